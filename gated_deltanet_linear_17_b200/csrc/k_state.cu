// Inter-chunk state passing: one CTA per (sequence, v-head, 32-column slice of Dv).
//
// Page "Qwen3Next Samples", "Recurrent State Attention" and "State Update",
// with the state held as S[Dk, Dv]:
//   v'    = k_cumdecay S                 -> U' = U - W S
//   S_new = S exp(g_last) + k_gexp^T (v_out - v'),  k_gexp = kh (.) exp(g_last - g_cum)
// g_last is the cumulative gate at the chunk's last valid token.  The CTA
// walks its sequence's chunks in order; the fp32 state slice [128 x 32] never
// leaves registers (16 warps, each 16 rows of Dk x 16 columns).  Each step writes the fp16 state
// entering the chunk (S_c) and U' for the output kernel.  The next chunk's W,
// k and U tiles are prefetched with cp.async while the current one computes.
// The state update multiplies the raw bf16 k rows (exact) by the decayed U'
// operand Ub = diag(rk e^{g_last - gamma}) U', with the normalisation 1/|k|
// folded in; Ub is split into two bf16 halves (hi + lo, ~16 significant bits)
// so the update keeps near-fp32 accuracy.  W S uses fp16 operands;
// accumulation is fp32 throughout.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kStateThreads = 512;
constexpr int DVT = 32;  // Dv columns per CTA

// per stage: W [128][128] fp16, K [128][128] bf16, U slice [128][32] fp16, gam[128], rkv[128]
constexpr int ST_W = 0, ST_K = 32768, ST_U = 65536, ST_G = 73728, ST_R = 74240;
constexpr int kStageBytes = 74752;
constexpr int OFF_SB = 2 * kStageBytes;      // fp16 [128 (Dk)][32] state operand
constexpr int OFF_UB = OFF_SB + 128 * 64;    // bf16 [128 (L)][32] decayed U' operand, high half
constexpr int OFF_UL = OFF_UB + 128 * 64;    // bf16 [128 (L)][32] decayed U' operand, low half
constexpr int kStateSmem = OFF_UL + 128 * 64;

__global__ void __launch_bounds__(kStateThreads, 1) state_kernel(
    const uint16_t *__restrict__ k, const float *__restrict__ pool, const int32_t *__restrict__ idx,
    float *__restrict__ final_state, int T, int Nqk, int Nv, const int4 *__restrict__ info,
    const int32_t *__restrict__ seq_chunk0, const float *__restrict__ rk, const float *__restrict__ gcum,
    const uint16_t *__restrict__ U, const uint16_t *__restrict__ W, uint16_t *__restrict__ Up,
    uint16_t *__restrict__ Sc)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int b = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * DVT;
    const int hq = h / (Nv / Nqk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // warp = (row block, column half): 16 rows (of Dk for the state, of L for U') x 16 columns
    const int r0 = (wid & 7) * 16, cb = (wid >> 3) * 16;
    const int c_begin = seq_chunk0[b], c_end = seq_chunk0[b + 1];
    // tokens of the sequence (the chunks of a sequence are consecutive 128-token runs)
    const int seq_t0 = c_begin < c_end ? info[c_begin].y : 0;
    const int seq_t1 = c_begin < c_end ? info[c_end - 1].y + info[c_end - 1].z : 0;

    // state slice: s[nt][e] is S[r0 + gid + 8*(e>>1)][col0 + cb + nt*8 + tig*2 + (e&1)]
    float s[2][4];
    {
        const float *src = nullptr;
        if (pool) {
            const int slot = idx ? idx[b] : b;
            src = pool + ((size_t)slot * Nv + h) * D * D;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = r0 + gid + hf * 8;
                const int col = col0 + cb + nt * 8 + tig * 2;
                float2 x = make_float2(0.f, 0.f);
                if (src) x = *reinterpret_cast<const float2 *>(src + (size_t)row * D + col);
                s[nt][2 * hf] = x.x;
                s[nt][2 * hf + 1] = x.y;
            }
    }

    auto issue = [&](int c, int st) {
        const int cstart = seq_t0 + (c - c_begin) * L, clen = min(L, seq_t1 - cstart);
        uint8_t *base = smem + st * kStageBytes;
        const uint32_t wsa = smem_addr(base + ST_W), ksa = smem_addr(base + ST_K), usa = smem_addr(base + ST_U);
        const uint16_t *wsrc = W + (size_t)(c * Nv + h) * L * D;
        const uint16_t *usrc = U + (size_t)(c * Nv + h) * L * D + col0;
        for (int e = tid; e < 128 * 16; e += kStateThreads) {
            const int r = e >> 4, cc = e & 15;
            cp_async16(wsa + sw256(r, cc), wsrc + r * D + cc * 8, true);
            const bool ok = r < clen;
            const int t = cstart + (ok ? r : 0);
            cp_async16(ksa + sw256(r, cc), k + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        }
        {
            const int r = tid >> 2, cc = tid & 3;  // 512 pieces: one per thread
            cp_async16(usa + sw64(r, cc), usrc + r * D + cc * 8, true);
        }
        // gamma (clamped to the last valid row) and 1/|k| (rows past the chunk read a real row; they
        // multiply zero rows of U' and K)
        if (tid < 128) {
            const int i = min(tid, clen - 1);
            cp_async4(smem_addr(base + ST_G) + tid * 4, gcum + (size_t)h * T + cstart + i);
            cp_async4(smem_addr(base + ST_R) + tid * 4, rk + (size_t)hq * T + cstart + i);
        }
    };

    uint8_t *Sb = smem + OFF_SB, *Ub = smem + OFF_UB, *Ul = smem + OFF_UL;
    const uint32_t sba = smem_addr(Sb), uba = smem_addr(Ub), ula = smem_addr(Ul);

    if (c_begin < c_end) issue(c_begin, 0);
    cp_async_commit();
    for (int c = c_begin, it = 0; c < c_end; ++c, ++it) {
        const int st = it & 1;
        if (c + 1 < c_end) issue(c + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait<1>();

        const int clen = min(L, seq_t1 - (seq_t0 + (c - c_begin) * L));
        uint8_t *base = smem + st * kStageBytes;
        const uint32_t wsa = smem_addr(base + ST_W), ksa = smem_addr(base + ST_K);
        const uint8_t *Us = base + ST_U;
        const float *gam = reinterpret_cast<const float *>(base + ST_G);
        const float *rkv = reinterpret_cast<const float *>(base + ST_R);
        const size_t tile = (size_t)(c * Nv + h) * L * D;

        // (1) state entering the chunk: fp16 copy to shared (MMA operand) and to Sc
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = r0 + gid + hf * 8;
                const int col = cb + nt * 8 + tig * 2;
                const uint32_t p = pack_h2(s[nt][2 * hf], s[nt][2 * hf + 1]);
                *reinterpret_cast<uint32_t *>(Sb + el64(row, col)) = p;
                *reinterpret_cast<uint32_t *>(Sc + tile + (size_t)row * D + col0 + col) = p;
            }
        __syncthreads();

        // (2) WS = W S for L rows r0..r0+15, columns cb..cb+15 (K = Dk)
        float wsacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) wsacc[nt][0] = wsacc[nt][1] = wsacc[nt][2] = wsacc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D; kk += 16) {
            uint32_t a[4], b0, b1, b2, b3;
            ldsm_x4(a_rowmajor_256(wsa, r0, kk, lane), a[0], a[1], a[2], a[3]);
            ldsm_x4_t(b_kmajor_64(sba, cb, kk, lane), b0, b1, b2, b3);
            mma16816(wsacc[0], a, b0, b1);
            mma16816(wsacc[1], a, b2, b3);
        }

        // (3) U' = U - W S -> Up; Ub = diag(rk e^{g_last - gamma}) U' as hi + lo (operand of the update)
        const float gl = gam[clen - 1];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int row = r0 + gid + hf * 8;
            const float sc = rkv[row] * __expf(gl - gam[row]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = cb + nt * 8 + tig * 2;
                const float2 u = unpack_h2(*reinterpret_cast<const uint32_t *>(Us + el64(row, col)));
                const float p0 = u.x - wsacc[nt][2 * hf];
                const float p1 = u.y - wsacc[nt][2 * hf + 1];
                *reinterpret_cast<uint32_t *>(Up + tile + (size_t)row * D + col0 + col) = pack_h2(p0, p1);
                uint32_t hi, lo;
                split_bf2(p0 * sc, p1 * sc, hi, lo);
                *reinterpret_cast<uint32_t *>(Ub + el64(row, col)) = hi;
                *reinterpret_cast<uint32_t *>(Ul + el64(row, col)) = lo;
            }
        }
        __syncthreads();

        // (4) S = e^{g_last} S + K^T (Ub_hi + Ub_lo) for Dk rows r0..r0+15, columns cb..cb+15 (K = L)
        const float dg = __expf(gl);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] *= dg;
#pragma unroll
        for (int kk = 0; kk < L; kk += 16) {
            uint32_t a[4], b0, b1, b2, b3;
            ldsm_x4_t(a_colmajor_256(ksa, r0, kk, lane), a[0], a[1], a[2], a[3]);
            ldsm_x4_t(b_kmajor_64(uba, cb, kk, lane), b0, b1, b2, b3);
            mma16816_bf16(s[0], a, b0, b1);
            mma16816_bf16(s[1], a, b2, b3);
            ldsm_x4_t(b_kmajor_64(ula, cb, kk, lane), b0, b1, b2, b3);
            mma16816_bf16(s[0], a, b0, b1);
            mma16816_bf16(s[1], a, b2, b3);
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    if (final_state) {
        float *dst = final_state + ((size_t)b * Nv + h) * D * D;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = r0 + gid + hf * 8;
                const int col = col0 + cb + nt * 8 + tig * 2;
                *reinterpret_cast<float2 *>(dst + (size_t)row * D + col) = make_float2(s[nt][2 * hf], s[nt][2 * hf + 1]);
            }
    }
}

cudaError_t launch_state(const uint16_t *k, const float *pool, const int32_t *idx, float *final_state, int T, int B,
                         int Nqk, int Nv, const Workspace &ws, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kStateSmem);
    if (e != cudaSuccess) return e;
    state_kernel<<<dim3(B, Nv, D / DVT), kStateThreads, kStateSmem, st>>>(
        k, pool, idx, final_state, T, Nqk, Nv, ws.chunk_info, ws.seq_chunk0, ws.rk, ws.gcum, ws.U, ws.W, ws.Up,
        ws.Sc);
    return cudaGetLastError();
}

}  // namespace gdn
