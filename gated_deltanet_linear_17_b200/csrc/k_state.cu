// Inter-chunk state passing: one CTA per (sequence, v-head, 32-column slice of Dv).
//
// Page "Qwen3Next Samples", "Recurrent State Attention" and "State Update",
// with the state held as S[Dk, Dv]:
//   v'    = k_cumdecay S                 -> U' = U - W S
//   S_new = S exp(g_last) + k_gexp^T (v_out - v'),  k_gexp = kh (.) exp(g_last - g_cum)
// g_last is the cumulative gate at the chunk's last valid token.  The CTA
// walks its sequence's chunks in order; the fp32 state slice [128 x 32] never
// leaves registers (4 warps x 32 rows of Dk).  Each step writes the fp16 state
// entering the chunk (S_c) and U' for the output kernel.  The next chunk's W,
// normalised k and U tiles are prefetched with cp.async while the current one
// computes.  Tensor-core operands are fp16 with fp32 accumulation.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kStateThreads = 128;
constexpr int DVT = 32;  // Dv columns per CTA

// per stage: W [128][128], Kh [128][128], U slice [128][32] (fp16), gam[128], (128 floats unused)
constexpr int ST_W = 0, ST_K = 32768, ST_U = 65536, ST_G = 73728, ST_R = 74240;
constexpr int kStageBytes = 74752;
constexpr int OFF_SB = 2 * kStageBytes;      // fp16 [128 (Dk)][32] state operand
constexpr int OFF_UB = OFF_SB + 128 * 64;    // fp16 [128 (L)][32] decayed U' operand
constexpr int kStateSmem = OFF_UB + 128 * 64;

__global__ void __launch_bounds__(kStateThreads, 1) state_kernel(
    const uint16_t *__restrict__ kn, const float *__restrict__ pool, const int32_t *__restrict__ idx,
    float *__restrict__ final_state, int T, int Nqk, int Nv, const int4 *__restrict__ info,
    const int32_t *__restrict__ seq_chunk0, const float *__restrict__ gcum,
    const uint16_t *__restrict__ U, const uint16_t *__restrict__ W, uint16_t *__restrict__ Up,
    uint16_t *__restrict__ Sc)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int b = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * DVT;
    const int hq = h / (Nv / Nqk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int c_begin = seq_chunk0[b], c_end = seq_chunk0[b + 1];

    // state slice: s[mt][nt][e] is S[wid*32 + mt*16 + gid + 8*(e>>1)][col0 + nt*8 + tig*2 + (e&1)]
    float s[2][4][4];
    {
        const float *src = nullptr;
        if (pool) {
            const int slot = idx ? idx[b] : b;
            src = pool + ((size_t)slot * Nv + h) * D * D;
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int row = wid * 32 + mt * 16 + gid + hf * 8;
                    const int col = col0 + nt * 8 + tig * 2;
                    float2 x = make_float2(0.f, 0.f);
                    if (src) x = *reinterpret_cast<const float2 *>(src + (size_t)row * D + col);
                    s[mt][nt][2 * hf] = x.x;
                    s[mt][nt][2 * hf + 1] = x.y;
                }
    }

    auto issue = [&](int c, int st) {
        const ChunkInfo ci = load_chunk(info, c);
        uint8_t *base = smem + st * kStageBytes;
        const uint32_t wsa = smem_addr(base + ST_W), ksa = smem_addr(base + ST_K), usa = smem_addr(base + ST_U);
        const uint16_t *wsrc = W + (size_t)(c * Nv + h) * L * D;
        const uint16_t *usrc = U + (size_t)(c * Nv + h) * L * D + col0;
        for (int e = tid; e < 128 * 16; e += kStateThreads) {
            const int r = e >> 4, cc = e & 15;
            cp_async16(wsa + sw256(r, cc), wsrc + r * D + cc * 8, true);
            const bool ok = r < ci.len;
            const int t = ci.start + (ok ? r : 0);
            cp_async16(ksa + sw256(r, cc), kn + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        }
        for (int e = tid; e < 128 * 4; e += kStateThreads) {
            const int r = e >> 2, cc = e & 3;
            cp_async16(usa + sw64(r, cc), usrc + r * D + cc * 8, true);
        }
        float *gam = reinterpret_cast<float *>(base + ST_G);
        const int i = tid;  // 128 threads: one row each
        gam[i] = gcum[(size_t)h * T + ci.start + min(i, ci.len - 1)];
    };

    uint8_t *Sb = smem + OFF_SB, *Ub = smem + OFF_UB;
    const uint32_t sba = smem_addr(Sb), uba = smem_addr(Ub);

    if (c_begin < c_end) issue(c_begin, 0);
    cp_async_commit();
    for (int c = c_begin, it = 0; c < c_end; ++c, ++it) {
        const int st = it & 1;
        if (c + 1 < c_end) issue(c + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        const ChunkInfo ci = load_chunk(info, c);
        uint8_t *base = smem + st * kStageBytes;
        const uint32_t wsa = smem_addr(base + ST_W), ksa = smem_addr(base + ST_K);
        const uint8_t *Us = base + ST_U;
        const float *gam = reinterpret_cast<const float *>(base + ST_G);
        const size_t tile = (size_t)(c * Nv + h) * L * D;

        // (1) state entering the chunk: fp16 copy to shared (MMA operand) and to Sc
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int row = wid * 32 + mt * 16 + gid + hf * 8;
                    const int col = nt * 8 + tig * 2;
                    const uint32_t p = pack_h2(s[mt][nt][2 * hf], s[mt][nt][2 * hf + 1]);
                    *reinterpret_cast<uint32_t *>(Sb + el64(row, col)) = p;
                    *reinterpret_cast<uint32_t *>(Sc + tile + (size_t)row * D + col0 + col) = p;
                }
        __syncthreads();

        // (2) WS = W S   (rows: L, 32 per warp; K = Dk)
        float wsacc[2][4][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) wsacc[mt][nt][0] = wsacc[mt][nt][1] = wsacc[mt][nt][2] = wsacc[mt][nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D; kk += 16) {
            uint32_t a0[4], a1[4];
            ldsm_x4(a_rowmajor_256(wsa, wid * 32, kk, lane), a0[0], a0[1], a0[2], a0[3]);
            ldsm_x4(a_rowmajor_256(wsa, wid * 32 + 16, kk, lane), a1[0], a1[1], a1[2], a1[3]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b_kmajor_64(sba, np * 16, kk, lane), b0, b1, b2, b3);
                mma16816(wsacc[0][2 * np], a0, b0, b1);
                mma16816(wsacc[0][2 * np + 1], a0, b2, b3);
                mma16816(wsacc[1][2 * np], a1, b0, b1);
                mma16816(wsacc[1][2 * np + 1], a1, b2, b3);
            }
        }

        // (3) U' = U - W S -> Up; Ub = diag(e^{g_last - gamma}) U' (operand of the update)
        const float gl = gam[ci.len - 1];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = wid * 32 + mt * 16 + gid + hf * 8;
                const float sc = __expf(gl - gam[row]);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int col = nt * 8 + tig * 2;
                    const uint32_t uu = *reinterpret_cast<const uint32_t *>(Us + el64(row, col));
                    const float2 u = unpack_h2(uu);
                    const float p0 = u.x - wsacc[mt][nt][2 * hf];
                    const float p1 = u.y - wsacc[mt][nt][2 * hf + 1];
                    *reinterpret_cast<uint32_t *>(Up + tile + (size_t)row * D + col0 + col) = pack_h2(p0, p1);
                    *reinterpret_cast<uint32_t *>(Ub + el64(row, col)) = pack_h2(p0 * sc, p1 * sc);
                }
            }
        __syncthreads();

        // (4) S = e^{g_last} S + Kh^T Ub   (rows: Dk, 32 per warp; K = L)
        const float dg = __expf(gl);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[mt][nt][e] *= dg;
#pragma unroll
        for (int kk = 0; kk < L; kk += 16) {
            uint32_t a0[4], a1[4];
            ldsm_x4_t(a_colmajor_256(ksa, wid * 32, kk, lane), a0[0], a0[1], a0[2], a0[3]);
            ldsm_x4_t(a_colmajor_256(ksa, wid * 32 + 16, kk, lane), a1[0], a1[1], a1[2], a1[3]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b_kmajor_64(uba, np * 16, kk, lane), b0, b1, b2, b3);
                mma16816(s[0][2 * np], a0, b0, b1);
                mma16816(s[0][2 * np + 1], a0, b2, b3);
                mma16816(s[1][2 * np], a1, b0, b1);
                mma16816(s[1][2 * np + 1], a1, b2, b3);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    if (final_state) {
        float *dst = final_state + ((size_t)b * Nv + h) * D * D;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int row = wid * 32 + mt * 16 + gid + hf * 8;
                    const int col = col0 + nt * 8 + tig * 2;
                    *reinterpret_cast<float2 *>(dst + (size_t)row * D + col) =
                        make_float2(s[mt][nt][2 * hf], s[mt][nt][2 * hf + 1]);
                }
    }
}

cudaError_t launch_state(const float *pool, const int32_t *idx, float *final_state, int T, int B, int Nqk,
                         int Nv, const Workspace &ws, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kStateSmem);
    if (e != cudaSuccess) return e;
    state_kernel<<<dim3(B, Nv, D / DVT), kStateThreads, kStateSmem, st>>>(
        ws.kn, pool, idx, final_state, T, Nqk, Nv, ws.chunk_info, ws.seq_chunk0, ws.gcum, ws.U, ws.W, ws.Up,
        ws.Sc);
    return cudaGetLastError();
}

}  // namespace gdn
