// Output kernel on the Blackwell tensor core: one CTA (8 warps) per (chunk, v-head),
// two CTAs per SM.
//
// Page "Qwen3Next Samples", "Recurrent State Attention":
//   o_inter = (q (.) exp(g_cum)) S^T
//   o_chunk = o_inter + (q k^T (.) D_decay (.) T_tril) (v_out - v'),  v' = k_cumdecay S
// with S held as [Dk, Dv] (so S^T there is S here), T_tril including the
// diagonal, v_out = U and k_cumdecay = W.  With P = q k^T (.) D_decay (.) T_tril
// and Q' = diag(e^gamma) q this is regrouped as
//   o = (Q' - P W) S_c + P U,
// so the chunk's state S_c enters one product.  Warp w handles rows
// 32(w%4)..32(w%4)+31 and, in the epilogues, one half of the columns.  Steps:
//   1. q k^T     -- tcgen05.mma M=128, N=128, K=128 on the raw bf16 rows (exact
//                   inputs), both K-major; fp32 accumulator in TMEM.
//   2. P = rq_i rk_j exp(gamma_i - gamma_j) (q k^T)_ij for j <= i, else 0, read
//      from TMEM and stored in fp16 as a K-major A tile over the now unused k
//      tile.  Since the gates are <= 0, gamma does not increase along the
//      chunk.  For a 16-column block below the diagonal the decay is factored
//      at the block's last column je as exp(gamma_i - gamma_je) exp(gamma_je -
//      gamma_j), both factors <= 1, so a row needs one exponential per block;
//      only the 32-column chunk on a warp's diagonal takes one per element.
//      Chunks above all of a warp's rows are written as zeros without reading
//      TMEM.
//   3. Z = P W  -- M=128, N=128, K=128, fp16 (W read MN-major); then
//      Qw = diag(rq e^gamma) q - Z in fp16, in place of q.
//   4. O = Qw S_c + P U for Dv columns 0..63, then 64..127 -- 16 tcgen05.mma
//      each (N = 64); S_c and U are staged one column half at a time in the
//      buffer W used, and each half is stored while the next one loads.
// One thread issues the MMAs and waits for their completion (mbarrier arrival
// from tcgen05.commit, bounded wait); a CTA barrier passes the outcome on.  If
// a wait gives up, the CTA sets bit 1 of status[2] in the workspace and skips
// the rest of its chunk after letting its MMAs drain.
#include "common.cuh"
#include "gdn_internal.h"
#include "tc100.cuh"

namespace gdn {

constexpr int kOutThreads = 256;
// shared memory, relative to a 1024-byte aligned base
constexpr int OO_Q = 0;         // q (bf16) then Qw (fp16): K-major over Dk, 2 halves x 128 rows x 128 B
constexpr int OO_K = 32768;     // k (bf16), K-major over Dk; then P (fp16), K-major over j
constexpr int OO_X = 65536;     // W (fp16) [L][Dk] in two 64-column blocks (MN-major B of P W); then
                                // S_c[:, half] (fp16) [Dk][64] and, 16 KiB on, U[:, half] (fp16) [L][64]
constexpr int OO_VEC = 98304;   // gam, rqv, rkv, kfe (rk_j e^{gamma_je - gamma_j})
constexpr int OO_BAR = OO_VEC + 4 * 512;
constexpr int kOutSmem = OO_BAR + 64 + 1024;

// byte offset of 16-byte chunk c (0..15) of row r in a 128-row, 128-element tile
__device__ __forceinline__ uint32_t t128(int r, int c) { return (uint32_t)((c >> 3) * 16384) + tc::sw128c(r, c & 7); }

__global__ void __launch_bounds__(kOutThreads, 2) output_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, uint16_t *__restrict__ out, int T, int Nqk,
    int Nv, const int4 *__restrict__ info, const float *__restrict__ rq, const float *__restrict__ rk,
    const float *__restrict__ gcum, const uint16_t *__restrict__ U, const uint16_t *__restrict__ W,
    const uint16_t *__restrict__ Sc, int32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int c = blockIdx.x, h = blockIdx.y;
    const ChunkInfo ci = load_chunk(info, c);
    if (ci.seq < 0) return;
    const int hq = h / (Nv / Nqk);
    const int n = ci.len, t0 = ci.start;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int quarter = wid & 3, half = wid >> 2;
    const int row = quarter * 32 + lane;
    float *gam = reinterpret_cast<float *>(smem + OO_VEC);
    float *rqv = gam + 128, *rkv = gam + 256, *kfe = gam + 384;
    const uint32_t bar_qk = sbase + OO_BAR, bar_z = sbase + OO_BAR + 8, bar_o = sbase + OO_BAR + 16;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OO_BAR + 24);
    const size_t tile = (size_t)(c * Nv + h) * L * D;

    // S_c and U columns [64 hf, 64 hf + 64) into the MN-major buffers
    auto load_su = [&](int hf) {
        for (int e = tid; e < 128 * 8; e += kOutThreads) {
            const int r = e >> 3, cc = e & 7;
            cp_async16(sbase + OO_X + tc::sw128c(r, cc), Sc + tile + (size_t)r * D + hf * 64 + cc * 8, true);
            cp_async16(sbase + OO_X + 16384 + tc::sw128c(r, cc), U + tile + (size_t)r * D + hf * 64 + cc * 8, true);
        }
    };

    // ---- async loads: q, k rows of the chunk (zero past n), W, gamma, rq, rk
    for (int e = tid; e < 128 * 16; e += kOutThreads) {
        const int r = e >> 4, cc = e & 15;
        const bool ok = r < n;
        const int t = t0 + (ok ? r : 0);
        const uint32_t off = t128(r, cc);
        cp_async16(sbase + OO_Q + off, q + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        cp_async16(sbase + OO_K + off, k + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        cp_async16(sbase + OO_X + off, W + tile + (size_t)r * D + cc * 8, true);
    }
    if (tid < 128) {
        const int i = min(tid, n - 1);
        cp_async4(smem_addr(gam + tid), gcum + (size_t)h * T + t0 + i);
        cp_async4(smem_addr(rqv + tid), rq + (size_t)hq * T + t0 + i);
        cp_async4(smem_addr(rkv + tid), rk + (size_t)hq * T + t0 + i);
    }
    cp_async_commit();
    if (tid == 0) {
        tc::mbar_init(bar_qk, 1);
        tc::mbar_init(bar_z, 1);
        tc::mbar_init(bar_o, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), 256);
    cp_async_wait<0>();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;  // columns [0, 128): q k^T, then O; [128, 256): Z = P W
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    uint32_t last_bar = bar_qk, last_par = 0;  // the most recent commit (thread 0)
    auto wait_mma = [&](uint32_t bar, uint32_t parity) {
        bool w_ok = true;
        if (tid == 0) w_ok = tc::mbar_wait_bounded(bar, parity);
        tc::fence_before_sync();
        ok = __syncthreads_and(w_ok) != 0;
        tc::fence_after_sync();
    };
    auto sync_operands = [&]() {  // generic-proxy shared-memory writes -> tensor core
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    // descriptor of K step kk of a K-major tile with two 64-column K halves
    auto kmaj = [](uint64_t d, int kk) { return d + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4); };

    // ---- (1) q k^T
    if (tid == 0) {
        const uint64_t dq = tc::desc_k128(sbase + OO_Q), dk = tc::desc_k128(sbase + OO_K);
        const uint32_t idesc = tc::idesc_f16(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_f16(tmem, kmaj(dq, kk), kmaj(dk, kk), idesc, kk > 0 ? 1u : 0u);
        tc::commit(bar_qk);
    }
    if (tid < 128) kfe[tid] = rkv[tid] * __expf(gam[tid | 15] - gam[tid]);
    wait_mma(bar_qk, 0);

    if (ok) {
        // ---- (2) P, this thread's 64 columns of its row (fp16 over the k tile)
        const float gi = gam[row], fr = rqv[row];
        const int rlo = quarter * 32;  // first row of this warp
#pragma unroll 1
        for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            if (j0 > rlo + 31) {  // above the diagonal for every row of the warp
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8)
                    *reinterpret_cast<uint4 *>(smem + OO_K + t128(row, (j0 >> 3) + c8)) = make_uint4(0, 0, 0, 0);
                continue;
            }
            float a[32];
            tc::tmem_ld32(t_row + j0, a);
            const bool diag = j0 == rlo;  // warp-uniform
#pragma unroll
            for (int q16 = 0; q16 < 2; ++q16) {
                const int jb = j0 + q16 * 16;
                const float eb = diag ? 0.f : fr * __expf(gi - gam[jb + 15]);
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float p[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int jj = q16 * 16 + q8 * 8 + 2 * e + u, j = j0 + jj;
                            float f;
                            if (diag)
                                f = j <= row ? fr * rkv[j] * __expf(fminf(gi - gam[j], 0.f)) : 0.f;
                            else
                                f = eb * kfe[j];
                            p[u] = f * a[jj];
                        }
                        w4[e] = pack_h2(p[0], p[1]);
                    }
                    *reinterpret_cast<uint4 *>(smem + OO_K + t128(row, (jb >> 3) + q8)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        sync_operands();

        // ---- (3) Z = P W, then Qw = diag(rq e^gamma) q - Z over q
        if (tid == 0) {
            const uint64_t dp = tc::desc_k128(sbase + OO_K), dw = tc::desc_mn(sbase + OO_X, 16384, 1024, 2);
            const uint32_t idesc = tc::idesc_f16(128, 128, false, false, false, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem + 128, kmaj(dp, kk), dw + (uint64_t)((kk * 2048) >> 4), idesc, kk > 0 ? 1u : 0u);
            tc::commit(bar_z);
            last_bar = bar_z;
        }
        wait_mma(bar_z, 0);
    }
    if (ok) {
        load_su(0);  // W is consumed
        cp_async_commit();
        const float qf = rqv[row] * __expf(gam[row]);
#pragma unroll 1
        for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            float z[32];
            tc::tmem_ld32(t_row + 128 + j0, z);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint4 *p = reinterpret_cast<uint4 *>(smem + OO_Q + t128(row, (j0 >> 3) + c4));
                const uint4 w = *p;
                const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o4[e] = pack_h2(__uint_as_float(w4[e] << 16) * qf - z[c4 * 8 + 2 * e],
                                    __uint_as_float(w4[e] & 0xffff0000u) * qf - z[c4 * 8 + 2 * e + 1]);
                *p = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        cp_async_wait<0>();
        sync_operands();

        const uint64_t dq = tc::desc_k128(sbase + OO_Q), dp = tc::desc_k128(sbase + OO_K);
        const uint64_t ds = tc::desc_mn(sbase + OO_X, 16384, 1024, 2), du = tc::desc_mn(sbase + OO_X + 16384, 16384, 1024, 2);
        const uint32_t idesc = tc::idesc_f16(128, 64, false, false, false, true);
#pragma unroll 1
        for (int hf = 0; hf < 2 && ok; ++hf) {
            // ---- (4) O[:, 64 hf : 64 hf + 64] = Qw S_c + P U
            if (tid == 0) {
                const uint32_t dst = tmem + hf * 64;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(dst, kmaj(dq, kk), ds + (uint64_t)((kk * 2048) >> 4), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(dst, kmaj(dp, kk), du + (uint64_t)((kk * 2048) >> 4), idesc, 1u);
                tc::commit(bar_o);
                last_bar = bar_o;
                last_par = (uint32_t)hf;
            }
            wait_mma(bar_o, (uint32_t)hf);
            if (!ok) break;
            if (hf == 0) {  // the buffers are free: start the second half's loads
                load_su(1);
                cp_async_commit();
            }
            // ---- this thread's 32 columns of the half, to bf16 (TMEM reads are warp-collective)
            {
                float a[32];
                tc::tmem_ld32(t_row + hf * 64 + half * 32, a);
                if (row < n) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + ((size_t)(t0 + row) * Nv + h) * D + hf * 64 + half * 32);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack_bf2(a[q8 * 8], a[q8 * 8 + 1]), pack_bf2(a[q8 * 8 + 2], a[q8 * 8 + 3]),
                                             pack_bf2(a[q8 * 8 + 4], a[q8 * 8 + 5]),
                                             pack_bf2(a[q8 * 8 + 6], a[q8 * 8 + 7]));
                }
            }
            if (hf == 0) {
                cp_async_wait<0>();
                sync_operands();
            }
        }
    }
    cp_async_wait<0>();
    if (!ok && tid == 0) {  // let the MMAs drain before TMEM is freed (a commit covers all earlier MMAs)
        atomicOr(status + 2, 2);
        tc::mbar_wait_bounded(last_bar, last_par);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, 256);
}

cudaError_t launch_output(const uint16_t *q, const uint16_t *k, uint16_t *out, int T, int Nqk, int Nv, int NC,
                          const Workspace &ws, cudaStream_t st)
{
    if (NC == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmem);
    if (e != cudaSuccess) return e;
    output_kernel<<<dim3(NC, Nv), kOutThreads, kOutSmem, st>>>(q, k, out, T, Nqk, Nv, ws.chunk_info, ws.rq, ws.rk,
                                                                ws.gcum, ws.U, ws.W, ws.Sc, ws.status);
    return cudaGetLastError();
}

}  // namespace gdn
