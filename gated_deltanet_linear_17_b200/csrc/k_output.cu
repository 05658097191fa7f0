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
//   0. TMA loads of the raw q and k rows and of W; rows past a short chunk are
//      zeroed after the load.
//   1. q k^T     -- tcgen05.mma M=128, N=128, K=128 on the raw 16-bit rows (bf16
//                   or fp16: exact inputs), both K-major; fp32 accumulator in TMEM.
//   2. P = rq_i rk_j exp(gamma_i - gamma_j) (q k^T)_ij for j <= i, else 0, read
//      from TMEM and written back to TMEM in fp16 pairs, where it is the A
//      operand of both products with P.  Since the gates are <= 0, gamma does not increase along the
//      chunk.  For a 16-column block below the diagonal the decay is factored
//      at the block's last column je as exp(gamma_i - gamma_je) exp(gamma_je -
//      gamma_j), both factors <= 1, so a row needs one exponential per block.
//      A row's own diagonal block takes the same split at its last row, where
//      the first factor is >= 1; it stays below e^kSpanMax unless the block's
//      gate span is wider, and then that block takes one exponential per
//      element.  Chunks above all of a warp's rows are written as zeros without
//      reading TMEM.
//   3. S_c starts loading into the k tile, free once q k^T is done.  Z = P W
//      -- M=128, N=128, K=128, fp16 (W read MN-major); then U starts loading
//      into W's tile, and Qw = diag(rq e^gamma) q - Z in fp16, in place of q.
//   4. O = Qw S_c + P U -- 16 tcgen05.mma (N = 128); the eight on U are issued
//      once it has landed, while the eight on S_c run.
//   5. O in out's type (bf16, fp16 or fp32): a full chunk of a 16-bit type is
//      staged over the consumed Qw tile and leaves by TMA; a short chunk's rows,
//      and fp32 rows, are stored by the threads, so rows of the next sequence are
//      never written.
// For an update rule without the retrieval (`delta` = 0: the LinearAttention
// page's gated and linear rules) W is zero: it is not loaded, Z is not formed and
// Qw = diag(rq e^gamma) q.
// One thread issues the MMAs and copies and waits for their completion
// (mbarriers, bounded waits); a CTA barrier passes the outcome on.  If a wait
// gives up, the CTA sets bit 1 of status[2] in the workspace and skips the rest
// of its chunk after letting its copies and MMAs drain.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"
#include "tc100.cuh"
#include "tma.cuh"

namespace gdn {

constexpr int kOutThreads = 256;
// shared memory, relative to a 1024-byte aligned base; 128 x 128 16-bit tiles are
// two 64-column halves of 128-byte rows with the 128-byte swizzle
constexpr int OO_Q = 0;        // q (bf16) -> Qw (fp16), K-major over Dk -> O (bf16) for the store
constexpr int OO_K = 32768;    // k (bf16), K-major over Dk -> S_c (fp16) [Dk][Dv], MN-major B of Qw S_c
constexpr int OO_X = 65536;    // W (fp16) [L][Dk], MN-major B of P W -> U (fp16) [L][Dv], MN-major B of P U
constexpr int OO_VEC = 98304;  // gam, rqv, rkv, kfe (rk_j e^{gamma_je - gamma_j})
constexpr int OO_BAR = OO_VEC + 4 * 512;  // mbarriers, TMEM slot, scan sums (72 bytes)
constexpr int kOutSmem = OO_BAR + 128 + 1024;

// byte offset of 16-byte chunk c (0..15) of row r in a 128 x 128 tile
__device__ __forceinline__ uint32_t t128(int r, int c) { return (uint32_t)((c >> 3) * 16384) + tc::sw128c(r, c & 7); }

// F16: the raw q and k rows are fp16 (else bf16); ODT: out's type (kTypeBF16 or kTypeF16 through a TMA
// store of the staged tile, kTypeF32 written by the threads)
template <bool F16, int ODT>
__global__ void __launch_bounds__(kOutThreads, 2) output_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_sc,
    const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_out, void *__restrict__ out,
    const float *__restrict__ g, float scale, float eps, int T, int Nqk, int Nv, const int4 *__restrict__ info,
    float *__restrict__ rq_out, int32_t *__restrict__ status, int c0, int delta, int m)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int c = c0 + blockIdx.x, h = blockIdx.y;
    const ChunkInfo ci = load_chunk(info, c);
    if (ci.seq < 0) return;
    const int hq = h / (Nv / Nqk);
    const int n = ci.len, t0 = ci.start;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int quarter = wid & 3, half = wid >> 2;
    const int row = quarter * 32 + lane;
    float *gam = reinterpret_cast<float *>(smem + OO_VEC);
    float *rqv = gam + 128, *rkv = gam + 256, *kfe = gam + 384;
    const uint32_t bar_ld = sbase + OO_BAR, bar_mma = sbase + OO_BAR + 8, bar_d = sbase + OO_BAR + 16;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OO_BAR + 24);
    const uint32_t bar_s = sbase + OO_BAR + 48, bar_u = sbase + OO_BAR + 56;  // S_c and U loads
    const uint32_t bar_w = sbase + OO_BAR + 64;                                 // W load (q, k on bar_ld)
    const int trow = (c * Nv + h) * L;  // first row of the chunk's tiles in the workspace

    if (tid == 0) {
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_d, 1);
        tc::mbar_init(bar_s, 1);
        tc::mbar_init(bar_u, 1);
        tc::mbar_init(bar_w, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), 256);
    __syncthreads();
    if (tid == 0) {  // q and k (64 KiB) on bar_ld, W (32 KiB) on bar_w
        tma::expect_tx(bar_ld, 65536);
        // q and k of the qk-head (columns past Dk = 64 read as zero)
        tma::load_3d(sbase + OO_Q, &tm_q, 0, hq, t0, bar_ld);
        tma::load_3d(sbase + OO_Q + 16384, &tm_q, 64, hq, t0, bar_ld);
        tma::load_3d(sbase + OO_K, &tm_k, 0, hq, t0, bar_ld);
        tma::load_3d(sbase + OO_K + 16384, &tm_k, 64, hq, t0, bar_ld);
        if (delta) {  // W enters only the rules with the retrieval
            tma::expect_tx(bar_w, 32768);
            tma::load_2d(sbase + OO_X, &tm_w, 0, trow, bar_w);
            tma::load_2d(sbase + OO_X + 16384, &tm_w, 64, trow, bar_w);
        }
    }
    // chunk-local cumulative gate while the rows load
    // the gate of the v-head (Nv counts sub-heads of 128 columns, m per v-head)
    chunk_gamma(g, Nv / m, h / m, t0, n, gam, reinterpret_cast<float *>(smem + OO_BAR + 32));
    // S_c, then U, as MN-major [128][128] tiles (two 64-column halves), each on its own barrier (thread 0)
    bool s_issued = false, u_issued = false;
    auto load_tile = [&](uint32_t dst, const CUtensorMap *m, uint32_t bar) {
        tma::expect_tx(bar, 32768);
        tma::load_2d(dst, m, 0, trow, bar);
        tma::load_2d(dst + 16384, m, 64, trow, bar);
    };
    bool ok = true;
    auto wait_bar = [&](uint32_t bar, uint32_t parity) {  // bounded, outcome shared with the CTA
        bool w_ok = true;
        if (tid == 0) w_ok = tc::mbar_wait_bounded(bar, parity);
        tc::fence_before_sync();
        ok = __syncthreads_and(w_ok) != 0 && ok;
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

    wait_bar(bar_ld, 0);
    if (n < L) {  // q and k rows past the chunk belong to the next sequence (W is zero there)
        for (int e = tid; e < (L - n) * 32; e += kOutThreads) {
            const int r = n + (e >> 5), tl = (e >> 4) & 1, blk = (e >> 3) & 1, cc = e & 7;
            *reinterpret_cast<uint4 *>(smem + (tl ? OO_K : OO_Q) + blk * 16384 + r * 128 + cc * 16) =
                make_uint4(0, 0, 0, 0);
        }
    }
    sync_operands();
    const uint32_t tmem = *tslot;  // columns [0, 128): q k^T, then Z = P W, then O; [128, 192): P (fp16 pairs)
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);

    // ---- (1) q k^T
    if (ok && tid == 0) {
        const uint64_t dq = tc::desc_k128(sbase + OO_Q), dk = tc::desc_k128(sbase + OO_K);
        const uint32_t idesc = tc::idesc_f16(128, 128, !F16, !F16);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_f16(tmem, kmaj(dq, kk), kmaj(dk, kk), idesc, kk > 0 ? 1u : 0u);
        tc::commit(bar_mma);
    }
    // while it runs: scale/|q| and 1/|k| of the valid rows ("L2 Normalization") and the decay factors
    {
        const int r = tid >> 1;  // two lanes per row
        const float xq = row_inv_norm_pair<F16>(smem + OO_Q, r, tid & 1, eps);
        const float xk = row_inv_norm_pair<F16>(smem + OO_K, r, tid & 1, eps);
        if ((tid & 1) == 0) {
            rqv[r] = r < n ? scale * xq : 0.f;
            rkv[r] = r < n ? xk : 0.f;
        }
    }
    __syncthreads();
    if (tid < 128) {
        kfe[tid] = rkv[tid] * __expf(gam[tid | 15] - gam[tid]);
        if (tid < n && h % (Nv / Nqk) == 0) rq_out[(size_t)hq * T + t0 + tid] = rqv[tid];  // for inspection
    }
    if (ok) wait_bar(bar_mma, 0);

    if (ok) {
        // ---- (2) P, this thread's 64 columns of its row, in fp16 pairs into TMEM columns [128, 192)
        const float gi = gam[row], fr = rqv[row];
        const int rlo = quarter * 32;  // first row of this warp
#pragma unroll 1
        for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            uint32_t pw[16];  // columns j0 .. j0 + 31 of the row, two to a word
            const uint32_t t_p = t_row + 128 + (j0 >> 1);
            if (j0 > rlo + 31) {  // above the diagonal for every row of the warp
#pragma unroll
                for (int e = 0; e < 16; ++e) pw[e] = 0u;
                tc::tmem_st16(t_p, pw);
                continue;
            }
            float a[32];
            tc::tmem_ld32(t_row + j0, a);
            if (j0 == rlo) {
                // The warp's diagonal chunk (warp-uniform).  Lanes 0-15 have their diagonal block at
                // columns j0..j0+15 and zeros right of it; lanes 16-31 have it at j0+16.. and the block
                // left of it at j0..j0+15.  Both blocks take the block factor, the diagonal one element
                // by element when its gate span is too wide for it.
                const bool hi = lane >= 16;
                const int rb = row & ~15;
                float kf[16], pd[16];
                lds_vec(kf, kfe + j0);  // the left block's column factors (lanes 16-31)
                const float eb = hi ? fr * __expf(gi - gam[j0 + 15]) : 0.f;
                const float gl = gam[rb + 15];
                if (gam[rb] - gl <= kSpanMax) {  // half-warp-uniform
                    float kd[16];
                    lds_vec(kd, kfe + rb);
                    const float ed = fr * __expf(gi - gl);
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 2) {
                        const float2 x = fmul2(fmul2(make_float2(ed, ed), make_float2(kd[jj], kd[jj + 1])),
                                               hi ? make_float2(a[16 + jj], a[17 + jj]) : make_float2(a[jj], a[jj + 1]));
                        pd[jj] = rb + jj <= row ? x.x : 0.f;
                        pd[jj + 1] = rb + jj + 1 <= row ? x.y : 0.f;
                    }
                } else {
                    float rkj[16], gmj[16];
                    lds_vec(rkj, rkv + rb);
                    lds_vec(gmj, gam + rb);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        pd[jj] = rb + jj <= row ? fr * rkj[jj] * __expf(fminf(gi - gmj[jj], 0.f)) * (hi ? a[16 + jj] : a[jj])
                                                : 0.f;
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = q8 * 8 + 2 * e, d = jj & 15;
                        const uint32_t left = pack_h2f(fmul2(fmul2(make_float2(eb, eb), make_float2(kf[d], kf[d + 1])),
                                                             make_float2(a[jj], a[jj + 1])));
                        const uint32_t dg = pack_h2(pd[d], pd[d + 1]);
                        pw[q8 * 4 + e] = q8 < 2 ? (hi ? left : dg) : (hi ? dg : 0u);
                    }
                }
                tc::tmem_st16(t_p, pw);
                continue;
            }
            // a chunk left of the warp's rows: the decay factored per 16-column block
            float kf[32];
            lds_vec(kf, kfe + j0);
            const float eb2[2] = {fr * __expf(gi - gam[j0 + 15]), fr * __expf(gi - gam[j0 + 31])};
#pragma unroll
            for (int q16 = 0; q16 < 2; ++q16) {
                const float eb = eb2[q16];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int jj = q16 * 16 + 2 * e;
                    pw[q16 * 8 + e] = pack_h2f(fmul2(fmul2(make_float2(eb, eb), make_float2(kf[jj], kf[jj + 1])),
                                                     make_float2(a[jj], a[jj + 1])));
                }
            }
            tc::tmem_st16(t_p, pw);
        }
        tc::tmem_wait_st();
    }
    sync_operands();

    // ---- (3) S_c starts loading over the consumed k tile; Z = P W (P from TMEM) into TMEM columns
    // [0, 128); U then loads over the consumed W; Qw = diag(rq e^gamma) q - Z in fp16, in place of q
    const uint32_t idesc_n128 = tc::idesc_f16(128, 128, false, false, false, true);
    if (ok) {
        bool w_ok = true;
        if (tid == 0) {
            load_tile(sbase + OO_K, &tm_sc, bar_s);
            s_issued = true;
            if (delta) w_ok = tc::mbar_wait_bounded(bar_w, 0);  // W has landed
            if (w_ok && delta) {
                const uint64_t dw = tc::desc_mn(sbase + OO_X, 16384, 1024, 2);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tmem, tmem + 128 + kk * 8, dw + (uint64_t)((kk * 2048) >> 4), idesc_n128,
                                   kk > 0 ? 1u : 0u);
            }
            tc::commit(bar_mma);  // (without the retrieval nothing new: the phase closes at once)
            w_ok = tc::mbar_wait_bounded(bar_mma, 1) && w_ok;  // second phase of bar_mma
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(w_ok) != 0 && ok;
        tc::fence_after_sync();
    }
    if (ok && tid == 0) {
        load_tile(sbase + OO_X, &tm_u, bar_u);
        u_issued = true;
    }
    float vmax = 0.f;  // largest magnitude of Qw (fp16 range check)
    if (ok) {
        const float qf = rqv[row] * __expf(gam[row]);
#pragma unroll 1
        for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            float z[32];
            if (delta) {
                tc::tmem_ld32(t_row + j0, z);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = 0.f;
            }
            uint4 qv[4];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) qv[c4] = *reinterpret_cast<const uint4 *>(smem + OO_Q + t128(row, (j0 >> 3) + c4));
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint4 *p = reinterpret_cast<uint4 *>(smem + OO_Q + t128(row, (j0 >> 3) + c4));
                const uint4 w = qv[c4];
                const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {  // q qf - z as one fused multiply-add per element, in pairs
                    const float2 x = ffma2(unpack2<F16>(w4[e]), make_float2(qf, qf),
                                           make_float2(-z[c4 * 8 + 2 * e], -z[c4 * 8 + 2 * e + 1]));
                    vmax = absmax_nan(absmax_nan(vmax, x.x), x.y);
                    o4[e] = pack_h2(x.x, x.y);
                }
                *p = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
    }
    sync_operands();

    // ---- (4) O = Qw S_c + P U into TMEM columns [0, 128): 8 MMAs on S_c, then 8 on U once it has landed
    if (ok) wait_bar(bar_s, 0);
    {
        bool w_ok = true;
        if (ok && tid == 0) {
            const uint64_t dq = tc::desc_k128(sbase + OO_Q), ds = tc::desc_mn(sbase + OO_K, 16384, 1024, 2);
            const uint64_t du = tc::desc_mn(sbase + OO_X, 16384, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem, kmaj(dq, kk), ds + (uint64_t)((kk * 2048) >> 4), idesc_n128, kk > 0 ? 1u : 0u);
            w_ok = tc::mbar_wait_bounded(bar_u, 0);
            if (w_ok) {
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ts(tmem, tmem + 128 + kk * 8, du + (uint64_t)((kk * 2048) >> 4), idesc_n128, 1u);
            }
            tc::commit(bar_mma);
            w_ok = w_ok && tc::mbar_wait_bounded(bar_mma, 0);  // third phase of bar_mma
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(w_ok) != 0 && ok;
        tc::fence_after_sync();
    }

    // ---- (5) O in out's type: a full chunk of a 16-bit type through shared memory (over Qw) and TMA, a
    // short one, or fp32, row by row
    if (ok) {
        const bool full = n == L && ODT != kTypeF32;
#pragma unroll 1
        for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            float a[32];
            tc::tmem_ld32(t_row + j0, a);
            if constexpr (ODT == kTypeF32) {
                if (row < n) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + ((size_t)(t0 + row) * Nv + h) * D + j0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) dst[q4] = make_float4(a[4 * q4], a[4 * q4 + 1], a[4 * q4 + 2], a[4 * q4 + 3]);
                }
                continue;
            }
            constexpr bool OF16 = ODT == kTypeF16;
            uint4 w[4];
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                w[q8] = make_uint4(pack2<OF16>(a[q8 * 8], a[q8 * 8 + 1]), pack2<OF16>(a[q8 * 8 + 2], a[q8 * 8 + 3]),
                                   pack2<OF16>(a[q8 * 8 + 4], a[q8 * 8 + 5]), pack2<OF16>(a[q8 * 8 + 6], a[q8 * 8 + 7]));
            if (full) {
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(smem + OO_Q + t128(row, (j0 >> 3) + q8)) = w[q8];
            } else if (row < n) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + ((size_t)(t0 + row) * Nv + h) * D + j0);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) dst[q8] = w[q8];
            }
        }
        if (full) {
            tc::fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                tma::store_2d(&tm_out, h * D, t0, sbase + OO_Q);
                tma::store_2d(&tm_out, h * D + 64, t0, sbase + OO_Q + 16384);
                tma::commit_group();
            }
        }
    } else if (tid == 0) {
        atomicOr(status + 2, GDN_DEV_WAIT_OUTPUT);
        // copies and MMAs still in flight land before shared and tensor memory are released:
        // a commit covers every MMA issued before it; then the last load phase issued
        tc::commit(bar_d);
        tc::mbar_wait_bounded(bar_d, 0);
        tc::mbar_wait_bounded(bar_ld, 0);
        if (delta) tc::mbar_wait_bounded(bar_w, 0);
        if (s_issued) tc::mbar_wait_bounded(bar_s, 0);
        if (u_issued) tc::mbar_wait_bounded(bar_u, 0);
    }
    if (tid == 0) tma::wait_read_all();  // the stores have read shared memory (the grid's end publishes them)
    if (__any_sync(0xffffffffu, out_of_fp16(vmax)) && lane == 0) atomicOr(status + 3, GDN_DEV_RANGE_OUTPUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, 256);
}

cudaError_t launch_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, void *out,
                          int T, int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st, bool delta,
                          bool f16, int out_type, Dims dims)
{
    if (nc <= 0 || T == 0) return cudaSuccess;
    if (c0 < 0 || c0 + nc > ws.NC) return cudaErrorInvalidValue;
    const uint64_t trows = (uint64_t)ws.NC * Nv * L;  // TMA coordinates are 32-bit signed
    if ((uint64_t)T >= (1ull << 31) || trows >= (1ull << 31)) return cudaErrorInvalidValue;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap m_q, m_k, m_w, m_sc, m_u, m_out;
    const auto AT = f16 ? HF : BF;
    cudaError_t e = tma::map_heads(&m_q, AT, q, (uint64_t)dims.Dk, (uint64_t)Nqk, (uint64_t)T, 128);
    if (e == cudaSuccess) e = tma::map_heads(&m_k, AT, k, (uint64_t)dims.Dk, (uint64_t)Nqk, (uint64_t)T, 128);
    if (e == cudaSuccess) e = tma::map2d(&m_w, HF, ws.W, D, trows, D * 2, 64, 128, SW);
    if (e == cudaSuccess) e = tma::map2d(&m_sc, HF, ws.Sc, D, trows, D * 2, 64, 128, SW);
    if (e == cudaSuccess) e = tma::map2d(&m_u, HF, ws.U, D, trows, D * 2, 64, 128, SW);
    if (e == cudaSuccess) {
        if (out_type == kTypeF32)  // written by the threads: the map is never used
            e = tma::map2d(&m_out, HF, ws.U, D, trows, D * 2, 64, 128, SW);
        else
            e = tma::map2d(&m_out, out_type == kTypeF16 ? HF : BF, out, (uint64_t)Nv * D, (uint64_t)T,
                           (uint64_t)Nv * D * 2, 64, 128, SW);
    }
    if (e != cudaSuccess) return e;
    auto kern = out_type == kTypeF32 ? (f16 ? output_kernel<true, kTypeF32> : output_kernel<false, kTypeF32>)
              : out_type == kTypeF16 ? (f16 ? output_kernel<true, kTypeF16> : output_kernel<false, kTypeF16>)
                                     : (f16 ? output_kernel<true, kTypeBF16> : output_kernel<false, kTypeBF16>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kOutSmem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(nc, Nv), kOutThreads, kOutSmem, st>>>(m_q, m_k, m_w, m_sc, m_u, m_out, out, g, scale, eps, T, Nqk, Nv,
                                                       ws.chunk_info, ws.rq, ws.status, c0, delta ? 1 : 0, dims.m);
    return cudaGetLastError();
}

}  // namespace gdn
