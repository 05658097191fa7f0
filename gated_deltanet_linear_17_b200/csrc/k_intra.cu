// Intra-chunk kernel: (chunk, v-head) items, two per CTA back to back, two CTAs per SM.
//
// Page "Qwen3Next Samples", chunk_gated_delta_rule, "Mathematical Formulas":
//   A  = (k_beta k^T) (.) D_decay (.) M_mask      "Pre-Attention Matrix"
//   (I - A)^-1                                     "Matrix Inversion"
//   v_out = (I - A)^-1 (v (.) beta)                "Value and Key Cumulative Decay"
//   k_cumdecay = (I - A)^-1 (k_beta (.) exp(g_cum))
// The page's A (with its negative mask) is the strictly lower matrix
// Ap_ij = -beta_i (kh_i . kh_j) Gamma_ij, j < i, and T = (I - Ap)^-1.  As the
// page's inverse_pto does, T is built from the inverses of its 16-row diagonal
// blocks, merged two at a time (16 -> 32 -> 64 -> 128): the inverse of
// [[M11, 0], [M21, M22]] with M = I - Ap is [[T11, 0], [T22 Ap21 T11, T22]].
// Steps, with the raw k and v rows (bf16, or fp16 when the caller's activations are
// fp16) staged by TMA:
//   1. k k^T     -- tcgen05.mma M=128, N=128, K=128 on the raw rows (exact inputs); the L2
//                   norms enter as the fp32 factors rk, taken from its diagonal.
//   2. Ap from TMEM in fp16 (the diagonal 16x16 blocks in fp32); the decay is
//      factored per 16-column block as in the output kernel, the diagonal
//      blocks included unless their gate span exceeds kSpanMax.
//   3. T_ii by forward substitution (fp32), then the three merge levels with
//      mma.sync on fp16 operands, in place over Ap.
//   4. [W | U] = T [diag(beta e^gamma rk) k | diag(beta) v] -- one tcgen05.mma
//      group, M=128, N=256, K=128, fp16; U and W are stored in fp16.
//   5. The state-independent factor of the state update ("State Update"): with
//      k_gexp = Kh (.) exp(g_last - g_cum) (fp16, |entries| <= 1),
//        S_new = e^{g_last} S + k_gexp^T U - Mk S,   Mk = k_gexp^T W  [Dk x Dk],
//      one tcgen05.mma group (M=128, N=128, K=128) on k_gexp (the k rows loaded
//      again) and W; Mk is stored in fp16, and the per-row factors
//      rk_t e^{g_last - gamma_t} and e^{g_last} go to fa for the state pass.
// Rows past a short chunk are zeroed after their TMA loads.  While an item's Mk
// product runs, the CTA loads the next item's k rows into the tile that held T
// and U (the two tiles swap roles) and, once Mk is done, its v rows; the next
// item's gate and beta values are fetched into registers at the start of the
// current one.  For an update rule without the retrieval (`delta` = 0: the
// LinearAttention page's gated and linear rules) the CTA takes one item, stores
// U = v in fp16 and the factor records, and skips T, W and Mk.  Each wait is
// bounded; if one gives up, the CTA sets bit 2 of
// status[2], lets its MMAs and open loads drain and stops.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"
#include "tc100.cuh"
#include "tma.cuh"

namespace gdn {

constexpr int kIntraThreads = 256;
// Chunks per CTA.  Two CTAs share an SM; each CTA runs its chunks back to back, loading the
// next chunk's k and v rows and gate values while the current one finishes, which saves the
// CTA start-up (barriers, tensor-memory allocation, the first loads) for every second chunk.
// Longer runs per CTA measured slower inside the pipelined forward pass: the state pass, which
// needs a whole SM, then waits longer for one to come free.
constexpr int kIntraItemsPerCta = 2;

// shared memory (bytes), relative to a 1024-byte aligned base; 128 x 128 16-bit
// tiles are two 64-column halves of 128-byte rows with the 128-byte swizzle
// Three tiles.  Tile 1 always holds raw v -> diag(beta) v (fp16) -> W (fp16).  Of tiles 0 and 2,
// the item's k tile holds raw k -> diag(beta e^gamma rk) k (fp16) -> raw k again -> k_gexp (fp16)
// -> Mk (fp16), and its A tile Ap (fp16) -> T (fp16), rows i, columns j -> U (fp16); the two swap roles
// from one item of a CTA to the next.
constexpr int OFF_T0 = 0;
constexpr int OFF_T1 = 32768;
constexpr int OFF_T2 = 65536;
constexpr int OFF_X = 98304;     // 8 KiB scratch: fp32 diagonal blocks of Ap, then fp16 merge products [64][64]
constexpr int OFF_VEC = OFF_X + 8192;  // fp32 gam[128], bet[128], rkv[128], kfe[128]
constexpr int OFF_BAR = OFF_VEC + 2048;  // mbarriers (loads, MMAs) + TMEM address slot
constexpr int kIntraSmem = OFF_BAR + 64 + 1024;  // + alignment slack

// byte offset of 16-byte chunk c (0..15) of row r in a 128 x 128 tile
__device__ __forceinline__ uint32_t t128(int r, int c) { return (uint32_t)((c >> 3) * 16384) + tc::sw128c(r, c & 7); }
// byte offset of 16-byte chunk c (0..7) of row r in the [64][64] fp16 scratch
__device__ __forceinline__ uint32_t x64(int r, int c) { return tc::sw128c(r, c); }

// One warp: acc (a 16 x 16 fp32 tile, two m16n8 fragments) += A[am0.., ak0 + k] B[bk0 + k, bn0..]
// for k in [0, 16 steps) in steps of 16 (steps <= KMAX); A and B are fp16 tiles addressed by
// the offset functions fa_ (row, chunk) and fb_ (row, chunk).  Every fragment load is issued
// before the first MMA.
template <int KMAX, typename FA, typename FB>
__device__ __forceinline__ void warp_mm(float (&acc)[2][4], uint32_t abase, FA fa_, int am0, int ak0, uint32_t bbase,
                                        FB fb_, int bk0, int bn0, int steps, int lane)
{
    uint32_t a[KMAX][4], b[KMAX][4];
#pragma unroll
    for (int s = 0; s < KMAX; ++s)
        if (s < steps) {
            const int kk = 16 * s;
            ldsm_x4(abase + fa_(am0 + (lane & 15), ((ak0 + kk) >> 3) + (lane >> 4)), a[s][0], a[s][1], a[s][2], a[s][3]);
            ldsm_x4_t(bbase + fb_(bk0 + kk + (lane & 7) + (((lane >> 3) & 1) << 3), (bn0 >> 3) + (lane >> 4)), b[s][0],
                      b[s][1], b[s][2], b[s][3]);
        }
#pragma unroll
    for (int s = 0; s < KMAX; ++s)
        if (s < steps) {
            mma16816(acc[0], a[s], b[s][0], b[s][1]);
            mma16816(acc[1], a[s], b[s][2], b[s][3]);
        }
}

// store a warp's 16 x 16 fp32 tile in fp16 at rows m0.., columns n0.. of a tile with offsets f_(row, chunk)
template <typename F>
__device__ __forceinline__ void warp_store16(const float (&acc)[2][4], uint8_t *base, F f_, int m0, int n0, int lane)
{
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int r = m0 + gid + hf * 8, col = n0 + nt * 8 + tig * 2;
            *reinterpret_cast<uint32_t *>(base + f_(r, col >> 3) + (col & 7) * 2) =
                pack_h2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
        }
}

// Rewrite a 128 x 128 tile of raw bf16 (F16: fp16) rows in place as fp16 rows scaled by fac(r),
// rows from nvalid on as zeros; NT threads (t = 0 .. NT - 1), thread t at chunk t % 16 of
// rows t / 16 + (NT / 16) i, eight rows at a time with their loads issued before any
// conversion.  With TRACK, vmax keeps the largest magnitude written (fp16 range check).
template <int NT, bool F16, bool TRACK = false, typename F>
__device__ __forceinline__ void scale_rows_f16(uint8_t *tile, int t, int nvalid, F fac, float *vmax = nullptr)
{
    constexpr int kStep = NT / 16, kRows = 128 / kStep;
#pragma unroll 1
    for (int b = 0; b < kRows; b += 8) {
        uint4 x[8];
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = (t >> 4) + kStep * (b + i);
            x[i] = *reinterpret_cast<const uint4 *>(tile + t128(r, t & 15));
            f[i] = fac(r);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = (t >> 4) + kStep * (b + i);
            const float m = f[i];
            if (TRACK && r < nvalid) {
                const uint32_t w4[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
                float mx = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                {
                    const float2 p = unpack2<F16>(w4[e]);
                    mx = absmax_nan(absmax_nan(mx, p.x), p.y);
                }
                *vmax = absmax_nan(*vmax, mx * m);
            }
            const float2 mm = make_float2(m, m);  // packed fp32 pairs: the same products
            const float2 p0 = fmul2(unpack2<F16>(x[i].x), mm), p1 = fmul2(unpack2<F16>(x[i].y), mm),
                         p2 = fmul2(unpack2<F16>(x[i].z), mm), p3 = fmul2(unpack2<F16>(x[i].w), mm);
            *reinterpret_cast<uint4 *>(tile + t128(r, t & 15)) =
                r < nvalid ? make_uint4(pack_h2(p0.x, p0.y), pack_h2(p1.x, p1.y), pack_h2(p2.x, p2.y),
                                        pack_h2(p3.x, p3.y))
                           : make_uint4(0, 0, 0, 0);
        }
    }
}

template <bool F16>  // raw q/k/v rows of fp16 (else bf16)
__global__ void __launch_bounds__(kIntraThreads, 2) intra_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_w,
    const __grid_constant__ CUtensorMap tm_mk, const float *__restrict__ g, const uint16_t *__restrict__ beta,
    float eps, int T, int Nqk, int Nv, const int4 *__restrict__ info, float *__restrict__ rk_out,
    float *__restrict__ gcum_out, float *__restrict__ betaf_out, float *__restrict__ fa, int32_t *__restrict__ status,
    int c0, int nc, int delta, int m)
{
    // Nv counts 128-column sub-heads: a v-head of Dv = 128 m columns is m sub-heads that share its gate,
    // beta and qk-head; g and beta are indexed by the v-head, Nv / m of them per token
    const int Nvr = Nv / m;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int quarter = wid & 3, half = wid >> 2;
    const int row = quarter * 32 + lane;  // TMEM lane of this thread
    const int items = nc * Nv, grid = (int)gridDim.x, grp = Nv / Nqk;
    // item `it` is chunk c0 + it % nc of v-head it / nc; the CTA takes items blockIdx.x + i gridDim.x,
    // passing over chunk rows past the last chunk
    auto next_item = [&](int it) {
        while (it < items && load_chunk(info, c0 + it % nc).seq < 0) it += grid;
        return it;
    };
    int it = next_item((int)blockIdx.x);
    if (it >= items) return;
    int h = it / nc, c = c0 + it % nc;
    ChunkInfo ci = load_chunk(info, c);

    float *gam = reinterpret_cast<float *>(smem + OFF_VEC);
    float *bet = gam + 128, *rkv = gam + 256, *kfe = gam + 384;
    const uint32_t bar_ld = sbase + OFF_BAR, bar_mma = sbase + OFF_BAR + 8, bar_d = sbase + OFF_BAR + 16;
    const uint32_t bar_v = sbase + OFF_BAR + 48;  // the v rows (k rows on bar_ld)
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 24);
    float *wsum = reinterpret_cast<float *>(smem + OFF_BAR + 32);

    if (tid == 0) {
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(bar_v, 1);
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_d, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), 256);
    // an item's raw k rows into tile `dst` (bar_ld) and its v rows into tile 1 (bar_v); rows past T read
    // as zero.  bar_ld completes twice per item (the rows, then the same rows again for k_gexp), bar_v
    // once; a load is issued only after the barrier's previous phase has been waited on.
    auto load_k = [&](uint32_t dst, int hq_, int t0_) {
        tma::expect_tx(bar_ld, 32768);
        tma::load_3d(sbase + dst, &tm_k, 0, hq_, t0_, bar_ld);  // columns past Dk (= 64) read as zero
        tma::load_3d(sbase + dst + 16384, &tm_k, 64, hq_, t0_, bar_ld);
    };
    auto load_v = [&](int h_, int t0_) {
        tma::expect_tx(bar_v, 32768);
        tma::load_2d(sbase + OFF_T1, &tm_v, h_ * D, t0_, bar_v);
        tma::load_2d(sbase + OFF_T1 + 16384, &tm_v, h_ * D + 64, t0_, bar_v);
    };
    if (tid == 0) {
        load_k(OFF_T0, h / grp, ci.start);
        load_v(h, ci.start);
    }
    // this thread's gate and beta of the current item (threads 0..127, zero past the chunk)
    float xg = 0.f, xb = 0.f;
    if (tid < 128 && tid < ci.len) {  // g == nullptr: a zero gate; beta == nullptr: not read (no retrieval)
        xg = g ? g[(size_t)(ci.start + tid) * Nvr + h / m] : 0.f;
        xb = beta ? bf2f(beta[(size_t)(ci.start + tid) * Nvr + h / m]) : 0.f;
    }
    bool ok = true;
    float vmax = 0.f;  // largest magnitude of the fp16 U tiles (range check; a NaN is kept)
    uint32_t mma_phase = 0, v_par = 0, ld_par = 0;
    bool ld_pend = true, v_pend = true;  // a load phase issued and not yet waited on
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
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16);
    auto kmaj = [](uint64_t d, int kk) { return d + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4); };

#pragma unroll 1
    for (int li = 0;; ++li) {
        // tiles of this item: k rows in tk, Ap / T / U in ta, v / W in tile 1; the next item's k rows
        // go to ta once U has left, so the two swap between consecutive items
        const uint32_t tk = (li & 1) ? OFF_T2 : OFF_T0, ta = (li & 1) ? OFF_T0 : OFF_T2;
        const int hq = h / grp, n = ci.len, t0 = ci.start;
        // the next item, and its gate and beta, fetched while this one runs
        const int nit = next_item(it + grid);
        float ng = 0.f, nb = 0.f;
        if (nit < items) {
            const int nh = nit / nc;
            const ChunkInfo nci = load_chunk(info, c0 + nit % nc);
            if (tid < 128 && tid < nci.len) {
                ng = g ? g[(size_t)(nci.start + tid) * Nvr + nh / m] : 0.f;
                nb = beta ? bf2f(beta[(size_t)(nci.start + tid) * Nvr + nh / m]) : 0.f;
            }
        }
        // chunk-local cumulative gate and beta while the rows load
        chunk_gamma_x(xg, gam, wsum);
        if (tid < 128) bet[tid] = xb;
        // zero the rows of a tile past the chunk (they belong to the next sequence)
        auto zero_tail = [&](uint32_t off) {
            for (int e = tid; e < (L - n) * 16; e += kIntraThreads) {
                const int r = n + (e >> 4), blk = (e >> 3) & 1, cc = e & 7;
                *reinterpret_cast<uint4 *>(smem + off + blk * 16384 + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            }
        };
        wait_bar(bar_ld, 0);
        if (ok) ld_pend = false;
        if (ok && n < L) zero_tail(tk);
        sync_operands();

        // ---- (1) k k^T into TMEM columns [0, 128)
        if (ok && tid == 0) {
            const uint64_t dk = tc::desc_k128(sbase + tk);
            const uint32_t idesc = tc::idesc_f16(128, 128, !F16, !F16);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) tc::mma_f16(tmem, kmaj(dk, kk), kmaj(dk, kk), idesc, kk > 0 ? 1u : 0u);
            tc::commit(bar_mma);
        }
        if (tid < n) {  // for inspection through the stage interface
            gcum_out[(size_t)h * T + t0 + tid] = gam[tid];
            betaf_out[(size_t)h * T + t0 + tid] = bet[tid];
        }
        if (tid == 0) tma::wait_read_all();  // the previous item's Mk store has read this item's A tile
        if (ok) {
            wait_bar(bar_mma, mma_phase);
            mma_phase ^= 1;
        }
        // 1/|k_i| ("L2 Normalization") from the diagonal of k k^T, the fp32 sum of the exact squares of
        // the raw 16-bit entries: warp q < 4 reads its 32 rows' diagonal block of columns and keeps lane l's
        // column l
        if (ok && half == 0) {
            float a[32];
            tc::tmem_ld32(t_row + quarter * 32, a);
            float d = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) d = jj == lane ? a[jj] : d;
            rkv[row] = row < n ? 1.0f / sqrtf(d + eps) : 0.f;
        }
        __syncthreads();
        // the decay factors of the columns
        if (tid < 128) {
            kfe[tid] = rkv[tid] * __expf(gam[tid | 15] - gam[tid]);
            if (tid < n && h % grp == 0) rk_out[(size_t)hq * T + t0 + tid] = rkv[tid];
        }
        __syncthreads();

        if (!delta) {
            // An update rule without the retrieval (the LinearAttention page's gated and linear rules):
            // S_new = e^{g_last} S + k_gexp^T v and o = Q'S + P v, so U = v in fp16 (rows past the chunk
            // zero) and there is no T, W or Mk.  One item per CTA in this mode.
            if (ok) wait_bar(bar_v, v_par);
            if (ok) {
                v_pend = false;
                scale_rows_f16<kIntraThreads, F16, true>(smem + OFF_T1, tid, n, [&](int) { return 1.f; }, &vmax);  // U = v
                if (tid < kFaStride) {
                    const float gl = gam[127];
                    fa[(size_t)(c * Nv + h) * kFaStride + tid] =
                        tid < 128 ? rkv[tid] * __expf(gl - gam[tid]) : (tid == 128 ? __expf(gl) : 0.f);
                }
            }
            tc::fence_proxy_async();
            __syncthreads();
            if (ok && tid == 0) {
                const int urow = (c * Nv + h) * L;
                tma::store_2d(&tm_u, 0, urow, sbase + OFF_T1);
                tma::store_2d(&tm_u, 64, urow, sbase + OFF_T1 + 16384);
                tma::commit_group();
            } else if (!ok && tid == 0) {
                atomicOr(status + 2, GDN_DEV_WAIT_INTRA);
                tc::commit(bar_d);
                tc::mbar_wait_bounded(bar_d, 0);
                if (ld_pend) tc::mbar_wait_bounded(bar_ld, ld_par);
                if (v_pend) tc::mbar_wait_bounded(bar_v, v_par);
            }
            break;
        }

        // ---- (2) Ap = -strict_tril(diag(beta rk) (k k^T) diag(rk) (.) Gamma): this thread's row and 64 columns.
        // Blocks left of the row's diagonal 16-block go to the A tile in fp16; the diagonal block goes to the
        // fp32 scratch (block b at OFF_X + 1024 b, row r at 64 r bytes, its 16-byte group q at position
        // q ^ ((r >> 1) & 3)); blocks right of it are zero.
        float *dsc = reinterpret_cast<float *>(smem + OFF_X);
        if (ok) {
            const float gi = gam[row], fr = -bet[row] * rkv[row];
            const int rb = row & ~15;  // first column of the row's diagonal block
#pragma unroll 1
            for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
                if (j0 > quarter * 32 + 31) {  // right of the diagonal for every row of the warp
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        *reinterpret_cast<uint4 *>(smem + ta + t128(row, (j0 >> 3) + c8)) = make_uint4(0, 0, 0, 0);
                    continue;
                }
                float a[32];
                tc::tmem_ld32(t_row + j0, a);
                if (j0 == quarter * 32) {
                    // The warp's diagonal chunk (warp-uniform).  Lanes 0-15 have their diagonal block at
                    // columns j0..j0+15 and nothing below the diagonal right of it; lanes 16-31 have it at
                    // j0+16.. and the block left of it at j0..j0+15.  The diagonal block goes to the fp32
                    // scratch, its decay element by element only when its gate span is too wide for the
                    // block factor; the left block goes to the fp16 tile, where the diagonal blocks are
                    // written later as T_ii.
                    const bool hi = lane >= 16;
                    float kf[16], dv[16];
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
                            dv[jj] = rb + jj < row ? x.x : 0.f;
                            dv[jj + 1] = rb + jj + 1 < row ? x.y : 0.f;
                        }
                    } else {
                        float rkj[16], gmj[16];
                        lds_vec(rkj, rkv + rb);
                        lds_vec(gmj, gam + rb);
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            dv[jj] = rb + jj < row ? fr * rkj[jj] * __expf(fminf(gi - gmj[jj], 0.f)) * (hi ? a[16 + jj] : a[jj])
                                                   : 0.f;
                    }
                    // row r of block b at OFF_X + 1024 b + 64 r, 16-byte group q at position q ^ ((r >> 1) & 3)
                    float4 *drow = reinterpret_cast<float4 *>(dsc + (rb >> 4) * 256 + (row - rb) * 16);
                    const int sw = ((row - rb) >> 1) & 3;
#pragma unroll
                    for (int q = 0; q < 4; ++q) drow[q ^ sw] = make_float4(dv[4 * q], dv[4 * q + 1], dv[4 * q + 2], dv[4 * q + 3]);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = (q8 & 1) * 8 + 2 * e;
                            w4[e] = (q8 < 2 && hi) ? pack_h2f(fmul2(fmul2(make_float2(eb, eb), make_float2(kf[jj], kf[jj + 1])),
                                                                    make_float2(a[jj], a[jj + 1])))
                                                   : 0u;
                        }
                        *reinterpret_cast<uint4 *>(smem + ta + t128(row, (j0 >> 3) + q8)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    continue;
                }
                // a chunk left of the warp's rows: the decay factored per 16-column block
                float kf[32];
                lds_vec(kf, kfe + j0);
                const float eb2[2] = {fr * __expf(gi - gam[j0 + 15]), fr * __expf(gi - gam[j0 + 31])};
#pragma unroll
                for (int q16 = 0; q16 < 2; ++q16) {
                    const int jb = j0 + q16 * 16;
                    const float eb = eb2[q16];
#pragma unroll
                    for (int q8 = 0; q8 < 2; ++q8) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = q16 * 16 + q8 * 8 + 2 * e;
                            w4[e] = pack_h2f(fmul2(fmul2(make_float2(eb, eb), make_float2(kf[jj], kf[jj + 1])),
                                                   make_float2(a[jj], a[jj + 1])));
                        }
                        *reinterpret_cast<uint4 *>(smem + ta + t128(row, (jb >> 3) + q8)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            // diag(beta e^gamma rk) k in fp16, in place (the k k^T product is complete)
            scale_rows_f16<kIntraThreads, F16>(smem + tk, tid, L, [&](int r) { return bet[r] * __expf(gam[r]) * rkv[r]; });
            // diag(beta) v in fp16, in place; rows past the chunk (the next sequence's) as zeros
            wait_bar(bar_v, v_par);
            if (ok) {
                v_pend = false;
                v_par ^= 1;
            }
            scale_rows_f16<kIntraThreads, F16>(smem + OFF_T1, tid, n, [&](int r) { return bet[r]; });
        }
        __syncthreads();

        // ---- (3) T_ii = (I - Ap_ii)^-1 by forward substitution: warp w, block w, lanes 0..15 own a column
        if (ok && lane < 16) {
            const float *ds = dsc + wid * 256;
            const int cidx = lane;
            float tcol[16];  // T_ii = I + Ap_ii T_ii, row by row; tcol[j] = 0 above the diagonal
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float nr[16];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (4 * q < i) {
                        const float4 x = reinterpret_cast<const float4 *>(ds + i * 16)[q ^ ((i >> 1) & 3)];
                        nr[4 * q] = x.x;
                        nr[4 * q + 1] = x.y;
                        nr[4 * q + 2] = x.z;
                        nr[4 * q + 3] = x.w;
                    }
                // even j into the first lane of the pair, odd j into the second (packed fp32 pairs)
                float2 s2 = make_float2(i == cidx ? 1.f : 0.f, 0.f);
#pragma unroll
                for (int j = 0; j + 1 < i; j += 2)
                    s2 = ffma2(make_float2(nr[j], nr[j + 1]), make_float2(tcol[j], tcol[j + 1]), s2);
                if (i & 1) s2.x = fmaf(nr[i - 1], tcol[i - 1], s2.x);
                tcol[i] = i < cidx ? 0.f : s2.x + s2.y;
            }
            const int col = wid * 16 + cidx;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __half hv = __float2half_rn(tcol[i]);
                *reinterpret_cast<uint16_t *>(smem + ta + t128(wid * 16 + i, col >> 3) + (col & 7) * 2) =
                    *reinterpret_cast<uint16_t *>(&hv);
            }
        }
        __syncthreads();
        // merge levels: T21 = T22 (Ap21 T11), the product in brackets through the fp16 scratch
        const uint32_t aA = sbase + ta, aX = sbase + OFF_X;
        uint8_t *pA = smem + ta, *pX = smem + OFF_X;
        auto fA = [](int r, int cc) { return t128(r, cc); };
        auto fX = [](int r, int cc) { return x64(r, cc); };
        if (ok) {
            // 16 -> 32: warp p < 4 merges blocks (32p + 16, 32p)
            if (wid < 4) {
                const int a = 32 * wid, bb = a + 16;
                float acc[2][4] = {};
                warp_mm<1>(acc, aA, fA, bb, a, aA, fA, a, a, 1, lane);
                warp_store16(acc, pX, fX, 16 * wid, 0, lane);
                __syncwarp();
                float acc2[2][4] = {};
                warp_mm<1>(acc2, aA, fA, bb, bb, aX, fX, 16 * wid, 0, 1, lane);
                warp_store16(acc2, pA, fA, bb, a, lane);
            }
            __syncthreads();
            // 32 -> 64: warps 4p .. 4p+3 merge 32-blocks (64p + 32, 64p), one 16 x 16 tile each
            {
                const int p = wid >> 2, mi = (wid >> 1) & 1, ni = wid & 1;
                const int a = 64 * p, bb = a + 32;
                float acc[2][4] = {};
                warp_mm<2>(acc, aA, fA, bb + 16 * mi, a + 16 * ni, aA, fA, a + 16 * ni, a + 16 * ni, 2 - ni, lane);
                warp_store16(acc, pX, fX, 32 * p + 16 * mi, 16 * ni, lane);
                __syncthreads();
                float acc2[2][4] = {};
                warp_mm<2>(acc2, aA, fA, bb + 16 * mi, bb, aX, fX, 32 * p, 16 * ni, mi + 1, lane);
                warp_store16(acc2, pA, fA, bb + 16 * mi, a + 16 * ni, lane);
            }
            __syncthreads();
            // 64 -> 128: the 64-blocks (64, 0).  X = Ap21 T11 takes 4 - ni k-steps for tile (mi, ni), so
            // warp w takes tiles (w / 2, w % 2) and (w / 2, 3 - w % 2): five steps for every warp
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int mi = wid >> 1, ni = rep ? 3 - (wid & 1) : (wid & 1);
                float acc[2][4] = {};
                warp_mm<4>(acc, aA, fA, 64 + 16 * mi, 16 * ni, aA, fA, 16 * ni, 16 * ni, 4 - ni, lane);
                warp_store16(acc, pX, fX, 16 * mi, 16 * ni, lane);
            }
            __syncthreads();
            // T21 = T22 X takes mi + 1 k-steps: warp w takes tiles (w % 2, w / 2) and (3 - w % 2, w / 2)
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int ni = wid >> 1, mi = rep ? 3 - (wid & 1) : (wid & 1);
                float acc[2][4] = {};
                warp_mm<4>(acc, aA, fA, 64 + 16 * mi, 64, aX, fX, 0, 16 * ni, mi + 1, lane);
                warp_store16(acc, pA, fA, 64 + 16 * mi, 16 * ni, lane);
            }
        }
        sync_operands();

        // ---- (4) [W | U] = T [diag(beta e^gamma rk) k | diag(beta) v] into TMEM columns [0, 256).  The B
        // operand is one N = 256 MN-major operand of four 64-column blocks 16 KiB apart: [k | v] from tile 0
        // when the k tile is tile 0, [v | k] from tile 1 when it is tile 2, so W lands in TMEM columns
        // [128 wsel, 128 wsel + 128) and U in the other half
        const int wsel = li & 1;
        if (ok && tid == 0) {
            const uint64_t dt = tc::desc_k128(sbase + ta), dr = tc::desc_mn(sbase + (wsel ? OFF_T1 : OFF_T0), 16384, 1024, 2);
            const uint32_t idesc = tc::idesc_f16(128, 256, false, false, false, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem, kmaj(dt, kk), dr + (uint64_t)((kk * 2048) >> 4), idesc, kk > 0 ? 1u : 0u);
            tc::commit(bar_mma);
        }
        if (ok) {
            wait_bar(bar_mma, mma_phase);
            mma_phase ^= 1;
        }
        if (ok && tid == 0) load_k(tk, hq, t0);  // the k rows again, for k_gexp (the first use of the tile is over)
        if (ok) {
            ld_pend = true;
            ld_par = 1;
        }
        if (ok) {
            // W into the v tile, where it is also Mk's B operand, and U into the A tile, in fp16 (warps
            // 4 wsel .. 4 wsel + 3 hold W); both leave for global memory by TMA
            uint8_t *dst = smem + (half == wsel ? OFF_T1 : ta);
#pragma unroll 1
            for (int j0 = 0; j0 < 128; j0 += 32) {
                float a[32];
                tc::tmem_ld32(t_row + half * 128 + j0, a);
                // U (v-derived; an out-of-range beta v shows up here as inf or NaN); W and Mk are bounded
                // by T, since their other factors have entries of magnitude <= 1
                if (half != wsel) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) vmax = absmax_nan(vmax, a[e]);
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(dst + t128(row, (j0 >> 3) + q8)) =
                        make_uint4(pack_h2(a[8 * q8], a[8 * q8 + 1]), pack_h2(a[8 * q8 + 2], a[8 * q8 + 3]),
                                   pack_h2(a[8 * q8 + 4], a[8 * q8 + 5]), pack_h2(a[8 * q8 + 6], a[8 * q8 + 7]));
            }
            // the state pass's per-row factors rk_t e^{g_last - gamma_t} (0 past the chunk) and e^{g_last}
            if (tid < kFaStride) {
                const float gl = gam[127];  // gam is clamped to the last valid row
                const float f = tid < 128 ? rkv[tid] * __expf(gl - gam[tid]) : (tid == 128 ? __expf(gl) : 0.f);
                fa[(size_t)(c * Nv + h) * kFaStride + tid] = f;
                if (tid < 128) kfe[tid] = f;  // k_gexp's row factors (the column factors are no longer needed)
            }
        }

        const int trow = (c * Nv + h) * L;  // first row of the chunk's tiles in the workspace
        tc::fence_proxy_async();
        __syncthreads();
        if (ok && tid == 0) {
            tma::store_2d(&tm_w, 0, trow, sbase + OFF_T1);
            tma::store_2d(&tm_w, 64, trow, sbase + OFF_T1 + 16384);
            tma::store_2d(&tm_u, 0, trow, sbase + ta);
            tma::store_2d(&tm_u, 64, trow, sbase + ta + 16384);
            tma::commit_group();
        }

        // ---- (5) k_gexp = fp16(rk e^{g_last - gamma} k) over the reloaded k rows (zero past the chunk), then Mk
        if (ok) wait_bar(bar_ld, 1);
        if (ok) scale_rows_f16<kIntraThreads, F16>(smem + tk, tid, n, [&](int r) { return kfe[r]; });
        sync_operands();
        // Mk = k_gexp^T W: A = k_gexp read MN-major (Dk contiguous), B = W MN-major; TMEM columns [0, 128)
        if (ok && tid == 0) {
            const uint64_t da = tc::desc_mn(sbase + tk, 16384, 1024, 2), db = tc::desc_mn(sbase + OFF_T1, 16384, 1024, 2);
            const uint32_t idesc = tc::idesc_f16(128, 128, false, false, true, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem, da + (uint64_t)((kk * 2048) >> 4), db + (uint64_t)((kk * 2048) >> 4), idesc,
                            kk > 0 ? 1u : 0u);
            tc::commit(bar_mma);
            if (nit < items) {
                // the next item's k rows into this item's A tile, once the U store has read it
                tma::wait_read_all();
                load_k(ta, (nit / nc) / grp, load_chunk(info, c0 + nit % nc).start);
            }
        }
        if (ok && nit < items) {
            ld_pend = true;
            ld_par = 0;
        }
        if (ok) {
            wait_bar(bar_mma, mma_phase);
            mma_phase ^= 1;
        }
        if (ok && nit < items) {
            // the next item's v rows, now that Mk has consumed W (the W store was read before)
            if (tid == 0) load_v(nit / nc, load_chunk(info, c0 + nit % nc).start);
            v_pend = true;
        }
        if (ok) {
            // warp w: row 32 (w % 4) + lane of Mk, columns 64 (w / 4) .. +63, into the (consumed) k tile
#pragma unroll 1
            for (int j0 = 0; j0 < 64; j0 += 32) {
                float a[32];
                tc::tmem_ld32(t_row + half * 64 + j0, a);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *reinterpret_cast<uint4 *>(smem + tk + t128(row, half * 8 + (j0 >> 3) + q8)) =
                        make_uint4(pack_h2(a[8 * q8], a[8 * q8 + 1]), pack_h2(a[8 * q8 + 2], a[8 * q8 + 3]),
                                   pack_h2(a[8 * q8 + 4], a[8 * q8 + 5]), pack_h2(a[8 * q8 + 6], a[8 * q8 + 7]));
            }
            tc::fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                tma::store_2d(&tm_mk, 0, trow, sbase + tk);
                tma::store_2d(&tm_mk, 64, trow, sbase + tk + 16384);
                tma::commit_group();
            }
        }
        if (!ok) {
            if (tid == 0) {
                atomicOr(status + 2, GDN_DEV_WAIT_INTRA);
                // MMAs and loads still in flight land before shared and tensor memory are released: a
                // commit covers every MMA issued before it; each barrier has at most one load phase open
                tc::commit(bar_d);
                tc::mbar_wait_bounded(bar_d, 0);
                if (ld_pend) tc::mbar_wait_bounded(bar_ld, ld_par);
                if (v_pend) tc::mbar_wait_bounded(bar_v, v_par);
            }
            break;
        }
        if (nit >= items) break;
        it = nit;
        h = it / nc;
        c = c0 + it % nc;
        ci = load_chunk(info, c);
        xg = ng;
        xb = nb;
    }
    if (tid == 0) tma::wait_read_all();  // the stores have read shared memory (the grid's end publishes them)
    if (__any_sync(0xffffffffu, out_of_fp16(vmax)) && lane == 0) atomicOr(status + 3, GDN_DEV_RANGE_INTRA);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, 256);
}

cudaError_t launch_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps, int T,
                         int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st, bool delta, bool f16,
                         Dims dims)
{
    if (nc <= 0 || T == 0) return cudaSuccess;
    if (c0 < 0 || c0 + nc > ws.NC) return cudaErrorInvalidValue;
    const uint64_t trows = (uint64_t)ws.NC * Nv * L;  // TMA coordinates are 32-bit signed
    if ((uint64_t)T >= (1ull << 31) || trows >= (1ull << 31)) return cudaErrorInvalidValue;
    CUtensorMap m_k, m_v, m_u, m_w, m_mk;
    const auto AT = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cudaError_t e = tma::map_heads(&m_k, AT, k, (uint64_t)dims.Dk, (uint64_t)Nqk, (uint64_t)T, 128);
    if (e == cudaSuccess)
        e = tma::map2d(&m_v, AT, v, (uint64_t)Nv * D, (uint64_t)T, (uint64_t)Nv * D * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = tma::map2d(&m_u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.U, D, trows, D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = tma::map2d(&m_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.W, D, trows, D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = tma::map2d(&m_mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.Mk, D, trows, D * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    auto kern = f16 ? intra_kernel<true> : intra_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kIntraSmem);
    if (e != cudaSuccess) return e;
    const int items = nc * Nv;  // below 2^31: nc Nv L rows are addressable
    const int per = delta ? kIntraItemsPerCta : 1;
    const int grid = (items + per - 1) / per;
    kern<<<grid, kIntraThreads, kIntraSmem, st>>>(m_k, m_v, m_u, m_w, m_mk, g, beta, eps, T, Nqk, Nv, ws.chunk_info,
                                                   ws.rk, ws.gcum, ws.betaf, ws.fa, ws.status, c0, nc, delta ? 1 : 0,
                                                   dims.m);
    return cudaGetLastError();
}

}  // namespace gdn
