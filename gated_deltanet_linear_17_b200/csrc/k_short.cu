// Fused short-sequence forward: one CTA per (sequence, v-head, 32-column slice of Dv;
// 64 columns with a bf16 pool).
//
// The decode page ("lite_boost.ops.recurrent_gated_delta_rule", algorithm
// flow) runs the Gated Delta Rule token by token for a few tokens per call,
// reading and writing a slot of a state pool.  For such batches the work is
// moving the states: 64 KiB of fp32 state per (sequence, v-head) in and out,
// against a few hundred bytes of q/k/v per token, so the kernel is a stream:
// each CTA issues the loads of its state slice (warp w holds Dk rows
// 32w..32w+31, lane j holds column j, one 128-byte row segment per warp load)
// together with cp.async copies of the token data of up to PRE tokens (q and
// k rows, the v slice, g), so that a single memory latency covers both.  The q
// and k rows are then normalised as in "L2 Normalization" into fp32 rows in
// shared memory (q with the scale), and the tokens are applied from registers,
//   S = e^g S;  kv = S^T kh;  S += kh (beta (v - kv))^T;  o = S^T qh,
// with the sums over Dk taken per warp and then across the four warps through
// shared memory (two barriers per token, the partial sums double-buffered by
// token parity), and the per-element work in packed fp32 pairs.  The final slice
// is written from registers.  Tokens past PRE are read directly from global
// memory, so the kernel is exact for any sequence length; it is only fast for
// short ones.  PRE is 8 when every sequence is known to have at most 8 tokens,
// else 16: the staging area then stays small enough for eight CTAs per SM (the
// register file holds eight state slices), where 16 staged tokens leave room for
// seven.
//
// With SLOTS the pool is updated in place with one slot index per token (page
// "lite_boost.ops.recurrent_gated_delta_rule": ssm_state_indices per token,
// num_accepted_tokens, state_out): a sequence starts from the slot of its last
// accepted token, slots[t0 + a - 1], and the state after token j is written to
// slots[t0 + j] whenever the next token's slot differs or j is the last token
// (a run of tokens on one slot keeps only its last state, so this writes every
// slot's final value).  A CTA reads its slice of the starting slot before it
// writes anything, and the slots of different sequences are disjoint, so the
// in-place update is race-free.  Two more options of that page's operator: a
// bf16 state pool (SBF: the state is widened to fp32 on load and rounded to bf16
// when written) and the key-dimension gate gk (GK: S = S e^g e^gk, row i of S
// decayed by e^{g + gk_i}; the 128 factors of each staged token are computed once
// per CTA into shared memory, and the state rows are decayed before the sum
// S^T kh).  With a state window (`win` = W > 0, the LinearAttention page's
// state_window) the pool is the window buffer [W, B, ...] seen as W B slots,
// slot w B + b holding entry w of sequence b: the sequence starts from entry
// W - 1 and the state after token j of its n goes to entry W - n + j when that
// is >= 0 (earlier tokens' states leave the window and are not written); the
// entries that a sequence shorter than the window keeps were moved down by
// window_shift_kernel before this kernel runs.  DECAY and DELTA select the update rule of the page
// "com.microsoft.LinearAttention" (update_rule): gated_delta (both), delta (no
// decay: g and gk unused), gated (S = e^g S + kh v^T: no retrieval, beta unused)
// and linear (S = S + kh v^T); without the retrieval a token needs one barrier.
#include "common.cuh"

#include <type_traits>
#include "gdn_internal.h"

namespace gdn {

constexpr int kTile = 32;  // Dv columns per CTA

// element types of the activations (q, k, v, out) and of the state pool
constexpr int kF32 = 0, kBF16 = 1, kF16 = 2;

template <int DT>  // a 16-bit value of type DT widened to fp32
__device__ __forceinline__ float wide16(uint16_t x)
{
    if constexpr (DT == kBF16) return bf2f(x);
    else return __half2float(__ushort_as_half(x));
}
template <int DT>  // fp32 rounded to nearest even in the 16-bit type DT
__device__ __forceinline__ uint16_t narrow16(float x)
{
    if constexpr (DT == kBF16) return f2bf(x);
    else return __half_as_ushort(__float2half_rn(x));
}
template <int DT>  // element i of an activation array of type DT
__device__ __forceinline__ float ld_act(const void *p, size_t i)
{
    if constexpr (DT == kF32) return static_cast<const float *>(p)[i];
    else return wide16<DT>(static_cast<const uint16_t *>(p)[i]);
}
template <int DT>
__device__ __forceinline__ void st_act(void *p, size_t i, float x)
{
    if constexpr (DT == kF32) static_cast<float *>(p)[i] = x;
    else static_cast<uint16_t *>(p)[i] = narrow16<DT>(x);
}
template <int DT>  // elements 2e, 2e + 1 of a staged row of type DT
__device__ __forceinline__ float2 pair_at(const uint16_t *row, int e)
{
    if constexpr (DT == kF32) return reinterpret_cast<const float2 *>(row)[e];
    else if constexpr (DT == kF16) return __half22float2(reinterpret_cast<const __half2 *>(row)[e]);
    else {
        const uint32_t w = reinterpret_cast<const uint32_t *>(row)[e];
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
}

// DK: key dimension (64 or 128); the CTA has DK threads, warp w holding state rows 32w .. 32w + 31.
// SDT: the pool's type; with a 16-bit pool the CTA covers 64 columns, its slice staged in shared
// memory (sst).  ADT: the activations' type (raw rows staged as bytes, 16-bit units).
template <int PRE, bool GK, int DK, int SDT, int ADT>  // tokens staged together with the state; key gate
struct ShortSmem {
    static constexpr int AU = ADT == kF32 ? 2 : 1;  // 16-bit units per activation element
    float kh[PRE][DK], qh[PRE][DK];   // normalised rows, fp32 (qh includes the scale)
    float gkd[GK ? PRE : 1][DK];      // gk rows, then the row decays e^{g + gk} (GK)
    uint16_t sst[SDT != kF32 ? DK : 1][SDT != kF32 ? 64 : 8];  // the 16-bit state slice
    uint16_t q[PRE][DK * AU], k[PRE][DK * AU];                  // raw rows
    uint16_t v[PRE][(SDT != kF32 ? 64 : 32) * AU];              // raw slice
    float g[PRE], dg[PRE], beta[PRE];
    int32_t slot[PRE + 1];  // token slots (SLOTS)
    float red[2][DK / 32][32], red2[2][DK / 32][32];
};

// sum over the warps of a [DK / 32][32] partial-sum array at this lane's column
template <int NW>
__device__ __forceinline__ float sum_warps(const float (&r)[NW][32], int lane)
{
    float a = r[0][lane];
#pragma unroll
    for (int w = 1; w < NW; ++w) a += r[w][lane];
    return a;
}

// The kernel body, entered through two kernels that differ only in their register budget:
// gdn_chunk_fwd's short path is held to 64 registers, eight CTAs per SM (without a bound the compiler
// takes 78 and fits six); the pool-slot variants keep the compiler's own choice (an explicit minimum of
// one CTA per SM makes it spend up to 142 registers and fit three; other explicit budgets measured
// slower at Dk = 64).
template <int PRE, bool SLOTS, bool GK, int SDT, bool DECAY, bool DELTA, int DK, int ADT>
__device__ __forceinline__ void short_body(
    const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
    const float *__restrict__ g, const uint16_t *__restrict__ beta, const float *__restrict__ gk,
    const int32_t *__restrict__ cu, const void *pool, const int32_t *__restrict__ idx,
    const int32_t *__restrict__ token_slots, const int32_t *__restrict__ num_accepted, void *pool_w, float scale,
    float eps, void *__restrict__ out, float *__restrict__ final_state, int T, int Nqk, int Nv, int Dv, int win,
    int Bw)
{
    constexpr bool SBF = SDT != kF32;          // a 16-bit pool
    constexpr int AES = ADT == kF32 ? 4 : 2;   // activation element bytes
    constexpr int NW = DK / 32, EL = DK / 32;  // warps; elements of a q/k row per lane
    // Dv columns per CTA: with a bf16 pool 64, the slice (16 KiB at Dk = 128) fetched by cp.async into
    // shared memory and the tokens applied to one 32-column half after the other, so a CTA keeps twice
    // the bytes in flight with the same registers
    constexpr int CW = SBF ? 64 : 32;
    __shared__ __align__(16) ShortSmem<PRE, GK, DK, SDT, ADT> sm;
    const int b = blockIdx.x, h = blockIdx.y, tl = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int col = tl * CW + lane;
    const int hq = h / (Nv / Nqk);
    const int t0 = min(max(cu[b], 0), T);
    const int t1 = min(max(cu[b + 1], t0), T);
    const int n = t1 - t0, npre = min(n, PRE);
    if (SLOTS && n == 0) return;  // no token: the pool keeps its slots

    // token data of the first kPre tokens: async copies
    constexpr int QC = DK * AES / 16, VC = CW * AES / 16;  // 16-byte pieces of a q/k row, of the v slice
    for (int e = tid; e < npre * QC; e += DK) {
        const int t = e / QC, c = e % QC;
        const size_t off = (((size_t)(t0 + t) * Nqk + hq) * DK) * AES + c * 16;
        cp_async16(smem_addr(&sm.q[t][c * 8]), static_cast<const char *>(q) + off, true);
        cp_async16(smem_addr(&sm.k[t][c * 8]), static_cast<const char *>(k) + off, true);
    }
    for (int e = tid; e < npre * VC; e += DK) {
        const int t = e / VC, c = e % VC;
        const size_t off = (((size_t)(t0 + t) * Nv + h) * Dv + tl * CW) * AES + c * 16;
        cp_async16(smem_addr(&sm.v[t][c * 8]), static_cast<const char *>(v) + off, true);
    }
    if (DECAY && tid < npre) cp_async4(smem_addr(&sm.g[tid]), g + (size_t)(t0 + tid) * Nv + h);
    // the window slot of token j (-1: its state leaves the window and is not written)
    auto win_slot = [&](int j) { return j >= n - win ? (win - n + j) * Bw + b : -1; };
    if (SLOTS && tid <= PRE && tid < n) {
        if (win > 0) sm.slot[tid] = win_slot(tid);
        else cp_async4(smem_addr(&sm.slot[tid]), token_slots + t0 + tid);
    }
    if (GK) {
        for (int e = tid; e < npre * (DK / 4); e += DK) {
            const int t = e / (DK / 4), c = e % (DK / 4);
            cp_async16(smem_addr(&sm.gkd[t][c * 4]), gk + ((size_t)(t0 + t) * Nv + h) * DK + c * 4, true);
        }
    }
    // the starting slot
    int slot0 = 0;
    if (pool) {
        if (SLOTS && win > 0) {  // the window's newest entry
            slot0 = (win - 1) * Bw + b;
        } else if (SLOTS) {  // the state after the last accepted token (n >= 1 here)
            const int a = min(max(num_accepted ? num_accepted[b] : n, 1), n);
            slot0 = token_slots[t0 + a - 1];
        } else {
            slot0 = idx ? idx[b] : b;
        }
    }
    if (SBF && pool) {  // the bf16 slice [DK][64] (128-byte row segments) into shared memory
        const unsigned short *src = static_cast<const unsigned short *>(pool) + ((size_t)slot0 * Nv + h) * DK * Dv + tl * CW;
        for (int e = tid; e < DK * 8; e += DK) {
            const int r = e >> 3, c = e & 7;
            cp_async16(smem_addr(&sm.sst[r][c * 8]), src + (size_t)r * Dv + c * 8, true);
        }
    }
    cp_async_commit();
    float bt_mine = 0.f;
    if (DELTA && tid < npre) bt_mine = bf2f(beta[(size_t)(t0 + tid) * Nv + h]);

    // fp32 pool: the state slice straight into registers, s2[m] holding rows 32 wid + 2m, 2m + 1
    // (bf16 pool: from shared memory, one half at a time, below)
    float2 s2[16];
    if (pool && !SBF) {
        const size_t off = (((size_t)slot0 * Nv + h) * DK + wid * 32) * Dv + col;
        {
            const float *src = static_cast<const float *>(pool) + off;
#pragma unroll
            for (int m = 0; m < 16; ++m)
                s2[m] = make_float2(__ldcs(src + (size_t)(2 * m) * Dv), __ldcs(src + (size_t)(2 * m + 1) * Dv));
        }
    } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) s2[m] = make_float2(0.f, 0.f);
    }

    // this thread's 32 values of the state into pool slot `slot` (SLOTS)
    auto write_slot = [&](int slot) {
        const size_t off = (((size_t)slot * Nv + h) * DK + wid * 32) * Dv + col;
        if (SBF) {
            unsigned short *dst = static_cast<unsigned short *>(pool_w) + off;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                __stcs(dst + (size_t)(2 * m) * Dv, (unsigned short)narrow16<SDT>(s2[m].x));
                __stcs(dst + (size_t)(2 * m + 1) * Dv, (unsigned short)narrow16<SDT>(s2[m].y));
            }
        } else {
            float *dst = static_cast<float *>(pool_w) + off;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                __stcs(dst + (size_t)(2 * m) * Dv, s2[m].x);
                __stcs(dst + (size_t)(2 * m + 1) * Dv, s2[m].y);
            }
        }
    };

    cp_async_wait<0>();
    if (tid < npre) sm.beta[tid] = bt_mine;
    __syncthreads();
    // normalised q and k rows in fp32 and the decay of every staged token: one warp per token,
    // lane l at elements EL l .. EL l + EL - 1
    for (int t = wid; t < npre; t += NW) {
        float qe[EL], ke[EL];
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e2 = 0; e2 < EL / 2; ++e2) {
            const float2 qp = pair_at<ADT>(&sm.q[t][0], lane * EL / 2 + e2);
            const float2 kp = pair_at<ADT>(&sm.k[t][0], lane * EL / 2 + e2);
            qe[2 * e2] = qp.x;
            qe[2 * e2 + 1] = qp.y;
            ke[2 * e2] = kp.x;
            ke[2 * e2 + 1] = kp.y;
        }
#pragma unroll
        for (int e = 0; e < EL; ++e) {
            sq = fmaf(qe[e], qe[e], sq);
            sk = fmaf(ke[e], ke[e], sk);
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        const float rq = scale / sqrtf(sq + eps), rk = 1.0f / sqrtf(sk + eps);
#pragma unroll
        for (int e2 = 0; e2 < EL / 2; ++e2) {
            reinterpret_cast<float2 *>(&sm.qh[t][lane * EL])[e2] = make_float2(qe[2 * e2] * rq, qe[2 * e2 + 1] * rq);
            reinterpret_cast<float2 *>(&sm.kh[t][lane * EL])[e2] = make_float2(ke[2 * e2] * rk, ke[2 * e2 + 1] * rk);
        }
        if (lane == 0) sm.dg[t] = DECAY ? __expf(sm.g[t]) : 1.f;
    }
    if (GK) {  // the row decays e^{g + gk_i} of every staged token, in place over gk (thread i: row i)
        for (int t = 0; t < npre; ++t) sm.gkd[t][tid] = __expf(sm.g[t] + sm.gkd[t][tid]);
    }
    __syncthreads();

#pragma unroll 1
    for (int half = 0; half < CW / 32; ++half) {
    if (SBF) {
        col = tl * CW + half * 32 + lane;
        if (half) __syncthreads();  // the previous half's last partial sums have been read
        if (pool) {
#pragma unroll
            for (int m = 0; m < 16; ++m)
                s2[m] = make_float2(wide16<SDT>(sm.sst[wid * 32 + 2 * m][half * 32 + lane]),
                                    wide16<SDT>(sm.sst[wid * 32 + 2 * m + 1][half * 32 + lane]));
        } else {
#pragma unroll
            for (int m = 0; m < 16; ++m) s2[m] = make_float2(0.f, 0.f);
        }
    }
    const int vc = half * 32 + lane;  // this thread's column in the staged v slice

    for (int j = 0; j < npre; ++j) {
        const int p = j & 1;
        const float4 *kr = reinterpret_cast<const float4 *>(&sm.kh[j][wid * 32]);
        const float4 *qr = reinterpret_cast<const float4 *>(&sm.qh[j][wid * 32]);
        // the decay as one factor (applied to the sum S^T kh and in the update), or per row (GK: applied
        // to the state rows first)
        const float dg = (GK || !DECAY) ? 1.f : sm.dg[j];
        float vj;
        if constexpr (ADT == kF32) vj = reinterpret_cast<const float *>(&sm.v[j][0])[vc];
        else vj = wide16<ADT>(sm.v[j][vc]);
        if (GK) {
            const float4 *dr = reinterpret_cast<const float4 *>(&sm.gkd[j][wid * 32]);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 d4 = dr[c];
                s2[2 * c] = fmul2(s2[2 * c], make_float2(d4.x, d4.y));
                s2[2 * c + 1] = fmul2(s2[2 * c + 1], make_float2(d4.z, d4.w));
            }
        }
        float u = vj;
        if (DELTA) {  // this warp's part of S^T kh, then u = beta (v - S^T kh)
            float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 kx = kr[c];
                a0 = ffma2(s2[2 * c], make_float2(kx.x, kx.y), a0);
                a1 = ffma2(s2[2 * c + 1], make_float2(kx.z, kx.w), a1);
            }
            sm.red[p][wid][lane] = (a0.x + a0.y) + (a1.x + a1.y);
            __syncthreads();
            const float kv = dg * sum_warps<NW>(sm.red[p], lane);
            u = sm.beta[j] * (vj - kv);
        }
        const float2 dg2 = make_float2(dg, dg), u2 = make_float2(u, u);
        // S = e^g S + kh u^T (GK: S already decayed), then this warp's part of S^T qh
        float2 b0 = make_float2(0.f, 0.f), b1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 kx = kr[c], qx = qr[c];
            if (GK || !DECAY) {
                s2[2 * c] = ffma2(make_float2(kx.x, kx.y), u2, s2[2 * c]);
                s2[2 * c + 1] = ffma2(make_float2(kx.z, kx.w), u2, s2[2 * c + 1]);
            } else {
                s2[2 * c] = ffma2(make_float2(kx.x, kx.y), u2, fmul2(s2[2 * c], dg2));
                s2[2 * c + 1] = ffma2(make_float2(kx.z, kx.w), u2, fmul2(s2[2 * c + 1], dg2));
            }
            b0 = ffma2(s2[2 * c], make_float2(qx.x, qx.y), b0);
            b1 = ffma2(s2[2 * c + 1], make_float2(qx.z, qx.w), b1);
        }
        sm.red2[p][wid][lane] = (b0.x + b0.y) + (b1.x + b1.y);
        if (SLOTS && sm.slot[j] >= 0 && (j == n - 1 || sm.slot[j + 1] != sm.slot[j])) write_slot(sm.slot[j]);
        __syncthreads();
        if (wid == 0)
            st_act<ADT>(out, ((size_t)(t0 + j) * Nv + h) * Dv + col, sum_warps<NW>(sm.red2[p], lane));
    }

    // beyond the staged tokens (longer sequences than the fused path is meant for): read directly
    for (int j = PRE; j < n; ++j) {
        const int t = t0 + j, p = j & 1;
        const size_t qrow = ((size_t)t * Nqk + hq) * DK;  // first element of the token's q and k rows
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int i = 0; i < EL; ++i) {
            const float a = ld_act<ADT>(q, qrow + lane + 32 * i), c = ld_act<ADT>(k, qrow + lane + 32 * i);
            sq = fmaf(a, a, sq);
            sk = fmaf(c, c, sk);
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        const float rq = scale / sqrtf(sq + eps), rk = 1.0f / sqrtf(sk + eps);
        const float vj = ld_act<ADT>(v, ((size_t)t * Nv + h) * Dv + col);
        const float gt = DECAY ? g[(size_t)t * Nv + h] : 0.f, bt = DELTA ? bf2f(beta[(size_t)t * Nv + h]) : 1.f;
        const float dg = (GK || !DECAY) ? 1.f : __expf(gt);
        if (GK) {  // this thread's 32 rows decayed by e^{g + gk_i}
            const float *gr = gk + ((size_t)t * Nv + h) * DK + wid * 32;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                s2[m].x *= __expf(gt + gr[2 * m]);
                s2[m].y *= __expf(gt + gr[2 * m + 1]);
            }
        }
        const size_t kr = qrow + wid * 32, qr = qrow + wid * 32;  // this warp's 32 rows
        float u = vj;
        if (DELTA) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                acc = fmaf(s2[m].x, ld_act<ADT>(k, kr + 2 * m) * rk, acc);
                acc = fmaf(s2[m].y, ld_act<ADT>(k, kr + 2 * m + 1) * rk, acc);
            }
            sm.red[p][wid][lane] = acc;
            __syncthreads();
            const float kv = dg * sum_warps<NW>(sm.red[p], lane);
            u = bt * (vj - kv);
        }
        float acc2 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            s2[m].x = fmaf(ld_act<ADT>(k, kr + 2 * m) * rk, u, s2[m].x * dg);
            s2[m].y = fmaf(ld_act<ADT>(k, kr + 2 * m + 1) * rk, u, s2[m].y * dg);
            acc2 = fmaf(s2[m].x, ld_act<ADT>(q, qr + 2 * m) * rq, acc2);
            acc2 = fmaf(s2[m].y, ld_act<ADT>(q, qr + 2 * m + 1) * rq, acc2);
        }
        sm.red2[p][wid][lane] = acc2;
        if (SLOTS) {
            const int sj = win > 0 ? win_slot(j) : token_slots[t];
            const int sn = j + 1 < n ? (win > 0 ? win_slot(j + 1) : token_slots[t + 1]) : -1;
            if (sj >= 0 && (j == n - 1 || sn != sj)) write_slot(sj);
        }
        __syncthreads();
        if (wid == 0)
            st_act<ADT>(out, ((size_t)t * Nv + h) * Dv + col, sum_warps<NW>(sm.red2[p], lane));
    }

    if (!SLOTS && final_state) {
        float *dst = final_state + (((size_t)b * Nv + h) * DK + wid * 32) * Dv + col;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            __stcs(dst + (size_t)(2 * m) * Dv, s2[m].x);
            __stcs(dst + (size_t)(2 * m + 1) * Dv, s2[m].y);
        }
    }
    }  // half
}

#define GDN_SHORT_PARAMS                                                                                           \
    const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,                          \
        const float *__restrict__ g, const uint16_t *__restrict__ beta, const float *__restrict__ gk,            \
        const int32_t *__restrict__ cu, const void *pool, const int32_t *__restrict__ idx,                       \
        const int32_t *__restrict__ token_slots, const int32_t *__restrict__ num_accepted, void *pool_w,         \
        float scale, float eps, void *__restrict__ out, float *__restrict__ final_state, int T, int Nqk, int Nv, \
        int Dv, int win, int Bw
#define GDN_SHORT_ARGS                                                                                              \
    q, k, v, g, beta, gk, cu, pool, idx, token_slots, num_accepted, pool_w, scale, eps, out, final_state, T, Nqk, Nv, \
        Dv, win, Bw

// Two entry kernels around one body, each with its own register budget.  The pool
// pass of the chunked forward (bf16 activations, fp32 state, one slot per sequence)
// is held to 64 registers, eight CTAs per SM: the register file then holds eight
// 32-column state slices, the most in flight.  The per-token-slot variants (key gate,
// 16-bit pools, other activation types and head dimensions) keep the compiler's own
// choice: capped at 64 they spill, and a minimum of one CTA per SM lets the compiler
// take so many registers that only three fit.
template <int PRE, bool GK, int SDT, bool DECAY, bool DELTA, int DK, int ADT>
__global__ void __launch_bounds__(DK) short_kernel_slots(GDN_SHORT_PARAMS)
{
    short_body<PRE, true, GK, SDT, DECAY, DELTA, DK, ADT>(GDN_SHORT_ARGS);
}

template <int PRE, bool DECAY, bool DELTA>
__global__ void __launch_bounds__(D, 8) short_kernel(GDN_SHORT_PARAMS)
{
    short_body<PRE, false, false, kF32, DECAY, DELTA, D, kBF16>(GDN_SHORT_ARGS);
}

template <int PRE, bool SLOTS, bool GK, int SDT, bool DECAY, bool DELTA, int DK, int ADT>
static void launch_variant(dim3 grid, cudaStream_t st, const void *q, const void *k, const void *v, const float *g,
                           const uint16_t *beta, const float *gk, const int32_t *cu, const void *pool,
                           const int32_t *idx, const int32_t *token_slots, const int32_t *num_accepted, void *pool_w,
                           float scale, float eps, void *out, float *final_state, int T, int Nqk, int Nv, int Dv,
                           int win = 0, int Bw = 0)
{
    if constexpr (SLOTS)
        short_kernel_slots<PRE, GK, SDT, DECAY, DELTA, DK, ADT><<<grid, DK, 0, st>>>(
            q, k, v, g, beta, gk, cu, pool, idx, token_slots, num_accepted, pool_w, scale, eps, out, final_state, T,
            Nqk, Nv, Dv, win, Bw);
    else
        short_kernel<PRE, DECAY, DELTA><<<grid, DK, 0, st>>>(q, k, v, g, beta, gk, cu, pool, idx, token_slots,
                                                               num_accepted, pool_w, scale, eps, out, final_state, T,
                                                               Nqk, Nv, Dv, 0, 0);
}

// Arguments of one pool-updating launch
struct RecArgs {
    const void *q, *k, *v;
    const float *g;
    const uint16_t *beta;
    const float *gk;
    const int32_t *cu;
    void *pool;
    const int32_t *token_slots, *num_accepted;
    float scale, eps;
    void *out;
    int T, Nqk, Nv, Dv;
    int win, Bw;  // state window (0: none) and the number of sequences
};

template <int PRE, bool GK, int SDT, bool DECAY, bool DELTA, int DK, int ADT>
static void launch_pool(const RecArgs &a, dim3 grid, cudaStream_t st)
{
    grid.z = a.Dv / (SDT != kF32 ? 64 : 32);  // Dv columns per CTA
    launch_variant<PRE, true, GK, SDT, DECAY, DELTA, DK, ADT>(grid, st, a.q, a.k, a.v, a.g, a.beta, a.gk, a.cu, a.pool,
                                                              nullptr, a.token_slots, a.num_accepted, a.pool, a.scale,
                                                              a.eps, a.out, nullptr, a.T, a.Nqk, a.Nv, a.Dv, a.win,
                                                              a.Bw);
}

// one activation type and pool type; a key gate only with a decaying rule.  A 16-bit pool stages 8
// tokens (the decode page's operator takes at most 8 per call, and 16 with the 64-column slice would not
// fit the static shared memory; longer sequences stay exact, their later tokens read directly)
template <int PRE, bool DECAY, bool DELTA, int DK, int ADT, int SDT>
static void launch_types(const RecArgs &a, dim3 grid, cudaStream_t st)
{
    constexpr int P = SDT != kF32 ? 8 : PRE;
    if (DECAY && a.gk) launch_pool<P, DECAY, SDT, DECAY, DELTA, DK, ADT>(a, grid, st);
    else launch_pool<P, false, SDT, DECAY, DELTA, DK, ADT>(a, grid, st);
}

// the type combinations: bf16 activations with an fp32 or bf16 pool (the decode page), fp16 or fp32
// activations with an fp16 or fp32 pool (the LinearAttention page; Dk = 128 only)
template <int PRE, bool DECAY, bool DELTA, int DK>
static void launch_rule(const RecArgs &a, int adt, int sdt, dim3 grid, cudaStream_t st)
{
    if (adt == kBF16) {
        if (sdt == kBF16) launch_types<PRE, DECAY, DELTA, DK, kBF16, kBF16>(a, grid, st);
        else launch_types<PRE, DECAY, DELTA, DK, kBF16, kF32>(a, grid, st);
    } else if constexpr (DK == 128) {
        if (adt == kF16) {
            if (sdt == kF16) launch_types<16, DECAY, DELTA, DK, kF16, kF16>(a, grid, st);
            else launch_types<16, DECAY, DELTA, DK, kF16, kF32>(a, grid, st);
        } else {
            if (sdt == kF16) launch_types<16, DECAY, DELTA, DK, kF32, kF16>(a, grid, st);
            else launch_types<16, DECAY, DELTA, DK, kF32, kF32>(a, grid, st);
        }
    }
}

template <int PRE, int DK>
static void launch_slots(const RecArgs &a, int rule, int adt, int sdt, dim3 grid, cudaStream_t st)
{
    switch (rule) {
    case kRuleDelta: launch_rule<PRE, false, true, DK>(a, adt, sdt, grid, st); break;
    case kRuleGated: launch_rule<PRE, true, false, DK>(a, adt, sdt, grid, st); break;
    case kRuleLinear: launch_rule<PRE, false, false, DK>(a, adt, sdt, grid, st); break;
    default: launch_rule<PRE, true, true, DK>(a, adt, sdt, grid, st);
    }
}

cudaError_t launch_short(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const uint16_t *beta, const int32_t *cu, const float *pool, const int32_t *idx, float scale,
                         float eps, uint16_t *out, float *final_state, int T, int B, int Nqk, int Nv, int max_seqlen,
                         cudaStream_t st, int rule)
{
    if (B == 0) return cudaSuccess;
    const dim3 grid(B, Nv, D / kTile);
    const bool few = max_seqlen >= 1 && max_seqlen <= 8;
    auto go = [&](auto pre, auto decay, auto delta) {
        launch_variant<decltype(pre)::value, false, false, kF32, decltype(decay)::value, decltype(delta)::value, D,
                       kBF16>(grid, st, q, k, v, g, beta, nullptr, cu, pool, idx, nullptr, nullptr, nullptr, scale, eps,
                              out, final_state, T, Nqk, Nv, D);
    };
    using P8 = std::integral_constant<int, 8>;
    using P16 = std::integral_constant<int, 16>;
    using Y = std::true_type;
    using N = std::false_type;
    switch (rule) {
    case kRuleDelta: few ? go(P8{}, N{}, Y{}) : go(P16{}, N{}, Y{}); break;
    case kRuleGated: few ? go(P8{}, Y{}, N{}) : go(P16{}, Y{}, N{}); break;
    case kRuleLinear: few ? go(P8{}, N{}, N{}) : go(P16{}, N{}, N{}); break;
    default: few ? go(P8{}, Y{}, Y{}) : go(P16{}, Y{}, Y{});
    }
    return cudaGetLastError();
}

// The window entries that a sequence of 1 <= n < W tokens keeps, moved n places towards entry 0 before
// the recurrence writes entries W - n .. W - 1: entry w <- entry w + n for w = 0 .. W - n - 1, in that
// order (each source is read before it is overwritten, and entry W - 1, the start of the recurrence, is
// not written here).  Grid (B, Nv, 16-byte pieces of a state / 256): each thread moves one 16-byte piece
// of the state through the entries.
__global__ void __launch_bounds__(256) window_shift_kernel(const int32_t *__restrict__ cu, uint4 *pool, int T, int B,
                                                           int Nv, int win, int pieces)
{
    const int b = blockIdx.x, h = blockIdx.y, i = blockIdx.z * 256 + threadIdx.x;
    const int t0 = min(max(cu[b], 0), T), n = min(max(cu[b + 1], t0), T) - t0;
    if (n < 1 || n >= win || i >= pieces) return;
    for (int w = 0; w + n < win; ++w)
        pool[(((size_t)w * B + b) * Nv + h) * pieces + i] = pool[(((size_t)(w + n) * B + b) * Nv + h) * pieces + i];
}

cudaError_t launch_recurrent(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                             const float *gk, const int32_t *cu, void *pool, int act_dtype, int state_dtype, int rule,
                             const int32_t *token_slots, const int32_t *num_accepted, float scale, float eps, void *out,
                             int T, int B, int Nqk, int Nv, int Dk, int Dv, int max_seqlen, cudaStream_t st, int win)
{
    if (B == 0) return cudaSuccess;
    if ((Dk != 64 && Dk != 128) || Dv <= 0 || Dv % kTile != 0) return cudaErrorInvalidValue;
    if (act_dtype != kBF16 && Dk != 128) return cudaErrorInvalidValue;
    if (win > 1) {
        const int pieces = Dk * Dv * (state_dtype == kF32 ? 4 : 2) / 16;
        window_shift_kernel<<<dim3(B, Nv, (pieces + 255) / 256), 256, 0, st>>>(cu, static_cast<uint4 *>(pool), T, B,
                                                                                Nv, win, pieces);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (max_seqlen == 1 && decode_supported(act_dtype, state_dtype, Dk, Dv, win))
        return launch_decode(q, k, v, g, beta, gk, cu, pool, state_dtype, rule, token_slots, num_accepted, scale, eps,
                             out, T, B, Nqk, Nv, Dk, Dv, st);
    const RecArgs a{q, k, v, g, beta, gk, cu, pool, token_slots, num_accepted, scale, eps, out, T, Nqk, Nv, Dv, win, B};
    const dim3 grid(B, Nv, Dv / kTile);
    const bool few = max_seqlen >= 1 && max_seqlen <= 8;
    if (Dk == 64) {
        if (few) launch_slots<8, 64>(a, rule, act_dtype, state_dtype, grid, st);
        else launch_slots<16, 64>(a, rule, act_dtype, state_dtype, grid, st);
    } else {
        if (few) launch_slots<8, 128>(a, rule, act_dtype, state_dtype, grid, st);
        else launch_slots<16, 128>(a, rule, act_dtype, state_dtype, grid, st);
    }
    return cudaGetLastError();
}

}  // namespace gdn
