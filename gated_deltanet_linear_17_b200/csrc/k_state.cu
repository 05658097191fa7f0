// Inter-chunk state passing on the Blackwell tensor core: one CTA per
// (sequence, v-head, 64-column slice of Dv), 8 epilogue warps, one warp that
// issues the tensor-core work and one that moves data with TMA.
//
// Page "Qwen3Next Samples", "Recurrent State Attention" and "State Update",
// with the state held as S[Dk, Dv]:
//   v'    = k_cumdecay S
//   S_new = S exp(g_last) + k_gexp^T (v_out - v'),  k_gexp = kh (.) exp(g_last - g_cum)
// regrouped as
//   S_new = e^{g_last} S + Kt - Mk S,   Kt = k_gexp^T U,  Mk = k_gexp^T W.
// Mk and the row factors f_t = rk_t e^{g_last - gamma_t} come from the
// intra-chunk kernel.  Kt is taken exactly as the raw 16-bit k rows times
// Ub = diag(f) U split into hi + lo halves of k's 16-bit type (about 16 significant
// bits with bf16, 22 with fp16).  Only
// Mk S depends on the state, so the serial chain over a sequence's chunks is
// one product per chunk; it accumulates -Mk S (the instruction negates A)
// onto the hi half of Kt, computed while the previous chunk's state update
// ran.  Warp w < 8 owns rows 32(w%4)..32(w%4)+31 and 32 columns (w/4) of the
// slice: each of its threads keeps 32 fp32 values of one row of S in registers
// for the whole sequence, and stages its row and columns of Ub.  Per chunk c
// (two stages, two TMEM accumulators of 128 columns, two fp16 copies of S):
//   issue warp: -Mk S_c onto Kt_c (tcgen05.mma M=128, N=64, K=128, fp16;
//               A = Mk K-major, B = S_c MN-major as the threads store it),
//               committed to an mbarrier; then, once the epilogue warps have
//               staged its operand, Kt of chunk c+1 = K^T [Ub_hi | Ub_lo]
//               (M=128, N=128, K=128, k's type; A = the raw k tile read MN-major)
//               into the other accumulator.
//   data warp:  a TMA store of S_c (fp16) to Sc; TMA loads of chunk c+2 into
//               the stage chunk c leaves: its raw k rows, U slice and factors
//               as soon as Kt of chunk c has completed (early in the chunk),
//               its Mk once the chain product of chunk c has.
//   epilogue:   stage Ub of chunk c+1 (hi over its U slice, lo beside it);
//               wait for the products of chunk c; S_{c+1} = e^{g_last} S_c +
//               D_hi + D_lo, whose fp16 copy is the next B operand (the other
//               buffer, so the TMA store of S_c can still be reading this one).
// One launch passes the chunks in a range [c_lo, c_hi): the forward pass runs
// the ranges one after another on a stream of its own (so that the other
// kernels of neighbouring ranges run beside it), and a sequence that crosses a
// range boundary carries its fp32 state through a workspace slot.  For an update
// rule without the retrieval (the LinearAttention page's gated and linear rules,
// `delta` = 0) the chain has no Mk S term: S_{c+1} = e^{g_last} S_c + Kt_c, and
// neither Mk nor its product is loaded or issued.
// The k rows of a chunk that ends before 128 tokens are zeroed after their TMA
// load, so the next sequence's rows never enter a product.  Every wait is
// bounded: if one gives up, the CTA sets bit 0 of status[2] in the workspace,
// stops, lets its copies and MMAs drain and frees its tensor memory.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"
#include "tc100.cuh"
#include "tma.cuh"

namespace gdn {

constexpr int kStateThreads = 320;  // 8 epilogue warps, the issue warp, the data warp
constexpr int DVT = 64;             // Dv columns per CTA

// shared memory, relative to a 1024-byte aligned base (bytes); 16-bit tiles
// with 128-byte rows use the 128-byte swizzle
constexpr int SG_MK = 0;       // fp16 Mk [Dk][Dk], K-major: two 64-column halves
constexpr int SG_K = 32768;    // bf16 k [L][Dk] in two 64-column blocks (MN-major A = k^T)
constexpr int SG_U = 65536;    // fp16 U slice [L][64] -> bf16 Ub_hi (MN-major B, first 64 columns)
constexpr int SG_UL = 81920;   // bf16 Ub_lo [L][64] (MN-major B, last 64 columns)
constexpr int kStage = 98304;  // a multiple of 1024
constexpr uint32_t kKUTx = 32768 + 16384 + kFaStride * 4;  // bytes of a stage's k / U / factor fill
constexpr int OFF_S = 2 * kStage;            // 2 x fp16 S [Dk][64] (MN-major B)
constexpr int OFF_F = OFF_S + 2 * 16384;     // 2 x fp32 factors: f_t (t < 128), e^{g_last} at 128
constexpr int OFF_BAR = OFF_F + 2 * kFaStride * 4;  // mbarriers; TMEM address slot
constexpr int kStateSmem = OFF_BAR + 96 + 1024;     // + alignment slack
constexpr int kTmemCols = 256;  // two accumulators [D_hi | D_lo], D_hi = Kt_hi - Mk S

// named barrier 1: the epilogue warps arrive once Ub is staged, the issue warp waits
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void named_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// bounded mbarrier wait by lane 0 of the warp, outcome shared with the warp
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane)
{
    bool w = true;
    if (lane == 0) w = tc::mbar_wait_bounded(bar, parity);
    return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
}

// F16: the raw k rows are fp16 (else bf16), and Ub's halves take the same type; SDT: the type of the
// pool and of the final state (kTypeF32, kTypeBF16 or kTypeF16; the carried state is always fp32)
template <bool F16, int SDT>
__global__ void __launch_bounds__(kStateThreads, 1) state_kernel(
    const __grid_constant__ CUtensorMap tm_mk, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_sc,
    const void *__restrict__ pool, const int32_t *__restrict__ idx, void *__restrict__ final_state, int Nqk,
    int Nv, const int4 *__restrict__ info, const int32_t *__restrict__ seq_chunk0, const float *__restrict__ fa,
    int32_t *__restrict__ status, int c_lo, int c_hi, int range, float *__restrict__ carry, int delta, int Dk, int Dv,
    int m)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int b = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * DVT;
    const int hq = h / (Nv / Nqk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const bool issuer = wid == 8, producer = wid == 9, epi = wid < 8;
    const int quarter = wid & 3, half = (wid >> 2) & 1;
    const int row = quarter * 32 + lane;  // row of the state (Dk) and of Ub (L)
    const int cbase = half * 32;          // first of this thread's 32 columns in the slice
    const int c_begin = seq_chunk0[b], c_end = seq_chunk0[b + 1];
    // This launch passes the sequence's chunks in [c_lo, c_hi).  A sequence that started in an
    // earlier range takes its state from carry slot range - 1, one that goes on past c_hi leaves it
    // in slot range (one slot per range boundary: at most one sequence crosses each).  A sequence
    // without chunks belongs to range 0.
    const bool empty_seq = c_begin >= c_end;
    if (empty_seq ? range != 0 : (c_end <= c_lo || c_begin >= c_hi)) return;
    const int lo = max(c_begin, c_lo), hi = min(c_end, c_hi);
    const bool from_carry = !empty_seq && c_begin < c_lo, to_carry = !empty_seq && c_end > c_hi;
    const int seq_t0 = c_begin < c_end ? info[c_begin].y : 0;
    const int seq_t1 = c_begin < c_end ? info[c_end - 1].y + info[c_end - 1].z : 0;
    auto chunk_len = [&](int c) { return min(L, seq_t1 - (seq_t0 + (c - c_begin) * L)); };

    // mbarriers (+ 8 s for stage s): ku (the stage's k rows, U slice and factors have landed), mk (its Mk
    // has landed), kt (the Kt product of the stage's chunk has completed); m (a chunk's chain product and
    // every product before it); d (drain on error)
    const uint32_t bar_ku = sbase + OFF_BAR, bar_mk = bar_ku + 16, bar_kt = bar_ku + 32;
    const uint32_t bar_m = bar_ku + 48, bar_d = bar_ku + 56;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 64);
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) tc::mbar_init(bar_ku + 8 * i, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), kTmemCols);
    __syncthreads();

    // TMA fills of stage st with chunk c (data lane): its k rows, U slice and factors; its Mk
    int fills_ku[2] = {0, 0}, fills_mk[2] = {0, 0};
    auto fill_ku = [&](int c, int st) {
        const uint32_t base = sbase + st * kStage, full = bar_ku + 8 * st;
        const int trow = (c * Nv + h) * L;  // first row of the chunk's tiles in the workspace
        const int cstart = seq_t0 + (c - c_begin) * L;
        tma::expect_tx(full, kKUTx);
        tma::load_3d(base + SG_K, &tm_k, 0, hq, cstart, full);  // columns past Dk (= 64) read as zero
        tma::load_3d(base + SG_K + 16384, &tm_k, 64, hq, cstart, full);
        tma::load_2d(base + SG_U, &tm_u, col0, trow, full);
        tma::load_1d(sbase + OFF_F + st * kFaStride * 4, fa + (size_t)(c * Nv + h) * kFaStride, kFaStride * 4,
                     full);
        ++fills_ku[st];
    };
    auto fill_mk = [&](int c, int st) {  // Mk enters only the rules with the retrieval
        const uint32_t base = sbase + st * kStage, full = bar_mk + 8 * st;
        const int trow = (c * Nv + h) * L;
        tma::expect_tx(full, 32768);
        tma::load_2d(base + SG_MK, &tm_mk, 0, trow, full);
        tma::load_2d(base + SG_MK + 16384, &tm_mk, 64, trow, full);
        ++fills_mk[st];
    };
    // After stage st has landed with chunk c (epilogue warps): zero the k rows
    // past a short chunk, and stage Ub = diag(f) U as bf16 hi (over U) and lo.
    // Returns e^{g_last} of the chunk.
    auto stage_ub = [&](int c, int st) {
        uint8_t *base = smem + st * kStage;
        const int clen = chunk_len(c);
        if (clen < L) {
            for (int e = tid; e < (L - clen) * 16; e += 256) {  // 2 blocks x 8 chunks per row
                const int r = clen + (e >> 4), blk = (e >> 3) & 1, cc = e & 7;
                *reinterpret_cast<uint4 *>(base + SG_K + blk * 16384 + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        const float *fr = reinterpret_cast<const float *>(smem + OFF_F + st * kFaStride * 4);
        const float f = fr[row];
        const float2 ff = make_float2(f, f);
        uint4 x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = *reinterpret_cast<const uint4 *>(base + SG_U + tc::sw128c(row, (cbase >> 3) + j));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t x4[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
            uint32_t h4[4], l4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // split2 in packed fp32 pairs (the same roundings)
                const float2 u = fmul2(unpack_h2(x4[e]), ff);
                h4[e] = pack2<F16>(u.x, u.y);
                const float2 r = fsub2(u, unpack2<F16>(h4[e]));
                l4[e] = pack2<F16>(r.x, r.y);
            }
            const uint32_t off = tc::sw128c(row, (cbase >> 3) + j);
            *reinterpret_cast<uint4 *>(base + SG_U + off) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            *reinterpret_cast<uint4 *>(base + SG_UL + off) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
        }
        return fr[128];
    };

    // initial state: this thread's 32 values
    // this thread's 32 values: in a carry slot [Nv sub-heads][128][128], and in a pool slot or a final
    // state [Nv / m v-heads][Dk][Dv] (sub-head h is columns 128 (h % m) .. of v-head h / m); state rows
    // past Dk stay zero and are neither read nor written
    float s[32];
    const size_t s_off = ((size_t)h * D + row) * D + col0 + cbase;
    const size_t p_off = ((size_t)(h / m) * Dk + row) * Dv + (size_t)(h % m) * D + col0 + cbase;
    const size_t p_slot = (size_t)(Nv / m) * Dk * Dv;  // elements of a pool slot
    const bool in_dk = row < Dk;
    if (epi && (from_carry || (pool && in_dk && SDT == kTypeF32))) {
        const float *src4 = from_carry ? carry + (size_t)(range - 1) * Nv * D * D + s_off
                                       : static_cast<const float *>(pool) + (size_t)(idx ? idx[b] : b) * p_slot + p_off;
        const float4 *src = reinterpret_cast<const float4 *>(src4);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v4 = src[j];
            s[4 * j] = v4.x;
            s[4 * j + 1] = v4.y;
            s[4 * j + 2] = v4.z;
            s[4 * j + 3] = v4.w;
        }
    } else if (epi && pool && in_dk) {  // a 16-bit pool, widened exactly
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(pool) +
                                                           (size_t)(idx ? idx[b] : b) * p_slot + p_off);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 w = src[j];
            const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 p = unpack2<SDT == kTypeF16>(w4[e]);
                s[8 * j + 2 * e] = p.x;
                s[8 * j + 2 * e + 1] = p.y;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = 0.f;
    }
    // S in fp16 as the MN-major B operand (buffer buf): row `row`, 16-byte chunks cbase/8 .. cbase/8 + 3
    auto store_state_operand = [&](int buf) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float *v8 = s + 8 * j;
            *reinterpret_cast<uint4 *>(smem + OFF_S + buf * 16384 + tc::sw128c(row, (cbase >> 3) + j)) =
                make_uint4(pack_h2(v8[0], v8[1]), pack_h2(v8[2], v8[3]), pack_h2(v8[4], v8[5]), pack_h2(v8[6], v8[7]));
        }
    };
    // vmax: the largest magnitude of the states converted to fp16 (range check), taken over each state
    // after its copy is stored, off the chain (at the start of the next chunk, and after the last)
    float vmax = 0.f;
    auto track_range = [&]() {
#pragma unroll
        for (int j = 0; j < 32; ++j) vmax = absmax_nan(vmax, s[j]);
    };

    bool ok = true;
    float dg = 1.f;  // e^{g_last} of the chunk in flight (epilogue warps)
    if (producer) {
        if (lane == 0) {
            tma::prefetch_map(&tm_mk);
            tma::prefetch_map(&tm_k);
            tma::prefetch_map(&tm_u);
            tma::prefetch_map(&tm_sc);
            for (int j = 0; j < 2 && lo + j < hi; ++j) {
                fill_ku(lo + j, j);
                if (delta) fill_mk(lo + j, j);
            }
        }
    } else if (epi) {
        store_state_operand(0);
        if (lo < hi) {
            ok = warp_wait(bar_ku, 0, lane);
            dg = stage_ub(lo, 0);
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();

    const uint32_t tmem = *tslot;
    const uint32_t t_mine = tmem + ((uint32_t)(quarter * 32) << 16) + cbase;
    const uint32_t idesc_kt = tc::idesc_f16(128, 128, !F16, !F16, true, true);
    const uint32_t idesc_mk = tc::idesc_f16(128, 64, false, false, false, true) | (1u << 13);  // A negated
    // Operand descriptors of k step 0; the start-address field holds (byte
    // address >> 4) and every address stays below 256 KiB, so the descriptor
    // of a k step is the base descriptor plus (byte offset >> 4).
    const uint64_t dMk0 = tc::desc_k128(sbase + SG_MK), dK0 = tc::desc_mn(sbase + SG_K, 16384, 1024, 2);
    const uint64_t dUb0 = tc::desc_mn(sbase + SG_U, 16384, 1024, 2), dS0 = tc::desc_mn(sbase + OFF_S, 0, 1024, 2);
    // Kt of the chunk in stage st into accumulator st (issue lane), tracked by kt[st]
    auto issue_kt = [&](int st) {
        const uint64_t so = (uint64_t)((st * kStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16(tmem + st * 128, dK0 + so + (uint64_t)((kk * 2048) >> 4),
                        dUb0 + so + (uint64_t)((kk * 2048) >> 4), idesc_kt, kk > 0 ? 1u : 0u);
        tc::commit(bar_kt + 8 * st);
    };
    bool issued = false;  // issue lane: any MMA in flight

    for (int c = lo, it = 0; ok && c < hi; ++c, ++it) {
        const int st = it & 1;  // stage, accumulator and S buffer of chunk c
        const bool has_next = c + 1 < hi;
        if (issuer) {
            bool w_ok = true;
            if (lane == 0) {
                if (it == 0) issue_kt(0);  // the first chunk's Kt, before its chain product
                const uint64_t so = (uint64_t)((st * kStage) >> 4), sb = (uint64_t)((st * 16384) >> 4);
                if (delta) {
                    w_ok = tc::mbar_wait_bounded(bar_mk + 8 * st, (uint32_t)((it >> 1) & 1));  // Mk of chunk c
                    tc::fence_after_sync();
                    if (w_ok) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_f16(tmem + st * 128,
                                        dMk0 + so + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                        dS0 + sb + (uint64_t)((kk * 2048) >> 4), idesc_mk, 1u);
                    }
                }
                tc::commit(bar_m);  // chunk c's products: Kt (issued before) and -Mk S
                issued = true;
            }
            ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0 && ok;
            if (has_next) {
                named_sync(1, 288);  // Ub of chunk c + 1 is staged
                if (lane == 0) issue_kt(st ^ 1);
                __syncwarp();
            }
        } else if (producer) {
            bool w_ok = true;
            if (lane == 0) {
                // the state entering chunk c, from its operand copy
                tma::store_2d(&tm_sc, col0, (c * Nv + h) * L, sbase + OFF_S + st * 16384);
                tma::commit_group();
                // stage st takes chunk c + 2: its k rows, U slice and factors once chunk c's Kt has read the
                // stage's (Kt was issued during the previous chunk), its Mk once chunk c's chain product has
                // read Mk
                if (c + 2 < hi) {
                    w_ok = tc::mbar_wait_bounded(bar_kt + 8 * st, (uint32_t)((it >> 1) & 1));
                    if (w_ok) fill_ku(c + 2, st);
                }
                const bool m_ok = tc::mbar_wait_bounded(bar_m, (uint32_t)(it & 1));
                w_ok = w_ok && m_ok;
                if (w_ok && delta && c + 2 < hi) fill_mk(c + 2, st);
                tma::wait_read_all();  // the store of S_c has read its buffer
            }
            ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0;
        } else {  // epilogue warps
            track_range();  // the state stored by the previous chunk (or the initial one), while loads land
            float dg_next = 1.f;
            if (has_next) {
                const bool f_ok = warp_wait(bar_ku + 8 * (st ^ 1), (uint32_t)(((it + 1) >> 1) & 1), lane);
                ok = ok && f_ok;
                dg_next = stage_ub(c + 1, st ^ 1);
                tc::fence_proxy_async();
                named_arrive(1, 288);
            }
            const bool m_ok = warp_wait(bar_m, (uint32_t)(it & 1), lane);
            tc::fence_after_sync();
            ok = ok && m_ok;
            float dh[32], dl[32];
            tc::tmem_ld32(t_mine + st * 128, dh);
            tc::tmem_ld32(t_mine + st * 128 + 64, dl);
            const float2 dg2 = make_float2(dg, dg);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {  // s = dg s + (dh + dl), in packed fp32 pairs
                const float2 r = ffma2(dg2, make_float2(s[j], s[j + 1]),
                                       fadd2(make_float2(dh[j], dh[j + 1]), make_float2(dl[j], dl[j + 1])));
                s[j] = r.x;
                s[j + 1] = r.y;
            }
            store_state_operand(st ^ 1);
            tc::fence_proxy_async();
            dg = dg_next;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(ok) != 0;
        tc::fence_after_sync();
    }

    // copies and MMAs still in flight land before shared and tensor memory are released
    if (producer && lane == 0) {
        for (int st = 0; st < 2; ++st) {
            if (fills_ku[st] > 0) tc::mbar_wait_bounded(bar_ku + 8 * st, (uint32_t)((fills_ku[st] - 1) & 1));
            if (fills_mk[st] > 0) tc::mbar_wait_bounded(bar_mk + 8 * st, (uint32_t)((fills_mk[st] - 1) & 1));
        }
        tma::wait_read_all();  // the stores have read shared memory (the grid's end publishes them)
    }
    if (issuer && lane == 0 && !ok && issued) {  // a commit covers every MMA issued before it
        tc::commit(bar_d);
        tc::mbar_wait_bounded(bar_d, 0);
    }
    if (epi) track_range();  // the last state stored (a repeat of the initial one when no chunk ran is harmless)
    if (epi && __any_sync(0xffffffffu, out_of_fp16(vmax)) && lane == 0) atomicOr(status + 3, GDN_DEV_RANGE_STATE);
    if (!ok) {
        if (tid == 0) atomicOr(status + 2, GDN_DEV_WAIT_STATE);
    } else if (epi && (to_carry || (final_state && in_dk && SDT == kTypeF32))) {
        float *dst4 = to_carry ? carry + (size_t)range * Nv * D * D + s_off
                               : static_cast<float *>(final_state) + (size_t)b * p_slot + p_off;
        float4 *dst = reinterpret_cast<float4 *>(dst4);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
    } else if (epi && final_state && in_dk) {  // a 16-bit final state, rounded to nearest even
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(final_state) + (size_t)b * p_slot + p_off);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float *v8 = s + 8 * j;
            dst[j] = make_uint4(pack2<SDT == kTypeF16>(v8[0], v8[1]), pack2<SDT == kTypeF16>(v8[2], v8[3]),
                                pack2<SDT == kTypeF16>(v8[4], v8[5]), pack2<SDT == kTypeF16>(v8[6], v8[7]));
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_state(const uint16_t *k, const void *pool, const int32_t *idx, void *final_state, int T, int B,
                         int Nqk, int Nv, int c_lo, int c_hi, int range, const Workspace &ws, cudaStream_t st,
                         bool delta, bool f16, int state_type, Dims dims)
{
    if (B == 0) return cudaSuccess;
    if (range < 0 || range >= kMaxRanges || c_lo < 0 || c_hi < c_lo) return cudaErrorInvalidValue;
    // tile rows of the workspace tensors; TMA coordinates are 32-bit signed
    const uint64_t trows = (uint64_t)ws.NC * Nv * L;
    if (trows >= (1ull << 31) || (uint64_t)T >= (1ull << 31)) return cudaErrorInvalidValue;
    const uint64_t rows = trows > 0 ? trows : 1;
    const auto HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16, BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap m_mk, m_k, m_u, m_sc;
    cudaError_t e = tma::map2d(&m_mk, HF, ws.Mk, D, rows, D * 2, 64, 128, SW);
    if (e == cudaSuccess) {
        if (T > 0)
            e = tma::map_heads(&m_k, f16 ? HF : BF, k, (uint64_t)dims.Dk, (uint64_t)Nqk, (uint64_t)T, 128);
        else  // no chunk exists, so the map is never used
            e = tma::map_heads(&m_k, BF, ws.Mk, D, 1, rows, 128);
    }
    if (e == cudaSuccess) e = tma::map2d(&m_u, HF, ws.U, D, rows, D * 2, DVT, 128, SW);
    if (e == cudaSuccess) e = tma::map2d(&m_sc, HF, ws.Sc, D, rows, D * 2, DVT, 128, SW);
    if (e != cudaSuccess) return e;
    auto kern = state_type == kTypeF16 ? (f16 ? state_kernel<true, kTypeF16> : state_kernel<false, kTypeF16>)
              : state_type == kTypeBF16 ? (f16 ? state_kernel<true, kTypeBF16> : state_kernel<false, kTypeBF16>)
                                        : (f16 ? state_kernel<true, kTypeF32> : state_kernel<false, kTypeF32>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(B, Nv, D / DVT), kStateThreads, kStateSmem, st>>>(
        m_mk, m_k, m_u, m_sc, pool, idx, final_state, Nqk, Nv, ws.chunk_info, ws.seq_chunk0, ws.fa, ws.status, c_lo,
        c_hi, range, ws.carry, delta ? 1 : 0, dims.Dk, dims.Dv, dims.m);
    return cudaGetLastError();
}

}  // namespace gdn
