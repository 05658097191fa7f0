// One-token decode on a state pool updated in place: gdn_recurrent_fwd with
// max_seqlen == 1 and bf16 activations (the decode page's operator in its
// commonest use, "lite_boost.ops.recurrent_gated_delta_rule": one token per
// sequence per call, bf16 activations, an fp32 or bf16 state pool).
//
// For one token the recurrence of the page's algorithm flow,
//   S' = D S  (D = diag(e^{g + gk_i}), or e^g, or 1);  kv = S'^T kh;
//   u = beta (v - kv);  S'' = S' + kh u^T;  o = S''^T qh,
// needs only two column sums of S' before the update, since
//   o = S'^T qh + u (kh . qh).
// So each state element is read once, used in both sums, and written once
// (S'' = D S + kh u^T): the kernel is a stream of the pool slices.  A
// persistent CTA (4 warps) walks (sequence, v-head, column slice) items: all Dk
// rows, 256 bytes of each (128 columns of a 16-bit pool, 64 of an fp32 one), so
// 32 KiB items at Dk = 128 (three CTAs per SM) and 16 KiB at Dk = 64 (six).  Half
// rows at Dk = 128 (16 KiB items, six CTAs per SM) measured 70 % of HBM on the
// one-token bf16 decode against 81 % for whole rows.  Each item's slots, gate and
// beta are read one item earlier still, so no dependent global load stands
// between an item and the copies of its slice.  While
// it computes one item from shared memory, the cp.async copies of the next
// item's state slice and token rows are in flight into the other of two
// buffers, so every SM keeps its loads going between items (a third buffer,
// with fewer CTAs per SM, measured slower).  Warp w owns rows
// w Dk/4 .. (w+1) Dk/4 - 1, lane l the columns of its 4 or 8 bytes of a row; the
// sums over rows go across the warps through shared memory.
//
// Slots as in gdn_recurrent_fwd: the sequence starts from the slot of its last
// accepted token and the state after each token goes to that token's slot.
// max_seqlen is a hint: a sequence with more tokens than one is still exact --
// its item then runs one column at a time with that column's state in fp32
// registers through all of its tokens, reading each token's rows directly
// (slow, and only reached when the hint is wrong).
#include <algorithm>

#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kDecodeThreads = 128;

template <int SDT>
__device__ __forceinline__ float2 load_pair(const uint8_t *p)  // the 4 bytes of a lane: 2 values or 1
{
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    if constexpr (SDT == kTypeF32) return make_float2(__uint_as_float(w), 0.f);
    else return unpack2<SDT == kTypeF16>(w);
}

template <int SDT>
__device__ __forceinline__ uint32_t store_bits(float a, float b)
{
    if constexpr (SDT == kTypeF32) return __float_as_uint(a);
    else return pack2<SDT == kTypeF16>(a, b);
}

}  // namespace

// Per-item values read from global memory one item ahead of their use, so that no dependent load
// (cu_seqlens, then the slots, then the gate) sits between an item's start and its slice copies
struct DecodeMeta {
    int b, h, z, t0, n, s0, ws;  // s0: starting slot; ws: the slot of the first token
    float gt, bt;                // the first token's gate and beta
};

constexpr int kDecodeBufs = 2;  // items in shared memory: the one computed and the next in flight

template <int DK, int SDT, bool GK, bool DECAY, bool DELTA>
__global__ void __launch_bounds__(kDecodeThreads, DK == 128 ? 3 : 6) decode_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
    const float *__restrict__ g, const uint16_t *__restrict__ beta, const float *__restrict__ gk,
    const int32_t *__restrict__ cu, void *pool, const int32_t *__restrict__ token_slots,
    const int32_t *__restrict__ num_accepted, float scale, float eps, uint16_t *__restrict__ out, int T, int B,
    int Nqk, int Nv, int Dv)
{
    constexpr int SE = SDT == kTypeF32 ? 4 : 2;  // bytes per state element
    constexpr int ROWB = 256;                    // bytes of an item's row: 32 KiB items at Dk = 128, 16 at 64
    constexpr int LB = ROWB / 32;                // bytes per lane in a row: 4 or 8
    constexpr int CPL = LB / SE;                 // columns per lane
    constexpr int CW = 32 * CPL;                 // columns per item
    constexpr int RW = DK / 4;                   // rows per warp
    constexpr int NB = kDecodeBufs;
    extern __shared__ __align__(16) uint8_t dyn_smem[];  // NB state slices of DK * ROWB bytes
    auto sbuf = [&](int bf) { return dyn_smem + bf * (DK * ROWB); };
    __shared__ __align__(16) uint16_t sq[NB][DK], sk[NB][DK], sv[NB][CW];
    __shared__ __align__(16) float sgk[NB][GK ? DK : 4];
    __shared__ __align__(16) float kh[DK], qh[DK], dd[DK];  // per row of the state: kh, qh, its decay
    __shared__ __align__(16) float red[4][32][2 * CPL];
    __shared__ float s_kq;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int nz = Dv / CW, G = Nv / Nqk;
    const int items = B * Nv * nz;
    uint8_t *const pool8 = static_cast<uint8_t *>(pool);
    auto meta_of = [&](int it) {
        DecodeMeta m{0, 0, 0, 0, 0, 0, 0, 0.f, 1.f};
        if (it < items) {
            m.z = it % nz;
            m.h = (it / nz) % Nv;
            m.b = it / (nz * Nv);
            m.t0 = min(max(cu[m.b], 0), T);
            m.n = min(max(cu[m.b + 1], m.t0), T) - m.t0;
            if (m.n > 0) {
                const int a = min(max(num_accepted ? num_accepted[m.b] : m.n, 1), m.n);
                m.s0 = token_slots[m.t0 + a - 1];
                m.ws = token_slots[m.t0];
                if (DECAY) m.gt = g[(size_t)m.t0 * Nv + m.h];
                if (DELTA) m.bt = bf2f(beta[(size_t)m.t0 * Nv + m.h]);
            }
        }
        return m;
    };
    // byte offset of row r of an item's columns in pool slot s
    auto slice_off = [&](const DecodeMeta &x, int s, int r) {
        return (((size_t)s * Nv + x.h) * DK + r) * (size_t)Dv * SE + (size_t)x.z * ROWB;
    };
    // cp.async copies of an item (its starting state slice and its first token's rows) into buffer bf
    auto stage = [&](const DecodeMeta &x, bool valid, int bf) {
        if (valid && x.n > 0) {
            for (int e = tid; e < DK * (ROWB / 16); e += kDecodeThreads) {
                const int r = e / (ROWB / 16), c = e % (ROWB / 16);
                cp_async16(smem_addr(sbuf(bf) + r * ROWB + c * 16), pool8 + slice_off(x, x.s0, r) + c * 16, true);
            }
            const size_t qo = ((size_t)x.t0 * Nqk + x.h / G) * DK;
            for (int e = tid; e < DK / 8; e += kDecodeThreads) {
                cp_async16(smem_addr(&sq[bf][e * 8]), q + qo + e * 8, true);
                cp_async16(smem_addr(&sk[bf][e * 8]), k + qo + e * 8, true);
            }
            if (tid < CW / 8)
                cp_async16(smem_addr(&sv[bf][tid * 8]), v + ((size_t)x.t0 * Nv + x.h) * Dv + x.z * CW + tid * 8, true);
            if (GK)
                for (int e = tid; e < DK / 4; e += kDecodeThreads)
                    cp_async16(smem_addr(&sgk[bf][e * 4]), gk + ((size_t)x.t0 * Nv + x.h) * DK + e * 4, true);
        }
        cp_async_commit();  // one group per item, possibly empty
    };
    // the normalised rows, k.q and the row decays (gate gt) from the 16-bit rows rq/rk (warp 0 for the rows,
    // threads < DK for the decays); the caller synchronises afterwards
    // (warp 0 for the rows and k.q, in one pass over the raw rows; threads < DK for the decays)
    auto token_prep = [&](float gt, const uint16_t *rq, const uint16_t *rk, const float *rgk) {
        if (wid == 0) {
            constexpr int EL = DK / 32;
            float qe[EL], ke[EL], sqq = 0.f, skk = 0.f, sqk = 0.f;
#pragma unroll
            for (int e = 0; e < EL; ++e) {
                qe[e] = bf2f(rq[lane * EL + e]);
                ke[e] = bf2f(rk[lane * EL + e]);
                sqq = fmaf(qe[e], qe[e], sqq);
                skk = fmaf(ke[e], ke[e], skk);
                sqk = fmaf(qe[e], ke[e], sqk);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sqq += __shfl_xor_sync(0xffffffffu, sqq, o);
                skk += __shfl_xor_sync(0xffffffffu, skk, o);
                sqk += __shfl_xor_sync(0xffffffffu, sqk, o);
            }
            const float rqn = scale / sqrtf(sqq + eps), rkn = 1.0f / sqrtf(skk + eps);
#pragma unroll
            for (int e = 0; e < EL; ++e) {
                qh[lane * EL + e] = qe[e] * rqn;
                kh[lane * EL + e] = ke[e] * rkn;
            }
            if (lane == 0) s_kq = sqk * rqn * rkn;
        }
        if (tid < DK) dd[tid] = DECAY ? __expf(GK ? gt + rgk[tid] : gt) : 1.f;
    };
    // this lane's CPL state values of row r of a slice
    auto row_vals = [&](const uint8_t *sb, int r, float (&x)[CPL]) {
        const uint8_t *p = sb + r * ROWB + lane * LB;
        if constexpr (SDT == kTypeF32) {
            if constexpr (CPL == 1) {
                x[0] = *reinterpret_cast<const float *>(p);
            } else {
                const float2 f = *reinterpret_cast<const float2 *>(p);
                x[0] = f.x;
                x[CPL - 1] = f.y;
            }
        } else {
            if constexpr (CPL == 2) {
                const float2 f = unpack2<SDT == kTypeF16>(*reinterpret_cast<const uint32_t *>(p));
                x[0] = f.x;
                x[CPL - 1] = f.y;
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(p);
                const float2 a = unpack2<SDT == kTypeF16>(w.x), b = unpack2<SDT == kTypeF16>(w.y);
                x[0] = a.x, x[1 % CPL] = a.y, x[2 % CPL] = b.x, x[3 % CPL] = b.y;
            }
        }
    };
    // this lane's CPL values of row r written to the pool (streaming stores of 4 or 8 bytes)
    auto row_store = [&](uint8_t *p, const float (&x)[CPL]) {
        if constexpr (SDT == kTypeF32) {
            if constexpr (CPL == 1) __stcs(reinterpret_cast<float *>(p), x[0]);
            else __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[CPL - 1]));
        } else {
            constexpr bool F = SDT == kTypeF16;
            if constexpr (CPL == 2) __stcs(reinterpret_cast<unsigned int *>(p), pack2<F>(x[0], x[CPL - 1]));
            else __stcs(reinterpret_cast<uint2 *>(p), make_uint2(pack2<F>(x[0], x[1 % CPL]), pack2<F>(x[2 % CPL], x[3 % CPL])));
        }
    };

    // items it, it + grid, it + 2 grid, ... of this CTA: the next one staged while one is computed, and the
    // values of the one after it read ahead into registers
    int it = blockIdx.x;
    const int gs = gridDim.x;
    DecodeMeta cur = meta_of(it), nxt = meta_of(it + gs);
    stage(cur, it < items, 0);
    for (int iter = 0; it < items; ++iter, it += gs) {
        const int bf = iter & 1;
        const DecodeMeta after = meta_of(it + 2 * gs);  // in flight while this item is computed
        const DecodeMeta x = cur;
        stage(nxt, it + gs < items, bf ^ 1);  // the next item's copies fly while this one is computed
        cur = nxt;
        nxt = after;
        cp_async_wait<1>();  // this item's copies
        __syncthreads();
        if (x.n == 0) continue;  // no token: the pool keeps its slots (CTA-uniform)
        token_prep(x.gt, sq[bf], sk[bf], sgk[bf]);
        __syncthreads();
        const float kq = s_kq;
        const uint8_t *sb = sbuf(bf);

        if (x.n == 1) {
            // sums over this warp's rows of S times d kh and d qh, for this lane's columns (factors of four
            // rows per 16-byte load, column pairs in packed fp32 arithmetic)
            float kv[CPL] = {}, qs[CPL] = {};
#pragma unroll 2
            for (int i = 0; i < RW; i += 4) {
                const int r0 = wid * RW + i;
                const float4 d4 = *reinterpret_cast<const float4 *>(dd + r0);
                const float4 a4 = *reinterpret_cast<const float4 *>(kh + r0);
                const float4 c4 = *reinterpret_cast<const float4 *>(qh + r0);
                const float av[4] = {d4.x * a4.x, d4.y * a4.y, d4.z * a4.z, d4.w * a4.w};
                const float cv[4] = {d4.x * c4.x, d4.y * c4.y, d4.z * c4.z, d4.w * c4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float sv_[CPL];
                    row_vals(sb, r0 + e, sv_);
                    if constexpr (CPL == 1) {
                        kv[0] = fmaf(sv_[0], av[e], kv[0]);
                        qs[0] = fmaf(sv_[0], cv[e], qs[0]);
                    } else {
#pragma unroll
                        for (int j = 0; j < CPL; j += 2) {
                            const float2 sp = make_float2(sv_[j], sv_[(j + 1) % CPL]);
                            const float2 kp = ffma2(sp, make_float2(av[e], av[e]), make_float2(kv[j], kv[(j + 1) % CPL]));
                            const float2 qp = ffma2(sp, make_float2(cv[e], cv[e]), make_float2(qs[j], qs[(j + 1) % CPL]));
                            kv[j] = kp.x, kv[(j + 1) % CPL] = kp.y, qs[j] = qp.x, qs[(j + 1) % CPL] = qp.y;
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                red[wid][lane][j] = kv[j];
                red[wid][lane][CPL + j] = qs[j];
            }
            __syncthreads();
            float u[CPL], o[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const float kvs = (red[0][lane][j] + red[1][lane][j]) + (red[2][lane][j] + red[3][lane][j]);
                const float qss = (red[0][lane][CPL + j] + red[1][lane][CPL + j]) +
                                  (red[2][lane][CPL + j] + red[3][lane][CPL + j]);
                const float vj = bf2f(sv[bf][lane * CPL + j]);
                u[j] = DELTA ? x.bt * (vj - kvs) : vj;
                o[j] = qss + u[j] * kq;
            }
            if (wid == 0) {
                uint16_t *op = out + ((size_t)x.t0 * Nv + x.h) * Dv + x.z * CW + lane * CPL;
#pragma unroll
                for (int j = 0; j < CPL; j += 2) {
                    if (j + 1 < CPL) *reinterpret_cast<uint32_t *>(op + j) = pack_bf2(o[j], o[(j + 1) % CPL]);
                    else op[j] = f2bf(o[j]);
                }
            }
            // S'' = D S + kh u^T into the token's slot
            uint8_t *dst = pool8 + slice_off(x, x.ws, wid * RW) + lane * LB;
            const size_t rstride = (size_t)Dv * SE;
#pragma unroll 2
            for (int i = 0; i < RW; i += 4) {
                const int r0 = wid * RW + i;
                const float4 d4 = *reinterpret_cast<const float4 *>(dd + r0);
                const float4 k4 = *reinterpret_cast<const float4 *>(kh + r0);
                const float dv[4] = {d4.x, d4.y, d4.z, d4.w}, kv4[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float sv_[CPL];
                    row_vals(sb, r0 + e, sv_);
                    if constexpr (CPL == 1) {
                        sv_[0] = fmaf(kv4[e], u[0], dv[e] * sv_[0]);
                    } else {
#pragma unroll
                        for (int j = 0; j < CPL; j += 2) {
                            const float2 n = ffma2(make_float2(kv4[e], kv4[e]), make_float2(u[j], u[(j + 1) % CPL]),
                                                   fmul2(make_float2(dv[e], dv[e]), make_float2(sv_[j], sv_[(j + 1) % CPL])));
                            sv_[j] = n.x, sv_[(j + 1) % CPL] = n.y;
                        }
                    }
                    row_store(dst + (size_t)(i + e) * rstride, sv_);
                }
            }
        } else {
            // more tokens than the hint: one column at a time, its state in fp32 registers through all tokens
#pragma unroll 1
            for (int j = 0; j < CPL; ++j) {
                float s[RW];
#pragma unroll
                for (int i = 0; i < RW; ++i) {
                    float p[CPL];
                    row_vals(sb, wid * RW + i, p);
                    s[i] = p[j];
                }
                const int col = x.z * CW + lane * CPL + j;
#pragma unroll 1
                for (int tj = 0; tj < x.n; ++tj) {
                    const int t = x.t0 + tj;
                    __syncthreads();  // the previous token's rows and sums have been read
                    if (tj > 0 || j > 0) {
                        const size_t qo = ((size_t)t * Nqk + x.h / G) * DK;
                        token_prep(DECAY ? g[(size_t)t * Nv + x.h] : 0.f, q + qo, k + qo,
                                   GK ? gk + ((size_t)t * Nv + x.h) * DK : nullptr);
                    }
                    __syncthreads();
                    float kv = 0.f, qs = 0.f;
#pragma unroll
                    for (int i = 0; i < RW; ++i) {
                        const int r = wid * RW + i;
                        s[i] *= dd[r];
                        kv = fmaf(s[i], kh[r], kv);
                        qs = fmaf(s[i], qh[r], qs);
                    }
                    red[wid][lane][0] = kv;
                    red[wid][lane][1] = qs;
                    __syncthreads();
                    const float kvs = (red[0][lane][0] + red[1][lane][0]) + (red[2][lane][0] + red[3][lane][0]);
                    const float qss = (red[0][lane][1] + red[1][lane][1]) + (red[2][lane][1] + red[3][lane][1]);
                    const float vj = bf2f(v[((size_t)t * Nv + x.h) * Dv + col]);
                    const float bt = DELTA ? bf2f(beta[(size_t)t * Nv + x.h]) : 1.f;
                    const float uj = DELTA ? bt * (vj - kvs) : vj;
                    if (wid == 0) out[((size_t)t * Nv + x.h) * Dv + col] = f2bf(qss + uj * s_kq);
#pragma unroll
                    for (int i = 0; i < RW; ++i) s[i] = fmaf(kh[wid * RW + i], uj, s[i]);
                    const int sj = token_slots[t], sn = tj + 1 < x.n ? token_slots[t + 1] : -1;
                    if (tj == x.n - 1 || sn != sj) {
#pragma unroll
                        for (int i = 0; i < RW; ++i) {
                            uint8_t *p = pool8 + slice_off(x, sj, wid * RW + i) + (size_t)(lane * CPL + j) * SE;
                            if constexpr (SDT == kTypeF32) *reinterpret_cast<float *>(p) = s[i];
                            else *reinterpret_cast<uint16_t *>(p) = (uint16_t)(pack2<SDT == kTypeF16>(s[i], 0.f) & 0xffffu);
                        }
                    }
                }
            }
        }
        __syncthreads();  // this item's buffer and rows are free again
    }
    cp_async_wait<0>();
}

namespace {

template <int DK, int SDT, bool GK, bool DECAY, bool DELTA>
cudaError_t launch_decode_variant(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                  const uint16_t *beta, const float *gk, const int32_t *cu, void *pool,
                                  const int32_t *token_slots, const int32_t *num_accepted, float scale, float eps,
                                  uint16_t *out, int T, int B, int Nqk, int Nv, int Dv, cudaStream_t st)
{
    auto kern = decode_kernel<DK, SDT, GK, DECAY, DELTA>;
    constexpr int dyn = kDecodeBufs * DK * 256;  // the state slices
    int per_sm = 0, dev = 0, sms = 0;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeThreads, dyn);
    if (e != cudaSuccess) return e;
    constexpr int CW = 256 / (SDT == kTypeF32 ? 4 : 2);  // columns per item
    const long long items = (long long)B * Nv * (Dv / CW);
    const long long grid = std::min<long long>(items, (long long)sms * std::max(per_sm, 1));
    if (grid <= 0) return cudaSuccess;
    kern<<<(unsigned)grid, kDecodeThreads, dyn, st>>>(q, k, v, g, beta, gk, cu, pool, token_slots, num_accepted, scale,
                                                   eps, out, T, B, Nqk, Nv, Dv);
    return cudaGetLastError();
}

template <int DK, int SDT>
cudaError_t launch_decode_rule(int rule, bool gk_on, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               const float *g, const uint16_t *beta, const float *gk, const int32_t *cu, void *pool,
                               const int32_t *slots, const int32_t *acc, float scale, float eps, uint16_t *out, int T,
                               int B, int Nqk, int Nv, int Dv, cudaStream_t st)
{
#define GDN_DECODE_ARGS q, k, v, g, beta, gk, cu, pool, slots, acc, scale, eps, out, T, B, Nqk, Nv, Dv, st
    switch (rule) {
    case kRuleDelta: return launch_decode_variant<DK, SDT, false, false, true>(GDN_DECODE_ARGS);
    case kRuleGated:
        return gk_on ? launch_decode_variant<DK, SDT, true, true, false>(GDN_DECODE_ARGS)
                     : launch_decode_variant<DK, SDT, false, true, false>(GDN_DECODE_ARGS);
    case kRuleLinear: return launch_decode_variant<DK, SDT, false, false, false>(GDN_DECODE_ARGS);
    default:
        return gk_on ? launch_decode_variant<DK, SDT, true, true, true>(GDN_DECODE_ARGS)
                     : launch_decode_variant<DK, SDT, false, true, true>(GDN_DECODE_ARGS);
    }
#undef GDN_DECODE_ARGS
}

}  // namespace

bool decode_supported(int act_dtype, int state_dtype, int Dk, int Dv, int win)
{
    // an item covers Dk rows of 256 bytes of a state
    const int cw = 256 / (state_dtype == kTypeF32 ? 4 : 2);
    return win == 0 && act_dtype == kTypeBF16 && (state_dtype == kTypeF32 || state_dtype == kTypeBF16) &&
           (Dk == 64 || Dk == 128) && Dv % cw == 0;
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                          const float *gk, const int32_t *cu, void *pool, int state_dtype, int rule,
                          const int32_t *token_slots, const int32_t *num_accepted, float scale, float eps, void *out,
                          int T, int B, int Nqk, int Nv, int Dk, int Dv, cudaStream_t st)
{
    const auto *q16 = static_cast<const uint16_t *>(q), *k16 = static_cast<const uint16_t *>(k),
               *v16 = static_cast<const uint16_t *>(v);
    auto *o16 = static_cast<uint16_t *>(out);
    const bool gk_on = gk != nullptr;
    if (Dk == 64)
        return state_dtype == kTypeF32
                   ? launch_decode_rule<64, kTypeF32>(rule, gk_on, q16, k16, v16, g, beta, gk, cu, pool, token_slots,
                                                      num_accepted, scale, eps, o16, T, B, Nqk, Nv, Dv, st)
                   : launch_decode_rule<64, kTypeBF16>(rule, gk_on, q16, k16, v16, g, beta, gk, cu, pool, token_slots,
                                                       num_accepted, scale, eps, o16, T, B, Nqk, Nv, Dv, st);
    return state_dtype == kTypeF32
               ? launch_decode_rule<128, kTypeF32>(rule, gk_on, q16, k16, v16, g, beta, gk, cu, pool, token_slots,
                                                   num_accepted, scale, eps, o16, T, B, Nqk, Nv, Dv, st)
               : launch_decode_rule<128, kTypeBF16>(rule, gk_on, q16, k16, v16, g, beta, gk, cu, pool, token_slots,
                                                    num_accepted, scale, eps, o16, T, B, Nqk, Nv, Dv, st);
}

}  // namespace gdn
