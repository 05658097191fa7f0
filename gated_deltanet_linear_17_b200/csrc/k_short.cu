// Fused short-sequence forward: one CTA per (sequence, v-head, 32-column slice of Dv).
//
// The decode page ("lite_boost.ops.recurrent_gated_delta_rule", algorithm
// flow) runs the Gated Delta Rule token by token for a few tokens per call,
// reading and writing a slot of a state pool.  For such batches the work is
// moving the states: 64 KiB of fp32 state per (sequence, v-head) in and out,
// against a few hundred bytes of q/k/v per token, so the kernel is a stream:
// each CTA issues the loads of its state slice (warp w holds Dk rows
// 32w..32w+31, lane j holds column j, one 128-byte row segment per warp load)
// together with cp.async copies of the token data of up to kPre tokens (q and
// k rows, the v slice, g), so that a single memory latency covers both; it then
// applies the tokens from registers and shared memory,
//   S = e^g S;  kv = S^T kh;  S += kh (beta (v - kv))^T;  o = S^T qh,
// with q and k normalised as in "L2 Normalization" and the cross-warp sums over
// Dk going through shared memory, and writes the final slice from registers.
// Tokens past kPre are read directly from global memory, so the kernel is exact
// for any sequence length; it is only fast for short ones.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kShortThreads = 128;
constexpr int kTile = 32;  // Dv columns per CTA
constexpr int kPre = 16;   // tokens staged together with the state

struct ShortSmem {
    uint16_t q[kPre][D], k[kPre][D];  // raw bf16 rows
    uint16_t v[kPre][kTile];          // raw bf16 slice
    float g[kPre], beta[kPre], rq[kPre], rk[kPre];
    float red[4][32], red2[4][32];
};

__global__ void __launch_bounds__(kShortThreads) short_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
    const float *__restrict__ g, const uint16_t *__restrict__ beta, const int32_t *__restrict__ cu,
    const float *__restrict__ pool, const int32_t *__restrict__ idx, float scale, float eps,
    uint16_t *__restrict__ out, float *__restrict__ final_state, int T, int Nqk, int Nv)
{
    __shared__ __align__(16) ShortSmem sm;
    const int b = blockIdx.x, h = blockIdx.y, tl = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = tl * kTile + lane;
    const int hq = h / (Nv / Nqk);
    const int t0 = min(max(cu[b], 0), T);
    const int t1 = min(max(cu[b + 1], t0), T);
    const int n = t1 - t0, npre = min(n, kPre);

    // token data of the first kPre tokens: async copies
    for (int e = tid; e < npre * 16; e += kShortThreads) {
        const int t = e >> 4, c = e & 15;
        const size_t off = ((size_t)(t0 + t) * Nqk + hq) * D + c * 8;
        cp_async16(smem_addr(&sm.q[t][c * 8]), q + off, true);
        cp_async16(smem_addr(&sm.k[t][c * 8]), k + off, true);
    }
    for (int e = tid; e < npre * 4; e += kShortThreads) {
        const int t = e >> 2, c = e & 3;
        cp_async16(smem_addr(&sm.v[t][c * 8]), v + ((size_t)(t0 + t) * Nv + h) * D + tl * kTile + c * 8, true);
    }
    if (tid < npre) cp_async4(smem_addr(&sm.g[tid]), g + (size_t)(t0 + tid) * Nv + h);
    cp_async_commit();
    float bt_mine = 0.f;
    if (tid < npre) bt_mine = bf2f(beta[(size_t)(t0 + tid) * Nv + h]);

    // the state slice, straight into registers
    float s[32];
    if (pool) {
        const int slot = idx ? idx[b] : b;
        const float *src = pool + (((size_t)slot * Nv + h) * D + wid * 32) * D + col;
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = __ldcs(src + (size_t)i * D);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = 0.f;
    }

    cp_async_wait<0>();
    if (tid < npre) sm.beta[tid] = bt_mine;
    __syncthreads();
    // norms of the staged q and k rows: one warp per token
    for (int t = wid; t < npre; t += kShortThreads / 32) {
        const uint2 qa = *reinterpret_cast<const uint2 *>(&sm.q[t][lane * 4]);
        const uint2 ka = *reinterpret_cast<const uint2 *>(&sm.k[t][lane * 4]);
        const uint32_t qw[2] = {qa.x, qa.y}, kw[2] = {ka.x, ka.y};
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xffff0000u);
            const float k0 = __uint_as_float(kw[e] << 16), k1 = __uint_as_float(kw[e] & 0xffff0000u);
            sq += q0 * q0 + q1 * q1;
            sk += k0 * k0 + k1 * k1;
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        if (lane == 0) {
            sm.rq[t] = scale / sqrtf(sq + eps);
            sm.rk[t] = 1.0f / sqrtf(sk + eps);
        }
    }

    for (int j = 0; j < n; ++j) {
        // this warp's 32 rows of the token's k and q (raw bf16) and the token's scalars
        const uint16_t *kr, *qr;
        float vj, gt, bt, rks, rqs;
        if (j < kPre) {
            __syncthreads();  // norms (first token) / previous token's reductions are complete
            kr = &sm.k[j][wid * 32];
            qr = &sm.q[j][wid * 32];
            vj = bf2f(sm.v[j][lane]);
            gt = sm.g[j];
            bt = sm.beta[j];
            rks = sm.rk[j];
            rqs = sm.rq[j];
        } else {  // beyond the staged tokens: read directly
            const int t = t0 + j;
            const uint16_t *qrow = q + ((size_t)t * Nqk + hq) * D, *krow = k + ((size_t)t * Nqk + hq) * D;
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = bf2f(qrow[lane + 32 * i]), c = bf2f(krow[lane + 32 * i]);
                sq += a * a;
                sk += c * c;
            }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            rqs = scale / sqrtf(sq + eps);
            rks = 1.0f / sqrtf(sk + eps);
            kr = krow + wid * 32;
            qr = qrow + wid * 32;
            vj = bf2f(v[((size_t)t * Nv + h) * D + col]);
            gt = g[(size_t)t * Nv + h];
            bt = bf2f(beta[(size_t)t * Nv + h]);
            __syncthreads();  // previous token's reductions are complete
        }
        const float dg = __expf(gt);
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            s[i] *= dg;
            acc += s[i] * bf2f(kr[i]);
        }
        sm.red[wid][lane] = acc;
        __syncthreads();
        const float u = bt * (vj - rks * (sm.red[0][lane] + sm.red[1][lane] + sm.red[2][lane] + sm.red[3][lane]));
        const float ku = u * rks;
        float acc2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            s[i] += bf2f(kr[i]) * ku;
            acc2 += s[i] * bf2f(qr[i]);
        }
        sm.red2[wid][lane] = acc2;
        __syncthreads();
        if (wid == 0)
            out[((size_t)(t0 + j) * Nv + h) * D + col] =
                f2bf(rqs * (sm.red2[0][lane] + sm.red2[1][lane] + sm.red2[2][lane] + sm.red2[3][lane]));
    }

    if (final_state) {
        float *dst = final_state + (((size_t)b * Nv + h) * D + wid * 32) * D + col;
#pragma unroll
        for (int i = 0; i < 32; ++i) __stcs(dst + (size_t)i * D, s[i]);
    }
}

cudaError_t launch_short(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const uint16_t *beta, const int32_t *cu, const float *pool, const int32_t *idx,
                         float scale, float eps, uint16_t *out, float *final_state, int T, int B, int Nqk,
                         int Nv, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    short_kernel<<<dim3(B, Nv, D / kTile), kShortThreads, 0, st>>>(q, k, v, g, beta, cu, pool, idx, scale, eps, out,
                                                                    final_state, T, Nqk, Nv);
    return cudaGetLastError();
}

}  // namespace gdn
