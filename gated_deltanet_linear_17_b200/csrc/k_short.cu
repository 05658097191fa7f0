// Fused short-sequence forward: one CTA per (sequence, v-head, 32-column slice of Dv).
//
// The decode page ("lite_boost.ops.recurrent_gated_delta_rule", algorithm
// flow) runs the Gated Delta Rule token by token for a few tokens per call,
// reading and writing a slot of a state pool.  For such batches the work is
// moving the states: 64 KiB of fp32 state per (sequence, v-head) in and out,
// against a few hundred bytes of q/k/v per token.  This kernel reads the
// state slice once into registers (warp w holds Dk rows 32w..32w+31, lane j
// holds column j), applies every token of the sequence,
//   S = e^g S;  kv = S^T kh;  S += kh (beta (v - kv))^T;  o = S^T qh,
// and writes the final slice once.  Cross-warp sums over Dk go through shared
// memory.  It is exact for any sequence length; it is only fast for short ones.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kShortThreads = 128;

__global__ void __launch_bounds__(kShortThreads) short_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
    const float *__restrict__ g, const uint16_t *__restrict__ beta, const int32_t *__restrict__ cu,
    const float *__restrict__ pool, const int32_t *__restrict__ idx, float scale, float eps,
    uint16_t *__restrict__ out, float *__restrict__ final_state, int T, int Nqk, int Nv)
{
    __shared__ float qs[D], ks[D], red[4][32], red2[4][32], nrm[2][4];
    const int b = blockIdx.x, h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int col = blockIdx.z * 32 + lane;
    const int hq = h / (Nv / Nqk);

    float s[32];
    if (pool) {
        const int slot = idx ? idx[b] : b;
        const float *src = pool + (((size_t)slot * Nv + h) * D + wid * 32) * D + col;
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = src[(size_t)i * D];
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = 0.f;
    }

    int t_begin = cu[b], t_end = cu[b + 1];
    t_begin = min(max(t_begin, 0), T);
    t_end = min(max(t_end, t_begin), T);
    for (int t = t_begin; t < t_end; ++t) {
        const float qv = bf2f(q[((size_t)t * Nqk + hq) * D + tid]);
        const float kv = bf2f(k[((size_t)t * Nqk + hq) * D + tid]);
        const float vj = bf2f(v[((size_t)t * Nv + h) * D + col]);
        const float gt = g[(size_t)t * Nv + h];
        const float bt = bf2f(beta[(size_t)t * Nv + h]);
        const float sq = warp_sum(qv * qv), sk = warp_sum(kv * kv);
        if (lane == 0) {
            nrm[0][wid] = sq;
            nrm[1][wid] = sk;
        }
        __syncthreads();
        const float rqs = scale / sqrtf(nrm[0][0] + nrm[0][1] + nrm[0][2] + nrm[0][3] + eps);
        const float rks = 1.0f / sqrtf(nrm[1][0] + nrm[1][1] + nrm[1][2] + nrm[1][3] + eps);
        qs[tid] = qv * rqs;
        ks[tid] = kv * rks;
        __syncthreads();

        const float dg = __expf(gt);
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            s[i] *= dg;
            acc += s[i] * ks[wid * 32 + i];
        }
        red[wid][lane] = acc;
        __syncthreads();
        const float u = bt * (vj - (red[0][lane] + red[1][lane] + red[2][lane] + red[3][lane]));
        float acc2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            s[i] += ks[wid * 32 + i] * u;
            acc2 += s[i] * qs[wid * 32 + i];
        }
        red2[wid][lane] = acc2;
        __syncthreads();
        if (wid == 0)
            out[((size_t)t * Nv + h) * D + col] = f2bf(red2[0][lane] + red2[1][lane] + red2[2][lane] + red2[3][lane]);
    }

    if (final_state) {
        float *dst = final_state + (((size_t)b * Nv + h) * D + wid * 32) * D + col;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[(size_t)i * D] = s[i];
    }
}

cudaError_t launch_short(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const uint16_t *beta, const int32_t *cu, const float *pool, const int32_t *idx,
                         float scale, float eps, uint16_t *out, float *final_state, int T, int B, int Nqk,
                         int Nv, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    short_kernel<<<dim3(B, Nv, D / 32), kShortThreads, 0, st>>>(q, k, v, g, beta, cu, pool, idx, scale, eps,
                                                                 out, final_state, T, Nqk, Nv);
    return cudaGetLastError();
}

}  // namespace gdn
