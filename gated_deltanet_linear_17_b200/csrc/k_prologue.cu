// Chunk table and prologue kernels.
//
// chunk_map: one CTA turns cu_seqlens into the table of 128-token chunks
//   ("Qwen3Next Samples": chunk length L = 128, act_seq_len as cumulative
//   sequence lengths).
// prologue : per chunk, the L2 normalisation of q (times the query scale) and
//   of k ("L2 Normalization", eps inside the square root) as fp32 factors
//   rq = scale / sqrt(|q|^2 + eps), rk = 1 / sqrt(|k|^2 + eps), the chunk-local
//   cumulative gate ("Gate Cumulative Sum") and beta in fp32, all laid out
//   head-major ([head][token]) so that later kernels read one chunk of one head
//   as a contiguous run.  The factors are applied where q and k are consumed
//   (as fp32 row/column scalings around tensor-core products on the raw rows,
//   which convert exactly from bf16 to fp16), so no rounded normalised copy of
//   q or k is ever made.  Bound by HBM: it streams q and k once.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kMapThreads = 1024;

__global__ void __launch_bounds__(kMapThreads) chunk_map_kernel(const int32_t *__restrict__ cu, int B,
                                                                int T, int NC, int4 *__restrict__ info,
                                                                int32_t *__restrict__ seq_chunk0,
                                                                int32_t *__restrict__ status)
{
    __shared__ int warp_tot[kMapThreads / 32];
    __shared__ int err_bits;
    const int tid = threadIdx.x;
    if (tid == 0) err_bits = 0;
    __syncthreads();

    // each thread owns a contiguous range of sequences
    const int per = (B + kMapThreads - 1) / kMapThreads;
    const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
    int my = 0, err = 0;
    for (int b = b0; b < b1; ++b) {
        int s = cu[b], e = cu[b + 1];
        if (b == 0 && s != 0) err |= 1;
        if (e < s) err |= 2;
        if (b == B - 1 && e != T) err |= 4;
        s = min(max(s, 0), T);
        e = min(max(e, s), T);
        my += (e - s + L - 1) / L;
    }
    if (err) atomicOr(&err_bits, err);

    // block-wide exclusive scan of `my`
    const int lane = tid & 31, wid = tid >> 5;
    int incl = my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int base = (wid ? warp_tot[wid - 1] : 0) + incl - my;
    const int total = warp_tot[kMapThreads / 32 - 1];

    int c = base;
    for (int b = b0; b < b1; ++b) {
        int s = cu[b], e = cu[b + 1];
        s = min(max(s, 0), T);
        e = min(max(e, s), T);
        seq_chunk0[b] = min(c, NC);
        for (int t = s, j = 0; t < e; t += L, ++j, ++c)
            if (c < NC) info[c] = make_int4(b, t, min(L, e - t), j);
    }
    if (tid == 0) {
        seq_chunk0[B] = min(total, NC);
        status[0] = err_bits;
        status[1] = total;
    }
    for (int i = total + tid; i < NC; i += kMapThreads) info[i] = make_int4(-1, 0, 0, 0);
}

constexpr int kProThreads = 256;
constexpr int kHeadGroup = 32;  // v-heads per pass of the gate scan
constexpr int kProSplit = 4;    // CTAs per chunk: each normalises a quarter of the chunk's rows
constexpr int kRowsInFlight = 4; // rows each half-warp loads before reducing

__global__ void __launch_bounds__(kProThreads) prologue_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const float *__restrict__ g,
    const uint16_t *__restrict__ beta, float scale, float eps, int T, int Nqk, int Nv,
    const int4 *__restrict__ info, float *__restrict__ rq, float *__restrict__ rk,
    float *__restrict__ gcum, float *__restrict__ betaf)
{
    __shared__ float gs[L][kHeadGroup + 1];
    const ChunkInfo ci = load_chunk(info, blockIdx.x);
    if (ci.seq < 0) return;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int n = ci.len, t0 = ci.start;
    const int part = blockIdx.y;

    // ---- gates (first CTA of the chunk): chunk-local inclusive cumsum of g per v-head, beta to fp32
    for (int hg = 0; part == 0 && hg < Nv; hg += kHeadGroup) {
        const int nh = min(kHeadGroup, Nv - hg);
        for (int e = tid; e < L * kHeadGroup; e += kProThreads) {
            const int i = e / kHeadGroup, j = e % kHeadGroup;
            gs[i][j] = (i < n && j < nh) ? g[(size_t)(t0 + i) * Nv + hg + j] : 0.f;
        }
        __syncthreads();
        for (int j = wid; j < nh; j += kProThreads / 32) {
            // lane holds tokens 4*lane .. 4*lane+3
            float v0 = gs[4 * lane][j], v1 = gs[4 * lane + 1][j], v2 = gs[4 * lane + 2][j],
                  v3 = gs[4 * lane + 3][j];
            v1 += v0;
            v2 += v1;
            v3 += v2;
            float incl = v3;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float off = incl - v3;
            const float cs[4] = {v0 + off, v1 + off, v2 + off, v3 + off};
            float *dst = gcum + (size_t)(hg + j) * T + t0;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (4 * lane + u < n) dst[4 * lane + u] = cs[u];
        }
        __syncthreads();
    }
    for (int e = tid; part == 0 && e < n * Nv; e += kProThreads) {
        const int i = e / Nv, h = e % Nv;
        betaf[(size_t)h * T + t0 + i] = bf2f(beta[(size_t)(t0 + i) * Nv + h]);
    }

    // ---- L2 norms: a half-warp per 128-element row, 16 bytes per lane,
    //      kRowsInFlight rows loaded before any is reduced
    const int rows = n * Nqk;  // rows of q (and of k) in this chunk, contiguous in memory
    const int half = lane >> 4, hl = lane & 15;
    const int stride = kProSplit * (kProThreads / 32) * 2 * kRowsInFlight;
    for (int rbase = (part * (kProThreads / 32) + wid) * 2 * kRowsInFlight; rbase < 2 * rows; rbase += stride) {
        uint4 w[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int r = rbase + 2 * u + half;  // r < rows: q row, else k row
            const bool isk = r >= rows;
            const int rr = isk ? r - rows : r;
            w[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < 2 * rows)
                w[u] = __ldg(reinterpret_cast<const uint4 *>((isk ? k : q) + ((size_t)t0 * Nqk + rr) * D + hl * 8));
        }
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const int r = rbase + 2 * u + half;
            const bool isk = r >= rows;
            const int rr = isk ? r - rows : r;
            const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = __uint_as_float(ws[e] << 16), b = __uint_as_float(ws[e] & 0xffff0000u);
                ss += a * a + b * b;
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (r < 2 * rows && hl == 0) {
                const int i = rr / Nqk, hq = rr % Nqk;
                const float f = (isk ? 1.0f : scale) / sqrtf(ss + eps);
                (isk ? rk : rq)[(size_t)hq * T + t0 + i] = f;
            }
        }
    }
}

cudaError_t launch_chunk_map(const int32_t *cu, int B, int T, int NC, const Workspace &ws,
                             cudaStream_t st)
{
    chunk_map_kernel<<<1, kMapThreads, 0, st>>>(cu, B, T, NC, ws.chunk_info, ws.seq_chunk0, ws.status);
    return cudaGetLastError();
}

cudaError_t launch_prologue(const uint16_t *q, const uint16_t *k, const float *g, const uint16_t *beta,
                            float scale, float eps, int T, int Nqk, int Nv, int NC, const Workspace &ws,
                            cudaStream_t st)
{
    if (NC == 0) return cudaSuccess;
    prologue_kernel<<<dim3(NC, kProSplit), kProThreads, 0, st>>>(q, k, g, beta, scale, eps, T, Nqk, Nv, ws.chunk_info,
                                                ws.rq, ws.rk, ws.gcum, ws.betaf);
    return cudaGetLastError();
}

}  // namespace gdn
