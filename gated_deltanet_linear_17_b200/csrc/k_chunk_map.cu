// Chunk table kernel: one CTA turns cu_seqlens into the table of 128-token
// chunks ("Qwen3Next Samples": chunk length L = 128, act_seq_len as cumulative
// sequence lengths), so that later grids are sized from an upper bound on the
// chunk count without a host round trip; rows past the last chunk hold -1 and
// their CTAs exit.
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

    // first chunk of every sequence, then the chunks themselves spread over the block: chunk c
    // belongs to the last sequence whose first chunk is <= c (binary search)
    {
        int c = base;
        for (int b = b0; b < b1; ++b) {
            int s = cu[b], e = cu[b + 1];
            s = min(max(s, 0), T);
            e = min(max(e, s), T);
            seq_chunk0[b] = min(c, NC);
            c += (e - s + L - 1) / L;
        }
    }
    if (tid == 0) seq_chunk0[B] = min(total, NC);
    __syncthreads();  // seq_chunk0 is complete (global writes of the block, ordered by the barrier)
    for (int c = tid; c < min(total, NC); c += kMapThreads) {
        int lo = 0, hi = B - 1;  // seq_chunk0[lo] <= c < seq_chunk0[hi + 1]
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seq_chunk0[mid] <= c) lo = mid;
            else hi = mid - 1;
        }
        const int s = min(max(cu[lo], 0), T), e = min(max(cu[lo + 1], s), T);
        const int j = c - seq_chunk0[lo], t = s + j * L;
        info[c] = make_int4(lo, t, min(L, e - t), j);
    }
    if (tid == 0) {
        // this kernel runs first in every chunked call, on the caller's stream: the wait and
        // range bits of an earlier call on this workspace are cleared before any kernel can set them
        status[0] = err_bits;
        status[1] = total;
        status[2] = 0;
        status[3] = 0;
    }
    for (int i = total + tid; i < NC; i += kMapThreads) info[i] = make_int4(-1, 0, 0, 0);
}

cudaError_t launch_chunk_map(const int32_t *cu, int B, int T, int NC, const Workspace &ws,
                             cudaStream_t st)
{
    chunk_map_kernel<<<1, kMapThreads, 0, st>>>(cu, B, T, NC, ws.chunk_info, ws.seq_chunk0, ws.status);
    return cudaGetLastError();
}

}  // namespace gdn
