// gdn_chunk_fwd_host: the forward pass from host buffers, with the host <-> device
// copies overlapped with the compute.
//
// The tokens are cut into segments at 128-token boundaries inside sequences (a
// cut never falls inside a chunk).  A sequence cut at such a boundary resumes
// from its fp32 state in the next segment, which the prefill page's "state
// reuse across sequence chunks" (streaming inference) and the decode page's
// state_out make exact: the chunks are the same chunks, and the state crosses
// the cut in fp32 as it crosses a chunk range inside one call.  So the result
// equals one gdn_chunk_fwd call over the whole batch bit for bit.
//
// Per segment s, on three streams: the H2D copies of its tokens (q, k, v, g,
// beta) on the library's upload stream; its gdn_chunk_fwd calls on the caller's
// stream once they have landed; the D2H copy of its output rows (and of the
// final states of the sequences that end in it) on the download stream once
// they are computed.  Segment s+1 uploads while s computes and s-1 downloads;
// the caller's stream joins the download stream before the call returns.
#include <algorithm>
#include <mutex>
#include <vector>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_stages.h"
#include "gdn_testing.h"

namespace {

constexpr int kD = 128, kL = 128;
constexpr int kMaxDev = 64;

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// cu of one call: dst[i] = clamp(cu[b0 + i], t0, t1) - t0 for i = 0 .. nb
__global__ void call_cu_kernel(const int32_t *__restrict__ cu, int b0, int nb, int t0, int t1, int32_t *__restrict__ dst)
{
    for (int i = threadIdx.x; i <= nb; i += blockDim.x) dst[i] = min(max(cu[b0 + i], t0), t1) - t0;
}

// the call's status words: those of one piece's workspace folded in (bits ORed, chunk counts added)
__global__ void status_fold_kernel(const int32_t *__restrict__ w, int32_t *__restrict__ acc)
{
    if (threadIdx.x == 0) {
        acc[0] |= w[0];
        acc[1] += w[1];
        acc[2] |= w[2];
        acc[3] |= w[3];
    }
}

struct Streams {
    cudaStream_t up = nullptr, down = nullptr;
    bool ready = false;
};
std::mutex g_lock;
Streams g_streams[kMaxDev];

cudaError_t copy_streams(Streams **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    Streams &s = g_streams[dev];
    if (!s.ready) {
        if ((e = cudaStreamCreateWithFlags(&s.up, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&s.down, cudaStreamNonBlocking)) != cudaSuccess) return e;
        s.ready = true;
    }
    *out = &s;
    return cudaSuccess;
}

// One gdn_chunk_fwd call of a segment: sequences b0 .. b0 + nb - 1 over tokens [t0, t1).
struct Call {
    int b0, nb, t0, t1;
    int src;  // initial states: 0 none, 1 the gathered pool slots (row b0 on), 2 the carry slot
    int dst;  // final states: 0 the final rows (b0 on), 1 the carry slot
};

struct Plan {
    std::vector<int> seg_t0;                 // first token of each segment (+ T at the end)
    std::vector<std::vector<Call>> calls;    // per segment
    std::vector<std::vector<int>> finished;  // per segment: sequences whose final state is complete there
    int64_t max_call_tokens = 0;
    int max_call_seqs = 0;
    size_t cu_slots = 0;  // int32 entries of all calls' cu arrays
};

// Cut [0, T) into about `segments` pieces.  A cut falls on a chunk start of the
// sequence it lies in, or on a sequence boundary.
Plan make_plan(const int32_t *cu, int64_t T, int B, int segments)
{
    Plan p;
    const int64_t target = std::max<int64_t>(kL, ((T + segments - 1) / segments + kL - 1) / kL * kL);
    std::vector<int64_t> cuts{0};
    int sb = 0;  // sequence that holds position `next`
    for (int64_t next = target; next < T;) {
        while (sb < B && cu[sb + 1] <= next) ++sb;  // cu[sb] <= next < cu[sb + 1]
        const int64_t s = cu[sb], e = cu[sb + 1];
        const int64_t c = std::min<int64_t>(e, s + (next - s + kL - 1) / kL * kL);
        if (c >= T) break;
        if (c > cuts.back()) cuts.push_back(c);
        next = std::max<int64_t>(c, cuts.back()) + target;
    }
    cuts.push_back(T);
    const int nseg = (int)cuts.size() - 1;
    int first = 0;  // first sequence that may overlap the current segment
    for (int si = 0; si < nseg; ++si) {
        const int64_t a = cuts[si], z = cuts[si + 1];
        const bool last = si + 1 == nseg;
        std::vector<Call> calls;
        std::vector<int> fin;
        while (first < B && cu[first + 1] <= a && !(cu[first] == cu[first + 1] && cu[first] >= a)) ++first;
        int b = first;
        for (; b < B; ++b) {
            const int64_t s = cu[b], e = cu[b + 1];
            const bool empty = s == e;
            if (empty ? !(s >= a && (s < z || last)) : !(s < z && e > a)) {
                if (s >= z) break;  // past the segment
                continue;
            }
            const int64_t t0 = std::max<int64_t>(s, a), t1 = std::min<int64_t>(e, z);
            const bool cont = t0 > s, cut = t1 < e;
            Call *run = calls.empty() ? nullptr : &calls.back();
            if (!cont && !cut && run && run->src == 1 && run->dst == 0 && run->b0 + run->nb == b) {
                run->nb += 1;  // joins the run of whole sequences before it
                run->t1 = (int)t1;
            } else {
                calls.push_back(Call{b, 1, (int)t0, (int)t1, cont ? 2 : 1, cut ? 1 : 0});
            }
            if (!cut) fin.push_back(b);
        }
        for (const Call &c : calls) {
            p.max_call_tokens = std::max<int64_t>(p.max_call_tokens, c.t1 - c.t0);
            p.max_call_seqs = std::max(p.max_call_seqs, c.nb);
            p.cu_slots += (size_t)c.nb + 1;
        }
        p.seg_t0.push_back((int)a);
        p.calls.push_back(calls);
        p.finished.push_back(fin);
    }
    p.seg_t0.push_back((int)T);
    return p;
}

struct Regions {
    size_t status, q, k, v, g, beta, cu, callcu, out, init, fin, carry, ws, ws_bytes, total;
};

Regions layout(int64_t T, int B, int Nqk, int Nv, bool pool, const Plan &p)
{
    Regions r{};
    size_t off = 0;
    auto take = [&](size_t n) { const size_t o = off; off = up256(off + n); return o; };
    const size_t sbytes = (size_t)Nv * kD * kD * 4;
    r.status = take(16);  // at offset 0: the call's four status words, read with gdn_read_status
    r.q = take((size_t)T * Nqk * kD * 2);
    r.k = take((size_t)T * Nqk * kD * 2);
    r.v = take((size_t)T * Nv * kD * 2);
    r.g = take((size_t)T * Nv * 4);
    r.beta = take((size_t)T * Nv * 2);
    r.cu = take((size_t)(B + 1) * 4);
    r.callcu = take(p.cu_slots * 4);
    r.out = take((size_t)T * Nv * kD * 2);
    r.init = take(pool ? (size_t)B * sbytes : 0);
    r.fin = take((size_t)B * sbytes);
    r.carry = take(2 * sbytes);
    r.ws_bytes = gdn_chunk_fwd_workspace_bytes(p.max_call_tokens, std::max(p.max_call_seqs, 1), Nqk, Nv);
    r.ws = take(r.ws_bytes);
    r.total = off;
    return r;
}

bool valid_cu(const int32_t *cu, int64_t T, int B)
{
    if (cu[0] != 0 || cu[B] != T) return false;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] < cu[b]) return false;
    return true;
}

int pick_segments(int64_t T, int segments)
{
    if (segments > 0) return segments;
    return T >= 8 * 4096 ? 8 : T >= 4096 ? 4 : 1;
}

}  // namespace

extern "C" int gdn_testing_host_plan(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t segments,
                                     int32_t *calls, int32_t max_calls)
{
    if (!cu_seqlens || !calls || T < 0 || B <= 0 || T >= (int64_t(1) << 31) || !valid_cu(cu_seqlens, T, B)) return -1;
    const Plan p = make_plan(cu_seqlens, T, B, pick_segments(T, segments));
    int n = 0;
    for (size_t s = 0; s < p.calls.size(); ++s)
        for (const Call &c : p.calls[s]) {
            if (n >= max_calls) return -1;
            int32_t *r = calls + 7 * n++;
            r[0] = (int32_t)s, r[1] = c.b0, r[2] = c.nb, r[3] = c.t0, r[4] = c.t1, r[5] = c.src, r[6] = c.dst;
        }
    return n;
}

extern "C" size_t gdn_chunk_fwd_host_bytes(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                                           int32_t with_pool, int32_t segments)
{
    if (!cu_seqlens || T < 0 || B <= 0 || Nqk <= 0 || Nv <= 0 || Nv % Nqk != 0) return 0;
    if (T >= (int64_t(1) << 31) || !valid_cu(cu_seqlens, T, B)) return 0;
    const Plan p = make_plan(cu_seqlens, T, B, pick_segments(T, segments));
    return layout(T, B, Nqk, Nv, with_pool != 0, p).total;
}

extern "C" int gdn_chunk_fwd_host(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                  const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                                  const int32_t *state_indices, float scale, float eps, uint16_t *out,
                                  float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                                  int32_t segments, void *device_buffer, size_t device_bytes, void *stream)
{
    if (T < 0 || B < 0 || Nqk <= 0 || Nv <= 0 || P < 0 || Nv % Nqk != 0) return GDN_ERR_BAD_SHAPE;
    if (T >= (int64_t(1) << 31) || Nqk > 64 || Nv > 256) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!cu_seqlens || !device_buffer) return GDN_ERR_NULL_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_NULL_ARG;
    if (!valid_cu(cu_seqlens, T, B)) return GDN_ERR_BAD_SHAPE;  // on the host the lengths are checked up front
    if (state_pool && P == 0) return GDN_ERR_BAD_SHAPE;
    if (state_pool && !state_indices && P < B) return GDN_ERR_BAD_SHAPE;
    if (state_pool && state_indices)
        for (int b = 0; b < B; ++b)
            if (state_indices[b] < 0 || state_indices[b] >= P) return GDN_ERR_BAD_SHAPE;
    if (reinterpret_cast<uintptr_t>(device_buffer) & 255u) return GDN_ERR_ALIGNMENT;
    const Plan p = make_plan(cu_seqlens, T, B, pick_segments(T, segments));
    const Regions r = layout(T, B, Nqk, Nv, state_pool != nullptr, p);
    if (device_bytes < r.total) return GDN_ERR_WORKSPACE;

    char *base = static_cast<char *>(device_buffer);
    auto dq = reinterpret_cast<uint16_t *>(base + r.q), dk = reinterpret_cast<uint16_t *>(base + r.k);
    auto dv = reinterpret_cast<uint16_t *>(base + r.v), db = reinterpret_cast<uint16_t *>(base + r.beta);
    auto dg = reinterpret_cast<float *>(base + r.g);
    auto dcu = reinterpret_cast<int32_t *>(base + r.cu), dcall = reinterpret_cast<int32_t *>(base + r.callcu);
    auto dout = reinterpret_cast<uint16_t *>(base + r.out);
    auto dinit = reinterpret_cast<float *>(base + r.init), dfin = reinterpret_cast<float *>(base + r.fin);
    auto dcarry = reinterpret_cast<float *>(base + r.carry);
    void *dws = base + r.ws;
    auto dstatus = reinterpret_cast<int32_t *>(base + r.status);
    gdn_workspace_layout_t wlay;
    gdn_workspace_layout(p.max_call_tokens, std::max(p.max_call_seqs, 1), Nqk, Nv, &wlay);
    const int32_t *ws_status = reinterpret_cast<const int32_t *>(static_cast<char *>(dws) + wlay.status);
    const size_t sfl = (size_t)Nv * kD * kD;  // floats per state

    const cudaStream_t st = (cudaStream_t)stream;
    std::lock_guard<std::mutex> guard(g_lock);
    Streams *ss = nullptr;
    cudaError_t e = copy_streams(&ss);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    const int S = (int)p.calls.size();
    std::vector<cudaEvent_t> ev(2 * S + 2, nullptr);
    for (auto &x : ev)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
    auto h2d = [&](void *dst, const void *src, size_t n, cudaStream_t s) {
        if (e == cudaSuccess && n) e = cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s);
    };
    auto d2h = [&](void *dst, const void *src, size_t n, cudaStream_t s) {
        if (e == cudaSuccess && n) e = cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s);
    };
    auto record = [&](cudaEvent_t x, cudaStream_t s) { if (e == cudaSuccess) e = cudaEventRecord(x, s); };
    auto wait = [&](cudaStream_t s, cudaEvent_t x) { if (e == cudaSuccess) e = cudaStreamWaitEvent(s, x, 0); };

    if ((e = cudaMemsetAsync(dstatus, 0, 16, st)) != cudaSuccess) return GDN_ERR_CUDA;
    // the copy streams start after the work the caller already enqueued on `stream`
    record(ev[2 * S], st);
    wait(ss->up, ev[2 * S]);
    wait(ss->down, ev[2 * S]);
    h2d(dcu, cu_seqlens, (size_t)(B + 1) * 4, ss->up);
    if (state_pool)  // the initial state of each sequence, gathered in sequence order
        for (int b = 0; b < B; ++b)
            h2d(dinit + (size_t)b * sfl, state_pool + (size_t)(state_indices ? state_indices[b] : b) * sfl, sfl * 4,
                ss->up);
    size_t cu_at = 0;
    int carry_in = 0;
    int rc = GDN_OK;
    for (int s = 0; s < S && e == cudaSuccess && rc == GDN_OK; ++s) {
        const size_t a = (size_t)p.seg_t0[s], z = (size_t)p.seg_t0[s + 1];
        h2d(dq + a * Nqk * kD, q + a * Nqk * kD, (z - a) * Nqk * kD * 2, ss->up);
        h2d(dk + a * Nqk * kD, k + a * Nqk * kD, (z - a) * Nqk * kD * 2, ss->up);
        h2d(dv + a * Nv * kD, v + a * Nv * kD, (z - a) * Nv * kD * 2, ss->up);
        h2d(dg + a * Nv, g + a * Nv, (z - a) * Nv * 4, ss->up);
        h2d(db + a * Nv, beta + a * Nv, (z - a) * Nv * 2, ss->up);
        record(ev[s], ss->up);
        wait(st, ev[s]);
        for (const auto &c : p.calls[s]) {
            if (e != cudaSuccess || rc != GDN_OK) break;
            int32_t *ccu = dcall + cu_at;
            cu_at += (size_t)c.nb + 1;
            call_cu_kernel<<<1, 256, 0, st>>>(dcu, c.b0, c.nb, c.t0, c.t1, ccu);
            if ((e = cudaGetLastError()) != cudaSuccess) break;
            const float *pool = c.src == 1 ? (state_pool ? dinit + (size_t)c.b0 * sfl : nullptr)
                              : c.src == 2 ? dcarry + (size_t)carry_in * sfl : nullptr;
            float *fin = c.dst == 1 ? dcarry + (size_t)(carry_in ^ 1) * sfl : dfin + (size_t)c.b0 * sfl;
            const size_t t0 = (size_t)c.t0;
            rc = gdn_chunk_fwd(dq + t0 * Nqk * kD, dk + t0 * Nqk * kD, dv + t0 * Nv * kD, dg + t0 * Nv,
                               db + t0 * Nv, ccu, pool, nullptr, scale, eps, dout + t0 * Nv * kD, fin, c.t1 - c.t0,
                               c.nb, Nqk, Nv, pool ? c.nb : 0, 0, dws, r.ws_bytes, stream);
            if (rc == GDN_OK) {  // this piece's status words, before the next piece clears them
                status_fold_kernel<<<1, 32, 0, st>>>(ws_status, dstatus);
                e = cudaGetLastError();
            }
            if (c.dst == 1) carry_in ^= 1;  // the next segment's first call resumes from this slot
        }
        record(ev[S + s], st);
        wait(ss->down, ev[S + s]);
        d2h(out + a * Nv * kD, dout + a * Nv * kD, (z - a) * Nv * kD * 2, ss->down);
        if (final_state)
            for (int b : p.finished[s]) d2h(final_state + (size_t)b * sfl, dfin + (size_t)b * sfl, sfl * 4, ss->down);
    }
    // join: nothing of this call runs outside `stream` after it returns
    record(ev[2 * S + 1], ss->down);
    cudaError_t j = cudaStreamWaitEvent(st, ev[2 * S + 1], 0);
    if (e == cudaSuccess) e = j;
    for (auto &x : ev)
        if (x) cudaEventDestroy(x);  // released once their recorded work completes
    if (rc != GDN_OK) return rc;
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
