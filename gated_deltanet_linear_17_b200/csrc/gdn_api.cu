// Host side of the C ABI (include/gdn.h, include/gdn_stages.h): argument
// checks, workspace layout and the launch sequence.  The chunked forward pass
// splits the chunks into ranges and runs them as a pipeline: the intra-chunk
// kernel on a low-priority stream, the state pass on a high-priority stream
// (range r after the intra-chunk kernel of range r and the state pass of range
// r - 1) and the output kernel on the caller's stream (range r after the state
// pass of range r), so the state pass, which keeps only part of the GPU busy,
// runs beside the other two kernels of neighbouring ranges.  The side streams
// fork from and join back into the caller's stream within the call.
#include <math.h>
#include <algorithm>
#include <string.h>

#include <atomic>
#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_stages.h"

using gdn::Workspace;

namespace {

constexpr int kVersion = 200;  // 0.2.0

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The pipeline's side streams and events, per device, created on first use and kept
// until the process exits; g_pipe_lock serialises their use (a call's record / wait
// pairs must not interleave with another host thread's).
constexpr int kMaxPipeDevices = 64;
struct SideStreams {
    cudaStream_t intra = nullptr, state = nullptr;
    cudaEvent_t ev[2 * gdn::kMaxRanges + 3] = {};
    bool ready = false;
};
std::mutex g_pipe_lock;
SideStreams g_side[kMaxPipeDevices];

cudaError_t side_streams(SideStreams **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxPipeDevices) return cudaErrorInvalidDevice;
    SideStreams &s = g_side[dev];
    if (!s.ready) {
        int least = 0, greatest = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&s.intra, cudaStreamNonBlocking, least)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&s.state, cudaStreamNonBlocking, greatest)) != cudaSuccess) return e;
        for (auto &x : s.ev)
            if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) return e;
        s.ready = true;
    }
    *out = &s;
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t max_chunks(int64_t T, int32_t B) { return (T + 127 * (int64_t)B) / gdn::L; }

// act_dtype: the activations' type; fp32 activations add the act16 region (their fp16 copies, q and k
// rows of Dk elements); Nv counts 128-column sub-heads (Nv Dv / 128 for a value dimension Dv)
int fill_layout(int64_t T, int32_t B, int32_t Nqk, int32_t Nv, gdn_workspace_layout_t *lay,
                int32_t act_dtype = GDN_DTYPE_BF16, int32_t Dk = gdn::D)
{
    if (T < 0 || B < 0 || Nqk <= 0 || Nv <= 0) return GDN_ERR_BAD_SHAPE;
    const int64_t NC = max_chunks(T, B);
    const size_t tile = (size_t)gdn::L * gdn::D * 2;
    size_t off = 0;
    lay->status = off;
    off = align256(off + 16);
    lay->chunk_info = off;
    off = align256(off + (size_t)NC * 16);
    lay->seq_chunk0 = off;
    off = align256(off + (size_t)(B + 1) * 4);
    lay->rq = off;
    off = align256(off + (size_t)Nqk * T * 4);
    lay->rk = off;
    off = align256(off + (size_t)Nqk * T * 4);
    lay->gcum = off;
    off = align256(off + (size_t)Nv * T * 4);
    lay->betaf = off;
    off = align256(off + (size_t)Nv * T * 4);
    lay->U = off;
    off += (size_t)NC * Nv * tile;
    lay->W = off;
    off += (size_t)NC * Nv * tile;
    lay->Mk = off;
    off += (size_t)NC * Nv * tile;
    lay->Sc = off;
    off += (size_t)NC * Nv * tile;
    lay->fa = off;
    off += (size_t)NC * Nv * gdn::kFaStride * 4;
    off = align256(off);
    lay->carry = off;
    off += (size_t)(gdn::pipeline_ranges(NC) - 1) * Nv * gdn::D * gdn::D * 4;
    off = align256(off);
    lay->act16 = off;
    if (act_dtype == GDN_DTYPE_FP32) off += ((size_t)2 * Nqk * Dk + (size_t)Nv * gdn::D) * T * 2;
    lay->total = align256(off);
    lay->max_chunks = NC;
    return GDN_OK;
}

Workspace views(void *base, const gdn_workspace_layout_t &lay)
{
    char *p = static_cast<char *>(base);
    Workspace w;
    w.status = reinterpret_cast<int32_t *>(p + lay.status);
    w.chunk_info = reinterpret_cast<int4 *>(p + lay.chunk_info);
    w.seq_chunk0 = reinterpret_cast<int32_t *>(p + lay.seq_chunk0);
    w.rq = reinterpret_cast<float *>(p + lay.rq);
    w.rk = reinterpret_cast<float *>(p + lay.rk);
    w.gcum = reinterpret_cast<float *>(p + lay.gcum);
    w.betaf = reinterpret_cast<float *>(p + lay.betaf);
    w.U = reinterpret_cast<uint16_t *>(p + lay.U);
    w.W = reinterpret_cast<uint16_t *>(p + lay.W);
    w.Mk = reinterpret_cast<uint16_t *>(p + lay.Mk);
    w.Sc = reinterpret_cast<uint16_t *>(p + lay.Sc);
    w.fa = reinterpret_cast<float *>(p + lay.fa);
    w.carry = reinterpret_cast<float *>(p + lay.carry);
    w.act16 = lay.total > lay.act16 ? reinterpret_cast<uint16_t *>(p + lay.act16) : nullptr;
    w.NC = static_cast<int>(lay.max_chunks);
    return w;
}

// sizes shared by every entry point
int check_sizes(int64_t T, int32_t B, int32_t Nqk, int32_t Nv)
{
    if (T < 0 || B < 0 || Nqk <= 0 || Nv <= 0) return GDN_ERR_BAD_SHAPE;
    if (Nv % Nqk != 0) return GDN_ERR_BAD_SHAPE;
    if (T >= (int64_t(1) << 31) || Nqk > 64 || Nv > 256) return GDN_ERR_UNSUPPORTED;
    if (max_chunks(T, B) >= (int64_t(1) << 31) / 256) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

int check_workspace(void *ws, size_t bytes, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                    gdn_workspace_layout_t *lay)
{
    int rc = fill_layout(T, B, Nqk, Nv, lay);
    if (rc) return rc;
    if (!ws) return GDN_ERR_NULL_ARG;
    if (!aligned16(ws)) return GDN_ERR_ALIGNMENT;
    if (bytes < lay->total) return GDN_ERR_WORKSPACE;
    return GDN_OK;
}

bool overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const char *x = static_cast<const char *>(a), *y = static_cast<const char *>(b);
    return a && b && na && nb && x < y + nb && y < x + na;
}

float resolve_scale(float scale) { return scale > 0.f ? scale : 1.0f / sqrtf((float)gdn::D); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

// arguments of the whole forward (shared by gdn_chunk_fwd and gdn_short_fwd); ae / se: bytes per
// activation / state element; Dk, Dv: head dimensions
int check_forward(const void *q, const void *k, const void *v, const float *g,
                  const uint16_t *beta, const int32_t *cu, const void *pool, const int32_t *idx,
                  const void *out, const void *final_state, int64_t T, int32_t B, int32_t Nqk,
                  int32_t Nv, int32_t P, bool need_g = true, bool need_beta = true, size_t ae = 2, size_t se = 4,
                  int32_t Dk = gdn::D, int32_t Dv = gdn::D)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    if (P < 0) return GDN_ERR_BAD_SHAPE;
    if (B == 0) return GDN_OK;
    if (!cu) return GDN_ERR_NULL_ARG;
    if (T > 0 && (!q || !k || !v || (need_g && !g) || (need_beta && !beta) || !out)) return GDN_ERR_NULL_ARG;
    if (pool && P == 0) return GDN_ERR_BAD_SHAPE;
    if (pool && !idx && P < B) return GDN_ERR_BAD_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(pool) ||
        !aligned16(final_state))
        return GDN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(g) & 3u) || (reinterpret_cast<uintptr_t>(beta) & 1u) ||
        (reinterpret_cast<uintptr_t>(cu) & 3u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return GDN_ERR_ALIGNMENT;
    const size_t sbytes = (size_t)Dk * Dv * se * Nv;
    if (overlap(final_state, sbytes * B, pool, sbytes * P)) return GDN_ERR_OVERLAP;
    const size_t obytes = (size_t)T * Nv * Dv * ae;
    if (overlap(out, obytes, q, (size_t)T * Nqk * Dk * ae) ||
        overlap(out, obytes, k, (size_t)T * Nqk * Dk * ae) || overlap(out, obytes, v, obytes))
        return GDN_ERR_OVERLAP;
    return GDN_OK;
}

}  // namespace

namespace {
std::atomic<int> g_value_checks{0};  // the process-wide switch of gdn_set_value_checks
}  // namespace

extern "C" {

const char *gdn_status_string(int status)
{
    switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_NULL_ARG: return "GDN_ERR_NULL_ARG: a required pointer is NULL";
    case GDN_ERR_BAD_SHAPE: return "GDN_ERR_BAD_SHAPE: invalid sizes";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: sizes beyond the supported limits";
    case GDN_ERR_ALIGNMENT: return "GDN_ERR_ALIGNMENT: pointer not aligned";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace too small";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA call failed";
    case GDN_ERR_OVERLAP: return "GDN_ERR_OVERLAP: an output overlaps an input";
    case GDN_ERR_SCRATCH_LIMIT:
        return "GDN_ERR_SCRATCH_LIMIT: these sizes need more workspace than the library's static scratch";
    default: return "GDN_ERR_UNKNOWN";
    }
}

int gdn_version(void) { return kVersion; }

int gdn_check_values(const float *g, const uint16_t *beta, const int32_t *state_indices, int64_t T, int32_t B,
                     int32_t Nv, int32_t P, int32_t *status_word, void *stream)
{
    if (!status_word) return GDN_ERR_NULL_ARG;
    if (T < 0 || B < 0 || Nv <= 0 || P < 0) return GDN_ERR_BAD_SHAPE;
    if (T * (int64_t)Nv >= (int64_t(1) << 40)) return GDN_ERR_UNSUPPORTED;
    const auto al = [](const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
    if (!al(g, 4) || !al(status_word, 4) || !al(beta, 2) || !al(state_indices, 4)) return GDN_ERR_ALIGNMENT;
    return cuda_status(gdn::launch_check_values(g, beta, state_indices, T, Nv, B, P, status_word,
                                                (cudaStream_t)stream));
}

int gdn_set_value_checks(int on) { return g_value_checks.exchange(on ? 1 : 0); }

int gdn_read_status(const void *workspace, int32_t *status_out, void *stream)
{
    if (!workspace || !status_out) return GDN_ERR_NULL_ARG;
    if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(status_out) & 3u)) return GDN_ERR_ALIGNMENT;
    return cuda_status(cudaMemcpyAsync(status_out, workspace, 4 * sizeof(int32_t), cudaMemcpyDefault,
                                       (cudaStream_t)stream));
}

int gdn_workspace_layout(int64_t T, int32_t B, int32_t Nqk, int32_t Nv, gdn_workspace_layout_t *layout)
{
    if (!layout) return GDN_ERR_NULL_ARG;
    return fill_layout(T, B, Nqk, Nv, layout);
}

size_t gdn_chunk_fwd_workspace_bytes(int64_t T, int32_t B, int32_t Nqk, int32_t Nv)
{
    gdn_workspace_layout_t lay;
    if (fill_layout(T, B, Nqk, Nv, &lay)) return 0;
    return lay.total;
}

int gdn_stage_chunk_map(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    gdn_workspace_layout_t lay;
    if ((rc = check_workspace(workspace, workspace_bytes, T, B, Nqk, Nv, &lay))) return rc;
    if (B == 0) return GDN_OK;
    if (!cu_seqlens) return GDN_ERR_NULL_ARG;
    const Workspace w = views(workspace, lay);
    return cuda_status(gdn::launch_chunk_map(cu_seqlens, B, (int)T, w.NC, w, (cudaStream_t)stream));
}

int gdn_stage_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps, int64_t T,
                    int32_t B, int32_t Nqk, int32_t Nv, void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    gdn_workspace_layout_t lay;
    if ((rc = check_workspace(workspace, workspace_bytes, T, B, Nqk, Nv, &lay))) return rc;
    if (B == 0 || T == 0) return GDN_OK;
    if (!k || !v || !g || !beta) return GDN_ERR_NULL_ARG;
    if (!aligned16(k) || !aligned16(v)) return GDN_ERR_ALIGNMENT;
    const Workspace w = views(workspace, lay);
    return cuda_status(gdn::launch_intra(k, v, g, beta, eps, (int)T, Nqk, Nv, 0, w.NC, w, (cudaStream_t)stream));
}

int gdn_stage_state(const uint16_t *k, const float *state_pool, const int32_t *state_indices, float *final_state,
                    int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P, void *workspace,
                    size_t workspace_bytes, void *stream)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    if (P < 0) return GDN_ERR_BAD_SHAPE;
    gdn_workspace_layout_t lay;
    if ((rc = check_workspace(workspace, workspace_bytes, T, B, Nqk, Nv, &lay))) return rc;
    if (B == 0) return GDN_OK;
    if (T > 0 && !k) return GDN_ERR_NULL_ARG;
    if (state_pool && P == 0) return GDN_ERR_BAD_SHAPE;
    if (state_pool && !state_indices && P < B) return GDN_ERR_BAD_SHAPE;
    if (!aligned16(k) || !aligned16(state_pool) || !aligned16(final_state)) return GDN_ERR_ALIGNMENT;
    const size_t sbytes = (size_t)gdn::D * gdn::D * 4 * Nv;
    if (overlap(final_state, sbytes * B, state_pool, sbytes * P)) return GDN_ERR_OVERLAP;
    const Workspace w = views(workspace, lay);
    return cuda_status(gdn::launch_state(k, state_pool, state_indices, final_state, (int)T, B, Nqk, Nv, 0, w.NC, 0, w,
                                         (cudaStream_t)stream));
}

int gdn_stage_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, uint16_t *out,
                     int64_t T, int32_t B, int32_t Nqk, int32_t Nv, void *workspace, size_t workspace_bytes,
                     void *stream)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    gdn_workspace_layout_t lay;
    if ((rc = check_workspace(workspace, workspace_bytes, T, B, Nqk, Nv, &lay))) return rc;
    if (B == 0 || T == 0) return GDN_OK;
    if (!q || !k || !g || !out) return GDN_ERR_NULL_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(out)) return GDN_ERR_ALIGNMENT;
    const Workspace w = views(workspace, lay);
    return cuda_status(gdn::launch_output(q, k, g, resolve_scale(scale), eps, out, (int)T, Nqk, Nv, 0, w.NC, w,
                                          (cudaStream_t)stream));
}

int gdn_short_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                  const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                  const int32_t *state_indices, float scale, float eps, uint16_t *out,
                  float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                  void *stream)
{
    int rc = check_forward(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, out, final_state, T, B,
                           Nqk, Nv, P);
    if (rc || B == 0) return rc;
    return cuda_status(gdn::launch_short(q, k, v, g, beta, cu_seqlens, state_pool, state_indices,
                                         resolve_scale(scale), eps, out, final_state, (int)T, B, Nqk, Nv, 0,
                                         (cudaStream_t)stream));
}

}  // extern "C"

namespace {

// Checks and launch shared by gdn_recurrent_fwd (win = 0: a pool of P slots, one slot per token) and
// gdn_recurrent_window_fwd (win >= 1: a window buffer of win * B slots, P = win * B, no token slots).
int recurrent_call(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                   const float *gk, const int32_t *cu_seqlens, void *state_pool, int32_t act_dtype,
                   int32_t state_dtype, int32_t update_rule, const int32_t *token_slots, const int32_t *num_accepted,
                   float scale, float eps, void *out, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t Dk,
                   int32_t Dv, int64_t P, int32_t max_seqlen, void *stream, int win)
{
    int rc = check_sizes(T, B, Nqk, Nv);
    if (rc) return rc;
    if (update_rule < GDN_RULE_GATED_DELTA || update_rule > GDN_RULE_LINEAR) return GDN_ERR_BAD_SHAPE;
    if (P <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_BAD_SHAPE;
    const auto known = [](int32_t d) { return d == GDN_DTYPE_FP32 || d == GDN_DTYPE_BF16 || d == GDN_DTYPE_FP16; };
    if (!known(act_dtype) || !known(state_dtype)) return GDN_ERR_BAD_SHAPE;
    // bf16 activations take an fp32 or bf16 pool; fp16 / fp32 activations an fp16 or fp32 pool at Dk = 128
    const bool types_ok = act_dtype == GDN_DTYPE_BF16 ? state_dtype != GDN_DTYPE_FP16
                                                      : state_dtype != GDN_DTYPE_BF16 && Dk == 128;
    const bool pool16 = state_dtype != GDN_DTYPE_FP32;
    if (!types_ok || (Dk != 64 && Dk != 128) || Dv % 32 != 0 || Dv > 1024 || (pool16 && Dv % 64 != 0))
        return GDN_ERR_UNSUPPORTED;
    if (win > 0 && (int64_t)win * B >= (int64_t(1) << 31) / 256) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    const bool decay = update_rule == GDN_RULE_GATED_DELTA || update_rule == GDN_RULE_GATED;
    const bool delta = update_rule == GDN_RULE_GATED_DELTA || update_rule == GDN_RULE_DELTA;
    if (!decay) g = nullptr, gk = nullptr;  // not read by this rule
    if (!delta) beta = nullptr;
    if (win > 0) token_slots = nullptr, num_accepted = nullptr;  // the window decides the slots
    if (!cu_seqlens || !state_pool) return GDN_ERR_NULL_ARG;
    if (T > 0 && (!q || !k || !v || !out || (win == 0 && !token_slots) || (decay && !g) || (delta && !beta)))
        return GDN_ERR_NULL_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state_pool) ||
        !aligned16(gk))
        return GDN_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(g) & 3u) || (reinterpret_cast<uintptr_t>(beta) & 1u) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(token_slots) & 3u) ||
        (reinterpret_cast<uintptr_t>(num_accepted) & 3u))
        return GDN_ERR_ALIGNMENT;
    const size_t ae = act_dtype == GDN_DTYPE_FP32 ? 4 : 2;
    const size_t obytes = (size_t)T * Nv * Dv * ae, qbytes = (size_t)T * Nqk * Dk * ae;
    const size_t pbytes = (size_t)Dk * Dv * (pool16 ? 2 : 4) * Nv * P;
    if (overlap(out, obytes, q, qbytes) || overlap(out, obytes, k, qbytes) || overlap(out, obytes, v, obytes) ||
        overlap(out, obytes, state_pool, pbytes) || overlap(out, obytes, gk, (size_t)T * Nv * Dk * 4))
        return GDN_ERR_OVERLAP;
    if (T == 0) return GDN_OK;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)Dk);
    return cuda_status(gdn::launch_recurrent(q, k, v, g, beta, gk, cu_seqlens, state_pool, act_dtype, state_dtype,
                                             update_rule, token_slots, num_accepted, sc, eps, out, (int)T, B, Nqk, Nv,
                                             Dk, Dv, max_seqlen, (cudaStream_t)stream, win));
}

}  // namespace

extern "C" {

int gdn_recurrent_fwd(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                      const float *gk, const int32_t *cu_seqlens, void *state_pool, int32_t act_dtype,
                      int32_t state_dtype, int32_t update_rule, const int32_t *token_slots,
                      const int32_t *num_accepted, float scale, float eps, void *out, int64_t T, int32_t B,
                      int32_t Nqk, int32_t Nv, int32_t Dk, int32_t Dv, int32_t P, int32_t max_seqlen, void *stream)
{
    return recurrent_call(q, k, v, g, beta, gk, cu_seqlens, state_pool, act_dtype, state_dtype, update_rule,
                          token_slots, num_accepted, scale, eps, out, T, B, Nqk, Nv, Dk, Dv, P, max_seqlen, stream, 0);
}

int gdn_recurrent_window_fwd(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                             const float *gk, const int32_t *cu_seqlens, void *state_window, int32_t window,
                             int32_t act_dtype, int32_t state_dtype, int32_t update_rule, float scale, float eps,
                             void *out, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t Dk, int32_t Dv,
                             int32_t max_seqlen, void *stream)
{
    if (window < 0 || window > GDN_MAX_STATE_WINDOW) return GDN_ERR_BAD_SHAPE;
    const int W = window > 0 ? window : 1;  // no window axis: the current state alone, one entry
    return recurrent_call(q, k, v, g, beta, gk, cu_seqlens, state_window, act_dtype, state_dtype, update_rule,
                          nullptr, nullptr, scale, eps, out, T, B, Nqk, Nv, Dk, Dv, std::max<int64_t>((int64_t)W * B, 1),
                          max_seqlen, stream, W);
}

int gdn_chunk_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                  const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                  const int32_t *state_indices, float scale, float eps, uint16_t *out,
                  float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                  int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream)
{
    return gdn_chunk_fwd_rule(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, scale, eps, out, final_state,
                              T, B, Nqk, Nv, P, GDN_RULE_GATED_DELTA, max_seqlen, workspace, workspace_bytes, stream);
}

int gdn_chunk_fwd_rule(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                       const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                       const int32_t *state_indices, float scale, float eps, uint16_t *out,
                       float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                       int32_t update_rule, int32_t max_seqlen, void *workspace, size_t workspace_bytes,
                       void *stream)
{
    return gdn_chunk_fwd_typed(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, scale, eps, out, final_state,
                               T, B, Nqk, Nv, P, update_rule, GDN_DTYPE_BF16, GDN_DTYPE_FP32, GDN_HEAD_DIM, GDN_HEAD_DIM,
                               max_seqlen, workspace, workspace_bytes, stream);
}

size_t gdn_chunk_fwd_typed_workspace_bytes(int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t act_dtype, int32_t Dk,
                                           int32_t Dv)
{
    if ((Dk != 64 && Dk != 128) || Dv <= 0 || Dv % 128 != 0 || Dv > 512 || Nv <= 0) return 0;
    gdn_workspace_layout_t lay;
    if (fill_layout(T, B, Nqk, Nv * (Dv / 128), &lay, act_dtype, Dk)) return 0;
    return lay.total;
}

int gdn_chunk_fwd_typed(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                        const int32_t *cu_seqlens, const void *state_pool, const int32_t *state_indices, float scale,
                        float eps, void *out, void *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                        int32_t P, int32_t update_rule, int32_t act_dtype, int32_t state_dtype, int32_t Dk, int32_t Dv,
                        int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream)
{
    if (update_rule < GDN_RULE_GATED_DELTA || update_rule > GDN_RULE_LINEAR) return GDN_ERR_BAD_SHAPE;
    const auto known = [](int32_t d) { return d == GDN_DTYPE_FP32 || d == GDN_DTYPE_BF16 || d == GDN_DTYPE_FP16; };
    if (!known(act_dtype) || !known(state_dtype)) return GDN_ERR_BAD_SHAPE;
    if (Dk <= 0 || Dv <= 0) return GDN_ERR_BAD_SHAPE;
    if ((Dk != 64 && Dk != 128) || Dv % 128 != 0 || Dv > 512) return GDN_ERR_UNSUPPORTED;
    gdn::Dims dims;
    dims.Dk = Dk, dims.Dv = Dv, dims.m = Dv / 128;
    if (Nv > 0 && (int64_t)Nv * dims.m > 256) return GDN_ERR_UNSUPPORTED;
    const bool decay = update_rule == GDN_RULE_GATED_DELTA || update_rule == GDN_RULE_GATED;
    const bool delta = update_rule == GDN_RULE_GATED_DELTA || update_rule == GDN_RULE_DELTA;
    if (!decay) g = nullptr;  // a zero gate
    if (!delta) beta = nullptr;
    const size_t ae = act_dtype == GDN_DTYPE_FP32 ? 4 : 2, se = state_dtype == GDN_DTYPE_FP32 ? 4 : 2;
    int rc = check_forward(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, out, final_state, T, B, Nqk, Nv,
                           P, decay, delta, ae, se, Dk, Dv);
    if (rc || B == 0) return rc;
    const cudaStream_t st = (cudaStream_t)stream;
    const float sc = resolve_scale(scale > 0.f ? scale : 1.0f / sqrtf((float)Dk));
    // the fused short-sequence kernel takes bf16 activations, an fp32 state and 128 x 128 heads; other
    // types and sizes take the chunked kernels whatever the lengths
    const bool short_ok = act_dtype == GDN_DTYPE_BF16 && state_dtype == GDN_DTYPE_FP32 && Dk == gdn::D &&
                          Dv == gdn::D;
    if (short_ok && max_seqlen >= 1 && max_seqlen <= GDN_SHORT_MAX)
        return cuda_status(gdn::launch_short(static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k),
                                             static_cast<const uint16_t *>(v), g, beta, cu_seqlens,
                                             static_cast<const float *>(state_pool), state_indices, sc, eps,
                                             static_cast<uint16_t *>(out), static_cast<float *>(final_state), (int)T,
                                             B, Nqk, Nv, max_seqlen, st, update_rule));

    const int32_t Nvs = Nv * dims.m;  // the kernels' head count: 128-column sub-heads
    gdn_workspace_layout_t lay;
    if ((rc = fill_layout(T, B, Nqk, Nvs, &lay, act_dtype, Dk))) return rc;
    bool owned = false;
    if (!workspace) {
        if (cudaMallocAsync(&workspace, lay.total, st) != cudaSuccess) return GDN_ERR_CUDA;
        owned = true;
    } else {
        if (!aligned16(workspace)) return GDN_ERR_ALIGNMENT;
        if (workspace_bytes < lay.total) return GDN_ERR_WORKSPACE;
    }
    const Workspace w = views(workspace, lay);
    const int Ti = (int)T, NC = w.NC;
    const bool f16 = act_dtype != GDN_DTYPE_BF16;  // fp16 rows (fp32 activations: their fp16 copies)
    const int sdt = state_dtype, odt = act_dtype;
    const uint16_t *q16 = static_cast<const uint16_t *>(q), *k16 = static_cast<const uint16_t *>(k),
                   *v16 = static_cast<const uint16_t *>(v);
    cudaError_t e = gdn::launch_chunk_map(cu_seqlens, B, Ti, NC, w, st);
    if (e == cudaSuccess && g_value_checks.load(std::memory_order_relaxed))  // into word 0, after the table clears it
        e = gdn::launch_check_values(g, beta, state_pool ? state_indices : nullptr, T, Nv, B, P, w.status, st);
    if (e == cudaSuccess && act_dtype == GDN_DTYPE_FP32 && T > 0) {
        uint16_t *aq = w.act16, *ak = aq + (size_t)T * Nqk * Dk, *av = ak + (size_t)T * Nqk * Dk;
        e = gdn::launch_act_to_f16(static_cast<const float *>(q), static_cast<const float *>(k),
                                   static_cast<const float *>(v), aq, ak, av, Ti, Nqk, Nvs, w.status, st, dims);
        q16 = aq, k16 = ak, v16 = av;
    }
    const int R = gdn::pipeline_ranges(NC);
    if (e == cudaSuccess && R == 1) {
        e = gdn::launch_intra(k16, v16, g, beta, eps, Ti, Nqk, Nvs, 0, NC, w, st, delta, f16, dims);
        if (e == cudaSuccess)
            e = gdn::launch_state(k16, state_pool, state_indices, final_state, Ti, B, Nqk, Nvs, 0, NC, 0, w, st, delta,
                                  f16, sdt, dims);
        if (e == cudaSuccess)
            e = gdn::launch_output(q16, k16, g, sc, eps, out, Ti, Nqk, Nvs, 0, NC, w, st, delta, f16, odt, dims);
    } else if (e == cudaSuccess) {
        std::lock_guard<std::mutex> guard(g_pipe_lock);
        SideStreams *ss = nullptr;
        e = side_streams(&ss);
        if (e == cudaSuccess) {
            // ev[0]: fork; ev[1 + r]: intra-chunk of range r done; ev[1 + R + r]: state pass of range r done;
            // ev[1 + 2R], ev[2 + 2R]: join
            cudaEvent_t *ev = ss->ev;
            auto c0 = [&](int r) { return gdn::range_begin(r, R, NC); };
            auto c1 = [&](int r) { return gdn::range_begin(r + 1, R, NC); };
            e = cudaEventRecord(ev[0], st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->intra, ev[0], 0);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->state, ev[0], 0);
            for (int r = 0; r < R && e == cudaSuccess; ++r) {
                e = gdn::launch_intra(k16, v16, g, beta, eps, Ti, Nqk, Nvs, c0(r), c1(r) - c0(r), w, ss->intra, delta,
                                      f16, dims);
                if (e == cudaSuccess) e = cudaEventRecord(ev[1 + r], ss->intra);
            }
            for (int r = 0; r < R && e == cudaSuccess; ++r) {
                e = cudaStreamWaitEvent(ss->state, ev[1 + r], 0);
                if (e == cudaSuccess)
                    e = gdn::launch_state(k16, state_pool, state_indices, final_state, Ti, B, Nqk, Nvs, c0(r), c1(r), r,
                                          w, ss->state, delta, f16, sdt, dims);
                if (e == cudaSuccess) e = cudaEventRecord(ev[1 + R + r], ss->state);
            }
            for (int r = 0; r < R && e == cudaSuccess; ++r) {
                e = cudaStreamWaitEvent(st, ev[1 + R + r], 0);
                if (e == cudaSuccess)
                    e = gdn::launch_output(q16, k16, g, sc, eps, out, Ti, Nqk, Nvs, c0(r), c1(r) - c0(r), w, st, delta,
                                           f16, odt, dims);
            }
            // join, also after a failed launch, so that nothing of this call runs outside `st` afterwards
            cudaError_t j = cudaEventRecord(ev[1 + 2 * R], ss->intra);
            if (j == cudaSuccess) j = cudaEventRecord(ev[2 + 2 * R], ss->state);
            if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ev[1 + 2 * R], 0);
            if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ev[2 + 2 * R], 0);
            if (e == cudaSuccess) e = j;
        }
    }
    if (owned) {
        cudaError_t f = cudaFreeAsync(workspace, st);
        if (e == cudaSuccess) e = f;
    }
    return cuda_status(e);
}

}  // extern "C"
