// Internal declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

constexpr int L = 128;  // chunk length
constexpr int D = 128;  // head dimension (Dk = Dv)
constexpr int kMaxRanges = 2;   // chunk ranges of the pipelined forward pass
constexpr int kFaStride = 132;  // floats per (chunk, v-head) record of the state-update factors (16-byte multiple)

// Chunk ranges of the pipelined forward pass for NC chunks: two halves from 32
// chunks on, one range (no pipeline) below.  Measured at 256 chunks (one-layer
// prefill, 32 v-heads): 2 ranges 0.89 ms, 3: 0.93, 4: 0.93, 8: 0.99, 16: 1.06,
// the kernels one after another 1.07 ms; every range adds a launch of each kernel
// and its tail, and the overlap is already near the GPU's busy time with two.
inline int pipeline_ranges(long long NC)
{
    const long long r = NC / 16;
    return (int)(r < 1 ? 1 : r > kMaxRanges ? kMaxRanges : r);
}
// first chunk of range r of R over NC chunks (range_begin(R) = NC)
inline int range_begin(int r, int R, int NC)
{
    return (int)((long long)NC * r / R);
}

// Typed views of the workspace regions (layout: gdn_workspace_layout in gdn_stages.h)
struct Workspace {
    int32_t *status;
    int4 *chunk_info;
    int32_t *seq_chunk0;
    float *rq, *rk;     // fp32 [Nqk][T]: scale / |q|, 1 / |k| (eps inside the square root)
    float *gcum, *betaf;
    uint16_t *U, *W, *Mk, *Sc;
    float *fa;     // [NC][Nv][kFaStride]: rk_t e^{gamma_L - gamma_t} (t < 128), e^{gamma_L} at 128
    float *carry;  // [kMaxRanges][Nv][D][D]: fp32 state crossing a chunk-range boundary
    int NC;  // max chunks
};

cudaError_t launch_chunk_map(const int32_t *cu, int B, int T, int NC, const Workspace &ws,
                             cudaStream_t st);
// intra and output run over chunks [c0, c0 + nc); the state pass over [c_lo, c_hi), range index `range`
cudaError_t launch_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps, int T,
                         int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st, bool delta = true);
cudaError_t launch_state(const uint16_t *k, const float *pool, const int32_t *idx, float *final_state, int T, int B,
                         int Nqk, int Nv, int c_lo, int c_hi, int range, const Workspace &ws, cudaStream_t st, bool delta = true);
cudaError_t launch_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, uint16_t *out,
                          int T, int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st, bool delta = true);
// delta == false (launch_intra / launch_state / launch_output): an update rule without the
// retrieval (U = v, no W or Mk); g == nullptr: a zero gate.
// Fused short-sequence kernel: sequence b starts from pool[idx ? idx[b] : b] (or
// zero without a pool) and ends in final_state[b].
cudaError_t launch_short(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const uint16_t *beta, const int32_t *cu, const float *pool, const int32_t *idx, float scale,
                         float eps, uint16_t *out, float *final_state, int T, int B, int Nqk, int Nv, int max_seqlen,
                         cudaStream_t st, int rule = 0);
// The same kernel on a pool updated in place (dtype codes: 0 fp32, 1 bf16, 2 fp16 for the activations
// q, k, v, out and for the pool), one slot per token,
// the start taken from the last accepted token's slot; key dimension Dk (64 or 128), value dimension
// Dv (a multiple of 32); gk [T, Nv, Dk] or nullptr (read only by the decaying rules).
// update rules of gdn_recurrent_fwd (GDN_RULE_* in gdn.h)
constexpr int kRuleGatedDelta = 0, kRuleDelta = 1, kRuleGated = 2, kRuleLinear = 3;
cudaError_t launch_recurrent(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                             const float *gk, const int32_t *cu, void *pool, int act_dtype, int state_dtype, int rule,
                             const int32_t *token_slots, const int32_t *num_accepted, float scale, float eps, void *out,
                             int T, int B, int Nqk, int Nv, int Dk, int Dv, int max_seqlen, cudaStream_t st,
                             int win = 0);
// win > 0: the pool is a state window [win, B, Nv, Dk, Dv] updated in place (token_slots and
// num_accepted unused); see gdn_recurrent_window_fwd in gdn.h.

}  // namespace gdn
