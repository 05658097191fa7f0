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
    uint16_t *act16;  // fp32 activations rounded to fp16: q [T][Nqk][D], k [T][Nqk][D], v [T][Nv][D] (or null)
    int NC;  // max chunks
};

// the value checks of gdn_check_values: bits GDN_DEV_VAL_* ORed into *word (g, beta [T][Nv] or null;
// idx [B] or null)
cudaError_t launch_check_values(const float *g, const uint16_t *beta, const int32_t *idx, long long T, int Nv, int B,
                                int P, int32_t *word, cudaStream_t st);
cudaError_t launch_chunk_map(const int32_t *cu, int B, int T, int NC, const Workspace &ws,
                             cudaStream_t st);
// intra and output run over chunks [c0, c0 + nc); the state pass over [c_lo, c_hi), range index `range`
// Head dimensions of the chunked path.  The kernels work on 128 x 128 states; a key dimension Dk of 64
// reads as 128 with the last 64 columns zero (the TMA copies of q and k fill them, and the state rows
// past Dk stay zero), and a value dimension Dv = 128 m runs as m sub-heads of 128 columns per v-head,
// which share the v-head's gate, beta and qk-head (the columns of the state evolve independently).
// Every kernel's Nv argument then counts sub-heads (Nv m).
struct Dims {
    int Dk = 128, Dv = 128, m = 1;
};

// element types of the chunked path: kActBF16 / kActF16 raw 16-bit q, k, v rows; outputs and states
// also kTypeF32 (the dtype codes of gdn.h: 0 fp32, 1 bf16, 2 fp16)
constexpr int kTypeF32 = 0, kTypeBF16 = 1, kTypeF16 = 2;
cudaError_t launch_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps, int T,
                         int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st, bool delta = true,
                         bool f16 = false, Dims dims = Dims());
cudaError_t launch_state(const uint16_t *k, const void *pool, const int32_t *idx, void *final_state, int T, int B,
                         int Nqk, int Nv, int c_lo, int c_hi, int range, const Workspace &ws, cudaStream_t st,
                         bool delta = true, bool f16 = false, int state_type = kTypeF32, Dims dims = Dims());
cudaError_t launch_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, void *out,
                          int T, int Nqk, int Nv, int c0, int nc, const Workspace &ws, cudaStream_t st,
                          bool delta = true, bool f16 = false, int out_type = kTypeBF16, Dims dims = Dims());
// delta == false (launch_intra / launch_state / launch_output): an update rule without the
// retrieval (U = v, no W or Mk); g == nullptr: a zero gate.  f16: q, k, v are fp16 rows (else bf16);
// state_type: the pool's and final state's type (fp32, bf16 or fp16); out_type: out's type.
// fp32 q, k, v rows rounded to fp16 (round to nearest even) into act16 [T][Nqk | Nqk | Nv][128]
// (the workspace's act16 region), before the fp16 kernels run
cudaError_t launch_act_to_f16(const float *q, const float *k, const float *v, uint16_t *q16, uint16_t *k16,
                              uint16_t *v16, int T, int Nqk, int Nv, int32_t *status, cudaStream_t st,
                              Dims dims = Dims());
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
// The one-token decode kernel (k_decode.cu): launch_recurrent routes to it when max_seqlen == 1 and
// decode_supported() holds (bf16 activations, an fp32 or bf16 pool, Dk 64 or 128, no window).
bool decode_supported(int act_dtype, int state_dtype, int Dk, int Dv, int win);
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g, const uint16_t *beta,
                          const float *gk, const int32_t *cu, void *pool, int state_dtype, int rule,
                          const int32_t *token_slots, const int32_t *num_accepted, float scale, float eps, void *out,
                          int T, int B, int Nqk, int Nv, int Dk, int Dv, cudaStream_t st);

}  // namespace gdn
