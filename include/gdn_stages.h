/*
 * gdn_stages.h -- the kernels of gdn_chunk_fwd as separate C-ABI calls.
 *
 * gdn_chunk_fwd (gdn.h) runs the same kernels as gdn_stage_chunk_map,
 * gdn_stage_intra, gdn_stage_state and gdn_stage_output enqueued in that order
 * on one stream with one workspace, with the same results: it splits the
 * chunks into R ranges (see `carry`) and overlaps the ranges' kernels on
 * streams of its own, which fork from and join back into the caller's stream
 * within the call.  The stages run over all chunks.  They are exposed so that each
 * kernel can be checked against the chunked form's intermediates and timed on
 * its own.  Conventions (device pointers, bf16 as uint16_t bits, asynchronous
 * on `stream`, status codes, alignment) are those of gdn.h.  Every stage takes
 * the sizes (T, B, Nqk, Nv) and the workspace that the chunk map was built
 * with; a stage reads the workspace regions that earlier stages wrote.
 *
 * Notation (page "Qwen3Next Samples", "Mathematical Formulas"; the state is
 * held as S[Dk, Dv] as on the decode page): per chunk of L = 128 tokens of one
 * sequence and v-head, gamma = chunk-local cumulative gate, Gamma_ij =
 * exp(gamma_i - gamma_j), kh/qh the normalised keys/queries, beta the update
 * rates.  A_ij = beta_i (kh_i . kh_j) Gamma_ij for j < i (the page's A with
 * its negative mask is -A); T = (I + A)^-1; U = T diag(beta) V;
 * W = T diag(beta e^gamma) Kh; S_c is the state entering chunk c;
 * U' = U - W S_c; S_{c+1} = e^{gamma_last} S_c + (Kh * e^{gamma_last - gamma})^T U';
 * o = diag(e^gamma) Qh S_c + (Qh Kh^T * Gamma * tril) U'.
 */
#ifndef GDN_STAGES_H_
#define GDN_STAGES_H_

#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Byte offsets of the workspace regions (each 256-byte aligned) for given
 * sizes.  NC = max_chunks = floor((T + 127 B) / 128), an upper bound on the
 * number of chunks of any packing of T tokens into B sequences.
 *   status      int32[4]: [0] cu_seqlens error bits (1: cu[0] != 0, 2: decreasing,
 *               4: cu[B] != T), [1] number of chunks, [2] tensor-core completion
 *               waits that gave up (bit 0: state pass, bit 1: output, bit 2:
 *               intra-chunk; the
 *               results are then incomplete); the caller clears [2] to read it
 *   chunk_info  int32[NC][4]: sequence, first token, tokens in the chunk (1..128),
 *               chunk index within its sequence; rows past the last chunk hold -1
 *   seq_chunk0  int32[B+1]: first chunk of each sequence, [B] = number of chunks
 *   rq          fp32 [Nqk][T]: scale / sqrt(|q|^2 + eps)
 *   rk          fp32 [Nqk][T]: 1 / sqrt(|k|^2 + eps)
 *   gcum        fp32 [Nv][T]: chunk-local cumulative gate gamma
 *   betaf       fp32 [Nv][T]: beta widened to fp32
 *   U, W        fp16 [NC][Nv][128 (L)][128]: U and W (columns Dk) of each chunk
 *   Mk          fp16 [NC][Nv][128 (Dk)][128 (Dk)]: Mk = k_gexp^T W, the factor of
 *               the state update that multiplies the state
 *   Sc          fp16 [NC][Nv][128 (Dk)][128 (Dv)]: state entering each chunk
 *   fa          fp32 [NC][Nv][132]: per chunk rk_t e^{gamma_L - gamma_t} for its
 *               rows t < 128 (0 past the chunk), e^{gamma_L} at 128, zeros after
 *   carry       fp32 [R-1][Nv][128][128]: the state of a sequence that crosses the
 *               boundary after chunk range r (the forward pass runs R chunk ranges
 *               as a pipeline: R = 2 from NC = 32 on, else 1; empty when R = 1)
 *   act16       fp16 q [T][Nqk][128], k [T][Nqk][128], v [T][Nv][128]: fp32
 *               activations of gdn_chunk_fwd_typed rounded to fp16 (empty for
 *               16-bit activations and in gdn_workspace_layout)
 * The tensor-core products take fp16 operands (11-bit significand) with fp32
 * accumulation: the raw bf16 q, k, v convert to fp16 exactly (magnitudes in
 * [2^-14, 65504]), the L2 norms enter as fp32 scalings, and the state update's
 * second operand is split into two fp16 halves; bf16 operands missed the
 * max-abs bound.  Values derived from v (U, U', S) must stay below 65504 in
 * magnitude.
 */
typedef struct {
    size_t total;
    size_t status;
    size_t chunk_info;
    size_t seq_chunk0;
    size_t rq;
    size_t rk;
    size_t gcum;
    size_t betaf;
    size_t U;
    size_t W;
    size_t Mk;
    size_t Sc;
    size_t fa;
    size_t carry;
    size_t act16;
    int64_t max_chunks;
} gdn_workspace_layout_t;

/* Fill *layout for these sizes; GDN_ERR_BAD_SHAPE on negative sizes. */
int gdn_workspace_layout(int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                         gdn_workspace_layout_t *layout);

/*
 * Chunk table from cu_seqlens (device int32 [B+1]): splits every sequence
 * into chunks of 128 tokens starting at its first token, the last chunk taking
 * the remainder ("Qwen3Next Samples": L = 128, act_seq_len).  Token ranges
 * are clamped to [0, T) so that a malformed cu_seqlens can never make a later
 * stage read or write out of bounds; the error bits in status say why.
 */
int gdn_stage_chunk_map(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t Nqk, int32_t Nv,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * Intra-chunk: per (chunk, v-head) the L2 normalisation factors of k ("L2
 * Normalization", eps inside the square root), the cumulative gate ("Gate
 * Cumulative Sum") restarting at every chunk start, A ("Pre-Attention
 * Matrix"), T = (I + A)^-1 by the block merge of inverse_pto / inverse_matmul
 * ("Matrix Inversion"), U and W ("Value and Key Cumulative Decay"), and
 * Mk = k_gexp^T W with k_gexp = Kh * exp(g_last - g_cum) ("State Update").
 * Reads k [T, Nqk, 128], v [T, Nv, 128] (bf16), g [T, Nv] fp32, beta [T, Nv]
 * bf16; writes U, W, Mk, fa, and rk, gcum, betaf (for inspection).
 */
int gdn_stage_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps,
                    int64_t T, int32_t B, int32_t Nqk, int32_t Nv, void *workspace, size_t workspace_bytes,
                    void *stream);

/*
 * Inter-chunk state passing: per (sequence, v-head, 64-column slice of Dv),
 * serially over the sequence's chunks, S <- e^{gamma_last} S + k_gexp^T U - Mk S
 * ("State Update" with v' = W S regrouped), the state kept in fp32 on chip.
 * S starts from state_pool[state_indices[b]] (or slot b, or zero without a
 * pool).  Reads k [T, Nqk, 128] bf16, fa, U and Mk; writes Sc for every chunk
 * and final_state (if not NULL).
 */
int gdn_stage_state(const uint16_t *k, const float *state_pool, const int32_t *state_indices, float *final_state,
                    int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P, void *workspace,
                    size_t workspace_bytes, void *stream);

/*
 * Output: per (chunk, v-head) o = (diag(e^gamma) Qh - P W) S_c + P U with
 * P = Qh Kh^T * Gamma * tril ("Recurrent State Attention": o_inter and
 * o_chunk regrouped; tril includes the diagonal).  Reads q, k [T, Nqk, 128]
 * bf16, g [T, Nv] fp32, W, U, Sc; writes out [T, Nv, 128] bf16 for every token
 * of every chunk, and rq (for inspection).  scale <= 0 selects 1/sqrt(128).
 */
int gdn_stage_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, uint16_t *out,
                     int64_t T, int32_t B, int32_t Nqk, int32_t Nv, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * Fused short-sequence forward: the token recurrence of the decode page
 * ("lite_boost.ops.recurrent_gated_delta_rule", algorithm flow, for up to 8
 * tokens per call there) run with each (sequence, v-head, 32-column slice)
 * state held in registers: one pass reads the initial state from the pool,
 * applies the sequence's tokens and writes out and final_state.  Correct for
 * any length (cost grows linearly with it); gdn_chunk_fwd routes here when
 * 1 <= max_seqlen <= GDN_SHORT_MAX.  Same arguments as gdn_chunk_fwd without
 * the workspace.
 */
int gdn_short_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                  const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                  const int32_t *state_indices, float scale, float eps, uint16_t *out,
                  float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                  void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_STAGES_H_ */
