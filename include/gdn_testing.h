/*
 * gdn_testing.h -- test hooks of the library (not part of the operator).
 *
 * gdn_selftest_umma: one CTA computes C[128, N] = sum_k A(m, k) B(n, k) on
 * the Blackwell tensor core (tcgen05.mma from swizzled shared-memory tiles,
 * fp32 accumulator in tensor memory, read back with tcgen05.ld).  It checks
 * the descriptor and layout conventions that the kernels build on, in
 * isolation, for K-major and MN-major operands.
 *   A       device fp16 (bf16 = 0) or bf16 (bf16 = 1): [128, K] row-major
 *           (a_mn = 0, K-major) or [K, 128] row-major (a_mn = 1, MN-major)
 *   B       device, same type: [N, K] (b_mn = 0) or [K, N] (b_mn = 1)
 *   C       device fp32 [128, N]
 *   N       32, 64, 128 or 256;  K  64 or 128
 *   status  device int32, set to 1 if the completion wait gave up (0 is not
 *           written: the caller clears it)
 * Returns a gdn_status_t code; the work is enqueued on `stream`.
 */
#ifndef GDN_TESTING_H_
#define GDN_TESTING_H_

#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

int gdn_selftest_umma(const uint16_t *A, const uint16_t *B, float *C, int32_t N, int32_t K, int32_t bf16,
                      int32_t a_mn, int32_t b_mn, int32_t *status, void *stream);

/*
 * gdn_selftest_wait: the bounded mbarrier wait of the kernels, run out on
 * purpose without faulting or hanging.  One thread initialises an mbarrier
 * that expects one arrival, arrives on it if `arrive` is nonzero, and waits
 * for its phase with at most `max_polls` polls (the kernels use 2^22, about
 * 0.3 s).  Without the arrival the wait gives up, and the thread sets
 * GDN_DEV_WAIT_SELFTEST in status word 2 of `workspace` (the word that the
 * chunked kernels use for their own waits; read it with gdn_read_status).
 * Nothing else is touched: no copy or tensor-core work is in flight.
 *   max_polls   1 .. 2^22
 *   workspace   device, 16-byte aligned, at least 16 bytes
 */
int gdn_selftest_wait(int32_t max_polls, int32_t arrive, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_testing_host_plan: the cut of gdn_chunk_fwd_host into pieces and calls,
 * on the host only (no CUDA call).  For host int32 cu_seqlens [B+1] and
 * `segments` (as for gdn_chunk_fwd_host) it writes up to max_calls rows of 7
 * int32 into calls: segment, first sequence, number of sequences, first token,
 * end token, initial-state source (1 the sequence's own initial state, 2 the
 * state carried from the previous piece), final-state target (0 the final
 * row, 1 carried to the next piece).  Returns the number of calls, or -1 for
 * invalid arguments or too small a max_calls.
 */
int gdn_testing_host_plan(const int32_t *cu_seqlens, int64_t T, int32_t B, int32_t segments, int32_t *calls,
                          int32_t max_calls);

#ifdef __cplusplus
}
#endif

#endif /* GDN_TESTING_H_ */
