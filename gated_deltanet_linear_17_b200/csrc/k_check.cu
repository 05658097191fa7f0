// Value checks of the operator's inputs on the device: the gate, beta and the slot indices.
//
// The decode page ("Raises") lists the operator's error cases and leaves the
// values themselves unchecked on the inference path: a check is a pass over the
// inputs.  On request (gdn_check_values, or the switch gdn_set_value_checks for
// the chunked entry points) this pass runs on the device and records what it
// finds as bits of a status word, without a host synchronisation:
//   GDN_DEV_VAL_GATE   a gate g[t, h] that is not <= 0 (a positive value or a NaN): the
//                      recurrence's decay exp(g) must not exceed 1 ("Gate Cumulative Sum").
//   GDN_DEV_VAL_BETA   a beta[t, h] outside [0, 1] (or a NaN): the page's beta is a sigmoid.
//   GDN_DEV_VAL_INDEX  a state index outside [0, P): the slot would lie outside the pool.
// One grid-stride pass reads g (fp32) and beta (bf16) once, so it is bound by HBM:
// 6 bytes per (token, v-head) and 4 per sequence.
#include <algorithm>

#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {

__global__ void __launch_bounds__(256) check_values_kernel(const float *__restrict__ g,
                                                           const uint16_t *__restrict__ beta,
                                                           const int32_t *__restrict__ idx, long long n, int B, int P,
                                                           int32_t *__restrict__ word)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    int bits = 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        if (g && !(g[i] <= 0.f)) bits |= GDN_DEV_VAL_GATE;
        if (beta) {
            const float b = bf2f(beta[i]);
            if (!(b >= 0.f && b <= 1.f)) bits |= GDN_DEV_VAL_BETA;
        }
    }
    if (idx)
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < B; i += stride)
            if (idx[i] < 0 || idx[i] >= P) bits |= GDN_DEV_VAL_INDEX;
    bits = __reduce_or_sync(0xffffffffu, bits);
    if (bits && (threadIdx.x & 31) == 0) atomicOr(word, bits);
}

cudaError_t launch_check_values(const float *g, const uint16_t *beta, const int32_t *idx, long long T, int Nv, int B,
                                int P, int32_t *word, cudaStream_t st)
{
    const long long n = T * Nv;
    if ((n == 0 || (!g && !beta)) && (!idx || B == 0)) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (std::max(n, (long long)B) + 255) / 256;
    const int grid = (int)std::max(1LL, std::min(want, (long long)sms * 8));
    check_values_kernel<<<grid, 256, 0, st>>>(g, beta, idx, n, B, P, word);
    return cudaGetLastError();
}

}  // namespace gdn
