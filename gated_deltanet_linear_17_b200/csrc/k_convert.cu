// fp32 activations for the chunked path: q, k and v rounded to fp16 (round to
// nearest even) into the workspace, so that the chunked kernels take them as fp16
// rows.  The LinearAttention page lets activations be fp32; the tensor-core
// operands of kind::f16 are 16-bit, and fp16 keeps 11 significant bits of each
// element (bf16 would keep 8).  A value beyond +-65504 (or a NaN) cannot be held
// and sets GDN_DEV_RANGE_INPUT in status word 3 instead of going on silently.
#include <algorithm>

#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {

// n8 groups of 8 elements of src -> dst; grid-stride
__global__ void __launch_bounds__(256) act_to_f16_kernel(const float4 *__restrict__ src, uint4 *__restrict__ dst,
                                                         size_t n8, int32_t *__restrict__ status)
{
    float m = 0.f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = src[2 * i], b = src[2 * i + 1];
        m = absmax_nan(absmax_nan(absmax_nan(absmax_nan(m, a.x), a.y), a.z), a.w);
        m = absmax_nan(absmax_nan(absmax_nan(absmax_nan(m, b.x), b.y), b.z), b.w);
        dst[i] = make_uint4(pack_h2(a.x, a.y), pack_h2(a.z, a.w), pack_h2(b.x, b.y), pack_h2(b.z, b.w));
    }
    if (__any_sync(0xffffffffu, out_of_fp16(m)) && (threadIdx.x & 31) == 0) atomicOr(status + 3, GDN_DEV_RANGE_INPUT);
}

cudaError_t launch_act_to_f16(const float *q, const float *k, const float *v, uint16_t *q16, uint16_t *k16,
                              uint16_t *v16, int T, int Nqk, int Nv, int32_t *status, cudaStream_t st, Dims dims)
{
    // q, k [T][Nqk][Dk]; v [T][Nv][128] with Nv counting 128-column sub-heads
    const size_t nqk = (size_t)T * Nqk * dims.Dk / 8, nv = (size_t)T * Nv * D / 8;
    const struct { const float *s; uint16_t *d; size_t n8; } parts[3] = {{q, q16, nqk}, {k, k16, nqk}, {v, v16, nv}};
    for (const auto &p : parts) {
        if (p.n8 == 0) continue;
        const size_t blocks = std::min<size_t>((p.n8 + 255) / 256, 148 * 8);
        act_to_f16_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(p.s),
                                                            reinterpret_cast<uint4 *>(p.d), p.n8, status);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdn
