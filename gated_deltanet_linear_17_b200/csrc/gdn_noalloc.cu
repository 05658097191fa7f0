// gdn_chunk_fwd_noalloc: the forward pass for callers that cannot allocate
// device memory.  The chunked path's workspace is a static device buffer that
// lives inside this library (one per GPU) instead of caller or cudaMalloc
// memory; everything else is gdn_chunk_fwd unchanged.
#include <mutex>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

// The scratch buffer.  On the host, `g_scratch` names a host-side stand-in of
// the variable, not its device address: handing it to a kernel would fault, or
// on a system where the GPU can reach host memory silently use the wrong
// memory.  Host code therefore asks the runtime for the device address of the
// current device's copy (cudaGetSymbolAddress) and passes that.
static __device__ __align__(256) unsigned char g_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_device_addr[kMaxDevices];  // device address of g_scratch, per device, set on first use

// Device address of the current device's scratch, looked up once per device.
int scratch_address(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_device_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
        g_device_addr[dev] = p;
    }
    *addr = g_device_addr[dev];
    return GDN_OK;
}

}  // namespace

extern "C" int gdn_chunk_fwd_noalloc(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                                     const uint16_t *beta, const int32_t *cu_seqlens, const float *state_pool,
                                     const int32_t *state_indices, float scale, float eps, uint16_t *out,
                                     float *final_state, int64_t T, int32_t B, int32_t Nqk, int32_t Nv, int32_t P,
                                     int32_t max_seqlen, void *stream)
{
    // sizes that gdn_chunk_fwd refuses get its code, before the scratch limit is looked at
    if (T < 0 || B < 0 || Nqk <= 0 || Nv <= 0 || P < 0 || Nv % Nqk != 0) return GDN_ERR_BAD_SHAPE;
    if (T >= (int64_t(1) << 31) || Nqk > 64 || Nv > 256) return GDN_ERR_UNSUPPORTED;
    const bool short_path = max_seqlen >= 1 && max_seqlen <= GDN_SHORT_MAX;
    // reject sizes whose workspace does not fit, before anything is enqueued
    if (!short_path && gdn_chunk_fwd_workspace_bytes(T, B, Nqk, Nv) > (size_t)GDN_NOALLOC_SCRATCH_BYTES)
        return GDN_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != GDN_OK) return rc;
    // Nothing in the workspace has to start at zero: the chunk-table kernel
    // clears the status words first, and every other region a kernel reads is
    // written earlier in the same call, so the previous call's leftovers are
    // never used.  A non-NULL workspace means no allocation.
    return gdn_chunk_fwd(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, scale, eps, out, final_state, T,
                         B, Nqk, Nv, P, max_seqlen, scratch, (size_t)GDN_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int gdn_noalloc_read_status(int32_t *status_out, void *stream)
{
    if (!status_out) return GDN_ERR_NULL_ARG;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != GDN_OK) return rc;
    return gdn_read_status(scratch, status_out, stream);
}
