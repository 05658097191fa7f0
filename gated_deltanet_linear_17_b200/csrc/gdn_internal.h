// Internal declarations shared by the host API and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

constexpr int L = 128;  // chunk length
constexpr int D = 128;  // head dimension (Dk = Dv)
constexpr int kFaStride = 132;  // floats per (chunk, v-head) record of the state-update factors (16-byte multiple)

// Typed views of the workspace regions (layout: gdn_workspace_layout in gdn_stages.h)
struct Workspace {
    int32_t *status;
    int4 *chunk_info;
    int32_t *seq_chunk0;
    float *rq, *rk;     // fp32 [Nqk][T]: scale / |q|, 1 / |k| (eps inside the square root)
    float *gcum, *betaf;
    uint16_t *U, *W, *Mk, *Sc;
    float *fa;  // [NC][Nv][kFaStride]: rk_t e^{gamma_L - gamma_t} (t < 128), e^{gamma_L} at 128
    int NC;  // max chunks
};

cudaError_t launch_chunk_map(const int32_t *cu, int B, int T, int NC, const Workspace &ws,
                             cudaStream_t st);
cudaError_t launch_intra(const uint16_t *k, const uint16_t *v, const float *g, const uint16_t *beta, float eps, int T,
                         int Nqk, int Nv, int NC, const Workspace &ws, cudaStream_t st);
cudaError_t launch_state(const uint16_t *k, const float *pool, const int32_t *idx, float *final_state, int T, int B,
                         int Nqk, int Nv, const Workspace &ws, cudaStream_t st);
cudaError_t launch_output(const uint16_t *q, const uint16_t *k, const float *g, float scale, float eps, uint16_t *out,
                          int T, int Nqk, int Nv, int NC, const Workspace &ws, cudaStream_t st);
cudaError_t launch_short(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                         const uint16_t *beta, const int32_t *cu, const float *pool, const int32_t *idx,
                         float scale, float eps, uint16_t *out, float *final_state, int T, int B, int Nqk,
                         int Nv, cudaStream_t st);

}  // namespace gdn
