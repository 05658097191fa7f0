// Output kernel: one CTA per (chunk, v-head).
//
// Page "Qwen3Next Samples", "Recurrent State Attention":
//   o_inter = (q (.) exp(g_cum)) S^T
//   o_chunk = o_inter + (q k^T (.) D_decay (.) T_tril) (v_out - v')
// with S held as [Dk, Dv] (so S^T there is S here), T_tril including the
// diagonal, and v_out - v' = U' from the state kernel.  q k^T is a bf16
// product of the raw rows (exact inputs); q is then converted to fp16 in place
// (exact) for the q S product with the fp16 state.  The normalisation and the
// query scale enter as the prologue's fp32 factors rq, rk, applied to the
// q k^T product and to the rows of q S.  Accumulation is fp32.  Each warp owns 16 rows of the chunk;
// its rows of P = (q k^T) (.) Gamma (.) tril never leave registers: the
// accumulator fragments of two adjacent 8-column tiles are exactly the A
// fragment of one 16-wide k step of the P U' product.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kOutThreads = 256;
constexpr int OO_Q = 0, OO_K = 32768, OO_S = 65536, OO_U = 98304, OO_VEC = 131072;
constexpr int kOutSmem = OO_VEC + 3 * 128 * 4;

__global__ void __launch_bounds__(kOutThreads, 1) output_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, uint16_t *__restrict__ out, int T,
    int Nqk, int Nv, const int4 *__restrict__ info, const float *__restrict__ rq, const float *__restrict__ rk,
    const float *__restrict__ gcum, const uint16_t *__restrict__ Up, const uint16_t *__restrict__ Sc)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int c = blockIdx.x, h = blockIdx.y;
    const ChunkInfo ci = load_chunk(info, c);
    if (ci.seq < 0) return;
    const int hq = h / (Nv / Nqk);
    const int n = ci.len, t0 = ci.start;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    const uint32_t qs = smem_addr(smem + OO_Q), ks = smem_addr(smem + OO_K), ss = smem_addr(smem + OO_S),
                   us = smem_addr(smem + OO_U);
    float *gam = reinterpret_cast<float *>(smem + OO_VEC);
    float *rqv = gam + 128, *rkv = gam + 256;

    const size_t tile = (size_t)(c * Nv + h) * L * D;
    for (int e = tid; e < 128 * 16; e += kOutThreads) {
        const int r = e >> 4, cc = e & 15;
        const bool ok = r < n;
        const int t = t0 + (ok ? r : 0);
        cp_async16(qs + sw256(r, cc), q + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        cp_async16(ks + sw256(r, cc), k + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
        cp_async16(ss + sw256(r, cc), Sc + tile + r * D + cc * 8, true);
        cp_async16(us + sw256(r, cc), Up + tile + r * D + cc * 8, true);
    }
    cp_async_commit();
    if (tid < 128) {
        const int i = tid;
        gam[i] = gcum[(size_t)h * T + t0 + min(i, n - 1)];
        rqv[i] = i < n ? rq[(size_t)hq * T + t0 + i] : 0.f;
        rkv[i] = i < n ? rk[(size_t)hq * T + t0 + i] : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    const int m0 = wid * 16;
    float acc[16][4];
    // ---- P = (Qh Kh^T) (.) Gamma (.) tril (diagonal included), rows of this warp only
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D; kk += 16) {
        uint32_t a[4];
        ldsm_x4(a_rowmajor_256(qs, m0, kk, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            if (np <= wid) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b_nmajor_256(ks, np * 16, kk, lane), b0, b1, b2, b3);
                mma16816_bf16(acc[2 * np], a, b0, b1);
                mma16816_bf16(acc[2 * np + 1], a, b2, b3);
            }
        }
    }
    __syncthreads();  // every warp is done with the bf16 q rows
    // q to fp16 in place for the q S product (each thread converts the chunks it copied)
    for (int e = tid; e < 128 * 16; e += kOutThreads) bf16_chunk_to_fp16(smem + OO_Q + sw256(e >> 4, e & 15));
    __syncthreads();
    // P as fp16 A fragments: pa[j] is k block j (columns 16j..16j+15) of this warp's 16 rows
    uint32_t pa[8][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int row = m0 + gid + hf * 8;
            const int col = nt * 8 + tig * 2;
            float p0 = 0.f, p1 = 0.f;
            if ((nt >> 1) <= wid) {
                const float fr = rqv[row];
                if (col <= row) p0 = fr * rkv[col] * acc[nt][2 * hf] * __expf(gam[row] - gam[col]);
                if (col + 1 <= row) p1 = fr * rkv[col + 1] * acc[nt][2 * hf + 1] * __expf(gam[row] - gam[col + 1]);
            }
            pa[nt >> 1][(nt & 1) * 2 + hf] = pack_h2(p0, p1);
        }
    }

    // ---- o = diag(rq e^gamma) Q S_c + P U'
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D; kk += 16) {
        uint32_t a[4];
        ldsm_x4(a_rowmajor_256(qs, m0, kk, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(b_kmajor_256(ss, np * 16, kk, lane), b0, b1, b2, b3);
            mma16816(acc[2 * np], a, b0, b1);
            mma16816(acc[2 * np + 1], a, b2, b3);
        }
    }
    {
        const float f0 = rqv[m0 + gid] * __expf(gam[m0 + gid]);
        const float f1 = rqv[m0 + gid + 8] * __expf(gam[m0 + gid + 8]);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            acc[nt][0] *= f0;
            acc[nt][1] *= f0;
            acc[nt][2] *= f1;
            acc[nt][3] *= f1;
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j <= wid) {
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b_kmajor_256(us, np * 16, j * 16, lane), b0, b1, b2, b3);
                mma16816(acc[2 * np], pa[j], b0, b1);
                mma16816(acc[2 * np + 1], pa[j], b2, b3);
            }
        }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int row = m0 + gid + hf * 8;
        if (row < n) {
            uint16_t *dst = out + ((size_t)(t0 + row) * Nv + h) * D;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt)
                *reinterpret_cast<uint32_t *>(dst + nt * 8 + tig * 2) =
                    pack_bf2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
        }
    }
}

cudaError_t launch_output(const uint16_t *q, const uint16_t *k, uint16_t *out, int T, int Nqk, int Nv, int NC,
                          const Workspace &ws, cudaStream_t st)
{
    if (NC == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kOutSmem);
    if (e != cudaSuccess) return e;
    output_kernel<<<dim3(NC, Nv), kOutThreads, kOutSmem, st>>>(q, k, out, T, Nqk, Nv, ws.chunk_info, ws.rq, ws.rk,
                                                                ws.gcum, ws.Up, ws.Sc);
    return cudaGetLastError();
}

}  // namespace gdn
