// Intra-chunk kernel: one CTA per (chunk, v-head).
//
// Page "Qwen3Next Samples", chunk_gated_delta_rule, "Mathematical Formulas":
//   A  = (k_beta k^T) (.) D_decay (.) M_mask      "Pre-Attention Matrix"
//   (I - A)^-1                                     "Matrix Inversion"
//   v_out = (I - A)^-1 (v (.) beta)                "Value and Key Cumulative Decay"
//   k_cumdecay = (I - A)^-1 (k_beta (.) exp(g_cum))
// Here A denotes the positive strictly-lower matrix beta_i (kh_i . kh_j) Gamma_ij
// (the page's A with its negative mask is -A), T = (I + A)^-1, U = v_out and
// W = k_cumdecay.  Keys arrive L2-normalised in fp16 from the prologue; v is
// converted from bf16 to fp16 while it is staged.  All tensor-core operands
// are fp16 with fp32 accumulation, and U and W are stored in fp16.
//
// The inverse is computed as on the page's inverse_pto / inverse_matmul: the
// 16x16 diagonal blocks are inverted by forward substitution (one warp each),
// then each block row i is completed from the rows above it,
//   T_ij = -T_ii sum_{j<=m<i} A_im T_mj,
// which is the 2x2 block merge applied block row by block row.
#include "common.cuh"
#include "gdn_internal.h"

namespace gdn {

constexpr int kIntraThreads = 256;
constexpr int FS = 132;  // fp32 row stride (floats) of the A and T scratch matrices

constexpr int OFF_K = 0;
constexpr int OFF_V = 32768;
constexpr int OFF_A = 65536;                  // fp32 [128][132]; later fp16 Tb and Tw
constexpr int OFF_T = OFF_A + 128 * FS * 4;   // fp32 [128][132]
constexpr int OFF_VEC = OFF_T + 128 * FS * 4; // gam, bet, (unused), egam
constexpr int kIntraSmem = OFF_VEC + 4 * 128 * 4;

__global__ void __launch_bounds__(kIntraThreads, 1) intra_kernel(
    const uint16_t *__restrict__ kn, const uint16_t *__restrict__ v, int T, int Nqk, int Nv,
    const int4 *__restrict__ info, const float *__restrict__ gcum, const float *__restrict__ betaf,
    uint16_t *__restrict__ U, uint16_t *__restrict__ W)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int c = blockIdx.x, h = blockIdx.y;
    const ChunkInfo ci = load_chunk(info, c);
    if (ci.seq < 0) return;
    const int hq = h / (Nv / Nqk);
    const int n = ci.len, t0 = ci.start;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    const uint32_t ks = smem_addr(smem + OFF_K), vs = smem_addr(smem + OFF_V);
    float *Af = reinterpret_cast<float *>(smem + OFF_A);
    float *Tf = reinterpret_cast<float *>(smem + OFF_T);
    float *gam = reinterpret_cast<float *>(smem + OFF_VEC);
    float *bet = gam + 128, *egam = gam + 384;

    // ---- stage the chunk's normalised keys (fp16, async) and values (bf16 -> fp16);
    //      rows past the chunk are zero
    for (int e = tid; e < 128 * 16; e += kIntraThreads) {
        const int r = e >> 4, cc = e & 15;
        const bool ok = r < n;
        const int t = t0 + (ok ? r : 0);
        cp_async16(ks + sw256(r, cc), kn + ((size_t)t * Nqk + hq) * D + cc * 8, ok);
    }
    cp_async_commit();
    for (int e = tid; e < 128 * 16; e += kIntraThreads) {
        const int r = e >> 4, cc = e & 15;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (r < n) {
            w = __ldg(reinterpret_cast<const uint4 *>(v + ((size_t)(t0 + r) * Nv + h) * D + cc * 8));
            w = make_uint4(bf2_to_h2(w.x), bf2_to_h2(w.y), bf2_to_h2(w.z), bf2_to_h2(w.w));
        }
        *reinterpret_cast<uint4 *>(smem + OFF_V + sw256(r, cc)) = w;
    }
    if (tid < 128) {
        const int i = tid;
        const bool ok = i < n;
        const float gi = gcum[(size_t)h * T + t0 + min(i, n - 1)];
        gam[i] = gi;
        egam[i] = __expf(gi);
        bet[i] = ok ? betaf[(size_t)h * T + t0 + i] : 0.f;
    }
    for (int e = tid; e < 128 * 128; e += kIntraThreads) {
        const int i = e >> 7, j = e & 127;
        if ((j >> 4) > (i >> 4)) Tf[i * FS + j] = 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    const int m0 = wid * 16;
    // ---- A = strict_tril(diag(beta) Kh Kh^T (.) Gamma): warp w owns rows 16w..16w+15
    {
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D; kk += 16) {
            uint32_t a[4];
            ldsm_x4(a_rowmajor_256(ks, m0, kk, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                if (np <= wid) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(b_nmajor_256(ks, np * 16, kk, lane), b0, b1, b2, b3);
                    mma16816(acc[2 * np], a, b0, b1);
                    mma16816(acc[2 * np + 1], a, b2, b3);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            if ((nt >> 1) <= wid) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = m0 + gid + ((e >> 1) << 3);
                    const int col = nt * 8 + tig * 2 + (e & 1);
                    float val = 0.f;
                    if (col < row) val = bet[row] * acc[nt][e] * __expf(gam[row] - gam[col]);
                    Af[row * FS + col] = val;
                }
            }
        }
    }
    __syncthreads();

    // ---- diagonal 16x16 blocks of T = (I + A)^-1: lanes 0..15 of warp w own one column each
    if (lane < 16) {
        const int b0 = wid * 16, cidx = lane;
        float tcol[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float val = (i == cidx) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j)
                if (j >= cidx) val -= Af[(b0 + i) * FS + b0 + j] * tcol[j];
            tcol[i] = (i < cidx) ? 0.f : val;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tf[(b0 + i) * FS + b0 + cidx] = tcol[i];
    }
    __syncthreads();

    // ---- off-diagonal blocks, block row by block row: T_ij = -T_ii sum_{m=j}^{i-1} A_im T_mj
    for (int bi = 1; bi < 8; ++bi) {
        if (wid < bi) {
            const int bj = wid;
            const int r = lane >> 1, c0 = (lane & 1) * 8;
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = 0.f;
            for (int bk = bj; bk < bi; ++bk) {
                const float *arow = Af + (bi * 16 + r) * FS + bk * 16;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float a = arow[m];
                    const float *trow = Tf + (bk * 16 + m) * FS + bj * 16 + c0;
#pragma unroll
                    for (int u = 0; u < 8; ++u) x[u] += a * trow[u];
                }
            }
            float *xdst = Tf + (bi * 16 + r) * FS + bj * 16 + c0;
#pragma unroll
            for (int u = 0; u < 8; ++u) xdst[u] = x[u];
            __syncwarp();
            float y[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] = 0.f;
            const float *tii = Tf + (bi * 16 + r) * FS + bi * 16;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float t = tii[m];
                const float *xrow = Tf + (bi * 16 + m) * FS + bj * 16 + c0;
#pragma unroll
                for (int u = 0; u < 8; ++u) y[u] += t * xrow[u];
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 8; ++u) xdst[u] = -y[u];
        }
        __syncthreads();
    }

    // ---- fp16 operands with the column scalings folded in (A scratch is dead now):
    //      Tb = T diag(beta), Tw = T diag(beta e^gamma)
    uint8_t *Tb = smem + OFF_A, *Tw = smem + OFF_A + 32768;
    for (int e = tid; e < 128 * 64; e += kIntraThreads) {
        const int i = e >> 6, j = (e & 63) * 2;
        const float t0v = Tf[i * FS + j], t1v = Tf[i * FS + j + 1];
        const float b0 = bet[j], b1 = bet[j + 1];
        *reinterpret_cast<uint32_t *>(Tb + el256(i, j)) = pack_h2(t0v * b0, t1v * b1);
        *reinterpret_cast<uint32_t *>(Tw + el256(i, j)) = pack_h2(t0v * b0 * egam[j], t1v * b1 * egam[j + 1]);
    }
    __syncthreads();

    // ---- U = Tb V and W = Tw K (T is lower triangular: k blocks up to the diagonal)
    const uint32_t tb = smem_addr(Tb), tw = smem_addr(Tw);
    const size_t tile = (size_t)(c * Nv + h) * L * D;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const uint32_t ta = pass ? tw : tb;
        const uint32_t tbm = pass ? ks : vs;
        uint16_t *dst = (pass ? W : U) + tile;
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        for (int kk = 0; kk < (wid + 1) * 16; kk += 16) {
            uint32_t a[4];
            ldsm_x4(a_rowmajor_256(ta, m0, kk, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b_kmajor_256(tbm, np * 16, kk, lane), b0, b1, b2, b3);
                mma16816(acc[2 * np], a, b0, b1);
                mma16816(acc[2 * np + 1], a, b2, b3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int col = nt * 8 + tig * 2;
            const int row = m0 + gid;
            *reinterpret_cast<uint32_t *>(dst + (size_t)row * D + col) = pack_h2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<uint32_t *>(dst + (size_t)(row + 8) * D + col) = pack_h2(acc[nt][2], acc[nt][3]);
        }
    }
}

cudaError_t launch_intra(const uint16_t *v, int T, int Nqk, int Nv, int NC, const Workspace &ws,
                         cudaStream_t st)
{
    if (NC == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kIntraSmem);
    if (e != cudaSuccess) return e;
    intra_kernel<<<dim3(NC, Nv), kIntraThreads, kIntraSmem, st>>>(ws.kn, v, T, Nqk, Nv, ws.chunk_info, ws.gcum,
                                                                   ws.betaf, ws.U, ws.W);
    return cudaGetLastError();
}

}  // namespace gdn
