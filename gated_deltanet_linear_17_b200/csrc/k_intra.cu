// Intra-chunk kernel: one CTA per (chunk, v-head), two CTAs per SM.
//
// Page "Qwen3Next Samples", chunk_gated_delta_rule, "Mathematical Formulas":
//   A  = (k_beta k^T) (.) D_decay (.) M_mask      "Pre-Attention Matrix"
//   (I - A)^-1                                     "Matrix Inversion"
//   v_out = (I - A)^-1 (v (.) beta)                "Value and Key Cumulative Decay"
//   k_cumdecay = (I - A)^-1 (k_beta (.) exp(g_cum))
// The page's A (with its negative mask) is the strictly lower matrix
// Ap_ij = -beta_i (kh_i . kh_j) Gamma_ij, j < i.  U = v_out and W = k_cumdecay
// solve (I - Ap) [U | W] = [diag(beta) V | diag(beta e^gamma) Kh].
//
// The solve is blocked on 16-row blocks, as the page's inverse_pto builds the
// inverse from 16-row diagonal blocks: each 16x16 diagonal block is inverted
// by forward substitution, T_ii = (I - Ap_ii)^-1, and then block row by block
// row
//   X_i = T_ii (R_i + sum_{j<i} Ap_ij X_j),
// which is forward substitution with block entries.  The right-hand side is
// 256 columns wide ([V | Kh]); each of the 8 warps owns 32 of those columns and
// runs the whole block recurrence on them by itself, on tensor cores, with no
// CTA-wide barrier inside the solve.  X overwrites R in place.
//
// The raw bf16 k and v rows are staged as they are; K K^T is a bf16 product of
// exact inputs, and the L2 normalisation of k enters as the prologue's fp32
// factors rk, applied to that product and to the right-hand side.  The solve
// itself runs on fp16 operands (the brackets and X overwrite the bf16
// right-hand side in place), with fp32 accumulation; U and W are stored in fp16.
//
// The state-independent factor of the state update ("State Update") is also
// formed here: with k_gexp = Kh (.) exp(g_last - g_cum) (fp16, |entries| <= 1),
//   S_new = e^{g_last} S + k_gexp^T (U - W S) = e^{g_last} S + k_gexp^T U - Mk S,
//   Mk = k_gexp^T W  [Dk x Dk],
// one tcgen05.mma group (M = 128, N = 128, K = 128) on the W half of the
// [U | W] tile as it lies in shared memory after the solve; Mk is stored in
// fp16.  The [V | K] / [U | W] tile is kept as four 64-column blocks of
// 128-byte rows with the 128-byte swizzle, which is the tensor core's MN-major
// operand layout.  The completion wait is bounded; if it gives up, the CTA sets
// bit 2 of status[2] and leaves Mk unwritten.
#include "common.cuh"
#include "gdn_internal.h"
#include "tc100.cuh"

namespace gdn {

constexpr int kIntraThreads = 256;

// shared memory (bytes), relative to a 1024-byte aligned base
constexpr int OFF_RX = 0;                 // [128][256]: bf16 [V | K], then fp16 [U | W]; 4 blocks of 64 columns
constexpr int OFF_AP = 65536;             // fp16 [128][128]: Ap off-diagonal blocks (256-byte rows); then k_gexp
constexpr int OFF_TD = OFF_AP + 32768;    // fp16 8 x [16][16]: T_ii (32-byte rows)
constexpr int OFF_DS = OFF_TD + 4096;     // fp32 8 x [16][16]: per-warp diagonal block scratch
constexpr int OFF_VEC = OFF_DS + 8192;    // fp32 gam[128], bet[128], egam[128], rkv[128]
constexpr int OFF_BAR = OFF_VEC + 4 * 128 * 4;  // mbarrier + TMEM address slot
constexpr int kIntraSmem = OFF_BAR + 64 + 1024;  // + alignment slack

// byte offset of 16-byte chunk c (0..31) of row r in the [128][256] tile: column
// block c / 8 (16 KiB each), 128-byte rows, 16-byte chunks swizzled with r % 8
__device__ __forceinline__ uint32_t sw512(int r, int c)
{
    return (uint32_t)((c >> 3) << 14) + (uint32_t)(r << 7) + (uint32_t)(((c & 7) ^ (r & 7)) << 4);
}

__global__ void __launch_bounds__(kIntraThreads, 2) intra_kernel(
    const uint16_t *__restrict__ k, const uint16_t *__restrict__ v, int T, int Nqk, int Nv,
    const int4 *__restrict__ info, const float *__restrict__ rk, const float *__restrict__ gcum,
    const float *__restrict__ betaf, uint16_t *__restrict__ U, uint16_t *__restrict__ W, uint16_t *__restrict__ Mk,
    float *__restrict__ fa, int32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int c = blockIdx.x, h = blockIdx.y;
    const ChunkInfo ci = load_chunk(info, c);
    if (ci.seq < 0) return;
    const int hq = h / (Nv / Nqk);
    const int n = ci.len, t0 = ci.start;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    const uint32_t rx = smem_addr(smem + OFF_RX), ap = smem_addr(smem + OFF_AP), td = smem_addr(smem + OFF_TD);
    float *gam = reinterpret_cast<float *>(smem + OFF_VEC);
    float *bet = gam + 128, *egam = gam + 256, *rkv = gam + 384;
    const uint32_t bar = smem_addr(smem + OFF_BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 16);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), 128);

    // ---- stage [V | K] (rows past the chunk are zero) with async copies
    for (int e = tid; e < 128 * 32; e += kIntraThreads) {
        const int r = e >> 5, cc = e & 31;
        const bool ok = r < n;
        const int t = t0 + (ok ? r : 0);
        const uint16_t *src = cc < 16 ? v + ((size_t)t * Nv + h) * D + cc * 8
                                      : k + ((size_t)t * Nqk + hq) * D + (cc - 16) * 8;
        cp_async16(rx + sw512(r, cc), src, ok);
    }
    cp_async_commit();
    if (tid < 128) {
        const int i = tid;
        const float gi = gcum[(size_t)h * T + t0 + min(i, n - 1)];
        gam[i] = gi;
        egam[i] = __expf(gi);
        bet[i] = i < n ? betaf[(size_t)h * T + t0 + i] : 0.f;
        rkv[i] = i < n ? rk[(size_t)hq * T + t0 + i] : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    const int m0 = wid * 16;  // this warp's row block in the KK^T step
    // ---- Ap = -strict_tril(diag(beta) Kh Kh^T (.) Gamma), Kh = diag(rk) K, rows of block `wid`
    {
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D; kk += 16) {
            uint32_t a[4];
            {
                const int r = m0 + (lane & 15);
                ldsm_x4(rx + sw512(r, 16 + (kk >> 3) + (lane >> 4)), a[0], a[1], a[2], a[3]);
            }
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                if (np <= wid) {
                    const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(rx + sw512(r, 16 + (kk >> 3) + ((lane >> 3) & 1)), b0, b1, b2, b3);
                    mma16816_bf16(acc[2 * np], a, b0, b1);
                    mma16816_bf16(acc[2 * np + 1], a, b2, b3);
                }
            }
        }
        float *ds = reinterpret_cast<float *>(smem + OFF_DS) + wid * 256;
        uint8_t *aps = smem + OFF_AP;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            if ((nt >> 1) <= wid) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int row = m0 + gid + hf * 8;
                    const int col = nt * 8 + tig * 2;
                    float p0 = 0.f, p1 = 0.f;
                    const float fr = -bet[row] * rkv[row];
                    if (col < row) p0 = fr * rkv[col] * acc[nt][2 * hf] * __expf(gam[row] - gam[col]);
                    if (col + 1 < row) p1 = fr * rkv[col + 1] * acc[nt][2 * hf + 1] * __expf(gam[row] - gam[col + 1]);
                    if ((nt >> 1) < wid) {
                        *reinterpret_cast<uint32_t *>(aps + el256(row, col)) = pack_h2(p0, p1);
                    } else {  // diagonal block: kept in fp32 for the inversion
                        ds[(row - m0) * 16 + (col - m0)] = p0;
                        ds[(row - m0) * 16 + (col - m0) + 1] = p1;
                    }
                }
            }
        }
        __syncwarp();
        // T_ii = (I - Ap_ii)^-1 by forward substitution: lanes 0..15 own one column each
        if (lane < 16) {
            const int cidx = lane;
            float tcol[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float val = (i == cidx) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < i; ++j)
                    if (j >= cidx) val += ds[i * 16 + j] * tcol[j];
                tcol[i] = (i < cidx) ? 0.f : val;
            }
            uint16_t *tdp = reinterpret_cast<uint16_t *>(smem + OFF_TD + wid * 512);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __half hv = __float2half_rn(tcol[i]);
                tdp[i * 16 + cidx] = *reinterpret_cast<uint16_t *>(&hv);
            }
        }
    }
    __syncthreads();

    // ---- block forward substitution on this warp's 32 columns of [V | K]
    {
        const int cb = wid * 4;  // first 16-byte chunk of this warp's 32 columns
        const bool kpart = wid >= 4;
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
            float acc[4][4];
            // R_i scaled by beta (V part) or beta e^gamma rk (K part)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = i * 16 + gid + hf * 8;
                const float f = kpart ? bet[row] * egam[row] * rkv[row] : bet[row];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const uint32_t off = sw512(row, cb + nt) + tig * 4;
                    const uint32_t x = *reinterpret_cast<const uint32_t *>(smem + OFF_RX + off);  // bf16 pair
                    acc[nt][2 * hf] = __uint_as_float(x << 16) * f;
                    acc[nt][2 * hf + 1] = __uint_as_float(x & 0xffff0000u) * f;
                }
            }
            // + sum_{j<i} Ap_ij X_j
            for (int j = 0; j < i; ++j) {
                uint32_t a[4];
                ldsm_x4(a_rowmajor_256(ap, i * 16, j * 16, lane), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int r = j * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(rx + sw512(r, cb + np * 2 + (lane >> 4)), b0, b1, b2, b3);
                    mma16816(acc[2 * np], a, b0, b1);
                    mma16816(acc[2 * np + 1], a, b2, b3);
                }
            }
            // stage the bracket in fp16 over R_i, then X_i = T_ii (bracket)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = i * 16 + gid + hf * 8;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    *reinterpret_cast<uint32_t *>(smem + OFF_RX + sw512(row, cb + nt) + tig * 4) =
                        pack_h2(acc[nt][2 * hf], acc[nt][2 * hf + 1]);
            }
            __syncwarp();
            float x[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
            {
                uint32_t a[4];
                // T_ii, 16 rows of 32 bytes: matrices (rows 0-7 | 8-15) x (cols 0-7 | 8-15)
                const uint32_t ta = td + i * 512 + (lane & 15) * 32 + (lane >> 4) * 16;
                ldsm_x4(ta, a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int r = i * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(rx + sw512(r, cb + np * 2 + (lane >> 4)), b0, b1, b2, b3);
                    mma16816(x[2 * np], a, b0, b1);
                    mma16816(x[2 * np + 1], a, b2, b3);
                }
            }
            __syncwarp();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int row = i * 16 + gid + hf * 8;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    *reinterpret_cast<uint32_t *>(smem + OFF_RX + sw512(row, cb + nt) + tig * 4) =
                        pack_h2(x[nt][2 * hf], x[nt][2 * hf + 1]);
            }
            __syncwarp();
        }
    }
    __syncthreads();

    // ---- reload the raw k rows into the free Ap region: [t][Dk] in two 64-column blocks
    const uint32_t kg = smem_addr(smem + OFF_AP);
    for (int e = tid; e < 128 * 16; e += kIntraThreads) {
        const int r = e >> 4, cc = e & 15;
        const bool ok = r < n;
        cp_async16(kg + sw512(r, cc), k + ((size_t)(t0 + (ok ? r : 0)) * Nqk + hq) * D + cc * 8, ok);
    }
    cp_async_commit();

    // ---- the state pass's per-row factors rk_t e^{g_last - gamma_t} (0 past the chunk) and e^{g_last}
    if (tid < kFaStride) {
        const float gl = gam[127];  // gam is clamped to the last valid row
        fa[(size_t)(c * Nv + h) * kFaStride + tid] =
            tid < 128 ? rkv[tid] * __expf(gl - gam[tid]) : (tid == 128 ? __expf(gl) : 0.f);
    }

    // ---- store [U | W] with 16-byte stores
    const size_t tile = (size_t)(c * Nv + h) * L * D;
    for (int e = tid; e < 128 * 32; e += kIntraThreads) {
        const int r = e >> 5, cc = e & 31;
        const uint4 w = *reinterpret_cast<const uint4 *>(smem + OFF_RX + sw512(r, cc));
        uint16_t *dst = (cc < 16 ? U : W) + tile + (size_t)r * D + (cc & 15) * 8;
        *reinterpret_cast<uint4 *>(dst) = w;
    }

    // ---- k_gexp = fp16(rk e^{g_last - gamma} k) in place (rows past the chunk are zero)
    cp_async_wait<0>();
    __syncthreads();
    {
        const float gl = gam[127];  // gam is clamped to the last valid row
        for (int e = tid; e < 128 * 16; e += kIntraThreads) {
            const int r = e >> 4, cc = e & 15;
            uint4 *p = reinterpret_cast<uint4 *>(smem + OFF_AP + sw512(r, cc));
            const float f = rkv[r] * __expf(gl - gam[r]);
            const uint4 x = *p;
            *p = make_uint4(pack_h2(__uint_as_float(x.x << 16) * f, __uint_as_float(x.x & 0xffff0000u) * f),
                            pack_h2(__uint_as_float(x.y << 16) * f, __uint_as_float(x.y & 0xffff0000u) * f),
                            pack_h2(__uint_as_float(x.z << 16) * f, __uint_as_float(x.z & 0xffff0000u) * f),
                            pack_h2(__uint_as_float(x.w << 16) * f, __uint_as_float(x.w & 0xffff0000u) * f));
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;

    // ---- Mk = k_gexp^T W: A = k_gexp read MN-major (Dk contiguous), B = W (column blocks 2, 3) MN-major
    if (tid == 0) {
        const uint64_t da = tc::desc_mn(kg, 16384, 1024, 2), db = tc::desc_mn(rx + 32768, 16384, 1024, 2);
        const uint32_t idesc = tc::idesc_f16(128, 128, false, false, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16(tmem, da + (uint64_t)((kk * 2048) >> 4), db + (uint64_t)((kk * 2048) >> 4), idesc,
                        kk > 0 ? 1u : 0u);
        tc::commit(bar);
    }
    bool w_ok = true;
    if (tid == 0) w_ok = tc::mbar_wait_bounded(bar, 0);
    tc::fence_before_sync();
    const bool ok = __syncthreads_and(w_ok) != 0;
    tc::fence_after_sync();
    if (ok) {
        // warp w: row 32 (w % 4) + lane of Mk, columns 64 (w / 4) .. +63
        const int quarter = wid & 3, part = wid >> 2;
        const int row = quarter * 32 + lane;
        uint4 *dst = reinterpret_cast<uint4 *>(Mk + tile + (size_t)row * D + part * 64);
        const uint32_t t_row = tmem + ((uint32_t)(quarter * 32) << 16) + part * 64;
#pragma unroll 1
        for (int j0 = 0; j0 < 64; j0 += 32) {
            float a[32];
            tc::tmem_ld32(t_row + j0, a);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                dst[(j0 >> 3) + q8] =
                    make_uint4(pack_h2(a[8 * q8], a[8 * q8 + 1]), pack_h2(a[8 * q8 + 2], a[8 * q8 + 3]),
                               pack_h2(a[8 * q8 + 4], a[8 * q8 + 5]), pack_h2(a[8 * q8 + 6], a[8 * q8 + 7]));
        }
    } else if (tid == 0) {
        atomicOr(status + 2, 4);
        tc::mbar_wait_bounded(bar, 0);  // let the MMAs drain before the tensor memory is released
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, 128);
}

cudaError_t launch_intra(const uint16_t *k, const uint16_t *v, int T, int Nqk, int Nv, int NC, const Workspace &ws,
                         cudaStream_t st)
{
    if (NC == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kIntraSmem);
    if (e != cudaSuccess) return e;
    intra_kernel<<<dim3(NC, Nv), kIntraThreads, kIntraSmem, st>>>(k, v, T, Nqk, Nv, ws.chunk_info, ws.rk, ws.gcum,
                                                                   ws.betaf, ws.U, ws.W, ws.Mk, ws.fa, ws.status);
    return cudaGetLastError();
}

}  // namespace gdn
