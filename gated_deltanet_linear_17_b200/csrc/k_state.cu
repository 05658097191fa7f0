// Inter-chunk state passing on the Blackwell tensor core: one CTA per
// (sequence, v-head, 32-column slice of Dv), 8 epilogue warps, one warp that
// issues the tensor-core work and one that moves data with TMA.
//
// Page "Qwen3Next Samples", "Recurrent State Attention" and "State Update",
// with the state held as S[Dk, Dv]:
//   v'    = k_cumdecay S
//   S_new = S exp(g_last) + k_gexp^T (v_out - v'),  k_gexp = kh (.) exp(g_last - g_cum)
// regrouped as
//   S_new = e^{g_last} S + Kt - Mk S,   Kt = k_gexp^T U,  Mk = k_gexp^T W.
// Mk and the row factors f_t = rk_t e^{g_last - gamma_t} come from the
// intra-chunk kernel.  Only Mk S depends on the state, so the serial chain over
// a sequence's chunks is one product per chunk; Kt of the next chunk runs on
// the tensor core while the current chunk's state update runs on the cores.
// Warp w < 8 owns rows 32(w%4)..32(w%4)+31 and 16 columns (w/4) of the slice:
// each of its threads keeps 16 fp32 values of one row of S in registers for the
// whole sequence.  Per chunk c:
//   issue warp: Mk S_c (tcgen05.mma M=128, N=32, K=128, fp16; A = Mk K-major,
//               B = S_c MN-major as the threads store it; two accumulation
//               chains over the halves of K), committed to an mbarrier; then,
//               once the epilogue warps have staged its operand, Kt of chunk
//               c+1 = K^T Ub (M=128, N=64, K=128, bf16; A = the raw k tile read
//               MN-major, B = [Ub_hi | Ub_lo]) into one of two TMEM buffers.
//   data warp:  a TMA store of S_c (fp16) to Sc; once Mk S_c has completed, TMA
//               loads of chunk c+2 (Mk, the raw k rows, the U slice and the
//               factors) into the freed stage.
//   epilogue:   Ub = diag(f) U of chunk c+1 split into bf16 hi + lo (~16
//               significant bits; k is exact in bf16); wait for Mk S_c (its
//               commit also covers Kt of chunk c, issued before it);
//               S_{c+1} = e^{g_last} S_c + Kt_c - Mk S_c, whose fp16 copy is the
//               next B operand (two buffers, so the TMA store of S_c can still
//               be reading the other).
// The k rows of a chunk that ends before 128 tokens are zeroed after their TMA
// load, so the next sequence's rows never enter a product.  Every wait is
// bounded: if one gives up, the CTA sets bit 0 of status[2] in the workspace,
// stops, lets its copies and MMAs drain and frees its tensor memory.
#include "common.cuh"
#include "gdn_internal.h"
#include "tc100.cuh"
#include "tma.cuh"

namespace gdn {

constexpr int kStateThreads = 320;  // 8 epilogue warps, the issue warp, the data warp
constexpr int DVT = 32;             // Dv columns per CTA

// shared memory, relative to a 1024-byte aligned base (bytes); two stages
constexpr int SG_MK = 0;            // fp16 Mk, K-major (rows Dk, K = Dk), 128B swizzle: 2 halves x 128 x 128 B
constexpr int SG_K = 32768;         // bf16 k [L][Dk] in two 64-column blocks, 128B swizzle (MN-major A = k^T)
constexpr int SG_U = 65536;         // fp16 U slice [L][32], 64B swizzle
constexpr int SG_F = 73728;         // fp32 factors: f_t (t < 128), e^{g_last} at 128
constexpr int kStage = 74752;       // a multiple of 1024
constexpr uint32_t kStageTx = 32768 + 32768 + 8192 + kFaStride * 4;  // bytes per stage fill
constexpr int OFF_S = 2 * kStage;        // 2 x fp16 S [Dk][32], MN-major, 64B swizzle
constexpr int OFF_UB = OFF_S + 16384;    // 2 x bf16 [L][64] = [Ub_hi | Ub_lo], MN-major, 128B swizzle
constexpr int OFF_BAR = OFF_UB + 32768;  // full[2], chain, drain mbarriers; TMEM address slot
constexpr int kStateSmem = OFF_BAR + 64 + 1024;  // + alignment slack
constexpr int kTmemCols = 256;  // [0, 64) Mk S (two chains), [64, 192) Kt (two buffers)

// named barrier 1: the epilogue warps arrive once Ub is staged, the issue warp waits
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void named_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// bounded mbarrier wait by lane 0 of the warp, outcome shared with the warp
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane)
{
    bool w = true;
    if (lane == 0) w = tc::mbar_wait_bounded(bar, parity);
    return __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
}

__global__ void __launch_bounds__(kStateThreads, 1) state_kernel(
    const __grid_constant__ CUtensorMap tm_mk, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_sc,
    const float *__restrict__ pool, const int32_t *__restrict__ idx, float *__restrict__ final_state, int Nqk,
    int Nv, const int4 *__restrict__ info, const int32_t *__restrict__ seq_chunk0, const float *__restrict__ fa,
    int32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int b = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * DVT;
    const int hq = h / (Nv / Nqk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const bool issuer = wid == 8, producer = wid == 9, epi = wid < 8;
    const int quarter = wid & 3, half = (wid >> 2) & 1;
    const int row = quarter * 32 + lane;  // row of the state (Dk) and of Ub (L)
    const int cbase = half * 16;          // first of this thread's 16 columns in the slice
    const int c_begin = seq_chunk0[b], c_end = seq_chunk0[b + 1];
    const int seq_t0 = c_begin < c_end ? info[c_begin].y : 0;
    const int seq_t1 = c_begin < c_end ? info[c_end - 1].y + info[c_end - 1].z : 0;
    auto chunk_len = [&](int c) { return min(L, seq_t1 - (seq_t0 + (c - c_begin) * L)); };

    const uint32_t bar_full = sbase + OFF_BAR;  // + 8 s: stage s holds its chunk
    const uint32_t bar_m = sbase + OFF_BAR + 16, bar_d = sbase + OFF_BAR + 24;  // chain product; drain on error
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 32);
    if (tid == 0) {
        tc::mbar_init(bar_full, 1);
        tc::mbar_init(bar_full + 8, 1);
        tc::mbar_init(bar_m, 1);
        tc::mbar_init(bar_d, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), kTmemCols);
    __syncthreads();

    // TMA fill of stage st with chunk c (data lane)
    int fills[2] = {0, 0};
    auto fill = [&](int c, int st) {
        const uint32_t base = sbase + st * kStage, full = bar_full + 8 * st;
        const int trow = (c * Nv + h) * L;  // first row of the chunk's tiles in the workspace
        const int cstart = seq_t0 + (c - c_begin) * L;
        tma::expect_tx(full, kStageTx);
        tma::load_2d(base + SG_MK, &tm_mk, 0, trow, full);
        tma::load_2d(base + SG_MK + 16384, &tm_mk, 64, trow, full);
        tma::load_2d(base + SG_K, &tm_k, hq * D, cstart, full);
        tma::load_2d(base + SG_K + 16384, &tm_k, hq * D + 64, cstart, full);
        tma::load_2d(base + SG_U, &tm_u, col0, trow, full);
        tma::load_1d(base + SG_F, fa + (size_t)(c * Nv + h) * kFaStride, kFaStride * 4, full);
        ++fills[st];
    };
    // After stage st has landed with chunk c (epilogue warps): zero the k rows
    // past a short chunk, and stage Ub = diag(f) U, hi and lo, in Ub buffer st.
    auto stage_ub = [&](int c, int st) {
        uint8_t *base = smem + st * kStage;
        const int clen = chunk_len(c);
        if (clen < L) {
            for (int e = tid; e < (L - clen) * 16; e += 256) {  // 2 blocks x 8 chunks per row
                const int r = clen + (e >> 4), blk = (e >> 3) & 1, cc = e & 7;
                *reinterpret_cast<uint4 *>(base + SG_K + blk * 16384 + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        const float f = reinterpret_cast<const float *>(base + SG_F)[row];
        uint8_t *dst = smem + OFF_UB + st * 16384;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 x = *reinterpret_cast<const uint4 *>(base + SG_U + sw64(row, (cbase >> 3) + j));
            const uint32_t x4[4] = {x.x, x.y, x.z, x.w};
            uint32_t h4[4], l4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 u = unpack_h2(x4[e]);
                split_bf2(u.x * f, u.y * f, h4[e], l4[e]);
            }
            *reinterpret_cast<uint4 *>(dst + tc::sw128c(row, (cbase >> 3) + j)) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            *reinterpret_cast<uint4 *>(dst + tc::sw128c(row, 4 + (cbase >> 3) + j)) =
                make_uint4(l4[0], l4[1], l4[2], l4[3]);
        }
        return reinterpret_cast<const float *>(base + SG_F)[128];  // e^{g_last}
    };

    // initial state: this thread's 16 values
    float s[16];
    if (epi && pool) {
        const int slot = idx ? idx[b] : b;
        const float4 *src =
            reinterpret_cast<const float4 *>(pool + (((size_t)slot * Nv + h) * D + row) * D + col0 + cbase);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 x = src[j];
            s[4 * j] = x.x;
            s[4 * j + 1] = x.y;
            s[4 * j + 2] = x.z;
            s[4 * j + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) s[j] = 0.f;
    }
    auto pack8 = [](const float *x) {
        return make_uint4(pack_h2(x[0], x[1]), pack_h2(x[2], x[3]), pack_h2(x[4], x[5]), pack_h2(x[6], x[7]));
    };
    // S in fp16 as the MN-major B operand (buffer buf): row `row`, 16-byte chunks (cbase/8, cbase/8 + 1)
    auto store_state_operand = [&](int buf) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
            *reinterpret_cast<uint4 *>(smem + OFF_S + buf * 8192 + sw64(row, (cbase >> 3) + j)) = pack8(s + 8 * j);
    };

    bool ok = true;
    float dg = 1.f;  // e^{g_last} of the chunk in flight (epilogue warps)
    if (producer) {
        if (lane == 0) {
            tma::prefetch_map(&tm_mk);
            tma::prefetch_map(&tm_k);
            tma::prefetch_map(&tm_u);
            tma::prefetch_map(&tm_sc);
            if (c_begin < c_end) fill(c_begin, 0);
            if (c_begin + 1 < c_end) fill(c_begin + 1, 1);
        }
    } else if (epi) {
        store_state_operand(0);
        if (c_begin < c_end) {
            ok = warp_wait(bar_full, 0, lane);
            dg = stage_ub(c_begin, 0);
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    ok = __syncthreads_and(ok) != 0;
    tc::fence_after_sync();

    const uint32_t tmem = *tslot;
    const uint32_t t_mine = tmem + ((uint32_t)(quarter * 32) << 16) + cbase;
    const uint32_t idesc_m = tc::idesc_f16(128, 32, false, false, false, true);
    const uint32_t idesc_k = tc::idesc_f16(128, 64, true, true, true, true);
    // Operand descriptors of k step 0; the start-address field holds (byte
    // address >> 4) and every address stays below 256 KiB, so the descriptor
    // of a k step is the base descriptor plus (byte offset >> 4).
    const uint64_t dMk0 = tc::desc_k128(sbase + SG_MK), dK0 = tc::desc_mn(sbase + SG_K, 16384, 1024, 2);
    const uint64_t dS0 = tc::desc_mn(sbase + OFF_S, 0, 512, 4);
    const uint64_t dUb0 = tc::desc_mn(sbase + OFF_UB, 16384, 1024, 2);
    // Kt of the chunk in stage st into TMEM buffer st, from Ub buffer st (issue lane)
    auto issue_kt = [&](int st) {
        const uint64_t so = (uint64_t)((st * kStage) >> 4), uo = (uint64_t)((st * 16384) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16(tmem + 64 + st * 64, dK0 + so + (uint64_t)((kk * 2048) >> 4),
                        dUb0 + uo + (uint64_t)((kk * 2048) >> 4), idesc_k, kk > 0 ? 1u : 0u);
    };
    bool issued = false;  // issue lane: any MMA in flight

    for (int c = c_begin, it = 0; ok && c < c_end; ++c, ++it) {
        const int st = it & 1;
        const bool has_next = c + 1 < c_end;
        if (issuer) {
            if (lane == 0) {
                if (it == 0) issue_kt(0);  // the first chunk's Kt, before its chain product
                const uint64_t so = (uint64_t)((st * kStage) >> 4), sb = (uint64_t)((st * 8192) >> 4);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16(tmem + (kk >> 2) * 32, dMk0 + so + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                dS0 + sb + (uint64_t)((kk * 1024) >> 4), idesc_m, (kk & 3) ? 1u : 0u);
                tc::commit(bar_m);
                issued = true;
            }
            __syncwarp();
            if (has_next) {
                named_sync(1, 288);  // Ub of chunk c + 1 is staged
                if (lane == 0) issue_kt(st ^ 1);
                __syncwarp();
            }
        } else if (producer) {
            bool w_ok = true;
            if (lane == 0) {
                // the state entering chunk c, from its operand copy
                tma::store_2d(&tm_sc, col0, (c * Nv + h) * L, sbase + OFF_S + st * 8192);
                tma::commit_group();
                // stage st is free once Mk S_c (and Kt_c before it) has completed
                w_ok = tc::mbar_wait_bounded(bar_m, (uint32_t)(it & 1));
                if (w_ok && c + 2 < c_end) fill(c + 2, st);
                tma::wait_read_all();  // the store of S_c has read its buffer
            }
            ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0;
        } else {  // epilogue warps
            float dg_next = 1.f;
            if (has_next) {
                const bool f_ok = warp_wait(bar_full + 8 * (st ^ 1), (uint32_t)(((it + 1) >> 1) & 1), lane);
                ok = ok && f_ok;
                dg_next = stage_ub(c + 1, st ^ 1);
                tc::fence_proxy_async();
                named_arrive(1, 288);
            }
            const bool m_ok = warp_wait(bar_m, (uint32_t)(it & 1), lane);
            tc::fence_after_sync();
            ok = ok && m_ok;
            float p0[16], p1[16], n0[16], n1[16];
            tc::tmem_ld16(t_mine, p0);
            tc::tmem_ld16(t_mine + 32, p1);
            tc::tmem_ld16(t_mine + 64 + st * 64, n0);
            tc::tmem_ld16(t_mine + 64 + st * 64 + 32, n1);
#pragma unroll
            for (int j = 0; j < 16; ++j) s[j] = dg * s[j] + ((n0[j] + n1[j]) - (p0[j] + p1[j]));
            store_state_operand(st ^ 1);
            tc::fence_proxy_async();
            dg = dg_next;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(ok) != 0;
        tc::fence_after_sync();
    }

    // copies and MMAs still in flight land before shared and tensor memory are released
    if (producer && lane == 0) {
        for (int st = 0; st < 2; ++st)
            if (fills[st] > 0) tc::mbar_wait_bounded(bar_full + 8 * st, (uint32_t)((fills[st] - 1) & 1));
        tma::wait_read_all();  // the stores have read shared memory (the grid's end publishes them)
    }
    if (issuer && lane == 0 && !ok && issued) {  // a commit covers every MMA issued before it
        tc::commit(bar_d);
        tc::mbar_wait_bounded(bar_d, 0);
    }
    if (!ok) {
        if (tid == 0) atomicOr(status + 2, 1);
    } else if (final_state && epi) {
        float4 *dst =
            reinterpret_cast<float4 *>(final_state + (((size_t)b * Nv + h) * D + row) * D + col0 + cbase);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_state(const uint16_t *k, const float *pool, const int32_t *idx, float *final_state, int T, int B,
                         int Nqk, int Nv, const Workspace &ws, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    // tile rows of the workspace tensors; TMA coordinates are 32-bit signed
    const uint64_t trows = (uint64_t)ws.NC * Nv * L;
    if (trows >= (1ull << 31) || (uint64_t)T >= (1ull << 31)) return cudaErrorInvalidValue;
    const uint64_t rows = trows > 0 ? trows : 1;
    CUtensorMap m_mk, m_k, m_u, m_sc;
    cudaError_t e = tma::map2d(&m_mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.Mk, D, rows, D * 2, 64, 128,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess) {
        if (T > 0)
            e = tma::map2d(&m_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, (uint64_t)Nqk * D, (uint64_t)T,
                           (uint64_t)Nqk * D * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
        else  // no chunk exists, so the map is never used
            e = tma::map2d(&m_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws.Mk, D, rows, D * 2, 64, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (e == cudaSuccess)
        e = tma::map2d(&m_u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.U, D, rows, D * 2, DVT, 128,
                       CU_TENSOR_MAP_SWIZZLE_64B);
    if (e == cudaSuccess)
        e = tma::map2d(&m_sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.Sc, D, rows, D * 2, DVT, 128,
                       CU_TENSOR_MAP_SWIZZLE_64B);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmem);
    if (e != cudaSuccess) return e;
    state_kernel<<<dim3(B, Nv, D / DVT), kStateThreads, kStateSmem, st>>>(
        m_mk, m_k, m_u, m_sc, pool, idx, final_state, Nqk, Nv, ws.chunk_info, ws.seq_chunk0, ws.fa, ws.status);
    return cudaGetLastError();
}

}  // namespace gdn
