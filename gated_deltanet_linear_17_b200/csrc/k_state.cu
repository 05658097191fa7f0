// Inter-chunk state passing on the Blackwell tensor core: one CTA (8 warps) per
// (sequence, v-head, 32-column slice of Dv).
//
// Page "Qwen3Next Samples", "Recurrent State Attention" and "State Update",
// with the state held as S[Dk, Dv]:
//   v'    = k_cumdecay S                 -> U' = U - W S
//   S_new = S exp(g_last) + k_gexp^T (v_out - v'),  k_gexp = kh (.) exp(g_last - g_cum)
// g_last is the cumulative gate at the chunk's last valid token.  The CTA walks
// its sequence's chunks in order.  Warp w owns rows 32(w%4)..32(w%4)+31 and
// columns 16(w/4)..16(w/4)+15 of the slice: each thread keeps 16 fp32 values of
// one row of the state S in registers for the whole sequence, and handles the
// same 16 values of one row of U'.  Per chunk:
//   1. W S     -- tcgen05.mma M=128 (L), N=32, K=128 (Dk), fp16: A = W
//                 (K-major), B = S (MN-major, as the threads store it); fp32
//                 accumulator in TMEM.
//   2. U' = U - W S (tcgen05.ld), written to Up; the decayed operand
//      Ub = diag(rk e^{g_last - gamma}) U' is split into bf16 hi + lo (~16
//      significant bits) and stored row-wise (MN-major).
//   3. K^T Ub  -- tcgen05.mma M=128 (Dk), N=32, K=128 (L), bf16: A = the raw k
//                 tile read MN-major (no transpose), B = Ub hi then lo, both
//                 accumulated into a second TMEM tile.
//   4. S = e^{g_last} S + K^T Ub (tcgen05.ld); S in fp16 becomes the next B
//      operand and, as the state entering the next chunk, goes to Sc.
// The next chunk's W, k, U, gamma and 1/|k| are prefetched with cp.async while
// the W S product runs, and each product is split into independent
// accumulation chains (partial sums over halves of K, and the hi / lo halves of
// Ub) that are added after one TMEM read, to shorten the serial chain.  One
// thread issues the MMAs and waits for their completion (an mbarrier arrival
// from tcgen05.commit); a CTA barrier passes the outcome on.  Every wait is
// bounded: if one gives up, the CTA sets bit 0 of status[2] in the workspace,
// stops, lets its MMAs drain and frees its tensor memory.
#include "common.cuh"
#include "gdn_internal.h"
#include "tc100.cuh"

namespace gdn {

constexpr int kStateThreads = 256;
constexpr int DVT = 32;  // Dv columns per CTA

// shared memory, relative to a 1024-byte aligned base (bytes)
constexpr int ST_W = 0;             // fp16 W, K-major over Dk, 128B swizzle: 2 halves x 128 rows x 128 B
constexpr int ST_K = 32768;         // bf16 k, MN-major over Dk (K rows = L), 128B swizzle: 2 halves x 128 x 128 B
constexpr int ST_U = 65536;         // fp16 U slice [L][32], 64-byte rows, 64B swizzle
constexpr int ST_G = 73728;         // fp32 gamma[128]
constexpr int ST_R = 74240;         // fp32 1/|k| [128]
constexpr int kStageBytes = 75776;  // rounded up to a multiple of 1024
constexpr int OFF_S = 2 * kStageBytes;  // fp16 S [Dk][32], MN-major, 64B swizzle
constexpr int OFF_UH = OFF_S + 8192;    // bf16 Ub high half [L][32], MN-major, 64B swizzle
constexpr int OFF_UL = OFF_UH + 8192;   // bf16 Ub low half
constexpr int OFF_BAR = OFF_UL + 8192;  // 2 mbarriers + TMEM address slot
constexpr int kStateSmem = OFF_BAR + 64 + 1024;  // + alignment slack

__global__ void __launch_bounds__(kStateThreads, 1) state_kernel(
    const uint16_t *__restrict__ k, const float *__restrict__ pool, const int32_t *__restrict__ idx,
    float *__restrict__ final_state, int T, int Nqk, int Nv, const int4 *__restrict__ info,
    const int32_t *__restrict__ seq_chunk0, const float *__restrict__ rk, const float *__restrict__ gcum,
    const uint16_t *__restrict__ U, const uint16_t *__restrict__ W, uint16_t *__restrict__ Up,
    uint16_t *__restrict__ Sc, int32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_addr(smem);
    const int b = blockIdx.x, h = blockIdx.y, col0 = blockIdx.z * DVT;
    const int hq = h / (Nv / Nqk);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int quarter = wid & 3, half = wid >> 2;
    const int row = quarter * 32 + lane;  // row of the state (Dk) and of U' (L)
    const int cbase = half * 16;          // first of this thread's 16 columns in the slice
    const int c_begin = seq_chunk0[b], c_end = seq_chunk0[b + 1];
    const int seq_t0 = c_begin < c_end ? info[c_begin].y : 0;
    const int seq_t1 = c_begin < c_end ? info[c_end - 1].y + info[c_end - 1].z : 0;

    const uint32_t bar_ws = sbase + OFF_BAR, bar_up = sbase + OFF_BAR + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 16);
    if (tid == 0) {
        tc::mbar_init(bar_ws, 1);
        tc::mbar_init(bar_up, 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(tslot), 256);

    // initial state: this thread's 16 values
    float s[16];
    if (pool) {
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
    // S in fp16 as the MN-major B operand: row `row`, 16-byte chunks (cbase/8, cbase/8 + 1)
    auto store_state_operand = [&]() {
#pragma unroll
        for (int j = 0; j < 2; ++j)
            *reinterpret_cast<uint4 *>(smem + OFF_S + sw64(row, (cbase >> 3) + j)) =
                make_uint4(pack_h2(s[8 * j], s[8 * j + 1]), pack_h2(s[8 * j + 2], s[8 * j + 3]),
                           pack_h2(s[8 * j + 4], s[8 * j + 5]), pack_h2(s[8 * j + 6], s[8 * j + 7]));
    };
    store_state_operand();

    // per-thread constant parts of the prefetch addresses
    const int wr = tid >> 4, wc = tid & 15;  // W / k pieces: rows wr + 16 j, chunk wc
    const uint32_t w_dst = (uint32_t)((wc >> 3) * 16384) + tc::sw128c(wr, wc & 7);
    const int ur = tid >> 2, uc = tid & 3;   // U pieces: rows ur + 64 j, chunk uc
    const uint32_t u_dst = sw64(ur, uc);
    auto issue = [&](int c, int st) {
        const int cstart = seq_t0 + (c - c_begin) * L, clen = min(L, seq_t1 - cstart);
        const uint32_t base = sbase + st * kStageBytes;
        const uint16_t *wsrc = W + (size_t)(c * Nv + h) * L * D + wr * D + wc * 8;
        const uint16_t *ksrc = k + ((size_t)cstart * Nqk + hq) * D + wc * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = wr + 16 * j;
            cp_async16(base + ST_W + w_dst + j * 2048, wsrc + (size_t)j * 16 * D, true);
            const bool valid = r < clen;
            cp_async16(base + ST_K + w_dst + j * 2048, ksrc + (size_t)(valid ? r : 0) * Nqk * D, valid);
        }
        const uint16_t *usrc = U + (size_t)(c * Nv + h) * L * D + col0 + ur * D + uc * 8;
#pragma unroll
        for (int j = 0; j < 2; ++j) cp_async16(base + ST_U + u_dst + j * 4096, usrc + (size_t)j * 64 * D, true);
        if (tid < 128) {
            // gamma (clamped to the last valid row) and 1/|k|; rows past the chunk multiply zeros
            const int i = min(tid, clen - 1);
            cp_async4(base + ST_G + tid * 4, gcum + (size_t)h * T + cstart + i);
            cp_async4(base + ST_R + tid * 4, rk + (size_t)hq * T + cstart + i);
        }
    };

    if (c_begin < c_end) issue(c_begin, 0);
    cp_async_commit();
    cp_async_wait<0>();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // TMEM columns: [0, 64) W S as two partial sums over the Dk halves;
    // [64, 192) K^T Ub as four partial sums (L half x hi / lo)
    const uint32_t tmem = *tslot;
    const uint32_t t_mine = tmem + ((uint32_t)(quarter * 32) << 16) + cbase;
    const uint32_t idesc_ws = tc::idesc_f16(128, 32, false, false, false, true);
    const uint32_t idesc_up = tc::idesc_f16(128, 32, true, true, true, true);
    // Operand descriptors of k step 0 of each tile; the start-address field holds
    // (byte address >> 4) and every address stays below 256 KiB, so the
    // descriptor of a k step is the base descriptor plus (byte offset >> 4).
    const uint64_t dW0 = tc::desc_k128(sbase + ST_W), dK0 = tc::desc_mn(sbase + ST_K, 16384, 1024, 2);
    const uint64_t dS = tc::desc_mn(sbase + OFF_S, 0, 512, 4);
    const uint64_t dUH = tc::desc_mn(sbase + OFF_UH, 0, 512, 4), dUL = tc::desc_mn(sbase + OFF_UL, 0, 512, 4);
    bool ok = true;

    // Each iteration starts with the chunk's data and the state operand in
    // shared memory (made visible to the tensor core before the barrier at the
    // end of the previous iteration).
    for (int c = c_begin, it = 0; c < c_end; ++c, ++it) {
        const int st = it & 1;
        const uint32_t parity = (uint32_t)(it & 1);
        const int clen = min(L, seq_t1 - (seq_t0 + (c - c_begin) * L));
        uint8_t *base = smem + st * kStageBytes;
        const float *gam = reinterpret_cast<const float *>(base + ST_G);
        const float *rkv = reinterpret_cast<const float *>(base + ST_R);
        const size_t tile = (size_t)(c * Nv + h) * L * D;

        const uint64_t stage_off = (uint64_t)((st * kStageBytes) >> 4);
        // (1) W S: two independent accumulation chains (Dk halves)
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                tc::mma_f16(tmem + (kk >> 2) * 32, dW0 + stage_off + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                            dS + (uint64_t)((kk * 1024) >> 4), idesc_ws, (kk & 3) ? 1u : 0u);
            tc::commit(bar_ws);
        }
        // while it runs: prefetch the next chunk, write the entering state, read U and the row factor
        if (c + 1 < c_end) issue(c + 1, st ^ 1);
        cp_async_commit();
        {
            uint4 *dst = reinterpret_cast<uint4 *>(Sc + tile + (size_t)row * D + col0 + cbase);
#pragma unroll
            for (int j = 0; j < 2; ++j)
                dst[j] = make_uint4(pack_h2(s[8 * j], s[8 * j + 1]), pack_h2(s[8 * j + 2], s[8 * j + 3]),
                                    pack_h2(s[8 * j + 4], s[8 * j + 5]), pack_h2(s[8 * j + 6], s[8 * j + 7]));
        }
        const float gl = gam[clen - 1];
        const float sc = rkv[row] * __expf(gl - gam[row]);
        const float dg = __expf(gl);
        uint4 uu[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) uu[j] = *reinterpret_cast<const uint4 *>(base + ST_U + sw64(row, (cbase >> 3) + j));
        {
            bool w_ok = true;
            if (tid == 0) w_ok = tc::mbar_wait_bounded(bar_ws, parity);
            tc::fence_before_sync();
            ok = __syncthreads_and(w_ok) != 0;
            tc::fence_after_sync();
        }
        if (!ok) break;

        // (2) U' = U - W S -> Up; Ub hi / lo
        {
            float ws[16], ws2[16];
            tc::tmem_ld16(t_mine, ws);
            tc::tmem_ld16(t_mine + 32, ws2);
            uint4 *updst = reinterpret_cast<uint4 *>(Up + tile + (size_t)row * D + col0 + cbase);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t w4[4] = {uu[j].x, uu[j].y, uu[j].z, uu[j].w};
                uint32_t o4[4], h4[4], l4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 u = unpack_h2(w4[e]);
                    const int i0 = 8 * j + 2 * e;
                    const float p0 = u.x - (ws[i0] + ws2[i0]), p1 = u.y - (ws[i0 + 1] + ws2[i0 + 1]);
                    o4[e] = pack_h2(p0, p1);
                    split_bf2(p0 * sc, p1 * sc, h4[e], l4[e]);
                }
                updst[j] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                *reinterpret_cast<uint4 *>(smem + OFF_UH + sw64(row, (cbase >> 3) + j)) =
                    make_uint4(h4[0], h4[1], h4[2], h4[3]);
                *reinterpret_cast<uint4 *>(smem + OFF_UL + sw64(row, (cbase >> 3) + j)) =
                    make_uint4(l4[0], l4[1], l4[2], l4[3]);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();

        // (3) K^T (Ub_hi + Ub_lo): four independent chains (L half x hi / lo)
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t ad = dK0 + stage_off + (uint64_t)((kk * 2048) >> 4);
                const uint32_t acc = (kk & 3) ? 1u : 0u;
                tc::mma_f16(tmem + 64 + (kk >> 2) * 32, ad, dUH + (uint64_t)((kk * 1024) >> 4), idesc_up, acc);
                tc::mma_f16(tmem + 128 + (kk >> 2) * 32, ad, dUL + (uint64_t)((kk * 1024) >> 4), idesc_up, acc);
            }
            tc::commit(bar_up);
        }
        {
            bool w_ok = true;
            if (tid == 0) w_ok = tc::mbar_wait_bounded(bar_up, parity);
            tc::fence_before_sync();
            ok = __syncthreads_and(w_ok) != 0;
            tc::fence_after_sync();
        }
        if (!ok) break;

        // (4) S = e^{g_last} S + K^T Ub; the next chunk's B operand
        {
            float p0[16], p1[16], p2[16], p3[16];
            tc::tmem_ld16(t_mine + 64, p0);
            tc::tmem_ld16(t_mine + 96, p1);
            tc::tmem_ld16(t_mine + 128, p2);
            tc::tmem_ld16(t_mine + 160, p3);
#pragma unroll
            for (int j = 0; j < 16; ++j) s[j] = dg * s[j] + ((p0[j] + p1[j]) + (p2[j] + p3[j]));
        }
        store_state_operand();
        cp_async_wait<0>();  // the next chunk's data
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }
    cp_async_wait<0>();

    if (!ok) {
        if (tid == 0) {
            atomicOr(status + 2, 1);
            // give the MMAs already issued time to finish before the tensor memory is released
            tc::mbar_wait_bounded(bar_ws, 0);
            tc::mbar_wait_bounded(bar_up, 0);
        }
    } else if (final_state) {
        float4 *dst =
            reinterpret_cast<float4 *>(final_state + (((size_t)b * Nv + h) * D + row) * D + col0 + cbase);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (wid == 0) tc::tmem_dealloc(tmem, 256);
}

cudaError_t launch_state(const uint16_t *k, const float *pool, const int32_t *idx, float *final_state, int T, int B,
                         int Nqk, int Nv, const Workspace &ws, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStateSmem);
    if (e != cudaSuccess) return e;
    state_kernel<<<dim3(B, Nv, D / DVT), kStateThreads, kStateSmem, st>>>(
        k, pool, idx, final_state, T, Nqk, Nv, ws.chunk_info, ws.seq_chunk0, ws.rk, ws.gcum, ws.U, ws.W, ws.Up,
        ws.Sc, ws.status);
    return cudaGetLastError();
}

}  // namespace gdn
