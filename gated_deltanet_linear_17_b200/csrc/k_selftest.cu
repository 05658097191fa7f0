// Self-test of the tcgen05 path (test hook, include/gdn_testing.h): one CTA
// computes C[128, N] = sum_k A(m, k) B(n, k) with each operand staged either
// K-major (128-byte swizzle) or MN-major (128-byte swizzle, or 64-byte for
// N = 32), the product accumulated in TMEM and read back with tcgen05.ld --
// the descriptor, swizzle and TMEM conventions that the kernels build on.
#include "common.cuh"
#include "gdn_internal.h"
#include "gdn_testing.h"
#include "tc100.cuh"

namespace gdn {

__global__ void __launch_bounds__(128, 1)
    umma_selftest_kernel(const uint16_t *__restrict__ A, const uint16_t *__restrict__ Bm, float *__restrict__ C,
                         int N, int K, int bf16, int a_mn, int b_mn, int32_t *__restrict__ status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the swizzle atoms need 1024-byte alignment of the shared-memory address itself
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int halves = K / 64;
    uint8_t *sA = smem;
    uint8_t *sB = smem + halves * 128 * 128;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sB + halves * N * 128);
    uint32_t *slot = reinterpret_cast<uint32_t *>(bar + 1);
    const uint32_t ncols = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;

    if (!a_mn) {  // A given as [128][K]
        for (int e = tid; e < 128 * (K / 8); e += 128) {
            const int r = e / (K / 8), c = e % (K / 8);
            *reinterpret_cast<uint4 *>(sA + (c / 8) * 128 * 128 + tc::sw128c(r, c % 8)) =
                *reinterpret_cast<const uint4 *>(A + (size_t)r * K + c * 8);
        }
    } else {      // A given as [K][128]: K rows of two 64-element MN halves
        for (int e = tid; e < K * 16; e += 128) {
            const int r = e / 16, c = e % 16;
            *reinterpret_cast<uint4 *>(sA + (c / 8) * K * 128 + tc::sw128c(r, c % 8)) =
                *reinterpret_cast<const uint4 *>(A + (size_t)r * 128 + c * 8);
        }
    }
    if (!b_mn) {  // B given as [N][K]
        for (int e = tid; e < N * (K / 8); e += 128) {
            const int r = e / (K / 8), c = e % (K / 8);
            *reinterpret_cast<uint4 *>(sB + (c / 8) * N * 128 + tc::sw128c(r, c % 8)) =
                *reinterpret_cast<const uint4 *>(Bm + (size_t)r * K + c * 8);
        }
    } else if (N == 32) {  // B given as [K][32]: 64-byte K rows, 64-byte swizzle
        for (int e = tid; e < K * 4; e += 128) {
            const int r = e / 4, c = e % 4;
            *reinterpret_cast<uint4 *>(sB + sw64(r, c)) = *reinterpret_cast<const uint4 *>(Bm + (size_t)r * 32 + c * 8);
        }
    } else {      // B given as [K][N]: K rows of N/64 MN halves of 128 bytes
        for (int e = tid; e < K * (N / 8); e += 128) {
            const int r = e / (N / 8), c = e % (N / 8);
            *reinterpret_cast<uint4 *>(sB + (c / 8) * K * 128 + tc::sw128c(r, c % 8)) =
                *reinterpret_cast<const uint4 *>(Bm + (size_t)r * N + c * 8);
        }
    }
    if (tid == 0) {
        tc::mbar_init(smem_addr(bar), 1);
        tc::mbar_init_fence();
    }
    if (wid == 0) tc::tmem_alloc(smem_addr(slot), ncols);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *slot;

    if (tid == 0) {
        const uint32_t idesc = tc::idesc_f16(128, N, bf16 != 0, bf16 != 0, a_mn != 0, b_mn != 0);
        const uint32_t a0 = smem_addr(sA), b0 = smem_addr(sB);
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint64_t ad = a_mn ? tc::desc_mn(a0 + kk * 2048, K * 128, 1024, 2)
                                     : tc::desc_k128(a0 + (kk / 4) * 128 * 128 + (kk % 4) * 32);
            const uint64_t bd = !b_mn     ? tc::desc_k128(b0 + (kk / 4) * N * 128 + (kk % 4) * 32)
                                : N == 32 ? tc::desc_mn(b0 + kk * 1024, 0, 512, 4)
                                          : tc::desc_mn(b0 + kk * 2048, K * 128, 1024, 2);
            tc::mma_f16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        tc::commit(smem_addr(bar));
    }
    bool ok = tc::mbar_wait_bounded(smem_addr(bar), 0);
    tc::fence_after_sync();
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tmem + ((uint32_t)(wid * 32) << 16) + c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) C[(size_t)(wid * 32 + lane) * N + c0 + j] = v[j];
        }
    } else {
        if (lane == 0) atomicExch(status, 1);
        tc::mbar_wait_bounded(smem_addr(bar), 0);  // let the MMAs drain before freeing TMEM
    }
    tc::fence_before_sync();
    __syncthreads();
    if (wid == 0) tc::tmem_dealloc(tmem, ncols);
}

// The bounded wait on an mbarrier that (without `arrive`) no one arrives on: it
// gives up after max_polls polls and the thread records that in status word 2.
__global__ void wait_selftest_kernel(uint32_t max_polls, int arrive, int32_t *__restrict__ status)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    tc::mbar_init(b, 1);
    tc::mbar_init_fence();
    if (arrive) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
    if (!tc::mbar_wait_bounded(b, 0, max_polls)) atomicOr(status + 2, GDN_DEV_WAIT_SELFTEST);
}

}  // namespace gdn

extern "C" int gdn_selftest_wait(int32_t max_polls, int32_t arrive, void *workspace, size_t workspace_bytes,
                                 void *stream)
{
    if (!workspace) return GDN_ERR_NULL_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return GDN_ERR_ALIGNMENT;
    if (workspace_bytes < 16) return GDN_ERR_WORKSPACE;
    if (max_polls < 1 || max_polls > (1 << 22)) return GDN_ERR_BAD_SHAPE;
    gdn::wait_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((uint32_t)max_polls, arrive,
                                                                 static_cast<int32_t *>(workspace));
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" int gdn_selftest_umma(const uint16_t *A, const uint16_t *B, float *C, int32_t N, int32_t K,
                                 int32_t bf16, int32_t a_mn, int32_t b_mn, int32_t *status, void *stream)
{
    if (!A || !B || !C || !status) return GDN_ERR_NULL_ARG;
    if (!(N == 32 || N == 64 || N == 128 || N == 256) || !(K == 64 || K == 128)) return GDN_ERR_BAD_SHAPE;
    const int smem = (K / 64) * (128 + N) * 128 + 64 + 1024;
    cudaError_t e = cudaFuncSetAttribute(gdn::umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    gdn::umma_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(A, B, C, N, K, bf16, a_mn, b_mn, status);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
