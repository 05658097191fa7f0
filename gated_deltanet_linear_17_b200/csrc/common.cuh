// Device helpers shared by the Gated Delta Rule kernels (sm_100a).
//
// Shared-memory tiles of bf16 are stored with 16-byte chunks XOR-swizzled by
// row, so that eight ldmatrix row addresses of one 8x8 matrix always land in
// eight different bank groups:
//   256-byte rows (128 bf16): chunk' = chunk ^ (row & 7)
//    64-byte rows ( 32 bf16): chunk' = chunk ^ ((row >> 1) & 3)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gdn_internal.h"

namespace gdn {

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- swizzled tiles

// byte offset of 16-byte chunk `c` of row `r` in a tile with 256-byte rows
__device__ __forceinline__ uint32_t sw256(int r, int c) { return (r << 8) + ((c ^ (r & 7)) << 4); }
// byte offset of 16-byte chunk `c` of row `r` in a tile with 64-byte rows
__device__ __forceinline__ uint32_t sw64(int r, int c) { return (r << 6) + ((c ^ ((r >> 1) & 3)) << 4); }
// byte offset of bf16 element (r, col) in those tiles
__device__ __forceinline__ uint32_t el256(int r, int col) { return sw256(r, col >> 3) + ((col & 7) << 1); }
__device__ __forceinline__ uint32_t el64(int r, int col) { return sw64(r, col >> 3) + ((col & 7) << 1); }

// ---------------------------------------------------------------- async copies

// 16-byte global->shared copy; when !valid the destination is zero-filled and
// nothing is read (src must still be a mapped address, callers pass a base pointer)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid)
{
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}
// 4-byte global->shared copy (always valid)
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- ldmatrix / mma

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D += A(16x16, row) * B(16x8, col), fp16 inputs, fp32 accumulate
__device__ __forceinline__ void mma16816(float *d, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma16816_bf16(float *d, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane addresses for ldmatrix.x4 on a 256-byte-row swizzled tile.
//  A operand, tile holds A[m][k] (k contiguous): 16x16 block at (m0, k0)
__device__ __forceinline__ uint32_t a_rowmajor_256(uint32_t base, int m0, int k0, int lane)
{
    const int r = m0 + (lane & 15);
    const int c = (k0 >> 3) + (lane >> 4);
    return base + sw256(r, c);
}
//  A operand, tile holds A^T[k][m] (m contiguous): 16x16 block at (m0, k0), use ldsm_x4_t
__device__ __forceinline__ uint32_t a_colmajor_256(uint32_t base, int m0, int k0, int lane)
{
    const int mi = lane >> 3;
    const int r = k0 + (lane & 7) + ((mi >> 1) << 3);
    const int c = (m0 >> 3) + (mi & 1);
    return base + sw256(r, c);
}
//  B operand, tile holds B^T[n][k] (k contiguous): n-tiles n0 and n0+8, k block k0; ldsm_x4
//  gives {b0,b1} of n-tile n0 then {b0,b1} of n-tile n0+8
__device__ __forceinline__ uint32_t b_nmajor_256(uint32_t base, int n0, int k0, int lane)
{
    const int r = n0 + (lane & 7) + ((lane >> 4) << 3);
    const int c = (k0 >> 3) + ((lane >> 3) & 1);
    return base + sw256(r, c);
}
//  B operand, tile holds B[k][n] (n contiguous): same fragment order, use ldsm_x4_t
__device__ __forceinline__ uint32_t b_kmajor_256(uint32_t base, int n0, int k0, int lane)
{
    const int r = k0 + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int c = (n0 >> 3) + (lane >> 4);
    return base + sw256(r, c);
}
//  B operand from a 64-byte-row tile B[k][n] (n contiguous, 32 columns), use ldsm_x4_t
__device__ __forceinline__ uint32_t b_kmajor_64(uint32_t base, int n0, int k0, int lane)
{
    const int r = k0 + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int c = (n0 >> 3) + (lane >> 4);
    return base + sw64(r, c);
}

// ---------------------------------------------------------------- conversions

__device__ __forceinline__ float bf2f(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }
__device__ __forceinline__ uint16_t f2bf(float x)
{
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
// two floats -> packed fp16 pair (round to nearest even), low half first
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_h2f(float2 v) { return pack_h2(v.x, v.y); }
__device__ __forceinline__ float2 unpack_h2(uint32_t x)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(&x));
}
// packed bf16 pair -> packed fp16 pair (exact for magnitudes in fp16's normal range)
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t x)
{
    return pack_h2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}

// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of a float2, each an
// IEEE round-to-nearest operation, so the results equal two fmaf / two multiplications).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)),
          "l"(*reinterpret_cast<const uint64_t *>(&c)));
    return *reinterpret_cast<const float2 *>(&d);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
    return *reinterpret_cast<const float2 *>(&d);
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
    return *reinterpret_cast<const float2 *>(&d);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)));
    return *reinterpret_cast<const float2 *>(&d);
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// convert one 16-byte chunk of 8 bf16 values in shared memory to 8 fp16 values in place
__device__ __forceinline__ void bf16_chunk_to_fp16(uint8_t *p)
{
    uint4 w = *reinterpret_cast<const uint4 *>(p);
    w = make_uint4(bf2_to_h2(w.x), bf2_to_h2(w.y), bf2_to_h2(w.z), bf2_to_h2(w.w));
    *reinterpret_cast<uint4 *>(p) = w;
}

// split x into a bf16 pair (hi, lo) with hi + lo = x to ~16 significant bits
__device__ __forceinline__ void split_bf2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf2(x0, x1);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
    lo = pack_bf2(x0 - h0, x1 - h1);
}

// ---------------------------------------------------------------- 16-bit activation types
// The chunked kernels take q, k, v as raw 16-bit rows, bf16 (F16 = false) or fp16 (F16 = true); both
// are exact tensor-core operands of kind::f16, and these helpers widen a packed pair of either type.
template <bool F16>
__device__ __forceinline__ float2 unpack2(uint32_t w)
{
    if constexpr (F16) return unpack_h2(w);
    else return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// split x into a pair (hi, lo) of the 16-bit type with hi + lo = x to about twice its significand
template <bool F16>
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    if constexpr (F16) {
        hi = pack_h2(x0, x1);
        const float2 h = unpack_h2(hi);
        lo = pack_h2(x0 - h.x, x1 - h.y);
    } else {
        split_bf2(x0, x1, hi, lo);
    }
}
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (F16) return pack_h2(lo, hi);
    else return pack_bf2(lo, hi);
}

// chunk table row: sequence, first token, tokens, chunk index within the sequence
struct ChunkInfo {
    int seq, start, len, idx;
};

__device__ __forceinline__ ChunkInfo load_chunk(const int4 *info, int c)
{
    const int4 v = info[c];
    return ChunkInfo{v.x, v.y, v.z, v.w};
}

// Chunk-local cumulative gate ("Gate Cumulative Sum"): gam[i] = sum_{j <= i} g[t0 + j][h]
// over the chunk's n rows; rows i >= n add nothing, so they repeat the last valid
// value.  Every thread of the CTA calls it (it holds barriers); threads 0..127
// produce gam[i]; wsum is 4 floats of shared scratch.  The kernels that need the
// gate all use this function, so they see the same fp32 values bit for bit.
// chunk_gamma_x takes the thread's gate value already loaded (0 for threads from n on and
// from 128 on), so that a kernel can fetch it ahead of time.
__device__ __forceinline__ void chunk_gamma_x(float x, float *gam, float *wsum)
{
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (tid < 128 && lane == 31) wsum[w] = x;
    __syncthreads();
    if (tid < 128) {
        float pre = 0.f;
        for (int j = 0; j < w; ++j) pre += wsum[j];
        gam[tid] = x + pre;
    }
    __syncthreads();
}

__device__ __forceinline__ void chunk_gamma(const float *__restrict__ g, int Nv, int h, int t0, int n, float *gam,
                                            float *wsum)
{
    const int tid = threadIdx.x;
    chunk_gamma_x((g && tid < 128 && tid < n) ? g[(size_t)(t0 + tid) * Nv + h] : 0.f, gam, wsum);  // g null: zero
}

// Largest gate span gamma_first - gamma_last of a 16-row block for which a row's
// decay inside the block is taken as e^{gamma_i - gamma_last} e^{gamma_last - gamma_j}:
// the first factor stays below e^64 and the second above e^-64, both normal fp32.
// Wider spans take e^{gamma_i - gamma_j} element by element.
constexpr float kSpanMax = 64.f;

// Largest finite fp16 magnitude: an fp32 value above it does not fit an fp16 operand tile
// (the kernels record that in status word 3 instead of computing on an infinity silently).
constexpr float kFp16Max = 65504.f;
// max(m, |x|) that keeps a NaN (a NaN operand never fits either), so that
// out_of_fp16(m) also catches NaN and infinite values
__device__ __forceinline__ float absmax_nan(float m, float x)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(fabsf(x)));
    return r;
}
__device__ __forceinline__ bool out_of_fp16(float m) { return !(m <= kFp16Max); }

// d[0..N) = s[0..N) from shared memory in 16-byte loads (s 16-byte aligned).  Loading
// a row's per-column factors into registers ahead of the row's stores keeps the
// loads from being ordered after stores the compiler cannot tell apart from them.
template <int N>
__device__ __forceinline__ void lds_vec(float (&d)[N], const float *s)
{
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 x = reinterpret_cast<const float4 *>(s)[i];
        d[4 * i] = x.x;
        d[4 * i + 1] = x.y;
        d[4 * i + 2] = x.z;
        d[4 * i + 3] = x.w;
    }
}

// 1 / sqrt(|x_r|^2 + eps) for row r of a 128 x 128 16-bit tile of raw bf16 (fp16 with F16) rows
// stored as two 64-column halves of 128-byte rows with the 128-byte swizzle
// ("L2 Normalization", eps inside the square root).  Two adjacent lanes share a
// row (part = lane & 1): part 0 sums the first 64 columns, part 1 the last 64, each
// 16-byte chunk in an order that keeps a quarter-warp on eight distinct bank
// groups, with four partial sums; both lanes get the result.  Same summation
// order in every kernel that calls it.
template <bool F16 = false>
__device__ __forceinline__ float row_inv_norm_pair(const uint8_t *tile, int r, int part, float eps)
{
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int cc = i ^ (part << 2);  // column chunk within the half
        const uint4 x = *reinterpret_cast<const uint4 *>(tile + part * 16384 + r * 128 + ((cc ^ (r & 7)) << 4));
        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 ab = unpack2<F16>(w4[e]);
            s[e] = fmaf(ab.y, ab.y, fmaf(ab.x, ab.x, s[e]));
        }
    }
    float t = (s[0] + s[1]) + (s[2] + s[3]);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    return 1.0f / sqrtf(t + eps);
}

}  // namespace gdn
