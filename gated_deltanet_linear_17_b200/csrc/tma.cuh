// Tensor Memory Accelerator (TMA) helpers for sm_100a: 2-D tiled tensor maps
// encoded on the host, bulk tensor copies global <-> shared memory completing
// on an mbarrier (loads) or a bulk group (stores), and 1-D bulk copies.
// Every copy is issued by one CTA for that CTA alone.
//
// A 2-D map describes `rows` rows of `cols` elements, rows `row_bytes` apart
// (a multiple of 16).  A copy moves a box of box_cols x box_rows elements whose
// first element is at column x, row y; with a 64- or 128-byte swizzle the box
// lands in shared memory as rows of box_cols elements (64 or 128 bytes), 16-byte
// chunk c of row r at chunk c ^ ((r >> 1) & 3) or c ^ (r & 7), which is the
// layout the tensor-core operand descriptors expect.  x * element size must be
// a multiple of 16 bytes.  Rows past the tensor read as zero.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {
namespace tma {

// Host: encode a 2-D tiled tensor map; cudaErrorInvalidValue if the encoder is
// unavailable or rejects the description.
cudaError_t map2d(CUtensorMap *m, CUtensorMapDataType dtype, const void *base, uint64_t cols, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// Host: a 3-D tiled map of rows of `heads` heads of `dim` elements (a [rows][heads][dim] tensor of
// 16-bit elements, row stride heads * dim elements), box of 64 elements x 1 head x box_rows rows with
// the 128-byte swizzle: box (x, head, row) lands as box_rows rows of 64 elements, the layout of one K
// half.  A head narrower than 128 elements reads its second half (x = 64) as zeros past dim.
cudaError_t map_heads(CUtensorMap *m, CUtensorMapDataType dtype, const void *base, uint64_t dim, uint64_t heads,
                      uint64_t rows, uint32_t box_rows);

__device__ __forceinline__ void prefetch_map(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// the mbarrier expects `bytes` more transaction bytes and gets one arrival
__device__ __forceinline__ void expect_tx(uint32_t mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// box at (x, y) of map m -> shared memory at dst; completes `bytes of the box` on mbar
__device__ __forceinline__ void load_2d(uint32_t dst, const CUtensorMap *m, int x, int y, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}

// box at (x, head, y) of a 3-D map (map_heads) -> shared memory at dst; completes on mbar
__device__ __forceinline__ void load_3d(uint32_t dst, const CUtensorMap *m, int x, int head, int y, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(head), "r"(y), "r"(mbar)
        : "memory");
}

// shared memory at src -> box at (x, y) of map m, in the current bulk group
__device__ __forceinline__ void store_2d(const CUtensorMap *m, int x, int y, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}

// contiguous `bytes` (a multiple of 16, both addresses 16-byte aligned) global -> shared, completing on mbar
__device__ __forceinline__ void load_1d(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed store group has finished reading its shared-memory source
__device__ __forceinline__ void wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed store group has completed
__device__ __forceinline__ void wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace tma
}  // namespace gdn
