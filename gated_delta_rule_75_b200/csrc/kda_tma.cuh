// TMA (cp.async.bulk.tensor) helpers and host-side tensor-map encoding.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {
namespace tma {

// 2-D tiled load of a box at (x = innermost element index, y = row) into
// shared memory; completion is signalled on `bar` as transferred bytes.
__device__ __forceinline__ void load_2d(void* dst_smem, const CUtensorMap* map, int32_t x, int32_t y,
                                        uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
          "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
          "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
        : "memory");
}

// Untiled bulk copy global -> shared, completion on `bar`.
__device__ __forceinline__ void load_bulk(void* dst_smem, const void* src, uint32_t bytes,
                                          uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :
        : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))), "l"(src), "r"(bytes),
          "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
        : "memory");
}

// 2-D tiled store of a box from shared memory to (x, y) of the tensor; rows past the tensor's
// last row are not written.  Completion is tracked by bulk groups (commit / wait below).
__device__ __forceinline__ void store_2d(const CUtensorMap* map, int32_t x, int32_t y, const void* src_smem)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 :
                 : "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
                   "r"(static_cast<uint32_t>(__cvta_generic_to_shared(src_smem)))
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until this thread's committed bulk stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Wait until this thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Arm `bar` (arrival count 1) for `bytes` of incoming transfers.
__device__ __forceinline__ void expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar))), "r"(bytes)
                 : "memory");
}

}  // namespace tma

// Host: a row-major 2-D tensor [rows][cols] of `elem_bytes`-sized elements with
// a row pitch of `row_bytes`, tiled in boxes of box_cols x box_rows; out-of-range
// rows read as zeros.  `swizzle128` selects the 128-byte swizzled smem layout.
// Returns cudaSuccess or the error of the driver call.
cudaError_t make_tensor_map_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t cols,
                               uint64_t rows, uint64_t row_bytes, uint32_t box_cols,
                               uint32_t box_rows, bool swizzle128);

}  // namespace kda
