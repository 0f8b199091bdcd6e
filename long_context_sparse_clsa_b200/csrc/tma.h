// TMA (tensor memory accelerator) helpers: host-side encoding of 2-D tiled tensor maps
// through the driver entry point (no link-time dependency on libcuda), and the
// device-side tiled bulk load into shared memory that completes on an mbarrier.
// Loads only; no cluster multicast.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace clsa {

// 2-D bf16 tensor [rows][cols] (row-major, row pitch `pitch_bytes`), box = box_cols x
// box_rows, 128-byte swizzle (box_cols * 2 must be 128).  Out-of-range rows read zero.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_rows, uint32_t box_cols);

#ifdef __CUDACC__
// box at (x = column, y = row) of `map` into shared memory `dst`, completing on `bar`.
// x * element size must be a multiple of 16 bytes (x is 0 or 64 here).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
      "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
      : "memory");
}
#endif

}  // namespace clsa
