// Tensor Memory Accelerator (TMA) helpers for sm_100a: tiled bulk tensor loads
// from global into shared memory, completed through an mbarrier transaction
// count, plus the mbarrier arrive forms the warp-specialised pipelines use.
//
// Rules the callers keep (checked on the host before a launch):
//  * the tensor map's base address is 16-byte aligned and every stride is a
//    multiple of 16 bytes;
//  * the innermost box extent times the element size is a multiple of 16
//    bytes, and so is every innermost start coordinate times the element size;
//  * destinations in shared memory are 128-byte aligned;
//  * loads only (no multicast, no stores or reductions through TMA).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc_util.cuh"

namespace fno {
namespace tma {

// 4-D tiled load of one box into shared memory; completion is signalled as
// transaction bytes on `mbar` (which must expect them, see arrive_expect_tx).
__device__ __forceinline__ void load_4d(void *dst, const CUtensorMap *map, uint64_t *mbar, int c0,
                                        int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(tc::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(tc::smem_u32(mbar))
      : "memory");
}

// Untiled bulk copy of `bytes` contiguous bytes from global into shared memory
// (both addresses 16-byte aligned, bytes a multiple of 16), completed as
// transaction bytes on `mbar`.
__device__ __forceinline__ void load_bulk(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(tc::smem_u32(mbar))
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// one arrival that also raises the phase's expected transaction count
__device__ __forceinline__ void arrive_expect_tx(uint64_t *mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc::smem_u32(mbar)),
               "r"(bytes)
               : "memory");
}

// plain arrival (release semantics at CTA scope)
__device__ __forceinline__ void arrive(uint64_t *mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(mbar)) : "memory");
}

// make freshly initialised mbarriers visible to the async proxy
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

}  // namespace tma

// Host: encode a 4-D tiled tensor map (no interleave, no OOB fill; optional
// 128-byte swizzle, whose box rows must then be exactly 128 bytes).  dims[0] is
// the contiguous axis; strides_bytes[i] is the byte stride of axis i + 1.
// Returns false (message set) if the driver refuses the map.
bool encode_tmap_4d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                    const uint64_t dims[4], const uint64_t strides_bytes[3],
                    const uint32_t box[4], bool swizzle128 = false);

}  // namespace fno
