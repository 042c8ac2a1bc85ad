// pa_tma.cuh -- tensor-memory-accelerator (TMA) loads shared by the kernels of
// libpa.so: the device-side copy instruction and the host-side tensor maps of
// the paged K/V pool.  Every load here fills only the issuing CTA's own shared
// memory.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace pa {

// One box of a 3-D tensor map into shared memory, completing on the mbarrier
// at `bar` (transaction bytes).  The innermost coordinate c0 is a multiple of
// 64 elements, so it starts on a 16-byte boundary.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// Orders this thread's earlier shared-memory accesses (generic proxy) before
// the TMA writes it issues next (async proxy) into the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Host: a 3-D bf16 tensor map (dim0 innermost, extents d0, d1, d2; byte
// strides of dims 1 and 2) with a (64, box1, box2) box and 128-byte swizzle;
// loads past the extents fill zeros.  False if the driver refuses it.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2);

}  // namespace pa
