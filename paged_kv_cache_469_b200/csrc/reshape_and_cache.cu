// reshape_and_cache.cu -- scatter this step's new K/V rows into their cache slots.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "PagedAttentionの仕組み":
// KV lives in 16-token blocks; a token's slot names its block and its offset
// in the block.  One warp moves one (token, kv-head) row of K and of V with
// 16-byte vector accesses: the source row is contiguous, and so is its
// destination ([block][kv-head][offset][:] in the cache).
#include "pa_internal.cuh"

namespace pa {
namespace {

template <int kVecPerRow>  // 16-byte vectors per row: head_dim * elem_bytes / 16
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                         uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                         const int64_t* __restrict__ slot_mapping, int num_tokens,
                         int num_kv_heads, int64_t num_slots) {
  // let the next kernel (the attention kernel) get launched now: it waits for
  // this grid's completion before it reads anything
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // launched as a programmatic dependent of the previous kernel on the stream:
  // nothing is read or written before that kernel has completed
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= (int64_t)num_tokens * num_kv_heads) return;
  const int64_t tok = row / num_kv_heads;
  const int h = (int)(row % num_kv_heads);
  const int64_t slot = slot_mapping[tok];
  if (slot < 0 || slot >= num_slots) return;  // padding / out-of-pool slot: no write
  const int64_t blk = slot / kBlockSize;
  const int off = (int)(slot % kBlockSize);
  const int64_t dst = ((blk * num_kv_heads + h) * kBlockSize + off) * kVecPerRow;
  const int64_t src = row * kVecPerRow;
#pragma unroll
  for (int i = lane; i < kVecPerRow; i += 32) {
    k_cache[dst + i] = k[src + i];
    v_cache[dst + i] = v[src + i];
  }
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int num_blocks,
                                     int elem_bytes, cudaStream_t stream) {
  const int64_t rows = (int64_t)num_tokens * num_kv_heads;
  if (rows == 0) return cudaSuccess;
  const int warps_per_cta = 8;
  const int64_t grid = (rows + warps_per_cta - 1) / warps_per_cta;
  const int vec = head_dim * elem_bytes / 16;
  const int64_t num_slots = (int64_t)num_blocks * kBlockSize;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(warps_per_cta * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto launch = [&](auto kernel) {
    return cudaLaunchKernelEx(&cfg, kernel, (const uint4*)k, (const uint4*)v, (uint4*)k_cache,
                              (uint4*)v_cache, slot_mapping, num_tokens, num_kv_heads, num_slots);
  };
  cudaError_t e;
  switch (vec) {
    case 8: e = launch(reshape_and_cache_kernel<8>); break;    // bf16 D=64
    case 16: e = launch(reshape_and_cache_kernel<16>); break;  // bf16 D=128, f32 D=64
    case 32: e = launch(reshape_and_cache_kernel<32>); break;  // f32 D=128
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pa
