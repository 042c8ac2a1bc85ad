// pa_static_scratch.cu -- paged attention for callers that cannot allocate.
//
// pa_attention_varlen needs a caller-provided workspace.  Some callers have no
// way to get one: code running inside a memory allocator's own callbacks (it
// may not re-enter the allocator), plugins whose host application owns all
// device memory and hands them only their inputs and outputs, and latency-
// critical paths whose rules forbid a cudaMalloc (which can synchronise the
// device and take milliseconds).  For them this file keeps a fixed scratch
// area in a file-scope __device__ array, which the CUDA runtime places on
// every GPU that loads the library when the module is loaded and keeps until
// the process exits, and runs the same kernels on it.
#include <cuda.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_pa_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// Per device: the CUDA context the address was looked up in, and the address.
// Each context holds its own copy of the array: after cudaDeviceReset (a new
// primary context) or under a context the caller made current through the
// driver API, the same device ordinal names another copy, so the address is
// looked up again whenever the current context is not the recorded one.
struct ScratchAddr {
  CUcontext ctx = nullptr;
  void* ptr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetCurrentFn)ptr;
  }
  return fn;
}

// Device address of g_pa_scratch in the current context, looked up once per
// (device, context).  In host code the symbol names a host-side stand-in,
// never the device array itself, so only this address may be handed to a
// kernel.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchAddr& a = g_scratch[dev];
  if (!ctx || a.ctx != ctx || !a.ptr) {
    // (a thread with no context yet gets the device's primary context bound
    // by this first runtime call that needs one)
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_pa_scratch) != cudaSuccess || !ptr) return PA_ERR_CUDA;
    if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return PA_ERR_CUDA;
    a.ctx = ctx;
    a.ptr = ptr;
  }
  *out = a.ptr;
  return PA_OK;
}

}  // namespace

extern "C" int pa_attention_varlen_static_scratch(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
    const int32_t* query_start_loc, int num_seqs, int num_tokens, int max_query_len,
    int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int num_blocks, float scale, pa_dtype dtype, const int32_t* seq_lens_host,
    const int32_t* query_start_loc_host, struct CUstream_st* stream) {
  // fp32 steps run the CUDA-core kernel, which uses no scratch at all
  if (dtype == PA_DTYPE_F32)
    return pa::attention_varlen_sequential(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                               seq_lens, query_start_loc, num_seqs, num_tokens, max_query_len,
                               max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size,
                               num_blocks, scale, dtype, nullptr, 0, seq_lens_host,
                               query_start_loc_host, stream);
  const size_t need =
      pa_attention_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len);
  if (need == 0) return PA_ERR_INVALID;
  if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_INVALID;  // step too large
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != PA_OK) return rc;
  if (num_seqs > 0 && num_tokens > 0) {
    // The array still holds whatever the previous call left there, possibly
    // under another layout: the status word and the decode grid's claim
    // counters must start at zero, so clear them (everything before the
    // partials).
    const pa::WorkspaceLayout w =
        pa::workspace_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len);
    if (cudaMemsetAsync(scratch, 0, w.o_off, (cudaStream_t)stream) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return pa::attention_varlen_sequential(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                             query_start_loc, num_seqs, num_tokens, max_query_len, max_seq_len,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                             dtype, scratch, (size_t)PA_STATIC_SCRATCH_BYTES, seq_lens_host,
                             query_start_loc_host, stream);
}
