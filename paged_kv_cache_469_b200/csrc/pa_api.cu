// pa_api.cu -- the C ABI of libpa.so: host-side argument checks, workspace
// layout and dispatch of the kernels (declared in include/pa.h).
#include <math.h>

#include "pa.h"
#include "pa_internal.cuh"

namespace pa {

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Keys per split-K partition: the largest power of two in [PA_PART_MIN,
// PA_PART_MAX] that still gives the GPU about PA_TARGET_CTAS CTAs when the
// sequences average half of max_seq_len.  Hardware CTA scheduling then spreads
// the partitions over the SMs as they free up.
#ifndef PA_PART_MIN
#define PA_PART_MIN 1024
#endif
#ifndef PA_PART_MAX
#define PA_PART_MAX 2048
#endif
#ifndef PA_TARGET_CTAS
#define PA_TARGET_CTAS (8 * 148)
#endif
static int choose_part_tokens(int num_seqs, int num_kv_heads, int max_seq_len) {
  const long units = (long)num_seqs * num_kv_heads;
  int part = PA_PART_MAX;
  while (part > PA_PART_MIN &&
         units * (((long)max_seq_len / 2 + part - 1) / part) < (long)PA_TARGET_CTAS)
    part /= 2;
  return part;
}

WorkspaceLayout workspace_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_seq_len) {
  WorkspaceLayout w{};
  w.part_tokens = choose_part_tokens(num_seqs, num_kv_heads, max_seq_len);
  w.max_parts = max(1, (max_seq_len + w.part_tokens - 1) / w.part_tokens);
  // prefill items: at most ceil(q_len / 128) <= ceil(max_seq_len / 128) per sequence and q-head
  const long items = (long)num_seqs * ((max_seq_len + kPrefillQTile - 1) / kPrefillQTile) *
                     num_q_heads;
  w.max_items = (int)min(items, (long)(1 << 30));
  const size_t units = (size_t)num_seqs * num_kv_heads;
  const size_t slots = units * w.max_parts * kDecodeRows;
  w.status_off = 0;
  w.counter_off = 256;
  w.o_off = align_up(w.counter_off + units * sizeof(int), 256);
  w.ml_off = align_up(w.o_off + slots * head_dim * sizeof(float), 256);
  w.items_off = align_up(w.ml_off + slots * 2 * sizeof(float), 256);
  w.total = align_up(w.items_off + (size_t)(w.max_items + 1) * 16, 256);
  return w;
}

}  // namespace pa

using namespace pa;

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

extern "C" const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape or dtype not implemented";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: kernel launch failed";
    default: return "unknown pa_status";
  }
}

static bool supported_head_dim(int d) { return d == 64 || d == 128; }

extern "C" int pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                    const int64_t* slot_mapping, int num_tokens,
                                    int num_kv_heads, int head_dim, int block_size,
                                    int num_blocks, pa_dtype dtype, struct CUstream_st* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks < 0) return PA_ERR_INVALID;
  if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
  if (block_size != kBlockSize || !supported_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const int elem = dtype == PA_DTYPE_F32 ? 4 : 2;
  cudaError_t e = launch_reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                           num_kv_heads, head_dim, num_blocks, elem,
                                           (cudaStream_t)stream);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" size_t pa_attention_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                              int head_dim, int max_seq_len) {
  if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || max_seq_len < 0) return 0;
  if (num_q_heads % num_kv_heads != 0 || !supported_head_dim(head_dim)) return 0;
  return workspace_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len).total;
}

extern "C" int pa_workspace_status(const void* workspace, size_t workspace_bytes,
                                   int* status_out, struct CUstream_st* stream) {
  if (!workspace || workspace_bytes < 256 || !status_out) return PA_ERR_INVALID;
  if (cudaMemcpyAsync(status_out, workspace, sizeof(int), cudaMemcpyDeviceToHost,
                      (cudaStream_t)stream) != cudaSuccess ||
      cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}

extern "C" int pa_workspace_init(void* workspace, size_t workspace_bytes,
                                 struct CUstream_st* stream) {
  if (!workspace && workspace_bytes) return PA_ERR_INVALID;
  if (!workspace_bytes) return PA_OK;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream) == cudaSuccess
             ? PA_OK
             : PA_ERR_CUDA;
}

extern "C" int pa_attention_varlen(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* seq_lens,
                                   const int32_t* query_start_loc, int num_seqs, int num_tokens,
                                   int max_query_len, int max_seq_len, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int num_blocks, float scale, pa_dtype dtype, void* workspace,
                                   size_t workspace_bytes, const int32_t* seq_lens_host,
                                   const int32_t* query_start_loc_host,
                                   struct CUstream_st* stream) {
  // ---- scalar checks
  if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0 || max_seq_len < 0 ||
      num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks < 0 || max_blocks_per_seq < 0)
    return PA_ERR_INVALID;
  if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
  if (block_size != kBlockSize || !supported_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID;
  const int group = num_q_heads / num_kv_heads;
  if (group > kDecodeRows) return PA_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !isfinite(scale)) return PA_ERR_INVALID;
  if (max_query_len > max_seq_len) return PA_ERR_INVALID;
  if ((long)max_blocks_per_seq * kBlockSize < (long)max_seq_len) return PA_ERR_INVALID;
  if (num_seqs == 0 || num_tokens == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !query_start_loc)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;

  // ---- optional host copies: check the step and see which kernels it needs
  bool any_decode = true, any_prefill = true;
  int prefill_items = -1;  // unknown without the host copies
  if (seq_lens_host && query_start_loc_host) {
    if (query_start_loc_host[0] != 0 || query_start_loc_host[num_seqs] != num_tokens)
      return PA_ERR_INVALID;
    any_decode = any_prefill = false;
    prefill_items = 0;
    for (int s = 0; s < num_seqs; ++s) {
      const int ql = query_start_loc_host[s + 1] - query_start_loc_host[s];
      const int L = seq_lens_host[s];
      if (ql < 0 || ql > L || L > max_seq_len || ql > max_query_len) return PA_ERR_INVALID;
      if (ql == 0) continue;
      if (ql * group <= kDecodeRows) {
        any_decode = true;
      } else {
        any_prefill = true;
        prefill_items += (ql + kPrefillQTile - 1) / kPrefillQTile * num_q_heads;
      }
    }
  } else if (max_query_len * group <= kDecodeRows) {
    any_prefill = false;
  }

  const WorkspaceLayout w =
      workspace_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len);
  if (w.max_parts > kDecodeMaxParts) return PA_ERR_UNSUPPORTED;
  AttnParams p{};
  p.out = out;
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.query_start_loc = query_start_loc;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_seq_len = max_seq_len;
  p.part_tokens = w.part_tokens;
  p.max_parts = w.max_parts;
  p.num_seqs = num_seqs;
  p.num_tokens = num_tokens;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.num_blocks = num_blocks;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = (cudaStream_t)stream;

  if (dtype == PA_DTYPE_F32) {
    cudaError_t e = launch_attention_simple(p, head_dim, false, 0, st);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }

  if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return PA_ERR_INVALID;
  char* ws = (char*)workspace;
  p.ws_status = (int*)(ws + w.status_off);
  p.ws_counter = (int*)(ws + w.counter_off);
  p.ws_o = (float*)(ws + w.o_off);
  p.ws_ml = (float*)(ws + w.ml_off);
  p.ws_items = (int4*)(ws + w.items_off);
  p.max_items = w.max_items;
  if (any_decode) {
    cudaError_t e = launch_decode_splitk(p, head_dim, max_query_len, st);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  if (any_prefill) {
    cudaError_t e = launch_prefill_tcgen05(p, head_dim, max_query_len, prefill_items, st);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}
