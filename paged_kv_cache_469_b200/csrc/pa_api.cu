// pa_api.cu -- the C ABI of libpa.so: host-side argument checks, workspace
// layout and dispatch of the kernels (declared in include/pa.h).
#include <math.h>

#include "pa.h"
#include "pa_internal.cuh"

namespace pa {

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split-K partial slots.  A decode unit (sequence, kv-head, row group) of
// nblk blocks is cut into pieces of P blocks, P chosen per launch; each piece
// of a unit that has more than one keeps an fp32 partial in the workspace.
// The workspace holds max_parts slots per (sequence, kv-head), shared by its
// row groups: kDecodePartsBase plus one per kDecodePartsPerBlocks blocks of
// the longest sequence, so that short sequences can be cut finely and long
// ones into pieces of a few hundred blocks at most.
int device_sm_count() {
  static std::atomic<int> n[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int v = n[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return 148;
    n[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

WorkspaceLayout workspace_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_seq_len) {
  WorkspaceLayout w{};
  const long max_blocks = ((long)max_seq_len + kBlockSize - 1) / kBlockSize;
  w.max_parts = (int)min((long)INT32_MAX,
                         kDecodePartsBase +
                             (max_blocks + kDecodePartsPerBlocks - 1) / kDecodePartsPerBlocks);
  // prefill items: at most ceil(q_len / 128) <= ceil(max_seq_len / 128) per sequence and q-head
  const long items = (long)num_seqs * ((max_seq_len + kPrefillQTile - 1) / kPrefillQTile) *
                     num_q_heads;
  w.max_items = (int)min(items, (long)(1 << 30));
  const size_t units = (size_t)num_seqs * num_kv_heads;
  // the device-built piece list: at most one piece per partial slot
  w.max_pieces = (int)min(units * (size_t)w.max_parts, (size_t)(1 << 30));
  const size_t slots = units * w.max_parts * kDecodeRows;
  w.status_off = 0;  // the 256-byte header: status word and the decode grid's counters
  w.o_off = 256;
  w.ml_off = align_up(w.o_off + slots * head_dim * sizeof(float), 256);
  w.pieces_off = align_up(w.ml_off + slots * 2 * sizeof(float), 256);
  w.items_off = align_up(w.pieces_off + (size_t)w.max_pieces * 16, 256);
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

static bool aligned_to(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

// A byte range [p, p + n) of caller memory (n = 0: empty, overlaps nothing).
struct Range {
  const void* p;
  size_t n;
  bool overlaps(const Range& o) const {
    if (!p || !o.p || n == 0 || o.n == 0) return false;
    const uintptr_t a = (uintptr_t)p, b = (uintptr_t)o.p;
    return a < b + o.n && b < a + n;
  }
};

extern "C" int pa_plan_step(const int32_t* free_queue, int queue_len, int32_t* planner_state,
                            const int32_t* num_computed, const int32_t* query_lens,
                            int num_seqs, int32_t* block_tables, int max_blocks_per_seq,
                            int block_size, int32_t* seq_lens, int32_t* query_start_loc,
                            int64_t* slot_mapping, int max_tokens, struct CUstream_st* stream) {
  if (queue_len < 0 || num_seqs < 0 || max_blocks_per_seq < 0 || max_tokens < 0)
    return PA_ERR_INVALID;
  if (block_size != kBlockSize || num_seqs > kPlanMaxSeqs) return PA_ERR_UNSUPPORTED;
  if (!planner_state || !query_start_loc) return PA_ERR_INVALID;
  if (num_seqs > 0 && (!num_computed || !query_lens || !block_tables || !seq_lens))
    return PA_ERR_INVALID;
  if ((queue_len > 0 && !free_queue) || (max_tokens > 0 && !slot_mapping)) return PA_ERR_INVALID;
  if (!aligned_to(planner_state, 16) || !aligned_to(query_start_loc, 4) ||
      !aligned_to(num_computed, 4) || !aligned_to(query_lens, 4) ||
      !aligned_to(block_tables, 4) || !aligned_to(seq_lens, 4) || !aligned_to(free_queue, 4) ||
      !aligned_to(slot_mapping, 8))
    return PA_ERR_INVALID;
  // The kernel's CTAs read num_computed and query_lens in full while other
  // CTAs already write seq_lens, query_start_loc and the slots: an output that
  // shares memory with an input would be read half old, half new.
  if (num_seqs > 0) {
    const Range in_nc{num_computed, (size_t)num_seqs * 4}, in_ql{query_lens, (size_t)num_seqs * 4};
    const Range outs[3] = {{seq_lens, (size_t)num_seqs * 4},
                           {query_start_loc, ((size_t)num_seqs + 1) * 4},
                           {slot_mapping, (size_t)max_tokens * 8}};
    for (const Range& o : outs)
      if (o.overlaps(in_nc) || o.overlaps(in_ql)) return PA_ERR_INVALID;
  }
  cudaError_t e = launch_plan_step(free_queue, queue_len, planner_state, num_computed,
                                   query_lens, num_seqs, block_tables, max_blocks_per_seq,
                                   seq_lens, query_start_loc, slot_mapping, max_tokens,
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

namespace {

// Rates one SM sustains while the two classes of a mixed step share the GPU,
// used only to split the SMs between them: the tensor-core prefill kernel
// (bf16 flops of unmasked query-key pairs per second; 5.5e12 when it has the
// GPU to itself, less beside a decode grid that keeps HBM busy) and the decode
// kernel (K/V bytes per second when every SM streams).  Measured on the
// Llama-3-8B mixed step: 3.3e12 to 4e12 (23 to 27 prefill SMs) gave the
// shortest step, 5e12 9 % longer, 6e12 16 % longer.
constexpr double kPrefillFlopsPerSm = 3.7e12;
constexpr double kDecodeBytesPerSm = 46.0e9;

// A side stream and two events, per thread and device, for the calls that run
// the prefill kernel beside the decode kernel.  Created on the first such call
// outside a stream capture; a capture that would need to create them runs the
// kernels one after the other instead.
struct ForkStreams {
  cudaStream_t side = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
};

ForkStreams* fork_streams(cudaStream_t st) {
  static thread_local ForkStreams per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  ForkStreams& f = per_dev[dev];
  if (f.side && f.start && f.done) return &f;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
    return nullptr;
  if ((!f.side && cudaStreamCreateWithFlags(&f.side, cudaStreamNonBlocking) != cudaSuccess) ||
      (!f.start && cudaEventCreateWithFlags(&f.start, cudaEventDisableTiming) != cudaSuccess) ||
      (!f.done && cudaEventCreateWithFlags(&f.done, cudaEventDisableTiming) != cudaSuccess))
    return nullptr;
  return &f;
}

// The new tokens' K/V rows a call writes into the cache before it reads it
// (pa_attention_varlen_write_cache); all null for pa_attention_varlen.
struct CacheWrite {
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const int64_t* slot_mapping = nullptr;
};

struct CallOptions {
  // may run the two classes of a mixed step side by side on a side stream
  // (created on first use); false for callers that must not create anything
  bool allow_fork = true;
};

int attention_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
                   const int32_t* query_start_loc, int num_seqs, int num_tokens,
                   int max_query_len, int max_seq_len, int num_q_heads, int num_kv_heads,
                   int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
                   void* workspace, size_t workspace_bytes, const int32_t* seq_lens_host,
                   const int32_t* query_start_loc_host, struct CUstream_st* stream,
                   const CacheWrite& cw, const CallOptions& opt) {
  const bool write_cache = cw.slot_mapping != nullptr;
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
  if (write_cache && (!cw.k_new || !cw.v_new || !aligned16(cw.k_new) || !aligned16(cw.v_new)))
    return PA_ERR_INVALID;

  // ---- optional host copies: check the step and see which kernels it needs
  bool any_decode = true, any_prefill = true;
  int prefill_items = -1;  // unknown without the host copies
  long decode_keys = -1;   // sum of the decode-class sequences' lengths, when known
  double prefill_flops = 0;  // of the prefill-class sequences, when known
  int decode_rows = min(max_query_len * group, kDecodeMaxRows);  // most rows of one of them
  if (seq_lens_host && query_start_loc_host) {
    if (query_start_loc_host[0] != 0 || query_start_loc_host[num_seqs] != num_tokens)
      return PA_ERR_INVALID;
    any_decode = any_prefill = false;
    prefill_items = 0;
    decode_keys = 0;
    decode_rows = 0;
    for (int s = 0; s < num_seqs; ++s) {
      const int ql = query_start_loc_host[s + 1] - query_start_loc_host[s];
      const int L = seq_lens_host[s];
      if (ql < 0 || ql > L || L > max_seq_len || ql > max_query_len) return PA_ERR_INVALID;
      if (ql == 0) continue;
      if (ql * group <= kDecodeMaxRows) {
        any_decode = true;
        decode_keys += L;
        decode_rows = max(decode_rows, ql * group);
      } else {
        any_prefill = true;
        prefill_items += (ql + kPrefillQTile - 1) / kPrefillQTile * num_q_heads;
        // unmasked (query, key) pairs: ql * (L - ql) of cached context + ql (ql + 1) / 2
        prefill_flops += 4.0 * head_dim * num_q_heads *
                         ((double)ql * (L - ql) + (double)ql * (ql + 1) / 2);
      }
    }
  } else if (max_query_len * group <= kDecodeMaxRows) {
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
  p.max_parts = w.max_parts;  // the workspace's partial slots per (sequence, kv-head)
  p.max_pieces = w.max_pieces;
  p.row_groups = max(1, (decode_rows + kDecodeRows - 1) / kDecodeRows);
  p.decode_rows = decode_rows;
  // the longest sequence must fit the slots of its (sequence, kv-head) in
  // pieces of at most kDecodeMaxPieceBlocks blocks
  {
    const long max_blocks = ((long)max_seq_len + kBlockSize - 1) / kBlockSize;
    const long slots_per_unit = w.max_parts / p.row_groups;
    if (any_decode && dtype == PA_DTYPE_BF16 &&
        (slots_per_unit < 1 ||
         (max_blocks + slots_per_unit - 1) / slots_per_unit > kDecodeMaxPieceBlocks))
      return PA_ERR_UNSUPPORTED;
  }
  p.num_seqs = num_seqs;
  p.num_tokens = num_tokens;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.num_blocks = num_blocks;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = (cudaStream_t)stream;
  const int elem_bytes = dtype == PA_DTYPE_F32 ? 4 : 2;
  // The decode kernel writes a sequence's new rows itself (each CTA those
  // that fall in its own key range, before it reads them back) when every
  // sequence of the step is decode-class; otherwise the cache write runs as
  // its own kernel first, since a prefill chunk's tiles need all of its rows.
  const bool fused_write = write_cache && dtype == PA_DTYPE_BF16 && !any_prefill;
  // every argument check comes before the first launch
  if (dtype != PA_DTYPE_F32 &&
      (!workspace || workspace_bytes < w.total || !aligned16(workspace)))
    return PA_ERR_INVALID;
  if (write_cache && !fused_write) {
    cudaError_t e = launch_reshape_and_cache(cw.k_new, cw.v_new, const_cast<void*>(k_cache),
                                             const_cast<void*>(v_cache), cw.slot_mapping,
                                             num_tokens, num_kv_heads, head_dim, num_blocks,
                                             elem_bytes, st);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }

  if (dtype == PA_DTYPE_F32) {
    cudaError_t e = launch_attention_simple(p, head_dim, false, 0, st);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }

  char* ws = (char*)workspace;
  p.ws_status = (int*)(ws + w.status_off);
  p.ws_header = p.ws_status;
  p.ws_o = (float*)(ws + w.o_off);
  p.ws_ml = (float*)(ws + w.ml_off);
  p.ws_pieces = (int4*)(ws + w.pieces_off);
  p.ws_items = (int4*)(ws + w.items_off);
  p.max_items = w.max_items;
  if (fused_write) {
    p.k_new = cw.k_new;
    p.v_new = cw.v_new;
    p.slot_mapping = cw.slot_mapping;
  }
  const int sms = device_sm_count();
  // A step with both classes of work (known from the host copies) runs them
  // side by side: the prefill kernel on a side stream, on a share of the SMs
  // proportional to its share of the step's work, the decode kernel on the
  // rest, joined back into `stream` before the call returns.
  ForkStreams* fork = nullptr;
  int prefill_ctas = sms, decode_ctas = sms;
  if (opt.allow_fork && any_decode && any_prefill && prefill_flops > 0 && decode_keys > 0) {
    fork = fork_streams(st);
    if (fork) {
      // SM-seconds of each class at the rates one SM sustains on its own
      const double a = prefill_flops / kPrefillFlopsPerSm;
      const double b = (double)decode_keys * 2 * num_kv_heads * head_dim * 2 / kDecodeBytesPerSm;
      prefill_ctas = (int)lround(sms * a / (a + b));
      prefill_ctas = max(1, min(prefill_ctas, sms / 2));
      decode_ctas = sms - prefill_ctas;
    }
  }
  if (fork) {
    if (cudaEventRecord(fork->start, st) != cudaSuccess ||
        cudaStreamWaitEvent(fork->side, fork->start, 0) != cudaSuccess)
      return PA_ERR_CUDA;
    cudaError_t e = launch_prefill_tcgen05(p, head_dim, max_query_len, prefill_items,
                                           seq_lens_host, query_start_loc_host, fork->side,
                                           prefill_ctas);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    e = launch_decode(p, head_dim, seq_lens_host, query_start_loc_host, st, decode_ctas);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    if (cudaEventRecord(fork->done, fork->side) != cudaSuccess ||
        cudaStreamWaitEvent(st, fork->done, 0) != cudaSuccess)
      return PA_ERR_CUDA;
    return PA_OK;
  }
  if (any_decode) {
    cudaError_t e = launch_decode(p, head_dim, seq_lens_host, query_start_loc_host, st, sms);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  if (any_prefill) {
    cudaError_t e = launch_prefill_tcgen05(p, head_dim, max_query_len, prefill_items,
                                           seq_lens_host, query_start_loc_host, st, sms);
    if (e != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace

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
  return attention_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                        query_start_loc, num_seqs, num_tokens, max_query_len, max_seq_len,
                        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                        workspace, workspace_bytes, seq_lens_host, query_start_loc_host, stream,
                        CacheWrite{}, CallOptions{});
}

namespace pa {

int attention_varlen_sequential(void* out, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* query_start_loc,
                                int num_seqs, int num_tokens, int max_query_len, int max_seq_len,
                                int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, float scale, pa_dtype dtype, void* workspace,
                                size_t workspace_bytes, const int32_t* seq_lens_host,
                                const int32_t* query_start_loc_host, struct CUstream_st* stream) {
  CallOptions opt;
  opt.allow_fork = false;
  return attention_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                        query_start_loc, num_seqs, num_tokens, max_query_len, max_seq_len,
                        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                        workspace, workspace_bytes, seq_lens_host, query_start_loc_host, stream,
                        CacheWrite{}, opt);
}

}  // namespace pa

extern "C" int pa_attention_varlen_write_cache(
    void* out, const void* q, const void* k_new, const void* v_new, void* k_cache,
    void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* seq_lens, const int32_t* query_start_loc,
    int num_seqs, int num_tokens, int max_query_len, int max_seq_len, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
    void* workspace, size_t workspace_bytes, const int32_t* seq_lens_host,
    const int32_t* query_start_loc_host, struct CUstream_st* stream) {
  if (!slot_mapping && num_tokens > 0) return PA_ERR_INVALID;
  CacheWrite cw;
  cw.k_new = k_new;
  cw.v_new = v_new;
  cw.slot_mapping = slot_mapping;
  return attention_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                        query_start_loc, num_seqs, num_tokens, max_query_len, max_seq_len,
                        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                        workspace, workspace_bytes, seq_lens_host, query_start_loc_host, stream,
                        slot_mapping ? cw : CacheWrite{}, CallOptions{});
}
