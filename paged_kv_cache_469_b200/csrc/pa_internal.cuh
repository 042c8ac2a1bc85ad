// pa_internal.cuh -- launch parameters and launchers shared by the kernels of
// libpa.so and its C-ABI front end (pa_api.cu).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "pa.h"

namespace pa {

// Raise a kernel's dynamic shared-memory limit only when a launch needs more
// than every earlier launch of it on this device (the attribute persists), so
// that a steady stream of calls makes no attribute call at all.  `done` is
// the kernel's own per-device record.
template <typename Kernel>
inline cudaError_t raise_smem_limit(Kernel kernel, int bytes, std::atomic<int> (&done)[64]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (done[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) {
    int cur = done[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !done[dev].compare_exchange_weak(cur, bytes)) {
    }
  }
  return e;
}

// SMs of the current device (looked up once per device; 148 if the query fails)
int device_sm_count();

constexpr int kBlockSize = 16;       // tokens per cache block (the pages' default)
constexpr int kDecodeRows = 16;      // query rows per kv-head one decode CTA holds (MMA M)
// A decode-class sequence has at most kDecodeMaxRows query rows per kv-head
// (q_len * q-heads per kv-head); they are split into 16-row groups, a unit of
// decode work each.  Longer queries are prefill chunks.
constexpr int kDecodeRowGroups = 4;
constexpr int kDecodeMaxRows = kDecodeRows * kDecodeRowGroups;
// split-K partial slots the workspace holds per (sequence, kv-head), shared by
// its row groups: kDecodePartsBase + ceil(max blocks / kDecodePartsPerBlocks)
constexpr int kDecodePartsBase = 8;
constexpr int kDecodePartsPerBlocks = 256;
// sanity bound on the slots of one (sequence, kv-head)
constexpr int kDecodeMaxParts = 1536;
// pieces of decode work: blocks per piece, and pieces per CTA the launch aims at
constexpr int kDecodeMaxPieceBlocks = 1024;
constexpr int kDecodeMinPieceBlocks = 4;
constexpr int kDecodePiecesPerCta = 4;
// K+V bytes of one (block, kv-head) per piece at most, unless a long unit
// needs bigger pieces to fit its partial slots
constexpr long kDecodeMaxPieceBytes = 2l << 20;
// pieces a launch can carry as a kernel parameter (more: the list is built on
// the device, in the workspace); with the per-CTA offsets and the two tensor
// maps the launch parameters stay under 32 KB
constexpr int kDecodeParamPieces = 1792;
// a list in the kernel parameters is dealt to at most this many CTAs on the
// host (longest first, each to the CTA with the least work so far, a piece
// counted as its blocks plus kDecodePieceCostBlocks for its staging and merge)
constexpr int kDecodeMaxDealtCtas = 256;
constexpr int kDecodePieceCostBlocks = 8;

// words of the workspace header (the first 256 bytes)
constexpr int kWsStatus = 0;       // error bits set by a kernel that gave up waiting
constexpr int kWsClaim = 1;        // decode pieces claimed past the first one per CTA
constexpr int kWsDone = 2;         // decode CTAs done claiming (the last resets both)
constexpr int kWsPieceCount = 3;   // decode pieces in the device-built list
constexpr int kWsPieceBlocks = 4;  // blocks per piece of that list

// Everything one attention launch reads; the same struct serves every kernel.
struct AttnParams {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const int32_t* query_start_loc;
  int max_blocks_per_seq;
  int max_seq_len;  // host bound: longer sequences are caller error and left unwritten
  int num_seqs;
  int num_tokens;
  int num_q_heads;
  int num_kv_heads;
  int group;  // num_q_heads / num_kv_heads
  int num_blocks;
  float scale;       // softmax scale (natural-log base)
  float scale_log2;  // scale * log2(e), for exp2-based softmax
  // decode-class steps of pa_attention_varlen_write_cache: the new tokens' K/V
  // rows [num_tokens][Hkv][D] and their slots, written by the decode kernel
  // (null otherwise)
  const void* k_new;
  const void* v_new;
  const int64_t* slot_mapping;
  int max_parts;     // partial slots per (sequence, kv-head): one per (piece, row group),
                     // piece-major
  int row_groups;    // 16-row groups per (sequence, kv-head) in this launch (1..4)
  int decode_rows;   // most query rows of one decode-class (sequence, kv-head)
  int max_pieces;    // capacity of ws_pieces
  float* ws_o;       // [num_seqs*Hkv][max_parts][16][D] unnormalised partial outputs
  float* ws_ml;      // [num_seqs*Hkv][max_parts][16][2] running max (log2 units), sum
  int* ws_status;    // the workspace header (kWs* words); [0]: error bits
  int* ws_header;    // = ws_status
  int4* ws_pieces;   // device-built decode piece list
  // prefill work list
  int4* ws_items;    // prefill items (seq, q-tile, q-head, kv tiles)
  int max_items;
};

// A decode launch's piece list carried as a kernel parameter (from_ws = 0), or
// a pointer to the device-built one in the workspace (from_ws = 1).  A piece is
// one int4: x = sequence, y = q_len << 24 | row group << 22 | kv-head << 12 |
// piece index in the unit, z = seq_len, w = query_start_loc of the sequence;
// piece j of a unit covers blocks j * piece_blocks .. of its sequence.
struct DecodeWork {
  int count;
  int piece_blocks;
  int from_ws;
  int split;  // some unit has more than one piece (its partials need the combine kernel)
  int dealt;  // CTA b takes items cta_off[b] .. cta_off[b + 1] - 1 (else: claims from a counter)
  int cta_off[kDecodeMaxDealtCtas + 1];
  int4 items[kDecodeParamPieces];
};

// bits of ws_status[0]
constexpr int kStatusWaitTimeout = 1;  // an mbarrier wait exceeded its time limit

// Workspace layout shared by the size query and the launch.
struct WorkspaceLayout {
  int max_parts;
  int max_items;
  int max_pieces;
  size_t status_off, o_off, ml_off, pieces_off, items_off, total;
};
WorkspaceLayout workspace_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_seq_len);

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int num_blocks,
                                     int elem_bytes, cudaStream_t stream);

// CUDA-core kernel: every query row whose sequence has more than
// min_rows_per_kv_head query rows per kv-head (0 = all rows).
cudaError_t launch_attention_simple(const AttnParams& p, int head_dim, bool is_bf16,
                                    int min_rows_per_kv_head, cudaStream_t stream);

// Persistent split-K decode kernel (bf16): sequences with q_len * group <=
// kDecodeMaxRows (64), in 16-row groups.  With host copies of the lengths the
// piece list is built on the host and passed with the launch; otherwise a
// one-CTA planning kernel builds it in the workspace first.
// At most max_ctas CTAs (the SMs left to decode when prefill runs beside it).
cudaError_t launch_decode(const AttnParams& p, int head_dim, const int32_t* seq_lens_host,
                          const int32_t* query_start_loc_host, cudaStream_t stream,
                          int max_ctas);

// Tensor-core prefill kernel (bf16): sequences with q_len * group > kDecodeMaxRows.
// num_items >= 0: the work list in ws_items was written by the host (exact
// count); num_items < 0: build it on the device first.
constexpr int kPrefillQTile = 128;  // query rows per Q tile (MMA M); a work item holds two
constexpr int kPrefillKvTile = 128;  // keys per pipeline step
// At most max_ctas persistent CTAs (one per SM).
cudaError_t launch_prefill_tcgen05(const AttnParams& p, int head_dim, int max_query_len,
                                   int num_items, const int32_t* seq_lens_host,
                                   const int32_t* query_start_loc_host, cudaStream_t stream,
                                   int max_ctas);

// pa_attention_varlen without the side stream of a mixed step (the two
// classes run one after the other): for the caller that must not create any
// CUDA object (the static-scratch entry point).
int attention_varlen_sequential(void* out, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* query_start_loc,
                                int num_seqs, int num_tokens, int max_query_len, int max_seq_len,
                                int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, float scale, pa_dtype dtype, void* workspace,
                                size_t workspace_bytes, const int32_t* seq_lens_host,
                                const int32_t* query_start_loc_host, struct CUstream_st* stream);

// On-GPU step planner (allocate_slots, seq_lens, query_start_loc, slot
// mapping).  planner state: int32[4] in device memory.
constexpr int kPlanStateHead = 0;      // index of the queue's front entry
constexpr int kPlanStateStatus = 1;    // error bits below (sticky)
constexpr int kPlanStateArrivals = 2;  // CTAs done with the current launch (0 between calls)
constexpr int kPlanMaxSeqs = 16384;    // sequences one call plans (their sums sit in shared memory)
constexpr int kPlanPoolEmpty = 1;      // the queue holds fewer blocks than the step needs
constexpr int kPlanRowFull = 2;        // a sequence would outgrow its block-table row
constexpr int kPlanSlotsFull = 4;      // more scheduled tokens than slot_mapping holds
constexpr int kPlanBadLength = 8;      // a negative count, or a length past int32
constexpr int kPlanBadHead = 16;       // the queue head lies outside the queue
size_t plan_step_smem(int num_seqs);
cudaError_t launch_plan_step(const int32_t* free_queue, int queue_len, int32_t* state,
                             const int32_t* num_computed, const int32_t* query_lens,
                             int num_seqs, int32_t* block_tables, int max_blocks_per_seq,
                             int32_t* seq_lens, int32_t* query_start_loc,
                             int64_t* slot_mapping, int max_tokens, cudaStream_t stream);

}  // namespace pa
