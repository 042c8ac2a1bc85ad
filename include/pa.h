/*
 * pa.h -- C ABI of the B200 (sm_100a) paged-attention library libpa.so.
 *
 * The method (page "LLM推論エンジンvLLMの内部構造を徹底解説", techfeed.io summary of
 * "Inside vLLM: Anatomy of a High-Throughput LLM Inference System"):
 *   section "PagedAttentionの仕組み" -- the KV cache is a pool of fixed-size
 *   blocks (16 tokens by default), each request owning a list of blocks (its
 *   row of the block table); a step's sequences are flattened into one
 *   super-sequence, and position indices plus a mask let each sequence attend
 *   only to its own tokens.
 *   section "高度な機能群" -- chunked prefill (a chunk attends to the context
 *   cached before it) and prefix caching (several block lists point at the
 *   same physical blocks).
 *   section "エンジンの中核" -- prefill is compute-bound, decode (the newest
 *   token only, against the cache) is memory-bandwidth-bound, and one step may
 *   mix both.
 *
 * Conventions of every call:
 *   - Every tensor pointer is DEVICE memory owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  The library allocates no device memory and
 *     keeps no data between calls; the caller's workspace holds all scratch.
 *     (It does remember, per device, the kernel attributes it has already
 *     set, and, per thread and device, the one side stream and two events it
 *     creates on the first call that runs a mixed step's two classes of work
 *     side by side; see pa_attention_varlen.)
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and keeps stream order: each kernel is launched
 *     as a programmatic dependent of the work before it, so its launch may
 *     overlap that work's tail, but it reads and writes nothing until that
 *     work has completed.  Argument checks run on the host before any launch
 *     and return PA_ERR_INVALID / PA_ERR_UNSUPPORTED with nothing launched;
 *     PA_ERR_CUDA reports a failed launch (cudaGetLastError).
 *   - Calls can be captured in a CUDA graph.  A capture records the launch
 *     plan of that call: with the optional host copies of seq_lens and
 *     query_start_loc, that plan follows them (kernel choice, the decode
 *     pieces, their order and their dealing to the CTAs, the prefill work
 *     list), so a replay needs device arrays that still hold those values.
 *   - Nothing traps on the device.  Slots or block ids outside the pool are
 *     never dereferenced (see each call).
 *   - dtype is the element type of q, k, v, the caches and out alike.
 *
 * Cache layout (the pages give none; this library's reading):
 *   k_cache, v_cache: [num_blocks][num_kv_heads][block_size][head_dim]; the
 *   16 tokens of one (block, kv-head) are one contiguous 2 KiB (D=64) or 4 KiB
 *   (D=128) bf16 tile.  Slot s is block s / block_size, offset s % block_size.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* = cudaStream_t without pulling in the CUDA headers */

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,     /* a size, pointer or alignment is wrong */
  PA_ERR_UNSUPPORTED = -2, /* valid, but not a shape this library implements */
  PA_ERR_CUDA = -3         /* a kernel launch failed */
} pa_status;

typedef enum { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1 } pa_dtype;

/* Human-readable name of a pa_status value (static string). */
const char* pa_status_string(int status);

/*
 * pa_reshape_and_cache -- write this step's new K/V rows into their cache slots.
 *
 * For every i < num_tokens with slot = slot_mapping[i] in [0, num_blocks *
 * block_size):  k_cache[slot / block_size][h][slot % block_size][:] = k[i][h][:]
 * and the same for v, for every kv-head h.  A slot outside that range (e.g. a
 * negative padding slot) skips the row.  The copy is bit-exact.  Two tokens
 * naming the same slot race (caller error).
 *
 *   k, v          [num_tokens][num_kv_heads][head_dim]
 *   k_cache,
 *   v_cache       [num_blocks][num_kv_heads][block_size][head_dim] (written)
 *   slot_mapping  int64 [num_tokens]
 * Supported: head_dim in {64, 128}; block_size 16; dtype f32 or bf16.
 * Slot of position p of a request: block_table[p / 16] * 16 + p % 16
 * (section "PagedAttentionの仕組み": blocks of 16 tokens, filled in order).
 */
int pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         struct CUstream_st* stream);

/*
 * Bytes of workspace pa_attention_varlen needs for a step of at most
 * num_seqs sequences, no sequence longer than max_seq_len tokens: a 256-byte
 * header (the status word, and counters the decode grid uses while it runs
 * and leaves at zero), fp32 split-K partials (running max, sum and
 * unnormalised output per piece of a sequence's keys), the decode work list
 * when it is built on the device, and the prefill work list.  0 means
 * invalid arguments.
 */
size_t pa_attention_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int max_seq_len);

/*
 * Read the workspace's status word (blocking: copies 4 bytes to *status_out
 * and synchronises `stream`).  0 = every kernel of the previous calls ran to
 * completion.  Bit 0 set = a kernel gave up waiting on one of its own
 * pipeline barriers after a time limit instead of hanging (a library bug or a
 * GPU fault); the outputs of that call are not valid.  The word stays set until
 * pa_workspace_init clears the workspace again.
 */
int pa_workspace_status(const void* workspace, size_t workspace_bytes, int* status_out,
                        struct CUstream_st* stream);

/*
 * Zero a workspace before its first use (a cudaMemsetAsync on `stream`).
 * Every pa_attention_varlen call leaves the counters at zero again, so this is
 * needed once per workspace allocation.
 */
int pa_workspace_init(void* workspace, size_t workspace_bytes, struct CUstream_st* stream);

/*
 * pa_attention_varlen -- paged attention over one flattened step.
 *
 * Sequence s owns query rows query_start_loc[s] .. query_start_loc[s+1]-1 of q
 * (q_len = their count) and seq_lens[s] keys (all of its tokens, this step's
 * new ones included; their K/V must already be in the cache, written by
 * pa_reshape_and_cache).  Query j of sequence s sits at position
 * seq_lens[s] - q_len + j and attends to keys 0..that position of its own
 * sequence, read through block_tables[s] (a decode is q_len = 1; a prefill
 * chunk over cached context is q_len > 1 with seq_lens[s] > q_len).  q-head h
 * reads kv-head h / (num_q_heads / num_kv_heads).
 *
 *   out[t][h][:] = sum_k softmax_k(scale * q[t][h] . K_k) V_k
 *
 *   out            [num_tokens][num_q_heads][head_dim] (written)
 *   q              [num_tokens][num_q_heads][head_dim]
 *   k_cache,
 *   v_cache        [num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]; entries beyond
 *                  ceil(seq_lens[s] / block_size) are never read; an entry
 *                  outside [0, num_blocks) is never dereferenced (the result
 *                  for that sequence is then not meaningful, but no memory
 *                  outside the pool is touched).  Slots of the last block past
 *                  seq_lens[s] are never used, whatever they hold.
 *   seq_lens       int32 [num_seqs]
 *   query_start_loc int32 [num_seqs + 1], query_start_loc[0] = 0,
 *                  nondecreasing, query_start_loc[num_seqs] = num_tokens.
 *                  The kernels trust these device arrays as given (a
 *                  malformed query_start_loc would index q and out out of
 *                  range); the host copies below, when given, are checked
 *   max_query_len, max_seq_len  host-side upper bounds over the step (they
 *                  size the launch grids; a sequence beyond them is caller
 *                  error and may be left unwritten)
 *   workspace      at least pa_attention_workspace_size(num_seqs, num_q_heads,
 *                  num_kv_heads, head_dim, max_seq_len) bytes, zeroed once by
 *                  pa_workspace_init; one workspace serves one call at a time
 *   seq_lens_host, query_start_loc_host  optional (NULL) host copies of the
 *                  two device arrays, equal to them: when given, the call
 *                  checks them, launches only the kernels the step needs,
 *                  cuts the decode work into pieces sized from the step's
 *                  total keys and passes their list (up to 1792 pieces) with
 *                  the launch, and (up to 1024 prefill work items) passes the
 *                  prefill work list with it, instead of building them on
 *                  the GPU
 *
 * Decode-class sequences (q_len * num_q_heads / num_kv_heads <= 64 query
 * rows per kv-head: single-token decodes and the few-token queries of
 * speculative verification) run the persistent split-K bandwidth-bound kernel
 * (one CTA per SM, pieces of the sequences' blocks claimed largest first, 16
 * query rows per unit of work); longer prefill chunks run the tensor-core
 * kernel.  fp32 steps run a CUDA-core kernel.  Without the host copies, a
 * one-CTA planning kernel first lists the decode work on the device.  When
 * the host copies show a bf16 step with both classes of sequences, the call
 * runs the tensor-core prefill kernel on a side stream of its own, on a share
 * of the SMs proportional to the prefill work, while the decode kernel
 * streams on the other SMs; `stream` waits for the side stream before the
 * call returns, so any work queued on `stream` afterwards sees every output
 * row.  (The side stream joins a stream capture the same way, as a fork and a
 * join of the captured graph.)
 * Supported: head_dim in {64, 128}; block_size 16; num_q_heads a multiple of
 * num_kv_heads with at most 16 q-heads per kv-head; dtype f32 or bf16;
 * max_seq_len up to 6.2M tokens (a longer bound returns PA_ERR_UNSUPPORTED).
 */
int pa_attention_varlen(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* seq_lens, const int32_t* query_start_loc, int num_seqs,
                        int num_tokens, int max_query_len, int max_seq_len, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                        const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                        struct CUstream_st* stream);

/*
 * pa_attention_varlen_write_cache -- pa_reshape_and_cache of the step's new
 * tokens followed by pa_attention_varlen, in one call.  (The pages describe
 * the two operations one after the other; this call gives the same results.)
 *
 * Arguments: those of pa_attention_varlen, plus the new rows k_new, v_new
 * ([num_tokens][num_kv_heads][head_dim], 16-byte aligned) and slot_mapping
 * (int64 [num_tokens]) as pa_reshape_and_cache takes them; k_cache and
 * v_cache are written.  Results: the cache bytes of pa_reshape_and_cache and
 * the output of pa_attention_varlen on the updated cache.
 *
 * When every sequence of the step is decode-class (bf16), the decode kernel
 * writes the rows itself: each CTA first stores the new tokens that fall in
 * its own range of its sequence's keys, then reads them back through the
 * block table.  One launch instead of two.  (When a sequence's query rows
 * span several 16-row groups, each group's CTA stores the same bytes to the
 * same slots; identical concurrent stores, so every read sees the new row.)  This requires the usual layout of
 * a step: a token's slot is the slot of its own position in its own
 * sequence's block table (block_tables[s][pos / 16] * 16 + pos % 16), and no
 * other sequence of the step reads that slot.  Otherwise (prefill chunks, or
 * fp32) the cache write runs as its own kernel first.
 */
int pa_attention_varlen_write_cache(
    void* out, const void* q, const void* k_new, const void* v_new, void* k_cache,
    void* v_cache, const int64_t* slot_mapping, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* seq_lens, const int32_t* query_start_loc,
    int num_seqs, int num_tokens, int max_query_len, int max_seq_len, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
    void* workspace, size_t workspace_bytes, const int32_t* seq_lens_host,
    const int32_t* query_start_loc_host, struct CUstream_st* stream);

/*
 * pa_attention_varlen_static_scratch -- pa_attention_varlen for callers that
 * cannot allocate device memory.  (The pages describe no such call; it has no
 * counterpart in the method itself.)
 *
 * Who needs it: code that must not call cudaMalloc or any allocating routine
 * -- a memory allocator's own callbacks (they would re-enter the allocator),
 * a plugin whose host application owns every device buffer and passes it only
 * inputs and outputs, or a latency-critical path where an allocation (which
 * may synchronise the device) is not allowed.  Such a caller has nowhere to
 * put the workspace pa_attention_varlen asks for.
 *
 * Same arguments and results as pa_attention_varlen, minus the workspace.
 * The scratch instead lives in one fixed array of PA_STATIC_SCRATCH_BYTES
 * (16 MiB) that every GPU which loads this library holds until the process
 * exits.  A step whose pa_attention_workspace_size(...) exceeds that is
 * rejected with PA_ERR_INVALID before anything is launched.  The call itself
 * allocates nothing.
 *
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address belongs to the CUDA context current at that call: a call
 *     under another context of the same device (after cudaDeviceReset, or one
 *     made current through the driver API) looks it up again, which must
 *     also happen outside a stream capture.
 *   - Every call, on every stream, shares the one array and it keeps the last
 *     call's contents: each call clears the parts that must start at zero.
 *     Calls that can overlap on the GPU (other streams, other threads) race
 *     on the array: serialise them.
 *   - A kernel's status word (see pa_workspace_status) lives in this array
 *     too and is cleared by the next call.  The caller has no workspace
 *     pointer to read it through, so a kernel that gave up on one of its
 *     time-bounded waits (a library bug or a GPU fault, never an input) is
 *     not reported by this entry point.  Callers that must see that status
 *     use pa_attention_varlen with a workspace of their own.
 *   - fp32 steps use no scratch: they are never refused for size.
 */
#define PA_STATIC_SCRATCH_BYTES (16u << 20)
int pa_attention_varlen_static_scratch(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
    const int32_t* query_start_loc, int num_seqs, int num_tokens, int max_query_len,
    int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int num_blocks, float scale, pa_dtype dtype, const int32_t* seq_lens_host,
    const int32_t* query_start_loc_host, struct CUstream_st* stream);

/*
 * pa_plan_step -- one scheduler step's block allocation and attention inputs,
 * computed on the GPU (no host round trip between the steps of a decode loop).
 *
 * Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "PagedAttentionの仕組み":
 * a request of n tokens holds ceil(n / 16) blocks, and allocate_slots takes
 * the blocks a request lacks from the front of free_block_queue into the
 * request's block list, requests in order; the step's sequences form one
 * super-sequence; a token at position p is stored in slot
 * block_table[p / 16] * 16 + p % 16.  Page "【ITニュース解説】Inside vLLM: Anatomy
 * of a High-Throughput LLM Inference System", its paragraph on Paging
 * Attention: blocks are handed out as the model produces new tokens, only as
 * many as are needed, so a running request grows by whole blocks step by
 * step.  (Step 2 of allocate_slots, preempting
 * requests when the pool runs dry, is scheduler policy: here a step that does
 * not fit is refused, see the status bits.)
 *
 * Sequence s already owns the blocks of its first num_computed[s] tokens
 * (entries 0 .. ceil(num_computed[s] / 16) - 1 of its row) and schedules
 * query_lens[s] new tokens.  The call writes
 *   seq_lens[s]        = num_computed[s] + query_lens[s]
 *   query_start_loc    = 0, then the running sum of query_lens  ([num_seqs + 1])
 *   block_tables[s][c] for c = ceil(num_computed[s] / 16) .. ceil(seq_lens[s] / 16) - 1:
 *                        the next queue entries, sequences in order, from the
 *                        queue head on (other entries are left as they are)
 *   slot_mapping[query_start_loc[s] + j] = slot of position num_computed[s] + j
 * and advances the queue head by the number of blocks taken.  These are the
 * arguments pa_reshape_and_cache and pa_attention_varlen(_write_cache) take
 * (with num_tokens = the sum of query_lens).
 *
 *   free_queue      int32 [queue_len]: block ids, front first
 *   planner_state   int32 [4], 16-byte aligned, caller-owned: [0] queue head
 *                   (index of the front entry, in and out), [1] status bits
 *                   (sticky: set, never cleared, by the call), [2] used inside
 *                   the call, must be 0 between calls, [3] unused.  Zero it
 *                   once, then set [0] to where the queue's free part starts.
 *   num_computed,
 *   query_lens      int32 [num_seqs] (device; e.g. a copy of the previous
 *                   step's seq_lens as num_computed).  Neither may share
 *                   memory with seq_lens, query_start_loc or slot_mapping:
 *                   the CTAs of one launch read both inputs in full while
 *                   others already write the outputs, so an aliased buffer
 *                   would be read half updated.  Such a call returns
 *                   PA_ERR_INVALID before anything is launched.
 *   block_tables    int32 [num_seqs][max_blocks_per_seq], updated in place
 *   seq_lens        int32 [num_seqs] (written)
 *   query_start_loc int32 [num_seqs + 1] (written)
 *   slot_mapping    int64 [max_tokens] (the first sum(query_lens) written)
 *
 * Status bits, set on the device (read planner_state[1] after the stream
 * has run; when any bit is set by a call, that call wrote nothing else and
 * left the head as it was):
 *   1  the queue holds fewer blocks than the step needs
 *   2  a sequence would need more than max_blocks_per_seq blocks
 *   4  sum(query_lens) > max_tokens
 *   8  a negative count, or a sequence longer than INT32_MAX tokens
 *  16  the queue head is outside [0, queue_len]
 * Supported: block_size 16; num_seqs up to 16384 (more returns
 * PA_ERR_UNSUPPORTED).  Entries of a row below num_computed's blocks are read
 * for the slots but not checked against the pool (pa_reshape_and_cache skips
 * slots outside it).
 */
int pa_plan_step(const int32_t* free_queue, int queue_len, int32_t* planner_state,
                 const int32_t* num_computed, const int32_t* query_lens, int num_seqs,
                 int32_t* block_tables, int max_blocks_per_seq, int block_size,
                 int32_t* seq_lens, int32_t* query_start_loc, int64_t* slot_mapping,
                 int max_tokens, struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
