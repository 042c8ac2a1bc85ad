// plan_step.cu -- a scheduler step's block allocation and device inputs, on the GPU.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "PagedAttentionの仕組み":
// a request of n tokens holds ceil(n / 16) blocks; allocate_slots counts the
// blocks a request needs and takes them from the front of free_block_queue
// into the request's block list (req_to_blocks), requests in order; the
// step's sequences are laid end to end as one super-sequence, and every new
// token is written to the slot of its position (block_table[p / 16] * 16 +
// p % 16).  Here the whole step does that in one launch, so a decode loop
// needs no host round trip between steps: sequence s already owns the blocks
// of its first num_computed[s] tokens and schedules query_lens[s] more.
//
// Every CTA scans the per-sequence counts (block-wide prefix sums over the
// sequences, in chunks of the block size) into shared memory, so all of them
// agree on the step's totals and on every sequence's offsets; then the CTAs
// split the writes: seq_lens and query_start_loc by sequence, the appended
// table entries by their index in the queue, the slots by token, each found
// by a binary search over the prefix sums.  The queue head is read by every
// CTA and advanced by the last one to finish (an arrival counter), so no CTA
// reads it after it has moved.  A step that does not fit (pool, row, slot
// buffer) writes nothing but a status bit.
#include "pa_internal.cuh"

namespace pa {
namespace {

constexpr int kPlanThreads = 1024;

// exclusive prefix sums of a and b over the block (kPlanThreads threads);
// returns the block totals in *ta, *tb
__device__ __forceinline__ void block_scan2(long long a, long long b, long long* ea,
                                            long long* eb, long long* ta, long long* tb,
                                            long long (*warp_tot)[2]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long ia = a, ib = b;  // inclusive within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long xa = __shfl_up_sync(0xffffffffu, ia, o);
    const long long xb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) ia += xa, ib += xb;
  }
  if (lane == 31) warp_tot[warp][0] = ia, warp_tot[warp][1] = ib;
  __syncthreads();
  if (warp == 0) {
    long long wa = warp_tot[lane][0], wb = warp_tot[lane][1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long xa = __shfl_up_sync(0xffffffffu, wa, o);
      const long long xb = __shfl_up_sync(0xffffffffu, wb, o);
      if (lane >= o) wa += xa, wb += xb;
    }
    warp_tot[lane][0] = wa, warp_tot[lane][1] = wb;  // inclusive over warps
  }
  __syncthreads();
  const long long pa_ = warp ? warp_tot[warp - 1][0] : 0, pb = warp ? warp_tot[warp - 1][1] : 0;
  *ea = pa_ + ia - a;
  *eb = pb + ib - b;
  *ta = warp_tot[31][0];
  *tb = warp_tot[31][1];
  __syncthreads();  // warp_tot is reused by the next chunk
}

// first index u in [0, n] with v[u] > x (v nondecreasing, v[n] > x)
__device__ __forceinline__ int upper_bound(const int* v, int n, long long x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (v[mid] > x) hi = mid; else lo = mid + 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kPlanThreads)
plan_step_kernel(const int32_t* __restrict__ free_queue, int queue_len, int32_t* state,
                 const int32_t* __restrict__ num_computed, const int32_t* __restrict__ query_lens,
                 int num_seqs, int32_t* block_tables, int max_blocks_per_seq,
                 int32_t* __restrict__ seq_lens, int32_t* __restrict__ query_start_loc,
                 int64_t* __restrict__ slot_mapping, int max_tokens) {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // inputs may come from the previous kernel on the stream (e.g. the last
  // step's seq_lens as this step's num_computed)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  extern __shared__ int plan_smem[];
  int* s_qsl = plan_smem;                     // [S+1] query_start_loc
  int* s_take = s_qsl + (num_seqs + 1);       // [S+1] first new block's queue offset
  int* s_nc = s_take + (num_seqs + 1);        // [S]   num_computed
  __shared__ long long warp_tot[32][2];
  __shared__ int s_head, s_bad;

  if (threadIdx.x == 0) {
    s_head = *(volatile int32_t*)&state[kPlanStateHead];
    s_bad = 0;
  }
  __syncthreads();
  long long carry_q = 0, carry_n = 0;
  int bad = 0;
  for (int base = 0; base < num_seqs; base += kPlanThreads) {
    const int s = base + threadIdx.x;
    long long ql = 0, need = 0;
    if (s < num_seqs) {
      const long long nc = num_computed[s];
      ql = query_lens[s];
      const long long L = nc + ql;
      if (nc < 0 || ql < 0 || L > 0x7fffffffLL) {
        bad |= kPlanBadLength;
        ql = 0;
      } else {
        const long long nb_old = (nc + kBlockSize - 1) / kBlockSize;
        const long long nb_new = (L + kBlockSize - 1) / kBlockSize;
        if (nb_new > max_blocks_per_seq) bad |= kPlanRowFull;
        need = nb_new - nb_old;
      }
      s_nc[s] = (int)max(0LL, nc);
    }
    long long eq, en, tq, tn;
    block_scan2(ql, need, &eq, &en, &tq, &tn, warp_tot);
    if (s < num_seqs) {
      // stored as int only when the totals fit (checked below before use)
      s_qsl[s] = (int)(carry_q + eq);
      s_take[s] = (int)(carry_n + en);
    }
    carry_q += tq;
    carry_n += tn;
  }
  // the block's error bits (a bitwise OR: each kind keeps its own bit)
  bad = (int)__reduce_or_sync(0xffffffffu, (unsigned)bad);
  if ((threadIdx.x & 31) == 0 && bad) atomicOr(&s_bad, bad);
  __syncthreads();  // also orders s_head and the scans for every thread
  bad = s_bad;
  const int head = s_head;
  const long long total_q = carry_q, total_n = carry_n;
  if (head < 0 || head > queue_len) bad |= kPlanBadHead;
  else if (total_n > (long long)(queue_len - head)) bad |= kPlanPoolEmpty;
  if (total_q > max_tokens) bad |= kPlanSlotsFull;
  if (bad) {
    // every CTA reaches the same verdict; one records it and nothing is written
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&state[kPlanStateStatus], bad);
    return;
  }
  if (threadIdx.x == 0) {
    s_qsl[num_seqs] = (int)total_q;
    s_take[num_seqs] = (int)total_n;
  }
  __syncthreads();

  const long long gthreads = (long long)gridDim.x * kPlanThreads;
  const long long gtid = (long long)blockIdx.x * kPlanThreads + threadIdx.x;
  // seq_lens and query_start_loc
  for (long long s = gtid; s <= num_seqs; s += gthreads) {
    query_start_loc[s] = s_qsl[s];
    if (s < num_seqs) seq_lens[s] = s_nc[s] + (s_qsl[s + 1] - s_qsl[s]);
  }
  // the new blocks: queue entries head .. head + total_n - 1, in sequence order
  for (long long j = gtid; j < total_n; j += gthreads) {
    const int s = upper_bound(s_take, num_seqs, j) - 1;
    const int nb_old = (s_nc[s] + kBlockSize - 1) / kBlockSize;
    block_tables[(long long)s * max_blocks_per_seq + nb_old + (j - s_take[s])] =
        free_queue[head + j];
  }
  // slots of the scheduled tokens (positions num_computed[s] .. seq_lens[s] - 1)
  for (long long i = gtid; i < total_q; i += gthreads) {
    const int s = upper_bound(s_qsl, num_seqs, i) - 1;
    const int nc = s_nc[s];
    const int pos = nc + (int)(i - s_qsl[s]);
    const int lb = pos / kBlockSize;
    const int nb_old = (nc + kBlockSize - 1) / kBlockSize;
    // an existing block comes from the table, a new one straight from the queue
    // (the table entry is being written by another thread of this launch)
    const int blk = lb < nb_old ? block_tables[(long long)s * max_blocks_per_seq + lb]
                                : free_queue[head + s_take[s] + (lb - nb_old)];
    slot_mapping[i] = (int64_t)blk * kBlockSize + pos % kBlockSize;
  }

  // the last CTA to arrive advances the queue head: every CTA has read it by then
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int arrived = atomicAdd(&state[kPlanStateArrivals], 1);
    if (arrived == (int)gridDim.x - 1) {
      state[kPlanStateHead] = head + (int)total_n;
      state[kPlanStateArrivals] = 0;
      __threadfence();
    }
  }
}

}  // namespace

size_t plan_step_smem(int num_seqs) { return (size_t)(3 * num_seqs + 2) * sizeof(int); }

cudaError_t launch_plan_step(const int32_t* free_queue, int queue_len, int32_t* state,
                             const int32_t* num_computed, const int32_t* query_lens,
                             int num_seqs, int32_t* block_tables, int max_blocks_per_seq,
                             int32_t* seq_lens, int32_t* query_start_loc,
                             int64_t* slot_mapping, int max_tokens, cudaStream_t stream) {
  // enough CTAs that each writes at most about two slots per thread
  const long long work = max((long long)max_tokens, 1LL);
  const int grid = (int)min((long long)device_sm_count(),
                            (work + 2 * kPlanThreads - 1) / (2 * kPlanThreads));
  const int smem = (int)plan_step_smem(num_seqs);
  if (smem > 48 * 1024) {
    static std::atomic<int> done[64];
    cudaError_t e = raise_smem_limit(plan_step_kernel, smem, done);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max(grid, 1));
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, plan_step_kernel, free_queue, queue_len, state,
                                     num_computed, query_lens, num_seqs, block_tables,
                                     max_blocks_per_seq, seq_lens, query_start_loc,
                                     slot_mapping, max_tokens);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pa
