// attention_simple.cu -- CUDA-core paged attention, one warp per query row.
//
// Runs the fp32 steps (fp32 tensor cores would round operands to tf32, too
// coarse for an fp32 result), one warp per (query token, q-head).  Page
// "LLM推論エンジンvLLMの内部構造を徹底解説", section "PagedAttentionの仕組み": the
// warp finds its sequence in the flattened super-sequence from
// query_start_loc, takes its position seq_len - q_len + j, and walks that
// sequence's keys 0..position through the block table in chunks of 32 (one
// key per lane), with an online (running max / running sum) softmax in fp32.
#include <math.h>

#include "pa_internal.cuh"

namespace pa {
namespace {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// index of the last sequence whose query rows start at or before token tok
__device__ __forceinline__ int find_sequence(const int32_t* qsl, int num_seqs, int tok) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (qsl[mid] <= tok) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) attention_simple_kernel(const AttnParams p,
                                                               int min_rows_per_kv_head) {
  constexpr int kPerLane = D / 32;
  __shared__ float q_sh[4][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;
  if (row >= (int64_t)p.num_tokens * p.num_q_heads) return;
  const int tok = (int)(row / p.num_q_heads);
  const int head = (int)(row % p.num_q_heads);
  const int s = find_sequence(p.query_start_loc, p.num_seqs, tok);
  const int q0 = p.query_start_loc[s];
  const int ql = p.query_start_loc[s + 1] - q0;
  const int L = p.seq_lens[s];
  if (tok < q0 || tok >= q0 + ql || ql > L) return;
  if ((L + kBlockSize - 1) / kBlockSize > p.max_blocks_per_seq) return;  // beyond its table row
  if (ql * p.group <= min_rows_per_kv_head) return;  // handled by the decode kernel
  const int pos = L - ql + (tok - q0);  // last visible key
  const int kvh = head / p.group;
  const T* q = (const T*)p.q + ((int64_t)tok * p.num_q_heads + head) * D;
  const T* kc = (const T*)p.k_cache;
  const T* vc = (const T*)p.v_cache;
  const int32_t* table = p.block_tables + (int64_t)s * p.max_blocks_per_seq;

  for (int d = lane; d < D; d += 32) q_sh[warp][d] = to_f32(q[d]);
  __syncwarp();

  float m = -INFINITY, l = 0.f;
  float acc[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) acc[i] = 0.f;

  for (int t0 = 0; t0 <= pos; t0 += 32) {
    const int t = t0 + lane;
    float x = -INFINITY;
    int64_t my_row = -1;  // element offset of key t's row in the caches
    if (t <= pos) {
      const int blk = table[t / kBlockSize];
      if (blk >= 0 && blk < p.num_blocks) {
        my_row = (((int64_t)blk * p.num_kv_heads + kvh) * kBlockSize + t % kBlockSize) * D;
        const T* kr = kc + my_row;
        float dot = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) dot = fmaf(q_sh[warp][d], to_f32(kr[d]), dot);
        x = dot * p.scale;
      }
    }
    float cm = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    const float m_new = fmaxf(m, cm);
    if (m_new == -INFINITY) continue;  // nothing visible in this chunk yet
    const float alpha = expf(m - m_new);
    const float pw = (x == -INFINITY) ? 0.f : expf(x - m_new);
    float ps = pw;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * alpha + ps;
    m = m_new;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) acc[i] *= alpha;
    const int nk = min(32, pos + 1 - t0);
    for (int kk = 0; kk < nk; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, pw, kk);
      const int64_t rk = __shfl_sync(0xffffffffu, my_row, kk);
      if (rk < 0) continue;
      const T* vr = vc + rk;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) acc[i] = fmaf(pk, to_f32(vr[lane + 32 * i]), acc[i]);
    }
  }
  T* o = (T*)p.out + ((int64_t)tok * p.num_q_heads + head) * D;
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) o[lane + 32 * i] = from_f32<T>(acc[i] * inv);
}

}  // namespace

cudaError_t launch_attention_simple(const AttnParams& p, int head_dim, bool is_bf16,
                                    int min_rows_per_kv_head, cudaStream_t stream) {
  const int64_t rows = (int64_t)p.num_tokens * p.num_q_heads;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 3) / 4);
  if (is_bf16) {
    if (head_dim == 64)
      attention_simple_kernel<__nv_bfloat16, 64><<<grid, 128, 0, stream>>>(p, min_rows_per_kv_head);
    else
      attention_simple_kernel<__nv_bfloat16, 128><<<grid, 128, 0, stream>>>(p, min_rows_per_kv_head);
  } else {
    if (head_dim == 64)
      attention_simple_kernel<float, 64><<<grid, 128, 0, stream>>>(p, min_rows_per_kv_head);
    else
      attention_simple_kernel<float, 128><<<grid, 128, 0, stream>>>(p, min_rows_per_kv_head);
  }
  return cudaGetLastError();
}

}  // namespace pa
