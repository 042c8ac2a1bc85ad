// decode_splitk.cu -- bandwidth-bound paged attention for decode-class sequences.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "エンジンの中核": a decode
// step runs the newest token against the KV cache and is bound by memory
// bandwidth; section "PagedAttentionの仕組み": the keys are read block by
// block through the sequence's block table.
//
// Work split.  One CTA (kWarps warps) per (partition, kv-head and row group,
// sequence): a sequence of L keys is cut into ceil(L / part_tokens)
// partitions of equal whole blocks; the hardware hands CTAs to SMs as they
// free up.  The query rows of a (sequence, kv-head) -- all q-heads of the
// kv-head times its query tokens, up to 64 -- are cut into 16-row groups, each
// the rows of one 16-row MMA tile in its own CTA; a single-token decode with
// up to 16 q-heads per kv-head is one group, so every K/V byte is read from
// HBM once per kv-head.  Warp w of the CTA takes blocks w, w+kWarps, ... of
// the partition.
//
// Staging.  Each warp streams its blocks through a private ring of kStages
// shared-memory slots (one (block, kv-head) K tile + V tile per slot) with
// 16-byte cp.async copies, kStages-1 blocks in flight ahead of the math.  The
// 16-byte chunks of every tile row are XOR-swizzled on the way in so that the
// fragment reads below hit 32 distinct banks.
//
// Per 16-token block:
//   S[16 rows x 16 keys]  = Q . K^T    mma.m16n8k16, two per 16 dims of D
//   online softmax (running max / sum in fp32, exp2 with log2(e) folded in)
//   O[16 rows x D]       += P . V      D/8 mma.m16n8k16
// The dot product's D axis is permuted identically on Q and K so that every
// lane's B-operand words are 8 consecutive bf16 of one key row, and the
// output's D axis is permuted so that every lane's V words are 8 consecutive
// bf16 of one key row (undone when the output is stored).
//
// Split-K.  A CTA reduces its warps' (max, sum, O) in shared memory.  A
// sequence that fits one partition writes its output directly; otherwise each
// partition stores its fp32 partial in the workspace and bumps a per
// (sequence, kv-head, row group) counter; the CTA that arrives last merges
// all partials and resets the counter.  No CTA ever waits for another.
//
// The kernel is launched as a programmatic dependent of whatever precedes it
// on the stream (typically the cache write), so its launch overlaps that
// kernel's tail; it reads nothing before griddepcontrol.wait.  In the
// one-call form (kWriteCache) it first stores the step's new K/V rows that
// fall in its own partition into their cache slots, then reads them back.
#include <math.h>

#include "pa_internal.cuh"

// ring slots per warp (shared memory per CTA: warps x stages x 2 tiles)
#ifndef PA_DECODE_STAGES_D64
#define PA_DECODE_STAGES_D64 4
#endif
#ifndef PA_DECODE_STAGES_D128
#define PA_DECODE_STAGES_D128 3
#endif

namespace pa {
namespace {

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async16(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// XOR applied to the 16-byte chunk index of tile row `row` (K and V tiles).
// K rows are read two at a time (rows 2k, 2k+1, chunk 4j..4j+3): flip the
// half of the 128-byte line on odd rows.  V rows are read four at a time
// (rows of equal parity), one chunk each: spread them by row bits 1-2.
__device__ __forceinline__ int k_swz(int row) { return (row & 1) << 2; }
__device__ __forceinline__ int v_swz(int row) { return row & 6; }

// Output column c (0..7) of n-tile nt sits at dimension 64*(nt/8) + 8*c + nt%8,
// so a lane owning columns 2*q4, 2*q4+1 of every n-tile owns, per 64-wide
// half of D, the 16 consecutive dimensions 16*q4 .. 16*q4+15.
__device__ __forceinline__ int out_dim(int nt, int c) { return 64 * (nt / 8) + 8 * c + (nt % 8); }

template <int D>
struct DecodeSmem {
  static constexpr int kChunks = D / 8;                 // 16-byte chunks per tile row
  static constexpr int kTileBytes = kBlockSize * D * 2;  // one (block, kv-head) tile
  static constexpr int kSlotBytes = 2 * kTileBytes;      // K tile + V tile
};

template <int D, bool kRows16, int kStages, int kWarps, bool kWriteCache>
__global__ void __launch_bounds__(kWarps * 32)
decode_splitk_kernel(const AttnParams p) {
  constexpr int NJ = D / 32;  // 16-byte K chunks per key row a lane reads
  constexpr int NV = D / 64;  // 16-byte V chunks per key row a lane reads
  constexpr int NT = D / 8;   // n-tiles of the P.V product
  constexpr int NC = D / 16;  // k-chunks of the Q.K^T product
  using SM = DecodeSmem<D>;
  constexpr int kChunks = SM::kChunks;
  constexpr int kCopies = kBlockSize * kChunks / 32;  // 16-byte copies per lane per tile

  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float sh_m[kWarps][kDecodeRows];
  __shared__ float sh_l[kWarps][kDecodeRows];
  __shared__ int sh_last;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, q4 = lane & 3;
  const int s = blockIdx.z, part = blockIdx.x;
  const int kvh = blockIdx.y / p.row_groups, rg = blockIdx.y % p.row_groups;

  // Launched as a programmatic dependent: the CTA may be resident before the
  // preceding kernel on the stream (typically the cache write) has finished;
  // nothing that kernel may write is read before this wait.  The next kernel
  // may then be launched at once: it waits for this grid in the same way.
  grid_dependency_wait();
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int q0 = p.query_start_loc[s];
  const int ql = p.query_start_loc[s + 1] - q0;
  const int L = p.seq_lens[s];
  const int G = p.group;
  // this CTA's query rows of the (sequence, kv-head): global rows row0 ..
  // row0 + rows - 1, global row i being token i / G, q-head kvh * G + i % G
  const int rows_all = ql * G;
  const int row0 = kDecodeRows * rg;
  const int rows = min(kDecodeRows, rows_all - row0);
  if (ql <= 0 || ql > L || rows_all > kDecodeMaxRows || rows <= 0 ||
      rows > (kRows16 ? 16 : 8))
    return;
  const int P = p.part_tokens;
  const int nparts = (L + P - 1) / P;
  // a sequence longer than the bounds the workspace was sized for is left
  // unwritten rather than overrunning the workspace or its block-table row
  if (part >= nparts || nparts * p.row_groups > p.max_parts || L > p.max_seq_len ||
      (L + kBlockSize - 1) / kBlockSize > p.max_blocks_per_seq)
    return;
  // nparts partitions of equal whole blocks (the last may be shorter; with
  // partitions of at least 32 blocks none is empty for up to 32 partitions,
  // and an empty one still reports (max -inf, sum 0) to the merge)
  const int nblk_seq = (L + kBlockSize - 1) / kBlockSize;
  const int pblk = (nblk_seq + nparts - 1) / nparts;
  const int blk_begin = part * pblk;
  const int blk_end = min(nblk_seq, blk_begin + pblk);

  if constexpr (kWriteCache) {
    // This step's new tokens of the sequence that fall in this partition's
    // key range go into their cache slots first (as pa_reshape_and_cache
    // would); only this CTA reads those keys of this kv-head, after the fence
    // and the barrier below.
    const int lo = max(L - ql, blk_begin * kBlockSize), hi = min(L, blk_end * kBlockSize);
    if (hi > lo) {
      constexpr int kVec = D * 2 / 16;  // 16-byte vectors per row
      const int n = (hi - lo) * kVec;
      const int64_t num_slots = (int64_t)p.num_blocks * kBlockSize;
      const uint4* kn = (const uint4*)p.k_new;
      const uint4* vn = (const uint4*)p.v_new;
      uint4* kcw = (uint4*)const_cast<void*>(p.k_cache);
      uint4* vcw = (uint4*)const_cast<void*>(p.v_cache);
      for (int i = threadIdx.x; i < 2 * n; i += blockDim.x) {
        const bool is_v = i >= n;
        const int ii = is_v ? i - n : i;
        const int j = ii / kVec, c = ii % kVec;
        const int tok = q0 + (lo - (L - ql)) + j;
        const int64_t slot = p.slot_mapping[tok];
        if (slot < 0 || slot >= num_slots) continue;  // padding / out-of-pool slot
        const int64_t dst =
            ((slot / kBlockSize * p.num_kv_heads + kvh) * kBlockSize + slot % kBlockSize) * kVec + c;
        const int64_t src = ((int64_t)tok * p.num_kv_heads + kvh) * kVec + c;
        if (is_v) vcw[dst] = vn[src];
        else kcw[dst] = kn[src];
      }
      __threadfence();
    }
    __syncthreads();
  }

  // ---- this warp's block ids, one per lane (lane i <-> i-th block of the warp)
  const int32_t* table = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
  const int my_nblk = (blk_end - blk_begin - warp + kWarps - 1) / kWarps;
  int win = -1, win_id = 0;  // block ids of the warp's blocks 32*win .. 32*win+31
  auto block_id = [&](int i) {
    if ((i >> 5) != win) {
      win = i >> 5;
      const int ii = (win << 5) + lane;
      win_id = ii < my_nblk ? table[blk_begin + warp + kWarps * ii] : 0;
    }
    return __shfl_sync(0xffffffffu, win_id, i & 31);
  };
  uint32_t bad = 0;  // bit (slot): that slot's block id was outside the pool

  // ---- Q as the A operand (rows r and r+8), D axis permuted as the K chunks
  const __nv_bfloat16* qg = (const __nv_bfloat16*)p.q;
  uint32_t qa[NC][2], qb[NC][2];
  {
    const bool va = r < rows, vb = kRows16 && (r + 8) < rows;
    const int ga = row0 + r, gb = row0 + r + 8;
    const int64_t ra = va ? ((int64_t)(q0 + ga / G) * p.num_q_heads + kvh * G + ga % G) * D : 0;
    const int64_t rb = vb ? ((int64_t)(q0 + gb / G) * p.num_q_heads + kvh * G + gb % G) * D : 0;
#pragma unroll
    for (int jp = 0; jp < NJ; ++jp) {
      uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
      if (va) xa = *reinterpret_cast<const uint4*>(qg + ra + 32 * jp + 8 * q4);
      if (vb) xb = *reinterpret_cast<const uint4*>(qg + rb + 32 * jp + 8 * q4);
      qa[2 * jp][0] = xa.x; qa[2 * jp][1] = xa.y; qa[2 * jp + 1][0] = xa.z; qa[2 * jp + 1][1] = xa.w;
      qb[2 * jp][0] = xb.x; qb[2 * jp][1] = xb.y; qb[2 * jp + 1][0] = xb.z; qb[2 * jp + 1][1] = xb.w;
    }
  }
  // causal limit of rows r and r+8: query j sees keys <= L - ql + j
  const int lim_a = L - ql + (row0 + min(r, rows - 1)) / G;
  const int lim_b = L - ql + (row0 + min(r + 8, rows - 1)) / G;
  const int first_masked = L - ql + 1;  // keys at or beyond this may be masked for some row

  const char* kc = (const char*)p.k_cache;
  const char* vc = (const char*)p.v_cache;
  const int64_t blk_bytes = (int64_t)SM::kTileBytes * p.num_kv_heads;
  const int64_t head_off = (int64_t)SM::kTileBytes * kvh;
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem) +
                        warp * kStages * SM::kSlotBytes;

  auto issue = [&](int i) {  // copy the warp's i-th block into slot i % kStages
    int id = block_id(i);
    if (id < 0 || id >= p.num_blocks) {  // never dereference outside the pool
      id = 0;
      bad |= 1u << (i % kStages);
    } else {
      bad &= ~(1u << (i % kStages));
    }
    const char* kt = kc + id * blk_bytes + head_off;
    const char* vt = vc + id * blk_bytes + head_off;
    const uint32_t ks = ring + (i % kStages) * SM::kSlotBytes;
    const uint32_t vs = ks + SM::kTileBytes;
#pragma unroll
    for (int j = 0; j < kCopies; ++j) {
      const int idx = lane + 32 * j;
      const int row = idx / kChunks, c = idx % kChunks;
      cp_async16(ks + (row * kChunks + (c ^ k_swz(row))) * 16, kt + idx * 16);
      cp_async16(vs + (row * kChunks + (c ^ v_swz(row))) * 16, vt + idx * 16);
    }
  };

  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < my_nblk) issue(st);
    cp_async_commit();
  }

  for (int i = 0; i < my_nblk; ++i) {
    __syncwarp();  // every lane is done reading the slot the next copy overwrites
    if (i + kStages - 1 < my_nblk) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();  // this lane's copies of block i have landed
    __syncwarp();                  // ... and every other lane's

    const int blk = blk_begin + warp + kWarps * i;
    const bool blk_ok = !((bad >> (i % kStages)) & 1u);
    const uint32_t ks = ring + (i % kStages) * SM::kSlotBytes;
    const uint32_t vs = ks + SM::kTileBytes;

    // ---- S = Q K^T (two 8-key halves of the block)
    float sc[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      sc[h][0] = sc[h][1] = sc[h][2] = sc[h][3] = 0.f;
      const int row = 8 * h + r;
#pragma unroll
      for (int jp = 0; jp < NJ; ++jp) {
        const uint4 kx = lds128(ks + (row * kChunks + ((4 * jp + q4) ^ k_swz(row))) * 16);
        mma_16816(sc[h], qa[2 * jp][0], kRows16 ? qb[2 * jp][0] : 0u, qa[2 * jp][1],
                  kRows16 ? qb[2 * jp][1] : 0u, kx.x, kx.y);
        mma_16816(sc[h], qa[2 * jp + 1][0], kRows16 ? qb[2 * jp + 1][0] : 0u,
                  qa[2 * jp + 1][1], kRows16 ? qb[2 * jp + 1][1] : 0u, kx.z, kx.w);
      }
    }
    // ---- V words: keys 2q4, 2q4+1, 2q4+8, 2q4+9; 8 dims 64u+8r.. each
    uint4 vw[4][NV];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 2 * q4 + (e & 1) + 8 * (e >> 1);
#pragma unroll
      for (int u = 0; u < NV; ++u)
        vw[e][u] = lds128(vs + (tok * kChunks + ((8 * u + r) ^ v_swz(tok))) * 16);
    }
    // slots of the last block past seq_len (and blocks outside the pool) may
    // hold anything, NaN included: their V words become zeros so that the
    // zero weights below cannot turn them into NaN in the P.V product
    if (blk * kBlockSize + kBlockSize > L || !blk_ok) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = blk * kBlockSize + 2 * q4 + (e & 1) + 8 * (e >> 1);
        if (!blk_ok || key >= L) {
#pragma unroll
          for (int u = 0; u < NV; ++u) vw[e][u] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    // ---- scale, mask, online softmax
    const int key0 = blk * kBlockSize + 2 * q4;  // keys key0, +1 (half 0), key0+8, +9 (half 1)
    const bool tail = (blk * kBlockSize + kBlockSize > first_masked) || !blk_ok;
    float xa[4], xb[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = key0 + (e & 1) + 8 * (e >> 1);
      xa[e] = sc[e >> 1][e & 1] * p.scale_log2;
      xb[e] = sc[e >> 1][2 + (e & 1)] * p.scale_log2;
      if (tail) {
        if (!blk_ok || key > lim_a) xa[e] = -INFINITY;
        if (!blk_ok || key > lim_b) xb[e] = -INFINITY;
      }
    }
    float bm_a = fmaxf(fmaxf(xa[0], xa[1]), fmaxf(xa[2], xa[3]));
    bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 1));
    bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 2));
    const float mn_a = fmaxf(m_a, bm_a);
    const float base_a = (mn_a == -INFINITY) ? 0.f : mn_a;
    const float al_a = exp2f(m_a - base_a);
    float pa[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pa[e] = exp2f(xa[e] - base_a);
    l_a = l_a * al_a + (pa[0] + pa[1]) + (pa[2] + pa[3]);
    m_a = mn_a;
    float pb[4] = {0.f, 0.f, 0.f, 0.f};
    float al_b = 1.f;
    if (kRows16) {
      float bm_b = fmaxf(fmaxf(xb[0], xb[1]), fmaxf(xb[2], xb[3]));
      bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 1));
      bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 2));
      const float mn_b = fmaxf(m_b, bm_b);
      const float base_b = (mn_b == -INFINITY) ? 0.f : mn_b;
      al_b = exp2f(m_b - base_b);
#pragma unroll
      for (int e = 0; e < 4; ++e) pb[e] = exp2f(xb[e] - base_b);
      l_b = l_b * al_b + (pb[0] + pb[1]) + (pb[2] + pb[3]);
      m_b = mn_b;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      o[nt][0] *= al_a; o[nt][1] *= al_a;
      if (kRows16) { o[nt][2] *= al_b; o[nt][3] *= al_b; }
    }
    // ---- O += P V
    const uint32_t pa0 = pack_bf16x2(pa[0], pa[1]), pa2 = pack_bf16x2(pa[2], pa[3]);
    const uint32_t pb1 = kRows16 ? pack_bf16x2(pb[0], pb[1]) : 0u;
    const uint32_t pb3 = kRows16 ? pack_bf16x2(pb[2], pb[3]) : 0u;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int u = nt / 8, idx = nt % 8;
      const uint32_t sel = (idx & 1) ? 0x7632u : 0x5410u;
      const uint32_t b0 = __byte_perm(word(vw[0][u], idx >> 1), word(vw[1][u], idx >> 1), sel);
      const uint32_t b1 = __byte_perm(word(vw[2][u], idx >> 1), word(vw[3][u], idx >> 1), sel);
      mma_16816(o[nt], pa0, pb1, pa2, pb3, b0, b1);
    }
  }
  cp_async_wait<0>();  // no copy may still target the ring when it is reused below

  // ---- per-warp results to shared memory (row sums reduced over the quad)
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  if (kRows16) {
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  }
  __syncthreads();  // every warp is done with its ring
  float(*sh_o)[kDecodeRows][D] = reinterpret_cast<float(*)[kDecodeRows][D]>(smem);
  if (q4 == 0) {
    sh_m[warp][r] = m_a; sh_l[warp][r] = l_a;
    sh_m[warp][r + 8] = m_b; sh_l[warp][r + 8] = l_b;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int d = out_dim(nt, 2 * q4 + c);
      sh_o[warp][r][d] = o[nt][c];
      if (kRows16) sh_o[warp][r + 8][d] = o[nt][2 + c];
    }
  }
  __syncthreads();

  // ---- merge the warps: row-wise max, rescaled sums
  const int unit = s * p.num_kv_heads + kvh;
  const bool direct = (nparts == 1);
  __nv_bfloat16* out = (__nv_bfloat16*)p.out;
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
    const int row = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh_m[w][row]);
    const float base = (M == -INFINITY) ? 0.f : M;
    float Ls = 0.f, Os = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = exp2f(sh_m[w][row] - base);
      Ls += sh_l[w][row] * f;
      Os += sh_o[w][row][d] * f;
    }
    if (direct) {
      const int tok = q0 + (row0 + row) / G, head = kvh * G + (row0 + row) % G;
      out[((int64_t)tok * p.num_q_heads + head) * D + d] =
          __float2bfloat16_rn(Ls > 0.f ? Os / Ls : 0.f);
    } else {
      const int64_t slot =
          ((int64_t)unit * p.max_parts + part * p.row_groups + rg) * kDecodeRows + row;
      p.ws_o[slot * D + d] = Os;
      if (d == 0) { p.ws_ml[slot * 2] = M; p.ws_ml[slot * 2 + 1] = Ls; }
    }
  }
  if (direct) return;

  // ---- split-K: the last partition to arrive merges every partition's partial
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.ws_counter + unit * kDecodeRowGroups + rg, 1);
    sh_last = (prev == nparts - 1);
    if (sh_last) __threadfence();
  }
  __syncthreads();
  if (!sh_last) return;
  // every partition's (max, sum) per row into shared memory (one round of
  // loads), then the rows' weights, then one round of 16-byte partial loads
  // per output chunk (the ring is free: every warp is past its last copy)
  float* sh_pm = reinterpret_cast<float*>(smem);  // [nparts][kDecodeRows] max, then weight
  float* sh_pl = sh_pm + nparts * kDecodeRows;    // [nparts][kDecodeRows] sum
  float* sh_inv = sh_pl + nparts * kDecodeRows;   // [kDecodeRows] 1 / merged sum
  // partition q of this row group is partial slot q * row_groups + rg of the unit
  const int64_t unit_slot = ((int64_t)unit * p.max_parts + rg) * kDecodeRows;
  const int slot_step = p.row_groups * kDecodeRows;
  for (int i = threadIdx.x; i < nparts * rows; i += blockDim.x) {
    const int q = i / rows, row = i % rows;
    const float2 ml =
        __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + unit_slot + q * slot_step + row);
    sh_pm[q * kDecodeRows + row] = ml.x;
    sh_pl[q * kDecodeRows + row] = ml.y;
  }
  __syncthreads();
  if (threadIdx.x < rows) {
    const int row = threadIdx.x;
    float M = -INFINITY;
    for (int q = 0; q < nparts; ++q) M = fmaxf(M, sh_pm[q * kDecodeRows + row]);
    const float base = (M == -INFINITY) ? 0.f : M;
    float Ls = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const float f = exp2f(sh_pm[q * kDecodeRows + row] - base);
      sh_pm[q * kDecodeRows + row] = f;
      Ls += sh_pl[q * kDecodeRows + row] * f;
    }
    sh_inv[row] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  constexpr int D4 = D / 4;
  const float4* po = reinterpret_cast<const float4*>(p.ws_o);
  for (int i = threadIdx.x; i < rows * D4; i += blockDim.x) {
    const int row = i / D4, d4 = i % D4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int q = 0; q < nparts; ++q) {
      const float4 v = __ldcg(po + (unit_slot + q * slot_step + row) * D4 + d4);
      const float f = sh_pm[q * kDecodeRows + row];
      acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
    }
    const float inv = sh_inv[row];
    const int tok = q0 + (row0 + row) / G, head = kvh * G + (row0 + row) % G;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(out + ((int64_t)tok * p.num_q_heads + head) * D + 4 * d4) = pk;
  }
  if (threadIdx.x == 0) p.ws_counter[unit * kDecodeRowGroups + rg] = 0;  // ready for the next call
}

template <int D, bool kRows16, int kStages, bool kWriteCache>
cudaError_t launch_one(const AttnParams& p, cudaStream_t stream) {
  constexpr int kWarps = kDecodeWarps;
  auto kernel = decode_splitk_kernel<D, kRows16, kStages, kWarps, kWriteCache>;
  const int ring = kWarps * kStages * DecodeSmem<D>::kSlotBytes;
  const int merge = kWarps * kDecodeRows * D * (int)sizeof(float);
  // the cross-partition merge: (max, sum) per partition and row, 1 / sum per row
  const int split = (2 * p.max_parts + 1) * kDecodeRows * (int)sizeof(float);
  int smem = ring > merge ? ring : merge;
  if (split > smem) smem = split;
  static std::atomic<int> smem_done[64];
  cudaError_t e = raise_smem_limit(kernel, smem, smem_done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  const int parts = (p.max_seq_len + p.part_tokens - 1) / p.part_tokens;  // <= p.max_parts
  cfg.gridDim = dim3(parts > 0 ? parts : 1, p.num_kv_heads * p.row_groups, p.num_seqs);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int D, bool kRows16, int kStages>
int wave_ctas_one() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  constexpr int kWarps = kDecodeWarps;
  const int ring = kWarps * kStages * DecodeSmem<D>::kSlotBytes;
  const int merge = kWarps * kDecodeRows * D * (int)sizeof(float);
  int per_sm = 0, sms = 0;
  auto kernel = decode_splitk_kernel<D, kRows16, kStages, kWarps, false>;
  static std::atomic<int> smem_done[64];
  raise_smem_limit(kernel, ring > merge ? ring : merge, smem_done);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarps * 32,
                                                    ring > merge ? ring : merge) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 2 * 148;
  n = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 148);
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace

int decode_wave_ctas(int head_dim, int rows) {
  constexpr int s64 = PA_DECODE_STAGES_D64, s128 = PA_DECODE_STAGES_D128;
  if (head_dim == 64)
    return rows > 8 ? wave_ctas_one<64, true, s64>() : wave_ctas_one<64, false, s64>();
  return rows > 8 ? wave_ctas_one<128, true, s128>() : wave_ctas_one<128, false, s128>();
}

cudaError_t launch_decode_splitk(const AttnParams& p, int head_dim, int max_query_len,
                                 cudaStream_t stream) {
  if (p.num_seqs == 0) return cudaSuccess;
  const int max_rows = min(p.decode_rows > 0 ? p.decode_rows : max_query_len * p.group,
                           kDecodeRows);
  const bool rows16 = max_rows > 8;
  cudaError_t e;
  constexpr int s64 = PA_DECODE_STAGES_D64, s128 = PA_DECODE_STAGES_D128;
  const bool wc = p.slot_mapping != nullptr;
  if (head_dim == 64)
    e = rows16 ? (wc ? launch_one<64, true, s64, true>(p, stream)
                     : launch_one<64, true, s64, false>(p, stream))
               : (wc ? launch_one<64, false, s64, true>(p, stream)
                     : launch_one<64, false, s64, false>(p, stream));
  else
    e = rows16 ? (wc ? launch_one<128, true, s128, true>(p, stream)
                     : launch_one<128, true, s128, false>(p, stream))
               : (wc ? launch_one<128, false, s128, true>(p, stream)
                     : launch_one<128, false, s128, false>(p, stream));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pa
