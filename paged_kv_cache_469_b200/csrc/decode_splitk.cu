// decode_splitk.cu -- bandwidth-bound paged attention for decode-class sequences.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "エンジンの中核": a decode
// step runs the newest token against the KV cache and is bound by memory
// bandwidth; section "PagedAttentionの仕組み": the keys are read block by
// block through the sequence's block table.
//
// Work split.  One CTA (4 warps) per (partition of part_tokens keys, kv-head,
// sequence).  All q-heads of the kv-head (and, for a short multi-token decode,
// all its query tokens) form the rows of one 16-row MMA tile, so every K/V
// byte is read from HBM once per kv-head.  Warp w of the CTA takes blocks
// w, w+4, ... of the partition.
//
// Per 16-token block (one (block, kv-head) tile: 16 x D bf16, contiguous):
//   S[16 rows x 16 keys]  = Q . K^T    two mma.m16n8k16 per 16 dims of D
//   online softmax (running max / sum in fp32, exp2 with log2(e) folded in)
//   O[16 rows x D]       += P . V      D/8 mma.m16n8k16
// Operands come straight from HBM into registers with 16-byte loads, no shared
// memory: the dot product's D axis is permuted identically on Q and K so that
// every lane's B-operand words are 8 consecutive bf16 of one key row, and the
// output's D axis is permuted so that every lane's V words are 8 consecutive
// bf16 of one key row (the permutation is undone when the output is stored).
// The next block's K/V loads are issued before the current block's math.
//
// Split-K.  A CTA reduces its 4 warps' (max, sum, O) in shared memory.  A
// sequence that fits one partition writes its output directly; otherwise each
// partition stores its fp32 partial in the workspace and bumps a per
// (sequence, kv-head) counter; the CTA that arrives last merges all partials
// and resets the counter.  No CTA ever waits for another.
#include <math.h>

#include "pa_internal.cuh"

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

__device__ __forceinline__ uint4 ldg_stream(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Output column c (0..7) of n-tile nt sits at dimension
//   64 * (nt / 8) + 8 * c + nt % 8
// so a lane that owns columns 2*q4, 2*q4+1 of every n-tile owns, per 64-wide
// half of D, the 16 consecutive dimensions 16*q4 .. 16*q4+15.
template <int D>
__device__ __forceinline__ int out_dim(int nt, int c) {
  return 64 * (nt / 8) + 8 * c + (nt % 8);
}

template <int D, bool kRows16>
__global__ void __launch_bounds__(kDecodeWarps * 32)
decode_splitk_kernel(const AttnParams p) {
  constexpr int NJ = D / 32;  // 16-byte K words per key row per lane
  constexpr int NV = D / 64;  // 16-byte V words per key row per lane
  constexpr int NT = D / 8;   // n-tiles of the P.V product
  constexpr int NC = D / 16;  // k-chunks of the Q.K^T product

  __shared__ float sh_o[kDecodeWarps][kDecodeRows][D];
  __shared__ float sh_m[kDecodeWarps][kDecodeRows];
  __shared__ float sh_l[kDecodeWarps][kDecodeRows];
  __shared__ int sh_last;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, q4 = lane & 3;
  const int s = blockIdx.z, kvh = blockIdx.y, part = blockIdx.x;

  const int q0 = p.query_start_loc[s];
  const int ql = p.query_start_loc[s + 1] - q0;
  const int L = p.seq_lens[s];
  const int G = p.group;
  const int rows = ql * G;
  if (ql <= 0 || ql > L || rows > (kRows16 ? 16 : 8)) return;
  const int P = p.part_tokens;
  const int nparts = (L + P - 1) / P;
  // a sequence longer than the bounds the workspace was sized for is left
  // unwritten rather than overrunning the workspace or its block-table row
  if (part >= nparts || nparts > p.max_parts ||
      (L + kBlockSize - 1) / kBlockSize > p.max_blocks_per_seq)
    return;
  const int t_begin = part * P;
  const int t_end = min(L, t_begin + P);
  const int blk_begin = t_begin / kBlockSize;
  const int blk_end = (t_end + kBlockSize - 1) / kBlockSize;

  const __nv_bfloat16* qg = (const __nv_bfloat16*)p.q;
  const char* kc = (const char*)p.k_cache;
  const char* vc = (const char*)p.v_cache;
  const int64_t tile_bytes = (int64_t)kBlockSize * D * 2;          // one (block, head) tile
  const int64_t blk_bytes = tile_bytes * p.num_kv_heads;            // one block, all heads
  const int64_t head_off = tile_bytes * kvh;

  // ---- Q as the A operand (rows r and r+8), D axis permuted as the K words
  uint32_t qa[NC][2], qb[NC][2];
  {
    const bool va = r < rows, vb = kRows16 && (r + 8) < rows;
    const int64_t ra = va ? ((int64_t)(q0 + r / G) * p.num_q_heads + kvh * G + r % G) * D : 0;
    const int64_t rb = vb ? ((int64_t)(q0 + (r + 8) / G) * p.num_q_heads + kvh * G + (r + 8) % G) * D : 0;
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
  const int lim_a = L - ql + min(r, rows - 1) / G;
  const int lim_b = L - ql + min(r + 8, rows - 1) / G;
  const int first_masked = L - ql + 1;  // keys at or beyond this may be masked for some row

  // ---- this warp's block ids, one per lane (lane i <-> i-th block of the warp)
  const int32_t* table = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
  const int my_nblk = (blk_end - blk_begin - warp + kDecodeWarps - 1) / kDecodeWarps;
  int my_id = 0;
  if (lane < my_nblk) my_id = table[blk_begin + warp + kDecodeWarps * lane];

  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  uint4 kw[2][NJ], vw[4][NV];
  auto load_block = [&](int i, uint4 (&kd)[2][NJ], uint4 (&vd)[4][NV]) {
    int id = __shfl_sync(0xffffffffu, my_id, i);
    if (id < 0 || id >= p.num_blocks) id = 0;  // never dereference outside the pool
    const char* kt = kc + id * blk_bytes + head_off;
    const char* vt = vc + id * blk_bytes + head_off;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int jp = 0; jp < NJ; ++jp)
        kd[h][jp] = ldg_stream(kt + ((8 * h + r) * D + 32 * jp + 8 * q4) * 2);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 2 * q4 + (e & 1) + 8 * (e >> 1);
#pragma unroll
      for (int u = 0; u < NV; ++u) vd[e][u] = ldg_stream(vt + (tok * D + 64 * u + 8 * r) * 2);
    }
  };

  if (my_nblk > 0) load_block(0, kw, vw);
  for (int i = 0; i < my_nblk; ++i) {
    uint4 kn[2][NJ], vn[4][NV];
    const bool has_next = i + 1 < my_nblk;
    if (has_next) load_block(i + 1, kn, vn);
    const int blk = blk_begin + warp + kDecodeWarps * i;
    const int id_raw = __shfl_sync(0xffffffffu, my_id, i);
    const bool blk_ok = id_raw >= 0 && id_raw < p.num_blocks;

    // ---- S = Q K^T (two 8-key halves of the block)
    float sc[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      sc[h][0] = sc[h][1] = sc[h][2] = sc[h][3] = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const uint4& kx = kw[h][c / 2];
        const uint32_t b0 = (c & 1) ? kx.z : kx.x;
        const uint32_t b1 = (c & 1) ? kx.w : kx.y;
        mma_16816(sc[h], qa[c][0], kRows16 ? qb[c][0] : 0u, qa[c][1], kRows16 ? qb[c][1] : 0u,
                  b0, b1);
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
    if (has_next) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int jp = 0; jp < NJ; ++jp) kw[h][jp] = kn[h][jp];
#pragma unroll
      for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int u = 0; u < NV; ++u) vw[e][u] = vn[e][u];
    }
  }

  // ---- per-warp results to shared memory (row sums reduced over the quad)
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  if (kRows16) {
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  }
  if (q4 == 0) {
    sh_m[warp][r] = m_a; sh_l[warp][r] = l_a;
    sh_m[warp][r + 8] = m_b; sh_l[warp][r + 8] = l_b;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int d = out_dim<D>(nt, 2 * q4 + c);
      sh_o[warp][r][d] = o[nt][c];
      if (kRows16) sh_o[warp][r + 8][d] = o[nt][2 + c];
    }
  }
  __syncthreads();

  // ---- merge the 4 warps: row-wise max, rescaled sums
  const int unit = s * p.num_kv_heads + kvh;
  const bool direct = (nparts == 1);
  __nv_bfloat16* out = (__nv_bfloat16*)p.out;
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
    const int row = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sh_m[w][row]);
    const float base = (M == -INFINITY) ? 0.f : M;
    float Ls = 0.f, Os = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float f = exp2f(sh_m[w][row] - base);
      Ls += sh_l[w][row] * f;
      Os += sh_o[w][row][d] * f;
    }
    if (direct) {
      const int tok = q0 + row / G, head = kvh * G + row % G;
      out[((int64_t)tok * p.num_q_heads + head) * D + d] =
          __float2bfloat16_rn(Ls > 0.f ? Os / Ls : 0.f);
    } else {
      const int64_t slot = ((int64_t)unit * p.max_parts + part) * kDecodeRows + row;
      p.ws_o[slot * D + d] = Os;
      if (d == 0) { p.ws_ml[slot * 2] = M; p.ws_ml[slot * 2 + 1] = Ls; }
    }
  }
  if (direct) return;

  // ---- split-K: the last partition to arrive merges every partition's partial
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.ws_counter + unit, 1);
    sh_last = (prev == nparts - 1);
    if (sh_last) __threadfence();
  }
  __syncthreads();
  if (!sh_last) return;
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
    const int row = idx / D, d = idx % D;
    const int64_t base_slot = (int64_t)unit * p.max_parts * kDecodeRows + row;
    float M = -INFINITY;
    for (int q = 0; q < nparts; ++q)
      M = fmaxf(M, __ldcg(p.ws_ml + (base_slot + (int64_t)q * kDecodeRows) * 2));
    const float base = (M == -INFINITY) ? 0.f : M;
    float Ls = 0.f, Os = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const int64_t slot = base_slot + (int64_t)q * kDecodeRows;
      const float f = exp2f(__ldcg(p.ws_ml + slot * 2) - base);
      Ls += __ldcg(p.ws_ml + slot * 2 + 1) * f;
      Os += __ldcg(p.ws_o + slot * D + d) * f;
    }
    const int tok = q0 + row / G, head = kvh * G + row % G;
    out[((int64_t)tok * p.num_q_heads + head) * D + d] =
        __float2bfloat16_rn(Ls > 0.f ? Os / Ls : 0.f);
  }
  if (threadIdx.x == 0) p.ws_counter[unit] = 0;  // ready for the next call
}

}  // namespace

cudaError_t launch_decode_splitk(const AttnParams& p, int head_dim, int max_query_len,
                                 cudaStream_t stream) {
  if (p.num_seqs == 0) return cudaSuccess;
  const int max_rows = min(max_query_len * p.group, kDecodeRows);
  const bool rows16 = max_rows > 8;
  dim3 grid(p.max_parts, p.num_kv_heads, p.num_seqs);
  dim3 block(kDecodeWarps * 32);
  if (head_dim == 64) {
    if (rows16) decode_splitk_kernel<64, true><<<grid, block, 0, stream>>>(p);
    else decode_splitk_kernel<64, false><<<grid, block, 0, stream>>>(p);
  } else {
    if (rows16) decode_splitk_kernel<128, true><<<grid, block, 0, stream>>>(p);
    else decode_splitk_kernel<128, false><<<grid, block, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace pa
