// prefill_tcgen05.cu -- tensor-core paged attention for prefill chunks.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説": section "エンジンの中核" -- a
// prefill runs the whole prompt and is compute-bound; section "高度な機能群"
// -- a chunked prefill attends to the context already cached before the chunk
// as well as to itself; section "PagedAttentionの仕組み" -- keys are read
// through the sequence's block table and a causal, position-based mask keeps
// each query on its own sequence's earlier tokens.
//
// Work item = (sequence, 128-query tile, q-head).  A persistent CTA walks its
// items; per item it streams the sequence's keys in 128-key tiles:
//
//   warp 0      TMA producer: Q tile once per item, then K and V tiles, each
//               tile eight 16-token cache blocks (one 16 x 64 box per block and
//               64-wide slice of D, 128-byte swizzled, straight from the pool
//               through the block table)
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (tcgen05.mma,
//               M=128, N=128, K=16 steps), then O += P V into TMEM
//   warps 2..5  softmax: one query row per thread; S from TMEM (tcgen05.ld),
//               causal mask, online softmax in fp32 (exp2, the running max is
//               only moved when it grows by more than 2^8, so O is rarely
//               rescaled), P as bf16 into shared memory for the second MMA;
//               at the end of the item O / l from TMEM to global memory
//
// S is double-buffered in TMEM so that Q K^T of tile j+1 overlaps the softmax
// of tile j.  The last, partly filled cache block of a sequence is loaded at a
// negative row offset so that its unwritten slots arrive as TMA zero fill
// (never uninitialised cache memory); blocks past the sequence, or block ids
// outside the pool, are loaded from beyond the tensor's extent (zeros).
//
// Every mbarrier wait is bounded by a time limit; a wait that runs out sets a
// status bit in the workspace and the CTA winds down instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "pa_internal.cuh"

namespace pa {
namespace {

constexpr int QT = kPrefillQTile;               // 128 query rows per item
constexpr int KT = kPrefillKvTile;              // 128 keys per tile
constexpr int kTileBlocks = KT / kBlockSize;    // 8 cache blocks per tile
constexpr int kKStages = 2, kVStages = 2;
constexpr int kThreads = 192;                   // 6 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;                  // S buffers at columns 0 and 128
constexpr uint32_t kTmemO = 256;                // O at columns 256 .. 256+D
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s
constexpr float kRescaleThreshold = 8.0f;       // log2 units: move the max only past 2^8

template <int D>
struct PrefillLayout {
  static constexpr int kPanels = D / 64;            // 64-wide slices of D
  static constexpr int kPanelBytes = 128 * 128;     // 128 rows x 128 bytes
  static constexpr int kQBytes = kPanels * kPanelBytes;
  static constexpr int kKvBytes = kPanels * kPanelBytes;
  static constexpr int kPBytes = 2 * kPanelBytes;   // 128 rows x 128 keys bf16
  static constexpr int q_off = 0;
  static constexpr int k_off = q_off + kQBytes;
  static constexpr int v_off = k_off + kKStages * kKvBytes;
  static constexpr int p_off = v_off + kVStages * kKvBytes;
  static constexpr int bar_off = p_off + kPBytes;
  static constexpr int used = bar_off + 256;
  // D = 64 would fit two CTAs per SM, whose TMEM allocations would then queue
  // behind each other: ask for enough shared memory to keep one CTA per SM.
  static constexpr int total = (used < 120 * 1024 ? 120 * 1024 : used) + 1024;
};

// mbarrier indices
enum : int {
  kBarQFull = 0, kBarQEmpty, kBarKFull0, kBarKFull1, kBarKEmpty0, kBarKEmpty1, kBarVFull0,
  kBarVFull1, kBarVEmpty0, kBarVEmpty1, kBarSFull0, kBarSFull1, kBarPFull, kBarODone, kNumBars
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with parity `parity` to complete.  Gives up
// (returns false) when another role of the CTA has given up, or after the time
// limit, in which case it records the timeout in the workspace status word.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

#define PA_R32(r)                                                                           \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),       \
      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),          \
      "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),          \
      "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define PA_W32(r)                                                                          \
  "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),   \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),      \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),    \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),    \
      "r"(r[29]), "r"(r[30]), "r"(r[31])

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : PA_R32(r)
      : "r"(taddr));
}
// 32 consecutive fp32 columns into elements OFF .. OFF+31 of a larger array
template <int OFF, int N>
__device__ __forceinline__ void tmem_ld32_at(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(OFF + 32 <= N, "tmem_ld32_at out of range");
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]),
        "=r"(r[OFF + 4]), "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]),
        "=r"(r[OFF + 8]), "=r"(r[OFF + 9]), "=r"(r[OFF + 10]), "=r"(r[OFF + 11]),
        "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]), "=r"(r[OFF + 15]),
        "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]),
        "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]),
        "=r"(r[OFF + 24]), "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]),
        "=r"(r[OFF + 28]), "=r"(r[OFF + 29]), "=r"(r[OFF + 30]), "=r"(r[OFF + 31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      PA_W32(r)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor (tcgen05): 128-byte swizzle, start address,
// leading / stride byte offsets (all in 16-byte units), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with bf16 operands and an fp32 accumulator.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
         ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct ItemInfo {
  int seq, qtile, head, ntiles;
  int q0, ql, L;
};

__device__ __forceinline__ ItemInfo load_item(const AttnParams& p, int w) {
  const int4 it = p.ws_items[1 + w];
  ItemInfo r;
  r.seq = it.x; r.qtile = it.y; r.head = it.z; r.ntiles = it.w;
  r.q0 = p.query_start_loc[r.seq];
  r.ql = p.query_start_loc[r.seq + 1] - r.q0;
  r.L = p.seq_lens[r.seq];
  return r;
}

// item index of the k-th item of CTA c (boustrophedon over rounds of gridDim)
__device__ __forceinline__ int item_index(int k) {
  const int g = gridDim.x, c = blockIdx.x;
  return k * g + ((k & 1) ? (g - 1 - c) : c);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tcgen05_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v) {
  using LY = PrefillLayout<D>;
  constexpr int kPanels = LY::kPanels;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t sh_tmem_base;
  __shared__ int sh_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = ((uint32_t)__cvta_generic_to_shared(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + LY::q_off, sK = base + LY::k_off, sV = base + LY::v_off,
                 sP = base + LY::p_off, sBar = base + LY::bar_off;
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = &sh_abort;

  if (threadIdx.x == 0) {
    sh_abort = 0;
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarKFull0 + i), 1);
      mbar_init(bar(kBarKEmpty0 + i), 1);
      mbar_init(bar(kBarVFull0 + i), 1);
      mbar_init(bar(kBarVEmpty0 + i), 1);
      mbar_init(bar(kBarSFull0 + i), 1);
    }
    mbar_init(bar(kBarPFull), 4);  // one arrival per softmax warp
    mbar_init(bar(kBarODone), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc((uint32_t)__cvta_generic_to_shared(&sh_tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh_tmem_base;

  // the work list and the cache must be complete before anything reads them
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int num_items = p.ws_items[0].x;
  int* status = p.ws_status;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    const int oob_bh = p.num_blocks * p.num_kv_heads;  // first block-head row past the pool
    uint32_t g = 0;                                     // global tile counter
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k);
      if (w >= num_items) break;
      const ItemInfo it = load_item(p, w);
      const int kvh = it.head / p.group;
      const int nblk = (it.L + kBlockSize - 1) / kBlockSize;
      const int shift = nblk * kBlockSize - it.L;  // unwritten slots of the last block
      const int32_t* table = p.block_tables + (int64_t)it.seq * p.max_blocks_per_seq;
      // ---- Q tile
      if (lane == 0) {
        if (k > 0) ok = wait_bar(bar(kBarQEmpty), (k - 1) & 1, abort_flag, status);
        if (ok) {
          mbar_expect_tx(bar(kBarQFull), LY::kQBytes);
          for (int pn = 0; pn < kPanels; ++pn)
            tma_load_3d(sQ + pn * LY::kPanelBytes, &tm_q, 64 * pn, it.head,
                        it.q0 + it.qtile * QT, bar(kBarQFull));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // ---- K and V tiles
      for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
        int id = -1;
        const int lb = t * kTileBlocks + lane;
        if (lane < kTileBlocks && lb < nblk && lb < p.max_blocks_per_seq) id = table[lb];
        int c1[kTileBlocks], c2[kTileBlocks];
#pragma unroll
        for (int b = 0; b < kTileBlocks; ++b) {
          const int idb = __shfl_sync(0xffffffffu, id, b);
          const int lbb = t * kTileBlocks + b;
          const bool valid = lbb < nblk && idb >= 0 && idb < p.num_blocks;
          c1[b] = (valid && lbb == nblk - 1) ? -shift : 0;
          c2[b] = valid ? idb * p.num_kv_heads + kvh : oob_bh;
        }
        if (lane == 0) {
          const int ks = g % kKStages, vs = g % kVStages;
          if (g >= kKStages)
            ok = wait_bar(bar(kBarKEmpty0 + ks), ((g / kKStages) - 1) & 1, abort_flag, status);
          if (ok) {
            mbar_expect_tx(bar(kBarKFull0 + ks), LY::kKvBytes);
            for (int pn = 0; pn < kPanels; ++pn)
              for (int b = 0; b < kTileBlocks; ++b)
                tma_load_3d(sK + ks * LY::kKvBytes + pn * LY::kPanelBytes + b * 2048, &tm_k,
                            64 * pn, c1[b], c2[b], bar(kBarKFull0 + ks));
          }
          if (ok && g >= kVStages)
            ok = wait_bar(bar(kBarVEmpty0 + vs), ((g / kVStages) - 1) & 1, abort_flag, status);
          if (ok) {
            mbar_expect_tx(bar(kBarVFull0 + vs), LY::kKvBytes);
            for (int pn = 0; pn < kPanels; ++pn)
              for (int b = 0; b < kTileBlocks; ++b)
                tma_load_3d(sV + vs * LY::kKvBytes + pn * LY::kPanelBytes + b * 2048, &tm_v,
                            64 * pn, c1[b], c2[b], bar(kBarVFull0 + vs));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
  } else if (warp == 1) {
    // =========================== MMA issuer ===========================
    constexpr uint32_t idesc_qk = instr_desc(128, KT, 0, 0);
    constexpr uint32_t idesc_pv = instr_desc(128, D, 0, 1);
    uint32_t g = 0;
    bool ok = true;
    auto issue_pv = [&](uint32_t gt, bool first_of_item) {
      const int vs = gt % kVStages;
      ok = wait_bar(bar(kBarPFull), gt & 1, abort_flag, status) &&
           wait_bar(bar(kBarVFull0 + vs), (gt / kVStages) & 1, abort_flag, status);
      if (!ok) return;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vbase = sV + vs * LY::kKvBytes;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint64_t a = smem_desc(sP + (kk / 4) * LY::kPanelBytes + (kk % 4) * 32, 16, 1024);
          const uint64_t b = smem_desc(vbase + kk * 2048, LY::kPanelBytes, 1024);
          umma_bf16(tmem + kTmemO, a, b, idesc_pv, (first_of_item && kk == 0) ? 0u : 1u);
        }
        umma_commit(bar(kBarVEmpty0 + vs));
        umma_commit(bar(kBarODone));
      }
      __syncwarp();
    };
    for (int k = 0; ok; ++k) {
      const int w = item_index(k);
      if (w >= num_items) break;
      const ItemInfo it = load_item(p, w);
      ok = wait_bar(bar(kBarQFull), k & 1, abort_flag, status);
      const uint32_t g_first = g;
      for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
        const int ks = g % kKStages;
        ok = wait_bar(bar(kBarKFull0 + ks), (g / kKStages) & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kbase = sK + ks * LY::kKvBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * LY::kPanelBytes + (kk % 4) * 32;
            umma_bf16(tmem + kTmemS + (g & 1) * KT, smem_desc(sQ + off, 16, 1024),
                      smem_desc(kbase + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(kBarKEmpty0 + ks));
          umma_commit(bar(kBarSFull0 + (g & 1)));
          if (t == it.ntiles - 1) umma_commit(bar(kBarQEmpty));
        }
        __syncwarp();
        if (t > 0) issue_pv(g - 1, g - 1 == g_first);
      }
      if (ok && it.ntiles > 0) issue_pv(g - 1, g - 1 == g_first);
    }
  } else {
    // =========================== softmax ===========================
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;        // query row of this thread
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    uint32_t g = 0;
    bool ok = true;
    const float sl2 = p.scale_log2;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k);
      if (w >= num_items) break;
      const ItemInfo it = load_item(p, w);
      const int jq = it.qtile * QT + row;
      const bool row_valid = jq < it.ql;
      const int pos = row_valid ? it.L - it.ql + jq : -1;  // last visible key
      const int nblk = (it.L + kBlockSize - 1) / kBlockSize;
      const int shift = nblk * kBlockSize - it.L;
      const int min_pos = it.L - it.ql + it.qtile * QT;    // smallest position in the tile
      float m_run = -INFINITY, l_run = 0.f;
      const uint32_t g_first = g;
      for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
        ok = wait_bar(bar(kBarSFull0 + (g & 1)), (g >> 1) & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[KT];
        {
          const uint32_t ta = tmem + lane_addr + kTmemS + (g & 1) * KT;
          tmem_ld32_at<0>(ta, sr);
          tmem_ld32_at<32>(ta + 32, sr);
          tmem_ld32_at<64>(ta + 64, sr);
          tmem_ld32_at<96>(ta + 96, sr);
        }
        tmem_ld_wait();
        float s[KT];
#pragma unroll
        for (int n = 0; n < KT; ++n) s[n] = __uint_as_float(sr[n]);
        // ---- mask: causal limit, the shifted last block, blocks past the sequence
        const bool need_mask = (t * KT + KT - 1 > min_pos) ||
                               ((t + 1) * kTileBlocks > nblk - 1);
        float mx = -INFINITY;
        if (need_mask) {
#pragma unroll
          for (int n = 0; n < KT; ++n) {
            const int lb = t * kTileBlocks + n / kBlockSize, i = n % kBlockSize;
            const int key = lb * kBlockSize + i - (lb == nblk - 1 ? shift : 0);
            const bool vis = lb < nblk && (lb != nblk - 1 || i >= shift) && key <= pos;
            s[n] = vis ? s[n] * sl2 : -INFINITY;
            mx = fmaxf(mx, s[n]);
          }
        } else {
#pragma unroll
          for (int n = 0; n < KT; ++n) {
            s[n] *= sl2;
            mx = fmaxf(mx, s[n]);
          }
        }
        // ---- running max: moved only when it grows past the threshold
        float alpha = 1.f;
        if (mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx > -INFINITY)) {
          alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - mx);
          m_run = mx;
        }
        const float base_m = (m_run == -INFINITY) ? 0.f : m_run;
        float sum = 0.f;
#pragma unroll
        for (int n = 0; n < KT; ++n) {
          s[n] = ex2(s[n] - base_m);
          sum += s[n];
        }
        l_run = l_run * alpha + sum;
        // ---- P (and O) may be touched once the previous P.V has finished
        if (g > 0) ok = wait_bar(bar(kBarODone), (g - 1) & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < KT / 8; ++c) {  // 16-byte chunks of 8 keys
          const uint32_t w0 = pack_bf16x2(s[8 * c + 0], s[8 * c + 1]);
          const uint32_t w1 = pack_bf16x2(s[8 * c + 2], s[8 * c + 3]);
          const uint32_t w2 = pack_bf16x2(s[8 * c + 4], s[8 * c + 5]);
          const uint32_t w3 = pack_bf16x2(s[8 * c + 6], s[8 * c + 7]);
          const uint32_t addr = sP + (c / 8) * LY::kPanelBytes + row * 128 +
                                (((c % 8) ^ (row % 8)) * 16);
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(w0), "r"(w1),
                       "r"(w2), "r"(w3)
                       : "memory");
        }
        if (g != g_first && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_addr + kTmemO + c * 32, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
              orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st32(tmem + lane_addr + kTmemO + c * 32, orr);
          }
          tmem_st_wait();
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull));
      }
      if (!ok || it.ntiles == 0) continue;
      // ---- epilogue: O / l to global memory
      ok = wait_bar(bar(kBarODone), (g - 1) & 1, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow =
          (__nv_bfloat16*)p.out + ((int64_t)(it.q0 + jq) * p.num_q_heads + it.head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(tmem + lane_addr + kTmemO + c * 32, orr);
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(orr[8 * v + 0]) * inv, __uint_as_float(orr[8 * v + 1]) * inv);
            pk.y = pack_bf16x2(__uint_as_float(orr[8 * v + 2]) * inv, __uint_as_float(orr[8 * v + 3]) * inv);
            pk.z = pack_bf16x2(__uint_as_float(orr[8 * v + 4]) * inv, __uint_as_float(orr[8 * v + 5]) * inv);
            pk.w = pack_bf16x2(__uint_as_float(orr[8 * v + 6]) * inv, __uint_as_float(orr[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + 8 * v) = pk;
          }
        }
      }
    }
  }

  // ---- wind down: every role is done (or gave up); free TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------- work list

// One CTA: list the prefill items of every sequence with q_len * group > 16,
// heaviest (most key tiles) first (a counting sort on the tile count), and
// store the count in ws_items[0].x.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(const AttnParams p, int max_tiles) {
  extern __shared__ int hist[];  // [max_tiles + 1] counters, then running offsets
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i <= max_tiles; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  // pass 1: histogram of items by tile count
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    if (ql * p.group <= kDecodeRows || ql > L) continue;
    const int nq = (ql + QT - 1) / QT;
    for (int i = 0; i < nq; ++i) {
      const int last = L - ql + min((i + 1) * QT, ql) - 1;
      const int nt = min(last / KT + 1, max_tiles);
      atomicAdd(&hist[nt], p.num_q_heads);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive offsets, descending tile count
    int run = 0;
    for (int nt = max_tiles; nt >= 0; --nt) {
      const int c = hist[nt];
      hist[nt] = run;
      run += c;
    }
    p.ws_items[0] = make_int4(min(run, p.max_items), 0, 0, 0);
  }
  __syncthreads();
  // pass 2: scatter
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    if (ql * p.group <= kDecodeRows || ql > L) continue;
    const int nq = (ql + QT - 1) / QT;
    for (int i = nq - 1; i >= 0; --i) {
      const int last = L - ql + min((i + 1) * QT, ql) - 1;
      const int nt = min(last / KT + 1, max_tiles);
      const int at = atomicAdd(&hist[nt], p.num_q_heads);
      for (int h = 0; h < p.num_q_heads; ++h)
        if (at + h < p.max_items) p.ws_items[1 + at + h] = make_int4(s, i, h, nt);
    }
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
  }
  return fn;
}

// 3-D bf16 tensor map (dim0 innermost) with a (64, box1, box2) box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {64, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!n[dev]) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
  return n[dev] > 0 ? n[dev] : 148;
}

template <int D>
cudaError_t launch_d(const AttnParams& p, int max_query_len, int num_items, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, p.q, D, p.num_q_heads, p.num_tokens, (uint64_t)D * 2,
                (uint64_t)p.num_q_heads * D * 2, 1, QT) ||
      !make_map(&tk, p.k_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1) ||
      !make_map(&tv, p.v_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1))
    return cudaErrorInvalidValue;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  // work list on the device
  {
    const int tiles = (p.max_blocks_per_seq * kBlockSize + KT - 1) / KT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = (tiles + 1) * sizeof(int);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cfg.dynamicSmemBytes > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(prefill_plan_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)cfg.dynamicSmemBytes);
      if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_plan_kernel, p, tiles);
    if (e != cudaSuccess) return e;
  }
  const int upper = num_items >= 0 ? num_items
                                   : (int)min((long)p.max_items,
                                              (long)p.num_seqs * ((max_query_len + QT - 1) / QT) *
                                                  p.num_q_heads);
  const int grid = max(1, min(sm_count(), upper));
  auto kernel = prefill_tcgen05_kernel<D>;
  const int smem = PrefillLayout<D>::total;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p, tq, tk, tv);
}

}  // namespace

cudaError_t launch_prefill_tcgen05(const AttnParams& p, int head_dim, int max_query_len,
                                   int num_items, cudaStream_t stream) {
  cudaError_t e = head_dim == 64 ? launch_d<64>(p, max_query_len, num_items, stream)
                                 : launch_d<128>(p, max_query_len, num_items, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pa
