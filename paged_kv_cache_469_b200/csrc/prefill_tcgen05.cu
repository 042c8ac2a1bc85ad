// prefill_tcgen05.cu -- tensor-core paged attention for prefill chunks.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説": section "エンジンの中核" -- a
// prefill runs the whole prompt and is compute-bound; section "高度な機能群"
// -- a chunked prefill attends to the context already cached before the chunk
// as well as to itself; section "PagedAttentionの仕組み" -- keys are read
// through the sequence's block table and a causal, position-based mask keeps
// each query on its own sequence's earlier tokens.
//
// Work item = (sequence, 128-query tile, two q-heads of one kv-head), or two
// consecutive 128-query tiles of one q-head when the group size is odd: two
// 128-row halves that read the same keys.  A persistent CTA (one per SM)
// walks its items, heaviest first; per item it streams the sequence's keys in
// 128-key tiles:
//
//   warp 8      TMA: the two Q tiles once per item, then every K tile -- eight
//               16-token cache blocks, one 16 x 64 box per block and 64-wide
//               slice of D, 128-byte swizzled, straight from the pool through
//               the block table; one lane issues each box
//   warp 10     TMA: every V tile, the same way
//   warp 9      MMA issuer (one thread): S_h = Q_h K^T into TMEM (tcgen05.mma,
//               M=128, N=128, K=16 steps, both operands in shared memory), and
//               O_h += P_h V with P_h read from TMEM
//   warps 0..3, 4..7  softmax of half 0 / half 1, one query row per thread:
//               S from TMEM (tcgen05.ld), causal mask, online softmax in fp32
//               (exp2; the running max moves only when it grows by more than
//               2^8, so O is rarely rescaled), P as bf16 written back over S
//               in TMEM (tcgen05.st); at the end of the item O / l to global
//               memory
//
// The MMA warp issues P.V of tile g-1 before Q K^T of tile g for each half, so
// the tensor pipe works on one half while the softmax of the other runs.  The
// last, partly filled cache block of a sequence is loaded at a negative row
// offset so that its unwritten slots arrive as TMA zero fill (never
// uninitialised cache memory); blocks past the sequence, or block ids outside
// the pool, are loaded from beyond the tensor's extent (zeros).
//
// Every mbarrier wait is bounded by a time limit; a wait that runs out sets a
// status bit in the workspace and the CTA winds down instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "pa_fastmath.cuh"
#include "pa_internal.cuh"
#include "pa_tma.cuh"
#include "pa_wait.cuh"

namespace pa {
namespace {

constexpr int QT = kPrefillQTile;               // 128 query rows per Q tile
constexpr int KT = kPrefillKvTile;              // 128 keys per K/V tile
constexpr int kTileBlocks = KT / kBlockSize;    // 8 cache blocks per tile
// K / V tile stages: a K tile is needed one MMA round after V's (P.V of a
// tile follows its Q K^T), so K benefits first from a deeper ring
#ifndef PA_PREFILL_K_STAGES
#define PA_PREFILL_K_STAGES 2
#endif
constexpr int kKStages = PA_PREFILL_K_STAGES, kVStages = 2;
constexpr int kThreads = 384;                   // 12 warps = 3 warpgroups
// warpgroup 0 (warps 0..3): softmax of half 0; warpgroup 1 (4..7): softmax of
// half 1 (a warp reads the TMEM lanes 32 * (warp % 4) ..); warpgroup 2: warp
// 8 TMA for Q and K, warp 9 MMA issuer, warp 10 TMA for V, warp 11 idle.
constexpr int kWarpK = 8, kWarpMma = 9, kWarpV = 10;
// Registers: launched at 168 each (384 x 168 = 64512); warpgroup 2 then gives
// back down to 88 and the softmax warpgroups take up to 208:
// 2 x 128 x 208 + 128 x 88 = 64512.
constexpr int kRegsLaunch = 168, kRegsSoftmax = 208, kRegsOther = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
// TMEM columns: O of half h at 128 h; S of half h at 256 + 128 h, its P (bf16,
// two per column) written over the first 64 columns of S once S is read
constexpr uint32_t kTmemO = 0, kTmemS = 256;
constexpr float kRescaleThreshold = 8.0f;       // log2 units: move the max only past 2^8
// independent max chains over a row of scores (a power of two, at most 32)
#ifndef PA_PREFILL_MAX_CHAINS
#define PA_PREFILL_MAX_CHAINS 8
#endif
constexpr int kMaxChains = PA_PREFILL_MAX_CHAINS;
static_assert((kMaxChains & (kMaxChains - 1)) == 0 && kMaxChains <= 32, "max chains");

template <int D>
struct PrefillLayout {
  static constexpr int kPanels = D / 64;            // 64-wide slices of D
  static constexpr int kQPanelBytes = QT * 128;     // 128 rows x 128 bytes
  static constexpr int kKvPanelBytes = KT * 128;    // 128 rows x 128 bytes
  static constexpr int kQBytes = kPanels * kQPanelBytes;   // one Q tile
  static constexpr int kKvBytes = kPanels * kKvPanelBytes; // one K or V tile
  static constexpr int q_off = 0;                   // two Q tiles (the two halves)
  static constexpr int k_off = q_off + 2 * kQBytes;
  static constexpr int v_off = k_off + kKStages * kKvBytes;
  static constexpr int bar_off = v_off + kVStages * kKvBytes;
  static constexpr int used = bar_off + 256;
  // D = 64 would fit two CTAs per SM, whose TMEM allocations would then queue
  // behind each other: ask for enough shared memory to keep one CTA per SM.
  static constexpr int total = (used < 120 * 1024 ? 120 * 1024 : used) + 1024;
  static_assert(total <= 227 * 1024, "shared memory of one CTA");
};

// mbarrier indices
enum : int {
  kBarQFull = 0, kBarQEmpty,
  kBarKFull = 2,                      // + stage
  kBarKEmpty = kBarKFull + kKStages,  // + stage
  kBarVFull = kBarKEmpty + kKStages,  // + stage
  kBarVEmpty = kBarVFull + kVStages,  // + stage
  kBarSFull = kBarVEmpty + kVStages,  // + half
  kBarPFull = kBarSFull + 2,          // + half
  kBarODone = kBarPFull + 2,          // + half
  kNumBars = kBarODone + 2
};
static_assert(kNumBars * 8 <= 256, "barriers must fit their 256-byte area");

// ------------------------------------------------------------------ PTX wrappers

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
// the same, with A (M x 16, bf16 packed two per 32-bit column) read from TMEM
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

// A work item is two 128-row Q tiles that read the same keys: two q-heads of
// one kv-head (pair_heads), or two consecutive query tiles of one q-head.
struct ItemInfo {
  int seq, qt0, head0, ntiles;
  int q0, ql, L;
};

// A work list the host built from its copies of the step's lengths, passed as
// a kernel parameter (count 0: the list is in the workspace, built by
// prefill_plan_kernel).
constexpr int kParamItems = 1024;
struct PrefillWork {
  int count;
  int pad[3];
  int4 items[kParamItems];
};

__device__ __forceinline__ ItemInfo load_item(const AttnParams& p, const PrefillWork& work,
                                              int w) {
  const int4 it = work.count > 0 ? work.items[w] : p.ws_items[1 + w];
  ItemInfo r;
  r.seq = it.x; r.qt0 = it.y; r.head0 = it.z; r.ntiles = it.w;
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
                       const __grid_constant__ CUtensorMap tm_v, int pair_heads,
                       const __grid_constant__ PrefillWork work) {
  using LY = PrefillLayout<D>;
  constexpr int kPanels = LY::kPanels;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t sh_tmem_base;
  __shared__ int sh_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = ((uint32_t)__cvta_generic_to_shared(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + LY::q_off, sK = base + LY::k_off, sV = base + LY::v_off,
                 sBar = base + LY::bar_off;
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = &sh_abort;

  if (threadIdx.x == 0) {
    sh_abort = 0;
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(bar(kBarKFull + i), 1);
      mbar_init(bar(kBarKEmpty + i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(bar(kBarVFull + i), 1);
      mbar_init(bar(kBarVEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarPFull + i), 4);  // one arrival per softmax warp of the half
      mbar_init(bar(kBarODone + i), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == kWarpMma) {
    tmem_alloc((uint32_t)__cvta_generic_to_shared(&sh_tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh_tmem_base;

  // the work list and the cache must be complete before anything reads them;
  // the next kernel on the stream may be launched from then on (it waits for
  // this grid before it reads anything)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int num_items = work.count > 0 ? work.count : p.ws_items[0].x;
  int* status = p.ws_status;

  if (warp >= 8) {
    // warpgroup 2 gives registers back before taking its role
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    if (warp == kWarpK || warp == kWarpV) {
      // ============ TMA producers: one warp loads the Q tiles and K, one loads V ============
      // (separate warps, so that a K tile never waits behind a V slot)
      const bool is_v = (warp == kWarpV);
      const int oob_bh = p.num_blocks * p.num_kv_heads;  // first block-head row past the pool
      uint32_t g = 0;                                     // global tile counter
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int w = item_index(k);
        if (w >= num_items) break;
        const ItemInfo it = load_item(p, work, w);
        const int kvh = it.head0 / p.group;
        const int nblk = (it.L + kBlockSize - 1) / kBlockSize;
        const int shift = nblk * kBlockSize - it.L;  // unwritten slots of the last block
        const int32_t* table = p.block_tables + (int64_t)it.seq * p.max_blocks_per_seq;
        // ---- the two Q tiles
        if (!is_v && lane == 0) {
          if (k > 0) ok = wait_bar(bar(kBarQEmpty), (k - 1) & 1, abort_flag, status);
          if (ok) {
            mbar_expect_tx(bar(kBarQFull), 2 * LY::kQBytes);
            for (int h = 0; h < 2; ++h) {
              const int head = pair_heads ? it.head0 + h : it.head0;
              const int qt = pair_heads ? it.qt0 : it.qt0 + h;
              for (int pn = 0; pn < kPanels; ++pn)
                tma_load_3d(sQ + h * LY::kQBytes + pn * LY::kQPanelBytes, &tm_q, 64 * pn, head,
                            it.q0 + qt * QT, bar(kBarQFull));
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        // ---- K or V tiles
        for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
          // lane b < kTileBlocks reads the id of the tile's block b; lane
          // pn * kTileBlocks + b then issues the box of block b, D-slice pn
          int id = -1;
          const int lb = t * kTileBlocks + lane;
          if (lane < kTileBlocks && lb < nblk && lb < p.max_blocks_per_seq) id = table[lb];
          const int b = lane % kTileBlocks, pn = lane / kTileBlocks;
          const int idb = __shfl_sync(0xffffffffu, id, b);
          const int lbb = t * kTileBlocks + b;
          const bool valid = lbb < nblk && idb >= 0 && idb < p.num_blocks;
          const int c1 = (valid && lbb == nblk - 1) ? -shift : 0;
          const int c2 = valid ? idb * p.num_kv_heads + kvh : oob_bh;
          const uint32_t nst = is_v ? kVStages : kKStages;
          const int st = g % nst;
          const int full = (is_v ? kBarVFull : kBarKFull) + st;
          const int empty = (is_v ? kBarVEmpty : kBarKEmpty) + st;
          if (lane == 0) {
            if (g >= nst) ok = wait_bar(bar(empty), ((g / nst) - 1) & 1, abort_flag, status);
            if (ok) mbar_expect_tx(bar(full), LY::kKvBytes);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);  // (also orders the expect_tx first)
          if (ok && lane < kPanels * kTileBlocks) {
            const uint32_t dst = (is_v ? sV : sK) + st * LY::kKvBytes;
            tma_load_3d(dst + pn * LY::kKvPanelBytes + b * 2048, is_v ? &tm_v : &tm_k, 64 * pn,
                        c1, c2, bar(full));
          }
          __syncwarp();
        }
      }
    } else if (warp == kWarpMma) {
      // =========================== MMA issuer ===========================
      // Per half h: S_h = Q_h K^T (both operands in shared memory), then, once
      // the softmax has written P_h over S_h in TMEM, O_h += P_h V (P from TMEM).
      // The tensor pipe runs a thread's MMAs in order, so P.V of tile g-1 has
      // finished with P_h before Q K^T of tile g overwrites S_h.
      // Descriptors are built once; a k-step, panel or stage moves the start
      // address, i.e. adds (byte offset >> 4) to the descriptor.
      constexpr uint32_t idesc_qk = instr_desc(128, KT, 0, 0);
      constexpr uint32_t idesc_pv = instr_desc(128, D, 0, 1);
      const uint64_t dq0 = smem_desc(sQ, 16, 1024);
      const uint64_t dk0 = smem_desc(sK, 16, 1024);
      const uint64_t dv0 = smem_desc(sV, LY::kKvPanelBytes, 1024);
      uint32_t g = 0;
      bool ok = true;
      auto issue_pv = [&](int h, uint32_t gt, bool first_of_item) {  // O_h += P_h V (tile gt)
        ok = wait_bar(bar(kBarPFull + h), gt & 1, abort_flag, status);
        if (!ok) return;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t dv = dv0 + (uint64_t)(((gt % kVStages) * LY::kKvBytes) >> 4);
          const uint32_t dst = tmem + kTmemO + 128 * h;
          const uint32_t pa = tmem + kTmemS + 128 * h;
  #pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk)
            umma_bf16_ts(dst, pa + 8 * kk, dv + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                         (first_of_item && kk == 0) ? 0u : 1u);
          umma_commit(bar(kBarODone + h));
        }
        __syncwarp();
      };
      auto issue_qk = [&](int h, uint32_t gt) {  // S_h = Q_h K^T (tile gt)
        if (lane == 0) {
          const uint64_t dk = dk0 + (uint64_t)(((gt % kKStages) * LY::kKvBytes) >> 4);
          const uint64_t dq = dq0 + (uint64_t)((h * LY::kQBytes) >> 4);
          const uint32_t dst = tmem + kTmemS + 128 * h;
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qo = ((kk / 4) * LY::kQPanelBytes + (kk % 4) * 32) >> 4;
            const uint32_t ko = ((kk / 4) * LY::kKvPanelBytes + (kk % 4) * 32) >> 4;
            umma_bf16(dst, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(kBarSFull + h));
        }
        __syncwarp();
      };
      for (int k = 0; ok; ++k) {
        const int w = item_index(k);
        if (w >= num_items) break;
        const ItemInfo it = load_item(p, work, w);
        ok = wait_bar(bar(kBarQFull), k & 1, abort_flag, status);
        const uint32_t g_first = g;
        for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
          ok = wait_bar(bar(kBarKFull + g % kKStages), (g / kKStages) & 1, abort_flag, status);
          if (ok && t > 0)
            ok = wait_bar(bar(kBarVFull + (g - 1) % kVStages), ((g - 1) / kVStages) & 1, abort_flag,
                          status);
          if (!ok) break;
          tc_fence_after();
          for (int h = 0; h < 2 && ok; ++h) {
            if (t > 0) issue_pv(h, g - 1, g - 1 == g_first);  // P_h of the previous tile
            if (ok) issue_qk(h, g);
          }
          if (ok && lane == 0) {
            umma_commit(bar(kBarKEmpty + g % kKStages));
            if (t > 0) umma_commit(bar(kBarVEmpty + (g - 1) % kVStages));
            if (t == it.ntiles - 1) umma_commit(bar(kBarQEmpty));
          }
          __syncwarp();
        }
        if (ok && it.ntiles > 0) {  // P.V of the item's last tile
          const uint32_t gl = g - 1;
          ok = wait_bar(bar(kBarVFull + gl % kVStages), (gl / kVStages) & 1, abort_flag, status);
          if (ok) tc_fence_after();
          for (int h = 0; h < 2 && ok; ++h) issue_pv(h, gl, gl == g_first);
          if (ok && lane == 0) umma_commit(bar(kBarVEmpty + gl % kVStages));
          __syncwarp();
        }
      }
    }
  } else {
    // =========================== softmax (two halves) ===========================
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int h = warp >> 2;                   // which Q tile
    const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;       // query row of this thread in its tile
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kTmemS + 128 * h;
    const uint32_t tO = tmem + lane_addr + kTmemO + 128 * h;
    uint32_t g = 0;
    bool ok = true;
    const float sl2 = p.scale_log2;
    for (int k = 0; ok; ++k) {
      const int w = item_index(k);
      if (w >= num_items) break;
      const ItemInfo it = load_item(p, work, w);
      const int head = pair_heads ? it.head0 + h : it.head0;
      const int qt = pair_heads ? it.qt0 : it.qt0 + h;
      const int jq = qt * QT + row;
      const bool row_valid = jq < it.ql;
      const int pos = row_valid ? it.L - it.ql + jq : -1;  // last visible key
      const int nblk = (it.L + kBlockSize - 1) / kBlockSize;
      const int shift = nblk * kBlockSize - it.L;
      const int min_pos = it.L - it.ql + qt * QT;          // smallest position in the tile
      float m_run = -INFINITY, l_run = 0.f;
      const uint32_t g_first = g;
      for (int t = 0; t < it.ntiles && ok; ++t, ++g) {
        // S_h of tile g is complete; so is P.V of tile g-1 (issued before it)
        ok = wait_bar(bar(kBarSFull + h), g & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[KT];
        tmem_ld32_at<0>(tS, sr);
        tmem_ld32_at<32>(tS + 32, sr);
        tmem_ld32_at<64>(tS + 64, sr);
        tmem_ld32_at<96>(tS + 96, sr);
        tmem_ld_wait();
        float s[KT];
#pragma unroll
        for (int n = 0; n < KT; ++n) s[n] = __uint_as_float(sr[n]);
        // ---- mask: column 16 b + i holds key t*KT + 16 b + i for blocks before
        // the sequence's last block; the last block was loaded shifted down by
        // `shift` rows, so its column 16 b + i holds key t*KT + 16 b + i - shift
        // and its first `shift` columns are empty; columns past it are empty.
        // Per block, slots lo .. hi are visible to this row.
        if (t * KT + KT - 1 > min_pos || (t + 1) * kTileBlocks > nblk - 1) {
          const int lim = pos - t * KT;  // last visible key, tile-relative
          const int lastb = nblk - 1 - t * kTileBlocks;
#pragma unroll
          for (int b = 0; b < kTileBlocks; ++b) {
            const int lo = b < lastb ? 0 : (b == lastb ? shift : 16);
            const int hi = lim - 16 * b + (b == lastb ? shift : 0);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              s[16 * b + i] = (i >= lo && i <= hi) ? s[16 * b + i] : -INFINITY;
          }
        }
        // ---- row max of the raw scores: kMaxChains independent chains of
        // three-input maxima, then a tree
        float mc[kMaxChains];
#pragma unroll
        for (int q = 0; q < kMaxChains; ++q) mc[q] = fmaxf(s[2 * q], s[2 * q + 1]);
#pragma unroll
        for (int n = 2 * kMaxChains; n < KT; n += 2 * kMaxChains) {
#pragma unroll
          for (int q = 0; q < kMaxChains; ++q) mc[q] = max3(mc[q], s[n + 2 * q], s[n + 2 * q + 1]);
        }
#pragma unroll
        for (int w = kMaxChains; w > 1; w /= 2) {
#pragma unroll
          for (int q = 0; q < w / 2; ++q) mc[q] = fmaxf(mc[q], mc[q + w / 2]);
        }
        const float mx = sl2 * mc[0];
        // ---- running max (log2 units): moved only when it grows past the threshold
        float alpha = 1.f;
        if (mx > m_run + kRescaleThreshold || (m_run == -INFINITY && mx > -INFINITY)) {
          alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - mx);
          m_run = mx;
        }
        const float neg_base = (m_run == -INFINITY) ? 0.f : -m_run;
        // ---- P = exp2(S * scale * log2(e) - max) on pairs of columns (the
        // scaling on the packed-pair FMA, the exponentials on the exponential
        // unit); two bf16 per word, written over the first half of S in
        // 32-word chunks (this thread has read all of S already)
        const uint64_t scale2 = f2(sl2, sl2), base2 = f2(neg_base, neg_base);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pw[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = 64 * c + 2 * j;
            const uint64_t x = fma2(f2(s[n], s[n + 1]), scale2, base2);
            float x0, x1;
            f2_split(x, x0, x1);
            const uint64_t e = f2(ex2(x0), ex2(x1));  // masked: ex2(-inf) = 0
            acc[j & 3] = add2(acc[j & 3], e);
            float e0, e1;
            f2_split(e, e0, e1);
            pw[j] = pack_bf16x2(e0, e1);
          }
          tmem_st32(tS + 32 * c, pw);
        }
        float sum;
        {
          float a0, a1;
          f2_split(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), a0, a1);
          sum = a0 + a1;
        }
        l_run = l_run * alpha + sum;
        // ---- O carries the old max: rescale it (P.V of tile g-1 is complete)
        if (g != g_first && __any_sync(0xffffffffu, alpha != 1.f)) {
          const uint64_t alpha2 = f2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tO + c * 32, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              uint32_t lo, hi;
              u2_split(mul2(u2(orr[2 * e], orr[2 * e + 1]), alpha2), lo, hi);
              orr[2 * e] = lo;
              orr[2 * e + 1] = hi;
            }
            tmem_st32(tO + c * 32, orr);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull + h));
      }
      if (!ok || it.ntiles == 0) continue;
      // ---- epilogue: O / l to global memory
      ok = wait_bar(bar(kBarODone + h), (g - 1) & 1, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow =
          (__nv_bfloat16*)p.out + ((int64_t)(it.q0 + jq) * p.num_q_heads + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(tO + c * 32, orr);
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
      // the next item's first P.V overwrites O: every lane has read it
      tc_fence_before();
    }
  }

  // ---- wind down: every role is done (or gave up); free TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------- work list

// One CTA: list the prefill items of every sequence with q_len * group > 64,
// heaviest (most key tiles) first (a counting sort on the tile count), and
// store the count in ws_items[0].x.  An item pairs two q-heads of one kv-head
// (pair_heads: the group is even) or two consecutive query tiles of one
// q-head; its tile count covers the later of its two query tiles.
__host__ __device__ __forceinline__ void prefill_item_range(int L, int ql, int pair_heads,
                                                            int i, int* last_row_pos) {
  const int hi_tile = pair_heads ? i : 2 * i + 1;
  const int last_row = min((hi_tile + 1) * QT, ql) - 1;
  *last_row_pos = L - ql + last_row;
}

__global__ void __launch_bounds__(1024)
prefill_plan_kernel(const AttnParams p, int max_tiles, int pair_heads) {
  extern __shared__ int hist[];  // [max_tiles + 1] counters, then running offsets
  // the prefill kernel may be launched at once: it waits for this grid before
  // it reads the work list
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i <= max_tiles; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int per_tile = pair_heads ? p.num_q_heads / 2 : p.num_q_heads;  // items per (seq, tile)
  // pass 1: histogram of items by tile count
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    if (ql * p.group <= kDecodeMaxRows || ql > L) continue;
    const int nq = (ql + QT - 1) / QT;
    const int ni = pair_heads ? nq : (nq + 1) / 2;
    for (int i = 0; i < ni; ++i) {
      int last;
      prefill_item_range(L, ql, pair_heads, i, &last);
      const int nt = min(last / KT + 1, max_tiles);
      atomicAdd(&hist[nt], per_tile);
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
    if (ql * p.group <= kDecodeMaxRows || ql > L) continue;
    const int nq = (ql + QT - 1) / QT;
    const int ni = pair_heads ? nq : (nq + 1) / 2;
    for (int i = ni - 1; i >= 0; --i) {
      int last;
      prefill_item_range(L, ql, pair_heads, i, &last);
      const int nt = min(last / KT + 1, max_tiles);
      const int at = atomicAdd(&hist[nt], per_tile);
      for (int h = 0; h < per_tile; ++h) {
        if (at + h >= p.max_items) break;
        p.ws_items[1 + at + h] = pair_heads ? make_int4(s, i, 2 * h, nt)
                                            : make_int4(s, 2 * i, h, nt);
      }
    }
  }
}

// ------------------------------------------------------------------ host side

// The work list of prefill_plan_kernel, built on the host from its copies of
// the step's lengths: the same items, heaviest first.  False when there are
// more items than a kernel parameter holds.
bool host_work_list(PrefillWork* work, const AttnParams& p, const int32_t* seq_lens_host,
                    const int32_t* query_start_loc_host, int max_tiles, int pair_heads) {
  const int per_tile = pair_heads ? p.num_q_heads / 2 : p.num_q_heads;
  static thread_local int hist[1 << 16];
  if (max_tiles + 1 > (1 << 16)) return false;
  for (int i = 0; i <= max_tiles; ++i) hist[i] = 0;
  long total = 0;
  auto for_each_item = [&](auto fn) {
    for (int s = 0; s < p.num_seqs; ++s) {
      const int ql = query_start_loc_host[s + 1] - query_start_loc_host[s];
      const int L = seq_lens_host[s];
      if (ql * p.group <= kDecodeMaxRows || ql > L) continue;
      const int nq = (ql + QT - 1) / QT;
      const int ni = pair_heads ? nq : (nq + 1) / 2;
      for (int i = 0; i < ni; ++i) {
        int last;
        prefill_item_range(L, ql, pair_heads, i, &last);
        fn(s, i, min(last / KT + 1, max_tiles));
      }
    }
  };
  for_each_item([&](int, int, int nt) { hist[nt] += per_tile; total += per_tile; });
  if (total > kParamItems || total > p.max_items) return false;
  int run = 0;
  for (int nt = max_tiles; nt >= 0; --nt) {
    const int c = hist[nt];
    hist[nt] = run;
    run += c;
  }
  for_each_item([&](int s, int i, int nt) {
    int at = hist[nt];
    hist[nt] += per_tile;
    for (int h = 0; h < per_tile; ++h, ++at)
      work->items[at] = pair_heads ? make_int4(s, i, 2 * h, nt) : make_int4(s, 2 * i, h, nt);
  });
  work->count = (int)total;
  return total > 0;
}

template <int D>
cudaError_t launch_d(const AttnParams& p, int max_query_len, int num_items,
                     const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                     cudaStream_t stream, int max_ctas) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, p.q, D, p.num_q_heads, p.num_tokens, (uint64_t)D * 2,
                (uint64_t)p.num_q_heads * D * 2, 1, QT) ||
      !make_map(&tk, p.k_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1) ||
      !make_map(&tv, p.v_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1))
    return cudaErrorInvalidValue;

  // two q-heads of one kv-head share every K/V tile when the group is even
  const int pair_heads = (p.group % 2 == 0) ? 1 : 0;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  // the work list: from the host copies when given and small enough, else
  // built on the device
  static thread_local PrefillWork work;  // 16 KB: kept off the stack
  const int tiles = (p.max_blocks_per_seq * kBlockSize + KT - 1) / KT;
  work.count = 0;
  if (!(seq_lens_host && query_start_loc_host &&
        host_work_list(&work, p, seq_lens_host, query_start_loc_host, tiles, pair_heads))) {
    work.count = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = (tiles + 1) * sizeof(int);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cfg.dynamicSmemBytes > 48 * 1024) {
      static std::atomic<int> plan_smem_done[64];
      cudaError_t e = raise_smem_limit(prefill_plan_kernel, (int)cfg.dynamicSmemBytes,
                                       plan_smem_done);
      if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_plan_kernel, p, tiles, pair_heads);
    if (e != cudaSuccess) return e;
  }
  const int upper = work.count > 0 ? work.count
                  : num_items >= 0 ? num_items
                                   : (int)min((long)p.max_items,
                                              (long)p.num_seqs * ((max_query_len + QT - 1) / QT) *
                                                  p.num_q_heads);
  const int grid = max(1, min(min(device_sm_count(), max_ctas), upper));
  auto kernel = prefill_tcgen05_kernel<D>;
  const int smem = PrefillLayout<D>::total;
  static std::atomic<int> smem_done[64];
  cudaError_t e = raise_smem_limit(kernel, smem, smem_done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p, tq, tk, tv, pair_heads, work);
}

}  // namespace

namespace {
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

}  // namespace

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


cudaError_t launch_prefill_tcgen05(const AttnParams& p, int head_dim, int max_query_len,
                                   int num_items, const int32_t* seq_lens_host,
                                   const int32_t* query_start_loc_host, cudaStream_t stream,
                                   int max_ctas) {
  cudaError_t e =
      head_dim == 64
          ? launch_d<64>(p, max_query_len, num_items, seq_lens_host, query_start_loc_host, stream,
                         max_ctas)
          : launch_d<128>(p, max_query_len, num_items, seq_lens_host, query_start_loc_host,
                          stream, max_ctas);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pa
