// decode_persistent.cu -- bandwidth-bound paged attention for decode-class
// sequences, as one persistent grid.
//
// Page "LLM推論エンジンvLLMの内部構造を徹底解説", section "エンジンの中核": a decode
// step runs the newest token against the KV cache and is bound by memory
// bandwidth; section "PagedAttentionの仕組み": the keys are read block by
// block through the sequence's block table.
//
// Work.  A unit is one (sequence, kv-head, 16-row group of query rows): all
// q-heads of the kv-head times the sequence's query tokens, up to 64 rows, cut
// into 16-row groups (a single-token decode with up to 16 q-heads per kv-head
// is one group, so every K/V byte is read from HBM once per kv-head).  A unit's
// nblk cache blocks are cut into pieces of P blocks (the last one shorter).
// The pieces of a launch form one list, largest first (every full piece, then
// the shorter last pieces by falling size), so that the work still left at the
// end of the launch is the finest.  P is chosen per launch: when no unit is
// much longer than a CTA's share of the step's blocks, every unit is one piece
// (the largest-first claims balance the SMs and nothing needs merging across
// CTAs); otherwise the long units are cut so that every CTA gets a few pieces.
//
// Grid.  One CTA per SM (its shared memory holds the streaming rings), each
// running until its work is done.  Pieces reach the CTAs in one of two ways:
//   claims  CTA b starts with piece b and claims the next piece from a global
//       counter once every compute warp with blocks in its current piece has
//       issued them all (their copies are still in flight while the claim
//       and the piece's staging complete), so the SMs that get through their
//       work first take the next pieces;
//   dealt   when every SM has a CTA and the list holds at least a few pieces
//       per CTA, the host deals the pieces to the CTAs beforehand (longest
//       first, each to the CTA with the least work so far, a piece counting
//       its blocks plus a fixed cost) and CTA b runs its own run of the list
//       in order.
// Inside a CTA:
//
//   scheduler warp (the last warp)  takes a piece, copies its block ids and
//       its query rows into a shared-memory piece slot (two slots: piece p
//       lives in slot p % 2) and publishes the slot.  When the call also
//       writes the step's new K/V rows, the scheduler stores the rows of a
//       claimed piece after publishing it and then raises a second flag of
//       the slot; a compute warp waits for that flag only before loading a
//       block that receives new rows.  (For dealt pieces the rows are
//       written before the slot is published.)
//   compute warps 0 .. kWarps-1     block subset c of a piece (its blocks c,
//       c + kWarps, ...) goes to warp (c + rot) % kWarps, where rot carries
//       on from the previous piece so that no warp gets every piece's ragged
//       remainder.  For the CTA's first piece the warps read their block ids
//       from the block table themselves and issue their first loads (blocks
//       receiving new rows excepted) before the slot is published.  Each warp streams its blocks through a
//       private ring of kStages shared-memory stages (K tile + V tile of one
//       (block, kv-head)) filled by TMA (16 x 64 boxes, one mbarrier per
//       stage), up to kStages blocks in flight, and the ring runs on from one
//       piece into the next without draining.  Per 16-token block, with the
//       keys on the MMA's M side and the (at most 8 per n-tile) query rows on
//       its N side, so that no MMA row is padding:
//         S^T[16 keys x 8 rows]  = K . Q^T   mma.m16n8k16 per 16 dims of D
//                                            (K by ldmatrix from the ring)
//         online softmax down the columns of S^T (fp32 running max and sum,
//         exp2 with log2(e) folded into the scale), the max moved lazily
//         P^T: the bf16 S^T fragment transposed in registers (movmatrix)
//         O^T[D x 8 rows]       += V^T . P^T  mma.m16n8k16 per 16 dims of D
//                                            (V^T by ldmatrix.trans)
//   piece merge  when a warp has computed its last block of a piece it puts
//       its (max, sum, O) in a shared merge slot, at the place of its block
//       subset; the warp whose blocks complete the piece's count merges the
//       parts in subset order (so the result does not depend on timing) and
//       stores the piece's result: the output rows when the
//       piece is the whole unit, else an fp32 partial in the workspace.  No
//       CTA ever waits for another, and no merge waits for global memory.
//   combine kernel  (launched right after, as a programmatic dependent) one
//       warp per unit cut into several pieces merges the unit's partials
//       into its output rows.
//
// The 16-byte chunks of every tile row are XOR-swizzled on their way into
// shared memory (the TMA 128-byte swizzle) so that every 8 x 8 matrix that
// ldmatrix reads hits eight distinct bank groups.
//
// Every wait on another warp of the CTA (a piece slot not yet published, a
// block's new rows not yet written, the merge slot still in use, the warps
// not yet past the current piece) is bounded by a time limit; one that runs out sets
// the workspace status bit and the CTA winds down instead of hanging.  The
// kernel is launched as a programmatic dependent of whatever precedes it on
// the stream; before griddepcontrol.wait it reads only its own parameters.
#include <math.h>

#include <algorithm>
#include <cstring>
#include <functional>
#include <queue>
#include <type_traits>
#include <utility>
#include <vector>

#include "pa_fastmath.cuh"
#include "pa_internal.cuh"
#include "pa_tma.cuh"
#include "pa_wait.cuh"

namespace pa {
namespace {

// compute warps and ring stages per CTA, by head_dim and most query rows per
// unit (shared memory: ring + merge slot + two piece slots, at most 227 KB).
// The copies a CTA keeps in flight (warps x stages x one block's K and V)
// must cover its share of HBM bandwidth times the load latency, about 64 KB
// to 96 KB; a warp's own loop over its blocks is bound by the latency of its
// dependent chain (shared-memory loads, MMAs, exponentials), a few hundred
// cycles per block.
template <int D, int kMaxRows>
struct DecodeCfg {
  static constexpr int kWarps = D == 64 ? 12 : (kMaxRows <= 4 ? 11 : kMaxRows <= 8 ? 10 : 8);
  static constexpr int kStages = D == 64 ? 3 : 2;
};

// What the scheduler publishes about one piece.
struct PieceInfo {
  int tag;  // CTA-local sequence number of the piece in this slot (-1: none yet)
  int end;  // 1: the list is exhausted, no piece in this slot
  int s, kvh, rg, j, nparts;
  int blk_begin, nb;  // the piece's blocks: blk_begin .. blk_begin + nb - 1 of the sequence
  int L, ql, q0;
  int rows, row0;  // this unit's query rows: global rows row0 .. row0 + rows - 1
  int rot;         // block subset c of the piece (blocks c, c + kWarps, ...) goes to warp (c + rot) % kWarps
  int cw_tag;      // = tag once the step's new K/V rows of the piece are in the cache (write path)
  int cw_first;    // the piece's first block receiving new rows (nb: none)
};

template <int D, int kMaxRows>
struct DecodeLayout {
  static constexpr int kWarps = DecodeCfg<D, kMaxRows>::kWarps;
  static constexpr int kStages = DecodeCfg<D, kMaxRows>::kStages;
  static constexpr int kTileBytes = kBlockSize * D * 2;  // one (block, kv-head) tile
  static constexpr int kStageBytes = 2 * kTileBytes;     // K tile + V tile
  static constexpr int ring_off = 0;  // 1024-byte aligned (128-byte swizzle atoms)
  static constexpr int ring_bytes = kWarps * kStages * kStageBytes;
  // merge slot: per compute warp its rows' max, sum and unnormalised O (rows
  // of D + 4 floats: the fragment stores of four rows hit distinct banks)
  static constexpr int kOStride = D + 4;
  static constexpr int mm_off = ring_off + ring_bytes;                // [kWarps][kMaxRows]
  static constexpr int ml_off = mm_off + kWarps * kMaxRows * 4;       // [kWarps][kMaxRows]
  static constexpr int mo_off = ml_off + kWarps * kMaxRows * 4;       // [kWarps][kMaxRows][kOStride]
  // the merged rows' max, sum and 1 / sum
  static constexpr int rs_off = mo_off + kWarps * kMaxRows * kOStride * 4;  // [3][kMaxRows]
  static constexpr int merge_end = rs_off + 3 * kMaxRows * 4;
  // two piece slots: info, block ids, query rows
  static constexpr int kInfoBytes = 128;
  static constexpr int kIdsBytes = kDecodeMaxPieceBlocks * 4;
  static constexpr int kQBytes = kMaxRows * D * 2;
  static constexpr int kSlotBytes = kInfoBytes + kIdsBytes + kQBytes;
  static constexpr int slot_off = (merge_end + 127) / 128 * 128;
  // per compute warp: (piece, block) of each ring stage
  static constexpr int meta_off = slot_off + 2 * kSlotBytes;
  // per compute warp and stage: the mbarrier its TMA loads complete on
  static constexpr int bar_off = meta_off + kWarps * kStages * 8;
  // (+1024: the dynamic shared memory base is rounded up to 1024 bytes)
  static constexpr int total = bar_off + kWarps * kStages * 8 + 1024;
  static_assert(sizeof(PieceInfo) <= kInfoBytes, "piece info");
  static_assert(kSlotBytes % 16 == 0, "piece slot alignment");
  static_assert(total <= 227 * 1024, "shared memory of one CTA");
};

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

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Four 8 x 8 bf16 matrices from shared memory (one row address per lane:
// lanes 8i .. 8i + 7 address the rows of matrix i), as MMA fragments; the
// .trans form delivers each matrix transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t (&a)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&a)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
// An 8 x 8 bf16 matrix held one pair per lane (row lane / 4, columns
// 2 (lane % 4), + 1), transposed in registers.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// CTA-scope hand-offs in shared memory: release stores, acquire loads and
// acq_rel adds order the memory accesses around them without a full fence
// (a fence could also wait for the warp's copies still in flight).
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v)
               : "r"((uint32_t)__cvta_generic_to_shared(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(p)),
               "r"(v) : "memory");
}
__device__ __forceinline__ int add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old)
               : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(v) : "memory");
  return old;
}

// Shared control words of a CTA.
struct DecodeCtl {
  int merged;     // CTA-local sequence number of the last piece merged (-1: none)
  int count;      // blocks covered by the parts of the current piece in the merge slot
  int abort;      // set by a bounded wait that ran out: every role winds down
  int passed[2];  // compute warps with blocks in the piece in each slot whose issue cursor has left it
};

// One piece of the list (see DecodeWork): x = sequence, y = ql << 24 | rg << 22
// | kvh << 12 | part, z = seq_len, w = query_start_loc of the sequence.
__device__ __forceinline__ int4 load_piece(const AttnParams& p, const DecodeWork& work, int g) {
  return work.from_ws ? p.ws_pieces[g] : work.items[g];
}

// kWriteCache: the call writes the step's new K/V rows (the scheduler stores
// them before the blocks holding them are read).  kLateRows (with it): a piece
// is published before its rows are written, and the compute warps load the
// blocks holding them only once the scheduler releases cw_tag; used when the
// pieces are claimed, while pieces dealt on the host, staged well ahead of
// their use, are written first and published after (that wait, compiled into
// the issue path, measured 3 % slower on the prefix-cached step).
template <int D, int kMaxRows, bool kWriteCache, bool kLateRows>
__global__ void __launch_bounds__((DecodeCfg<D, kMaxRows>::kWarps + 1) * 32, 1)
decode_persistent_kernel(const AttnParams p, const __grid_constant__ DecodeWork work,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
  using LY = DecodeLayout<D, kMaxRows>;
  constexpr int kWarps = LY::kWarps;
  constexpr int kStages = LY::kStages;
  constexpr int kN = (kMaxRows + 7) / 8;  // 8-row n-tiles of query rows
  constexpr int NK = D / 16;  // 16-dim steps of K Q^T, 16-dim m-tiles of V^T P^T
  constexpr int kOStride = LY::kOStride;
  constexpr float kRescaleLog2 = 8.f;  // lazy-rescale threshold, log2 units
  constexpr int kChunks = D / 8;    // 16-byte chunks per tile row
  constexpr int kPanels = D / 64;   // 64-wide slices of D: one 16 x 64 TMA box each

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ DecodeCtl ctl;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t sraw = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (sbase - sraw);
  auto slot_info = [&](int p_) {
    return reinterpret_cast<PieceInfo*>(smem + LY::slot_off + (p_ & 1) * LY::kSlotBytes);
  };
  auto slot_ids = [&](int p_) {
    return reinterpret_cast<int*>(smem + LY::slot_off + (p_ & 1) * LY::kSlotBytes +
                                  LY::kInfoBytes);
  };
  auto slot_q = [&](int p_) {  // shared address of the slot's query rows [kMaxRows][D] bf16
    return sbase + LY::slot_off + (p_ & 1) * LY::kSlotBytes + LY::kInfoBytes + LY::kIdsBytes;
  };
  float* msl_m = reinterpret_cast<float*>(smem + LY::mm_off);
  float* msl_l = reinterpret_cast<float*>(smem + LY::ml_off);
  float* msl_o = reinterpret_cast<float*>(smem + LY::mo_off);
  float* row_m = reinterpret_cast<float*>(smem + LY::rs_off);
  float* row_l = row_m + kMaxRows;
  float* row_inv = row_l + kMaxRows;
  int* meta = reinterpret_cast<int*>(smem + LY::meta_off);  // [kWarps][kStages][2]
  const uint32_t bars = sbase + LY::bar_off;                 // [kWarps][kStages] mbarriers
  volatile int* vabort = &ctl.abort;
  int* status = p.ws_status;

  if (threadIdx.x == 0) {
    ctl.merged = -1;
    ctl.count = 0;
    ctl.abort = 0;
    ctl.passed[0] = ctl.passed[1] = 0;
    slot_info(0)->tag = -1;
    slot_info(1)->tag = -1;
    slot_info(0)->cw_tag = -1;
    slot_info(1)->cw_tag = -1;
    for (int i = 0; i < kWarps * kStages; ++i) mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  // A piece list in the kernel's parameters does not depend on the preceding
  // kernel: its size and the CTA's first piece are read before the wait.
  int num_pieces = 0, P = 0, g_begin = 0, g_end = 0;
  int4 first = make_int4(0, 0, 0, 0);
  if (warp == kWarps && !work.from_ws) {
    num_pieces = work.count;
    P = work.piece_blocks;
    if (work.dealt) {
      g_begin = work.cta_off[blockIdx.x];
      g_end = work.cta_off[blockIdx.x + 1];
    } else {
      g_begin = blockIdx.x;
      g_end = num_pieces;
    }
    if (g_begin < g_end) first = work.items[g_begin];
  }
  // Launched as a programmatic dependent: nothing the preceding kernel may
  // write is read before this wait; the next kernel may then be launched (it
  // waits for this grid in the same way).
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int G = p.group;

  if (warp == kWarps) {
    // =============================== scheduler ===============================
    if (work.from_ws) {
      num_pieces = p.ws_header[kWsPieceCount];
      P = p.ws_header[kWsPieceBlocks];
      g_begin = blockIdx.x;
      g_end = num_pieces;
    }
    const bool dealt = !work.from_ws && work.dealt;
    int prev_nb = 1;  // blocks of the piece staged last
    // the CTA's pieces are dealt to the compute warps as one round-robin:
    // each piece starts at the warp after the one that got the previous
    // piece's last block, so that no warp gets every piece's ragged remainder
    int rot = 0;
    for (int pc = 0;; ++pc) {
      // the next piece is claimed only once every block of the current one
      // has been issued (every compute warp with blocks there has moved its
      // issue cursor past it; the copies in flight then keep the warps busy
      // while the claim and the staging complete), so that the list's
      // largest-first order goes to the SMs that are free.  (Claiming when
      // the first warp moves on hides more of the staging but lets a CTA hold
      // pieces ahead of its progress, which costs more at the list's end.)
      // (pieces dealt on the host are staged as soon as their slot is free)
      if (pc >= 1 && !dealt &&
          !spin_until([&] { return ld_acquire(&ctl.passed[(pc - 1) & 1]) >= min(kWarps, prev_nb); },
                      vabort, status))
        break;
      // slot pc % 2 is free once piece pc - 2 has been merged
      if (pc >= 2 &&
          !spin_until([&] { return ld_acquire(&ctl.merged) >= pc - 2; }, vabort, status))
        break;
      int g = g_begin + pc;
      if (pc > 0 && !dealt) {
        if (lane == 0) g = gridDim.x + atomicAdd(p.ws_header + kWsClaim, 1);
        g = __shfl_sync(0xffffffffu, g, 0);
      }
      PieceInfo* inf = slot_info(pc);
      if (g >= g_end) {
        if (lane == 0) {
          inf->end = 1;
          st_release(&inf->tag, pc);
        }
        break;
      }
      const int4 it = (pc == 0 && !work.from_ws) ? first : load_piece(p, work, g);
      const int s = it.x;
      const int j = it.y & 0xfff, kvh = (it.y >> 12) & 0x3ff, rg = (it.y >> 22) & 3;
      const int ql = (it.y >> 24) & 0x7f;
      const int L = it.z, q0 = it.w;
      const int nblk = (L + kBlockSize - 1) / kBlockSize;
      const int nparts = (nblk + P - 1) / P;
      const int blk_begin = j * P;
      const int nb = min(P, nblk - blk_begin);
      const int rows_all = ql * G;
      const int row0 = kDecodeRows * rg;
      const int rows = min(kDecodeRows, rows_all - row0);
      // block ids and query rows (rows past the unit's are zero): every load
      // of a round is issued before its results are stored, so that a piece
      // is staged in one round trip to global memory (two for long pieces)
      const int32_t* table = p.block_tables + (int64_t)s * p.max_blocks_per_seq + blk_begin;
      int* ids = slot_ids(pc);
      constexpr int kQv = (kMaxRows * kChunks + 31) / 32;  // 16-byte query loads per lane
      // This step's new tokens of the sequence that fall in the piece's key
      // range (the one-call path writes them into their cache slots, as
      // pa_reshape_and_cache would): 16-byte chunks, K then V.  Lane t's
      // first chunk is loaded with the block ids and the query rows (with
      // kLateRows; otherwise when the rows are written).  When a unit's
      // query rows span several row groups, the pieces of each row group
      // over these keys store the same rows: identical bytes, so a CTA that
      // has completed its own stores reads the new values whatever the
      // others' stores are doing.
      int lo = 0, hi = 0;
      if constexpr (kWriteCache) {
        lo = max(L - ql, blk_begin * kBlockSize);
        hi = min(L, (blk_begin + nb) * kBlockSize);
      }
      const int ncw = hi > lo ? (hi - lo) * kChunks : 0;  // chunks per K (and per V)
      auto cw_src = [&](int i, bool& is_v, int& tok, int& c) {  // chunk i of the K and V rows
        is_v = i >= ncw;
        const int ii = is_v ? i - ncw : i;
        tok = q0 + (lo - (L - ql)) + ii / kChunks;
        c = ii % kChunks;
        return ((int64_t)tok * p.num_kv_heads + kvh) * kChunks + c;
      };
      int64_t cw_slot = -1;
      uint4 cw_val = make_uint4(0, 0, 0, 0);
      bool cw_isv = false;
      int cw_c = 0;
      if (kLateRows && lane < 2 * ncw) {
        int tok;
        const int64_t src = cw_src(lane, cw_isv, tok, cw_c);
        cw_slot = p.slot_mapping[tok];
        cw_val = cw_isv ? ((const uint4*)p.v_new)[src] : ((const uint4*)p.k_new)[src];
      }
      {
        const uint4* qg = (const uint4*)p.q;
        uint4 qv[kQv];
        int iv[8];
#pragma unroll
        for (int k = 0; k < kQv; ++k) {
          const int c = lane + 32 * k, i = c / kChunks, ch = c % kChunks;
          qv[k] = make_uint4(0, 0, 0, 0);
          if (c < kMaxRows * kChunks && i < rows) {
            const int gi = row0 + i;
            const int64_t tok = q0 + gi / G, head = (int64_t)kvh * G + gi % G;
            qv[k] = qg[(tok * p.num_q_heads + head) * kChunks + ch];
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) iv[k] = lane + 32 * k < nb ? table[lane + 32 * k] : 0;
        const uint32_t qs = slot_q(pc);
#pragma unroll
        for (int k = 0; k < kQv; ++k) {
          const int c = lane + 32 * k;
          if (c < kMaxRows * kChunks)
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(qs + c * 16),
                         "r"(qv[k].x), "r"(qv[k].y), "r"(qv[k].z), "r"(qv[k].w)
                         : "memory");
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (lane + 32 * k < nb) ids[lane + 32 * k] = iv[k];
        for (int base = 256; base < nb; base += 256) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int i = base + lane + 32 * k;
            iv[k] = i < nb ? table[i] : 0;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (base + lane + 32 * k < nb) ids[base + lane + 32 * k] = iv[k];
        }
      }
      prev_nb = nb;
      if (lane == 0) {
        ctl.passed[pc & 1] = 0;
        inf->end = 0;
        inf->s = s; inf->kvh = kvh; inf->rg = rg; inf->j = j; inf->nparts = nparts;
        inf->blk_begin = blk_begin; inf->nb = nb;
        inf->L = L; inf->ql = ql; inf->q0 = q0;
        inf->rows = rows; inf->row0 = row0;
        inf->rot = rot;
        inf->cw_first = ncw > 0 ? max(0, (L - ql) / kBlockSize - blk_begin) : nb;
      }
      rot = (rot + nb) % kWarps;
      __syncwarp();
      auto write_rows = [&]() {
        // With several 16-row groups, every row group's piece of the same
        // (sequence, kv-head, blocks) stores the same bytes to the same slots,
        // possibly while another CTA reads them: identical concurrent stores,
        // so every read sees the new row.  No other piece reads these slots.
        const int64_t num_slots = (int64_t)p.num_blocks * kBlockSize;
        uint4* kcw = (uint4*)const_cast<void*>(p.k_cache);
        uint4* vcw = (uint4*)const_cast<void*>(p.v_cache);
        auto store = [&](int64_t slot, bool is_v, int c, const uint4& v) {
          if (slot < 0 || slot >= num_slots) return;  // padding / out-of-pool slot
          const int64_t dst =
              ((slot / kBlockSize * p.num_kv_heads + kvh) * kBlockSize + slot % kBlockSize) *
                  kChunks + c;
          if (is_v) vcw[dst] = v;
          else kcw[dst] = v;
        };
        if (kLateRows && lane < 2 * ncw) store(cw_slot, cw_isv, cw_c, cw_val);
        for (int i = kLateRows ? lane + 32 : lane; i < 2 * ncw; i += 32) {  // (the rest)
          bool is_v;
          int tok, c;
          const int64_t src = cw_src(i, is_v, tok, c);
          const uint4 v = is_v ? ((const uint4*)p.v_new)[src] : ((const uint4*)p.k_new)[src];
          store(p.slot_mapping[tok], is_v, c, v);
        }
        // the compute warps read these rows with TMA (the async proxy)
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0) st_release(&inf->cw_tag, pc);
      };
      // With kLateRows the piece is published before the cache write (a
      // release after the write would wait for its global stores), and only
      // the blocks that receive new rows wait for cw_tag: the write's round
      // trips then stay off the path of the piece's other blocks.
      if (kWriteCache && !kLateRows && ncw > 0) write_rows();
      if (lane == 0) st_release(&inf->tag, pc);
      if (kLateRows && ncw > 0) write_rows();
    }
    // the last CTA to finish claiming resets the claim counter for the next call
    if (lane == 0 && !dealt) {
      __threadfence();
      const int prev = atomicAdd(p.ws_header + kWsDone, 1);
      if (prev == (int)gridDim.x - 1) {
        atomicExch(p.ws_header + kWsClaim, 0);
        atomicExch(p.ws_header + kWsDone, 0);
      }
    }
    return;
  }

  // ================================ compute warps ================================
  const int r = lane >> 2, q4 = lane & 3;
  const int oob_bh = p.num_blocks * p.num_kv_heads;  // first (block, kv-head) row past the pool
  const uint32_t ring = sbase + LY::ring_off + warp * kStages * LY::kStageBytes;
  int* my_meta = meta + warp * kStages * 2;
  // ldmatrix rows this lane addresses: matrix lane / 8, row lane % 8 of it.
  // K as the A operand (keys x dims): matrix mi holds keys 8 * (mi & 1) + 0..7
  // of the 16-byte chunk 2 * kk + (mi >> 1); V^T as the A operand (dims x
  // keys): matrix mi holds keys 8 * (mi >> 1) + 0..7 of chunk 2 * mt + (mi & 1).
  // With the 128-byte swizzle, chunk c of row t sits at chunk c ^ (t % 8) of
  // its 128-byte row, and the chunk pairs (2k, 2k + 1) never straddle a box.
  const int mi = lane >> 3, mrow = lane & 7;
  const uint32_t k_row = (8 * (mi & 1) + mrow) * 128;
  const int k_hx = (mi >> 1) ^ mrow;
  const uint32_t v_row = LY::kTileBytes + (8 * (mi >> 1) + mrow) * 128;
  const int v_hx = (mi & 1) ^ mrow;

  // State of piece pc's slot as this warp sees it: 0 not published yet, 1
  // published, 2 already reused for a later piece.  The tag is read (with
  // acquire order) only until the warp has seen the piece published.  A slot
  // is reused for piece pc + 2 only after piece pc has been merged, which
  // needs every warp with blocks in it: a warp that finds the slot reused had
  // none there (it lagged behind while the piece went by) and skips it.
  int seen = -1;  // the latest piece this warp has seen published
  auto slot_state = [&](int pc) -> int {
    if (pc <= seen) return 1;
    const int tag = ld_acquire(&slot_info(pc)->tag);
    if (tag < pc) return 0;
    if (tag > pc) return 2;
    seen = pc;
    return 1;
  };

  int ip = 0, ii = -1;  // issue cursor: next candidate (piece, block of the piece; -1: its first)
  // blocks receiving the step's new rows wait for them (kLateRows: the piece
  // is published before the write)
  constexpr bool cw_wait = kLateRows;
  bool issue_done = false;
  int n_issued = 0, n_comp = 0;
  uint32_t bad = 0;  // bit (stage): that stage's block id was outside the pool

  // The copies of block i of piece pc (id: its cache block, kvh: the piece's
  // kv-head) into the next ring stage.
  auto issue_stage = [&](int pc, int i, int id, int kvh) {
    const int st = n_issued % kStages;
    // a block id outside the pool is never dereferenced: the box is read from
    // past the tensor's extent (zeros) and its keys are masked
    const bool id_ok = id >= 0 && id < p.num_blocks;
    if (id_ok) bad &= ~(1u << st);
    else bad |= 1u << st;
    const int row_bh = id_ok ? id * p.num_kv_heads + kvh : oob_bh;
    if (lane == 0) {
      const uint32_t ks = ring + st * LY::kStageBytes;
      const uint32_t bar = bars + 8 * (warp * kStages + st);
      // (the warp's earlier reads of this stage have completed: their values
      // went into MMAs before the stage was freed)
      mbar_expect_tx(bar, LY::kStageBytes);
#pragma unroll
      for (int pn = 0; pn < kPanels; ++pn) {
        tma_load_3d(ks + pn * 2048, &tm_k, 64 * pn, 0, row_bh, bar);
        tma_load_3d(ks + LY::kTileBytes + pn * 2048, &tm_v, 64 * pn, 0, row_bh, bar);
      }
    }
    // (every lane stores the same values and reads back only what it stored)
    my_meta[2 * st] = pc;
    my_meta[2 * st + 1] = i;
    ++n_issued;
  };

  // Issue the copies of this warp's next block; false when there is none yet
  // (the next piece is not published and `block` is false) or none at all.
  // Warp w takes the blocks c, c + kWarps, ... of every piece, c = (w - rot)
  // mod kWarps: a fixed grouping, so that the piece's result does not depend
  // on timing.
  auto try_issue = [&](bool block) -> bool {
    const PieceInfo* inf;
    while (true) {
      int state = slot_state(ip);
      if (state == 0) {
        if (!block) return false;
        if (!spin_until([&] { return (state = slot_state(ip)) != 0; }, vabort, status)) {
          issue_done = true;
          return false;
        }
      }
      if (state == 2) {  // a piece without blocks of this warp, gone by
        ++ip;
        ii = -1;
        continue;
      }
      inf = slot_info(ip);
      if (inf->end) {
        issue_done = true;
        return false;
      }
      const int first = (warp - inf->rot + kWarps) % kWarps;
      if (ii < 0) ii = first;
      if (ii < inf->nb) break;
      // this warp leaves piece ip (counted when it had blocks there)
      if (lane == 0 && first < inf->nb) atomicAdd(&ctl.passed[ip & 1], 1);
      ++ip;
      ii = -1;
    }
    // a block that receives the step's new rows is loaded only once the
    // scheduler has written them (the piece is published before that write)
    if (cw_wait && ii >= inf->cw_first && ld_acquire(&inf->cw_tag) < ip) {
      if (!block) return false;
      if (!spin_until([&] { return ld_acquire(&inf->cw_tag) >= ip; }, vabort, status)) {
        issue_done = true;
        return false;
      }
    }
    issue_stage(ip, ii, slot_ids(ip)[ii], inf->kvh);
    ii += kWarps;
    return true;
  };

  // per-piece state of this warp.  Fragment ownership: lane (r, q4) holds the
  // query rows 8n + 2q4 and 8n + 2q4 + 1 of n-tile n (h = 0, 1), the keys r
  // and r + 8 of a block in S^T, and the dims 16mt + r and 16mt + r + 8 of
  // m-tile mt in O^T.
  int cur = -1;   // piece being accumulated
  int n_cur = 0;  // blocks of it this warp has accumulated
  uint32_t qf[kN][NK][2];  // Q^T as the B operand: rows 8n + r, dims 16kk + 2q4 (+8)
  float o[kN][NK][4];      // O^T: [dim 16mt + r (+8)][row 8n + 2q4 (+1)]
  float m[kN][2], mb[kN][2], l[kN][2];  // running max, exponent base, this lane's partial sum
  int lim[kN][2], first_masked = 0;

  // The warp's part of piece pc is done: its (max, sum, O) go to the merge
  // slot; the last warp to arrive merges and stores the piece's result.
  auto flush = [&](int pc, const PieceInfo* inf) -> bool {
#pragma unroll
    for (int n = 0; n < kN; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // the sum over the eight lanes holding the row's keys
        l[n][h] += __shfl_xor_sync(0xffffffffu, l[n][h], 4);
        l[n][h] += __shfl_xor_sync(0xffffffffu, l[n][h], 8);
        l[n][h] += __shfl_xor_sync(0xffffffffu, l[n][h], 16);
      }
    // the merge slot holds one piece at a time: the previous one must be
    // merged.  The warp's part goes to the place of its block subset c.
    if (!spin_until([&] { return ld_acquire(&ctl.merged) >= pc - 1; }, vabort, status))
      return false;
    const int rot = inf->rot;
    const int sub = warp >= rot ? warp - rot : warp - rot + kWarps;
    if (r == 0) {
#pragma unroll
      for (int n = 0; n < kN; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = 8 * n + 2 * q4 + h;
          if (row < kMaxRows) {
            msl_m[sub * kMaxRows + row] = m[n][h];
            msl_l[sub * kMaxRows + row] = l[n][h];
          }
        }
    }
    float* mo = msl_o + sub * kMaxRows * kOStride;
#pragma unroll
    for (int n = 0; n < kN; ++n)
#pragma unroll
      for (int mt = 0; mt < NK; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = 8 * n + 2 * q4 + (c & 1);
          if (row < kMaxRows) mo[row * kOStride + 16 * mt + r + 8 * (c >> 1)] = o[n][mt][c];
        }
    __syncwarp();
    int last = 0;  // the blocks of every part are in: this warp merges
    if (lane == 0) last = add_acq_rel(&ctl.count, n_cur) + n_cur == inf->nb;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return true;
    __syncwarp();  // every lane reads the other warps' parts after lane 0's acquire

    // ---- merge the warps' parts of the piece: shared memory in, global
    // stores out, then the merge slot is free again (no round trip to global
    // memory while the other warps may wait for the slot).  The parts are
    // placed and combined in block-subset order whichever warp merges, so the
    // result does not depend on timing or on the piece's rotation.
    const int rows = inf->rows, row0 = inf->row0, q0 = inf->q0;
    const int kvh = inf->kvh, rg = inf->rg, np = inf->nparts, ql = inf->ql;
    const int nw = min(kWarps, inf->nb);  // parts present: block subsets 0 .. nw - 1
    const int unit = inf->s * p.num_kv_heads + kvh;
    __nv_bfloat16* out = (__nv_bfloat16*)p.out;
    constexpr int D4 = D / 4;
    const bool direct = np == 1;
    const int64_t slot0 = ((int64_t)unit * p.max_parts + inf->j * p.row_groups + rg) * kDecodeRows;
    {
      // per row: the max over the parts, each part's weight 2^(m_c - max)
      // (written over its max), and the weighted sum of the parts' sums; the
      // 32 / kMaxRows lanes of a row share its parts
      constexpr int W = 32 / kMaxRows;
      constexpr int kPer = (kWarps + W - 1) / W;
      const int i = lane % kMaxRows, wg = lane / kMaxRows;
      float mv[kPer], lv[kPer];
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = wg + W * k;
        const bool has = c < nw;
        mv[k] = has ? msl_m[c * kMaxRows + i] : -INFINITY;
        lv[k] = has ? msl_l[c * kMaxRows + i] : 0.f;
        M = fmaxf(M, mv[k]);
      }
#pragma unroll
      for (int off = kMaxRows; off < 32; off <<= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      const float base = (M == -INFINITY) ? 0.f : M;
      float Ls = 0.f;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = wg + W * k;
        const float wt = ex2(mv[k] - base);  // 0 for a missing part
        Ls += lv[k] * wt;
        if (c < kWarps) msl_m[c * kMaxRows + i] = wt;
      }
#pragma unroll
      for (int off = kMaxRows; off < 32; off <<= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
      if (wg == 0) {
        row_m[i] = M;
        row_l[i] = Ls;
        row_inv[i] = Ls > 0.f ? 1.f / Ls : 0.f;
      }
    }
    __syncwarp();
    // the weighted sums of the parts' O rows, each written back over part
    // 0's element (read by this lane only), then the stores from there; the
    // merge slot is released last.  No global store is issued among the
    // shared-memory loads of the sums, where it would hold them up.
    const uint32_t part0 = sbase + LY::mo_off;
    auto sums = [&](auto all_parts) {
      constexpr bool kAll = decltype(all_parts)::value;
      for (int e = lane; e < rows * D4; e += 32) {
        const int i = e / D4, d4 = e % D4;
        const uint32_t wrow = sbase + LY::mm_off + i * 4;
        const uint32_t orow = part0 + (i * kOStride + 4 * d4) * 4;
        // in batches of parts, every load of a batch issued before its sums
        // (a part past nw reads stale bytes, replaced by 0)
        constexpr int kB = kWarps > 6 ? (kWarps + 1) / 2 : kWarps;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int b = 0; b < kWarps; b += kB) {
          float wt[kB];
          float4 v[kB];
#pragma unroll
          for (int k = 0; k < kB && b + k < kWarps; ++k) {
            wt[k] = __uint_as_float(lds32(wrow + (b + k) * (kMaxRows * 4)));
            v[k] = lds_f4(orow + (b + k) * (kMaxRows * kOStride * 4));
          }
#pragma unroll
          for (int k = 0; k < kB && b + k < kWarps; ++k) {
            const bool has = kAll || b + k < nw;
            acc.x = fmaf(has ? v[k].x : 0.f, wt[k], acc.x);
            acc.y = fmaf(has ? v[k].y : 0.f, wt[k], acc.y);
            acc.z = fmaf(has ? v[k].z : 0.f, wt[k], acc.z);
            acc.w = fmaf(has ? v[k].w : 0.f, wt[k], acc.w);
          }
        }
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(orow), "f"(acc.x),
                     "f"(acc.y), "f"(acc.z), "f"(acc.w)
                     : "memory");
      }
    };
    if (nw == kWarps) sums(std::true_type{});
    else sums(std::false_type{});
    __syncwarp();
    if (direct) {  // 8 dims (16 bytes of output) per lane and store
      constexpr int D8 = D / 8;
      for (int e = lane; e < rows * D8; e += 32) {
        const int i = e / D8, d8 = e % D8;
        const float4 a0 = lds_f4(part0 + (i * kOStride + 8 * d8) * 4);
        const float4 a1 = lds_f4(part0 + (i * kOStride + 8 * d8 + 4) * 4);
        const float inv = row_inv[i];
        const int gi = row0 + i;
        // one query token: its rows are consecutive heads of the kv-head
        const int64_t tok = ql == 1 ? q0 : q0 + gi / G;
        const int64_t head = (int64_t)kvh * G + (ql == 1 ? gi : gi % G);
        uint4 pk;
        pk.x = pack_bf16x2(a0.x * inv, a0.y * inv);
        pk.y = pack_bf16x2(a0.z * inv, a0.w * inv);
        pk.z = pack_bf16x2(a1.x * inv, a1.y * inv);
        pk.w = pack_bf16x2(a1.z * inv, a1.w * inv);
        *reinterpret_cast<uint4*>(out + (tok * p.num_q_heads + head) * D + 8 * d8) = pk;
      }
    } else {
      for (int e = lane; e < rows * D4; e += 32) {
        const int i = e / D4, d4 = e % D4;
        reinterpret_cast<float4*>(p.ws_o)[(slot0 + i) * D4 + d4] =
            lds_f4(part0 + (i * kOStride + 4 * d4) * 4);
      }
      if (lane < rows)
        reinterpret_cast<float2*>(p.ws_ml)[slot0 + lane] = make_float2(row_m[lane], row_l[lane]);
    }
    __syncwarp();  // every lane is done with the merge slot and the piece slot
    if (lane == 0) {
      ctl.count = 0;
      st_release(&ctl.merged, pc);
    }
    __syncwarp();
    return true;
  };

  // The CTA's first piece, when the list is in the kernel parameters: the
  // warp's first blocks of it are issued straight from the block table (the
  // piece's rotation is 0), while the scheduler stages the piece, so the
  // first K/V tiles are on their way one round trip earlier.  Blocks that
  // receive this step's new K/V rows are left to the normal path, which
  // issues them only after the scheduler has written those rows.
  if (!work.from_ws) {
    const int gb = work.dealt ? work.cta_off[blockIdx.x] : (int)blockIdx.x;
    const int ge = work.dealt ? work.cta_off[blockIdx.x + 1] : work.count;
    if (gb < ge) {
      const int4 it = work.items[gb];
      const int s0 = it.x, j0 = it.y & 0xfff, kvh0 = (it.y >> 12) & 0x3ff;
      const int ql0 = (it.y >> 24) & 0x7f, L0 = it.z;
      const int P0 = work.piece_blocks;
      const int blk_begin = j0 * P0;
      const int nb0 = min(P0, (L0 + kBlockSize - 1) / kBlockSize - blk_begin);
      const int lim = kWriteCache ? min(nb0, max(0, (L0 - ql0) / kBlockSize - blk_begin)) : nb0;
      const int32_t* table = p.block_tables + (int64_t)s0 * p.max_blocks_per_seq + blk_begin;
      int id = 0;
      if (lane < kStages && warp + lane * kWarps < lim) id = table[warp + lane * kWarps];
#pragma unroll
      for (int k = 0; k < kStages; ++k) {
        const int idk = __shfl_sync(0xffffffffu, id, k);
        if (warp + k * kWarps < lim) issue_stage(0, warp + k * kWarps, idk, kvh0);
      }
      ii = warp + n_issued * kWarps;  // the next block of the piece to issue
    }
  }

  while (true) {
    // keep kStages blocks in flight; wait for a piece to be published only
    // when nothing is in flight
    while (!issue_done && n_issued - n_comp < kStages) {
      if (!try_issue(n_issued == n_comp)) break;
    }
    if (n_issued == n_comp) break;  // the list is exhausted (or the CTA aborted)
    if (!wait_bar(bars + 8 * (warp * kStages + n_comp % kStages), (n_comp / kStages) & 1, vabort,
                  status))
      break;  // the oldest stage's K and V tiles have landed (or the CTA gave up)

    const int st = n_comp % kStages;
    const int pc = my_meta[2 * st], i = my_meta[2 * st + 1];
    // (a block issued before its piece was published: the piece's query rows
    // and fields are read once it is)
    if (pc > seen && !spin_until([&] { return slot_state(pc) == 1; }, vabort, status)) break;
    const PieceInfo* inf = slot_info(pc);
    const int L = inf->L;
    if (pc != cur) {
      // ---- a new piece: its query rows as the B operand (rows past the
      // unit's are zero), fresh running max, sum and O
      cur = pc;
      n_cur = 0;
      const uint32_t qs = slot_q(pc);
#pragma unroll
      for (int n = 0; n < kN; ++n) {
        const int row = 8 * n + r;
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
          qf[n][kk][0] = row < kMaxRows ? lds32(qs + (row * D + 16 * kk + 2 * q4) * 2) : 0u;
          qf[n][kk][1] = row < kMaxRows ? lds32(qs + (row * D + 16 * kk + 8 + 2 * q4) * 2) : 0u;
        }
      }
      const int rows = inf->rows, ql = inf->ql;
#pragma unroll
      for (int n = 0; n < kN; ++n) {
#pragma unroll
        for (int mt = 0; mt < NK; ++mt) o[n][mt][0] = o[n][mt][1] = o[n][mt][2] = o[n][mt][3] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          m[n][h] = -INFINITY;
          mb[n][h] = 0.f;
          l[n][h] = 0.f;
          // causal limit of the row: query j of the sequence sees keys <= L - ql + j
          lim[n][h] = L - ql + (inf->row0 + min(8 * n + 2 * q4 + h, rows - 1)) / G;
        }
      }
      first_masked = L - ql + 1;  // keys at or beyond this may be masked for some row
    }

    const int kb = (inf->blk_begin + i) * kBlockSize;  // first key of the block
    const bool blk_ok = !((bad >> st) & 1u);
    const uint32_t ks = ring + st * LY::kStageBytes;

    // ---- S^T = K Q^T: keys on the MMA's M side, query rows on N; per n-tile
    // two accumulators (even and odd 16-dim steps) keep the chains short
    float x[kN][4];
    {
      float sa[kN][2][4];
#pragma unroll
      for (int n = 0; n < kN; ++n)
#pragma unroll
        for (int a = 0; a < 2; ++a) sa[n][a][0] = sa[n][a][1] = sa[n][a][2] = sa[n][a][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, ks + (kk >> 2) * 2048 + k_row + ((((2 * kk) & 7) ^ k_hx) << 4));
#pragma unroll
        for (int n = 0; n < kN; ++n)
          mma_16816(sa[n][kk & 1], a[0], a[1], a[2], a[3], qf[n][kk][0], qf[n][kk][1]);
      }
#pragma unroll
      for (int n = 0; n < kN; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) x[n][c] = (sa[n][0][c] + sa[n][1][c]) * p.scale_log2;
    }
    // ---- mask: keys past a row's causal limit (past seq_len for a decode)
    // and every key of a block outside the pool
    if (kb + kBlockSize > first_masked || !blk_ok) {
#pragma unroll
      for (int n = 0; n < kN; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (!blk_ok || kb + r + 8 * (c >> 1) > lim[n][c & 1]) x[n][c] = -INFINITY;
    }
    // ---- online softmax with a lazy rescale: the running max of a row moves
    // (and O and the sums are rescaled) only when some score exceeds it by
    // more than kRescaleLog2, so exp2(score - base) stays below
    // 2^kRescaleLog2 and most blocks skip the row reduction
    bool need = false;
#pragma unroll
    for (int n = 0; n < kN; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) need |= fmaxf(x[n][h], x[n][h + 2]) > m[n][h] + kRescaleLog2;
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int n = 0; n < kN; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float bm = fmaxf(x[n][h], x[n][h + 2]);
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
          bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
          const float mn = fmaxf(m[n][h], bm);
          if (mn > m[n][h]) {
            const float al = ex2(m[n][h] - mn);  // 0 while the row had no finite score
            m[n][h] = mn;
            mb[n][h] = mn;
            l[n][h] *= al;
#pragma unroll
            for (int mt = 0; mt < NK; ++mt) {
              o[n][mt][h] *= al;
              o[n][mt][h + 2] *= al;
            }
          }
        }
    }
    // ---- P^T as the B operand of O^T += V^T P^T: the bf16 pairs of P in the
    // S^T fragment (keys r / r + 8, rows 2q4, 2q4 + 1) are transposed 8 x 8 to
    // the B fragment (keys 2q4, 2q4 + 1 / + 8, row r)
    uint32_t pb[kN][2];
#pragma unroll
    for (int n = 0; n < kN; ++n) {
      float pr[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) pr[c] = ex2(x[n][c] - mb[n][c & 1]);
      l[n][0] += pr[0] + pr[2];
      l[n][1] += pr[1] + pr[3];
      pb[n][0] = movm_t(pack_bf16x2(pr[0], pr[1]));
      pb[n][1] = movm_t(pack_bf16x2(pr[2], pr[3]));
    }
    // slots of the last block past seq_len (and blocks outside the pool) may
    // hold anything, NaN included: their V elements become zeros so that the
    // zero weights cannot turn them into NaN in the P.V product
    uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;  // keys 2q4, 2q4 + 1 / 2q4 + 8, 2q4 + 9
    const bool vtail = kb + kBlockSize > L || !blk_ok;
    if (vtail) {
      const int k0 = kb + 2 * q4;
      vm0 = !blk_ok ? 0u : (k0 < L ? 0xffffu : 0u) | (k0 + 1 < L ? 0xffff0000u : 0u);
      vm1 = !blk_ok ? 0u : (k0 + 8 < L ? 0xffffu : 0u) | (k0 + 9 < L ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < NK; ++mt) {
      uint32_t a[4];
      ldsm_x4_t(a, ks + (mt >> 2) * 2048 + v_row + ((((2 * mt) & 7) ^ v_hx) << 4));
      if (vtail) {
        a[0] &= vm0; a[1] &= vm0; a[2] &= vm1; a[3] &= vm1;
      }
#pragma unroll
      for (int n = 0; n < kN; ++n) mma_16816(o[n][mt], a[0], a[1], a[2], a[3], pb[n][0], pb[n][1]);
    }
    ++n_comp;
    ++n_cur;
    if (i + kWarps >= inf->nb) {  // this warp's last block of the piece
      __syncwarp();  // every lane is done with the stage before it is refilled
      if (!flush(pc, inf)) break;
    }
    __syncwarp();  // every lane is done with the stage freed above before it is refilled
  }
  // no TMA load may still target the ring when the CTA exits (only after a
  // wait gave up: a normal exit has consumed every stage it loaded)
  for (int n = n_comp; n < n_issued; ++n) {  // loaded, never waited for
    const uint32_t b = bars + 8 * (warp * kStages + n % kStages);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(b, (n / kStages) & 1) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
}

template <int D, int kMaxRows, bool kWriteCache, bool kLateRows>
cudaError_t launch_one(const AttnParams& p, const DecodeWork& work, int grid,
                       cudaStream_t stream) {
  using LY = DecodeLayout<D, kMaxRows>;
  CUtensorMap tk, tv;
  if (!make_map(&tk, p.k_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1) ||
      !make_map(&tv, p.v_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1))
    return cudaErrorInvalidValue;
  auto kernel = decode_persistent_kernel<D, kMaxRows, kWriteCache, kLateRows>;
  static std::atomic<int> smem_done[64];
  cudaError_t e = raise_smem_limit(kernel, LY::total, smem_done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((LY::kWarps + 1) * 32);
  cfg.dynamicSmemBytes = LY::total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p, work, tk, tv);
}

template <int D, bool kWriteCache, bool kLateRows>
cudaError_t launch_rows(const AttnParams& p, const DecodeWork& work, int grid, int max_rows,
                        cudaStream_t stream) {
  if (max_rows <= 4) return launch_one<D, 4, kWriteCache, kLateRows>(p, work, grid, stream);
  if (max_rows <= 8) return launch_one<D, 8, kWriteCache, kLateRows>(p, work, grid, stream);
  return launch_one<D, 16, kWriteCache, kLateRows>(p, work, grid, stream);
}

// ------------------------------------------------------------------ piece lists

// Decode-class test and block count of sequence s (0: no decode work).
__host__ __device__ __forceinline__ int decode_blocks(int ql, int L, int group, int max_seq_len,
                                                      int max_blocks_per_seq) {
  if (ql <= 0 || ql > L || ql * group > kDecodeMaxRows || L > max_seq_len) return 0;
  const int nblk = (L + kBlockSize - 1) / kBlockSize;
  return nblk <= max_blocks_per_seq ? nblk : 0;
}

// Blocks per piece: about total / (kDecodePiecesPerCta * ctas), so that every
// CTA gets a few pieces, and no more than kDecodeMaxPieceBytes of K+V, so
// that the last pieces of a big step stay short; but never fewer than the
// workspace's partial slots allow for the longest unit.
__host__ __device__ __forceinline__ int choose_piece_blocks(long long total_blocks, int max_nblk,
                                                            int ctas, int slots_per_unit,
                                                            int head_dim) {
  // Whole units when none is much longer than a CTA's share of the step: the
  // largest-first claims then balance the SMs, and no unit needs a merge of
  // partials across CTAs.
  const long long share = total_blocks / max(1, ctas);
  if (max_nblk <= kDecodeMaxPieceBlocks && 5ll * max_nblk <= 6 * share + 5 * 16) return max(1, max_nblk);
  long long want = (total_blocks + (long long)kDecodePiecesPerCta * ctas - 1) /
                   ((long long)kDecodePiecesPerCta * ctas);
  if (want < kDecodeMinPieceBlocks) want = kDecodeMinPieceBlocks;
  const long long cap = kDecodeMaxPieceBytes / (2 * kBlockSize * head_dim * 2);
  if (want > cap) want = cap;
  const long long need = (max_nblk + slots_per_unit - 1) / max(1, slots_per_unit);
  if (want < need) want = need;
  if (want > kDecodeMaxPieceBlocks) want = kDecodeMaxPieceBlocks;
  return (int)want;
}

__host__ __device__ __forceinline__ int4 make_piece(int s, int kvh, int rg, int j, int ql, int L,
                                                    int q0) {
  return make_int4(s, (ql << 24) | (rg << 22) | (kvh << 12) | j, L, q0);
}

// One CTA: the piece list of every decode-class sequence, written to the
// workspace (count, blocks per piece, then the pieces, largest first).
__global__ void __launch_bounds__(1024)
decode_plan_kernel(const AttnParams p, int ctas, int head_dim, int whole_units) {
  __shared__ unsigned long long sh_total;
  __shared__ int sh_max_nblk, sh_P, sh_full, sh_count;
  __shared__ int hist[kDecodeMaxPieceBlocks + 1];  // tail pieces by size, then offsets
  // the decode kernel may be launched at once: it waits for this grid before
  // it reads the list
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) {
    sh_total = 0;
    sh_max_nblk = 0;
    sh_full = 0;
  }
  for (int i = threadIdx.x; i <= kDecodeMaxPieceBlocks; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int G = p.group, H = p.num_kv_heads;
  auto groups_of = [&](int ql) { return (ql * G + kDecodeRows - 1) / kDecodeRows; };
  // pass 1: total blocks over the units, longest unit
  unsigned long long tot = 0;
  int mx = 0;
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    const int nblk = decode_blocks(ql, L, G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    tot += (unsigned long long)nblk * H * groups_of(ql);
    mx = max(mx, nblk);
  }
  atomicAdd(&sh_total, tot);
  atomicMax(&sh_max_nblk, mx);
  __syncthreads();
  if (threadIdx.x == 0)
    sh_P = whole_units ? max(1, sh_max_nblk)
                       : choose_piece_blocks((long long)sh_total, sh_max_nblk, ctas,
                                             p.max_parts / max(1, p.row_groups), head_dim);
  __syncthreads();
  const int P = sh_P;
  // pass 2: count the full pieces and the tail pieces by size
  int full = 0;
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    const int nblk = decode_blocks(ql, L, G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    const int units = H * groups_of(ql);
    full += units * (nblk / P);
    if (nblk % P) atomicAdd(&hist[nblk % P], units);
  }
  atomicAdd(&sh_full, full);
  __syncthreads();
  if (threadIdx.x == 0) {  // offsets: full pieces from 0, then tails by falling size
    int run = sh_full;
    for (int sz = P - 1; sz >= 1; --sz) {
      const int c = hist[sz];
      hist[sz] = run;
      run += c;
    }
    sh_count = min(run, p.max_pieces);
    sh_full = 0;  // becomes the running offset of the full pieces
    p.ws_header[kWsPieceCount] = sh_count;
    p.ws_header[kWsPieceBlocks] = P;
  }
  __syncthreads();
  // pass 3: scatter
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
    const int nblk = decode_blocks(ql, L, G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    const int ng = groups_of(ql), nf = nblk / P;
    if (nf) {
      int at = atomicAdd(&sh_full, H * ng * nf);
      for (int kvh = 0; kvh < H; ++kvh)
        for (int rg = 0; rg < ng; ++rg)
          for (int j = 0; j < nf; ++j, ++at)
            if (at < p.max_pieces) p.ws_pieces[at] = make_piece(s, kvh, rg, j, ql, L, q0);
    }
    if (nblk % P) {
      int at = atomicAdd(&hist[nblk % P], H * ng);
      for (int kvh = 0; kvh < H; ++kvh)
        for (int rg = 0; rg < ng; ++rg, ++at)
          if (at < p.max_pieces) p.ws_pieces[at] = make_piece(s, kvh, rg, nf, ql, L, q0);
    }
  }
}

// The same list built on the host from its copies of the lengths; false when
// it holds more pieces than a kernel parameter carries.
bool host_piece_list(DecodeWork* work, const AttnParams& p, const int32_t* seq_lens_host,
                     const int32_t* query_start_loc_host, int ctas, int head_dim) {
  const int G = p.group, H = p.num_kv_heads;
  auto groups_of = [&](int ql) { return (ql * G + kDecodeRows - 1) / kDecodeRows; };
  long long total = 0;
  int mx = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int ql = query_start_loc_host[s + 1] - query_start_loc_host[s];
    const int nblk = decode_blocks(ql, seq_lens_host[s], G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    total += (long long)nblk * H * groups_of(ql);
    mx = max(mx, nblk);
  }
  const int P =
      choose_piece_blocks(total, mx, ctas, p.max_parts / max(1, p.row_groups), head_dim);
  static thread_local int hist[kDecodeMaxPieceBlocks + 1];
  for (int i = 0; i <= P; ++i) hist[i] = 0;
  long long full = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int ql = query_start_loc_host[s + 1] - query_start_loc_host[s];
    const int nblk = decode_blocks(ql, seq_lens_host[s], G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    const int units = H * groups_of(ql);
    full += (long long)units * (nblk / P);
    if (nblk % P) hist[nblk % P] += units;
  }
  long long run = full;
  for (int sz = P - 1; sz >= 1; --sz) {
    const int c = hist[sz];
    hist[sz] = (int)min(run, (long long)INT32_MAX);
    run += c;
  }
  if (run > kDecodeParamPieces) return false;
  int at_full = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int q0 = query_start_loc_host[s], ql = query_start_loc_host[s + 1] - q0;
    const int L = seq_lens_host[s];
    const int nblk = decode_blocks(ql, L, G, p.max_seq_len, p.max_blocks_per_seq);
    if (!nblk || ql * G > p.decode_rows) continue;
    const int ng = groups_of(ql), nf = nblk / P;
    for (int kvh = 0; kvh < H; ++kvh)
      for (int rg = 0; rg < ng; ++rg) {
        for (int j = 0; j < nf; ++j) work->items[at_full++] = make_piece(s, kvh, rg, j, ql, L, q0);
        if (nblk % P) work->items[hist[nblk % P]++] = make_piece(s, kvh, rg, nf, ql, L, q0);
      }
  }
  work->count = (int)run;
  work->piece_blocks = P;
  work->from_ws = 0;
  work->split = mx > P;  // some unit has more than one piece
  work->dealt = 0;
  return true;
}

// Deals the list's pieces (longest first) to `ctas` CTAs: each to the CTA
// with the least work so far, a piece costing its blocks plus
// kDecodePieceCostBlocks.  CTA b's pieces then sit at items cta_off[b] ..
// cta_off[b + 1] - 1, in the order dealt, so that each CTA can stage its next
// piece while the current one streams instead of claiming it when it is
// nearly done.  (The claims of a shared counter adapt to SMs that run slower,
// but every claim's round trips and staging then sit on the CTA's path.)
constexpr int kDecodeDealPiecesPerCta = 4;
// a device-listed launch keeps units whole when no unit can exceed this many
// blocks (by the host's bound on the lengths)
constexpr int kDecodeWholeUnitBlocks = 256;

void deal_pieces(DecodeWork* work, int ctas) {
  const int n = work->count, P = work->piece_blocks;
  if (ctas <= 0 || ctas > kDecodeMaxDealtCtas || n < ctas) return;
  static thread_local int4 items[kDecodeParamPieces];
  static thread_local int owner[kDecodeParamPieces];
  static thread_local int count[kDecodeMaxDealtCtas];
  using Load = std::pair<long long, int>;  // (work so far, CTA)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int b = 0; b < ctas; ++b) {
    heap.push({0, b});
    count[b] = 0;
  }
  for (int g = 0; g < n; ++g) {  // the list is longest first
    const int4 it = work->items[g];
    const int nblk = (it.z + kBlockSize - 1) / kBlockSize, j = it.y & 0xfff;
    const int nb = std::min(P, nblk - j * P);
    Load l = heap.top();
    heap.pop();
    owner[g] = l.second;
    ++count[l.second];
    l.first += nb + kDecodePieceCostBlocks;
    heap.push(l);
  }
  work->cta_off[0] = 0;
  for (int b = 0; b < ctas; ++b) work->cta_off[b + 1] = work->cta_off[b] + count[b];
  for (int b = 0; b < ctas; ++b) count[b] = work->cta_off[b];
  for (int g = 0; g < n; ++g) items[count[owner[g]]++] = work->items[g];
  std::memcpy(work->items, items, sizeof(int4) * n);
  work->dealt = 1;
}

// ------------------------------------------------------------------ combine

// One warp per unit (sequence, kv-head, row group) whose blocks were cut into
// more than one piece: merges the pieces' fp32 partials (running max, sum,
// unnormalised O per row) into the output rows.  Launched as a programmatic
// dependent of the decode kernel: it reads the partials only after that grid
// has completed.
template <int D>
__global__ void __launch_bounds__(256)
decode_combine_kernel(const AttnParams p, int piece_blocks, int from_ws) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long u = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int RG = p.row_groups, G = p.group;
  if (u >= (long)p.num_seqs * p.num_kv_heads * RG) return;
  const int rg = (int)(u % RG);
  const int kvh = (int)((u / RG) % p.num_kv_heads);
  const int s = (int)(u / ((long)RG * p.num_kv_heads));
  const int P = from_ws ? p.ws_header[kWsPieceBlocks] : piece_blocks;
  const int q0 = p.query_start_loc[s], ql = p.query_start_loc[s + 1] - q0, L = p.seq_lens[s];
  const int nblk = decode_blocks(ql, L, G, p.max_seq_len, p.max_blocks_per_seq);
  if (!nblk || ql * G > p.decode_rows || P <= 0) return;
  const int np = (nblk + P - 1) / P;
  const int row0 = kDecodeRows * rg, rows = min(kDecodeRows, ql * G - row0);
  if (np <= 1 || rows <= 0) return;
  constexpr int D4 = D / 4;
  const int64_t unit = (int64_t)s * p.num_kv_heads + kvh;
  const int64_t uslot = (unit * p.max_parts + rg) * kDecodeRows;
  const int64_t step = (int64_t)RG * kDecodeRows;  // the next part's same row
  const float2* pml = reinterpret_cast<const float2*>(p.ws_ml);
  const float4* po = reinterpret_cast<const float4*>(p.ws_o);
  __nv_bfloat16* out = (__nv_bfloat16*)p.out;
  // lane t handles (row, 4 dims) elements t, t + 32, ...; per element the max
  // over the parts, then the weighted sums, the parts' loads issued together
  for (int e = lane; e < rows * D4; e += 32) {
    const int i = e / D4, d4 = e % D4;
    float M = -INFINITY;
    for (int q = 0; q < np; ++q) M = fmaxf(M, __ldcg(pml + uslot + q * step + i).x);
    const float base = (M == -INFINITY) ? 0.f : M;
    float Ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int q = 0; q < np; ++q) {
      const int64_t sl = uslot + q * step + i;
      const float2 ml = __ldcg(pml + sl);
      const float f = ex2(ml.x - base);
      const float4 v = __ldcg(po + sl * D4 + d4);
      Ls += ml.y * f;
      acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    const int gi = row0 + i;
    const int64_t tok = q0 + gi / G, head = (int64_t)kvh * G + gi % G;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(out + (tok * p.num_q_heads + head) * D + 4 * d4) = pk;
  }
}

template <int D, int kMaxRows>
int max_ctas_one() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  using LY = DecodeLayout<D, kMaxRows>;
  auto kernel = decode_persistent_kernel<D, kMaxRows, false, false>;
  static std::atomic<int> smem_done[64];
  int per_sm = 0;
  if (raise_smem_limit(kernel, LY::total, smem_done) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, (LY::kWarps + 1) * 32,
                                                    LY::total) != cudaSuccess ||
      per_sm <= 0)
    per_sm = 1;
  n = per_sm * device_sm_count();
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

int max_ctas(int head_dim, int max_rows) {
  if (head_dim == 64)
    return max_rows <= 4 ? max_ctas_one<64, 4>() : max_rows <= 8 ? max_ctas_one<64, 8>()
                                                                 : max_ctas_one<64, 16>();
  return max_rows <= 4 ? max_ctas_one<128, 4>() : max_rows <= 8 ? max_ctas_one<128, 8>()
                                                                : max_ctas_one<128, 16>();
}

}  // namespace

cudaError_t launch_decode(const AttnParams& p, int head_dim, const int32_t* seq_lens_host,
                          const int32_t* query_start_loc_host, cudaStream_t stream,
                          int max_ctas_allowed) {
  if (p.num_seqs == 0) return cudaSuccess;
  const int max_rows = max(1, min(p.decode_rows, kDecodeRows));  // rows of one unit at most
  const int full = max_ctas(head_dim, max_rows);
  const int ctas = max(1, min(full, max_ctas_allowed));
  static thread_local DecodeWork work;  // 30 KB: kept off the stack
  int grid = ctas;
  if (seq_lens_host && query_start_loc_host &&
      host_piece_list(&work, p, seq_lens_host, query_start_loc_host, ctas, head_dim)) {
    if (work.count == 0) return cudaSuccess;
    grid = min(ctas, work.count);
    // Dealt on the host when the kernel has every SM to itself and each CTA
    // gets several pieces: the claims' latency then adds up on every CTA.
    // With few pieces per CTA, or SMs shared with a prefill running beside
    // it, the claims' adapting to each SM's actual pace is worth more.
    if (ctas == full && work.count >= kDecodeDealPiecesPerCta * grid) deal_pieces(&work, grid);
  } else {
    // Listed on the device.  When the host's bound on the lengths keeps every
    // unit short and there are at least as many units as CTAs, the units stay
    // whole (the claims balance them), so no partial needs merging and the
    // combine kernel is not launched.
    const long long bound_blocks =
        (min((long long)p.max_seq_len, (long long)p.max_blocks_per_seq * kBlockSize) +
         kBlockSize - 1) / kBlockSize;
    const long long units = (long long)p.num_seqs * p.num_kv_heads * p.row_groups;
    const int whole = bound_blocks <= kDecodeWholeUnitBlocks && units >= ctas;
    work.count = 0;
    work.piece_blocks = 0;
    work.from_ws = 1;
    work.split = !whole;
    work.dealt = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1024);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_plan_kernel, p, ctas, head_dim, whole);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e;
  const bool wc = p.slot_mapping != nullptr;
  const bool late = !work.dealt;  // (the write path's pieces are claimed: kLateRows)
  if (head_dim == 64)
    e = !wc   ? launch_rows<64, false, false>(p, work, grid, max_rows, stream)
        : late ? launch_rows<64, true, true>(p, work, grid, max_rows, stream)
               : launch_rows<64, true, false>(p, work, grid, max_rows, stream);
  else
    e = !wc   ? launch_rows<128, false, false>(p, work, grid, max_rows, stream)
        : late ? launch_rows<128, true, true>(p, work, grid, max_rows, stream)
               : launch_rows<128, true, false>(p, work, grid, max_rows, stream);
  if (e != cudaSuccess) return e;
  if (work.split) {
    // the units cut into several pieces: merge their partials
    const long units = (long)p.num_seqs * p.num_kv_heads * p.row_groups;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((units + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = head_dim == 64
            ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<64>, p, work.piece_blocks, work.from_ws)
            : cudaLaunchKernelEx(&cfg, decode_combine_kernel<128>, p, work.piece_blocks,
                                 work.from_ws);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace pa
