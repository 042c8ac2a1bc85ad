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
// running until the list is exhausted.  CTA b starts with piece b and claims
// the next piece from a global counter once all blocks of its current piece
// have been issued (their copies are still in flight while the claim and the
// piece's staging complete), so the SMs that get through their work first
// take the next pieces.  Inside a CTA:
//
//   scheduler warp (the last warp)  claims a piece, copies its block ids and
//       its query rows into a shared-memory piece slot (two slots: piece p
//       lives in slot p % 2), writes the step's new K/V rows of the piece into
//       the cache first when the call asks for it, and publishes the slot.
//   compute warps 0 .. kWarps-1     warp w takes blocks w, w + kWarps, ... of
//       every piece.  It streams them through a private ring of kStages
//       shared-memory stages (K tile + V tile of one (block, kv-head)) with
//       16-byte cp.async copies, up to kStages blocks in flight, and
//       the ring runs on from one piece into the next without draining.  Per
//       16-token block:
//         S[16 rows x 16 keys] = Q . K^T     mma.m16n8k16 (two per 16 dims of D)
//         online softmax (fp32 running max and sum, exp2 with log2(e) folded in)
//         O[16 rows x D]      += P . V       D/8 mma.m16n8k16
//   piece merge  when a warp has computed its last block of a piece it puts
//       its (max, sum, O) in a shared merge slot; the last warp to arrive
//       merges them and stores the piece's result: the output rows when the
//       piece is the whole unit, else an fp32 partial in the workspace.  No
//       CTA ever waits for another, and no merge waits for global memory.
//   combine kernel  (launched right after, as a programmatic dependent) one
//       warp per unit cut into several pieces merges the unit's partials
//       into its output rows.
//
// The dot product's D axis is permuted identically on Q and K so that every
// lane's B-operand words are 8 consecutive bf16 of one key row, and the
// output's D axis is permuted so that every lane's V words are 8 consecutive
// bf16 of one key row (undone when the output is stored).  The 16-byte chunks
// of every tile row are XOR-swizzled on their way into shared memory so that
// these fragment reads hit distinct banks.
//
// Every wait on another warp of the CTA (a piece slot not yet published, the
// merge slot still in use) is bounded by a time limit; one that runs out sets
// the workspace status bit and the CTA winds down instead of hanging.  The
// kernel is launched as a programmatic dependent of whatever precedes it on
// the stream; it reads nothing before griddepcontrol.wait.
#include <math.h>

#include "pa_internal.cuh"
#include "pa_tma.cuh"
#include "pa_wait.cuh"

namespace pa {
namespace {

// compute warps and ring stages per CTA, by head_dim and most query rows per
// unit (shared memory: ring + merge slot + two piece slots, at most 227 KB)
// A warp's loop over its blocks is bound by the latency of its own dependent
// chain (loads, MMAs, shuffles, exponentials), about 2,000 cycles per block,
// so an SM needs about a dozen compute warps to keep up with its share of
// HBM bandwidth; the register budget of a quarter-SM (16K registers) and the
// shared memory of the rings set how many fit.
template <int D, int kMaxRows>
struct DecodeCfg {
  static constexpr int kWarps =
      D == 64 ? (kMaxRows <= 8 ? 11 : 8) : (kMaxRows <= 4 ? 8 : kMaxRows <= 8 ? 7 : 6);
  static constexpr int kStages = D == 64 ? 4 : 3;
};

// What the scheduler publishes about one piece.
struct PieceInfo {
  int tag;  // CTA-local sequence number of the piece in this slot (-1: none yet)
  int end;  // 1: the list is exhausted, no piece in this slot
  int s, kvh, rg, j, nparts;
  int blk_begin, nb;  // the piece's blocks: blk_begin .. blk_begin + nb - 1 of the sequence
  int L, ql, q0;
  int rows, row0;  // this unit's query rows: global rows row0 .. row0 + rows - 1
};

template <int D, int kMaxRows>
struct DecodeLayout {
  static constexpr int kWarps = DecodeCfg<D, kMaxRows>::kWarps;
  static constexpr int kStages = DecodeCfg<D, kMaxRows>::kStages;
  static constexpr int kTileBytes = kBlockSize * D * 2;  // one (block, kv-head) tile
  static constexpr int kStageBytes = 2 * kTileBytes;     // K tile + V tile
  static constexpr int ring_off = 0;  // 1024-byte aligned (128-byte swizzle atoms)
  static constexpr int ring_bytes = kWarps * kStages * kStageBytes;
  // merge slot: per compute warp its rows' max, sum and unnormalised O
  static constexpr int mm_off = ring_off + ring_bytes;                // [kWarps][kMaxRows]
  static constexpr int ml_off = mm_off + kWarps * kMaxRows * 4;       // [kWarps][kMaxRows]
  static constexpr int mo_off = ml_off + kWarps * kMaxRows * 4;       // [kWarps][kMaxRows][D]
  static constexpr int merge_end = mo_off + kWarps * kMaxRows * D * 4;
  // two piece slots: info, block ids, query rows
  static constexpr int kInfoBytes = 64;
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

// Byte offset of 16-byte chunk c of row `row` in a tile that TMA loaded as
// 16 x 64 boxes with 128-byte swizzle: box (64-wide slice of D) c / 8 at
// 2048 bytes per box, rows of 128 bytes, chunk c % 8 XOR row % 8.
__device__ __forceinline__ uint32_t swz128(int row, int c) {
  return (uint32_t)((c >> 3) * 2048 + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}
// 16-byte chunk of a key row (and of a query row) that lane q4 holds for the
// jp-th pair of Q.K^T MMAs: the dot product's D axis is permuted so that the
// eight lanes of one shared-memory phase (two rows, four q4) read eight
// distinct banks after the swizzle (rows r and r+1 differ in row % 8 bit 0).
__device__ __forceinline__ int k_chunk(int q4, int jp) { return 8 * (jp >> 1) + 2 * q4 + (jp & 1); }

// Output column c (0..7) of n-tile nt sits at dimension 64*(nt/8) + 8*c + nt%8,
// so a lane owning columns 2*q4, 2*q4+1 of every n-tile owns, per 64-wide
// half of D, the 16 consecutive dimensions 16*q4 .. 16*q4+15.
__device__ __forceinline__ int out_dim(int nt, int c) { return 64 * (nt / 8) + 8 * c + (nt % 8); }

// Shared control words of a CTA.
struct DecodeCtl {
  int merged;     // CTA-local sequence number of the last piece merged (-1: none)
  int count;      // compute warps that have put their part of the current piece in the merge slot
  int abort;      // set by a bounded wait that ran out: every role winds down
  int passed[2];  // compute warps whose issue cursor has left the piece in each slot
};

// One piece of the list (see DecodeWork): x = sequence, y = ql << 24 | rg << 22
// | kvh << 12 | part, z = seq_len, w = query_start_loc of the sequence.
__device__ __forceinline__ int4 load_piece(const AttnParams& p, const DecodeWork& work, int g) {
  return work.from_ws ? p.ws_pieces[g] : work.items[g];
}

template <int D, int kMaxRows, bool kWriteCache>
__global__ void __launch_bounds__((DecodeCfg<D, kMaxRows>::kWarps + 1) * 32, 1)
decode_persistent_kernel(const AttnParams p, const __grid_constant__ DecodeWork work,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
  using LY = DecodeLayout<D, kMaxRows>;
  constexpr int kWarps = LY::kWarps;
  constexpr int kStages = LY::kStages;
  constexpr bool kRows16 = kMaxRows > 8;
  constexpr int NJ = D / 32;  // 16-byte K chunks per key row a lane reads
  constexpr int NV = D / 64;  // 16-byte V chunks per key row a lane reads
  constexpr int NT = D / 8;   // n-tiles of the P.V product
  constexpr int NC = D / 16;  // k-chunks of the Q.K^T product
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
    for (int i = 0; i < kWarps * kStages; ++i) mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  // Launched as a programmatic dependent: nothing the preceding kernel may
  // write is read before this wait; the next kernel may then be launched (it
  // waits for this grid in the same way).
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int G = p.group;
  const int num_pieces = work.from_ws ? p.ws_header[kWsPieceCount] : work.count;
  const int P = work.from_ws ? p.ws_header[kWsPieceBlocks] : work.piece_blocks;

  if (warp == kWarps) {
    // =============================== scheduler ===============================
    for (int pc = 0;; ++pc) {
      // the next piece is claimed only once every block of the current one
      // has been issued (every compute warp's issue cursor has left it; the
      // copies then keep the warps busy for a while), so that the list's
      // largest-first order goes to the SMs that are free
      if (pc >= 1 &&
          !spin_until([&] { return ld_acquire(&ctl.passed[(pc - 1) & 1]) >= kWarps; }, vabort,
                      status))
        break;
      // slot pc % 2 is free once piece pc - 2 has been merged
      if (pc >= 2 &&
          !spin_until([&] { return ld_acquire(&ctl.merged) >= pc - 2; }, vabort, status))
        break;
      int g = blockIdx.x;
      if (pc > 0) {
        if (lane == 0) g = gridDim.x + atomicAdd(p.ws_header + kWsClaim, 1);
        g = __shfl_sync(0xffffffffu, g, 0);
      }
      PieceInfo* inf = slot_info(pc);
      if (g >= num_pieces) {
        if (lane == 0) {
          inf->end = 1;
          st_release(&inf->tag, pc);
        }
        break;
      }
      const int4 it = load_piece(p, work, g);
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
      if constexpr (kWriteCache) {
        // This step's new tokens of the sequence that fall in the piece's key
        // range go into their cache slots first (as pa_reshape_and_cache
        // would); the compute warps read them only after the publication
        // below.  With several 16-row groups, every row group's piece of the
        // same (sequence, kv-head, blocks) stores the same bytes to the same
        // slots, possibly while another CTA reads them: identical concurrent
        // stores, so every read sees the new row.  No other piece reads
        // these slots.
        const int lo = max(L - ql, blk_begin * kBlockSize);
        const int hi = min(L, (blk_begin + nb) * kBlockSize);
        if (hi > lo) {
          const int n = (hi - lo) * kChunks;
          const int64_t num_slots = (int64_t)p.num_blocks * kBlockSize;
          const uint4* kn = (const uint4*)p.k_new;
          const uint4* vn = (const uint4*)p.v_new;
          uint4* kcw = (uint4*)const_cast<void*>(p.k_cache);
          uint4* vcw = (uint4*)const_cast<void*>(p.v_cache);
          for (int i = lane; i < 2 * n; i += 32) {
            const bool is_v = i >= n;
            const int ii = is_v ? i - n : i;
            const int r = ii / kChunks, c = ii % kChunks;
            const int tok = q0 + (lo - (L - ql)) + r;
            const int64_t slot = p.slot_mapping[tok];
            if (slot < 0 || slot >= num_slots) continue;  // padding / out-of-pool slot
            const int64_t dst =
                ((slot / kBlockSize * p.num_kv_heads + kvh) * kBlockSize + slot % kBlockSize) *
                    kChunks + c;
            const int64_t src = ((int64_t)tok * p.num_kv_heads + kvh) * kChunks + c;
            if (is_v) vcw[dst] = vn[src];
            else kcw[dst] = kn[src];
          }
          // the compute warps read these rows with TMA (the async proxy)
          __threadfence();
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
      }
      if (lane == 0) {
        ctl.passed[pc & 1] = 0;
        inf->end = 0;
        inf->s = s; inf->kvh = kvh; inf->rg = rg; inf->j = j; inf->nparts = nparts;
        inf->blk_begin = blk_begin; inf->nb = nb;
        inf->L = L; inf->ql = ql; inf->q0 = q0;
        inf->rows = rows; inf->row0 = row0;
      }
      __syncwarp();
      if (lane == 0) st_release(&inf->tag, pc);
    }
    // the last CTA to finish claiming resets the claim counter for the next call
    if (lane == 0) {
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

  // the piece in slot pc, once published (nullptr before); the tag is read
  // (with acquire order) only until the warp has seen the piece published
  int seen = -1;  // the latest piece this warp has seen published
  auto published = [&](int pc) -> const PieceInfo* {
    const PieceInfo* inf = slot_info(pc);
    if (pc <= seen) return inf;
    if (ld_acquire(&inf->tag) != pc) return nullptr;
    seen = pc;
    return inf;
  };

  int ip = 0, ii = warp;  // issue cursor: next candidate (piece, block of the piece)
  bool issue_done = false;
  int n_issued = 0, n_comp = 0;
  uint32_t bad = 0;  // bit (stage): that stage's block id was outside the pool

  // Issue the copies of this warp's next block; false when there is none yet
  // (the next piece is not published and `block` is false) or none at all.
  auto try_issue = [&](bool block) -> bool {
    const PieceInfo* inf;
    while (true) {
      inf = published(ip);
      if (!inf) {
        if (!block) return false;
        if (!spin_until([&] { return published(ip) != nullptr; }, vabort, status)) {
          issue_done = true;
          return false;
        }
        inf = published(ip);
      }
      if (inf->end) {
        issue_done = true;
        return false;
      }
      if (ii < inf->nb) break;
      if (lane == 0) atomicAdd(&ctl.passed[ip & 1], 1);  // this warp leaves piece ip
      ++ip;
      ii = warp;
    }
    const int st = n_issued % kStages;
    const int id = slot_ids(ip)[ii];
    // a block id outside the pool is never dereferenced: the box is read from
    // past the tensor's extent (zeros) and its keys are masked
    const bool id_ok = id >= 0 && id < p.num_blocks;
    if (id_ok) bad &= ~(1u << st);
    else bad |= 1u << st;
    const int row_bh = id_ok ? id * p.num_kv_heads + inf->kvh : oob_bh;
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
    if (lane == 0) {
      my_meta[2 * st] = ip;
      my_meta[2 * st + 1] = ii;
    }
    ++n_issued;
    ii += kWarps;
    return true;
  };

  // per-piece state of this warp
  int cur = -1;  // piece being accumulated
  uint32_t qa[NC][2], qb[NC][2];
  float o[NT][4];
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  int lim_a = 0, lim_b = 0, first_masked = 0;

  // The warp's part of piece pc is done: its (max, sum, O) go to the merge
  // slot; the last warp to arrive merges and stores the piece's result.
  auto flush = [&](int pc, const PieceInfo* inf) -> bool {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    if (kRows16) {
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    }
    // the merge slot holds one piece at a time: the previous one must be merged
    if (!spin_until([&] { return ld_acquire(&ctl.merged) >= pc - 1; }, vabort, status))
      return false;
    if (q4 == 0) {
      if (r < kMaxRows) { msl_m[warp * kMaxRows + r] = m_a; msl_l[warp * kMaxRows + r] = l_a; }
      if (kRows16 && r + 8 < kMaxRows) {
        msl_m[warp * kMaxRows + r + 8] = m_b;
        msl_l[warp * kMaxRows + r + 8] = l_b;
      }
    }
    float* mo = msl_o + warp * kMaxRows * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int d = out_dim(nt, 2 * q4 + c);
        if (r < kMaxRows) mo[r * D + d] = o[nt][c];
        if (kRows16 && r + 8 < kMaxRows) mo[(r + 8) * D + d] = o[nt][2 + c];
      }
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) last = add_acq_rel(&ctl.count, 1) + 1 == min(kWarps, inf->nb);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return true;
    __syncwarp();  // every lane reads the other warps' parts after lane 0's acquire

    // ---- merge the warps' parts of the piece: shared memory in, global
    // stores out, then the merge slot is free again (no round trip to global
    // memory while the other warps may wait for the slot)
    const int nw = min(kWarps, inf->nb);
    const int rows = inf->rows, row0 = inf->row0, q0 = inf->q0;
    const int kvh = inf->kvh, rg = inf->rg, np = inf->nparts;
    const int unit = inf->s * p.num_kv_heads + kvh;
    __nv_bfloat16* out = (__nv_bfloat16*)p.out;
    constexpr int D4 = D / 4;
    const bool direct = np == 1;
    const int64_t slot0 = ((int64_t)unit * p.max_parts + inf->j * p.row_groups + rg) * kDecodeRows;
    for (int e = lane; e < rows * D4; e += 32) {
      const int i = e / D4, d4 = e % D4;
      // every warp's value loaded first (unrolled over the CTA's warps), then
      // the max and the weighted sums
      float mw[kWarps];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) mw[w] = w < nw ? msl_m[w * kMaxRows + i] : -INFINITY;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mw[w]);
      const float base = (M == -INFINITY) ? 0.f : M;
      float Ls = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (w < nw) {
          const float f = exp2f(mw[w] - base);
          Ls += msl_l[w * kMaxRows + i] * f;
          const float4 v =
              *reinterpret_cast<const float4*>(msl_o + (w * kMaxRows + i) * D + 4 * d4);
          acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
        }
      }
      if (direct) {
        const int gi = row0 + i;
        const int64_t tok = q0 + gi / G, head = (int64_t)kvh * G + gi % G;
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(out + (tok * p.num_q_heads + head) * D + 4 * d4) = pk;
      } else {
        reinterpret_cast<float4*>(p.ws_o)[(slot0 + i) * D4 + d4] = acc;
        if (d4 == 0) reinterpret_cast<float2*>(p.ws_ml)[slot0 + i] = make_float2(M, Ls);
      }
    }
    __syncwarp();  // every lane is done with the merge slot and the piece slot
    if (lane == 0) {
      ctl.count = 0;
      st_release(&ctl.merged, pc);
    }
    __syncwarp();
    return true;
  };

  // The loop is software-pipelined by one block: iteration n computes
  // S = Q K^T and P of block n (phase A) and adds P V of block n-1 (phase B),
  // two independent dependency chains; O is then rescaled to block n's
  // running max.  A block whose P.V is still pending keeps its stage.  The
  // warp's last block of a piece finishes at once, before the piece is
  // flushed, so nothing is pending across pieces.
  bool pend = false;
  int pend_st = 0, pend_blk = 0, pend_L = 0;
  bool pend_ok = true;
  uint32_t pp0 = 0u, pp1 = 0u, pp2 = 0u, pp3 = 0u;  // P of the pending block, bf16 pairs
  int n_done = 0;  // blocks whose stage is free again (their P.V is in O)

  auto phase_b = [&]() {  // O += P V of the pending block
    const uint32_t vs = ring + pend_st * LY::kStageBytes + LY::kTileBytes;
    // V words: keys 2q4, 2q4+1, 2q4+8, 2q4+9; 8 dims 64u+8r.. each
    uint4 vw[4][NV];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 2 * q4 + (e & 1) + 8 * (e >> 1);
#pragma unroll
      for (int u = 0; u < NV; ++u) vw[e][u] = lds128(vs + swz128(tok, 8 * u + r));
    }
    // slots of the last block past seq_len (and blocks outside the pool) may
    // hold anything, NaN included: their V words become zeros so that the
    // zero weights cannot turn them into NaN in the P.V product
    if (pend_blk * kBlockSize + kBlockSize > pend_L || !pend_ok) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = pend_blk * kBlockSize + 2 * q4 + (e & 1) + 8 * (e >> 1);
        if (!pend_ok || key >= pend_L) {
#pragma unroll
          for (int u = 0; u < NV; ++u) vw[e][u] = make_uint4(0, 0, 0, 0);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int u = nt / 8, idx = nt % 8;
      const uint32_t sel = (idx & 1) ? 0x7632u : 0x5410u;
      const uint32_t b0 = __byte_perm(word(vw[0][u], idx >> 1), word(vw[1][u], idx >> 1), sel);
      const uint32_t b1 = __byte_perm(word(vw[2][u], idx >> 1), word(vw[3][u], idx >> 1), sel);
      mma_16816(o[nt], pp0, pp1, pp2, pp3, b0, b1);
    }
    pend = false;
    ++n_done;
  };

  while (true) {
    // keep kStages blocks in flight (a pending block's stage included); wait
    // for a piece to be published only when nothing is in flight
    while (!issue_done && n_issued - n_done < kStages) {
      if (!try_issue(n_issued == n_done)) break;
    }
    if (n_issued == n_comp) break;  // the list is exhausted (or the CTA aborted)
    if (!wait_bar(bars + 8 * (warp * kStages + n_comp % kStages), (n_comp / kStages) & 1, vabort,
                  status))
      break;  // the oldest stage's K and V tiles have landed (or the CTA gave up)

    const int st = n_comp % kStages;
    const int pc = my_meta[2 * st], i = my_meta[2 * st + 1];
    const PieceInfo* inf = slot_info(pc);
    const int L = inf->L;
    if (pc != cur) {
      // ---- a new piece: its query rows as the A operand (rows r and r+8), D
      // axis permuted as the K chunks; fresh running max, sum and O
      cur = pc;
      const uint32_t qs = slot_q(pc);
#pragma unroll
      for (int jp = 0; jp < NJ; ++jp) {
        uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
        const int cc = k_chunk(q4, jp);
        if (r < kMaxRows) xa = lds128(qs + (r * kChunks + cc) * 16);
        if (kRows16 && r + 8 < kMaxRows) xb = lds128(qs + ((r + 8) * kChunks + cc) * 16);
        qa[2 * jp][0] = xa.x; qa[2 * jp][1] = xa.y; qa[2 * jp + 1][0] = xa.z; qa[2 * jp + 1][1] = xa.w;
        qb[2 * jp][0] = xb.x; qb[2 * jp][1] = xb.y; qb[2 * jp + 1][0] = xb.z; qb[2 * jp + 1][1] = xb.w;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
      m_a = m_b = -INFINITY;
      l_a = l_b = 0.f;
      const int rows = inf->rows, ql = inf->ql;
      // causal limit of rows r and r+8: query j sees keys <= L - ql + j
      lim_a = L - ql + (inf->row0 + min(r, rows - 1)) / G;
      lim_b = L - ql + (inf->row0 + min(r + 8, rows - 1)) / G;
      first_masked = L - ql + 1;  // keys at or beyond this may be masked for some row
    }

    const int blk = inf->blk_begin + i;
    const bool blk_ok = !((bad >> st) & 1u);
    const uint32_t ks = ring + st * LY::kStageBytes;

    // ---- phase A: S = Q K^T (two 8-key halves of the block), each half
    // summed in two accumulators (even and odd k-chunks) so the MMA chains
    // are short
    float sc[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float acc2[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a) acc2[a][0] = acc2[a][1] = acc2[a][2] = acc2[a][3] = 0.f;
      const int row = 8 * h + r;
#pragma unroll
      for (int jp = 0; jp < NJ; ++jp) {
        const uint4 kx = lds128(ks + swz128(row, k_chunk(q4, jp)));
        mma_16816(acc2[0], qa[2 * jp][0], kRows16 ? qb[2 * jp][0] : 0u, qa[2 * jp][1],
                  kRows16 ? qb[2 * jp][1] : 0u, kx.x, kx.y);
        mma_16816(acc2[1], qa[2 * jp + 1][0], kRows16 ? qb[2 * jp + 1][0] : 0u,
                  qa[2 * jp + 1][1], kRows16 ? qb[2 * jp + 1][1] : 0u, kx.z, kx.w);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) sc[h][c] = acc2[0][c] + acc2[1][c];
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
    ++n_comp;

    // ---- phase B of the block before (same running max as O so far), then
    // O to this block's running max
    if (pend) phase_b();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      o[nt][0] *= al_a; o[nt][1] *= al_a;
      if (kRows16) { o[nt][2] *= al_b; o[nt][3] *= al_b; }
    }
    pend = true;
    pend_st = st;
    pend_blk = blk;
    pend_L = L;
    pend_ok = blk_ok;
    pp0 = pack_bf16x2(pa[0], pa[1]);
    pp2 = pack_bf16x2(pa[2], pa[3]);
    pp1 = kRows16 ? pack_bf16x2(pb[0], pb[1]) : 0u;
    pp3 = kRows16 ? pack_bf16x2(pb[2], pb[3]) : 0u;
    if (i + kWarps >= inf->nb) {  // this warp's last block of the piece
      phase_b();
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

template <int D, int kMaxRows, bool kWriteCache>
cudaError_t launch_one(const AttnParams& p, const DecodeWork& work, int grid,
                       cudaStream_t stream) {
  using LY = DecodeLayout<D, kMaxRows>;
  CUtensorMap tk, tv;
  if (!make_map(&tk, p.k_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1) ||
      !make_map(&tv, p.v_cache, D, kBlockSize, (uint64_t)p.num_blocks * p.num_kv_heads,
                (uint64_t)D * 2, (uint64_t)kBlockSize * D * 2, kBlockSize, 1))
    return cudaErrorInvalidValue;
  auto kernel = decode_persistent_kernel<D, kMaxRows, kWriteCache>;
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

template <int D, bool kWriteCache>
cudaError_t launch_rows(const AttnParams& p, const DecodeWork& work, int grid, int max_rows,
                        cudaStream_t stream) {
  if (max_rows <= 4) return launch_one<D, 4, kWriteCache>(p, work, grid, stream);
  if (max_rows <= 8) return launch_one<D, 8, kWriteCache>(p, work, grid, stream);
  return launch_one<D, 16, kWriteCache>(p, work, grid, stream);
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
decode_plan_kernel(const AttnParams p, int ctas, int head_dim) {
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
    sh_P = choose_piece_blocks((long long)sh_total, sh_max_nblk, ctas,
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
  return true;
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
      const float f = exp2f(ml.x - base);
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
  auto kernel = decode_persistent_kernel<D, kMaxRows, false>;
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
  const int ctas = max(1, min(max_ctas(head_dim, max_rows), max_ctas_allowed));
  static thread_local DecodeWork work;  // 16 KB: kept off the stack
  int grid = ctas;
  if (seq_lens_host && query_start_loc_host &&
      host_piece_list(&work, p, seq_lens_host, query_start_loc_host, ctas, head_dim)) {
    if (work.count == 0) return cudaSuccess;
    grid = min(ctas, work.count);
  } else {
    work.count = 0;
    work.piece_blocks = 0;
    work.from_ws = 1;
    work.split = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1024);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_plan_kernel, p, ctas, head_dim);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e;
  const bool wc = p.slot_mapping != nullptr;
  if (head_dim == 64)
    e = wc ? launch_rows<64, true>(p, work, grid, max_rows, stream)
           : launch_rows<64, false>(p, work, grid, max_rows, stream);
  else
    e = wc ? launch_rows<128, true>(p, work, grid, max_rows, stream)
           : launch_rows<128, false>(p, work, grid, max_rows, stream);
  if (e != cudaSuccess) return e;
  if (work.from_ws || work.split) {
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
