// attn_mma_kernel.cu -- pooled hybrid-head decode attention of one launch
// (two, four or eight consecutive layers), bf16 inputs, tensor cores.
//
// Computes, for every segment of the launch's work pool (lyc_plan.h):
//   retrieval rows, page "LycheeDecode ..." (paper-graph-ui summary),
//   section 3.4 Eq. (1): o = softmax(q K^T / sqrt(d)) V over all n cached rows,
//   sparse rows, section 3.4 Eq. (3): the same over the rows of the set they
//   inherit,
// plus the selection key of every cached row for the sets refreshed at its
// layer (Eq. 2 then runs in topk_kernel.cu).  The pieces of a segment cut
// over several CTAs are merged with log-sum-exp (Appendix C, Algorithm 2
// steps 5-6) by the epilogue warps of the next launch, so no CTA waits for
// another's partials.
//
// Design (B200 / sm_100a):
//   * decode attention reads every K/V byte once and does 2-8 flop per byte:
//     HBM bound.  A CUDA-core version of this loop was issue bound (IPC 0.2,
//     DRAM 12% busy in ncu), so both contractions run as bf16 mma with fp32
//     accumulation, transposed so that the up-to-8 query heads of a KV group
//     are the N=8 side and nothing is padded: S^T = K Q^T (M = 16 keys) and
//     O^T = V^T P^T (M = 16 output columns); P^T's fragments come from S^T's
//     by an 8x8 movmatrix transpose;
//   * a STAGES-deep ring of 64-row K/V tiles in shared memory, 128-byte rows
//     with the 128B XOR swizzle so that ldmatrix reads are conflict-free.
//     Dense (contiguous) tiles arrive by TMA tensor copies from a 5-D tensor
//     map of the whole cache (rows past n come back as zeros).  Gathered
//     (sparse) rows arrive by 16-byte cp.async issued by NP producer warps: a
//     gather issues from many warps or not at all (about 0.9 TB/s per issuing
//     warp per SM measured on B200), and the zero-fill form covers the
//     ragged tail.  The gather's indices come ahead in a small ring by bulk copy;
//   * NC consumer warps take whole tiles in turn (each stage of the ring
//     belongs to one of them), keep an online softmax per
//     query head in log2 units (p rounded to bf16 before both P.V and the row
//     sum, so the weights stay normalised), and merge their states at the
//     end of each piece.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "lyc_device.cuh"
#include "lyc_plan.h"

namespace lyc {

typedef uint16_t bf16_t;  // bf16 bit pattern

template <int D, int NC, int NP, int STAGES, bool GT>
struct MmaCfg {
  // warps: NC consumers, one epilogue warp, one scheduler warp, NP producers
  static constexpr int kThreads = (NC + 2 + NP) * 32;
  static constexpr int kProducerThreads = NP * 32;
  static constexpr int kScheduler = (NC + 1) * 32;      // thread index of its warp
  static constexpr int kFirstProducer = (NC + 2) * 32;  // thread index
  // arrivals that complete a full barrier: with row gathers by TMA the one
  // leader thread arms every tile; otherwise every producer thread arrives
  static constexpr int kFullCount = GT ? 1 : NP * 32;
  static constexpr int HALVES = D / 64;                    // 128-byte column blocks per row
  static constexpr int BLOCKB = kTileRows * 128;           // one swizzled 64 x 128 B block
  static constexpr int TILEB = HALVES * BLOCKB;            // K (or V) tile bytes
  static constexpr int IR = 16;                            // index ring slots
  static_assert(kTileRows % (2 * NP) == 0, "rows per producer warp");
  // Tile t sits in stage t % STAGES and is consumed by warp t % NC.  With
  // STAGES a multiple of NC every stage belongs to one consumer warp, which
  // takes that stage's tiles in order; so when it waits for tile t, tile
  // t - STAGES (the stage's previous phase) is already consumed and the
  // parity wait cannot match a phase that has not started.
  static_assert(STAGES % NC == 0, "each stage must belong to one consumer warp");
  static_assert(NC <= kMaxConsumerWarps, "piece-state ring sized for kMaxConsumerWarps");
  // warps that read the pool ring (all but the scheduler, which writes it)
  static constexpr int kRingReaders = NC + 1 + NP;
  // shared memory (bytes from a 1024-aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * TILEB;
  static constexpr int OFF_IDX = OFF_V + STAGES * TILEB;
  static constexpr int OFF_BAR = OFF_IDX + IR * kTileRows * 4;
  // barriers: full[STAGES], empty[STAGES], idx[IR], slot_full[PS], slot_free[PS],
  // unit_full[R], unit_empty[R], idx_free[IR]
  static constexpr int BAR_UNIT = 2 * STAGES + IR + 2 * kPartSlots;
  static constexpr int BAR_IDXFREE = BAR_UNIT + 2 * kPoolRing;
  // prev_ok: the epilogue warp has seen the previous launch complete (from
  // then on this launch may write its partial states)
  static constexpr int BAR_PREVOK = BAR_IDXFREE + IR;
  static constexpr int OFF_FLAGS = OFF_BAR + (BAR_PREVOK + 1) * 8;
  static constexpr int OFF_RING = OFF_FLAGS + 16;  // kPoolRing pool pieces
  static constexpr int SMEM = OFF_RING + kPoolRing * 16 + 1024;  // + alignment slack
};

// Piece i of the CTA, for every warp but the scheduler: its own pieces
// first, then the pool pieces the scheduler took, from the ring (false at the
// end of both).  Each warp calls it for i = 0, 1, ... in order.
template <class C>
// pbeg, pend: the CTA's range in the piece list (read only when needed, so
// that a CTA whose first piece is in the launch parameters does not wait for
// that read before its first piece).
__device__ __forceinline__ bool cta_piece(const AttnParams& p, unsigned char* smem, int pbeg, int pend,
                                          int i, int lane, Piece* out, const FirstPiece* fp = nullptr) {
  if (i == 0 && fp && fp->pc.seg >= 0) {  // from the launch parameters
    *out = fp->pc;
    return true;
  }
  const int nhome = pend - pbeg;
  if (i < nhome) {
    *out = p.pieces[pbeg + i];
    return true;
  }
  if (p.pool_n <= 0) return false;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* unit_full = bars + C::BAR_UNIT;
  uint64_t* unit_empty = unit_full + kPoolRing;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const int k = i - nhome;
  const int r = k % kPoolRing;
  if (!mbar_wait(&unit_full[r], (k / kPoolRing) & 1, abort_flag, p.status)) return false;
  const Piece pc = reinterpret_cast<const Piece*>(smem + C::OFF_RING)[r];
  __syncwarp();
  if (lane == 0) mbar_arrive(&unit_empty[r]);
  *out = pc;
  return pc.seg >= 0;
}

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate
__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// two floats -> bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// 8x8 bf16 matrix transpose across the warp (fragment layout in and out)
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, int c4, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// four rows (coordinates y0..y3 of a 2-D tensor map with a one-row box) at
// column x, into 4 consecutive box rows at dst; rows outside the map read as zeros
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int x, int4 y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y.x), "r"(y.y), "r"(y.z), "r"(y.w),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// byte offset of 16-byte chunk `ch` (0 .. D/8-1) of tile row `r`
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * (kTileRows * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

}  // namespace lyc


namespace lyc {

// ---------------------------------------------------------------- scheduler
// One thread walks the CTA's pieces ahead of the producers: its own pieces,
// then pool units it takes by the launch's atomic cursor, each published as a
// ring entry, ending with an entry of segment -1.  For every gathered tile it
// copies the tile's slice of the index list into the index ring (a bulk
// copy) once the ring slot is free, i.e. once the tile IR places earlier has
// been consumed; a pool unit is taken at that same point for its first tile,
// so every CTA holds about IR tiles of work ahead, however early it started.
// Before the first tile of a set written by a selection of this step it
// waits for that selection's ready flag.  Its waits hold up no copy issue.
template <int D, int NC, int NP, int STAGES, bool GT>
__device__ __forceinline__ void mma_scheduler(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                              int pend) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  const AttnParams& p = P.p;
  int32_t* idxring = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* idxbar = bars + 2 * STAGES;
  uint64_t* unit_full = bars + C::BAR_UNIT;
  uint64_t* unit_empty = unit_full + kPoolRing;
  uint64_t* idx_free = bars + C::BAR_IDXFREE;
  Piece* ring = reinterpret_cast<Piece*>(smem + C::OFF_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const int nhome = pend - pbeg;
  int32_t* cursor = p.pool_n > 0
                        ? p.pool_cursors + static_cast<int64_t>(*p.epoch & 1u) * p.pool_stride + p.layer
                        : nullptr;
  // Slot of tile tt in the index ring is free once tile tt - IR is consumed.
  // The scheduler waits on every tile in order, dense ones included: a
  // parity wait tells phases apart only when the waiter is at most one phase
  // ahead of the barrier.
  auto slot_free = [&](int tt) {
    return tt < C::IR || mbar_wait(&idx_free[tt % C::IR], ((tt / C::IR) - 1) & 1, abort_flag, p.status);
  };
  const uint32_t* acquired = nullptr;  // the last ready flag waited on
  bool waited = false;                 // the previous launch has completed
  int t = 0;                           // CTA-wide tile sequence number
  // the pool unit taken last: segment, rows, ordinal (none: row == end)
  int useg = 0, urow = 0, uend = 0, uord = 0;
  // the current segment's fields
  int cseg = -1, ckind = 0, cdep = 0;
  const uint32_t* cready = nullptr;
  const int32_t* cidx = nullptr;
  bool cpad = false;
  auto seg_fields = [&](int seg) {  // the segment's fields, kept across its consecutive pieces
    if (seg == cseg) return;
    const Segment& sg = p.segs[seg];
    cseg = seg;
    ckind = sg.kind;
    cready = sg.ready;
    cdep = sg.dep;
    cidx = sg.idx;
    cpad = sg.pad_ok != 0;
  };
  // A set that a selection of this step writes is read once that selection
  // has raised its ready flag (the selection may still be running).
  // Otherwise a set the previous launch writes is read once that launch has
  // completed.  The bulk copies read the set through the async proxy, hence
  // the proxy fence after the acquire.
  auto wait_set = [&]() {
    if (cready) {
      if (cready != acquired) {
        wait_flag(cready, *p.epoch + 1u, abort_flag, p.status);
        fence_proxy_async_global();
        acquired = cready;
      }
    } else if (cdep && !waited) {
      pdl_wait();
      waited = true;
    }
  };
  for (int i = 0;; ++i) {
    Piece pc;
    if (i < nhome) {
      pc = p.pieces[pbeg + i];
    } else {
      if (!cursor) break;
      const int k = i - nhome;
      const int r = k % kPoolRing;
      if (!slot_free(t)) break;
      if (k >= kPoolRing && !mbar_wait(&unit_empty[r], ((k / kPoolRing) - 1) & 1, abort_flag, p.status))
        break;
      // the next unit, or the end (seg -1)
      if (urow >= uend) {
        const int u = atomicAdd(cursor, 1);
        if (u < p.pool_n) {
          const Piece un = p.pool_units[u];
          useg = un.seg;
          urow = un.r0;
          uend = un.r1;
          uord = un.ordinal;
        } else {
          useg = -1;
        }
      }
      pc.seg = -1;
      pc.r0 = pc.r1 = pc.ordinal = 0;
      if (useg >= 0) {
        pc.seg = useg;
        pc.r0 = urow;
        pc.r1 = uend;
        pc.ordinal = uord;
        urow = uend;
        seg_fields(pc.seg);
        // A set of a rule that may leave it shorter than its capacity is
        // ascending with -1 padding at its end: the unit keeps its tiles up
        // to the first one that starts with padding (at least one tile, so
        // that the piece still writes its partial state: an empty softmax,
        // which the cross-piece combine skips).  The tiles dropped here
        // would have fetched no bytes, but they would still take their
        // turn in the pipeline.
        if (ckind == kSparse && cpad) {
          wait_set();
          constexpr int UT = kPoolTiles > kPoolTilesDep ? kPoolTiles : kPoolTilesDep;
          int32_t first[UT];
          const int nt = (pc.r1 - pc.r0 + kTileRows - 1) / kTileRows;
#pragma unroll
          for (int j = 0; j < UT; ++j) first[j] = j < nt ? __ldcg(cidx + pc.r0 + j * kTileRows) : -1;
          int keep = 1;
#pragma unroll
          for (int j = 1; j < UT; ++j)
            if (keep == j && first[j] >= 0) keep = j + 1;
          if (first[0] < 0) pc.r1 = pc.r0 + 1;  // one padding row
          else pc.r1 = min(pc.r1, pc.r0 + keep * kTileRows);
        }
      }
      ring[r] = pc;
      mbar_arrive(&unit_full[r]);  // release: the entry above
      if (pc.seg < 0) break;
    }
    seg_fields(pc.seg);
    if (ckind != kSparse) {
      for (int r0 = pc.r0; r0 < pc.r1; r0 += kTileRows, ++t)
        if (!slot_free(t)) return;
      continue;
    }
    wait_set();
    for (int r0 = pc.r0; r0 < pc.r1; r0 += kTileRows, ++t) {
      const int slot = t % C::IR;
      if (!slot_free(t)) return;
      const int nrows = min(kTileRows, pc.r1 - r0);
      const uint32_t bytes = static_cast<uint32_t>(((nrows * 4) + 15) & ~15);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&idxbar[slot], bytes);
      bulk_g2s(idxring + slot * kTileRows, cidx + r0, bytes, &idxbar[slot]);
    }
  }
}

// ---------------------------------------------------------------- producers
// NP warps walk the CTA's tiles together.  Dense tile: one thread issues the
// TMA copies, everyone arrives.  Gathered tile: warp pw copies rows
// [pw*64/NP, (pw+1)*64/NP) with cp.async and every lane arrives when its own
// copies have landed.
template <int D, int NC, int NP, int STAGES, bool GT, bool PG>
__device__ __forceinline__ void mma_producers(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                              int pend) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  const AttnParams& p = P.p;
  const int ptid = threadIdx.x - C::kFirstProducer;  // 0 .. NP*32-1
  const int pw = ptid >> 5;
  const int lane = ptid & 31;
  unsigned char* Ks = smem + C::OFF_K;
  unsigned char* Vs = smem + C::OFF_V;
  int32_t* idxring = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* idxbar = bars + 2 * STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const uint64_t pol = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_normal();  // gathered rows may be read again
  const bool leader = ptid == 0;

  constexpr int CH = D / 8;                  // 16-byte chunks per row
  constexpr int ROWS_W = kTileRows / NP;     // rows per producer warp
  uint32_t idx_phase = 0;
  int t = 0;
  // the current segment's constants in registers (the copies below are asm
  // with a memory clobber: fields read through the segment would be reloaded
  // after each), kept while consecutive pieces stay in one segment
  int cseg = -1;
  bool dense = false;
  int64_t s_token = 0, s_page = 0;
  const bf16_t* kb = nullptr;
  const bf16_t* vb = nullptr;
  const int32_t* bt = nullptr;
  int sl = 0, sb = 0, sgg = 0, nvalid = 0, page_rows = 0;
  int32_t pad_ok = 0, row_base = 0;
  const FirstPiece* fp = static_cast<int>(blockIdx.x) < P.nfirst ? &P.first[blockIdx.x] : nullptr;
  for (int pi = 0;; ++pi) {
    Piece pc;
    if (!cta_piece<C>(p, smem, pbeg, pend, pi, lane, &pc, fp)) break;
    if (pi == 0 && fp && fp->pc.seg >= 0) {
      // a dense piece of the launch's first layer: the tile copies need no more
      // (the next piece reads its segment's fields)
      dense = true;
      sgg = fp->g;
      sb = fp->b;
      sl = p.layer;
      cseg = -1;
    } else if (pc.seg != cseg) {
      const Segment& sg = p.segs[pc.seg];
      cseg = pc.seg;
      dense = sg.kind == kDense;
      s_token = sg.s_token;
      kb = static_cast<const bf16_t*>(sg.k);
      vb = static_cast<const bf16_t*>(sg.v);
      sl = sg.l;
      sb = sg.b;
      sgg = sg.g;
      nvalid = sg.nvalid;
      pad_ok = sg.pad_ok;
      bt = sg.bt;
      page_rows = sg.page_rows;
      s_page = sg.s_page;
      row_base = sg.row_base;
    }
    for (int r0 = pc.r0; r0 < pc.r1; r0 += kTileRows, ++t) {
      const int nrows = min(kTileRows, pc.r1 - r0);
      const int stage = t % STAGES;
      if (t >= STAGES) {
        if (!mbar_wait(&empty[stage], ((t / STAGES) - 1) & 1, abort_flag, p.status)) return;
      }
      unsigned char* kdst = Ks + stage * C::TILEB;
      unsigned char* vdst = Vs + stage * C::TILEB;
      if (dense) {
        // TMA tensor copies; rows past n are filled with zeros by the copy
        if (leader) {
          mbar_arrive_expect_tx(&full[stage], 2u * C::TILEB);
          // contiguous: map (d, row, g, b, l); paged: map (d, g, row in page, page, l),
          // a tile never crosses a page (page_rows is a multiple of 64)
          int c1 = r0, c2 = sgg, c3 = sb;
          if (PG) {
            c1 = sgg;
            c2 = r0 % page_rows;
            c3 = __ldg(&bt[r0 / page_rows]);
          }
#pragma unroll
          for (int h = 0; h < C::HALVES; ++h) {
            tma_load_5d(kdst + h * C::BLOCKB, &P.tmk, h * 64, c1, c2, c3, sl, &full[stage], pol);
            tma_load_5d(vdst + h * C::BLOCKB, &P.tmv, h * 64, c1, c2, c3, sl, &full[stage], pol);
          }
        } else if (!GT) {
          mbar_arrive(&full[stage]);
        }
      } else if (GT) {
        // TMA row gathers: lane j < 16 brings K rows 4j .. 4j+3, lane 16 + j the
        // same V rows, one 128-byte column block per copy.  Rows past the
        // tile's end and out-of-range indices get a coordinate past the map,
        // which reads as zeros (and is reported below, never followed).
        const int slot = t % C::IR;
        if (!mbar_wait(&idxbar[slot], (idx_phase >> slot) & 1u, abort_flag, p.status)) return;
        idx_phase ^= 1u << slot;
        if (leader) mbar_arrive_expect_tx(&full[stage], 2u * C::TILEB);
        const int j = lane & 15;
        const int4 ix = reinterpret_cast<const int4*>(idxring + slot * kTileRows)[j];
        const int xs[4] = {ix.x, ix.y, ix.z, ix.w};
        int ys[4];
        bool bad = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in_tile = 4 * j + e < nrows;
          const bool ok = xs[e] >= 0 && xs[e] < nvalid;
          bad |= in_tile && index_bad(xs[e], nvalid, pad_ok);
          ys[e] = (in_tile && ok) ? row_base + xs[e] : p.gather_rows;
        }
        if (bad) atomicOr(p.status, kStatusBadIndex);
        const bool isv = lane >= 16;
        unsigned char* dst = (isv ? vdst : kdst) + 4 * j * 128;
        const CUtensorMap* map = isv ? &P.tgv : &P.tgk;
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_gather4(dst + h * C::BLOCKB, map, h * 64, make_int4(ys[0], ys[1], ys[2], ys[3]),
                      &full[stage], pol_keep);
      } else {
        const int slot = t % C::IR;
        if (!mbar_wait(&idxbar[slot], (idx_phase >> slot) & 1u, abort_flag, p.status)) return;
        idx_phase ^= 1u << slot;
        const int32_t* ring = idxring + slot * kTileRows;
        if (pw == 0) {  // bounds of the inherited indices (reported, never followed)
          const int32_t ia = (lane < nrows) ? ring[lane] : 0;
          const int32_t ib = (lane + 32 < nrows) ? ring[lane + 32] : 0;
          if (index_bad(ia, nvalid, pad_ok) || index_bad(ib, nvalid, pad_ok))
            atomicOr(p.status, kStatusBadIndex);
        }
        const uint32_t kbase = smem_u32(kdst), vbase = smem_u32(vdst);
        // lane: chunk (lane % CH) of rows pw*ROWS_W + (lane / CH) + (32/CH)*i
        constexpr int RPI = 32 / CH;         // rows per warp instruction
#pragma unroll
        for (int i = 0; i < ROWS_W / RPI; ++i) {
          const int r = pw * ROWS_W + i * RPI + lane / CH;
          const int c = lane % CH;
          const int32_t ix = (r < nrows) ? ring[r] : -1;
          const bool ok = ix >= 0 && ix < nvalid;
          // contiguous rows, or row ix % page_rows of page bt[ix / page_rows]
          int64_t off = 0;
          if (ok) {
            if (PG)
              off = static_cast<int64_t>(__ldg(&bt[ix / page_rows])) * s_page +
                    static_cast<int64_t>(ix % page_rows) * s_token;
            else
              off = static_cast<int64_t>(ix) * s_token;
          }
          cp_async_16(kbase + swz(r, c), kb + off + c * 8, ok ? 16u : 0u);
          cp_async_16(vbase + swz(r, c), vb + off + c * 8, ok ? 16u : 0u);
        }
        cp_async_arrive(&full[stage]);
      }
    }
  }
}

}  // namespace lyc

namespace lyc {

// The ring of piece states this CTA uses (chosen at its start, kept in
// shared memory): the SM's own when CTAs of two launches may run at once (a
// CTA of this kernel has the SM to itself: the shared memory of two does not
// fit), else the block's.
template <class C>
__device__ __forceinline__ int cta_ring(const unsigned char* smem) {
  return *reinterpret_cast<const volatile int*>(smem + C::OFF_FLAGS + 4);
}

// One arrival of `cnt` on the step counter of layer `layer`'s selection keys
// (the counters of a launch's layers are consecutive, from the first
// layer's; release: the caller's warp or CTA barrier orders its threads' key
// stores before it); that layer's selection starts once its counter reaches
// (CTAs with dense pieces of the layer) * NC.
__device__ __forceinline__ void keys_arrive(const AttnParams& p, int layer, uint32_t cnt) {
  red_release_add_u32(p.keys_done + (*p.epoch & 1u) * p.pool_stride + (layer - p.layer), cnt);
}

// A one-tile piece's result from the warp that computed it, for one of the
// lane's two queries (h = 0: query 2c, columns in oa[md][0] and [2]; h = 1:
// query 2c+1, oa[md][1] and [3]); oi = that query's output index, or -1.
// m, l are the warp-wide running maximum (log2 units) and sum.
template <int D>
__device__ __forceinline__ void solo_write(const AttnParams& p, const Segment& sg, const Piece& pc, int oi,
                                           float m, float l, const float (*oa)[4], int h, int g, int c) {
  if (oi < 0) return;
  constexpr int MD = D / 16;
  if (sg.npieces == 1) {
    float* out = (sg.out ? sg.out : p.out) + (static_cast<int64_t>(sg.b) * p.Hq + sg.head[2 * c + h]) * D;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (l <= 0.f && g == 0) atomicOr(p.status, kStatusEmptySoftmax);
#pragma unroll
    for (int md = 0; md < MD; ++md) {
      out[16 * md + g] = oa[md][h] * inv;
      out[16 * md + g + 8] = oa[md][2 + h] * inv;
    }
  } else {
    const int64_t idx = sg.part_base + static_cast<int64_t>(pc.ordinal) * sg.nout + oi;
    float* po = p.part_o + idx * D;
#pragma unroll
    for (int md = 0; md < MD; ++md) {
      po[16 * md + g] = oa[md][h];
      po[16 * md + g + 8] = oa[md][2 + h];
    }
    if (g == 0) p.part_ml[idx] = make_float2(m, l);
  }
}

// ---------------------------------------------------------------- consumers
// Fragment bookkeeping (m16n8k16, g = lane/4, c = lane%4):
//   S^T tile mt (16 keys):  st[mt][0..1] = keys 16mt+g,   queries 2c, 2c+1
//                           st[mt][2..3] = keys 16mt+g+8, queries 2c, 2c+1
//   O^T tile md (16 cols):  oa[md][0..1] = cols 16md+g,   queries 2c, 2c+1
//                           oa[md][2..3] = cols 16md+g+8, queries 2c, 2c+1
// so every lane owns queries q0 = 2c and q1 = 2c+1 in both, and the softmax
// rescale needs no data movement.
template <int D, int NC, int NP, int STAGES, bool GT>
__device__ __forceinline__ void mma_consumers(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                              int pend) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int KSTEPS = D / 16;   // q.K k-steps over d
  constexpr int MD = D / 16;       // O^T m-tiles
  const AttnParams& p = P.p;
  const int tid = threadIdx.x;     // 0 .. NC*32-1
  const int w = tid >> 5;
  const int lane = tid & 31;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int q0 = 2 * c, q1 = 2 * c + 1;
  const uint32_t ksm = smem_u32(smem + C::OFF_K);
  const uint32_t vsm = smem_u32(smem + C::OFF_V);
  const int32_t* idxring = reinterpret_cast<const int32_t*>(smem + C::OFF_IDX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* slot_full = bars + 2 * STAGES + C::IR;
  uint64_t* slot_free = slot_full + kPartSlots;
  uint64_t* idx_free = bars + C::BAR_IDXFREE;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const float sl2 = p.scale_log2;
  const int mi = lane >> 3, r8 = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const int wq = p.wpart_q > 0 ? p.wpart_q : kMaxQ;  // query rows per ring record

  int t = 0;   // CTA-wide tile sequence number
  int mp = 0;  // pieces of more than one tile so far (they take ring slots in turn)
  bool prev_ok = false;  // the previous launch has completed (partials may be written)
  // the current segment's constants and query fragments
  int cseg = -1, nq = 0, nout = 0, b = 0, oi0 = -1, oi1 = -1, nvalid = 0;
  bool dense = false;
  int64_t koff0 = -1, koff1 = -1, key_mean_off = -1;
  float mean_scale = 0.f;
  uint32_t qb[KSTEPS][2];
  const FirstPiece* fp = static_cast<int>(blockIdx.x) < P.nfirst ? &P.first[blockIdx.x] : nullptr;
  // The CTA's own pieces (its dense runs, the only writers of selection keys,
  // in layer order) come first: once past a layer's, this warp's keys of
  // that layer are written.  home_l: the layer of the own pieces so far.
  int home_l = -1;
  auto keys_written = [&](int layer) {
    __syncwarp();
    if (lane == 0) keys_arrive(p, layer, 1u);
    __syncwarp();
  };
  for (int pi = 0;; ++pi) {
    if (home_l >= 0 && pi == pend - pbeg) {
      keys_written(home_l);
      home_l = -1;
    }
    Piece pc;
    if (!cta_piece<C>(p, smem, pbeg, pend, pi, lane, &pc, fp)) break;
    // an own piece of another layer: the keys of the layer before are done
    // (every warp sees every piece, those it leaves to others included)
    if (p.keys_done && ((pi == 0 && fp && fp->pc.seg >= 0) || pi < pend - pbeg)) {
      // (a first piece from the parameters is of the launch's first layer)
      const int sl = (pi == 0 && fp && fp->pc.seg >= 0) ? p.layer : p.segs[pc.seg].l;
      if (home_l >= 0 && sl != home_l) keys_written(home_l);
      home_l = sl;
    }
    const int ntile = (pc.r1 - pc.r0 + kTileRows - 1) / kTileRows;
    // A piece of one tile belongs to the one warp that takes its tile: that
    // warp writes the piece's partial state (or, for a segment of one piece,
    // its outputs) itself, with no ring slot and no epilogue merge.
    const bool solo = ntile == 1;
    if (solo && (t % NC) != w) {
      ++t;
      continue;
    }
    const Segment& sg = p.segs[pc.seg];
    if (pc.seg != cseg) {
      // a new segment: its constants and Q^T as the B operand (this lane
      // holds query g, d = 16kk + 2c (+8)); kept while the warp's pieces stay
      // in the segment (consecutive one-tile pieces of a pool unit)
      cseg = pc.seg;
      nq = sg.nq;
      nout = sg.nout;
      b = sg.b;
      dense = sg.kind == kDense;
      oi0 = oi1 = -1;
      for (int o = 0; o < nout; ++o) {
        if (sg.out_row[o] == q0) oi0 = o;
        if (sg.out_row[o] == q1) oi1 = o;
      }
      koff0 = (q0 < nq) ? sg.key_off[q0] : -1;
      koff1 = (q1 < nq) ? sg.key_off[q1] : -1;
      key_mean_off = sg.key_mean_off;
      mean_scale = p.scale / static_cast<float>(nq);
      nvalid = sg.nvalid;
      const bf16_t* q = static_cast<const bf16_t*>(sg.q ? sg.q : p.q);  // the segment's layer
      const bf16_t* qrow = q + (static_cast<int64_t>(b) * p.Hq + sg.head[g < nq ? g : 0]) * D;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        qb[kk][0] = (g < nq) ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * c) : 0u;
        qb[kk][1] = (g < nq) ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * c) : 0u;
      }
    }
    const bool out0 = oi0 >= 0, out1 = oi1 >= 0;

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float oa[MD][4];
#pragma unroll
    for (int md = 0; md < MD; ++md) oa[md][0] = oa[md][1] = oa[md][2] = oa[md][3] = 0.f;

    for (int u = 0; u < ntile; ++u, ++t) {
      if ((t % NC) != w) continue;
      const int r0 = pc.r0 + u * kTileRows;
      const int nrows = min(kTileRows, pc.r1 - r0);
      const int stage = t % STAGES;
      mbar_wait(&full[stage], (t / STAGES) & 1, abort_flag, p.status);
      // validity of the 64 rows (ragged tail; inherited indices out of range)
      bool va = lane < nrows, vb = lane + 32 < nrows;
      if (!dense) {
        const int32_t* ring = idxring + (t % C::IR) * kTileRows;
        if (va) { const int32_t x = ring[lane]; va = x >= 0 && x < nvalid; }
        if (vb) { const int32_t x = ring[lane + 32]; vb = x >= 0 && x < nvalid; }
      }
      const uint64_t vmask = static_cast<uint64_t>(__ballot_sync(FULL, va)) |
                             (static_cast<uint64_t>(__ballot_sync(FULL, vb)) << 32);
      const uint32_t kt_base = ksm + stage * C::TILEB;
      const uint32_t vt_base = vsm + stage * C::TILEB;

      // ---- S^T = K Q^T: 4 m-tiles of 16 keys x 8 queries
      float st[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) st[mt][0] = st[mt][1] = st[mt][2] = st[mt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t a[4];
          ldsm_x4(a, kt_base + swz(16 * mt + (mi & 1) * 8 + r8, 2 * kk + (mi >> 1)));
          mma_bf16(st[mt], a[0], a[1], a[2], a[3], qb[kk][0], qb[kk][1]);
        }
      }

      // ---- selection keys (dense segments only)
      if (dense && (koff0 >= 0 || koff1 >= 0)) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int key = 16 * mt + g + 8 * h;
            if ((vmask >> key) & 1ull) {
              if (koff0 >= 0) p.keys[koff0 + r0 + key] = st[mt][2 * h] * p.scale;
              if (koff1 >= 0) p.keys[koff1 + r0 + key] = st[mt][2 * h + 1] * p.scale;
            }
          }
        }
      }
      if (dense && key_mean_off >= 0) {
        // queries >= nq hold zero logits, so the sum over all 8 is the sum over nq
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float x = st[mt][2 * h] + st[mt][2 * h + 1];
            x += __shfl_xor_sync(FULL, x, 1);
            x += __shfl_xor_sync(FULL, x, 2);
            const int key = 16 * mt + g + 8 * h;
            if (c == 0 && ((vmask >> key) & 1ull)) p.keys[key_mean_off + r0 + key] = x * mean_scale;
          }
        }
      }

      // ---- online softmax for queries q0, q1 (log2 units)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const bool ok = (vmask >> (16 * mt + g + 8 * h)) & 1ull;
          st[mt][2 * h] = ok ? st[mt][2 * h] * sl2 : -INFINITY;
          st[mt][2 * h + 1] = ok ? st[mt][2 * h + 1] * sl2 : -INFINITY;
          mx0 = fmaxf(mx0, st[mt][2 * h]);
          mx1 = fmaxf(mx1, st[mt][2 * h + 1]);
        }
      }
#pragma unroll
      for (int s = 4; s <= 16; s <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, s));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, s));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const bool live0 = out0 && mn0 != -INFINITY, live1 = out1 && mn1 != -INFINITY;
      const float sc0 = live0 ? exp2f(m0 - mn0) : 1.f;
      const float sc1 = live1 ? exp2f(m1 - mn1) : 1.f;
      if (out0) m0 = mn0;
      if (out1) m1 = mn1;
      uint32_t pb[4][2];  // P^T fragments, per 16-key step: keys +0..7, +8..15
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float pv0 = live0 ? exp2f(st[mt][2 * h] - mn0) : 0.f;
          const float pv1 = live1 ? exp2f(st[mt][2 * h + 1] - mn1) : 0.f;
          const uint32_t pk = pack_bf16(pv0, pv1);  // (key, q0) low, (key, q1) high
          ls0 += __uint_as_float(pk << 16);
          ls1 += __uint_as_float(pk & 0xffff0000u);
          pb[mt][h] = movmatrix_t(pk);  // -> (query g, keys 2c, 2c+1)
        }
      }
      l0 = l0 * sc0 + ls0;
      l1 = l1 * sc1 + ls1;
#pragma unroll
      for (int md = 0; md < MD; ++md) {
        oa[md][0] *= sc0;
        oa[md][1] *= sc1;
        oa[md][2] *= sc0;
        oa[md][3] *= sc1;
      }

      // ---- O^T += V^T P^T: 4 k-steps of 16 keys, MD m-tiles of 16 columns
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
#pragma unroll
        for (int md = 0; md < MD; ++md) {
          uint32_t a[4];
          ldsm_x4_t(a, vt_base + swz(16 * kt + (mi >> 1) * 8 + r8, 2 * md + (mi & 1)));
          mma_bf16(oa[md], a[0], a[1], a[2], a[3], pb[kt][0], pb[kt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[stage]);
        mbar_arrive(&idx_free[t % C::IR]);  // the tile's index slice is no longer read
      }
    }

#pragma unroll
    for (int s2 = 4; s2 <= 16; s2 <<= 1) {
      l0 += __shfl_xor_sync(FULL, l0, s2);
      l1 += __shfl_xor_sync(FULL, l1, s2);
    }
    if (solo) {
      // ---- this warp holds the whole piece: its partial state, or the
      // normalised outputs when the segment is this one piece.  Partial
      // states share their buffer with the launch two launches back, whose
      // merge runs in the previous launch: write them once that launch has
      // completed (seen by the epilogue warp).
      if (sg.npieces > 1 && !prev_ok) {
        mbar_wait(&bars[C::BAR_PREVOK], 0, abort_flag, p.status);
        prev_ok = true;
      }
      solo_write<D>(p, sg, pc, oi0, m0, l0, oa, 0, g, c);
      solo_write<D>(p, sg, pc, oi1, m1, l1, oa, 1, g, c);
      continue;
    }
    // ---- hand this warp's state of the piece to the epilogue warp: slot
    // (multi-tile piece % kPartSlots) of this CTA's ring, rows that produce
    // an output
    {
      const int slot = mp % kPartSlots;
      if (mp >= kPartSlots)
        mbar_wait(&slot_free[slot], ((mp / kPartSlots) - 1) & 1, abort_flag, p.status);
      ++mp;
      const int64_t rec = ((static_cast<int64_t>(cta_ring<C>(smem)) * kPartSlots + slot) * NC + w) * wq;
      if (g == 0) {
        if (out0) p.wpart_ml[rec + q0] = make_float2(m0, l0);
        if (out1) p.wpart_ml[rec + q1] = make_float2(m1, l1);
      }
      float* o0 = p.wpart_o + (rec + q0) * D;
      float* o1 = p.wpart_o + (rec + q1) * D;
#pragma unroll
      for (int md = 0; md < MD; ++md) {
        if (out0) {
          o0[16 * md + g] = oa[md][0];
          o0[16 * md + g + 8] = oa[md][2];
        }
        if (out1) {
          o1[16 * md + g] = oa[md][1];
          o1[16 * md + g + 8] = oa[md][3];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_full[slot]);  // release: the writes above
    }
  }
}

// ---------------------------------------------------------------- epilogue warp
// Two jobs (Appendix C, Algorithm 2, steps 5-6):
//  1. first, the cross-piece combine of the previous attention launch: this
//     CTA takes the (segment, output) tasks t = blockIdx.x, blockIdx.x +
//     gridDim.x, ... and folds each output's piece partials (log-sum-exp)
//     into the output of the segment's layer, once that launch's done counter
//     is complete (its partials are then in place; this launch may start
//     while that one still runs); running the combine here keeps it off the
//     critical path;
//  2. then, per piece of this CTA in order: wait for the NC consumer warps'
//     states, merge them per output, and write the piece's partial (or, for a
//     segment of one piece, the output itself).
// The consumers never wait for this work unless they run kPartSlots pieces
// ahead.  Lane j owns columns 4j .. 4j+3.

// Running log-sum-exp state of one lane (4 columns).
struct LseAcc {
  float M, L;
  float4 o;
};
__device__ __forceinline__ void lse_init(LseAcc& a) {
  a.M = -INFINITY;
  a.L = 0.f;
  a.o = make_float4(0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ void lse_add(LseAcc& a, float2 ml, float4 ov) {
  if (ml.x == -INFINITY) return;
  const float mn = fmaxf(a.M, ml.x);
  const float s = (a.M == -INFINITY) ? 0.f : exp2f(a.M - mn);
  const float f = exp2f(ml.x - mn);
  a.L = a.L * s + f * ml.y;
  a.o.x = a.o.x * s + f * ov.x;
  a.o.y = a.o.y * s + f * ov.y;
  a.o.z = a.o.z * s + f * ov.z;
  a.o.w = a.o.w * s + f * ov.w;
  a.M = mn;
}

// out[b][head of output o] = the normalised state (0 and a status bit if the
// softmax had no valid row)
__device__ __forceinline__ void lse_finish(const LseAcc& a, float* out, const AttnParams& p,
                                           const Segment& sg, int o, int lane, bool col, int D) {
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.L > 0.f) {
    const float inv = 1.f / a.L;
    res = make_float4(a.o.x * inv, a.o.y * inv, a.o.z * inv, a.o.w * inv);
  } else if (lane == 0) {
    atomicOr(p.status, kStatusEmptySoftmax);
  }
  if (col)
    *reinterpret_cast<float4*>(
        &out[(static_cast<int64_t>(sg.b) * p.Hq + sg.head[sg.out_row[o]]) * D + lane * 4]) = res;
}

template <int D, int NC, int NP, int STAGES, bool GT>
__device__ __forceinline__ void mma_epilogue(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                             int pend) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  const AttnParams& p = P.p;
  const int lane = threadIdx.x & 31;
  const bool col = lane * 4 < D;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* slot_full = bars + 2 * STAGES + C::IR;
  uint64_t* slot_free = slot_full + kPartSlots;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const int wq = p.wpart_q > 0 ? p.wpart_q : kMaxQ;  // query rows per ring record

  // ---- 1. the previous launch's cross-piece combine, after that launch has
  // completed.  The wait also comes before any partial of this launch is
  // written: this launch may start while the previous attention launch still
  // runs, and that launch reads the partials of the launch before it, which
  // share this launch's buffer.  With a flag for it, wait on the flag (the
  // selection in between may still run); else on griddepcontrol.wait, which
  // returns once every earlier launch of the chain has completed.
  if (p.prev_done) {
    if (lane == 0)
      wait_flag(p.prev_done + (*p.epoch & 1u) * p.pool_stride, p.prev_done_expect, abort_flag, p.status);
    __syncwarp();
  } else {
    pdl_wait();
  }
  // the consumer warps that write one-tile pieces' partial states themselves
  // wait for this (release: the acquire above)
  if (lane == 0) mbar_arrive(&bars[C::BAR_PREVOK]);
  for (int t = blockIdx.x; t < p.prev_ntasks; t += gridDim.x) {
    const int2 task = p.prev_tasks[t];
    const Segment& sg = p.prev_segs[task.x];
    const int o = task.y, nout = sg.nout, np = sg.npieces;
    const int64_t idx0 = sg.part_base + o;
    LseAcc acc;
    lse_init(acc);
    for (int u0 = 0; u0 < np; u0 += 8) {  // eight partials in flight per lane
      float2 ml[8];
      float4 ov[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t idx = idx0 + static_cast<int64_t>(min(u0 + j, np - 1)) * nout;
        ml[j] = __ldcg(&p.prev_part_ml[idx]);
        ov[j] = col ? __ldcg(reinterpret_cast<const float4*>(&p.prev_part_o[idx * D + lane * 4]))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (u0 + j < np) lse_add(acc, ml[j], ov[j]);
    }
    lse_finish(acc, sg.out ? sg.out : p.prev_out, p, sg, o, lane, col, D);
  }

  // ---- 2. this launch's pieces of more than one tile (a one-tile piece's
  // warp writes its result itself).  Tile j of a piece whose first tile is
  // the CTA's tile t0 went to consumer warp (t0 + j) % NC, which took tiles
  // j, j + NC, ... of the piece in order; merging the warps' states in the
  // order of j makes the piece's result independent of t0, i.e. of which
  // CTA took the piece and what it did before (results repeat bit for bit).
  int mp = 0;
  int t = 0;  // CTA-wide tile sequence number, as the consumers count it
  for (int pi = 0;; ++pi) {
    Piece pc;
    if (!cta_piece<C>(p, smem, pbeg, pend, pi, lane, &pc)) break;
    const int t0 = t;
    t += (pc.r1 - pc.r0 + kTileRows - 1) / kTileRows;
    if (pc.r1 - pc.r0 <= kTileRows) continue;
    const Segment& sg = p.segs[pc.seg];
    const int nout = sg.nout;
    const int slot = mp % kPartSlots;
    if (!mbar_wait(&slot_full[slot], (mp / kPartSlots) & 1, abort_flag, p.status)) return;
    ++mp;
    const int64_t rec0 = (static_cast<int64_t>(cta_ring<C>(smem)) * kPartSlots + slot) * NC * wq;
    // load every output's NC warp states first (all in flight), then merge
    for (int o0 = 0; o0 < nout; o0 += 2) {
      float2 ml[2][NC];
      float4 ov[2][NC];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = sg.out_row[min(o0 + h, nout - 1)];
#pragma unroll
        for (int j = 0; j < NC; ++j) {  // entry j: the warp that took tiles j, j + NC, ...
          const int ww = (t0 + j) % NC;
          ml[h][j] = p.wpart_ml[rec0 + ww * wq + r];
          ov[h][j] = col ? *reinterpret_cast<const float4*>(p.wpart_o + (rec0 + ww * wq + r) * D + lane * 4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int o = o0 + h;
        if (o >= nout) break;
        LseAcc acc;
        lse_init(acc);
#pragma unroll
        for (int j = 0; j < NC; ++j) lse_add(acc, ml[h][j], ov[h][j]);
        if (sg.npieces == 1) {
          lse_finish(acc, sg.out ? sg.out : p.out, p, sg, o, lane, col, D);  // the whole segment
        } else {
          const int64_t idx = sg.part_base + static_cast<int64_t>(pc.ordinal) * nout + o;
          if (col) *reinterpret_cast<float4*>(&p.part_o[idx * D + lane * 4]) = acc.o;
          if (lane == 0) p.part_ml[idx] = make_float2(acc.M, acc.L);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&slot_free[slot]);  // the consumers may reuse the slot
  }
}

// ---------------------------------------------------------------- kernel
template <int D, int NC, int NP, int STAGES, bool GT, bool PG>
__global__ void __launch_bounds__(MmaCfg<D, NC, NP, STAGES, GT>::kThreads, 1)
    attn_mma_layer_kernel(const __grid_constant__ AttnMmaParams P) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  const uint64_t t_start = P.p.timeline ? global_timer_ns() : 0;
  extern __shared__ unsigned char smem_raw[];
  // the 128B-swizzled TMA destination needs 1024-byte alignment
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars[s], C::kFullCount);  // full: arrivals + TMA bytes
      mbar_init(&bars[STAGES + s], 1);           // empty: the one warp that consumed the tile
    }
    for (int r = 0; r < C::IR; ++r) mbar_init(&bars[2 * STAGES + r], 1);
    for (int r = 0; r < kPartSlots; ++r) {
      mbar_init(&bars[2 * STAGES + C::IR + r], NC);  // slot full: every consumer warp
      mbar_init(&bars[2 * STAGES + C::IR + kPartSlots + r], 1);  // slot free: the epilogue warp
    }
    for (int r = 0; r < kPoolRing; ++r) {
      mbar_init(&bars[C::BAR_UNIT + r], 1);                             // unit full: the scheduler
      mbar_init(&bars[C::BAR_UNIT + kPoolRing + r], C::kRingReaders);  // unit empty: every reader
    }
    for (int r = 0; r < C::IR; ++r) mbar_init(&bars[C::BAR_IDXFREE + r], 1);  // the tile's consumer
    mbar_init(&bars[C::BAR_PREVOK], 1);                                       // the epilogue warp
    *reinterpret_cast<int*>(smem + C::OFF_FLAGS) = 0;
    // this CTA's ring of piece states: its SM's (CTAs of consecutive
    // launches may overlap in time), else the block's
    reinterpret_cast<int*>(smem + C::OFF_FLAGS)[1] =
        P.p.wpart_by_sm ? static_cast<int>(sm_index()) : static_cast<int>(blockIdx.x);
    fence_mbar_init();
  }
  if (threadIdx.x == C::kFirstProducer) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmv)) : "memory");
    if (GT) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tgk)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tgv)) : "memory");
    }
  }
  __syncthreads();
  pdl_launch_dependents();
  if (P.p.wait_prev) pdl_wait();  // the previous launch writes what this one reads or writes
  static_assert(2 * C::SMEM > 232448, "the per-SM ring needs one CTA per SM");
  if (cta_ring<C>(smem) >= P.p.wpart_slots) {
    if (threadIdx.x == 0) {
      atomicOr(P.p.status, kStatusScratch);
      // no work, but the arrivals of its consumer warps for every layer it
      // has own pieces of, so that no selection waits out its limit
      if (P.p.keys_done) {
        int last = -1;
        for (int i = P.p.cta_begin[blockIdx.x]; i < P.p.cta_begin[blockIdx.x + 1]; ++i) {
          const int sl = P.p.segs[P.p.pieces[i].seg].l;
          if (sl != last) keys_arrive(P.p, sl, NC);
          last = sl;
        }
      }
    }
  } else {
    const int pbeg = P.p.cta_begin[blockIdx.x];
    const int pend = P.p.cta_begin[blockIdx.x + 1];
    if (threadIdx.x >= C::kFirstProducer) {
      mma_producers<D, NC, NP, STAGES, GT, PG>(P, smem, pbeg, pend);
    } else if (threadIdx.x >= C::kScheduler) {
      if (threadIdx.x == C::kScheduler) mma_scheduler<D, NC, NP, STAGES, GT>(P, smem, pbeg, pend);
    } else if (threadIdx.x >= NC * 32) {
      mma_epilogue<D, NC, NP, STAGES, GT>(P, smem, pbeg, pend);
    } else {
      mma_consumers<D, NC, NP, STAGES, GT>(P, smem, pbeg, pend);
    }
  }
  // every write of the CTA is done before its arrival on the launch's done
  // counter; the last CTA to arrive raises the flag.  Release: the CTA
  // barrier orders every thread's writes before thread 0's device-scope
  // fence, which precedes the arrival (one fence per CTA: a fence in every
  // thread stalls every warp on its own outstanding stores).
  __syncthreads();
  if (threadIdx.x == 0 && P.p.done) red_release_add_u32(P.p.done + (*P.p.epoch & 1u) * P.p.pool_stride, 1u);
  // This grid completes only after the one it depends on, so that the
  // launches of the step complete in launch order (dense-only CTAs never
  // waited above).  With a completion counter, one CTA waits and the others
  // leave at once: a CTA that waits here holds its SM idle, and the next
  // launch's CTAs need the SMs.  The timeline's end is the end of the CTA's
  // last warp.
  if (threadIdx.x == 0) {
    if (!P.p.done || blockIdx.x == 0) pdl_wait();
    timeline_record(P.p.timeline, P.p.timeline_cap, t_start,
                    (kTagAttention << 32) | (static_cast<unsigned long long>(P.p.layer) << 16) | blockIdx.x);
  }
}

// ---------------------------------------------------------------- host side
template <int D, int NC, int NP, int STAGES, bool GT, bool PG = false>
static cudaError_t mma_run(const AttnMmaParams* P, int grid, cudaStream_t stream, int* smem_out,
                           bool configure_only) {
  using C = MmaCfg<D, NC, NP, STAGES, GT>;
  auto kern = attn_mma_layer_kernel<D, NC, NP, STAGES, GT, PG>;
  if (configure_only) {
    if (smem_out) *smem_out = C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    // every kernel of the step asks for the same shared-memory carveout, so an
    // SM never has to reconfigure between consecutive kernels
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, *P);
}

// Consumer warps of the instantiation for head_dim D (the key counter of a
// launch reaches keys_ctas times this).
int attn_mma_consumer_warps(int D) { return D == 64 ? 4 : 6; }

// bf16 inputs.  configure_only: set the shared-memory attribute, report the size.
cudaError_t attn_mma_dispatch(int D, const AttnMmaParams* P, int grid, cudaStream_t stream,
                              int* smem_out, bool configure_only) {
  // gathered rows by TMA (one producer warp) when the planner built the
  // row-gather maps, else by cp.async from eight producer warps
  if (configure_only) {
    int s1 = 0, s2 = 0;
    cudaError_t e = cudaErrorInvalidValue;
    if (D == 128) {
      e = mma_run<128, 6, 8, 6, false>(P, grid, stream, &s1, true);
      if (e == cudaSuccess) e = mma_run<128, 6, 8, 6, false, true>(P, grid, stream, &s1, true);
      if (e == cudaSuccess) e = mma_run<128, 6, 1, 6, true>(P, grid, stream, &s2, true);
    } else if (D == 64) {
      e = mma_run<64, 4, 8, 8, false>(P, grid, stream, &s1, true);
      if (e == cudaSuccess) e = mma_run<64, 4, 8, 8, false, true>(P, grid, stream, &s1, true);
      if (e == cudaSuccess) e = mma_run<64, 4, 1, 8, true>(P, grid, stream, &s2, true);
    }
    if (smem_out) *smem_out = s1 > s2 ? s1 : s2;
    return e;
  }
  // a paged cache (the planner never pairs it with the row-gather maps) runs
  // on its own instantiation, so the contiguous one carries no paging code
  const bool gt = P->p.gather_rows > 0;
  const bool pg = P->p.paged != 0;
  if (D == 128)
    return gt ? mma_run<128, 6, 1, 6, true>(P, grid, stream, smem_out, false)
           : pg ? mma_run<128, 6, 8, 6, false, true>(P, grid, stream, smem_out, false)
                : mma_run<128, 6, 8, 6, false>(P, grid, stream, smem_out, false);
  if (D == 64)
    return gt ? mma_run<64, 4, 1, 8, true>(P, grid, stream, smem_out, false)
           : pg ? mma_run<64, 4, 8, 8, false, true>(P, grid, stream, smem_out, false)
                : mma_run<64, 4, 8, 8, false>(P, grid, stream, smem_out, false);
  return cudaErrorInvalidValue;
}

}  // namespace lyc
