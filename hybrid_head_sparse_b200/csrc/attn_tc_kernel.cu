// attn_tc_kernel.cu -- pooled hybrid-head decode attention for one layer,
// bf16 inputs, head_dim 128, on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// Computes the same as attn_mma_kernel.cu (page "LycheeDecode ...",
// paper-graph-ui summary, section 3.4 Eq. 1 for retrieval rows, Eq. 3 for
// gathered rows, the selection keys of the refreshed sets for Eq. 2, and the
// piece partials of Appendix C / Algorithm 2), with the work in 128-row tiles:
//   S^T[128 keys x 16 queries] = K[128 x 128] . Q^T       (one M=128 N=16 MMA
//                                                          per 16 columns of d)
//   O^T[128 d x 16 queries]   += V^T[128 x 128 keys] . P^T (M=128 N=16, per 16 keys)
// Queries of a segment (at most 8: the GQA group) are the N side, padded to
// 16; the K/V tile is the M side, read by the tensor core straight from the
// shared-memory stage it was loaded into (128-byte swizzle: K-major for K,
// MN-major for V^T), so no thread touches K or V.
//
// Warps: 0 issues the MMAs (one thread) and owns the tensor memory; 1-4 are
// the softmax warps, thread i of them owning key row i of S^T and d row i of
// O^T (tensor-memory lane i); 5 runs the previous layer's cross-piece combine;
// 6-13 load the tiles (TMA tensor copies for contiguous rows, 16-byte
// cp.async gathers for inherited rows).  Two S^T buffers let the QK MMA of
// tile t+1 run while the softmax of tile t does; the online softmax keeps a
// running maximum per query and rescales O^T (in tensor memory) only when the
// maximum grows by more than 2^8, so the rescale is rare.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "lyc_device.cuh"
#include "lyc_plan.h"
#include "tc_ptx.cuh"

namespace lyc {

namespace {

typedef uint16_t bf16_t;
constexpr int kTcRows = 128;  // rows per tile: the M side of one MMA

template <int STAGES>
struct TcCfg {
  static constexpr int D = 128;
  static constexpr int NQ = 16;               // MMA N: query rows padded to 16
  static constexpr int NP = 8;                // producer warps
  static constexpr int kSoftThreads = 128;    // warps 1-4
  static constexpr int kEpiWarp = 5;
  static constexpr int kFirstProducer = 6 * 32;
  static constexpr int kThreads = (6 + NP) * 32;
  static constexpr int HALF = kTcRows * 128;  // one 64-column half of a K or V tile
  static constexpr int TILEB = 2 * HALF;      // K (or V) tile bytes
  static constexpr int IR = 8;                // index ring slots
  static constexpr int LA = 4;                // index lookahead (tiles)
  static_assert(IR > LA + STAGES, "index ring too small for the lookahead");
  // shared memory (bytes from a 1024-aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * TILEB;
  static constexpr int OFF_Q = OFF_V + STAGES * TILEB;   // [2 pieces][2 halves][16 rows][128 B]
  static constexpr int OFF_P = OFF_Q + 2 * 2 * NQ * 128; // [2][16 key groups][2][8 keys][16 B]
  static constexpr int PBYTES = kTcRows * NQ * 2;
  static constexpr int OFF_IDX = OFF_P + 2 * PBYTES;
  static constexpr int OFF_RED = OFF_IDX + IR * kTcRows * 4;  // tile maxima [2][4][8], sums [4][8]
  static constexpr int OFF_BAR = OFF_RED + 1024;
  // barriers: full[S], empty[S], idx[IR], s_ready[2], s_free[2], p_ready[2],
  // pv_done[2], o_free, mma_idle
  static constexpr int NBAR = 2 * STAGES + IR + 8 + 2;
  static constexpr int OFF_FLAGS = OFF_BAR + NBAR * 8;  // abort flag, tensor-memory address
  static constexpr int SMEM = OFF_FLAGS + 16 + 1024;
  static constexpr uint32_t kTmemCols = 64;  // S^T x2 (cols 0, 16), O^T (col 32)
};

// byte offset of 16-byte chunk `ch` (0 .. 15) of tile row `r` (128-byte swizzle)
__device__ __forceinline__ uint32_t tswz(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * (kTcRows * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
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
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// order-preserving float -> uint (for warp max reductions)
__device__ __forceinline__ uint32_t f2o(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float o2f(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace
}  // namespace lyc

namespace lyc {
namespace {

// ---------------------------------------------------------------- producers
// NP warps walk the CTA's tiles.  Dense tile: one thread issues the TMA
// tensor copies (counted in bytes), everyone arrives.  Gathered tile: warp pw
// copies rows [16 pw, 16 pw + 16) with cp.async and every lane arrives when
// its own copies have landed (cp.async.mbarrier.arrive), the pattern the
// tensor core's reads of a cp.async-filled stage follow in CUTLASS's sm100
// cp.async pipelines.
template <int STAGES>
__device__ __forceinline__ void tc_producers(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                             int pend) {
  using C = TcCfg<STAGES>;
  const AttnParams& p = P.p;
  const int ptid = threadIdx.x - C::kFirstProducer;
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
  const bool leader = ptid == 0;

  // lookahead cursor (leader only): index-list copies of gathered tiles
  int la_pc = pbeg, la_r0 = (pbeg < pend) ? p.pieces[pbeg].r0 : 0, la_t = 0;
  bool waited = false;
  auto la_step = [&]() {
    if (la_pc >= pend) return;
    const Piece pc = p.pieces[la_pc];
    const Segment& ls = p.segs[pc.seg];
    if (ls.kind == kSparse) {
      // a set the previous launch writes is read only once it has completed;
      // sets of earlier selections were complete before that launch began
      if (ls.dep && !waited) {
        pdl_wait();
        waited = true;
      }
      const int slot = la_t % C::IR;
      const int nrows = min(kTcRows, pc.r1 - la_r0);
      const uint32_t bytes = static_cast<uint32_t>(((nrows * 4) + 15) & ~15);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&idxbar[slot], bytes);
      bulk_g2s(idxring + slot * kTcRows, ls.idx + la_r0, bytes, &idxbar[slot]);
    }
    ++la_t;
    la_r0 += kTcRows;
    if (la_r0 >= pc.r1) {
      ++la_pc;
      if (la_pc < pend) la_r0 = p.pieces[la_pc].r0;
    }
  };
  if (leader)
    for (int a = 0; a < C::LA; ++a) la_step();

  constexpr int CH = C::D / 8;            // 16-byte chunks per row
  constexpr int ROWS_W = kTcRows / C::NP; // rows per producer warp
  constexpr int RPI = 32 / CH;            // rows per warp instruction
  uint32_t idx_phase = 0;
  int t = 0;
  for (int pcI = pbeg; pcI < pend && !*abort_flag; ++pcI) {
    const Piece pc = p.pieces[pcI];
    const Segment& sg = p.segs[pc.seg];
    const bool dense = sg.kind == kDense;
    const int64_t s_token = sg.s_token;
    const bf16_t* kb = static_cast<const bf16_t*>(sg.k);
    const bf16_t* vb = static_cast<const bf16_t*>(sg.v);
    const int sl = sg.l, sb = sg.b, sgg = sg.g;
    for (int r0 = pc.r0; r0 < pc.r1; r0 += kTcRows, ++t) {
      if (leader) la_step();
      const int nrows = min(kTcRows, pc.r1 - r0);
      const int stage = t % STAGES;
      if (t >= STAGES) {
        if (!mbar_wait(&empty[stage], ((t / STAGES) - 1) & 1, abort_flag, p.status)) break;
      }
      unsigned char* kdst = Ks + stage * C::TILEB;
      unsigned char* vdst = Vs + stage * C::TILEB;
      if (dense) {
        // TMA tensor copies; rows past n are filled with zeros by the copy
        if (leader) {
          mbar_arrive_expect_tx(&full[stage], 2u * C::TILEB);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_5d(kdst + h * C::HALF, &P.tmk, h * 64, r0, sgg, sb, sl, &full[stage], pol);
            tma_load_5d(vdst + h * C::HALF, &P.tmv, h * 64, r0, sgg, sb, sl, &full[stage], pol);
          }
        }
        if (!leader) mbar_arrive(&full[stage]);  // the leader's arrival carries the bytes
      } else {
        const int slot = t % C::IR;
        if (!mbar_wait(&idxbar[slot], (idx_phase >> slot) & 1u, abort_flag, p.status)) break;
        idx_phase ^= 1u << slot;
        const int32_t* ring = idxring + slot * kTcRows;
        if (pw == 0) {  // bounds of the inherited indices (reported, never followed)
          bool bad = false;
#pragma unroll
          for (int i = 0; i < kTcRows / 32; ++i) {
            const int r = lane + 32 * i;
            const int32_t ix = (r < nrows) ? ring[r] : 0;
            bad |= index_bad(ix, sg.nvalid, sg.pad_ok);
          }
          if (bad) atomicOr(p.status, kStatusBadIndex);
        }
        const uint32_t kbase = smem_u32(kdst), vbase = smem_u32(vdst);
#pragma unroll
        for (int i = 0; i < ROWS_W / RPI; ++i) {
          const int r = pw * ROWS_W + i * RPI + lane / CH;
          const int c = lane % CH;
          const int32_t ix = (r < nrows) ? ring[r] : -1;
          const bool ok = ix >= 0 && ix < sg.nvalid;
          const int64_t off = ok ? static_cast<int64_t>(ix) * s_token : 0;
          cp_async_16(kbase + tswz(r, c), kb + off + c * 8, ok ? 16u : 0u);
          cp_async_16(vbase + tswz(r, c), vb + off + c * 8, ok ? 16u : 0u);
        }
        cp_async_arrive(&full[stage]);
      }
    }
  }
}

}  // namespace
}  // namespace lyc

namespace lyc {
namespace {

// barrier indices within the block of barriers
template <int STAGES>
struct TcBars {
  uint64_t* full;     // [STAGES] producers -> MMA: stage loaded (NP*32 arrivals + bytes)
  uint64_t* empty;    // [STAGES] MMA commit -> producers: stage free
  uint64_t* idx;      // [IR]     index ring
  uint64_t* s_ready;  // [2] MMA commit -> softmax: S^T buffer written
  uint64_t* s_free;   // [2] softmax (128) -> MMA: S^T buffer read
  uint64_t* p_ready;  // [2] softmax (128) -> MMA: P^T buffer written (and O^T rescaled)
  uint64_t* pv_done;  // [2] MMA commit -> softmax: the PV of the tile using P^T buffer b done
  uint64_t* o_free;   // softmax (128) -> MMA: O^T of the piece read out
  uint64_t* mma_idle; // MMA commit -> MMA: everything issued has completed
  __device__ explicit TcBars(unsigned char* smem) {
    using C = TcCfg<STAGES>;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    full = b;
    empty = b + STAGES;
    idx = b + 2 * STAGES;
    s_ready = idx + C::IR;
    s_free = s_ready + 2;
    p_ready = s_free + 2;
    pv_done = p_ready + 2;
    o_free = pv_done + 2;
    mma_idle = o_free + 1;
  }
};

// ---------------------------------------------------------------- MMA warp
// Two streams of work, each in tile order: the QK of tile t (stage t %
// STAGES loaded; S^T buffer t & 1 read by the softmax two tiles ago): eight
// M=128 N=16 K=16 MMAs, S^T = K Q^T, committed to s_ready; and the PV of tile
// t (its P^T written): eight MMAs, O^T += V^T P^T, committed to the stage's
// `empty` and to pv_done.  Lane 0 polls both and issues whichever is ready,
// (non-blocking tests), so a stage is freed as soon as its PV can run, never
// behind the arrival of a later tile.
template <int STAGES>
__device__ __forceinline__ void tc_mma(const AttnMmaParams& P, unsigned char* smem, int pbeg, int pend,
                                       uint32_t tmem) {
  using C = TcCfg<STAGES>;
  constexpr unsigned FULL = 0xffffffffu;
  const AttnParams& p = P.p;
  const int lane = threadIdx.x & 31;
  TcBars<STAGES> br(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  constexpr uint32_t IDESC_QK = tc::idesc_bf16(128, C::NQ, 0, 0);  // K-major K and Q
  constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, C::NQ, 1, 1);  // MN-major V^T and P^T
  const uint32_t kbase = smem_u32(smem + C::OFF_K);
  const uint32_t vbase = smem_u32(smem + C::OFF_V);
  const uint32_t qbase = smem_u32(smem + C::OFF_Q);
  const uint32_t pbase = smem_u32(smem + C::OFF_P);
  const bf16_t* qg = static_cast<const bf16_t*>(p.q);

  // a cursor over the CTA's tiles: piece, tile within it, CTA-wide tile number
  struct Cursor {
    int pc, u, ntile, t;
  };
  auto ntiles_of = [&](int pcI) {
    const Piece pc = p.pieces[pcI];
    return (pc.r1 - pc.r0 + kTcRows - 1) / kTcRows;
  };
  auto advance = [&](Cursor& c) {
    ++c.t;
    if (++c.u >= c.ntile) {
      c.u = 0;
      ++c.pc;
      c.ntile = (c.pc < pend) ? ntiles_of(c.pc) : 0;
    }
  };
  Cursor qk{pbeg, 0, pbeg < pend ? ntiles_of(pbeg) : 0, 0};
  Cursor pv = qk;

  // the QK of the tile under qk (its stage and S^T buffer must be ready)
  auto qk_ready = [&](bool block) -> int {
    const int t = qk.t, stage = t % STAGES, b = t & 1;
    int ready = 1;
    if (lane == 0) {
      if (block) {
        ready = mbar_wait(&br.full[stage], (t / STAGES) & 1, abort_flag, p.status) &&
                (t < 2 || mbar_wait(&br.s_free[b], ((t - 2) >> 1) & 1, abort_flag, p.status));
      } else {
        ready = mbar_test_wait(&br.full[stage], (t / STAGES) & 1) &&
                (t < 2 || mbar_test_wait(&br.s_free[b], ((t - 2) >> 1) & 1));
      }
    }
    return __shfl_sync(FULL, ready, 0);
  };
  auto issue_qk = [&]() {
    const int t = qk.t, stage = t % STAGES, b = t & 1;
    const int pi = qk.pc - pbeg;
    if (qk.u == 0) {
      // this piece's query rows into Q buffer pi & 1 (K-major, 128-byte
      // swizzle, rows >= nq zero); its previous user, piece pi-2, had its
      // last QK complete before the softmax freed the S^T buffer this QK
      // waited for
      const Piece pc = p.pieces[qk.pc];
      const Segment& sg = p.segs[pc.seg];
      unsigned char* qb = smem + C::OFF_Q + (pi & 1) * (2 * C::NQ * 128);
      for (int c = lane; c < C::NQ * 16; c += 32) {
        const int row = c >> 4, ch = c & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < sg.nq)
          v = *reinterpret_cast<const uint4*>(
              qg + (static_cast<int64_t>(sg.b) * p.Hq + sg.head[row]) * C::D + ch * 8);
        *reinterpret_cast<uint4*>(qb + (ch >> 3) * (C::NQ * 128) + row * 128 +
                                  (((ch & 7) ^ (row & 7)) << 4)) = v;
      }
      tc::fence_async_smem();
      __syncwarp();
    }
    tc::fence_after_sync();
    if (lane == 0) {
      const uint32_t qpiece = qbase + (pi & 1) * (2 * C::NQ * 128);
#pragma unroll
      for (int kk = 0; kk < C::D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * C::HALF + (kk & 3) * 32;
        const uint32_t qoff = (kk >> 2) * (C::NQ * 128) + (kk & 3) * 32;
        const uint64_t a = tc::smem_desc(kbase + stage * C::TILEB + koff, 16, 1024, 2);
        const uint64_t bd = tc::smem_desc(qpiece + qoff, 16, 1024, 2);
        tc::mma_bf16_ss(tmem + b * C::NQ, a, bd, IDESC_QK, kk > 0 ? 1u : 0u);
      }
      tc::commit(&br.s_ready[b]);
    }
    __syncwarp();
    advance(qk);
  };

  // QK runs one tile ahead of PV: before each PV, the next QK is issued if
  // its stage is already loaded; after it, the next QK waits for its stage,
  // so a late tile never holds back the PV that frees an earlier stage.
  bool ok = true;
  if (qk.pc < pend) ok = qk_ready(true) != 0;
  if (ok && qk.pc < pend) issue_qk();
  while (ok && pv.pc < pend) {
    const bool ahead_open = qk.pc < pend && qk.t == pv.t + 1;
    if (ahead_open && qk_ready(false)) issue_qk();
    // PV of the tile under pv
    {
      const int t = pv.t, stage = t % STAGES, b = t & 1;
      const int piece = pv.pc - pbeg;
      const bool first = pv.u == 0;
      int ready = 1;
      if (lane == 0)
        ready = mbar_wait(&br.p_ready[b], (t >> 1) & 1, abort_flag, p.status) &&
                (!first || piece == 0 || mbar_wait(br.o_free, (piece - 1) & 1, abort_flag, p.status));
      if (!__shfl_sync(FULL, ready, 0)) break;
      tc::fence_after_sync();
      if (lane == 0) {
#pragma unroll
        for (int kt = 0; kt < kTcRows / 16; ++kt) {
          const uint64_t a = tc::smem_desc(vbase + stage * C::TILEB + kt * 16 * 128, C::HALF, 1024, 2);
          const uint64_t bd = tc::smem_desc(pbase + b * C::PBYTES + kt * 512, 256, 128, 0);
          tc::mma_bf16_ss(tmem + 32, a, bd, IDESC_PV, (kt > 0 || !first) ? 1u : 0u);
        }
        tc::commit(&br.empty[stage]);
        tc::commit(&br.pv_done[b]);
      }
      __syncwarp();
      advance(pv);
    }
    if (qk.pc < pend && qk.t == pv.t) {  // the next PV needs this QK
      if (!qk_ready(true)) break;
      issue_qk();
    }
  }
  // every MMA issued has completed before the tensor memory is released
  if (lane == 0) tc::commit(br.mma_idle);
  __syncwarp();
  mbar_wait(br.mma_idle, 0, abort_flag, p.status);
}

}  // namespace
}  // namespace lyc

namespace lyc {
namespace {

__device__ __forceinline__ void st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// named barrier `id` over `n` threads that also ORs a predicate across them
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- softmax warps
// Thread i (of 128) owns tensor-memory lane i: key row i of each S^T tile and
// d row i of O^T.  Per tile: read its 16 logits, write the selection keys of
// a dense segment, exchange per-query tile maxima through shared memory,
// rescale O^T if a maximum grew by more than 2^8, and write its row of P^T
// (bf16) for the PV MMA.  At a piece's end: sum the per-thread softmax
// denominators, read O^T, and write the piece's partial (or, for a segment of
// one piece, the output).
template <int STAGES>
__device__ __forceinline__ void tc_softmax(const AttnMmaParams& P, unsigned char* smem, int pbeg,
                                           int pend, uint32_t tmem) {
  using C = TcCfg<STAGES>;
  constexpr unsigned FULL = 0xffffffffu;
  const AttnParams& p = P.p;
  const int lane = threadIdx.x & 31;
  const int quarter = (threadIdx.x >> 5) & 3;  // this warp's quarter of the 128 lanes
  const int kr = quarter * 32 + lane;
  TcBars<STAGES> br(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][8] maxima, then [4][8] sums
  const int32_t* idxring = reinterpret_cast<const int32_t*>(smem + C::OFF_IDX);
  unsigned char* pbuf = smem + C::OFF_P;
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const float sl2 = p.scale_log2;
  int t = 0;
  for (int pcI = pbeg; pcI < pend; ++pcI) {
    const Piece pc = p.pieces[pcI];
    const Segment& sg = p.segs[pc.seg];
    const int nq = sg.nq, nout = sg.nout;
    const bool dense = sg.kind == kDense;
    const int64_t key_mean_off = sg.key_mean_off;
    const float mean_scale = p.scale / static_cast<float>(nq);
    int64_t koff[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) koff[q] = (dense && q < nq) ? sg.key_off[q] : -1;
    float m[8], l[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
    }
    const int ntile = (pc.r1 - pc.r0 + kTcRows - 1) / kTcRows;
    for (int u = 0; u < ntile; ++u, ++t) {
      const int b = t & 1;
      const int r0 = pc.r0 + u * kTcRows;
      const int nrows = min(kTcRows, pc.r1 - r0);
      if (!mbar_wait(&br.s_ready[b], (t >> 1) & 1, abort_flag, p.status)) return;
      tc::fence_after_sync();
      uint32_t sr[16];
      tc::ld_32x32b_x16(tl + b * C::NQ, sr);
      tc::wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&br.s_free[b]);
      bool valid = kr < nrows;
      if (!dense && valid) {
        // the stage's arrival orders the index ring's contents (the producers
        // waited for them) before this read
        if (!mbar_wait(&br.full[t % STAGES], (t / STAGES) & 1, abort_flag, p.status)) return;
        const int32_t x = idxring[(t % C::IR) * kTcRows + kr];
        valid = x >= 0 && x < sg.nvalid;
      }
      float x[8];  // logits in log2 units; -inf for rows or queries not in use
      bool over = false;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float sq = __uint_as_float(sr[q]);
        x[q] = (valid && q < nq) ? sq * sl2 : -INFINITY;
        if (q < nq) {
          if (valid && koff[q] >= 0) p.keys[koff[q] + r0 + kr] = sq * p.scale;  // selection key
          over |= x[q] > m[q] + 8.f;
        }
      }
      if (dense && valid && key_mean_off >= 0) {
        float xs = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) xs += (q < nq) ? __uint_as_float(sr[q]) : 0.f;
        p.keys[key_mean_off + r0 + kr] = xs * mean_scale;
      }
      // The running maximum of each query moves only when a logit exceeds it
      // by more than 2^8 (or on a piece's first rows): one barrier with an OR
      // tells every thread; then, rarely, the tile's maxima are exchanged and
      // O^T is rescaled.  Weights up to 2^8 are exact enough in bf16 and far
      // from fp32 overflow.
      if (named_bar_or(1, C::kSoftThreads, over)) {
        float* rmax = red + (t & 1) * 32;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < nq) {
            const uint32_t mx = __reduce_max_sync(FULL, f2o(x[q]));
            if (lane == 0) rmax[quarter * 8 + q] = o2f(mx);
          }
        named_bar_sync(1, C::kSoftThreads);
        float alpha[8];
        bool resc = false;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          alpha[q] = 1.f;
          if (q < nq) {
            const float tm = fmaxf(fmaxf(rmax[q], rmax[8 + q]), fmaxf(rmax[16 + q], rmax[24 + q]));
            if (m[q] == -INFINITY) {
              m[q] = tm;  // nothing accumulated for this query yet (its P was all zero)
            } else if (tm > m[q] + 8.f) {
              alpha[q] = exp2f(m[q] - tm);
              m[q] = tm;
              resc = true;
            }
          }
        }
        if (resc) {  // the same decision in every thread: O^T = O^T * alpha, by column
          if (!mbar_wait(&br.pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, p.status)) return;
          tc::fence_after_sync();
          uint32_t o[16];
          tc::ld_32x32b_x16(tl + 32, o);
          tc::wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
          st_32x32b_x16(tl + 32, o);
          wait_st();
#pragma unroll
          for (int q = 0; q < 8; ++q) l[q] *= alpha[q];
        }
      }
      // this row of P^T into buffer b, once the PV that last read it (tile t-2) is done
      if (t >= 2 && !mbar_wait(&br.pv_done[b], ((t - 2) >> 1) & 1, abort_flag, p.status)) return;
      uint32_t pk[4];
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        float pv[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = 2 * q2 + h;
          pv[h] = (q < nq && x[q] != -INFINITY) ? exp2f(x[q] - m[q]) : 0.f;
        }
        pk[q2] = pack_bf16(pv[0], pv[1]);
        l[2 * q2] += __uint_as_float(pk[q2] << 16);  // the rounded weights, as the PV sees them
        l[2 * q2 + 1] += __uint_as_float(pk[q2] & 0xffff0000u);
      }
      *reinterpret_cast<uint4*>(pbuf + b * C::PBYTES + (kr >> 3) * 256 + (kr & 7) * 16) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
      tc::fence_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&br.p_ready[b]);
    }
    // ---- piece end: the denominators, O^T, the partial
    const int tl_last = t - 1;
    if (!mbar_wait(&br.pv_done[tl_last & 1], (tl_last >> 1) & 1, abort_flag, p.status)) return;
    tc::fence_after_sync();
    uint32_t o[16];
    tc::ld_32x32b_x16(tl + 32, o);
    tc::wait_ld();
    tc::fence_before_sync();
    mbar_arrive(br.o_free);
    float* rsum = red + 64;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float x = l[q];
#pragma unroll
      for (int s2 = 16; s2 >= 1; s2 >>= 1) x += __shfl_xor_sync(FULL, x, s2);
      if (lane == 0) rsum[quarter * 8 + q] = x;
    }
    named_bar_sync(1, C::kSoftThreads);
    for (int oo = 0; oo < nout; ++oo) {
      const int q = sg.out_row[oo];
      float L = 0.f, ov = 0.f, mq = -INFINITY;
#pragma unroll
      for (int qq = 0; qq < 8; ++qq)
        if (qq == q) {
          L = rsum[qq] + rsum[8 + qq] + rsum[16 + qq] + rsum[24 + qq];
          ov = __uint_as_float(o[qq]);
          mq = m[qq];
        }
      if (sg.npieces == 1) {
        float res = 0.f;
        if (L > 0.f) {
          res = ov / L;
        } else if (kr == 0) {
          atomicOr(p.status, kStatusEmptySoftmax);
        }
        p.out[(static_cast<int64_t>(sg.b) * p.Hq + sg.head[q]) * C::D + kr] = res;
      } else {
        const int64_t idx = sg.part_base + static_cast<int64_t>(pc.ordinal) * nout + oo;
        p.part_o[idx * C::D + kr] = ov;
        if (kr == 0) p.part_ml[idx] = make_float2(mq, L);
      }
    }
  }
}

}  // namespace
}  // namespace lyc

namespace lyc {
namespace {

// ---------------------------------------------------------------- combine warp
// The previous layer's cross-piece combine (Appendix C, Algorithm 2, steps
// 5-6): this CTA takes the (segment, output) tasks blockIdx.x,
// blockIdx.x + gridDim.x, ... and folds each output's piece partials
// (log-sum-exp, log2 units) into that layer's output.  That layer's attention
// completed before this launch began (the launch in between waited for it;
// without one, this waits), so its partials are in place.  Lane j owns
// columns 4j .. 4j+3.
__device__ __forceinline__ void tc_combine_prev(const AttnParams& p) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  if (p.prev_ntasks > 0) pdl_wait();
  for (int t = blockIdx.x; t < p.prev_ntasks; t += gridDim.x) {
    const int2 task = p.prev_tasks[t];
    const Segment& sg = p.prev_segs[task.x];
    const int o = task.y, nout = sg.nout, np = sg.npieces;
    const int64_t idx0 = sg.part_base + o;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int u0 = 0; u0 < np; u0 += 8) {  // eight partials in flight per lane
      float2 ml[8];
      float4 ov[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t idx = idx0 + static_cast<int64_t>(min(u0 + j, np - 1)) * nout;
        ml[j] = __ldcg(&p.prev_part_ml[idx]);
        ov[j] = __ldcg(reinterpret_cast<const float4*>(&p.prev_part_o[idx * D + lane * 4]));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (u0 + j >= np || ml[j].x == -INFINITY) continue;
        const float mn = fmaxf(M, ml[j].x);
        const float a = (M == -INFINITY) ? 0.f : exp2f(M - mn);
        const float f = exp2f(ml[j].x - mn);
        L = L * a + f * ml[j].y;
        acc.x = acc.x * a + f * ov[j].x;
        acc.y = acc.y * a + f * ov[j].y;
        acc.z = acc.z * a + f * ov[j].z;
        acc.w = acc.w * a + f * ov[j].w;
        M = mn;
      }
    }
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    if (L > 0.f) {
      const float inv = 1.f / L;
      res = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else if (lane == 0) {
      atomicOr(p.status, kStatusEmptySoftmax);
    }
    *reinterpret_cast<float4*>(
        &p.prev_out[(static_cast<int64_t>(sg.b) * p.Hq + sg.head[sg.out_row[o]]) * D + lane * 4]) = res;
  }
}

// ---------------------------------------------------------------- kernel
template <int STAGES>
__global__ void __launch_bounds__(TcCfg<STAGES>::kThreads, 1)
    attn_tc_layer_kernel(const __grid_constant__ AttnMmaParams P) {
  using C = TcCfg<STAGES>;
  const uint64_t t_start = P.p.timeline ? global_timer_ns() : 0;
  extern __shared__ unsigned char smem_raw[];
  // the 128-byte swizzle needs 1024-byte aligned tiles
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_FLAGS);  // [0] abort, [1] tmem
  if (threadIdx.x == 0) {
    TcBars<STAGES> br(smem);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&br.full[s], C::NP * 32);
      mbar_init(&br.empty[s], 1);
    }
    for (int r = 0; r < C::IR; ++r) mbar_init(&br.idx[r], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&br.s_ready[b], 1);
      mbar_init(&br.s_free[b], C::kSoftThreads);
      mbar_init(&br.p_ready[b], C::kSoftThreads);
      mbar_init(&br.pv_done[b], 1);
    }
    mbar_init(br.o_free, C::kSoftThreads);
    mbar_init(br.mma_idle, 1);
    flags[0] = 0u;
    fence_mbar_init();
  }
  // P^T buffers: the columns of queries 8..15 stay zero; the rest is written per tile
  for (int i = threadIdx.x; i < 2 * C::PBYTES / 16; i += C::kThreads)
    reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 0) {
    tc::tmem_alloc(flags + 1, C::kTmemCols);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == C::kFirstProducer) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmv)) : "memory");
  }
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  pdl_launch_dependents();
  if (P.p.wait_prev) pdl_wait();  // the previous launch writes what this one reads or writes
  const uint32_t tmem = flags[1];
  const int pbeg = P.p.cta_begin[blockIdx.x];
  const int pend = P.p.cta_begin[blockIdx.x + 1];
  if (threadIdx.x >= C::kFirstProducer) {
    tc_producers<STAGES>(P, smem, pbeg, pend);
  } else if (warp == C::kEpiWarp) {
    tc_combine_prev(P.p);
  } else if (warp >= 1) {
    tc_softmax<STAGES>(P, smem, pbeg, pend, tmem);
  } else {
    tc_mma<STAGES>(P, smem, pbeg, pend, tmem);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
  // this grid completes only after the one it depends on (CTAs that waited
  // for nothing above), so completion order follows launch order
  if (threadIdx.x == 0) {
    pdl_wait();
    timeline_record(P.p.timeline, P.p.timeline_cap, t_start,
                    (kTagAttention << 32) | (static_cast<unsigned long long>(P.p.layer) << 16) | blockIdx.x);
  }
}

constexpr int kTcStages = 3;

}  // namespace

// bf16, head_dim 128.  configure_only: set the shared-memory attributes, report the size.
cudaError_t attn_tc_dispatch(const AttnMmaParams* P, int grid, cudaStream_t stream, int* smem_out,
                             bool configure_only) {
  using C = TcCfg<kTcStages>;
  auto kern = attn_tc_layer_kernel<kTcStages>;
  if (configure_only) {
    if (smem_out) *smem_out = C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
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

int attn_tc_tile_rows() { return kTcRows; }

}  // namespace lyc
