// correction_kernel.cu -- Cache Correction's dense attention on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes (page "LycheeDecode ...", paper-graph-ui summary, section
// 4.2.2 and the decoding setup of section 4.1): every 32 decoded tokens the T
// most recent positions are prefilled again with dense attention.  Its
// attention part, for every layer l, batch element b and query head h: query
// t, at position p = n - T + t, attends rows 0..p of the cache (causal):
//   o = softmax(q K[0..p]^T / sqrt(d)) V[0..p].
// Rows n-T .. n-1 hold the refreshed K/V (written first when the caller
// passes them).
//
// Design (B200, bf16, d = 128).  The G query heads of a KV group times the T
// positions are one block of G*T <= 128 query rows: the M side of the MMAs.
// K/V tiles of 128 rows arrive by TMA (128-byte swizzle) and are read by the
// tensor core in place:
//   S[128 q x 128 keys]  = Q[128 x 128 d] . K^T      (8 MMAs, K=16 each, into TMEM)
//   O[128 q x 128 d]    += P[128 x 128 keys] . V     (8 MMAs, into TMEM: keys
//                                                     0-63 and 64-127 into O_a, O_b)
// Warps 0-7 are the softmax warps: warp w owns query rows 32*(w%4) .. +31
// (their tensor-memory lanes) and key half w/4 of every tile.  Each half
// keeps its own running maximum (O rescaled in tensor memory only when it
// grows by more than 2^8), sum and O accumulator, and writes its half of the
// row of P (bf16, 128-byte swizzle) for the PV MMA.  Warp 8 issues the MMAs
// (one thread) and owns the tensor memory; warp 9 issues the TMA copies (one
// thread).  Two S buffers and two P buffers let the QK MMA of tile t+1 and
// the softmax of tile t overlap.  Tensor memory: S x2 (columns 0, 128), O of
// key half 0 (256) and of key half 1 (384).
//
// Work pooling (Appendix C, Algorithm 2, applied to this dense pass): the
// (l, b, g) groups times their ceil(n/128) tiles are cut into equal runs, one
// per CTA; a run that crosses groups becomes several pieces.  Each piece
// writes two partial states (m, l, O) per query row, one per key half; a
// second launch merges the records of each group (log-sum-exp) into the
// output.
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
constexpr int kCcRows = 128;  // keys per tile; query rows per block

struct CcCfg {
  static constexpr int D = 128;
  static constexpr int STAGES = 2;
  static constexpr int kSoftThreads = 256;  // warps 0-7
  static constexpr int kMmaWarp = 8;
  static constexpr int kLoadWarp = 9;
  static constexpr int kThreads = 10 * 32;
  static constexpr int HALF = kCcRows * 128;  // one 64-column half of a tile (bytes)
  static constexpr int TILEB = 2 * HALF;      // a K, V, Q or P tile (bytes)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + TILEB;           // [2] P buffers
  static constexpr int OFF_K = OFF_P + 2 * TILEB;       // [STAGES]
  static constexpr int OFF_V = OFF_K + STAGES * TILEB;  // [STAGES]
  static constexpr int OFF_BAR = OFF_V + STAGES * TILEB;
  // kfull[S], vfull[S], kempty[S], vempty[S], s_ready[2], s_free[2],
  // p_ready[2], pv_done[2], q_ready, o_free, mma_idle
  static constexpr int NBAR = 4 * STAGES + 8 + 3;
  static constexpr int OFF_FLAGS = OFF_BAR + NBAR * 8;  // abort flag, tensor-memory address
  static constexpr int SMEM = OFF_FLAGS + 16 + 1024;    // + alignment slack
  static constexpr uint32_t kTmemCols = 512;            // S x2 (cols 0, 128), O (col 256)
};

struct CcBars {
  uint64_t *kfull, *vfull, *kempty, *vempty, *s_ready, *s_free, *p_ready, *pv_done, *q_ready,
      *o_free, *mma_idle;
  __device__ explicit CcBars(unsigned char* smem) {
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + CcCfg::OFF_BAR);
    constexpr int S = CcCfg::STAGES;
    kfull = b;
    vfull = b + S;
    kempty = b + 2 * S;
    vempty = b + 3 * S;
    s_ready = b + 4 * S;
    s_free = s_ready + 2;
    p_ready = s_free + 2;
    pv_done = p_ready + 2;
    q_ready = pv_done + 2;
    o_free = q_ready + 1;
    mma_idle = o_free + 1;
  }
};

// byte offset of 16-byte chunk `ch` (0 .. 15) of row `r` of a tile (128-byte swizzle)
__device__ __forceinline__ uint32_t cswz(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * CcCfg::HALF + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cc_tma_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                          int c3, int c4, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint32_t cc_pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void cc_st_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void cc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- loads
// One thread walks the CTA's tiles: K then V of each, into stage t % STAGES
// once the MMAs that read the stage's previous tile are done.
__device__ __forceinline__ void cc_loads(const CorrParams& P, unsigned char* smem, int pbeg, int pend) {
  constexpr int S = CcCfg::STAGES;
  CcBars br(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + CcCfg::OFF_FLAGS);
  const uint64_t pol = l2_policy_evict_first();
  int t = 0;
  for (int pc = pbeg; pc < pend; ++pc) {
    const CorrPiece piece = P.pieces[pc];
    for (int tile = piece.t0; tile < piece.t1; ++tile, ++t) {
      const int stage = t % S;
      if (t >= S && !mbar_wait(&br.kempty[stage], ((t / S) - 1) & 1, abort_flag, P.status)) return;
      unsigned char* kdst = smem + CcCfg::OFF_K + stage * CcCfg::TILEB;
      mbar_arrive_expect_tx(&br.kfull[stage], CcCfg::TILEB);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cc_tma_5d(kdst + h * CcCfg::HALF, &P.tmk, h * 64, tile * kCcRows, piece.g, piece.b, piece.l,
                  &br.kfull[stage], pol);
      if (t >= S && !mbar_wait(&br.vempty[stage], ((t / S) - 1) & 1, abort_flag, P.status)) return;
      unsigned char* vdst = smem + CcCfg::OFF_V + stage * CcCfg::TILEB;
      mbar_arrive_expect_tx(&br.vfull[stage], CcCfg::TILEB);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        cc_tma_5d(vdst + h * CcCfg::HALF, &P.tmv, h * 64, tile * kCcRows, piece.g, piece.b, piece.l,
                  &br.vfull[stage], pol);
    }
  }
}

// ---------------------------------------------------------------- MMA warp
// Per tile t: the QK MMA (S buffer t & 1 = Q K^T; K stage loaded, the S
// buffer read by the softmax two tiles ago, the piece's Q written), committed
// to s_ready and to the K stage's `kempty`; then the PV MMA of tile t
// (O += P V; P buffer t & 1 written; V stage loaded; at a piece's first tile
// the previous piece's O read out), committed to pv_done and `vempty`.  The
// QK of tile t+1 is issued before the PV of tile t, so the tensor core
// computes the next logits while the softmax works on this tile.
__device__ __forceinline__ void cc_mma(const CorrParams& P, unsigned char* smem, int pbeg, int pend,
                                       uint32_t tmem) {
  constexpr int S = CcCfg::STAGES;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr uint32_t IDESC_QK = tc::idesc_bf16(128, 128, 0, 0);  // K-major Q and K
  constexpr uint32_t IDESC_PV = tc::idesc_bf16(128, 128, 0, 1);  // K-major P, MN-major V
  const int lane = threadIdx.x & 31;
  CcBars br(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + CcCfg::OFF_FLAGS);
  const uint32_t qbase = smem_u32(smem + CcCfg::OFF_Q);
  const uint32_t pbase = smem_u32(smem + CcCfg::OFF_P);
  const uint32_t kbase = smem_u32(smem + CcCfg::OFF_K);
  const uint32_t vbase = smem_u32(smem + CcCfg::OFF_V);

  // tile cursors: piece, tile within it, CTA-wide tile number
  struct Cursor {
    int pc, u, ntile, t;
  };
  auto ntiles_of = [&](int pc) { return P.pieces[pc].t1 - P.pieces[pc].t0; };
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

  auto issue_qk = [&]() -> bool {
    const int t = qk.t, stage = t % S, b = t & 1;
    int ok = 1;
    if (lane == 0) {
      ok = mbar_wait(&br.kfull[stage], (t / S) & 1, abort_flag, P.status) &&
           (t < 2 || mbar_wait(&br.s_free[b], ((t - 2) >> 1) & 1, abort_flag, P.status)) &&
           (qk.u != 0 || mbar_wait(br.q_ready, (qk.pc - pbeg) & 1, abort_flag, P.status));
    }
    ok = __shfl_sync(FULL, ok, 0);
    if (!ok) return false;
    tc::fence_after_sync();
    if (lane == 0) {
#pragma unroll
      for (int kk = 0; kk < CcCfg::D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * CcCfg::HALF + (kk & 3) * 32;
        const uint64_t a = tc::smem_desc(qbase + off, 16, 1024, 2);
        const uint64_t bd = tc::smem_desc(kbase + stage * CcCfg::TILEB + off, 16, 1024, 2);
        tc::mma_bf16_ss(tmem + b * 128, a, bd, IDESC_QK, kk > 0 ? 1u : 0u);
      }
      tc::commit(&br.kempty[stage]);
      tc::commit(&br.s_ready[b]);
    }
    __syncwarp();
    advance(qk);
    return true;
  };

  bool ok = true;
  if (qk.pc < pend) ok = issue_qk();
  while (ok && pv.pc < pend) {
    // the look-ahead QK stays within the piece: a piece's first QK needs its
    // Q, which the softmax warps write only after this piece's last PV
    if (qk.pc < pend && qk.t == pv.t + 1 && qk.u != 0 && !issue_qk()) break;
    const int t = pv.t, stage = t % S, b = t & 1;
    const int piece = pv.pc - pbeg;
    const bool first = pv.u == 0;
    int ready = 1;
    if (lane == 0)
      ready = mbar_wait(&br.p_ready[b], (t >> 1) & 1, abort_flag, P.status) &&
              mbar_wait(&br.vfull[stage], (t / S) & 1, abort_flag, P.status) &&
              (!first || piece == 0 || mbar_wait(br.o_free, (piece - 1) & 1, abort_flag, P.status));
    if (!__shfl_sync(FULL, ready, 0)) break;
    tc::fence_after_sync();
    if (lane == 0) {
#pragma unroll
      for (int kt = 0; kt < kCcRows / 16; ++kt) {
        const uint64_t a =
            tc::smem_desc(pbase + b * CcCfg::TILEB + (kt >> 2) * CcCfg::HALF + (kt & 3) * 32, 16, 1024, 2);
        const uint64_t bd = tc::smem_desc(vbase + stage * CcCfg::TILEB + kt * 16 * 128, CcCfg::HALF, 1024, 2);
        // keys 0-63 accumulate into O_a (column 256), keys 64-127 into O_b (384)
        tc::mma_bf16_ss(tmem + 256 + (kt >> 2) * 128, a, bd, IDESC_PV, ((kt & 3) > 0 || !first) ? 1u : 0u);
      }
      tc::commit(&br.vempty[stage]);
      tc::commit(&br.pv_done[b]);
    }
    __syncwarp();
    advance(pv);
    if (qk.pc < pend && qk.t == pv.t && !issue_qk()) break;
  }
  // every MMA issued has completed before the tensor memory is released
  if (lane == 0) tc::commit(br.mma_idle);
  __syncwarp();
  mbar_wait(br.mma_idle, 0, abort_flag, P.status);
}

// ---------------------------------------------------------------- softmax warps
// Warps 0-7.  Warp w owns tensor-memory lanes 32*(w%4) .. +31, i.e. query rows
// i = 32*(w%4) + lane, and key half hf = w/4 of every tile (keys 64*hf ..
// 64*hf+63).  Each half keeps its own running maximum, sum and O accumulator
// (columns 256 + 128*hf): the two halves are two split-K partial states of
// the same rows, merged by the combine launch like any other pieces.  So the
// two warps of a row never exchange anything, and every SM sub-partition runs
// two softmax warps.
// Per piece: write this half of the query row into Q (128-byte swizzle; rows
// >= G*T zero).  Per tile: read the half's 64 logits, mask keys past the
// row's position (only in the tiles that reach past the first query's
// position), keep the running maximum (O rescaled in place only when it grows
// by more than 2^8: a warp-wide decision, since tensor-memory accesses are
// warp-wide), write P = 2^(x - max) as bf16 for the PV MMA.  At the piece's
// end: read O and write the half's partial state.
__device__ __forceinline__ float cc_ex2(float x) {  // 2^x (ex2.approx.ftz: 2^-inf = +0)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cc_softmax(const CorrParams& P, unsigned char* smem, int pbeg, int pend,
                                           uint32_t tmem) {
  constexpr unsigned FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3, hf = warp >> 2;
  const int i = quarter * 32 + lane;  // query row, tensor-memory lane
  CcBars br(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + CcCfg::OFF_FLAGS);
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const uint32_t tl_o = tl + 256 + hf * 128;  // this half's O accumulator
  const float sl2 = P.scale_log2;
  const bool live = i < P.rows;
  const int pos = P.n - P.T + (live ? i % P.T : 0);  // keys 0 .. pos are visible to this row
  const int pos_min = P.n - P.T;                      // the first query's position
  const bf16_t* qg = static_cast<const bf16_t*>(P.q);
  unsigned char* qbuf = smem + CcCfg::OFF_Q;
  unsigned char* pbuf = smem + CcCfg::OFF_P;
  int t = 0;
  for (int pc = pbeg; pc < pend; ++pc) {
    const CorrPiece piece = P.pieces[pc];
    {  // this piece's queries: row i is head g*G + i/T at position n - T + i%T
      const bf16_t* src =
          qg + (((static_cast<int64_t>(piece.l) * P.B + piece.b) * P.Hq + static_cast<int64_t>(piece.g) * P.G) *
                    P.T + i) * CcCfg::D;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const int ch = hf * 8 + c8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (live) v = *reinterpret_cast<const uint4*>(src + ch * 8);
        *reinterpret_cast<uint4*>(qbuf + cswz(i, ch)) = v;
      }
      tc::fence_async_smem();
      mbar_arrive(br.q_ready);
    }
    float m_used = -INFINITY, lsum = 0.f;
    const int ntile = piece.t1 - piece.t0;
    for (int u = 0; u < ntile; ++u, ++t) {
      const int b = t & 1;
      if (!mbar_wait(&br.s_ready[b], (t >> 1) & 1, abort_flag, P.status)) return;
      tc::fence_after_sync();
      uint32_t r[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::ld_32x32b_x16(tl + b * 128 + hf * 64 + c * 16, r[c]);
      tc::wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&br.s_free[b]);
      const int kb = (piece.t0 + u) * kCcRows + hf * 64;  // this half's first key
      float mraw = -INFINITY;
      if (live && kb + 63 <= pos_min) {  // every key of the half is visible to every row
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j) mraw = fmaxf(mraw, __uint_as_float(r[c][j]));
      } else {  // causal mask (key kb + x is visible if kb + x <= pos); rows >= G*T see nothing
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const bool vis = live && kb + c * 16 + j <= pos;
            const float x = vis ? __uint_as_float(r[c][j]) : -INFINITY;
            r[c][j] = __float_as_uint(x);
            mraw = fmaxf(mraw, x);
          }
      }
      const float mx = mraw * sl2;                       // sl2 > 0: the scaled maximum
      const bool grow = mx > m_used + 8.f;               // includes the first finite maximum
      const bool rescale = grow && m_used != -INFINITY;  // O already holds earlier tiles
      if (__any_sync(FULL, rescale)) {
        // O holds the tiles before this one: wait for the last PV, rescale in place
        if (!mbar_wait(&br.pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, P.status)) return;
        tc::fence_after_sync();
        const float sc = rescale ? cc_ex2(m_used - mx) : 1.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[16];
          tc::ld_32x32b_x16(tl_o + c * 16, o);
          tc::wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * sc);
          cc_st_x16(tl_o + c * 16, o);
        }
        cc_wait_st();
        lsum *= sc;
      }
      if (grow) m_used = mx;
      // p = 2^(x sl2 - m_used); a row with no visible key yet has m_used = -inf
      // and only masked (-inf) logits, which give 0
      const float mneg = m_used == -INFINITY ? 0.f : -m_used;
      // P buffer b was last read by the PV of tile t-2
      if (t >= 2 && !mbar_wait(&br.pv_done[b], ((t - 2) >> 1) & 1, abort_flag, P.status)) return;
      unsigned char* prow = pbuf + b * CcCfg::TILEB;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = cc_ex2(fmaf(__uint_as_float(r[c8 >> 1][(c8 & 1) * 8 + 2 * e]), sl2, mneg));
          const float p1 = cc_ex2(fmaf(__uint_as_float(r[c8 >> 1][(c8 & 1) * 8 + 2 * e + 1]), sl2, mneg));
          w[e] = cc_pack_bf16(p0, p1);
          lsum += p0 + p1;
        }
        *reinterpret_cast<uint4*>(prow + cswz(i, hf * 8 + c8)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&br.p_ready[b]);
    }
    // the half's O, once the PV of the piece's last tile is done
    const int tl_last = t - 1;
    if (!mbar_wait(&br.pv_done[tl_last & 1], (tl_last >> 1) & 1, abort_flag, P.status)) return;
    tc::fence_after_sync();
    const int64_t rec = 2 * static_cast<int64_t>(piece.part) + hf;  // this half's partial record
    float* dst = P.part_o + (rec * kCcRows + i) * CcCfg::D;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t o[16];
      tc::ld_32x32b_x16(tl_o + c * 16, o);
      tc::wait_ld();
      if (live)
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(dst + c * 16 + j) =
              make_float4(__uint_as_float(o[j]), __uint_as_float(o[j + 1]), __uint_as_float(o[j + 2]),
                          __uint_as_float(o[j + 3]));
    }
    if (live) P.part_ml[rec * kCcRows + i] = make_float2(m_used, lsum);
    tc::fence_before_sync();
    mbar_arrive(br.o_free);
  }
}

__global__ void __launch_bounds__(CcCfg::kThreads, 1)
    correction_tc_kernel(const __grid_constant__ CorrParams P) {
  using C = CcCfg;
  extern __shared__ unsigned char smem_raw[];
  // the 128-byte swizzle needs 1024-byte aligned tiles
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  uint32_t* flags = reinterpret_cast<uint32_t*>(smem + C::OFF_FLAGS);  // [0] abort, [1] tmem
  if (threadIdx.x == 0) {
    CcBars br(smem);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&br.kfull[s], 1);
      mbar_init(&br.vfull[s], 1);
      mbar_init(&br.kempty[s], 1);
      mbar_init(&br.vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&br.s_ready[b], 1);
      mbar_init(&br.s_free[b], C::kSoftThreads);
      mbar_init(&br.p_ready[b], C::kSoftThreads);
      mbar_init(&br.pv_done[b], 1);
    }
    mbar_init(br.q_ready, C::kSoftThreads);
    mbar_init(br.o_free, C::kSoftThreads);
    mbar_init(br.mma_idle, 1);
    flags[0] = 0u;
    fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    tc::tmem_alloc(flags + 1, C::kTmemCols);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == C::kLoadWarp * 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.tmv)) : "memory");
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = flags[1];
  const int pbeg = P.cta_begin[blockIdx.x];
  const int pend = P.cta_begin[blockIdx.x + 1];
  if (warp < 8) {
    cc_softmax(P, smem, pbeg, pend, tmem);
  } else if (warp == C::kMmaWarp) {
    cc_mma(P, smem, pbeg, pend, tmem);
  } else if ((threadIdx.x & 31) == 0) {
    cc_loads(P, smem, pbeg, pend);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == C::kMmaWarp) tc::tmem_dealloc(tmem, C::kTmemCols);
}

// One warp per (KV group, query row): the log-sum-exp merge of the group's
// partial records (two per piece) into the output.  Lane j owns columns
// 4j .. 4j+3.
__global__ void correction_combine_kernel(const CorrParams P) {
  const int warps = blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * warps + (threadIdx.x >> 5);
  const int64_t ngroups = static_cast<int64_t>(P.L) * P.B * P.Hkv;
  if (w >= ngroups * P.rows) return;
  const int grp = static_cast<int>(w / P.rows), i = static_cast<int>(w % P.rows);
  // two partial records (key halves) per piece
  const int f = 2 * P.group_first[grp], e = 2 * P.group_first[grp + 1];
  float M = -INFINITY;
  for (int pc = f; pc < e; ++pc) M = fmaxf(M, P.part_ml[static_cast<int64_t>(pc) * kCcRows + i].x);
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int pc = f; pc < e; ++pc) {
    const float2 ml = P.part_ml[static_cast<int64_t>(pc) * kCcRows + i];
    if (ml.x == -INFINITY) continue;
    const float a = exp2f(ml.x - M);
    L += ml.y * a;
    const float4 o = *reinterpret_cast<const float4*>(
        P.part_o + (static_cast<int64_t>(pc) * kCcRows + i) * CcCfg::D + 4 * lane);
    acc.x += o.x * a;
    acc.y += o.y * a;
    acc.z += o.z * a;
    acc.w += o.w * a;
  }
  if (!(L > 0.f)) {
    if (lane == 0) atomicOr(P.status, kStatusEmptySoftmax);
    L = 1.f;
  }
  const float inv = 1.f / L;
  const int g = grp % P.Hkv;
  const int lb = grp / P.Hkv;  // l * B + b
  const int h = g * P.G + i / P.T, tq = i % P.T;
  *reinterpret_cast<float4*>(P.out + ((static_cast<int64_t>(lb) * P.Hq + h) * P.T + tq) * CcCfg::D + 4 * lane) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// The refreshed rows: one block per (l, b, g, t), 16-byte chunks of the K
// row, then of the V row.
__global__ void write_rows_kernel(const WriteRowsParams p) {
  const int64_t x = blockIdx.x;
  const int t = static_cast<int>(x % p.T);
  const int g = static_cast<int>((x / p.T) % p.Hkv);
  const int b = static_cast<int>((x / (static_cast<int64_t>(p.T) * p.Hkv)) % p.B);
  const int l = static_cast<int>(x / (static_cast<int64_t>(p.T) * p.Hkv * p.B));
  const int64_t row = p.n - p.T + t;
  const int64_t dst = (l * p.s_layer + b * p.s_batch + g * p.s_head + row * p.s_token) * p.elem_bytes;
  const int64_t src = x * p.row_bytes;
  for (int c = threadIdx.x; c < p.row_bytes / 16; c += blockDim.x) {
    *reinterpret_cast<uint4*>(p.k + dst + 16 * c) = *reinterpret_cast<const uint4*>(p.k_new + src + 16 * c);
    *reinterpret_cast<uint4*>(p.v + dst + 16 * c) = *reinterpret_cast<const uint4*>(p.v_new + src + 16 * c);
  }
}

}  // namespace

int correction_smem_bytes() { return CcCfg::SMEM; }

cudaError_t correction_configure() {
  return cudaFuncSetAttribute(correction_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CcCfg::SMEM);
}

cudaError_t correction_launch(const CorrParams* P, int grid, const WriteRowsParams* rows, cudaStream_t stream) {
  if (rows) {
    const int64_t nrow = static_cast<int64_t>(rows->L) * rows->B * rows->Hkv * rows->T;
    write_rows_kernel<<<static_cast<unsigned>(nrow), 32, 0, stream>>>(*rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  correction_tc_kernel<<<grid, CcCfg::kThreads, CcCfg::SMEM, stream>>>(*P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t warps = static_cast<int64_t>(P->L) * P->B * P->Hkv * P->rows;
  correction_combine_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(*P);
  return cudaGetLastError();
}

}  // namespace lyc
