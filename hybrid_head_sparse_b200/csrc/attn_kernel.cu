// attn_kernel.cu -- pooled hybrid-head decode attention for one layer, fp32
// inputs (CUDA-core path; bf16 inputs use attn_mma_kernel.cu).
//
// Computes, for every segment of the layer's work pool (see lyc_plan.h):
//   retrieval heads, page "LycheeDecode ..." (paper-graph-ui summary),
//   section 3.4 Eq. (1):  o = softmax(q K^T / sqrt(d)) V over all n rows,
//   sparse heads, section 3.4 Eq. (3): the same over the rows of the
//   inherited set, and writes the selection key of every row for the heads
//   (or group mean queries) whose set is refreshed (Eq. 2 runs afterwards in
//   topk_kernel.cu).  Partial softmax states of a segment's pieces are
//   merged with log-sum-exp by the last piece to finish (Appendix C,
//   Algorithm 2 steps 5-6, done here without a second launch).
//
// Design (B200 / sm_100a):
//   * one producer warp per CTA streams 64-row K and V tiles into a
//     STAGES-deep shared-memory ring with bulk (TMA) copies: one 16 KiB copy
//     per tile for a contiguous dense range, one 256-byte copy per row for a
//     gathered (sparse) tile, whose indices arrive ahead in their own small
//     ring, also by bulk copy;
//   * eight consumer warps each own 8 rows of every tile: q.K with fp32
//     FMAs on CUDA cores (decode is bandwidth bound: ~1-4 flop per byte),
//     an online softmax per warp in log2 units, and P.V with each lane
//     owning d/32 output columns;
//   * row-major tiles are read conflict-free without swizzling: each lane
//     reads a quarter of a row, visiting its 16-byte chunks in a rotated
//     order so that the 8 lanes of a quarter-warp always hit 8 different
//     bank groups.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "lyc_device.cuh"
#include "lyc_plan.h"

namespace lyc {

typedef uint16_t bf16_t;  // bf16 bit pattern

template <typename T>
__device__ __forceinline__ float load_elem(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_elem<bf16_t>(const bf16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}
template <>
__device__ __forceinline__ float load_elem<float>(const float* p, int64_t i) {
  return p[i];
}

// 16 bytes of shared memory -> 16 / sizeof(T) floats
template <typename T>
__device__ __forceinline__ void load_chunk(const unsigned char* s, float* v);
template <>
__device__ __forceinline__ void load_chunk<bf16_t>(const unsigned char* s, float* v) {
  const uint4 w = *reinterpret_cast<const uint4*>(s);
  v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
  v[4] = bf16lo(w.z); v[5] = bf16hi(w.z); v[6] = bf16lo(w.w); v[7] = bf16hi(w.w);
}
template <>
__device__ __forceinline__ void load_chunk<float>(const unsigned char* s, float* v) {
  const float4 w = *reinterpret_cast<const float4*>(s);
  v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
}

// VE consecutive elements of a V row -> floats
template <typename T, int VE>
__device__ __forceinline__ void load_vslice(const unsigned char* s, float* v) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (VE == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(s);
      v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(s);
      v[0] = bf16lo(w); v[1] = bf16hi(w);
    }
  } else {
    if constexpr (VE == 4) {
      const float4 w = *reinterpret_cast<const float4*>(s);
      v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
    } else {
      const float2 w = *reinterpret_cast<const float2*>(s);
      v[0] = w.x; v[1] = w.y;
    }
  }
}

template <typename T, int D, int NQ, int STAGES>
struct AttnCfg {
  static constexpr int kConsumerWarps = 8;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  static constexpr int ROWB = D * (int)sizeof(T);         // bytes per K/V row
  static constexpr int TILEB = kTileRows * ROWB;          // bytes per K (or V) tile
  static constexpr int CQ = ROWB / 64;                    // 16-byte chunks per quarter row
  static constexpr int EPC = 16 / (int)sizeof(T);         // elements per chunk
  static constexpr int QE = D / 4;                        // elements per quarter
  static constexpr int QPAD = QE + 4;                     // padded quarter (floats)
  static constexpr int VE = D / 32;                       // output columns per lane
  static constexpr int IR = 8;                            // index ring slots
  static constexpr int LA = IR - 1;                       // index lookahead (tiles)
  // shared memory layout (bytes)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + STAGES * TILEB;
  static constexpr int OFF_IDX = OFF_V + STAGES * TILEB;
  static constexpr int OFF_Q = OFF_IDX + IR * kTileRows * 4;
  static constexpr int OFF_P = OFF_Q + NQ * 4 * QPAD * 4;
  static constexpr int OFF_MO = OFF_P + kConsumerWarps * NQ * 8 * 4;
  static constexpr int OFF_MML = OFF_MO + kConsumerWarps * NQ * D * 4;
  static constexpr int OFF_BAR = OFF_MML + kConsumerWarps * NQ * 8;
  static constexpr int OFF_MASK = OFF_BAR + (2 * STAGES + IR) * 8;
  static constexpr int OFF_FLAGS = OFF_MASK + STAGES * 8;
  static constexpr int SMEM = OFF_FLAGS + (NQ + 2) * 4;
};

}  // namespace lyc

namespace lyc {

// ---------------------------------------------------------------- producer
template <typename T, int D, int NQ, int STAGES>
__device__ __forceinline__ void attn_producer(const AttnParams& p, unsigned char* smem, int pbeg,
                                              int pend) {
  using C = AttnCfg<T, D, NQ, STAGES>;
  const int lane = threadIdx.x & 31;
  unsigned char* Ks = smem + C::OFF_K;
  unsigned char* Vs = smem + C::OFF_V;
  int32_t* idxring = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* idxbar = bars + 2 * STAGES;
  uint64_t* rowmask = reinterpret_cast<uint64_t*>(smem + C::OFF_MASK);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  const uint64_t pol = l2_policy_evict_first();

  // Lookahead cursor: issues the index-list copy of sparse tiles LA tiles
  // before the main cursor needs them.
  int la_pc = pbeg, la_r0 = (pbeg < pend) ? p.pieces[pbeg].r0 : 0, la_t = 0;
  bool waited = false;  // the previous layer's selection has completed
  auto la_step = [&]() {
    if (la_pc >= pend) return;
    const Piece pc = p.pieces[la_pc];
    const Segment& sg = p.segs[pc.seg];
    if (sg.kind == kSparse && lane == 0) {
      if (!waited) {  // the inherited sets are that kernel's output
        pdl_wait();
        waited = true;
      }
      const int slot = la_t % C::IR;
      const int nrows = min(kTileRows, pc.r1 - la_r0);
      const uint32_t bytes = static_cast<uint32_t>(((nrows * 4) + 15) & ~15);
      fence_proxy_async_smem();  // earlier reads of this slot precede the new copy
      mbar_arrive_expect_tx(&idxbar[slot], bytes);
      bulk_g2s(idxring + slot * kTileRows, sg.idx + la_r0, bytes, &idxbar[slot]);
    }
    ++la_t;
    la_r0 += kTileRows;
    if (la_r0 >= pc.r1) {
      ++la_pc;
      if (la_pc < pend) la_r0 = p.pieces[la_pc].r0;
    }
  };
  for (int a = 0; a < C::LA; ++a) la_step();

  uint32_t idx_phase = 0;  // per ring slot: parity of its next completion
  int t = 0;
  for (int pcI = pbeg; pcI < pend; ++pcI) {
    const Piece pc = p.pieces[pcI];
    const Segment& sg = p.segs[pc.seg];
    const int kind = sg.kind;
    const int64_t s_token = sg.s_token;
    const T* kb = static_cast<const T*>(sg.k);
    const T* vb = static_cast<const T*>(sg.v);
    const bool contiguous = (kind == kDense) && (s_token == D);
    for (int r0 = pc.r0; r0 < pc.r1; r0 += kTileRows, ++t) {
      la_step();
      const int nrows = min(kTileRows, pc.r1 - r0);
      const int stage = t % STAGES;
      if (t >= STAGES) {
        if (!mbar_wait(&empty[stage], ((t / STAGES) - 1) & 1, abort_flag, p.status)) return;
      }
      unsigned char* kdst = Ks + stage * C::TILEB;
      unsigned char* vdst = Vs + stage * C::TILEB;
      if (contiguous) {
        if (lane == 0) {
          rowmask[stage] = (nrows == 64) ? ~0ull : ((1ull << nrows) - 1ull);
          const uint32_t bytes = static_cast<uint32_t>(nrows * C::ROWB);
          mbar_arrive_expect_tx(&full[stage], 2u * bytes);
          bulk_g2s_stream(kdst, kb + static_cast<int64_t>(r0) * D, bytes, &full[stage], pol);
          bulk_g2s_stream(vdst, vb + static_cast<int64_t>(r0) * D, bytes, &full[stage], pol);
        }
      } else {
        int64_t ia, ib;
        if (kind == kSparse) {
          const int slot = t % C::IR;
          if (!mbar_wait(&idxbar[slot], (idx_phase >> slot) & 1u, abort_flag, p.status)) return;
          idx_phase ^= 1u << slot;
          const int32_t* ring = idxring + slot * kTileRows;
          ia = (lane < nrows) ? ring[lane] : -1;
          ib = (lane + 32 < nrows) ? ring[lane + 32] : -1;
        } else {
          ia = r0 + lane;
          ib = r0 + lane + 32;
        }
        const bool va = lane < nrows && ia >= 0 && ia < sg.nvalid;
        const bool vb2 = lane + 32 < nrows && ib >= 0 && ib < sg.nvalid;
        if ((lane < nrows && index_bad(ia, sg.nvalid, sg.pad_ok)) ||
            (lane + 32 < nrows && index_bad(ib, sg.nvalid, sg.pad_ok)))
          atomicOr(p.status, kStatusBadIndex);
        const uint32_t ma = __ballot_sync(0xffffffffu, va);
        const uint32_t mb = __ballot_sync(0xffffffffu, vb2);
        if (lane == 0) {
          rowmask[stage] = static_cast<uint64_t>(ma) | (static_cast<uint64_t>(mb) << 32);
          const uint32_t nvalid = __popc(ma) + __popc(mb);
          mbar_arrive_expect_tx(&full[stage], nvalid * 2u * C::ROWB);
        }
        __syncwarp();
        if (va) {
          bulk_g2s(kdst + lane * C::ROWB, kb + ia * s_token, C::ROWB, &full[stage]);
          bulk_g2s(vdst + lane * C::ROWB, vb + ia * s_token, C::ROWB, &full[stage]);
        }
        if (vb2) {
          bulk_g2s(kdst + (lane + 32) * C::ROWB, kb + ib * s_token, C::ROWB, &full[stage]);
          bulk_g2s(vdst + (lane + 32) * C::ROWB, vb + ib * s_token, C::ROWB, &full[stage]);
        }
      }
    }
  }
}

}  // namespace lyc

namespace lyc {

// ---------------------------------------------------------------- consumers
template <typename T, int D, int NQ, int STAGES>
__device__ __forceinline__ void attn_consumers(const AttnParams& p, unsigned char* smem, int pbeg,
                                               int pend) {
  using C = AttnCfg<T, D, NQ, STAGES>;
  constexpr unsigned FULL = 0xffffffffu;
  const int tid = threadIdx.x;  // 0..255
  const int w = tid >> 5;
  const int lane = tid & 31;
  // lane -> (row i of the warp's 8, quarter c of the row); see the file header
  const int i = (lane & 3) | (((lane >> 3) & 1) << 2);
  const int c = ((lane >> 2) & 1) | (((lane >> 4) & 1) << 1);
  const unsigned char* Ks = smem + C::OFF_K;
  const unsigned char* Vs = smem + C::OFF_V;
  float* qs = reinterpret_cast<float*>(smem + C::OFF_Q);
  float* pb = reinterpret_cast<float*>(smem + C::OFF_P) + w * NQ * 8;
  float* mo = reinterpret_cast<float*>(smem + C::OFF_MO);
  float2* mml = reinterpret_cast<float2*>(smem + C::OFF_MML);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  const uint64_t* rowmask = reinterpret_cast<const uint64_t*>(smem + C::OFF_MASK);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  int* lastflag = reinterpret_cast<int*>(smem + C::OFF_FLAGS) + 1;
  const T* q = static_cast<const T*>(p.q);

  int t = 0;
  for (int pcI = pbeg; pcI < pend; ++pcI) {
    const Piece pc = p.pieces[pcI];
    const Segment& sg = p.segs[pc.seg];
    const int nq = sg.nq;
    const int nout = sg.nout;
    const int b = sg.b;
    const bool dense = sg.kind == kDense;
    uint32_t outmask = 0;
    for (int o = 0; o < nout; ++o) outmask |= 1u << sg.out_row[o];
    const int64_t key_mean_off = sg.key_mean_off;

    // ---- query vectors of this segment -> shared memory (fp32, padded quarters)
    named_bar_sync(1, 256);  // previous piece is done with qs / merge area
    for (int x = tid; x < nq * D; x += 256) {
      const int j = x / D, e = x % D;
      const float val = load_elem<T>(q, (static_cast<int64_t>(b) * p.Hq + sg.head[j]) * D + e);
      qs[(j * 4 + e / C::QE) * C::QPAD + (e % C::QE)] = val;
    }
    named_bar_sync(1, 256);

    float m_run[NQ], l_lane[NQ], o[NQ][C::VE];
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      m_run[j] = -INFINITY;
      l_lane[j] = 0.f;
#pragma unroll
      for (int e = 0; e < C::VE; ++e) o[j][e] = 0.f;
    }

    for (int r0 = pc.r0; r0 < pc.r1; r0 += kTileRows, ++t) {
      const int stage = t % STAGES;
      mbar_wait(&full[stage], (t / STAGES) & 1, abort_flag, p.status);
      const uint64_t mask = rowmask[stage];
      const unsigned char* Kt = Ks + stage * C::TILEB;
      const unsigned char* Vt = Vs + stage * C::TILEB;
      const int row = w * 8 + i;
      const bool valid = (mask >> row) & 1ull;

      // ---- logits: lane (i, c) sums a quarter row, then the 4 quarters combine
      float acc[NQ];
#pragma unroll
      for (int j = 0; j < NQ; ++j) acc[j] = 0.f;
      const unsigned char* krow = Kt + row * C::ROWB;
#pragma unroll
      for (int m = 0; m < C::CQ; ++m) {
        const int cc = (m + i) & (C::CQ - 1);
        float kv[C::EPC];
        load_chunk<T>(krow + (c * C::CQ + cc) * 16, kv);
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
          if (j < nq) {
            const float* qp = qs + (j * 4 + c) * C::QPAD + cc * C::EPC;
#pragma unroll
            for (int u = 0; u < C::EPC; u += 4) {
              const float4 qv = *reinterpret_cast<const float4*>(qp + u);
              acc[j] = fmaf(qv.x, kv[u + 0], acc[j]);
              acc[j] = fmaf(qv.y, kv[u + 1], acc[j]);
              acc[j] = fmaf(qv.z, kv[u + 2], acc[j]);
              acc[j] = fmaf(qv.w, kv[u + 3], acc[j]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        if (j < nq) {
          acc[j] += __shfl_xor_sync(FULL, acc[j], 4);
          acc[j] += __shfl_xor_sync(FULL, acc[j], 16);
        }
      }

      // ---- selection keys, online softmax (log2 units), probabilities -> smem
      if (dense && c == 0 && valid && key_mean_off >= 0) {
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < NQ; ++j)
          if (j < nq) sum += acc[j];
        p.keys[key_mean_off + r0 + row] = sum / static_cast<float>(nq) * p.scale;
      }
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        if (j < nq) {
          if (dense && c == 0 && valid && sg.key_off[j] >= 0)
            p.keys[sg.key_off[j] + r0 + row] = acc[j] * p.scale;
          if ((outmask >> j) & 1u) {
            const float tj = valid ? acc[j] * p.scale_log2 : -INFINITY;
            float mx = fmaxf(tj, __shfl_xor_sync(FULL, tj, 1));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
            const float mnew = fmaxf(m_run[j], mx);
            float pj = 0.f, sc = 1.f;
            if (mnew != -INFINITY) {
              sc = exp2f(m_run[j] - mnew);  // 0 when m_run is -inf
              pj = valid ? exp2f(tj - mnew) : 0.f;
            }
            m_run[j] = mnew;
            l_lane[j] = l_lane[j] * sc + (c == 0 ? pj : 0.f);
#pragma unroll
            for (int e = 0; e < C::VE; ++e) o[j][e] *= sc;
            if (c == 0) pb[j * 8 + i] = pj;
          }
        }
      }
      __syncwarp();

      // ---- P.V: lane owns output columns [lane*VE, lane*VE + VE)
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if ((mask >> (w * 8 + r)) & 1ull) {
          float v[C::VE];
          load_vslice<T, C::VE>(Vt + (w * 8 + r) * C::ROWB + lane * C::VE * (int)sizeof(T), v);
#pragma unroll
          for (int j = 0; j < NQ; ++j) {
            if ((outmask >> j) & 1u) {
              const float pj = pb[j * 8 + r];
#pragma unroll
              for (int e = 0; e < C::VE; ++e) o[j][e] = fmaf(pj, v[e], o[j][e]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }

    // ---- merge the 8 warps' states of this piece into one partial record
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      if ((outmask >> j) & 1u) {
        float l = l_lane[j];
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) l += __shfl_xor_sync(FULL, l, s);
        if (lane == 0) mml[w * NQ + j] = make_float2(m_run[j], l);
#pragma unroll
        for (int e = 0; e < C::VE; ++e) mo[(w * NQ + j) * D + lane * C::VE + e] = o[j][e];
      }
    }
    named_bar_sync(1, 256);
    for (int x = tid; x < nout * D; x += 256) {
      const int o = x / D, e = x % D;
      const int j = sg.out_row[o];
      float M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) M = fmaxf(M, mml[ww * NQ + j].x);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) {
          const float2 ml = mml[ww * NQ + j];
          const float f = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
          L = fmaf(f, ml.y, L);
          O = fmaf(f, mo[(ww * NQ + j) * D + e], O);
        }
      }
      const int part = sg.part_base + pc.ordinal * nout + o;
      p.part_o[static_cast<int64_t>(part) * D + e] = O;
      if (e == 0) p.part_ml[part] = make_float2(M, L);
    }
    __threadfence();
    named_bar_sync(1, 256);
    if (tid == 0) {
      for (int j = 0; j < nout; ++j) {
        const int old = atomicAdd(&p.counters[sg.cnt_base + j], 1);
        lastflag[j] = (old == sg.npieces - 1);
      }
      __threadfence();
    }
    named_bar_sync(1, 256);

    // ---- the last piece of the segment combines every piece (log-sum-exp)
    for (int o = 0; o < nout; ++o) {
      if (!lastflag[o]) continue;
      const int base = sg.part_base + o;
      const int np = sg.npieces;
      for (int e = tid; e < D; e += 256) {
        float M = -INFINITY;
        for (int u = 0; u < np; ++u) M = fmaxf(M, __ldcg(&p.part_ml[base + u * nout]).x);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
          for (int u = 0; u < np; ++u) {
            const float2 ml = __ldcg(&p.part_ml[base + u * nout]);
            const float f = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
            L = fmaf(f, ml.y, L);
            O = fmaf(f, __ldcg(&p.part_o[static_cast<int64_t>(base + u * nout) * D + e]), O);
          }
        }
        float res = 0.f;
        if (L > 0.f) {
          res = O / L;
        } else if (e == 0) {
          atomicOr(p.status, kStatusEmptySoftmax);
        }
        p.out[(static_cast<int64_t>(b) * p.Hq + sg.head[sg.out_row[o]]) * D + e] = res;
      }
      if (tid == 0) p.counters[sg.cnt_base + o] = 0;
    }
  }
}

// ---------------------------------------------------------------- kernel
template <typename T, int D, int NQ, int STAGES>
__global__ void __launch_bounds__(AttnCfg<T, D, NQ, STAGES>::kThreads, 1)
    attn_layer_kernel(const AttnParams p) {
  using C = AttnCfg<T, D, NQ, STAGES>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars[s], 1);                           // full: producer arrival + bytes
      mbar_init(&bars[STAGES + s], C::kConsumerWarps);  // empty: one arrival per warp
    }
    for (int r = 0; r < C::IR; ++r) mbar_init(&bars[2 * STAGES + r], 1);
    *reinterpret_cast<int*>(smem + C::OFF_FLAGS) = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  if (p.wait_prev) pdl_wait();  // the previous launch writes what this one reads or writes
  const int pbeg = p.cta_begin[blockIdx.x];
  const int pend = p.cta_begin[blockIdx.x + 1];
  if (threadIdx.x >= C::kConsumerWarps * 32) {
    attn_producer<T, D, NQ, STAGES>(p, smem, pbeg, pend);
  } else {
    attn_consumers<T, D, NQ, STAGES>(p, smem, pbeg, pend);
  }
  if (threadIdx.x == 0) pdl_wait();  // complete only after the grid this one depends on
}

}  // namespace lyc

namespace lyc {

// ---------------------------------------------------------------- host side
template <typename T, int D>
constexpr int attn_stages() {
  // about 128 KiB of K/V tiles in flight per CTA (one CTA per SM)
  constexpr int per_stage = 2 * kTileRows * D * (int)sizeof(T);
  constexpr int s = (128 * 1024) / per_stage;
  return s > 6 ? 6 : (s < 2 ? 2 : s);
}

template <typename T, int D, int NQ>
static cudaError_t attn_run(const AttnParams* p, int grid, cudaStream_t stream, int* smem_out,
                            bool configure_only) {
  constexpr int S = attn_stages<T, D>();
  using C = AttnCfg<T, D, NQ, S>;
  auto kern = attn_layer_kernel<T, D, NQ, S>;
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
  return cudaLaunchKernelEx(&cfg, kern, *p);
}

template <typename T, int D>
static cudaError_t attn_by_nq(int nqb, const AttnParams* p, int grid, cudaStream_t stream,
                              int* smem_out, bool configure_only) {
  switch (nqb) {
    case 1: return attn_run<T, D, 1>(p, grid, stream, smem_out, configure_only);
    case 2: return attn_run<T, D, 2>(p, grid, stream, smem_out, configure_only);
    case 4: return attn_run<T, D, 4>(p, grid, stream, smem_out, configure_only);
    case 8: return attn_run<T, D, 8>(p, grid, stream, smem_out, configure_only);
    default: return cudaErrorInvalidValue;
  }
}

// Smallest compiled query-row count >= nq (both attention kernels).
int attn_nq_bucket(int nq) {
  if (nq <= 1) return 1;
  if (nq <= 2) return 2;
  if (nq <= 4) return 4;
  return 8;
}

// fp32 inputs (CUDA-core kernel).  configure_only: set the kernel's
// shared-memory attribute and report its size, launch nothing.
cudaError_t attn_simt_dispatch(int D, int nqb, const AttnParams* p, int grid, cudaStream_t stream,
                               int* smem_out, bool configure_only) {
  if (D == 64) return attn_by_nq<float, 64>(nqb, p, grid, stream, smem_out, configure_only);
  if (D == 128) return attn_by_nq<float, 128>(nqb, p, grid, stream, smem_out, configure_only);
  return cudaErrorInvalidValue;
}

}  // namespace lyc
