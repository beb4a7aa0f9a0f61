// topk_kernel.cu -- exact argsTopK over one row of selection keys per task.
//
// What it computes (page "LycheeDecode ...", paper-graph-ui summary,
// section 3.4 Eq. 2): S = the k_eff = min(k, n) indices with the largest
// keys, ties to the lower index (-0 == +0), written in ascending index
// order, positions k_eff..k-1 set to -1.
//
// Design (B200 / sm_100a): radix select of tau, the k_eff-th largest key, on
// order-preserving 32-bit encodings (digits of 11, 11 and 10 bits), then one
// stable compaction.  One thread-block cluster of CL CTAs per task; each CTA
// owns a contiguous chunk of the keys, loaded once into shared memory.
// Three cluster barriers in the common case:
//   (1) after every CTA zeroed its totals and histogrammed its chunk's top
//       digit with shared-memory atomics;
//   (2) after every CTA added its non-zero bins into every CTA's totals through
//       distributed shared memory (the adds are spread over all threads); each
//       CTA then finds the top digit of tau by itself;
//   (3) after every CTA copied its candidates (keys whose top digit is tau's,
//       a few per cent of the keys), in index order, into every CTA, with its
//       count of keys above that digit.
// Each CTA then finds tau among the candidates, the per-CTA counts of keys
// > tau and == tau, hence its output offset and how many of its ties (lowest
// indices first) it takes, and writes its indices with warp ballots.  If the
// candidates do not fit (heavily tied keys), two more radix digits run over
// the chunks with totals pushed into every CTA, and the CTA counts are
// exchanged instead.
//
// Selection rules other than a fixed k (page "LycheeDecode ...", section
// 4.4.1, Figure 6, Tables 5-6): the number of keys to select is found first,
// then the same selection runs with it.
//  * top-p (the fewest largest keys whose probabilities reach p) and
//    threshold (the keys of probability >= tau): the cluster's maximum key M
//    is exchanged first; every key gets the weight W = round(2^40 exp(x - M))
//    (an integer: sums are exact whatever their order, so every CTA takes the
//    same decision).  Threshold counts W >= ceil(tau * sum W).  Top-p finds
//    the key value at which the running mass, larger keys first, reaches
//    T = ceil(p * sum W): a radix descent on the same digits as the
//    selection, with per-digit counts and masses pushed into every CTA
//    (one more cluster barrier per digit; lanes of a warp that share a bin
//    add once), then how many of the keys equal to that value it takes;
//  * block selection: each CTA scores the blocks of its chunk from the key
//    rows as it loads them (log(sum exp(key)) over the block's rows, which
//    orders blocks by their summed probability), selects among the blocks,
//    and writes each selected block out as its rows.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lyc_device.cuh"
#include "lyc_plan.h"

namespace cg = cooperative_groups;

namespace lyc {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkCandCap = 4096;  // pivot-digit candidates gathered from the whole cluster
constexpr int kTopkSelCap = 4096;   // one CTA's keys at or above the pivot digit
// words of the size-rule exchange area: vx[16], vcnt[16] (u32), then 40 u64
constexpr int kTopkRuleWords = 32 + 80;

// The fp32 key an order-preserving encoding stands for (-0 comes back as +0).
__device__ __forceinline__ float key_from_order(uint32_t u) {
  const uint32_t b = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
  return __uint_as_float(b);
}

// 40-bit fixed-point weight of a key relative to the maximum M (x <= M):
// round(2^40 exp(x - M)), at most 2^40.
__device__ __forceinline__ unsigned long long key_weight(uint32_t u, float M) {
  return __float2ull_rn(expf(key_from_order(u) - M) * 1099511627776.0f);
}

// 64-bit add into shared or distributed shared memory as two 32-bit atomic
// adds, the low word's carry passed on to the high word: the exact sum once
// every add has landed, without 64-bit atomics.
__device__ __forceinline__ void atomic_add_u64_split(unsigned long long* a, unsigned long long v) {
  uint32_t* w = reinterpret_cast<uint32_t*>(a);
  const uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
  const uint32_t old = atomicAdd(w, lo);
  const uint32_t up = hi + (old + lo < old ? 1u : 0u);
  if (up) atomicAdd(w + 1, up);
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, s));
  return v;
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// Exclusive prefix sum of one value per warp (lane 0's) over the CTA; also the total.
__device__ __forceinline__ void cta_warp_scan(uint32_t* scratch, uint32_t mine, int warp, int lane,
                                              uint32_t* prefix, uint32_t* total) {
  if (lane == 0) scratch[warp] = mine;
  __syncthreads();
  uint32_t acc = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) {
    const uint32_t v = scratch[w];
    acc += (w < warp) ? v : 0u;
    tot += v;
  }
  *prefix = acc;
  *total = tot;
  __syncthreads();
}

// Find the digit d with  sum(hist[> d]) < krem <= sum(hist[>= d]).  Every
// thread returns the same (digit, count above it).  hist has kKeyBins entries
// (shared or global memory).
__device__ __forceinline__ void find_digit(const uint32_t* hist, uint32_t krem, uint32_t* scratch,
                                           uint32_t* found, int tid, int lane, int warp,
                                           uint32_t* digit, uint32_t* above_out) {
  constexpr int per = kKeyBins / kTopkThreads;
  uint32_t c[per];
  uint32_t mine = 0u;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = hist[tid * per + q];
    mine += c[q];
  }
  uint32_t suf = mine;  // inclusive suffix sum within the warp
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, s);
    if (lane + s < 32) suf += v;
  }
  if (lane == 0) scratch[warp] = suf;
  __syncthreads();
  uint32_t above = suf - mine;
  for (int w2 = warp + 1; w2 < kTopkWarps; ++w2) above += scratch[w2];
#pragma unroll
  for (int q = per - 1; q >= 0; --q) {
    if (above < krem && above + c[q] >= krem) {
      found[0] = static_cast<uint32_t>(tid * per + q);
      found[1] = above;
    }
    above += c[q];
  }
  __syncthreads();
  *digit = found[0];
  *above_out = found[1];
  __syncthreads();
}

// Find the digit d with  mass(> d) < target <= mass(>= d)  over NB bins of
// (count, mass); every thread returns the same digit and the count and mass
// of the bins above it.  Integer sums: the same in every CTA.
template <int NB>
__device__ __forceinline__ void find_digit_mass(const unsigned long long* mass, const uint32_t* cntb,
                                                unsigned long long target, unsigned long long* scr64,
                                                uint32_t* scr32, unsigned long long* res, int tid,
                                                int lane, int warp, uint32_t* digit, uint32_t* cabove,
                                                unsigned long long* mabove) {
  constexpr int per = NB >= kTopkThreads ? NB / kTopkThreads : 1;  // bins per thread
  unsigned long long m[per];
  uint32_t c[per];
  unsigned long long mm = 0ull;
  uint32_t mc = 0u;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    const bool in = tid * per + q < NB;
    m[q] = in ? mass[tid * per + q] : 0ull;
    c[q] = in ? cntb[tid * per + q] : 0u;
    mm += m[q];
    mc += c[q];
  }
  unsigned long long sm = mm;  // inclusive suffix sums within the warp
  uint32_t sc = mc;
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const unsigned long long vm = __shfl_down_sync(0xffffffffu, sm, s);
    const uint32_t vc = __shfl_down_sync(0xffffffffu, sc, s);
    if (lane + s < 32) {
      sm += vm;
      sc += vc;
    }
  }
  if (lane == 0) {
    scr64[warp] = sm;
    scr32[warp] = sc;
  }
  __syncthreads();
  unsigned long long am = sm - mm;
  uint32_t ac = sc - mc;
  for (int w2 = warp + 1; w2 < kTopkWarps; ++w2) {
    am += scr64[w2];
    ac += scr32[w2];
  }
#pragma unroll
  for (int q = per - 1; q >= 0; --q) {
    if (am < target && am + m[q] >= target) {
      res[0] = static_cast<unsigned long long>(tid * per + q);
      res[1] = ac;
      res[2] = am;
    }
    am += m[q];
    ac += c[q];
  }
  __syncthreads();
  *digit = static_cast<uint32_t>(res[0]);
  *cabove = static_cast<uint32_t>(res[1]);
  *mabove = res[2];
  __syncthreads();
}

}  // namespace lyc

namespace lyc {

// Lists the non-zero bins of hist[kKeyBins] as (bin, count) pairs in `out`
// (bin order) and returns how many there are.
__device__ __forceinline__ uint32_t compact_nonzero(const uint32_t* hist, uint2* out,
                                                    uint32_t* scratch, int tid, int lane, int warp) {
  constexpr int per = kKeyBins / kTopkThreads;
  uint32_t c[per];
  uint32_t mine = 0u;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = hist[tid * per + q];
    mine += c[q] != 0u;
  }
  uint32_t inc = mine;  // inclusive prefix within the warp
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, s);
    if (lane >= s) inc += v;
  }
  uint32_t before, total;
  cta_warp_scan(scratch, __shfl_sync(0xffffffffu, inc, 31), warp, lane, &before, &total);
  uint32_t pos = before + inc - mine;
#pragma unroll
  for (int q = 0; q < per; ++q)
    if (c[q]) out[pos++] = make_uint2(static_cast<uint32_t>(tid * per + q), c[q]);
  __syncthreads();
  return total;
}

// CTA-local radix select over the gathered candidates (source r's entries
// at cand[r*rcap .. r*rcap + cnt[r]), all sharing the digits in `prefix`):
// returns the krem-th largest encoded key; *krem becomes the number of
// candidates equal to it that are to be taken.
template <int CL>
__device__ __forceinline__ uint32_t select_in_candidates(const uint2* cand, const uint32_t* cnt,
                                                         int rcap, uint32_t prefix, uint32_t pmask,
                                                         uint32_t* krem, uint32_t* hist,
                                                         uint32_t* scratch, uint32_t* found, int tid,
                                                         int lane, int warp) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int sh = pass == 0 ? 10 : 0;
    const uint32_t dmask = pass == 0 ? 0x7ffu : 0x3ffu;
    for (int b = tid; b < kKeyBins; b += kTopkThreads) hist[b] = 0u;
    __syncthreads();
    for (int x = tid; x < CL * rcap; x += kTopkThreads) {
      if (static_cast<uint32_t>(x % rcap) < cnt[x / rcap]) {
        const uint32_t u = cand[x].x;
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> sh) & dmask], 1u);
      }
    }
    __syncthreads();
    uint32_t dg, ab;
    find_digit(hist, *krem, scratch, found, tid, lane, warp, &dg, &ab);
    *krem -= ab;
    prefix |= dg << sh;
    pmask |= dmask << sh;
  }
  return prefix;
}

// Every CTA of a task calls this once its writes of S are issued: the last of
// the CL to arrive resets the arrival counter and raises the task's ready
// flag to the step's epoch + 1.  Release: the CTA barrier orders every
// thread's writes before thread 0's device-scope fence, which precedes its
// arrival; the last arrival fences again before the flag store.  (One fence
// per CTA: a fence in every thread stalls the whole CTA on memory barriers.)
template <int CL>
__device__ __forceinline__ void topk_signal_done(const TopkParams& p, const TopkTask& task, int tid) {
  if (task.done) {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const uint32_t prev = atomicAdd(&task.done[0], 1u);
      if (prev == static_cast<uint32_t>(CL - 1)) {
        task.done[0] = 0u;
        __threadfence();
        st_release_u32(&task.done[1], (p.epoch ? *p.epoch : 0u) + 1u);
      }
    }
  }
  // a launch that started on the key flag rather than on griddepcontrol.wait
  // still completes only after the attention launch before it, so that the
  // launches of the step complete in launch order
  if (p.keys_ready && tid == 0) pdl_wait();
}

// VAR: a size rule or block expansion may be in use (an instantiation of its
// own, so that the fixed-k selection carries none of their code)
template <int CL, bool VAR>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_cluster_kernel(const TopkParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int CAP = kTopkCandCap;   // gathered candidates (all CTAs together)
  constexpr int RCAP = CAP / CL;      // candidates one CTA may contribute
  constexpr int SELCAP = kTopkSelCap; // this CTA's keys at or above the pivot digit
  constexpr unsigned FULL = 0xffffffffu;
  const int rank = static_cast<int>(cluster.block_rank());
  const TopkTask task = p.tasks ? p.tasks[blockIdx.y] : p.single;
  const int n = task.n > 0 ? task.n : p.n;
  const int k = p.k;                                 // entries of the output set
  const int kcap = task.k > 0 ? task.k : k;          // keys selected at most
  const int E = (VAR && p.expand > 1) ? p.expand : 1;  // rows per selected key
  const int rows = task.rows > 0 ? task.rows : n * E;
  const int rule = VAR ? p.size_rule : static_cast<int>(kSizeFixed);
  int keff = kcap < n ? kcap : n;
  const int chunk = (((n + CL - 1) / CL) + 3) & ~3;
  const int lo = rank * chunk;
  const int cnt = max(0, min(n, lo + chunk) - lo);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  // The keys are the attention kernel's output: read only once it has
  // written them.  The next kernel (the next selection, or the next
  // attention launch) may start its launch before that when its readers of
  // this selection's sets wait on the ready flags (p.early), else only after.
  // With a key counter, the keys are complete once every consumer warp of the
  // attention launch that writes them has finished its dense rows of this
  // layer (the counter reaches keys_expect); the rest of that launch may
  // still run.  The sets this launch writes replace sets that the attention
  // launch before that one may still read: wait for its done counter as
  // well.  Both writers were resident before this launch began (each launch
  // of the step starts only once every CTA of the one before it has), so the
  // waits end.
  if (p.early) pdl_launch_dependents();
  if (p.keys_ready) {
    __shared__ int wait_abort;
    if (tid == 0) {
      wait_abort = 0;
      const uint32_t par = (*p.epoch & 1u) * p.cnt_stride;
      if (wait_flag(p.keys_ready + par, p.keys_expect, &wait_abort, p.status) && p.prev_done)
        wait_flag(p.prev_done + par, p.prev_done_expect, &wait_abort, p.status);
    }
    __syncthreads();
  } else {
    pdl_wait();
  }
  if (!p.early) pdl_launch_dependents();
  const uint64_t t_start = p.timeline ? global_timer_ns() : 0;  // work starts here

  extern __shared__ __align__(16) unsigned char smem[];
  uint2* cand = reinterpret_cast<uint2*>(smem);        // [CAP] (encoded key, index) by source CTA
  uint2* sel = cand + CAP;                             // [SELCAP] this CTA's keys >= pivot digit
  uint32_t* loc = reinterpret_cast<uint32_t*>(sel + SELCAP);  // [kKeyBins] this CTA's histogram
  uint32_t* tot = loc + kKeyBins;                      // [kKeyBins] cluster totals, top digit
  uint32_t* src_cnt = tot + kKeyBins;                  // [CL] candidates per source CTA
  uint32_t* src_above = src_cnt + CL;                  // [CL] keys above the pivot digit per source
  uint32_t* src_gt = src_above + CL;                   // [CL] per source: keys > tau
  uint32_t* src_eq = src_gt + CL;                      // [CL] per source: keys == tau
  uint32_t* xchg = src_eq + CL;                        // [CL][2] (fallback path)
  uint32_t* scratch = xchg + 2 * CL;                   // [kTopkWarps]
  uint32_t* found = scratch + kTopkWarps;              // [4]
  uint32_t* vx = found + 4;                            // [16] size rules: per source, max key
  uint32_t* vcnt = vx + 16;                            // [16] per source: keys counted
  unsigned long long* vsum = reinterpret_cast<unsigned long long*>(vcnt + 16);  // [16] masses
  unsigned long long* scr64 = vsum + 16;               // [16]
  unsigned long long* res64 = scr64 + 16;              // [8]
  uint32_t* us = reinterpret_cast<uint32_t*>(res64 + 8);  // [chunk] encoded keys (16-byte aligned)
  // top-p, before the selection proper: `cand` holds the local histograms
  // (digit 0: three 16-bit limbs of the masses, u32 [3][2048]; digits 1-3:
  // count and limbs, u32 [4][128]); `sel` the cluster totals (digit 0: masses,
  // u64 [2048], its counts are `tot`; digits 1-3: masses u64 [3][128], then
  // counts u32 [3][128])
  constexpr int kFineBins = 128;  // digits 1-3 have 7 bits
  uint32_t* limb0 = reinterpret_cast<uint32_t*>(cand);
  uint32_t* fine_loc = limb0 + 3 * kKeyBins;
  unsigned long long* mt0 = reinterpret_cast<unsigned long long*>(sel);
  unsigned long long* mtf = mt0 + kKeyBins;
  uint32_t* ctf = reinterpret_cast<uint32_t*>(mtf + 3 * kFineBins);

  // the output: selected key j at position pos (its rows with block selection)
  // (and the same entry into the trace row, when there is one)
  int32_t* const trace = task.trace;
  auto store = [&](int64_t pos, int32_t v) {
    task.S[pos] = v;
    if (trace) trace[pos] = v;
  };
  auto put = [&](uint32_t pos, int32_t j) {
    if (E == 1) {
      store(pos, j);
    } else {
      for (int t = 0; t < E; ++t) {
        const int64_t r = static_cast<int64_t>(j) * E + t;
        store(static_cast<int64_t>(pos) * E + t, r < rows ? static_cast<int32_t>(r) : -1);
      }
    }
  };
  auto all_selected = [&]() {  // every key is selected
    for (int x = tid; x < cnt; x += kTopkThreads) put(static_cast<uint32_t>(lo + x), lo + x);
    if (rank == 0)
      for (int x = keff * E + tid; x < k; x += kTopkThreads) store(x, -1);
    topk_signal_done<CL>(p, task, tid);
    if (tid == 0)
      timeline_record(p.timeline, p.timeline_cap, t_start,
                      (kTagTopk << 32) | (static_cast<unsigned long long>(p.layer) << 16) |
                          (blockIdx.y * CL + rank));
  };
  if (rule == kSizeFixed && keff == n) {
    all_selected();
    return;
  }

  for (int b = tid; b < kKeyBins; b += kTopkThreads) {
    tot[b] = 0u;
    loc[b] = 0u;
  }
  if (rule != kSizeFixed) {
    if (tid < 8) res64[tid] = 0ull;
    if (rule == kSizeTopP) {  // every total of the descent, and the local masses
      uint32_t* a = reinterpret_cast<uint32_t*>(cand);
      uint32_t* b2 = reinterpret_cast<uint32_t*>(sel);
      for (int x = tid; x < 2 * kTopkCandCap; x += kTopkThreads) a[x] = 0u;
      for (int x = tid; x < 2 * kTopkSelCap; x += kTopkThreads) b2[x] = 0u;
    }
  }
  __syncthreads();
  // size rules and blocks: this CTA has started (and zeroed what other CTAs
  // add into); the wait below, before the first access to another CTA's
  // shared memory, lets the largest key go out before barrier (1)
  if (VAR) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // Every pass over the chunk gives warp w the contiguous range [wlo, whi)
  // and walks it 128 keys at a time, lane l holding keys 4l .. 4l+3 of the
  // step: 16-byte shared-memory accesses without bank conflicts, and index
  // order = (step, lane, element).
  const int span = ((cnt + kTopkWarps - 1) / kTopkWarps + 127) & ~127;
  const int wlo = min(cnt, warp * span);
  const int whi = min(cnt, wlo + span);
  auto load4 = [&](int x0, uint32_t* u) {  // four encoded keys from shared memory
    if (x0 + 3 < whi) {
      const uint4 v = *reinterpret_cast<const uint4*>(us + x0);
      u[0] = v.x; u[1] = v.y; u[2] = v.z; u[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) u[e] = (x0 + e < whi) ? us[x0 + e] : 0u;
    }
  };

  // ---- the chunk, encoded, into shared memory, and its top-digit histogram
  uint32_t umax = 0u;  // size rules: the largest encoded key of this thread
  if (VAR && E > 1) {
    // block selection: the chunk's keys are block scores, log(sum exp(key))
    // over the block's rows (max + log(sum exp(key - max))), one warp per block
    for (int x = warp; x < cnt; x += kTopkWarps) {
      const int64_t r0 = static_cast<int64_t>(lo + x) * E;
      const int64_t r1 = min(static_cast<int64_t>(rows), r0 + E);
      float m = -INFINITY, z = 0.f;
      if (E <= 128) {  // the block's keys in registers: one read of the rows
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t r = r0 + lane + 32 * j;
          v[j] = r < r1 ? task.keys[r] : -INFINITY;
          m = fmaxf(m, v[j]);
        }
        m = warp_max_f32(m);
#pragma unroll
        for (int j = 0; j < 4; ++j) z += v[j] == -INFINITY ? 0.f : expf(v[j] - m);
      } else {
        for (int64_t r = r0 + lane; r < r1; r += 32) m = fmaxf(m, task.keys[r]);
        m = warp_max_f32(m);
        for (int64_t r = r0 + lane; r < r1; r += 32) z += expf(task.keys[r] - m);
      }
      z = warp_sum_f32(z);
      if (lane == 0) {
        const uint32_t u = order_key(m + logf(z));
        us[x] = u;
        atomicAdd(&loc[u >> kKeyDigitShift], 1u);
        umax = max(umax, u);
      }
    }
  } else {
    // The keys were just written by the attention launch, which may still
    // stream beside this one, so each read waits on a loaded memory system.
    // A warp issues kLoadBatch steps' reads before it uses any of them: the
    // histogram's shared-memory atomics would otherwise hold each step's
    // read back until the step before it is done.
    constexpr int kLoadBatch = 8;
    const float* src = task.keys + lo;
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    for (int base = wlo; base < whi; base += 128 * kLoadBatch) {
      float4 v[kLoadBatch];
#pragma unroll
      for (int j = 0; j < kLoadBatch; ++j) {
        const int x0 = base + 128 * j + 4 * lane;
        if (vec && x0 + 3 < whi) {
          v[j] = *reinterpret_cast<const float4*>(src + x0);
        } else {
          v[j].x = x0 < whi ? src[x0] : 0.f;
          v[j].y = x0 + 1 < whi ? src[x0 + 1] : 0.f;
          v[j].z = x0 + 2 < whi ? src[x0 + 2] : 0.f;
          v[j].w = x0 + 3 < whi ? src[x0 + 3] : 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < kLoadBatch; ++j) {
        const int x0 = base + 128 * j + 4 * lane;
        const uint32_t u[4] = {order_key(v[j].x), order_key(v[j].y), order_key(v[j].z),
                               order_key(v[j].w)};
        if (x0 + 3 < whi) {
          *reinterpret_cast<uint4*>(us + x0) = make_uint4(u[0], u[1], u[2], u[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (x0 + e < whi) us[x0 + e] = u[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (x0 + e < whi) {
            atomicAdd(&loc[u[e] >> kKeyDigitShift], 1u);
            if (VAR) umax = max(umax, u[e]);
          }
      }
    }
  }
  if (rule != kSizeFixed) {
    umax = __reduce_max_sync(FULL, umax);
    if (lane == 0) atomicMax(reinterpret_cast<uint32_t*>(&res64[5]), umax);  // low word
  }
  __syncthreads();
  if (VAR) {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (rule != kSizeFixed && tid < CL)
      cluster.map_shared_rank(vx, tid)[rank] = static_cast<uint32_t>(res64[5]);
  }
  cluster.sync();  // (1) every CTA's totals are zero and its histogram complete

  // ---- size rules, first part: the cluster's largest key M; threshold's
  // local mass, top-p's local digit-0 masses (three 16-bit limbs per bin in
  // 32-bit words: sums of at most 2^16 keys per CTA cannot overflow, and no
  // add needs its result)
  float M = 0.f;
  if (rule != kSizeFixed) {
    uint32_t um = 0u;
    for (int r = 0; r < CL; ++r) um = max(um, vx[r]);
    M = key_from_order(um);
    if (rule == kSizeThreshold) {
      unsigned long long sw = 0ull;
      for (int x = tid; x < cnt; x += kTopkThreads) sw += key_weight(us[x], M);
      sw = warp_sum_u64(sw);
      if (lane == 0) atomic_add_u64_split(&res64[4], sw);
    } else {
      for (int x = tid; x < cnt; x += kTopkThreads) {
        const uint32_t u = us[x];
        const uint32_t d = u >> kKeyDigitShift;
        const unsigned long long w = key_weight(u, M);
        atomicAdd(&limb0[d], static_cast<uint32_t>(w & 0xffffu));
        atomicAdd(&limb0[kKeyBins + d], static_cast<uint32_t>((w >> 16) & 0xffffu));
        if (w >> 32) atomicAdd(&limb0[2 * kKeyBins + d], static_cast<uint32_t>(w >> 32));
      }
    }
    __syncthreads();
  }

  // ---- top digit: add the non-zero local bins into every CTA's totals (and
  // the size rules' local masses)
  if (rule == kSizeTopP) {
    for (int x = tid; x < CL * kKeyBins; x += kTopkThreads) {
      const int b = x % kKeyBins, r = x / kKeyBins;
      const uint32_t c = loc[b];
      if (c) {
        atomicAdd(cluster.map_shared_rank(tot, r) + b, c);
        const unsigned long long w = static_cast<unsigned long long>(limb0[b]) +
                                     (static_cast<unsigned long long>(limb0[kKeyBins + b]) << 16) +
                                     (static_cast<unsigned long long>(limb0[2 * kKeyBins + b]) << 32);
        if (w) atomicAdd(cluster.map_shared_rank(mt0, r) + b, w);
      }
    }
  } else {
    if (rule == kSizeThreshold && tid < CL) cluster.map_shared_rank(vsum, tid)[rank] = res64[4];
    uint2* nz = cand;  // (bin, count) of the non-zero local bins; free until the gather
    const uint32_t nnz = compact_nonzero(loc, nz, scratch, tid, lane, warp);
    for (uint32_t x = tid; x < nnz * CL; x += kTopkThreads) {
      const uint2 e = nz[x / CL];
      atomicAdd(cluster.map_shared_rank(tot, static_cast<int>(x % CL)) + e.x, e.y);
    }
  }
  cluster.sync();  // (2)

  // ---- size rules, second part: how many keys to select
  if (rule != kSizeFixed) {
    if (rule == kSizeThreshold) {
      unsigned long long total = 0ull;
      for (int r = 0; r < CL; ++r) total += vsum[r];
      const double tg = ceil(p.size_x * static_cast<double>(total));
      const unsigned long long thr = tg <= 0.0 ? 0ull : static_cast<unsigned long long>(tg);
      uint32_t c = 0u;
      for (int x0 = 0; x0 < cnt; x0 += kTopkThreads) {  // every lane takes part in the reduce
        const int x = x0 + tid;
        c += (x < cnt && key_weight(us[x], M) >= thr) ? 1u : 0u;
      }
      c = __reduce_add_sync(FULL, c);
      if (lane == 0) atomicAdd(reinterpret_cast<uint32_t*>(&res64[6]), c);  // low word
      __syncthreads();
      if (tid < CL) cluster.map_shared_rank(vcnt, tid)[rank] = static_cast<uint32_t>(res64[6]);
      cluster.sync();
      uint32_t m = 0u;
      for (int r = 0; r < CL; ++r) m += vcnt[r];
      m = max(m, 1u);
      keff = min(keff, static_cast<int>(m));
    } else {
      // top-p: a radix descent (digits of 11, 7, 7 and 7 bits) to the key
      // value at which the running mass, larger keys first, reaches
      // T = ceil(p * total mass); digits 1-3 as digit 0, with local counts
      uint32_t prefix = 0u, pmask = 0u, m_above = 0u;
      unsigned long long target = 0ull;
      uint32_t dg = 0u, ca = 0u;
      unsigned long long ma = 0ull;
      {  // the mass to reach, and digit 0
        unsigned long long tm = 0ull;
        for (int b = tid; b < kKeyBins; b += kTopkThreads) tm += mt0[b];
        tm = warp_sum_u64(tm);
        if (lane == 0) scr64[warp] = tm;
        __syncthreads();
        unsigned long long total = 0ull;
        for (int w2 = 0; w2 < kTopkWarps; ++w2) total += scr64[w2];
        __syncthreads();
        const double tg = ceil(p.size_x * static_cast<double>(total));
        target = tg >= static_cast<double>(total)
                     ? total
                     : (tg < 1.0 ? 1ull : static_cast<unsigned long long>(tg));
        find_digit_mass<kKeyBins>(mt0, tot, target, scr64, scratch, res64, tid, lane, warp, &dg, &ca,
                                  &ma);
        m_above += ca;
        target -= ma;
        prefix = dg << kKeyDigitShift;
        pmask = 0xffe00000u;
      }
#pragma unroll 1
      for (int pass = 1; pass < 4; ++pass) {
        const int sh = 21 - 7 * pass;
        const uint32_t dmask = kFineBins - 1;
        uint32_t* lc = fine_loc;              // local counts
        uint32_t* lm = fine_loc + kFineBins;  // local limbs [3][kFineBins]
        unsigned long long* mt = mtf + (pass - 1) * kFineBins;
        uint32_t* ct = ctf + (pass - 1) * kFineBins;
        for (int b = tid; b < 4 * kFineBins; b += kTopkThreads) fine_loc[b] = 0u;
        __syncthreads();
        for (int x = tid; x < cnt; x += kTopkThreads) {
          const uint32_t u = us[x];
          if ((u & pmask) != prefix) continue;
          const uint32_t d = (u >> sh) & dmask;
          const unsigned long long w = key_weight(u, M);
          atomicAdd(&lc[d], 1u);
          atomicAdd(&lm[d], static_cast<uint32_t>(w & 0xffffu));
          atomicAdd(&lm[kFineBins + d], static_cast<uint32_t>((w >> 16) & 0xffffu));
          if (w >> 32) atomicAdd(&lm[2 * kFineBins + d], static_cast<uint32_t>(w >> 32));
        }
        __syncthreads();
        for (int x = tid; x < CL * kFineBins; x += kTopkThreads) {
          const int b = x % kFineBins, r = x / kFineBins;
          const uint32_t c = lc[b];
          if (c) {
            atomicAdd(cluster.map_shared_rank(ct, r) + b, c);
            const unsigned long long w = static_cast<unsigned long long>(lm[b]) +
                                         (static_cast<unsigned long long>(lm[kFineBins + b]) << 16) +
                                         (static_cast<unsigned long long>(lm[2 * kFineBins + b]) << 32);
            if (w) atomicAdd(cluster.map_shared_rank(mt, r) + b, w);
          }
        }
        cluster.sync();
        find_digit_mass<kFineBins>(mt, ct, target, scr64, scratch, res64, tid, lane, warp, &dg, &ca,
                                   &ma);
        m_above += ca;
        target -= ma;
        prefix |= dg << sh;
        pmask |= dmask << sh;
      }
      // `prefix` is now the key value that reaches the mass: its keys all
      // have the same weight; take as many of them as the rest of the mass needs
      const uint32_t cv = ctf[2 * kFineBins + dg];
      const unsigned long long wv = mtf[2 * kFineBins + dg] / (cv ? cv : 1u);
      unsigned long long r = wv ? (target + wv - 1ull) / wv : cv;
      r = r < 1ull ? 1ull : (r > cv ? cv : r);
      keff = min(keff, static_cast<int>(m_above + static_cast<uint32_t>(r)));
    }
    __syncthreads();  // every read of `sel` precedes the selection's writes to it
  }
  if (rule != kSizeFixed && keff == n) {
    all_selected();
    return;
  }
  uint32_t d0, above;
  find_digit(tot, static_cast<uint32_t>(keff), scratch, found, tid, lane, warp, &d0, &above);
  uint32_t krem = static_cast<uint32_t>(keff) - above;
  const uint32_t ncand = tot[d0];

  // ---- pass over the chunk: per warp, keys above the pivot digit and keys
  // on it (the candidates)
  uint32_t my_cand = 0u, my_above = 0u, c_before = 0u, a_before = 0u;
  {
    uint32_t wc = 0u, wa = 0u;
    for (int base = wlo; base < whi; base += 128) {
      const int x0 = base + 4 * lane;
      uint32_t u[4];
      load4(x0, u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = x0 + e < whi;
        const uint32_t dg = u[e] >> kKeyDigitShift;
        wc += (ok && dg == d0) ? 1u : 0u;
        wa += (ok && dg > d0) ? 1u : 0u;
      }
    }
#pragma unroll
    for (int s2 = 16; s2 >= 1; s2 >>= 1) {
      wc += __shfl_xor_sync(FULL, wc, s2);
      wa += __shfl_xor_sync(FULL, wa, s2);
    }
    cta_warp_scan(scratch, wc, warp, lane, &c_before, &my_cand);
    cta_warp_scan(scratch, wa, warp, lane, &a_before, &my_above);
  }
  // this CTA's keys at or above the pivot digit, in index order, into `sel`
  // (when they fit), and its candidates into its region of `cand`
  const bool sel_fits = my_above + my_cand <= static_cast<uint32_t>(SELCAP);
  const bool cand_fits = my_cand <= static_cast<uint32_t>(RCAP);
  uint2* mine = cand + rank * RCAP;
  if (sel_fits || cand_fits) {
    uint32_t cpos = c_before, spos = a_before + c_before;
    for (int base = wlo; base < whi; base += 128) {
      const int x0 = base + 4 * lane;
      uint32_t u[4];
      load4(x0, u);
      // one ballot per element slot: a lane's entries come after every entry
      // of the lanes below it (index order is lane, then element)
      unsigned bc[4], bs[4];
      uint32_t oc = cpos, os = spos, tc = 0u, ts = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = x0 + e < whi;
        const uint32_t dg = u[e] >> kKeyDigitShift;
        bc[e] = __ballot_sync(FULL, ok && dg == d0);
        bs[e] = __ballot_sync(FULL, ok && dg >= d0);
        oc += __popc(bc[e] & lt);
        os += __popc(bs[e] & lt);
        tc += __popc(bc[e]);
        ts += __popc(bs[e]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint2 ent = make_uint2(u[e], static_cast<uint32_t>(lo + x0 + e));
        if ((bs[e] >> lane) & 1u) {
          if (sel_fits) sel[os] = ent;
          ++os;
        }
        if ((bc[e] >> lane) & 1u) {
          if (cand_fits) mine[oc] = ent;
          ++oc;
        }
      }
      cpos += tc;
      spos += ts;
    }
  }
  __syncthreads();
  // candidates into the other CTAs, (entry, CTA) pairs spread over the threads
  if (cand_fits) {
    for (uint32_t x = tid; x < my_cand * (CL - 1); x += kTopkThreads) {
      const uint32_t j = x / (CL - 1);
      const int r = static_cast<int>(x % (CL - 1));
      const int dst = r < rank ? r : r + 1;
      cluster.map_shared_rank(cand, dst)[rank * RCAP + j] = mine[j];
    }
  }
  if (tid < CL) {
    cluster.map_shared_rank(src_cnt, tid)[rank] = my_cand;
    cluster.map_shared_rank(src_above, tid)[rank] = my_above;
  }
  cluster.sync();  // (3) candidates and counts of every CTA are here

  bool fits = ncand <= static_cast<uint32_t>(CAP);
  for (int r = 0; r < CL; ++r) fits = fits && src_cnt[r] <= static_cast<uint32_t>(RCAP);

  uint32_t tau, out_base, take;
  if (fits) {
    // ---- tau among the gathered candidates, the same in every CTA
    tau = select_in_candidates<CL>(cand, src_cnt, RCAP, d0 << kKeyDigitShift, 0xffe00000u, &krem,
                                   loc, scratch, found, tid, lane, warp);
    // per source: keys > tau and == tau (warp w counts the sources w, w+16, ...)
    for (int r = warp; r < CL; r += kTopkWarps) {
      const uint32_t c = src_cnt[r];
      uint32_t g = 0u, e = 0u;
      for (uint32_t base = 0; base < c; base += 32) {
        const uint32_t x = base + lane;
        const uint32_t u = (x < c) ? cand[r * RCAP + x].x : 0u;
        g += __popc(__ballot_sync(0xffffffffu, x < c && u > tau));
        e += __popc(__ballot_sync(0xffffffffu, x < c && u == tau));
      }
      if (lane == 0) {
        src_gt[r] = src_above[r] + g;
        src_eq[r] = e;
      }
    }
    __syncthreads();
    out_base = 0u;
    uint32_t eq_prev = 0u;
    for (int r = 0; r < rank; ++r) {
      const uint32_t e = src_eq[r];
      const uint32_t tk = (krem > eq_prev) ? min(krem - eq_prev, e) : 0u;
      out_base += src_gt[r] + tk;
      eq_prev += e;
    }
    take = (krem > eq_prev) ? min(krem - eq_prev, src_eq[rank]) : 0u;
  } else {
    // ---- too many candidates (heavily tied keys): two more radix digits over
    // the chunks, totals pushed into every CTA, then a count exchange
    uint32_t* tot12 = reinterpret_cast<uint32_t*>(cand);  // the candidates are not needed here
    for (int b = tid; b < 2 * kKeyBins; b += kTopkThreads) tot12[b] = 0u;
    cluster.sync();  // every CTA's digit-1/2 totals are zero
    uint32_t prefix = d0 << kKeyDigitShift, pmask = 0xffe00000u;
#pragma unroll
    for (int pass = 1; pass <= 2; ++pass) {
      const int sh = pass == 1 ? 10 : 0;
      const uint32_t dmask = pass == 1 ? 0x7ffu : 0x3ffu;
      uint32_t* tp = tot12 + (pass - 1) * kKeyBins;
      for (int b = tid; b < kKeyBins; b += kTopkThreads) loc[b] = 0u;
      __syncthreads();
      for (int x = tid; x < cnt; x += kTopkThreads) {
        const uint32_t u = us[x];
        if ((u & pmask) == prefix) atomicAdd(&loc[(u >> sh) & dmask], 1u);
      }
      __syncthreads();
      for (int x = tid; x < CL * kKeyBins; x += kTopkThreads) {
        const int b = x % kKeyBins, r = x / kKeyBins;
        const uint32_t c = loc[b];
        if (c) atomicAdd(cluster.map_shared_rank(tp, r) + b, c);
      }
      cluster.sync();
      uint32_t dg, ab;
      find_digit(tp, krem, scratch, found, tid, lane, warp, &dg, &ab);
      krem -= ab;
      prefix |= dg << sh;
      pmask |= dmask << sh;
    }
    tau = prefix;
    uint32_t g = 0u, e = 0u;
    for (int x = tid; x < cnt; x += kTopkThreads) {
      const uint32_t u = us[x];
      g += u > tau;
      e += u == tau;
    }
    uint32_t dummy, gt_cta, eq_cta;
    const unsigned FULL = 0xffffffffu;
#pragma unroll
    for (int s2 = 16; s2 >= 1; s2 >>= 1) {
      g += __shfl_xor_sync(FULL, g, s2);
      e += __shfl_xor_sync(FULL, e, s2);
    }
    cta_warp_scan(scratch, g, warp, lane, &dummy, &gt_cta);
    cta_warp_scan(scratch, e, warp, lane, &dummy, &eq_cta);
    if (tid < CL) {
      uint32_t* xd = cluster.map_shared_rank(xchg, tid);
      xd[2 * rank] = gt_cta;
      xd[2 * rank + 1] = eq_cta;
    }
    cluster.sync();
    out_base = 0u;
    uint32_t eq_prev = 0u;
    for (int r = 0; r < rank; ++r) {
      const uint32_t gg = xchg[2 * r], ee = xchg[2 * r + 1];
      const uint32_t tk = (krem > eq_prev) ? min(krem - eq_prev, ee) : 0u;
      out_base += gg + tk;
      eq_prev += ee;
    }
    take = (krem > eq_prev) ? min(krem - eq_prev, eq_cta) : 0u;
  }

  // ---- write this CTA's selected indices in index order, from `sel` when it
  // holds every key at or above the pivot digit (few), else from the whole
  // chunk.  Warp w owns entries [w*span, (w+1)*span) of the list, span a
  // multiple of 128, four ballot rows per step.
  auto emit = [&](auto get, int len) {
    const int sp = ((len + kTopkWarps - 1) / kTopkWarps + 127) & ~127;
    const int elo = min(len, warp * sp);
    const int ehi = min(len, elo + sp);
    uint32_t wgt = 0u, weq = 0u;
    for (int base = elo; base < ehi; base += 128) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int x = base + 32 * j + lane;
        const uint32_t u = (x < ehi) ? get(x).x : 0u;
        wgt += __popc(__ballot_sync(FULL, x < ehi && u > tau));
        weq += __popc(__ballot_sync(FULL, x < ehi && u == tau));
      }
    }
    uint32_t gt_before, eq_before, dummy2;
    cta_warp_scan(scratch, wgt, warp, lane, &gt_before, &dummy2);
    cta_warp_scan(scratch, weq, warp, lane, &eq_before, &dummy2);
    uint32_t run_eq = eq_before;
    uint32_t run_sel = out_base + gt_before + min(eq_before, take);
    for (int base = elo; base < ehi; base += 128) {
      uint2 ent[4];
      unsigned gb[4], eb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int x = base + 32 * j + lane;
        ent[j] = (x < ehi) ? get(x) : make_uint2(0u, 0u);
        gb[j] = __ballot_sync(FULL, x < ehi && ent[j].x > tau);
        eb[j] = __ballot_sync(FULL, x < ehi && ent[j].x == tau);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool is_eq = (eb[j] >> lane) & 1u;
        const bool pick = ((gb[j] >> lane) & 1u) || (is_eq && run_eq + __popc(eb[j] & lt) < take);
        const unsigned sb = __ballot_sync(FULL, pick);
        const uint32_t pos = run_sel + __popc(sb & lt);
        if (pick && pos < static_cast<uint32_t>(keff)) put(pos, static_cast<int32_t>(ent[j].y));
        run_sel += __popc(sb);
        run_eq += __popc(eb[j]);
      }
    }
  };
  if (fits && sel_fits)
    emit([&](int x) { return sel[x]; }, static_cast<int>(my_above + my_cand));
  else
    emit([&](int x) { return make_uint2(us[x], static_cast<uint32_t>(lo + x)); }, cnt);
  if (rank == 0)
    for (int x = keff * E + tid; x < k; x += kTopkThreads) store(x, -1);
  topk_signal_done<CL>(p, task, tid);
  if (tid == 0)
    timeline_record(p.timeline, p.timeline_cap, t_start,
                    (kTagTopk << 32) | (static_cast<unsigned long long>(p.layer) << 16) |
                        (blockIdx.y * CL + rank));
  // no CTA leaves while another may still access its shared memory: every
  // remote access precedes the last cluster barrier on its path.
}

// ---------------------------------------------------------------- host side
static size_t topk_smem_bytes(int cl, int n) {
  const int chunk = (((n + cl - 1) / cl) + 3) & ~3;
  return static_cast<size_t>(2 * kTopkCandCap + 2 * kTopkSelCap + 2 * kKeyBins + 6 * cl + kTopkWarps +
                             4 + kTopkRuleWords + chunk) * 4u;
}

template <int CL>
static cudaError_t topk_run(const TopkParams* p, int ntasks, cudaStream_t stream, bool configure_only,
                            size_t max_smem, bool force_var = false) {
  if (configure_only) {
    for (auto kern : {topk_cluster_kernel<CL, false>, topk_cluster_kernel<CL, true>}) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(max_smem));
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      if (CL > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const bool var = force_var || p->size_rule != kSizeFixed || p->expand > 1;
  auto kern = var ? topk_cluster_kernel<CL, true> : topk_cluster_kernel<CL, false>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, ntasks, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = topk_smem_bytes(CL, p->n);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, *p);
}

size_t topk_smem_for(int cl, int n) { return topk_smem_bytes(cl, n); }

// Largest cluster size (16, else 8) that can be resident with `smem` bytes.
int topk_pick_cluster(size_t smem) {
  if (topk_run<16>(nullptr, 0, nullptr, true, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<16, false>, &cfg) == cudaSuccess &&
        nclusters > 0)
      return 16;
  }
  cudaGetLastError();
  return 8;
}

// How many clusters of `cl` CTAs with `smem` bytes each can be resident at
// once (0 if unknown); cl must have been configured.
template <int CL>
static int topk_max_clusters_t(size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel<CL, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int topk_max_clusters(int cl, size_t smem) {
  switch (cl) {
    case 16: return topk_max_clusters_t<16>(smem);
    case 8: return topk_max_clusters_t<8>(smem);
    case 4: return topk_max_clusters_t<4>(smem);
  }
  return 0;
}

cudaError_t topk_configure(int cl, size_t smem) {
  switch (cl) {
    case 16: return topk_run<16>(nullptr, 0, nullptr, true, smem);
    case 8: return topk_run<8>(nullptr, 0, nullptr, true, smem);
    case 4: return topk_run<4>(nullptr, 0, nullptr, true, smem);
  }
  return cudaErrorInvalidValue;
}

// force_var: run the instantiation of the size rules even for a fixed k
// (test hook: the same selection through both instantiations)
cudaError_t topk_launch(int cl, const TopkParams* p, int ntasks, cudaStream_t stream, bool force_var) {
  switch (cl) {
    case 16: return topk_run<16>(p, ntasks, stream, false, 0, force_var);
    case 8: return topk_run<8>(p, ntasks, stream, false, 0, force_var);
    case 4: return topk_run<4>(p, ntasks, stream, false, 0, force_var);
  }
  return cudaErrorInvalidValue;
}


}  // namespace lyc
