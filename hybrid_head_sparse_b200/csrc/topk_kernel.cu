// topk_kernel.cu -- exact argsTopK over one row of selection keys per task.
//
// What it computes (page "LycheeDecode ...", paper-graph-ui summary,
// section 3.4 Eq. 2): S = the k_eff = min(k, n) indices with the largest
// keys, ties to the lower index (-0 == +0), written in ascending index
// order, positions k_eff..k-1 set to -1.
//
// Design (B200 / sm_100a): one thread-block cluster of CL CTAs per task.
//   1. each CTA loads its contiguous chunk of n/CL keys once into shared
//      memory as order-preserving unsigned integers;
//   2. radix select, most significant digit first (11 + 11 + 10 bits): each
//      CTA histograms its candidates (warp-aggregated shared atomics), the
//      cluster sums the histograms through distributed shared memory, and
//      every CTA finds the same digit of the k-th largest key tau;
//   3. stable compaction: CTAs exchange their counts of keys > tau and == tau,
//      which fixes each CTA's output offset and how many of its ties (lowest
//      indices first) it takes; inside a CTA warps compact in index order
//      with ballots.
// No pass reads global memory again after step 1.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lyc_device.cuh"
#include "lyc_plan.h"

namespace cg = cooperative_groups;

namespace lyc {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 == +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive prefix sum of one value per warp (lane 0 holds it) over the CTA.
// Returns the exclusive prefix for the caller's warp and the CTA total.
__device__ __forceinline__ void warp_exclusive_scan(uint32_t* scratch, uint32_t mine, int warp,
                                                    int lane, uint32_t* prefix, uint32_t* total) {
  if (lane == 0) scratch[warp] = mine;
  __syncthreads();
  uint32_t acc = 0, tot = 0;
  for (int w = 0; w < kTopkWarps; ++w) {
    const uint32_t v = scratch[w];
    if (w < warp) acc += v;
    tot += v;
  }
  *prefix = acc;
  *total = tot;
  __syncthreads();
}

template <int CL>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_cluster_kernel(const TopkParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const TopkTask task = p.tasks ? p.tasks[blockIdx.y] : p.single;
  const int n = p.n;
  const int k = p.k;
  const int keff = k < n ? k : n;
  const int chunk = (n + CL - 1) / CL;
  const int lo = rank * chunk;
  const int cnt = max(0, min(n, lo + chunk) - lo);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);            // [kBins]
  uint32_t* total = hist + kBins;                                // [kBins]
  uint32_t* xchg = total + kBins;                                // [CL][2]
  uint32_t* scratch = xchg + 2 * CL;                             // [kTopkWarps]
  uint32_t* found = scratch + kTopkWarps;                        // [2]: digit, count above
  uint32_t* us = found + 4;                                      // [chunk]

  // all indices selected: no ordering work
  if (keff == n) {
    for (int x = tid; x < cnt; x += kTopkThreads) task.S[lo + x] = lo + x;
    if (rank == 0)
      for (int x = keff + tid; x < k; x += kTopkThreads) task.S[x] = -1;
    return;
  }

  for (int x = tid; x < cnt; x += kTopkThreads) us[x] = order_key(task.keys[lo + x]);

  // ---- radix select of tau, the k-th largest key
  uint32_t prefix = 0u, pmask = 0u;
  uint32_t krem = static_cast<uint32_t>(keff);
#pragma unroll
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3ffu : 0x7ffu;
    for (int b = tid; b < kBins; b += kTopkThreads) hist[b] = 0u;
    __syncthreads();
    for (int base = 0; base < cnt; base += kTopkThreads) {
      const int x = base + tid;
      const uint32_t u = (x < cnt) ? us[x] : 0u;
      const bool cand = (x < cnt) && ((u & pmask) == prefix);
      const unsigned act = __ballot_sync(0xffffffffu, cand);
      if (cand) {
        const uint32_t dg = (u >> sh) & dmask;
        const unsigned peers = __match_any_sync(act, dg);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[dg], static_cast<uint32_t>(__popc(peers)));
      }
    }
    cluster.sync();
    // this CTA sums its slice of bins over the cluster and hands the sums to all
    constexpr int slice = kBins / CL;
    for (int b = rank * slice + tid; b < (rank + 1) * slice; b += kTopkThreads) {
      uint32_t s = 0u;
#pragma unroll
      for (int r = 0; r < CL; ++r) s += cluster.map_shared_rank(hist, r)[b];
#pragma unroll
      for (int r = 0; r < CL; ++r) cluster.map_shared_rank(total, r)[b] = s;
    }
    cluster.sync();
    // digit of tau: the one where the count of larger candidates crosses krem
    constexpr int per = kBins / kTopkThreads;  // bins per thread
    uint32_t mine = 0u;
#pragma unroll
    for (int q = 0; q < per; ++q) mine += total[tid * per + q];
    // inclusive sum of `mine` over threads with a larger id (suffix), per warp then CTA
    uint32_t suf = mine;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, suf, s);
      if (lane + s < 32) suf += v;
    }
    if (lane == 0) scratch[warp] = suf;  // warp total
    __syncthreads();
    uint32_t above = suf - mine;  // strictly larger threads within the warp
    for (int w2 = warp + 1; w2 < kTopkWarps; ++w2) above += scratch[w2];
#pragma unroll
    for (int q = per - 1; q >= 0; --q) {
      const uint32_t c = total[tid * per + q];
      if (above < krem && above + c >= krem) {
        found[0] = static_cast<uint32_t>(tid * per + q);
        found[1] = above;
      }
      above += c;
    }
    __syncthreads();
    const uint32_t dg = found[0];
    krem -= found[1];
    prefix |= dg << sh;
    pmask |= dmask << sh;
    __syncthreads();
  }
  const uint32_t tau = prefix;  // krem = how many keys equal to tau are taken

  // ---- counts of this CTA, exchanged across the cluster
  uint32_t gt = 0u, eq = 0u;
  for (int base = 0; base < cnt; base += kTopkThreads) {
    const int x = base + tid;
    const uint32_t u = (x < cnt) ? us[x] : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, x < cnt && u > tau));
    eq += __popc(__ballot_sync(0xffffffffu, x < cnt && u == tau));
  }
  uint32_t gt_cta, eq_cta, dummy;
  warp_exclusive_scan(scratch, gt, warp, lane, &dummy, &gt_cta);
  warp_exclusive_scan(scratch, eq, warp, lane, &dummy, &eq_cta);
  if (tid < CL) {
    uint32_t* dst = cluster.map_shared_rank(xchg, tid);
    dst[2 * rank] = gt_cta;
    dst[2 * rank + 1] = eq_cta;
  }
  cluster.sync();
  uint32_t out_base = 0u, eq_before = 0u;
  for (int r = 0; r < rank; ++r) {
    const uint32_t g = xchg[2 * r], e = xchg[2 * r + 1];
    const uint32_t tk = (krem > eq_before) ? min(krem - eq_before, e) : 0u;
    out_base += g + tk;
    eq_before += e;
  }
  const uint32_t take = (krem > eq_before) ? min(krem - eq_before, eq_cta) : 0u;

  // ---- stable compaction: warp w owns elements [w*span, (w+1)*span)
  const int span = ((cnt + kTopkWarps - 1) / kTopkWarps + 31) & ~31;
  const int wlo = warp * span;
  const int whi = min(cnt, wlo + span);
  const unsigned lt = (1u << lane) - 1u;
  uint32_t weq = 0u;
  for (int base = wlo; base < whi; base += 32) {
    const int x = base + lane;
    weq += __popc(__ballot_sync(0xffffffffu, x < whi && us[x] == tau));
  }
  uint32_t eq_base, eq_tot;
  warp_exclusive_scan(scratch, weq, warp, lane, &eq_base, &eq_tot);
  uint32_t wsel = 0u;
  {
    uint32_t run_eq = eq_base;
    for (int base = wlo; base < whi; base += 32) {
      const int x = base + lane;
      const uint32_t u = (x < whi) ? us[x] : 0u;
      const bool is_eq = x < whi && u == tau;
      const unsigned eb = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = (x < whi) && (u > tau || (is_eq && run_eq + __popc(eb & lt) < take));
      wsel += __popc(__ballot_sync(0xffffffffu, sel));
      run_eq += __popc(eb);
    }
  }
  uint32_t sel_base, sel_tot;
  warp_exclusive_scan(scratch, wsel, warp, lane, &sel_base, &sel_tot);
  {
    uint32_t run_eq = eq_base, run_sel = out_base + sel_base;
    for (int base = wlo; base < whi; base += 32) {
      const int x = base + lane;
      const uint32_t u = (x < whi) ? us[x] : 0u;
      const bool is_eq = x < whi && u == tau;
      const unsigned eb = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = (x < whi) && (u > tau || (is_eq && run_eq + __popc(eb & lt) < take));
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      const uint32_t pos = run_sel + __popc(sb & lt);
      if (sel && pos < static_cast<uint32_t>(keff)) task.S[pos] = lo + x;
      run_sel += __popc(sb);
      run_eq += __popc(eb);
    }
  }
  if (rank == 0)
    for (int x = keff + tid; x < k; x += kTopkThreads) task.S[x] = -1;
  (void)eq_tot;
  (void)sel_tot;
  // no CTA leaves while another may still read its shared memory: the last
  // remote access (the count exchange) precedes the cluster.sync above.
}

// ---------------------------------------------------------------- host side
static size_t topk_smem_bytes(int cl, int n) {
  const int chunk = (n + cl - 1) / cl;
  return static_cast<size_t>(2 * kBins + 2 * cl + kTopkWarps + 4 + chunk) * 4u;
}

template <int CL>
static cudaError_t topk_run(const TopkParams* p, int ntasks, cudaStream_t stream, bool configure_only,
                            size_t max_smem) {
  auto kern = topk_cluster_kernel<CL>;
  if (configure_only) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(max_smem));
    if (e != cudaSuccess) return e;
    if (CL > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, ntasks, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = topk_smem_bytes(CL, p->n);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
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
    if (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<16>, &cfg) == cudaSuccess &&
        nclusters > 0)
      return 16;
  }
  cudaGetLastError();
  return 8;
}

cudaError_t topk_configure(int cl, size_t smem) {
  return cl == 16 ? topk_run<16>(nullptr, 0, nullptr, true, smem)
                  : topk_run<8>(nullptr, 0, nullptr, true, smem);
}

cudaError_t topk_launch(int cl, const TopkParams* p, int ntasks, cudaStream_t stream) {
  return cl == 16 ? topk_run<16>(p, ntasks, stream, false, 0) : topk_run<8>(p, ntasks, stream, false, 0);
}

}  // namespace lyc
