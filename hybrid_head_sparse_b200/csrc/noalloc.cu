// noalloc.cu -- lyc_sparse_attention_noalloc: the sparse-head attention of
// one layer for callers that cannot allocate device memory.  The paper has no
// counterpart for this entry point; the arithmetic is the library's sparse
// head, o = softmax(q K[S]^T / sqrt(d)) V[S] over the rows of a given set.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not
// acceptable -- inside a framework whose caching allocator owns all device
// memory (a raw cudaMalloc there fragments its pool and can fail when the
// pool holds the free memory), or on a latency-critical serving path where
// cudaMalloc / cudaFree may synchronize the device.  lyc_create allocates its
// scratch with cudaMalloc, so such callers cannot create a context; this
// entry point needs none.
//
// How: the pooled attention kernel of the bf16 path (attn_mma_kernel.cu) is
// launched unchanged; everything it needs beyond the caller's tensors --
// work lists, partial softmax states, the per-CTA ring of consumer-warp
// states, arrival counters, the status word -- lives in one file-scope
// device array of fixed size, g_noalloc_scratch.  Its address is looked up
// once per device with cudaGetSymbolAddress.  Per call a small kernel on the
// caller's stream writes the work list into the array and clears the
// counters and the status word (the call's sizes and pointers are its
// by-value arguments), so a call enqueues kernels and one status copy only:
// no host-to-device copy, no cudaMalloc, cudaFree or allocating library
// routine.
//
// Every call shares the array, which keeps the last call's contents: calls
// that may overlap on the GPU (two streams, two host threads without an
// ordering between their streams) race on it.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/lyc.h"
#include "lyc_plan.h"

namespace lyc {

cudaError_t attn_mma_dispatch(int D, const AttnMmaParams* P, int grid, cudaStream_t stream,
                              int* smem_out, bool configure_only);

namespace {

// Limits of one call (they size the array below).  Every segment has one
// query row, so the consumer-warp ring keeps one row per warp record.
constexpr int kNaMaxSets = LYC_NOALLOC_MAX_SETS;   // batch * query heads
constexpr int kNaMaxCtas = LYC_NOALLOC_MAX_CTAS;   // CTAs of the attention launch
constexpr int kNaMaxD = 128;
constexpr int kNaMaxPieces = kNaMaxCtas + kNaMaxSets;  // one per CTA run and segment cut
constexpr int kNaMaxParts = kNaMaxPieces;              // one partial per piece (one output each)
constexpr int kNaMaxCounters = kNaMaxSets;

constexpr size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
// scratch layout (byte offsets)
constexpr size_t kOffSegs = 0;
constexpr size_t kOffPieces = align256(kOffSegs + sizeof(Segment) * kNaMaxSets);
constexpr size_t kOffCta = align256(kOffPieces + sizeof(Piece) * kNaMaxPieces);
// the combine launch: (segment, output) tasks and CTA offsets with no pieces
constexpr size_t kOffTasks = align256(kOffCta + sizeof(int32_t) * (kNaMaxCtas + 1));
constexpr size_t kOffEmptyCta = align256(kOffTasks + sizeof(int2) * kNaMaxSets);
constexpr size_t kPlanBytes = align256(kOffEmptyCta + sizeof(int32_t) * (kNaMaxCtas + 1));
constexpr size_t kOffCounters = kPlanBytes;  // [kNaMaxCounters] int32, then the status word
constexpr size_t kOffStatus = kOffCounters + sizeof(int32_t) * kNaMaxCounters;
constexpr size_t kZeroBytes = align256(kOffStatus + 16) - kOffCounters;
constexpr size_t kOffPartO = kOffCounters + kZeroBytes;
constexpr size_t kOffPartMl = align256(kOffPartO + sizeof(float) * kNaMaxParts * kNaMaxD);
constexpr int kNaRingQ = 1;  // query rows per consumer-warp record (AttnParams::wpart_q)
constexpr size_t kRingRecs = static_cast<size_t>(kNaMaxCtas) * kPartSlots * kMaxConsumerWarps * kNaRingQ;
constexpr size_t kOffWpartO = align256(kOffPartMl + sizeof(float2) * kNaMaxParts);
constexpr size_t kOffWpartMl = align256(kOffWpartO + sizeof(float) * kRingRecs * kNaMaxD);
constexpr size_t kScratchUsed = align256(kOffWpartMl + sizeof(float2) * kRingRecs);
static_assert(kScratchUsed <= LYC_NOALLOC_SCRATCH_BYTES, "scratch layout exceeds the array");

}  // namespace

// The one scratch array of the allocation-free entry point.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LYC_NOALLOC_SCRATCH_BYTES];

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

// The CTA whose run of tiles holds tile T, when NT tiles are cut into `grid`
// equal runs [NT*c/grid, NT*(c+1)/grid): the largest c with
// floor(NT*c/grid) <= T.
__host__ __device__ inline int64_t cta_of_tile(int64_t T, int64_t NT, int64_t grid) {
  return ((T + 1) * grid + NT - 1) / NT - 1;
}

// One call's work list, computed by the plan kernel below (and its sizes by
// the host, with the same formulas): one gathered segment per (b, h) of
// tiles_per 64-row tiles, the NT = nsets * tiles_per tiles cut into equal
// runs, one per CTA (the pooling of the full step); a run that crosses
// segments becomes several pieces.
struct NaPlanArgs {
  unsigned char* base;        // device address of g_noalloc_scratch
  const unsigned char* kc;    // K and V of the cache (bf16)
  const unsigned char* vc;
  const int32_t* S;           // [B][Hq][k]
  int64_t s_batch, s_head, s_token;
  int64_t NT;                 // tiles of the call
  int32_t B, Hq, G, k, keff, n;
  int32_t tiles_per;          // tiles of one segment
  int32_t grid, cgrid;        // CTAs of the attention and of the combine launch
};

constexpr int kNaPlanThreads = 512;
static_assert(kNaPlanThreads >= kNaMaxSets && kNaPlanThreads >= kNaMaxCtas, "one thread per set and CTA");

// Exclusive prefix sum of one value per thread over the block; *total gets the sum.
__device__ int na_block_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) tmp[warp] = inc;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kNaPlanThreads / 32; ++w) {
    before += w < warp ? tmp[w] : 0;
    all += tmp[w];
  }
  __syncthreads();
  *total = all;
  return before + inc - v;
}

__global__ void __launch_bounds__(kNaPlanThreads) noalloc_plan_kernel(const NaPlanArgs a) {
  __shared__ int tmp[kNaPlanThreads / 32];
  const int t = threadIdx.x;
  const int nsets = a.B * a.Hq;
  const int64_t tp = a.tiles_per;
  // counters and status word start at zero
  uint32_t* zero = reinterpret_cast<uint32_t*>(a.base + kOffCounters);
  for (size_t i = t; i < kZeroBytes / 4; i += kNaPlanThreads) zero[i] = 0u;
  // per segment: the CTAs its tiles fall in
  int npieces = 0;
  int64_t cfirst = 0;
  if (t < nsets) {
    cfirst = cta_of_tile(t * tp, a.NT, a.grid);
    npieces = static_cast<int>(cta_of_tile((t + 1) * tp - 1, a.NT, a.grid) - cfirst + 1);
  }
  // per CTA: the segments its run crosses
  int64_t t0 = 0, t1 = 0, s0 = 0;
  int mine = 0;
  if (t < a.grid) {
    t0 = a.NT * t / a.grid;
    t1 = a.NT * (t + 1) / a.grid;
    s0 = t0 / tp;
    mine = static_cast<int>((t1 - 1) / tp - s0 + 1);
  }
  int parts = 0, pieces = 0, ntasks = 0;
  const int part_base = na_block_scan(npieces, tmp, &parts);
  const int task_pos = na_block_scan(npieces > 1 ? 1 : 0, tmp, &ntasks);
  const int piece0 = na_block_scan(mine, tmp, &pieces);
  Segment* segs = reinterpret_cast<Segment*>(a.base + kOffSegs);
  Piece* pcs = reinterpret_cast<Piece*>(a.base + kOffPieces);
  int32_t* cta = reinterpret_cast<int32_t*>(a.base + kOffCta);
  int2* tasks = reinterpret_cast<int2*>(a.base + kOffTasks);
  int32_t* empty_cta = reinterpret_cast<int32_t*>(a.base + kOffEmptyCta);
  if (t < nsets) {
    const int b = t / a.Hq, h = t % a.Hq, g = h / a.G;
    const int64_t off = b * a.s_batch + g * a.s_head;
    Segment sg{};
    sg.k = a.kc + off * 2;
    sg.v = a.vc + off * 2;
    sg.idx = a.S + static_cast<int64_t>(t) * a.k;
    sg.s_token = a.s_token;
    for (int j = 0; j < kMaxQ; ++j) sg.key_off[j] = -1;
    sg.key_mean_off = -1;
    sg.kind = kSparse;
    sg.b = b;
    sg.g = g;
    sg.rows = a.keff;
    sg.nvalid = a.n;
    sg.nq = sg.nout = 1;
    sg.dep = 1;  // the caller's sets: read after whatever ran before on the stream
    sg.head[0] = h;
    sg.part_base = part_base;
    sg.npieces = npieces;
    sg.cnt_base = t;
    segs[t] = sg;
    if (npieces > 1) tasks[task_pos] = make_int2(t, 0);
  }
  if (t < a.grid) {
    cta[t] = piece0;
    for (int i = 0; i < mine; ++i) {
      const int64_t si = s0 + i;
      const int64_t lo = (t0 > si * tp ? t0 : si * tp) - si * tp;
      const int64_t hi = (t1 < (si + 1) * tp ? t1 : (si + 1) * tp) - si * tp;
      Piece pc;
      pc.seg = static_cast<int32_t>(si);
      pc.r0 = static_cast<int32_t>(lo * kTileRows);
      pc.r1 = static_cast<int32_t>(hi * kTileRows < a.keff ? hi * kTileRows : a.keff);
      pc.ordinal = static_cast<int32_t>(t - cta_of_tile(si * tp, a.NT, a.grid));
      pcs[piece0 + i] = pc;
    }
  }
  if (t == 0) cta[a.grid] = pieces;
  if (t <= a.cgrid) empty_cta[t] = 0;
}

// Once per device, with that device current: the array's address, the
// driver's tensor-map encoder and the kernel's shared-memory attribute.
lyc_status setup_device(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return LYC_ERR_UNSUPPORTED;
  DeviceState& ds = g_dev[dev];
  if (!ds.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return LYC_ERR_CUDA;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess)
        return LYC_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    int smem = 0;
    for (int D : {64, 128})
      if (attn_mma_dispatch(D, nullptr, 0, nullptr, &smem, true) != cudaSuccess) return LYC_ERR_CUDA;
    ds.scratch = static_cast<unsigned char*>(ptr);
    ds.ready = true;
  }
  *out = &ds;
  return LYC_OK;
}

// 5-D map (d, row, KV head, batch, 1 layer) of one cache tensor, as the
// kernel expects; only the gathered path runs here, but the kernel
// prefetches the maps it is given, so they are real ones.
bool encode_map(CUtensorMap* map, const void* base, const lyc_kv_cache* kv, int B, int Hkv, int d) {
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(kv->n),
                              static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(B), 1};
  int64_t st[4] = {kv->s_token * 2, kv->s_head * 2, kv->s_batch * 2, 0};
  if (Hkv == 1 && st[1] == 0) st[1] = st[0] * static_cast<int64_t>(kv->n);
  if (B == 1 && st[2] == 0) st[2] = st[1] * Hkv;
  st[3] = st[2] * B;
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(st[0]), static_cast<cuuint64_t>(st[1]),
                                 static_cast<cuuint64_t>(st[2]), static_cast<cuuint64_t>(st[3])};
  const cuuint32_t box[5] = {64, static_cast<cuuint32_t>(kTileRows), 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace lyc

extern "C" lyc_status lyc_sparse_attention_noalloc(const void* q, const lyc_kv_cache* kv, int batch,
                                                   int num_q_heads, int num_kv_heads, int head_dim,
                                                   const int32_t* S, int k, float* out,
                                                   uint32_t* status, void* stream_) {
  using namespace lyc;
  // ---- arguments
  if (!q || !kv || !kv->k || !kv->v || !S || !out) return LYC_ERR_INVALID_ARG;
  if (batch < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0)
    return LYC_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LYC_ERR_UNSUPPORTED;
  if (num_q_heads / num_kv_heads > kMaxGroup) return LYC_ERR_UNSUPPORTED;
  if (k < 1 || (k & 3) != 0 || kv->n < 1 || kv->n > 0x7fffffffll) return LYC_ERR_INVALID_ARG;
  if (kv->s_token < head_dim || kv->s_batch < 0 || kv->s_head < 0) return LYC_ERR_INVALID_ARG;
  if (((kv->s_token | kv->s_head | kv->s_batch) * 2) % 16 != 0) return LYC_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(kv->k) | reinterpret_cast<uintptr_t>(kv->v) |
        reinterpret_cast<uintptr_t>(S)) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(out) & 15u) != 0)
    return LYC_ERR_INVALID_ARG;
  const int B = batch, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
  const int G = Hq / Hkv;
  const int nsets = B * Hq;
  if (nsets > kNaMaxSets) return LYC_ERR_SCRATCH_LIMIT;
  const int n = static_cast<int>(kv->n);
  const int keff = std::min(k, n);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LYC_ERR_CUDA;
  DeviceState* ds = nullptr;
  lyc_status st = setup_device(dev, &ds);
  if (st != LYC_OK) return st;

  // ---- the work list's sizes (the plan kernel builds the list itself)
  unsigned char* dbase = ds->scratch;
  const int tiles_per = (keff + kTileRows - 1) / kTileRows;
  const int64_t NT = static_cast<int64_t>(tiles_per) * nsets;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LYC_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>({NT, static_cast<int64_t>(kNaMaxCtas),
                                                       static_cast<int64_t>(sms)}));
  int64_t part = 0;
  int ntasks = 0;
  for (int s = 0; s < nsets; ++s) {
    const int64_t np = cta_of_tile(static_cast<int64_t>(s + 1) * tiles_per - 1, NT, grid) -
                       cta_of_tile(static_cast<int64_t>(s) * tiles_per, NT, grid) + 1;
    part += np;
    ntasks += np > 1 ? 1 : 0;
  }
  // pieces = partials (one output each); a cut of NT tiles into `grid` runs
  // and nsets segments has at most grid + nsets - 1 of them
  if (part > kNaMaxParts || part > kNaMaxPieces) return LYC_ERR_SCRATCH_LIMIT;
  const int cgrid = std::max(1, std::min(ntasks, grid));
  NaPlanArgs pa;
  pa.base = dbase;
  pa.kc = static_cast<const unsigned char*>(kv->k);
  pa.vc = static_cast<const unsigned char*>(kv->v);
  pa.S = S;
  pa.s_batch = kv->s_batch;
  pa.s_head = kv->s_head;
  pa.s_token = kv->s_token;
  pa.NT = NT;
  pa.B = B;
  pa.Hq = Hq;
  pa.G = G;
  pa.k = k;
  pa.keff = keff;
  pa.n = n;
  pa.tiles_per = tiles_per;
  pa.grid = grid;
  pa.cgrid = cgrid;

  AttnMmaParams mp;
  memset(&mp, 0, sizeof mp);
  if (!encode_map(&mp.tmk, kv->k, kv, B, Hkv, D) || !encode_map(&mp.tmv, kv->v, kv, B, Hkv, D))
    return LYC_ERR_INVALID_ARG;
  mp.tgk = mp.tmk;
  mp.tgv = mp.tmv;
  AttnParams& ap = mp.p;
  ap.segs = reinterpret_cast<const Segment*>(dbase + kOffSegs);
  ap.pieces = reinterpret_cast<const Piece*>(dbase + kOffPieces);
  ap.cta_begin = reinterpret_cast<const int32_t*>(dbase + kOffCta);
  ap.q = q;
  ap.out = out;
  ap.keys = nullptr;
  ap.part_o = reinterpret_cast<float*>(dbase + kOffPartO);
  ap.part_ml = reinterpret_cast<float2*>(dbase + kOffPartMl);
  ap.counters = reinterpret_cast<int32_t*>(dbase + kOffCounters);
  ap.wpart_o = reinterpret_cast<float*>(dbase + kOffWpartO);
  ap.wpart_ml = reinterpret_cast<float2*>(dbase + kOffWpartMl);
  ap.wpart_by_sm = 0;  // one ring per CTA: the two launches of a call never overlap on an SM ring
  ap.wpart_slots = kNaMaxCtas;
  ap.wpart_q = kNaRingQ;
  ap.wait_prev = 1;    // the plan kernel's work list is complete before any CTA reads it
  ap.status = reinterpret_cast<uint32_t*>(dbase + kOffStatus);
  ap.timeline = nullptr;
  ap.timeline_cap = 0;
  ap.layer = 0;
  ap.Hq = Hq;
  ap.G = G;
  ap.n = n;
  ap.gather_rows = 0;  // gathered rows by cp.async
  ap.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(D)));
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));

  // the combine launch: no pieces, this launch's partials as its "previous layer"
  AttnMmaParams cmp = mp;
  cmp.p.cta_begin = reinterpret_cast<const int32_t*>(dbase + kOffEmptyCta);
  cmp.p.prev_segs = ap.segs;
  cmp.p.prev_tasks = reinterpret_cast<const int2*>(dbase + kOffTasks);
  cmp.p.prev_ntasks = ntasks;
  cmp.p.prev_part_o = ap.part_o;
  cmp.p.prev_part_ml = ap.part_ml;
  cmp.p.prev_out = out;

  // ---- enqueue: the work list (and cleared counters and status), the
  // kernel, the combine, the status out
  noalloc_plan_kernel<<<1, kNaPlanThreads, 0, stream>>>(pa);
  if (cudaGetLastError() != cudaSuccess || attn_mma_dispatch(D, &mp, grid, stream, nullptr, false) != cudaSuccess)
    return LYC_ERR_CUDA;
  if (ntasks > 0 && attn_mma_dispatch(D, &cmp, cgrid, stream, nullptr, false) != cudaSuccess)
    return LYC_ERR_CUDA;
  if (status && cudaMemcpyAsync(status, dbase + kOffStatus, sizeof(uint32_t), cudaMemcpyDefault,
                                stream) != cudaSuccess)
    return LYC_ERR_CUDA;
  return LYC_OK;
}
