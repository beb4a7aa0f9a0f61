// noalloc.cu -- lyc_sparse_attention_noalloc: the sparse-head attention of
// one layer (page "LycheeDecode ...", paper-graph-ui summary, section 3.4
// Eq. 3) for callers that cannot allocate device memory.
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
// once per device with cudaGetSymbolAddress.  Per call the host builds the
// work list in a fixed host buffer and copies it in; the counters and the
// status word are cleared on the stream first.  No cudaMalloc, cudaFree or
// allocating library routine is called.
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

struct AttnMmaParams {  // layout shared with attn_mma_kernel.cu
  CUtensorMap tmk;
  CUtensorMap tmv;
  CUtensorMap tgk;
  CUtensorMap tgv;
  AttnParams p;
};
cudaError_t attn_mma_dispatch(int D, const AttnMmaParams* P, int grid, cudaStream_t stream,
                              int* smem_out, bool configure_only);

namespace {

// Limits of one call (they size the array below).
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
constexpr size_t kRingRecs = static_cast<size_t>(kNaMaxCtas) * kPartSlots * kMaxConsumerWarps * kMaxQ;
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
// host staging of one call's work list (guarded by g_mu)
unsigned char g_host_plan[kPlanBytes];

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

  // ---- work list: one gathered segment per (b, h), its rows cut into equal
  // runs of 64-row tiles, one run per CTA (the pooling of the full step)
  unsigned char* dbase = ds->scratch;
  Segment* segs = reinterpret_cast<Segment*>(g_host_plan + kOffSegs);
  Piece* pieces = reinterpret_cast<Piece*>(g_host_plan + kOffPieces);
  int32_t* cta = reinterpret_cast<int32_t*>(g_host_plan + kOffCta);
  const int tiles_per = (keff + kTileRows - 1) / kTileRows;
  const int64_t NT = static_cast<int64_t>(tiles_per) * nsets;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LYC_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>({NT, static_cast<int64_t>(kNaMaxCtas),
                                                       static_cast<int64_t>(sms)}));
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      Segment& sg = segs[b * Hq + h];
      memset(&sg, 0, sizeof sg);
      const int g = h / G;
      const int64_t off = b * kv->s_batch + g * kv->s_head;
      sg.k = static_cast<const unsigned char*>(kv->k) + off * 2;
      sg.v = static_cast<const unsigned char*>(kv->v) + off * 2;
      sg.idx = S + static_cast<int64_t>(b * Hq + h) * k;
      sg.s_token = kv->s_token;
      for (int j = 0; j < kMaxQ; ++j) sg.key_off[j] = -1;
      sg.key_mean_off = -1;
      sg.kind = kSparse;
      sg.l = 0;
      sg.b = b;
      sg.g = g;
      sg.rows = keff;
      sg.nvalid = static_cast<int32_t>(n);
      sg.nq = sg.nout = 1;
      sg.dep = 1;  // the caller's sets: read after whatever ran before on the stream
      sg.head[0] = h;
      sg.out_row[0] = 0;
    }
  }
  int npc = 0;
  {
    int64_t si = 0;
    for (int c = 0; c < grid; ++c) {
      cta[c] = npc;
      const int64_t t0 = NT * c / grid, t1 = NT * (c + 1) / grid;
      for (si = t0 / tiles_per; si < nsets && si * tiles_per < t1; ++si) {
        const int64_t a = std::max(t0, si * tiles_per) - si * tiles_per;
        const int64_t e = std::min(t1, (si + 1) * tiles_per) - si * tiles_per;
        if (e <= a) continue;
        Piece& pc = pieces[npc++];
        pc.seg = static_cast<int32_t>(si);
        pc.r0 = static_cast<int32_t>(a * kTileRows);
        pc.r1 = static_cast<int32_t>(std::min<int64_t>(e * kTileRows, keff));
        pc.ordinal = segs[si].npieces++;
      }
    }
    cta[grid] = npc;
  }
  if (npc > kNaMaxPieces) return LYC_ERR_SCRATCH_LIMIT;
  // partials: one per piece; segments cut into several pieces are combined
  // by a second launch of the same kernel, one (segment, output 0) task each
  int2* tasks = reinterpret_cast<int2*>(g_host_plan + kOffTasks);
  int32_t* empty_cta = reinterpret_cast<int32_t*>(g_host_plan + kOffEmptyCta);
  int part = 0, ntasks = 0;
  for (int s = 0; s < nsets; ++s) {
    segs[s].part_base = part;
    segs[s].cnt_base = s;
    part += segs[s].npieces;
    if (segs[s].npieces > 1) tasks[ntasks++] = make_int2(s, 0);
  }
  if (part > kNaMaxParts) return LYC_ERR_SCRATCH_LIMIT;
  const int cgrid = std::max(1, std::min(ntasks, grid));
  for (int c = 0; c <= cgrid; ++c) empty_cta[c] = 0;

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

  // ---- enqueue: work list in, counters and status cleared, the kernel, the
  // combine, the status out
  if (cudaMemcpyAsync(dbase, g_host_plan, kPlanBytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemsetAsync(dbase + kOffCounters, 0, kZeroBytes, stream) != cudaSuccess ||
      attn_mma_dispatch(D, &mp, grid, stream, nullptr, false) != cudaSuccess)
    return LYC_ERR_CUDA;
  if (ntasks > 0 && attn_mma_dispatch(D, &cmp, cgrid, stream, nullptr, false) != cudaSuccess)
    return LYC_ERR_CUDA;
  if (status && cudaMemcpyAsync(status, dbase + kOffStatus, sizeof(uint32_t), cudaMemcpyDefault,
                                stream) != cudaSuccess)
    return LYC_ERR_CUDA;
  return LYC_OK;
}
