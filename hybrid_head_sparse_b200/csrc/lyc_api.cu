// lyc_api.cu -- host side of liblyc.so: argument checks, the per-layer work
// planner (workload pooling), set-buffer bookkeeping, CUDA-graph capture and
// the C entry points declared in include/lyc.h.
//
// The step follows the decode loop of page "LycheeDecode ..." (paper-graph-ui
// summary), Appendix B / Algorithm 1, attention part: per layer, retrieval
// heads attend densely and re-select their set, sparse heads attend over the
// set they inherit and pass it on; layer 0 is all retrieval.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <list>
#include <memory>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/lyc.h"
#include "lyc_plan.h"

namespace lyc {
int attn_nq_bucket(int nq);
cudaError_t attn_simt_dispatch(int D, int nqb, const AttnParams* p, int grid, cudaStream_t stream,
                               int* smem_out, bool configure_only);
int attn_mma_consumer_warps(int D);
cudaError_t attn_mma_dispatch(int D, const AttnMmaParams* P, int grid, cudaStream_t stream,
                              int* smem_out, bool configure_only);
cudaError_t attn_tc_dispatch(const AttnMmaParams* P, int grid, cudaStream_t stream, int* smem_out,
                             bool configure_only);
int attn_tc_tile_rows();
size_t topk_smem_for(int cl, int n);
int topk_pick_cluster(size_t smem);
cudaError_t topk_configure(int cl, size_t smem);
cudaError_t topk_launch(int cl, const TopkParams* p, int ntasks, cudaStream_t stream, bool force_var);
int topk_max_clusters(int cl, size_t smem);
cudaError_t copy_sets_launch(const CopySetsParams* p, cudaStream_t stream);
cudaError_t append_rows_launch(const AppendParams* p, cudaStream_t stream);
cudaError_t validate_sets_launch(const ValidateSetsParams* p, cudaStream_t stream);
int correction_smem_bytes();
cudaError_t correction_configure();
cudaError_t correction_launch(const CorrParams* P, int grid, const WriteRowsParams* rows,
                              cudaStream_t stream);
}  // namespace lyc

using namespace lyc;

namespace {

constexpr int kMaxCtxLimit = 655360;  // 16-CTA top-k keeps every key in shared memory
constexpr int kPlanCacheSize = 16;
// Layers per attention launch (mma kernel): each launch runs the dense rows
// and gathered rows of several consecutive layers, so that a CTA's fixed
// cost (its start, the wait for its first tiles, its drain: ~7 us, about
// what the step streams in 45 MB) is paid once per that many layers; the
// selections stay one launch per layer.  Two layers per launch for layers
// that read at least kSmallLayerBytes; below, four with per-head selection
// and eight with KV-group selection, whose gathered rows (one set per
// sparse group, not per sparse head) are a small share of a layer's bytes.
// Measured on B200: 128K Llama3-8B shapes, ~151 MB per later layer: 1047
// steps/s with two layers per launch, 1026 with three, 1037 with four,
// ~1001 with one; 32K, ~50 MB per layer: 2081, 2149, 2182 and ~1750.  With
// selections on clusters of 4: 128K 1078 with two against 1065 with four;
// 32K KV-group 2287 with eight against 2230 with four, per head 1451
// against 1476.  When no layer after the first selects (every later head a
// sparse head, so layer 0's sets serve the whole step), only layer 0's
// readers are deferred and a launch holds eight layers (128K with no later
// retrieval heads: 3889 against 3478 steps/s with four).
constexpr int kLayersPerLaunch = 8;  // at most
constexpr double kSmallLayerBytes = 96e6;
// Buffers per set slot.  A selection overwrites the set that its slot held
// kSetBuffers refreshes earlier.  That set's last readers run in the launch
// of the layer that last read it, or, for a deferred pass, of the layer
// after; a selection waits only for the attention launch before its own
// layer's launch, so kLayersPerLaunch + 2 buffers keep every reader of the
// overwritten set in a launch that has completed.
constexpr int kSetBuffers = kLayersPerLaunch + 2;


int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// One layer of a plan: offsets of its records in the plan's device buffer.
struct LayerPlan {
  int nseg = 0, npieces = 0, grid = 0, nqb = 1;
  size_t off_segs = 0, off_pieces = 0, off_cta = 0;
  int ntasks = 0;
  size_t off_tasks = 0;
  size_t off_combine = 0;    // bf16: (segment, output) pairs combined by the next launch
  int ncombine = 0;
  size_t off_pool = 0;       // mma kernel: the pool's units
  int pool_n = 0;             // units in the pool
  int64_t pool_tiles = 0, tiles = 0;  // tiles in the pool, in the whole layer
  int topk_cl = 16;          // cluster size of the selection launch
  int topk_n = 0;            // keys of the longest selection task
  int keys_ctas = 0;         // CTAs with dense pieces of this layer (the writers of its keys)
  std::vector<FirstPiece> first;  // mma kernel: each CTA's first piece, for the launch parameters
  // the attention launch: this layer's record holds it when the layer is the
  // first of the launch's layers [layer, layer + nlayers); the other layers
  // of the launch have none (attn false) but keep their selection launch
  bool attn = true;
  int nlayers = 1;
  int launch = 0;            // ordinal of the attention launch in the step
};

struct Plan {
  std::vector<LayerPlan> layers;
  unsigned char* dev = nullptr;  // all records of all layers
  size_t dev_bytes = 0;
  size_t off_final_src = 0;      // copy table: current buffer of each set -> caller S
  // set trace: the selections write their rows of it; one copy at the end of
  // the step fills the rows of the sets a layer did not refresh
  size_t off_fill_src = 0, off_fill_dst = 0;
  int nfill = 0;
  int nsets = 0;
  int combine_grid = 1;       // bf16: CTAs of the launch that combines the last layer
  size_t off_empty_cta = 0;   // its CTA offsets (all zero: no pieces)
  int k = 0, keff = 0, n = 0;
  std::vector<int64_t> nb;        // rows of each batch element
  std::vector<int> set_rows;      // capacity of each batch element's sets (rows)
  bool variable = false;          // sets may be shorter than their capacity (-1 padded)
  lyc_selection sel{};            // the selection rule the plan was built for
  bool append = false;            // the step writes the current token's K and V first
  bool paged = false;             // the cache is paged
  AppendParams ap_append{};       // (its n array lives in the plan buffer)
  size_t off_n = 0;
  uint32_t flags = 0;
  const void* q = nullptr;
  float* out = nullptr;
  int32_t* S = nullptr;
  int32_t* trace = nullptr;
  bool timing = false;
  unsigned long long* timeline = nullptr;
  int timeline_cap = 0;
  CUtensorMap tmk{}, tmv{};       // bf16 path: 5-D maps of the whole K and V cache
  CUtensorMap tgk{}, tgv{};       // bf16 path: 2-D row-gather maps (when gather_rows > 0)
  int32_t gather_rows = 0;        // rows of the row-gather maps; 0 = none
  bool use_tc = false;            // bf16: the tcgen05 attention kernel
  cudaGraphExec_t exec = nullptr;
  // timing: event-record nodes of the graph, in launch order (2 per kernel)
  std::vector<cudaGraphNode_t> ev_nodes;
  cudaGraph_t graph = nullptr;
  std::vector<int> kernel_kind, kernel_layer;  // per timed kernel
};

}  // namespace

struct lyc_ctx {
  lyc_config cfg{};
  int G = 1, Hs = 1, sms = 1, topk_cl = 8;
  unsigned topk_cls = 0;  // bit c: cluster size c is configured for max_ctx (c in 4, 8, 16)
  int topk_resident[17] = {};  // clusters of size c resident at once (at max_ctx's smem)
  int64_t nstride = 0;  // row stride of the key buffer
  int KS = 0;           // row stride of the set buffers
  std::string err;
  uint32_t* status = nullptr;
  float* keys = nullptr;
  int32_t* sbuf = nullptr;  // [kSetBuffers][B][Hs][KS]
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  // bf16 path: per CTA ring of the consumer warps' piece states
  float* wpart_o = nullptr;
  float2* wpart_ml = nullptr;
  int wpart_slots = 0;
  // per (layer, b, slot): {arrival counter, ready flag} of the selection task
  // that writes the slot at that layer; then the step counters; then the
  // step epoch
  uint32_t* flags = nullptr;
  // step counters [2][3][L + 1], by epoch parity: the pool cursor, the
  // completion counter and the selection-key counter of each attention launch
  // (zeroed for the next step by the step's last launch)
  int32_t* pool_cursors = nullptr;
  uint32_t* epoch = nullptr;
  int32_t* counters = nullptr;
  size_t max_parts = 0, max_counters = 0;
  // host-buffer entry point staging
  void* q_dev = nullptr;
  float* out_dev = nullptr;
  int32_t* S_dev = nullptr;
  int32_t* trace = nullptr;
  cudaStream_t last_stream = nullptr;
  int last_launches[3] = {-1, 0, 0};  // the most recent step's attention, selection, other launches
  bool timing = false;
  unsigned long long* timeline = nullptr;  // caller's buffer, or NULL
  int timeline_cap = 0;
  // the selection rule of the steps (lyc_set_selection)
  lyc_selection sel{};
  // Cache Correction: the work pool of the last (n, T) (pieces, CTA offsets,
  // group offsets in one device buffer) and the piece partials
  unsigned char* corr_dev = nullptr;
  int64_t corr_n = -1;
  int corr_T = -1, corr_grid = 0, corr_npieces = 0;
  size_t corr_off_cta = 0, corr_off_group = 0;
  float* corr_part_o = nullptr;
  float2* corr_part_ml = nullptr;
  size_t corr_parts_cap = 0;
  bool corr_configured = false;
  // plans, most recent first
  std::list<std::pair<std::string, std::unique_ptr<Plan>>> plans;
  // timing pool
  std::vector<cudaEvent_t> events;        // kTimingSets * events_per_set
  int events_per_set = 0;
  struct Recorded { int set; Plan* plan; };
  std::vector<Recorded> recorded;
  int next_set = 0;
};

namespace {

lyc_status fail(lyc_ctx* c, lyc_status s, const std::string& msg) {
  if (c) c->err = msg;
  return s;
}

lyc_status cuda_fail(lyc_ctx* c, cudaError_t e, const char* what) {
  if (c) c->err = std::string(what) + ": " + cudaGetErrorString(e);
  return LYC_ERR_CUDA;
}

#define LYC_CUDA(call, what)                        \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_fail(ctx, e_, what); \
  } while (0)

void free_plan(Plan* p) {
  if (!p) return;
  if (p->exec) cudaGraphExecDestroy(p->exec);
  if (p->graph) cudaGraphDestroy(p->graph);
  if (p->dev) cudaFree(p->dev);
  p->exec = nullptr;
  p->graph = nullptr;
  p->dev = nullptr;
}

}  // namespace

namespace {

// ---------------------------------------------------------------- KV views
// The KV cache of one step, from either entry point: every batch element's
// row count, and contiguous or paged rows (the layout of lyc_kv_batch).
struct KvView {
  const void* k = nullptr;
  const void* v = nullptr;
  int64_t nmax = 0;
  std::vector<int64_t> n;  // per batch element
  int64_t s_layer = 0, s_batch = 0, s_head = 0, s_token = 0, s_page = 0;
  const int32_t* bt = nullptr;
  int32_t page_rows = 0, max_blocks = 0;
  int64_t num_pages = 0;
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  bool paged() const { return bt != nullptr; }
};

KvView view_of(const lyc_kv_cache* kv, int B) {
  KvView w;
  w.k = kv->k;
  w.v = kv->v;
  w.nmax = kv->n;
  w.n.assign(B, kv->n);
  w.s_layer = kv->s_layer;
  w.s_batch = kv->s_batch;
  w.s_head = kv->s_head;
  w.s_token = kv->s_token;
  return w;
}

KvView view_of(const lyc_kv_batch* kv, int B) {
  KvView w;
  w.k = kv->k;
  w.v = kv->v;
  w.n.assign(kv->n, kv->n + B);
  for (int64_t x : w.n) w.nmax = std::max(w.nmax, x);
  w.s_layer = kv->s_layer;
  w.s_batch = kv->s_batch;
  w.s_head = kv->s_head;
  w.s_token = kv->s_token;
  w.s_page = kv->s_page;
  w.bt = kv->block_table;
  w.page_rows = kv->page_rows;
  w.max_blocks = kv->max_blocks;
  w.num_pages = kv->num_pages;
  w.k_new = kv->k_new;
  w.v_new = kv->v_new;
  return w;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 5-D map of one cache tensor, 64 x 64 boxes of 128-byte rows with the 128B
// swizzle: contiguous rows (d, row, KV head, batch, layer), rows at or past
// the longest element's n read as zeros; or paged (d, KV head, row in page,
// page, layer), a box never crossing a page.
lyc_status encode_cache_map(lyc_ctx* ctx, CUtensorMap* map, const void* base, const KvView& kv,
                            int tile_rows) {
  const lyc_config& c = ctx->cfg;
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return fail(ctx, LYC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const int64_t es = 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(c.head_dim), static_cast<cuuint64_t>(kv.nmax),
                        static_cast<cuuint64_t>(c.num_kv_heads), static_cast<cuuint64_t>(c.batch),
                        static_cast<cuuint64_t>(c.num_layers)};
  int64_t st[4] = {kv.s_token * es, kv.s_head * es, kv.s_batch * es, kv.s_layer * es};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(tile_rows), 1, 1, 1};
  if (kv.paged()) {
    dims[1] = static_cast<cuuint64_t>(c.num_kv_heads);
    dims[2] = static_cast<cuuint64_t>(kv.page_rows);
    dims[3] = static_cast<cuuint64_t>(kv.num_pages);
    st[0] = kv.s_head * es;
    st[1] = kv.s_token * es;
    st[2] = kv.s_page * es;
    box[1] = 1;
    box[2] = static_cast<cuuint32_t>(tile_rows);
  }
  // a dimension of extent 1 is only ever read at coordinate 0: give it a
  // harmless stride if the caller passed 0
  for (int i = 0; i < 4; ++i)
    if (dims[i + 1] == 1 && st[i] == 0) st[i] = (i == 0 ? c.head_dim * es : st[i - 1] * static_cast<int64_t>(dims[i]));
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(st[0]), static_cast<cuuint64_t>(st[1]),
                                 static_cast<cuuint64_t>(st[2]), static_cast<cuuint64_t>(st[3])};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, LYC_ERR_INVALID_ARG, "cuTensorMapEncodeTiled rejected the cache layout (code " +
                                              std::to_string(static_cast<int>(r)) + ")");
  return LYC_OK;
}

// Rows of a flattened 2-D view (d, row) of the cache in which row
// (l*s_layer + b*s_batch + g*s_head)/s_token + i is token i of (l, b, g), or 0
// when the strides do not allow one (a head, batch or layer stride that is
// not a whole number of rows) or the rows do not fit a 32-bit coordinate.
int64_t gather_map_rows(const lyc_config& c, const KvView& kv) {
  const int64_t st = kv.s_token;
  if (st <= 0 || kv.paged()) return 0;
  if ((c.num_kv_heads > 1 && kv.s_head % st) || (c.batch > 1 && kv.s_batch % st) ||
      (c.num_layers > 1 && kv.s_layer % st))
    return 0;
  if (kv.s_head < 0 || kv.s_batch < 0 || kv.s_layer < 0) return 0;
  const int64_t last = (c.num_layers - 1) * kv.s_layer + (c.batch - 1) * kv.s_batch +
                       (c.num_kv_heads - 1) * kv.s_head;
  const int64_t rows = last / st + kv.nmax;
  return rows < 0x7fffffffll ? rows : 0;
}

// The 2-D row-gather map of one cache tensor: boxes of one 128-byte row
// (64 bf16), 128B swizzle, so that a four-row gather lands in the same
// swizzled tile layout as the 5-D map's tiles.
lyc_status encode_gather_map(lyc_ctx* ctx, CUtensorMap* map, const void* base, const KvView& kv,
                             int64_t rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return fail(ctx, LYC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(ctx->cfg.head_dim), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kv.s_token * 2)};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(ctx, LYC_ERR_INVALID_ARG, "cuTensorMapEncodeTiled rejected the row-gather view (code " +
                                              std::to_string(static_cast<int>(r)) + ")");
  return LYC_OK;
}

// Cluster size of a selection launch of `ntasks` sets.  A small selection (a
// few sets) takes clusters of 4 and runs beside the attention launches, on
// SMs that the planner leaves out of their grid: room for two selections, so
// that a layer's selection can start on its keys while the one before still
// runs.  Its time is off the step's critical path (passes over its sets run
// in later launches), so the SMs it does not take are worth more to the
// attention grid.  (Measured on B200 at 128K keys, 2 retrieval heads per
// layer, two layers per attention launch: clusters of 4, grid 132, 1082
// steps/s against 1047 with clusters of 8, grid 116; per head 840 against
// 801; 32K 2230 against 2172.  With one layer per launch clusters of 8
// won, 999 against 983.)  The size rules and block selection (variable) do
// more work per key, and on clusters of 4 their selections last long enough
// to hold up the passes over their sets: clusters of 8 (measured: top-p 0.5
// 998 against 894 steps/s, threshold 1120 against 1082, block 1040 against
// 1030).  Layer 0's selection (first), when its sets fit on clusters of 4
// in a quarter of the SMs, takes clusters of 4: it starts as its launch ends
// and holds SMs that the next launch's CTAs are waiting for (measured: 1084
// against 1077-1079 steps/s with clusters of 8, 8 sets at 128K).  Another
// large selection takes the largest size whose clusters are all resident at
// once, so that it runs in one wave and the next layer starts right away;
// else the smallest size.
int pick_topk_cluster(const lyc_ctx* ctx, int ntasks, bool variable, bool first) {
  auto resident = [&](int cl) {
    return ctx->topk_resident[cl] > 0 ? ctx->topk_resident[cl] : ctx->sms / cl;
  };
  const int small = variable ? 8 : 4;
  if (2 * ntasks * small <= ctx->sms / 4 && (ctx->topk_cls & (1u << small)) && ntasks <= resident(small))
    return small;
  if (first && !variable && ntasks * 4 <= ctx->sms / 4 && (ctx->topk_cls & (1u << 4)) && ntasks <= resident(4))
    return 4;
  int best = 0, smallest = 0;
  for (int cl : {16, 8, 4}) {
    if (!(ctx->topk_cls & (1u << cl))) continue;
    smallest = cl;
    if (!best && ntasks <= resident(cl)) best = cl;
  }
  return best ? best : smallest;
}

// ---------------------------------------------------------------- planner
//
// Builds every launch's work pool for one (role mask, n, k, flags, pointers)
// combination and uploads it in one buffer.  Set buffers: each set slot has
// kSetBuffers buffers; a refreshed slot is written into the next one in turn,
// never one that a pass still in flight may read (see kSetBuffers), and
// unrefreshed slots cost no copy.
lyc_status build_plan(lyc_ctx* ctx, Plan* plan, const uint8_t* role, const KvView& kv,
                      int k, uint32_t flags) {
  const lyc_config& cfg = ctx->cfg;
  const int L = cfg.num_layers, B = cfg.batch, Hq = cfg.num_q_heads, Hkv = cfg.num_kv_heads;
  const int G = ctx->G, Hs = ctx->Hs;
  const bool kvmode = cfg.select_mode == LYC_SELECT_KVGROUP_MEAN;
  const bool s_in = (flags & LYC_STEP_S_IN) != 0;
  const int n = static_cast<int>(kv.nmax);  // the longest element's rows
  const int keff = std::min(k, n);
  const size_t es = cfg.dtype == LYC_BF16 ? 2 : 4;
  plan->k = k;
  plan->keff = keff;
  plan->n = n;
  plan->nb = kv.n;
  // the selection rule: how many keys a task selects at most (blocks, for
  // block selection), and the capacity of the sets it writes (rows)
  const lyc_selection sel = ctx->sel;
  plan->sel = sel;
  const int E = sel.rule == LYC_RULE_BLOCK_TOPK ? sel.block : 1;
  if (sel.rule == LYC_RULE_BLOCK_TOPK && k < E)
    return fail(ctx, LYC_ERR_INVALID_ARG, "block selection needs k >= block");
  plan->variable = sel.rule == LYC_RULE_BLOCK_TOPK || sel.rule == LYC_RULE_TOPP ||
                   sel.rule == LYC_RULE_THRESHOLD;
  auto select_cap = [&](int64_t nb) -> int {  // keys (blocks) selected at most
    if (sel.rule == LYC_RULE_RATIO) {
      const int64_t m = (sel.ratio_num * nb + sel.ratio_den - 1) / sel.ratio_den;
      return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({m, k, nb})));
    }
    if (sel.rule == LYC_RULE_BLOCK_TOPK) return static_cast<int>(std::min<int64_t>(k / E, (nb + E - 1) / E));
    return static_cast<int>(std::min<int64_t>(k, nb));
  };
  auto set_rows = [&](int64_t nb) -> int {  // rows a set holds at most
    if (sel.rule == LYC_RULE_BLOCK_TOPK) return static_cast<int>(std::min<int64_t>((k / E) * E, nb));
    return select_cap(nb);
  };
  plan->set_rows.clear();
  for (int b = 0; b < B; ++b) plan->set_rows.push_back(set_rows(kv.n[b]));
  plan->paged = kv.paged();
  plan->nsets = B * Hs;
  plan->gather_rows = 0;
  // bf16 with head_dim 128 runs on the tcgen05 kernel (128-row tiles) when
  // the config asks for it (and q is 16-byte aligned), else on the mma.sync one
  plan->use_tc = cfg.dtype == LYC_BF16 && cfg.head_dim == 128 && (cfg.flags & LYC_CFG_TCGEN05) &&
                 !(cfg.flags & LYC_CFG_TMA_GATHER) && (reinterpret_cast<uintptr_t>(plan->q) & 15u) == 0;
  const int TR = plan->use_tc ? attn_tc_tile_rows() : kTileRows;
  // the mma kernel takes gathered rows from a pool at run time (its launches
  // of consecutive layers may overlap, see enqueue)
  const bool use_pool = cfg.dtype == LYC_BF16 && !plan->use_tc;
  if (cfg.dtype == LYC_BF16) {
    lyc_status st = encode_cache_map(ctx, &plan->tmk, kv.k, kv, TR);
    if (st == LYC_OK) st = encode_cache_map(ctx, &plan->tmv, kv.v, kv, TR);
    if (st != LYC_OK) return st;
    const int64_t rows = (cfg.flags & LYC_CFG_TMA_GATHER) ? gather_map_rows(cfg, kv) : 0;
    if (rows > 0) {
      st = encode_gather_map(ctx, &plan->tgk, kv.k, kv, rows);
      if (st == LYC_OK) st = encode_gather_map(ctx, &plan->tgv, kv.v, kv, rows);
      if (st != LYC_OK) return st;
      plan->gather_rows = static_cast<int32_t>(rows);
    }
  }

  struct HostLayer {
    std::vector<Segment> segs;
    std::vector<Piece> pieces;
    std::vector<int32_t> cta;
    std::vector<TopkTask> tasks;
    int topk_n = 0;
    std::vector<const int32_t*> final_src;  // the current buffer of each set after the layer
    std::vector<int2> combine;  // bf16: (segment, output) left to the next launch
    int nqb = 1;
    int grid = 0;
    int topk_cl = 16;           // cluster size of this layer's selection launch
    std::vector<Piece> pool_units;   // mma kernel: the pool's units, in order
    int64_t tiles = 0, pool_tiles = 0;
    // mma kernel: sparse passes of earlier layers deferred to this layer's
    // rows (see push_sparse below)
    std::vector<Segment> deferred;
    int keys_ctas = 0;        // CTAs with dense pieces of this layer
    bool attn = true;         // this layer's record holds an attention launch
    int nlayers = 1;          // ... of the layers [this one, this one + nlayers)
  };
  std::vector<HostLayer> hl(L);
  std::vector<int> cur(Hs, 0);
  auto set_ptr = [&](int buf, int b, int s) {
    return ctx->sbuf + ((static_cast<int64_t>(buf) * B + b) * Hs + s) * ctx->KS;
  };
  const char* kbase = static_cast<const char*>(kv.k);
  const char* vbase = static_cast<const char*>(kv.v);
  // Deferred sparse passes (mma kernel).  A sparse pass of layer l over a set
  // that layer l-1's selection writes must wait for that selection, which
  // starts only once layer l-1's dense rows are done.  Run in layer l's own
  // launch, the CTAs that take it hold their SMs while they wait, and the
  // next launch's CTAs that need those SMs start late (the chain: selection
  // -> waiting gathers -> late dense runs -> late keys -> next selection).
  // So such a pass runs in layer l+1's launch instead, after that launch's
  // dense rows, by which time the selection is long done; its partial states
  // and outputs are those of layer l (Segment::q, Segment::out).  The last
  // layer keeps its own.
  const bool defer_dep = use_pool;
  // The attention launches (mma kernel): LG consecutive layers each (two,
  // four or eight, see kLayersPerLaunch), the last layer alone (it keeps its passes over the sets of the
  // selection just before it, which is enqueued before its launch).
  // launch_first[l]: the first layer of l's launch; next_launch[l]: the first
  // layer of the launch after it (L: none).
  std::vector<int> launch_first(L), next_launch(L);
  {
    // the K/V bytes a later layer reads, on average (its dense groups' rows,
    // and k rows per sparse-only group)
    double layer_bytes = 0.0;
    for (int l = 1; l < L; ++l)
      for (int g = 0; g < Hkv; ++g) {
        bool dense = false;
        for (int h = g * G; h < (g + 1) * G; ++h) dense = dense || role[static_cast<int64_t>(l) * Hq + h] != 0;
        for (int b = 0; b < B; ++b)
          layer_bytes += static_cast<double>(dense ? kv.n[b] : std::min<int64_t>(k, kv.n[b]));
      }
    layer_bytes *= static_cast<double>(cfg.head_dim) * es * 2.0 / std::max(1, L - 1);
    bool later_sel = false;  // a layer after the first has a retrieval head
    for (int64_t i = Hq; i < static_cast<int64_t>(L) * Hq && !later_sel; ++i) later_sel = role[i] != 0;
    const int LG = !use_pool                        ? 1
                   : !later_sel                     ? kLayersPerLaunch
                   : layer_bytes >= kSmallLayerBytes ? 2
                   : kvmode                          ? kLayersPerLaunch
                                                    : 4;
    for (int l0 = 0, l1 = 0; l0 < L; l0 = l1) {
      l1 = std::min(L, l0 + LG);
      if (l1 == L && l1 - l0 > 1) l1 = L - 1;
      for (int l = l0; l < l1; ++l) {
        launch_first[l] = l0;
        next_launch[l] = l1;
      }
    }
  }

  // the set trace [L][B][Hs][k]: row (l, b, s) holds the set slot s passes on
  // after layer l.  A refreshed slot's row is written by its selection; the
  // others are copies of the row of the slot's last writer (or of S^(0) in
  // set-input mode), made by one launch at the end of the step.
  auto trace_row = [&](int l, int b, int s) -> int32_t* {
    if (!plan->trace) return nullptr;
    return plan->trace + ((static_cast<int64_t>(l) * B + b) * Hs + s) * k;
  };
  std::vector<const int32_t*> fill_src;
  std::vector<int32_t*> fill_dst;
  std::vector<char> prev_fresh(Hs, 1);  // slots the previous layer's selection wrote
  std::vector<int> writer(Hs, -1);      // layer whose selection wrote each slot's current set
  auto ready_flag = [&](int s, int b) -> const uint32_t* {
    if (writer[s] < 0) return nullptr;
    return ctx->flags + ((static_cast<int64_t>(writer[s]) * B + b) * Hs + s) * 2 + 1;
  };
  for (int l = 0; l < L; ++l) {
    HostLayer& H = hl[l];
    // every layer has key rows of its own, so no attention launch writes keys
    // that an earlier selection may still read (launches of consecutive
    // layers may overlap in time)
    const int64_t keys_base = l * static_cast<int64_t>(B) * Hs * ctx->nstride;
    std::vector<char> is_ret(Hq), fresh(Hs, 0);
    for (int h = 0; h < Hq; ++h) {
      is_ret[h] = (l == 0 && !s_in) || role[static_cast<int64_t>(l) * Hq + h] != 0;
      if (is_ret[h]) fresh[kvmode ? h / G : h] = 1;
    }
    // a sparse pass of this layer: into this launch, or (a set the previous
    // layer's selection writes) into the next one, where it needs no wait
    // order (dep 0: its selection has long completed)
    // w: the layer whose selection wrote the set (-1: the caller's)
    auto push_sparse = [&](Segment ss, int layer, int w) {
      if (defer_dep && w >= 0 && launch_first[w] == launch_first[layer] && next_launch[layer] < L) {
        // a set of a selection of this pass's own launch: that selection is
        // enqueued after the launch, so the pass goes to the next launch
        ss.dep = 0;
        hl[next_launch[layer]].deferred.push_back(ss);
      } else if (defer_dep && layer + 1 < L && ss.dep && ss.ready) {
        ss.dep = 0;
        hl[layer + 1].deferred.push_back(ss);
      } else {
        H.segs.push_back(ss);
      }
    };
    int maxnq = 1;
    for (int b = 0; b < B; ++b) {
      const int nb = static_cast<int>(kv.n[b]);  // this element's rows
      const int keffb = plan->set_rows[b];       // rows of its sets at most
      for (int g = 0; g < Hkv; ++g) {
        // row 0 of (l, b, g); paged: of page 0, rows found through b's block table
        const int64_t off = l * kv.s_layer + (kv.paged() ? 0 : b * kv.s_batch) + g * kv.s_head;
        Segment base{};
        base.k = kbase + off * es;
        base.v = vbase + off * es;
        base.s_token = kv.s_token;
        base.row_base = plan->gather_rows > 0 ? static_cast<int32_t>(off / kv.s_token) : 0;
        base.nvalid = nb;
        if (kv.paged()) {
          base.bt = kv.bt + static_cast<int64_t>(b) * kv.max_blocks;
          base.page_rows = kv.page_rows;
          base.s_page = kv.s_page;
        }
        base.l = l;
        base.b = b;
        base.g = g;
        base.q = static_cast<const char*>(plan->q) + static_cast<size_t>(l) * B * Hq * cfg.head_dim * es;
        base.out = plan->out + static_cast<size_t>(l) * B * Hq * cfg.head_dim;
        base.key_mean_off = -1;
        for (int j = 0; j < kMaxQ; ++j) {
          base.key_off[j] = -1;
          base.head[j] = 0;
          base.out_row[j] = 0;
        }
        // dense segment: the group's retrieval heads; in group mode every head
        // of the group, whose mean logit is the group's selection key
        Segment ds = base;
        ds.kind = kDense;
        ds.rows = nb;
        int nret = 0;
        for (int h = g * G; h < (g + 1) * G; ++h) nret += is_ret[h];
        if (nret > 0) {
          int j = 0, o = 0;
          for (int h = g * G; h < (g + 1) * G; ++h) {
            if (!kvmode && !is_ret[h]) continue;
            ds.head[j] = h;
            if (is_ret[h]) ds.out_row[o++] = j;
            if (!kvmode) ds.key_off[j] = keys_base + (static_cast<int64_t>(b) * Hs + h) * ctx->nstride;
            ++j;
          }
          ds.nq = j;
          ds.nout = o;
          if (kvmode) ds.key_mean_off = keys_base + (static_cast<int64_t>(b) * Hs + g) * ctx->nstride;
          maxnq = std::max(maxnq, j);
          H.segs.push_back(ds);
        }
        // sparse segments: one per inherited set that sparse heads read
        if (kvmode) {
          Segment ss = base;
          ss.kind = kSparse;
          ss.rows = keffb;
          ss.idx = set_ptr(cur[g], b, g);
          ss.pad_ok = plan->variable ? 1 : 0;
          int js = 0;
          for (int h = g * G; h < (g + 1) * G; ++h)
            if (!is_ret[h]) {
              ss.out_row[js] = js;
              ss.head[js++] = h;
            }
          if (js > 0) {
            ss.nq = ss.nout = js;
            ss.dep = prev_fresh[g];
            ss.ready = ready_flag(g, b);
            maxnq = std::max(maxnq, js);
            push_sparse(ss, l, writer[g]);
          }
        } else {
          for (int h = g * G; h < (g + 1) * G; ++h) {
            if (is_ret[h]) continue;
            Segment ss = base;
            ss.kind = kSparse;
            ss.rows = keffb;
            ss.idx = set_ptr(cur[h], b, h);
            ss.pad_ok = plan->variable ? 1 : 0;
            ss.head[0] = h;
            ss.out_row[0] = 0;
            ss.nq = ss.nout = 1;
            ss.dep = prev_fresh[h];
            ss.ready = ready_flag(h, b);
            push_sparse(ss, l, writer[h]);
          }
        }
      }
    }
    // the sparse passes deferred to this layer, after its own
    for (const Segment& ds : H.deferred) {
      H.segs.push_back(ds);
      maxnq = std::max(maxnq, ds.nq);
    }
    H.nqb = attn_nq_bucket(maxnq);


    // selection tasks of this layer, then flip the refreshed slots
    for (int s = 0; s < Hs; ++s) {
      if (!fresh[s]) continue;
      for (int b = 0; b < B; ++b) {
        TopkTask tk{};
        tk.keys = ctx->keys + keys_base + (static_cast<int64_t>(b) * Hs + s) * ctx->nstride;
        tk.S = set_ptr((cur[s] + 1) % kSetBuffers, b, s);
        tk.done = ctx->flags + ((static_cast<int64_t>(l) * B + b) * Hs + s) * 2;
        tk.trace = trace_row(l, b, s);
        tk.n = static_cast<int32_t>(kv.n[b]);
        tk.k = select_cap(kv.n[b]);
        if (sel.rule == LYC_RULE_BLOCK_TOPK) {
          // the selection runs over the element's blocks (scored from its keys)
          tk.rows = tk.n;
          tk.n = static_cast<int32_t>((kv.n[b] + E - 1) / E);
        }
        H.topk_n = std::max(H.topk_n, static_cast<int>(tk.n));
        H.tasks.push_back(tk);
      }
    }
    if (plan->trace)
      for (int b = 0; b < B; ++b)
        for (int s = 0; s < Hs; ++s) {
          if (fresh[s]) continue;
          fill_dst.push_back(trace_row(l, b, s));
          fill_src.push_back(writer[s] >= 0 ? trace_row(writer[s], b, s)
                                            : plan->S + (static_cast<int64_t>(b) * Hs + s) * k);
        }
    for (int s = 0; s < Hs; ++s)
      if (fresh[s]) {
        cur[s] = (cur[s] + 1) % kSetBuffers;
        writer[s] = l;
      }
    prev_fresh = fresh;
    H.topk_cl = pick_topk_cluster(ctx, static_cast<int>(H.tasks.size()), plan->variable, l == 0);
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < Hs; ++s) H.final_src.push_back(set_ptr(cur[s], b, s));
  }


  // ---- phase B: the attention launches.  With the mma kernel a launch runs
  // several consecutive layers: their segments are concatenated in
  // layer order (each layer's own passes, then the passes deferred into it).
  // No pass of a launch waits for a selection enqueued after that launch
  // (the selection could find no free SM while the launch's CTAs wait): a
  // pass over a set of a selection of its own launch goes to the next launch
  // (see push_sparse), and the last layer, which keeps its passes over the
  // sets of the selection just before it, has a launch of its own.
  {
    int prev_l0 = -1;
    for (int l0 = 0, l1 = 0; l0 < L; l0 = l1) {
      l1 = next_launch[l0];  // the launch's layers [l0, l1)
      HostLayer& H = hl[l0];
      std::vector<size_t> seg_begin(1, 0);
      seg_begin.push_back(H.segs.size());
      for (int li = l0 + 1; li < l1; ++li) {
        for (const Segment& sg : hl[li].segs) H.segs.push_back(sg);
        seg_begin.push_back(H.segs.size());
        H.nqb = std::max(H.nqb, hl[li].nqb);
        hl[li].segs.clear();
        hl[li].attn = false;
      }
      H.nlayers = l1 - l0;
      // Workload pooling.  The dense rows are cut into equal runs of tiles, one
      // per CTA.  The gathered rows:
      //  * mma kernel: go to a pool of kPoolTiles-tile units, which the CTAs
      //    take at run time once their dense run is done (an atomic cursor per
      //    launch), sets of earlier selections first, those the previous
      //    layer's selection writes (the only rows that wait for it) last.  A
      //    CTA that starts late (the launches of consecutive layers overlap) or
      //    streams slowly then simply takes fewer units;
      //  * other kernels: are cut into equal runs too, taken after the dense
      //    run, the previous selection's sets last, so that few CTAs wait, and
      //    late.
      int64_t NT = 0;
      for (const Segment& sg : H.segs) NT += (sg.rows + TR - 1) / TR;
      // The previous layer's selection runs beside this layer's attention (the
      // attention streams its dense rows meanwhile and waits for the sets only
      // before its gathered rows).  When that selection is small, leave its SMs
      // to it: fewer SMs still stream at full HBM bandwidth, and no CTA of this
      // kernel then starts late behind it.
      int avail = ctx->sms;
      {
        // the largest selection among the one before this launch and its own
        int prev = 0;
        for (int li = std::max(0, l0 - 1); li < l1; ++li)
          prev = std::max(prev, static_cast<int>(hl[li].tasks.size()) * hl[li].topk_cl);
        if (l0 > 0 && prev > 0 && 2 * prev <= ctx->sms / 4) avail = ctx->sms - 2 * prev;
        else if (l0 > 0 && prev > 0 && prev <= ctx->sms / 4) avail = ctx->sms - prev;
      }
      // The grid leaves the SMs of the previous selection and of this layer's
      // own to them: the selection of this layer starts on its key flag, while
      // the previous one may still run, and takes free SMs at once (measured on
      // B200: +1.9 % in KV-group mode for a grid that leaves one selection's SMs
      // against one with CTAs that take them back for pool units).
      H.tiles = NT;
      // A launch with no rows of its own (a layer without retrieval heads whose
      // sparse passes all moved to the next launch) still runs: its CTAs merge
      // the previous launch's split rows and raise its done flag.
      int grid = static_cast<int>(std::min<int64_t>(NT, avail));
      if (grid == 0)
        grid = std::max(1, std::min(avail, prev_l0 >= 0 ? static_cast<int>(hl[prev_l0].combine.size()) : 1));
      H.grid = grid;
      std::vector<int> npieces(H.segs.size(), 0);
      std::vector<std::vector<Piece>> per_cta(grid);
      // phase 0 (dense segments) is cut per layer of the launch, so that every
      // CTA streams a run of each layer's dense rows in layer order (the keys of
      // the first layer are then complete early, and its selection starts)
      for (int pass = 0; pass < (use_pool ? l1 - l0 : 2); ++pass) {
        const int phase = use_pool ? 0 : pass;
        const size_t sg_lo = use_pool ? seg_begin[pass] : 0;
        const size_t sg_hi = use_pool ? seg_begin[pass + 1] : H.segs.size();
        std::vector<size_t> ids;
        std::vector<int64_t> tstart(1, 0);
        for (int dep = 0; dep < 2; ++dep) {
          for (size_t s2 = sg_lo; s2 < sg_hi; ++s2) {
            const Segment& cs = H.segs[s2];
            if ((cs.kind == kDense ? 0 : 1) != phase || (phase == 1 && cs.dep != dep) ||
                (phase == 0 && dep == 1))
              continue;
            ids.push_back(s2);
            tstart.push_back(tstart.back() + (cs.rows + TR - 1) / TR);
          }
        }
        const int64_t nt = tstart.back();
        const int cut = grid;
        size_t si = 0;
        for (int c = 0; c < cut; ++c) {
          const int64_t t0 = nt * c / cut, t1 = nt * (c + 1) / cut;
          while (si < ids.size() && tstart[si + 1] <= t0) ++si;
          for (size_t q = si; q < ids.size() && tstart[q] < t1; ++q) {
            const int64_t a = std::max(t0, tstart[q]) - tstart[q];
            const int64_t e = std::min(t1, tstart[q + 1]) - tstart[q];
            if (e <= a) continue;
            Piece pc;
            pc.seg = static_cast<int32_t>(ids[q]);
            pc.r0 = static_cast<int32_t>(a * TR);
            pc.r1 = static_cast<int32_t>(std::min<int64_t>(e * TR, H.segs[ids[q]].rows));
            pc.ordinal = npieces[ids[q]]++;
            per_cta[c].push_back(pc);
          }
        }
      }
      if (use_pool) {
        // a gathered segment of r rows is cut into units of kPoolTiles tiles
        // (kPoolTilesDep for a set the previous selection writes), unit q =
        // piece q (its ordinal); CTAs take them at run time.  The pool lists
        // the units in order, earlier selections' sets first.  (Measured on
        // B200 against one-tile pieces whose warp writes its own partial state:
        // per-head selection 1231 against 1348 us per step, KV-group even.)
        for (int dep = 0; dep < 2; ++dep)
          for (size_t s2 = 0; s2 < H.segs.size(); ++s2)
            if (H.segs[s2].kind == kSparse && H.segs[s2].dep == dep) {
              const int unit_tiles = dep ? kPoolTilesDep : kPoolTiles;
              const int rows = H.segs[s2].rows;
              int tile = 0;
              for (int r0 = 0; r0 < rows; r0 += unit_tiles * kTileRows, tile += unit_tiles) {
                Piece pc;
                pc.seg = static_cast<int32_t>(s2);
                pc.r0 = r0;
                pc.r1 = std::min(r0 + unit_tiles * kTileRows, rows);
                pc.ordinal = tile / unit_tiles;
                H.pool_units.push_back(pc);
              }
              npieces[s2] = (rows + unit_tiles * kTileRows - 1) / (unit_tiles * kTileRows);
              H.pool_tiles += (rows + TR - 1) / TR;
            }
      }
      for (int c = 0; c < grid; ++c) {
        H.cta.push_back(static_cast<int32_t>(H.pieces.size()));
        for (const Piece& pc : per_cta[c]) H.pieces.push_back(pc);
      }
      H.cta.push_back(static_cast<int32_t>(H.pieces.size()));
      // partial records (one per piece and output) and arrival counters (one
      // per output; the fp32 kernel's last-arrival combine); the bf16 kernel
      // leaves the cross-piece combine of segments cut into several pieces to
      // the next launch, as (segment, output) tasks
      int part = 0, cnt = 0;
      for (size_t s = 0; s < H.segs.size(); ++s) {
        H.segs[s].npieces = npieces[s];
        H.segs[s].part_base = part;
        H.segs[s].cnt_base = cnt;
        part += npieces[s] * H.segs[s].nout;
        cnt += H.segs[s].nout;
        if (npieces[s] > 1)
          for (int o = 0; o < H.segs[s].nout; ++o) H.combine.push_back(make_int2(static_cast<int>(s), o));
      }
      if (static_cast<size_t>(part) > ctx->max_parts || static_cast<size_t>(cnt) > ctx->max_counters)
        return fail(ctx, LYC_ERR_UNSUPPORTED, "work pool larger than the scratch sized at create");
      // the CTAs that write each layer's selection keys (their dense pieces)
      for (int li = l0; li < l1; ++li) {
        int n_ctas = 0;
        for (int c = 0; c < grid; ++c) {
          bool has = false;
          for (const Piece& pc : per_cta[c])
            has = has || (H.segs[pc.seg].kind == kDense && H.segs[pc.seg].l == li);
          n_ctas += has ? 1 : 0;
        }
        hl[li].keys_ctas = n_ctas;
      }
      prev_l0 = l0;
    }
  }

  // ---- one device buffer for every record
  size_t bytes = 0;
  auto take = [&](size_t sz) {
    bytes = round_up(bytes, 64);
    const size_t o = bytes;
    bytes += sz;
    return o;
  };
  plan->layers.resize(L);
  int attn_launches = 0;
  for (int l = 0; l < L; ++l) {
    LayerPlan& lp = plan->layers[l];
    HostLayer& H = hl[l];
    lp.nseg = static_cast<int>(H.segs.size());
    lp.npieces = static_cast<int>(H.pieces.size());
    lp.grid = H.grid;
    lp.nqb = H.nqb;
    lp.ntasks = static_cast<int>(H.tasks.size());
    lp.topk_cl = H.topk_cl;
    lp.off_segs = take(H.segs.size() * sizeof(Segment));
    lp.off_pieces = take(H.pieces.size() * sizeof(Piece));
    lp.off_cta = take(H.cta.size() * sizeof(int32_t));
    lp.off_tasks = take(std::max<size_t>(1, H.tasks.size()) * sizeof(TopkTask));
    lp.topk_n = H.topk_n;
    lp.ncombine = static_cast<int>(H.combine.size());
    lp.off_combine = take(std::max<size_t>(1, H.combine.size()) * sizeof(int2));
    lp.pool_n = static_cast<int>(H.pool_units.size());
    lp.tiles = H.tiles;
    lp.pool_tiles = H.pool_tiles;
    lp.off_pool = take(std::max<size_t>(1, H.pool_units.size()) * sizeof(Piece));
    lp.keys_ctas = H.keys_ctas;
    lp.attn = H.attn;
    lp.nlayers = H.nlayers;
    lp.launch = attn_launches;
    if (H.attn) ++attn_launches;
    // the first piece of each CTA, when it is a dense piece of a contiguous
    // cache (the only kind the kernel can start from the parameters)
    lp.first.clear();
    if (use_pool && !plan->paged && H.attn) {
      const int nf = std::min(H.grid, kFirstPieces);
      lp.first.resize(nf);
      for (int c = 0; c < nf; ++c) {
        FirstPiece& f = lp.first[c];
        f.pc.seg = -1;
        f.pc.r0 = f.pc.r1 = f.pc.ordinal = 0;
        f.g = f.b = 0;
        if (H.cta[c + 1] <= H.cta[c]) continue;
        const Piece& pc = H.pieces[H.cta[c]];
        const Segment& sg = H.segs[pc.seg];
        if (sg.kind != kDense || sg.l != l) continue;
        f.pc = pc;
        f.g = static_cast<int16_t>(sg.g);
        f.b = static_cast<int16_t>(sg.b);
      }
    }
  }
  plan->off_final_src = take(hl[L - 1].final_src.size() * sizeof(void*));
  plan->nfill = static_cast<int>(fill_src.size());
  plan->off_fill_src = take(std::max<size_t>(1, fill_src.size()) * sizeof(void*));
  plan->off_fill_dst = take(std::max<size_t>(1, fill_dst.size()) * sizeof(void*));
  plan->off_n = take(static_cast<size_t>(B) * sizeof(int64_t));
  // the last layer's combine runs in a launch of its own, whose CTAs have no pieces
  int last_attn = 0;  // the first layer of the last attention launch
  for (int l = 0; l < L; ++l)
    if (plan->layers[l].attn) last_attn = l;
  plan->combine_grid = std::max(1, std::min(ctx->sms, plan->layers[last_attn].ncombine));
  plan->off_empty_cta = take((plan->combine_grid + 1) * sizeof(int32_t));
  std::vector<unsigned char> host(bytes, 0);
  for (int l = 0; l < L; ++l) {
    const LayerPlan& lp = plan->layers[l];
    HostLayer& H = hl[l];
    memcpy(host.data() + lp.off_segs, H.segs.data(), H.segs.size() * sizeof(Segment));
    memcpy(host.data() + lp.off_pieces, H.pieces.data(), H.pieces.size() * sizeof(Piece));
    memcpy(host.data() + lp.off_cta, H.cta.data(), H.cta.size() * sizeof(int32_t));
    if (!H.tasks.empty())
      memcpy(host.data() + lp.off_tasks, H.tasks.data(), H.tasks.size() * sizeof(TopkTask));
    if (!H.combine.empty())
      memcpy(host.data() + lp.off_combine, H.combine.data(), H.combine.size() * sizeof(int2));
    if (!H.pool_units.empty())
      memcpy(host.data() + lp.off_pool, H.pool_units.data(), H.pool_units.size() * sizeof(Piece));
  }
  memcpy(host.data() + plan->off_final_src, hl[L - 1].final_src.data(),
         hl[L - 1].final_src.size() * sizeof(void*));
  if (!fill_src.empty()) {
    memcpy(host.data() + plan->off_fill_src, fill_src.data(), fill_src.size() * sizeof(void*));
    memcpy(host.data() + plan->off_fill_dst, fill_dst.data(), fill_dst.size() * sizeof(void*));
  }
  memcpy(host.data() + plan->off_n, kv.n.data(), static_cast<size_t>(B) * sizeof(int64_t));
  LYC_CUDA(cudaMalloc(&plan->dev, bytes), "cudaMalloc(plan)");
  plan->dev_bytes = bytes;
  if (kv.k_new) {
    AppendParams& a = plan->ap_append;
    a.k_new = static_cast<const unsigned char*>(kv.k_new);
    a.v_new = static_cast<const unsigned char*>(kv.v_new);
    a.k = static_cast<unsigned char*>(const_cast<void*>(kv.k));
    a.v = static_cast<unsigned char*>(const_cast<void*>(kv.v));
    a.n = reinterpret_cast<const int64_t*>(plan->dev + plan->off_n);
    a.s_layer = kv.s_layer;
    a.s_batch = kv.s_batch;
    a.s_head = kv.s_head;
    a.s_token = kv.s_token;
    a.s_page = kv.s_page;
    a.bt = kv.bt;
    a.page_rows = kv.page_rows;
    a.max_blocks = kv.max_blocks;
    a.L = L;
    a.B = B;
    a.Hkv = Hkv;
    a.elem_bytes = static_cast<int32_t>(es);
    a.row_bytes = static_cast<int32_t>(cfg.head_dim * es);
    plan->append = true;
  }
  LYC_CUDA(cudaMemcpy(plan->dev, host.data(), bytes, cudaMemcpyHostToDevice), "upload plan");
  return LYC_OK;
}

}  // namespace

namespace {

// ---------------------------------------------------------------- enqueue
// Records an event of timing set `set` (or, while capturing, of set 0, whose
// nodes are re-pointed at other sets before each replay).
lyc_status record_event(lyc_ctx* ctx, Plan* plan, int set, int idx, cudaStream_t stream,
                        bool capturing) {
  if (!plan->timing) return LYC_OK;
  cudaEvent_t ev = ctx->events[static_cast<size_t>(set) * ctx->events_per_set + idx];
  if (capturing) {
    LYC_CUDA(cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal), "event record node");
  } else {
    LYC_CUDA(cudaEventRecord(ev, stream), "cudaEventRecord");
  }
  return LYC_OK;
}

// Enqueue the whole step of `plan` on `stream` (or record it, while capturing).
// Layer `pl`'s cross-piece combine tasks, for the launch that follows it.
void set_prev_combine(lyc_ctx* ctx, Plan* plan, int pl, AttnParams* ap) {
  const lyc_config& cfg = ctx->cfg;
  const LayerPlan& pp = plan->layers[pl];
  const int D = cfg.head_dim;
  ap->prev_segs = reinterpret_cast<const Segment*>(plan->dev + pp.off_segs);
  ap->prev_tasks = reinterpret_cast<const int2*>(plan->dev + pp.off_combine);
  ap->prev_ntasks = pp.ncombine;
  ap->prev_part_o = ctx->part_o + (pp.launch & 1) * ctx->max_parts * D;
  ap->prev_part_ml = ctx->part_ml + (pp.launch & 1) * ctx->max_parts;
  ap->prev_out = plan->out + static_cast<size_t>(pl) * cfg.batch * cfg.num_q_heads * D;
}

lyc_status enqueue_step(lyc_ctx* ctx, Plan* plan, cudaStream_t stream, int set, bool capturing) {
  const lyc_config& cfg = ctx->cfg;
  const int L = cfg.num_layers, B = cfg.batch, Hq = cfg.num_q_heads, D = cfg.head_dim;
  const size_t es = cfg.dtype == LYC_BF16 ? 2 : 4;
  const int dtype = cfg.dtype == LYC_BF16 ? 0 : 1;
  // the current token's K and V into the cache, before any layer reads it
  if (plan->append) LYC_CUDA(append_rows_launch(&plan->ap_append, stream), "append K/V rows");
  if (plan->flags & LYC_STEP_S_IN) {
    LYC_CUDA(cudaMemcpy2DAsync(ctx->sbuf, ctx->KS * sizeof(int32_t), plan->S, plan->k * sizeof(int32_t),
                               plan->k * sizeof(int32_t), static_cast<size_t>(B) * ctx->Hs,
                               cudaMemcpyDeviceToDevice, stream),
             "copy S^(0) in");
    if (plan->flags & LYC_STEP_VALIDATE_S) {
      // per batch element: its sets hold min(k, n[b]) indices below n[b]
      for (int b = 0; b < B; ++b) {
        const int nb = static_cast<int>(plan->nb[b]);
        const int cap = plan->set_rows[b];
        ValidateSetsParams vp{ctx->sbuf + static_cast<int64_t>(b) * ctx->Hs * ctx->KS, ctx->status, ctx->Hs,
                              ctx->KS, plan->k, cap, nb, plan->variable ? std::min(1, cap) : cap};
        LYC_CUDA(validate_sets_launch(&vp, stream), "validate S^(0)");
      }
    }
  }
  plan->kernel_kind.clear();
  plan->kernel_layer.clear();
  int ev = 0;
  // bf16 on the mma kernel: ready and done flags, the per-SM piece-state
  // ring and the pool make it safe for its launches to overlap the previous
  // layer's (the previous attention, and the selection between them)
  const bool early = dtype == 0 && !plan->use_tc;
  // ... and each selection lets the next attention launch at its start
  // (before its keys are complete), so that the next attention's CTAs take
  // the SMs of the previous attention's tail as they free up.  They then
  // start staggered; the pool of gathered rows (taken at run time) absorbs
  // the stagger.  (Measured on B200 with the selection started on the key
  // flag: per-head selection unchanged, KV-group selection +1.3 % against
  // letting it launch only once the selection has its keys.)
  // step counters of the attention launch whose first layer is l (parity-0
  // addresses), and of layer l's selection keys
  const int cstride = 3 * (L + 1);
  uint32_t* cnt_base = reinterpret_cast<uint32_t*>(ctx->pool_cursors);
  auto done_cnt = [&](int l) { return cnt_base + (L + 1) + l; };
  auto keys_cnt = [&](int l) { return cnt_base + 2 * (L + 1) + l; };
  const uint32_t nc = static_cast<uint32_t>(attn_mma_consumer_warps(D));
  int prev_l0 = -1;  // the first layer of the previous attention launch
  for (int l0 = 0; l0 < L; ++l0) {
    const LayerPlan& lp = plan->layers[l0];
    if (!lp.attn) continue;  // a later layer of a launch: enqueued with the launch
    const int l1 = l0 + lp.nlayers;  // the launch's layers [l0, l1)
    bool any_tasks = false;
    for (int li = l0; li < l1; ++li) any_tasks = any_tasks || plan->layers[li].ntasks > 0;
    AttnParams ap{};
    ap.segs = reinterpret_cast<const Segment*>(plan->dev + lp.off_segs);
    ap.pieces = reinterpret_cast<const Piece*>(plan->dev + lp.off_pieces);
    ap.cta_begin = reinterpret_cast<const int32_t*>(plan->dev + lp.off_cta);
    ap.q = static_cast<const char*>(plan->q) + static_cast<size_t>(l0) * B * Hq * D * es;
    ap.out = plan->out + static_cast<size_t>(l0) * B * Hq * D;
    ap.keys = ctx->keys;
    // partial records: double-buffered by launch (the next launch merges them)
    ap.part_o = ctx->part_o + (lp.launch & 1) * ctx->max_parts * D;
    ap.part_ml = ctx->part_ml + (lp.launch & 1) * ctx->max_parts;
    ap.wpart_o = ctx->wpart_o;
    ap.wpart_ml = ctx->wpart_ml;
    ap.wpart_by_sm = 1;
    ap.wpart_slots = ctx->wpart_slots;
    ap.epoch = ctx->epoch;
    if (early) {
      // done counters between consecutive attention launches, and the pool of
      // gathered rows (mma kernel only)
      ap.done = done_cnt(l0);
      ap.prev_done = prev_l0 >= 0 ? done_cnt(prev_l0) : nullptr;
      ap.prev_done_expect = prev_l0 >= 0 ? static_cast<uint32_t>(plan->layers[prev_l0].grid) : 0u;
      ap.pool_units = reinterpret_cast<const Piece*>(plan->dev + lp.off_pool);
      ap.pool_n = lp.pool_n;
      ap.pool_stride = cstride;
      ap.pool_cursors = ctx->pool_cursors;
      // each layer's selection starts once that layer's keys are written (its
      // dense runs), not once the whole launch is done: the consumer warps
      // count their arrivals per layer, from the first layer's counter on
      if (any_tasks) {
        ap.keys_done = keys_cnt(l0);
        ap.keys_ctas = lp.keys_ctas;
      }
    }
    ap.counters = ctx->counters;
    ap.status = ctx->status;
    ap.timeline = plan->timeline;
    ap.timeline_cap = plan->timeline_cap;
    ap.layer = l0;
    ap.Hq = Hq;
    ap.G = ctx->G;
    ap.n = plan->n;
    ap.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    // Without a selection launch in between, the previous layer's attention
    // may still be running.  The mma kernel needs no wait for it: its
    // readers of sets wait on the sets' ready flags, its partials are written
    // only after its epilogue has seen the previous launch complete, and its
    // piece-state ring is the SM's own.  The other kernels wait for it at
    // their start.
    ap.wait_prev = (l0 > 0 && plan->layers[l0 - 1].ntasks == 0 && !early) ? 1 : 0;
    lyc_status st = record_event(ctx, plan, set, ev++, stream, capturing);
    if (st != LYC_OK) return st;
    if (dtype == 0) {
      AttnMmaParams mp;
      memset(&mp, 0, sizeof mp);
      mp.tmk = plan->tmk;
      mp.tmv = plan->tmv;
      mp.tgk = plan->tgk;
      mp.tgv = plan->tgv;
      mp.p = ap;
      mp.p.gather_rows = plan->gather_rows;
      mp.p.paged = plan->paged ? 1 : 0;
      if (prev_l0 >= 0) set_prev_combine(ctx, plan, prev_l0, &mp.p);
      if (!plan->use_tc && !lp.first.empty()) {
        mp.nfirst = static_cast<int32_t>(lp.first.size());
        memcpy(mp.first, lp.first.data(), lp.first.size() * sizeof(FirstPiece));
      }
      LYC_CUDA(plan->use_tc ? attn_tc_dispatch(&mp, lp.grid, stream, nullptr, false)
                            : attn_mma_dispatch(D, &mp, lp.grid, stream, nullptr, false),
               "attention launch");
    } else {
      LYC_CUDA(attn_simt_dispatch(D, lp.nqb, &ap, lp.grid, stream, nullptr, false), "attention launch");
    }
    if ((st = record_event(ctx, plan, set, ev++, stream, capturing)) != LYC_OK) return st;
    plan->kernel_kind.push_back(0);
    plan->kernel_layer.push_back(l0);
    // the launch's selections, one launch per layer, in layer order.  Each
    // lets the next kernel of the step launch at its own start (the next
    // selection, or the next attention launch, whose CTAs then take the SMs
    // of this launch's tail as they free up; its pool of gathered rows absorbs
    // their staggered start).  (Measured on B200 with the selection started
    // on its keys: per-head selection unchanged, KV-group selection +1.3 %
    // against letting the next attention launch only once the selection has
    // its keys.)
    for (int li = l0; li < l1; ++li) {
      const LayerPlan& sp = plan->layers[li];
      if (sp.ntasks == 0) continue;
      TopkParams tp{};
      tp.tasks = reinterpret_cast<const TopkTask*>(plan->dev + sp.off_tasks);
      tp.epoch = ctx->epoch;
      tp.early = (early && li + 1 < L) ? 1 : 0;
      tp.n = sp.topk_n;
      tp.k = plan->k;
      tp.size_rule = plan->sel.rule == LYC_RULE_TOPP        ? kSizeTopP
                     : plan->sel.rule == LYC_RULE_THRESHOLD ? kSizeThreshold
                                                            : kSizeFixed;
      tp.size_x = plan->sel.rule == LYC_RULE_TOPP ? plan->sel.p : plan->sel.tau;
      tp.expand = plan->sel.rule == LYC_RULE_BLOCK_TOPK ? plan->sel.block : 1;
      tp.timeline = plan->timeline;
      tp.timeline_cap = plan->timeline_cap;
      tp.layer = li;
      tp.status = ctx->status;
      if (ap.keys_done && sp.keys_ctas > 0) {
        // its keys, and the previous attention launch done (it may still read
        // the set buffers this selection overwrites)
        tp.keys_ready = keys_cnt(li);
        tp.keys_expect = static_cast<uint32_t>(sp.keys_ctas) * nc;
        tp.prev_done = ap.prev_done;
        tp.prev_done_expect = ap.prev_done_expect;
        tp.cnt_stride = cstride;
      }
      if ((st = record_event(ctx, plan, set, ev++, stream, capturing)) != LYC_OK) return st;
      LYC_CUDA(topk_launch(sp.topk_cl, &tp, sp.ntasks, stream, false), "top-k launch");
      if ((st = record_event(ctx, plan, set, ev++, stream, capturing)) != LYC_OK) return st;
      plan->kernel_kind.push_back(1);
      plan->kernel_layer.push_back(li);
    }
    prev_l0 = l0;
  }
  if (dtype == 0) {
    // the last launch's cross-piece combine: the same kernel with no pieces
    AttnMmaParams mp;
    memset(&mp, 0, sizeof mp);
    mp.tmk = plan->tmk;
    mp.tmv = plan->tmv;
    mp.tgk = plan->tgk;
    mp.tgv = plan->tgv;
    AttnParams& ap = mp.p;
    ap = AttnParams{};
    const LayerPlan& lp = plan->layers[prev_l0];
    ap.segs = reinterpret_cast<const Segment*>(plan->dev + lp.off_segs);
    ap.pieces = reinterpret_cast<const Piece*>(plan->dev + lp.off_pieces);
    ap.cta_begin = reinterpret_cast<const int32_t*>(plan->dev + plan->off_empty_cta);
    ap.q = plan->q;
    ap.out = plan->out;
    ap.status = ctx->status;
    ap.wpart_o = ctx->wpart_o;
    ap.wpart_ml = ctx->wpart_ml;
    ap.wpart_by_sm = 1;
    ap.wpart_slots = ctx->wpart_slots;
    ap.epoch = ctx->epoch;
    if (early) {
      ap.prev_done = done_cnt(prev_l0);
      ap.prev_done_expect = static_cast<uint32_t>(lp.grid);
      ap.pool_stride = cstride;
    }
    ap.layer = L;
    ap.Hq = Hq;
    ap.G = ctx->G;
    ap.n = plan->n;
    set_prev_combine(ctx, plan, prev_l0, &ap);
    lyc_status st = record_event(ctx, plan, set, ev++, stream, capturing);
    if (st != LYC_OK) return st;
    LYC_CUDA(plan->use_tc ? attn_tc_dispatch(&mp, plan->combine_grid, stream, nullptr, false)
                          : attn_mma_dispatch(D, &mp, plan->combine_grid, stream, nullptr, false),
             "combine launch");
    if ((st = record_event(ctx, plan, set, ev++, stream, capturing)) != LYC_OK) return st;
    plan->kernel_kind.push_back(0);
    plan->kernel_layer.push_back(L - 1);
  }
  if (plan->trace && plan->nfill > 0) {
    // the trace rows of the sets a layer passed on unchanged (before the final
    // copy: in set-input mode some of them come from the caller's S^(0))
    CopySetsParams fp{};
    fp.src = reinterpret_cast<const int32_t* const*>(plan->dev + plan->off_fill_src);
    fp.dsts = reinterpret_cast<int32_t* const*>(plan->dev + plan->off_fill_dst);
    fp.nsets = plan->nfill;
    fp.k = plan->k;
    LYC_CUDA(copy_sets_launch(&fp, stream), "trace fill");
  }
  CopySetsParams cp{reinterpret_cast<const int32_t* const*>(plan->dev + plan->off_final_src), plan->S,
                    B * ctx->Hs, plan->k, ctx->epoch, ctx->pool_cursors, cstride, nullptr};
  LYC_CUDA(copy_sets_launch(&cp, stream), "final set copy");
  return LYC_OK;
}

lyc_status capture_plan(lyc_ctx* ctx, Plan* plan) {
  cudaStream_t cs;
  LYC_CUDA(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking), "capture stream");
  cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) {
    cudaStreamDestroy(cs);
    return cuda_fail(ctx, e, "begin capture");
  }
  lyc_status st = enqueue_step(ctx, plan, cs, 0, true);
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  if (st != LYC_OK) {
    if (graph) cudaGraphDestroy(graph);
    return st;
  }
  if (e != cudaSuccess) return cuda_fail(ctx, e, "end capture");
  e = cudaGraphInstantiate(&plan->exec, graph, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(graph);
    return cuda_fail(ctx, e, "graph instantiate");
  }
  plan->graph = graph;
  if (plan->timing) {
    // map each event-record node to its position via the set-0 event it records
    size_t nn = 0;
    LYC_CUDA(cudaGraphGetNodes(graph, nullptr, &nn), "graph nodes");
    std::vector<cudaGraphNode_t> nodes(nn);
    LYC_CUDA(cudaGraphGetNodes(graph, nodes.data(), &nn), "graph nodes");
    plan->ev_nodes.assign(ctx->events_per_set, nullptr);
    for (cudaGraphNode_t nd : nodes) {
      cudaGraphNodeType ty;
      LYC_CUDA(cudaGraphNodeGetType(nd, &ty), "node type");
      if (ty != cudaGraphNodeTypeEventRecord) continue;
      cudaEvent_t ev;
      LYC_CUDA(cudaGraphEventRecordNodeGetEvent(nd, &ev), "node event");
      for (int i = 0; i < ctx->events_per_set; ++i)
        if (ctx->events[i] == ev) plan->ev_nodes[i] = nd;
    }
  }
  return LYC_OK;
}

std::string plan_key(const uint8_t* role, int L, int Hq, const KvView& kv, int k,
                     uint32_t flags, const void* q, const float* out, const int32_t* S,
                     const int32_t* trace, bool timing) {
  std::string key(reinterpret_cast<const char*>(role), static_cast<size_t>(L) * Hq);
  auto add = [&](const void* p, size_t n) { key.append(static_cast<const char*>(p), n); };
  add(&kv.k, sizeof kv.k);
  add(&kv.v, sizeof kv.v);
  add(kv.n.data(), kv.n.size() * sizeof(int64_t));
  const int64_t st[5] = {kv.s_layer, kv.s_batch, kv.s_head, kv.s_token, kv.s_page};
  add(st, sizeof st);
  add(&kv.bt, sizeof kv.bt);
  const int64_t pg[3] = {kv.page_rows, kv.max_blocks, kv.num_pages};
  add(pg, sizeof pg);
  add(&kv.k_new, sizeof kv.k_new);
  add(&kv.v_new, sizeof kv.v_new);
  add(&k, sizeof k);
  const uint32_t f = flags & (LYC_STEP_S_IN | LYC_STEP_VALIDATE_S);
  add(&f, sizeof f);
  add(&q, sizeof q);
  add(&out, sizeof out);
  add(&S, sizeof S);
  add(&trace, sizeof trace);
  const char t = timing ? 1 : 0;
  add(&t, 1);
  return key;
}

}  // namespace

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int now = -1;
    if (prev >= 0 && cudaGetDevice(&now) == cudaSuccess && now != prev) cudaSetDevice(prev);
  }
};

struct TimedStep {
  int set;
  std::vector<int> kind, layer;
};
std::unordered_map<const lyc_ctx*, std::vector<TimedStep>>& timed_steps() {
  static std::unordered_map<const lyc_ctx*, std::vector<TimedStep>> m;
  return m;
}

int timing_sets() { return 64; }

lyc_status check_kv(lyc_ctx* ctx, const lyc_kv_cache* kv) {
  const lyc_config& c = ctx->cfg;
  const int64_t es = c.dtype == LYC_BF16 ? 2 : 4;
  if (!kv || !kv->k || !kv->v) return fail(ctx, LYC_ERR_INVALID_ARG, "kv cache pointer is NULL");
  if (kv->n < 1 || kv->n > c.max_ctx) return fail(ctx, LYC_ERR_INVALID_ARG, "kv->n outside [1, max_ctx]");
  if (kv->s_token < c.head_dim) return fail(ctx, LYC_ERR_INVALID_ARG, "s_token < head_dim");
  if (kv->s_layer < 0 || kv->s_batch < 0 || kv->s_head < 0)
    return fail(ctx, LYC_ERR_INVALID_ARG, "negative kv stride");
  const int64_t strides[4] = {kv->s_layer, kv->s_batch, kv->s_head, kv->s_token};
  for (int64_t s : strides)
    if ((s * es) % 16 != 0) return fail(ctx, LYC_ERR_INVALID_ARG, "kv strides must be multiples of 16 bytes");
  if ((reinterpret_cast<uintptr_t>(kv->k) | reinterpret_cast<uintptr_t>(kv->v)) & 15u)
    return fail(ctx, LYC_ERR_INVALID_ARG, "kv base pointers must be 16-byte aligned");
  return LYC_OK;
}

lyc_status check_kv_batch(lyc_ctx* ctx, const lyc_kv_batch* kv) {
  const lyc_config& c = ctx->cfg;
  const int64_t es = c.dtype == LYC_BF16 ? 2 : 4;
  if (!kv || !kv->k || !kv->v || !kv->n) return fail(ctx, LYC_ERR_INVALID_ARG, "kv pointer is NULL");
  int64_t nmax = 0;
  for (int b = 0; b < c.batch; ++b) {
    if (kv->n[b] < 1 || kv->n[b] > c.max_ctx)
      return fail(ctx, LYC_ERR_INVALID_ARG, "kv->n[b] outside [1, max_ctx]");
    nmax = std::max(nmax, kv->n[b]);
  }
  const bool paged = kv->block_table != nullptr;
  if (kv->s_token < c.head_dim || kv->s_head < c.head_dim)
    return fail(ctx, LYC_ERR_INVALID_ARG, "s_token and s_head must be at least head_dim");
  if (kv->s_layer < 0 || kv->s_batch < 0 || kv->s_page < 0)
    return fail(ctx, LYC_ERR_INVALID_ARG, "negative kv stride");
  const int64_t strides[5] = {kv->s_layer, paged ? 0 : kv->s_batch, kv->s_head, kv->s_token,
                              paged ? kv->s_page : 0};
  for (int64_t s : strides)
    if ((s * es) % 16 != 0) return fail(ctx, LYC_ERR_INVALID_ARG, "kv strides must be multiples of 16 bytes");
  if ((reinterpret_cast<uintptr_t>(kv->k) | reinterpret_cast<uintptr_t>(kv->v)) & 15u)
    return fail(ctx, LYC_ERR_INVALID_ARG, "kv base pointers must be 16-byte aligned");
  if (paged) {
    if (c.dtype != LYC_BF16 || (c.flags & LYC_CFG_TCGEN05))
      return fail(ctx, LYC_ERR_UNSUPPORTED, "a paged cache needs bf16 on the default (mma.sync) kernel");
    if (kv->page_rows < 64 || kv->page_rows % 64 != 0)
      return fail(ctx, LYC_ERR_INVALID_ARG, "page_rows must be a positive multiple of 64");
    if (kv->max_blocks < (nmax + kv->page_rows - 1) / kv->page_rows || kv->num_pages < 1 || kv->s_page < 1)
      return fail(ctx, LYC_ERR_INVALID_ARG, "block table too short, or no pages");
  }
  if ((kv->k_new == nullptr) != (kv->v_new == nullptr))
    return fail(ctx, LYC_ERR_INVALID_ARG, "k_new and v_new must both be given or both NULL");
  if ((reinterpret_cast<uintptr_t>(kv->k_new) | reinterpret_cast<uintptr_t>(kv->v_new)) & 15u)
    return fail(ctx, LYC_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  return LYC_OK;
}

}  // namespace

extern "C" {

const char* lyc_status_string(lyc_status s) {
  switch (s) {
    case LYC_OK: return "ok";
    case LYC_ERR_INVALID_ARG: return "invalid argument";
    case LYC_ERR_UNSUPPORTED: return "unsupported configuration";
    case LYC_ERR_OOM: return "out of device memory";
    case LYC_ERR_CUDA: return "CUDA error";
    case LYC_ERR_BAD_INDEX: return "inherited set holds an index outside [0, n)";
    case LYC_ERR_TIMEOUT: return "device-side wait timed out";
    case LYC_ERR_SCRATCH_LIMIT:
      return "request exceeds the fixed scratch of the allocation-free entry point "
             "(LYC_NOALLOC_MAX_SETS / LYC_NOALLOC_MAX_CTAS)";
  }
  return "unknown status";
}

const char* lyc_last_error(const lyc_ctx* ctx) { return ctx ? ctx->err.c_str() : "NULL context"; }

lyc_status lyc_create(const lyc_config* cfg, lyc_ctx** out) {
  if (!cfg || !out) return LYC_ERR_INVALID_ARG;
  *out = nullptr;
  const lyc_config& c = *cfg;
  if (c.num_layers < 1 || c.batch < 1 || c.num_q_heads < 1 || c.num_kv_heads < 1 ||
      c.num_q_heads % c.num_kv_heads != 0 || c.max_ctx < 1 || c.max_k < 1 ||
      (c.flags & ~(LYC_CFG_TMA_GATHER | LYC_CFG_TCGEN05)) != 0)
    return LYC_ERR_INVALID_ARG;
  if (c.dtype != LYC_BF16 && c.dtype != LYC_FP32) return LYC_ERR_INVALID_ARG;
  if (c.select_mode != LYC_SELECT_PER_QHEAD && c.select_mode != LYC_SELECT_KVGROUP_MEAN)
    return LYC_ERR_INVALID_ARG;
  if (c.head_dim != 64 && c.head_dim != 128) return LYC_ERR_UNSUPPORTED;
  if (c.num_q_heads / c.num_kv_heads > kMaxGroup) return LYC_ERR_UNSUPPORTED;
  if (c.max_ctx > kMaxCtxLimit) return LYC_ERR_UNSUPPORTED;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || c.device < 0 || c.device >= ndev)
    return LYC_ERR_INVALID_ARG;
  DeviceGuard guard(c.device);
  if (!guard.ok) return LYC_ERR_CUDA;

  std::unique_ptr<lyc_ctx> holder(new lyc_ctx());
  lyc_ctx* ctx = holder.get();
  ctx->cfg = c;
  ctx->G = c.num_q_heads / c.num_kv_heads;
  ctx->Hs = c.select_mode == LYC_SELECT_KVGROUP_MEAN ? c.num_kv_heads : c.num_q_heads;
  LYC_CUDA(cudaDeviceGetAttribute(&ctx->sms, cudaDevAttrMultiProcessorCount, c.device), "SM count");
  ctx->nstride = round_up(c.max_ctx, 4);
  ctx->KS = static_cast<int>(round_up(c.max_k, 4));
  const int B = c.batch, Hq = c.num_q_heads, Hkv = c.num_kv_heads, D = c.head_dim, L = c.num_layers;
  const size_t es = c.dtype == LYC_BF16 ? 2 : 4;
  // segments of one layer: dense and sparse of its own, plus the sparse
  // passes deferred to it
  const size_t nseg_max = static_cast<size_t>(B) * (Hkv + 2 * Hq);
  // pieces per layer <= 2 * sms + segments (two pooling phases), plus the
  // pool units of the mma kernel (every sparse segment cut into units, at
  // most of the smaller unit size); a launch holds up to kLayersPerLaunch
  // layers
  const size_t unit_rows = static_cast<size_t>(std::min(kPoolTiles, kPoolTilesDep)) * kTileRows;
  const size_t units = (static_cast<size_t>(c.max_k) + unit_rows - 1) / unit_rows;
  ctx->max_parts = (2 * static_cast<size_t>(ctx->sms) + nseg_max + nseg_max * units) * kMaxQ * kLayersPerLaunch;
  ctx->max_counters = nseg_max * kMaxQ;
  auto alloc = [&](void** p, size_t bytes) -> lyc_status {
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return fail(ctx, LYC_ERR_OOM, "cudaMalloc failed");
    }
    return LYC_OK;
  };
  lyc_status st;
  // ready flags: two words per (layer, b, slot); then the step counters;
  // then the epoch
  const size_t flag_words = static_cast<size_t>(L) * B * ctx->Hs * 2 + 2 * 3 * (static_cast<size_t>(L) + 1) + 4;
  if ((st = alloc(reinterpret_cast<void**>(&ctx->status), 16)) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->keys),
                  static_cast<size_t>(L) * B * ctx->Hs * ctx->nstride * sizeof(float))) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->flags), flag_words * sizeof(uint32_t))) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->sbuf),
                  static_cast<size_t>(kSetBuffers) * B * ctx->Hs * ctx->KS * sizeof(int32_t) + 64)) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->part_o), 2 * ctx->max_parts * D * sizeof(float))) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->part_ml), 2 * ctx->max_parts * sizeof(float2))) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->counters), ctx->max_counters * sizeof(int32_t))) != LYC_OK ||
      (st = alloc(&ctx->q_dev, static_cast<size_t>(L) * B * Hq * D * es)) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->out_dev), static_cast<size_t>(L) * B * Hq * D * sizeof(float))) != LYC_OK ||
      (st = alloc(reinterpret_cast<void**>(&ctx->S_dev), static_cast<size_t>(B) * ctx->Hs * c.max_k * sizeof(int32_t))) != LYC_OK) {
    lyc_destroy(holder.release());
    return st;
  }
  ctx->pool_cursors = reinterpret_cast<int32_t*>(ctx->flags + static_cast<size_t>(L) * B * ctx->Hs * 2);
  ctx->epoch = ctx->flags + (flag_words - 4);
  if (c.dtype == LYC_BF16) {
    // one ring per SM index (the SM a CTA runs on owns it; SM indices need
    // not be dense, so twice the count, at least 256)
    ctx->wpart_slots = std::max(256, 2 * ctx->sms);
    const size_t recs = static_cast<size_t>(ctx->wpart_slots) * kPartSlots * kMaxConsumerWarps * kMaxQ;
    if ((st = alloc(reinterpret_cast<void**>(&ctx->wpart_o), recs * D * sizeof(float))) != LYC_OK ||
        (st = alloc(reinterpret_cast<void**>(&ctx->wpart_ml), recs * sizeof(float2))) != LYC_OK) {
      lyc_destroy(holder.release());
      return st;
    }
  }
  if (cudaMemset(ctx->status, 0, 16) != cudaSuccess ||
      cudaMemset(ctx->flags, 0, flag_words * sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(ctx->counters, 0, ctx->max_counters * sizeof(int32_t)) != cudaSuccess ||
      cudaMemset(ctx->sbuf, 0xff, static_cast<size_t>(kSetBuffers) * B * ctx->Hs * ctx->KS * sizeof(int32_t) + 64) !=
          cudaSuccess) {
    lyc_destroy(holder.release());
    return LYC_ERR_CUDA;
  }
  cudaError_t e;
  // kernel attributes: shared-memory sizes and the top-k cluster size
  const int dtype = c.dtype == LYC_BF16 ? 0 : 1;
  if (dtype == 0) {
    int smem = 0;
    e = attn_mma_dispatch(D, nullptr, 0, nullptr, &smem, true);
    if (e == cudaSuccess && D == 128) e = attn_tc_dispatch(nullptr, 0, nullptr, &smem, true);
  } else {
    e = cudaSuccess;
    for (int nqb : {1, 2, 4, 8}) {
      int smem = 0;
      if (e == cudaSuccess) e = attn_simt_dispatch(D, nqb, nullptr, 0, nullptr, &smem, true);
    }
  }
  if (e != cudaSuccess) {
    lyc_destroy(holder.release());
    return LYC_ERR_CUDA;
  }
  const size_t smem16 = topk_smem_for(16, static_cast<int>(c.max_ctx));
  const size_t smem8 = topk_smem_for(8, static_cast<int>(c.max_ctx));
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c.device);
  ctx->topk_cl = (smem16 <= static_cast<size_t>(optin)) ? topk_pick_cluster(smem16) : 8;
  if (ctx->topk_cl == 8) {
    if (smem8 > static_cast<size_t>(optin) || topk_configure(8, smem8) != cudaSuccess) {
      lyc_destroy(holder.release());
      return LYC_ERR_UNSUPPORTED;
    }
  }
  ctx->topk_cls = 1u << ctx->topk_cl;
  // smaller clusters (bigger chunks per CTA) for layers with many sets, so
  // that one selection launch fits the GPU in one wave
  for (int cl : {8, 4}) {
    if (cl >= ctx->topk_cl) continue;
    const size_t sm = topk_smem_for(cl, static_cast<int>(c.max_ctx));
    if (sm <= static_cast<size_t>(optin) && topk_configure(cl, sm) == cudaSuccess) ctx->topk_cls |= 1u << cl;
  }
  for (int cl : {16, 8, 4})
    if (ctx->topk_cls & (1u << cl))
      ctx->topk_resident[cl] = topk_max_clusters(cl, topk_smem_for(cl, static_cast<int>(c.max_ctx)));
  cudaGetLastError();
  *out = holder.release();
  return LYC_OK;
}

void lyc_destroy(lyc_ctx* ctx) {
  if (!ctx) return;
  DeviceGuard guard(ctx->cfg.device);
  for (auto& kv : ctx->plans) free_plan(kv.second.get());
  ctx->plans.clear();
  for (cudaEvent_t ev : ctx->events) cudaEventDestroy(ev);
  void* bufs[] = {ctx->status, ctx->keys, ctx->flags, ctx->sbuf, ctx->part_o, ctx->part_ml,
                  ctx->wpart_o, ctx->wpart_ml, ctx->counters, ctx->q_dev, ctx->out_dev,
                  ctx->S_dev, ctx->corr_dev, ctx->corr_part_o, ctx->corr_part_ml};
  for (void* b : bufs)
    if (b) cudaFree(b);
  timed_steps().erase(ctx);
  delete ctx;
}

}  // extern "C"

namespace {

// The step on a checked KV view (both entry points).
lyc_status step_impl(lyc_ctx* ctx, const void* q, const KvView& kv, const uint8_t* role_mask, int k,
                     float* out, int32_t* S, void* stream_, uint32_t step_flags) {
  lyc_status st = LYC_OK;
  DeviceGuard guard(ctx->cfg.device);
  if (!guard.ok) return fail(ctx, LYC_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const lyc_config& c = ctx->cfg;

  std::string key = plan_key(role_mask, c.num_layers, c.num_q_heads, kv, k, step_flags, q, out, S,
                             ctx->trace, ctx->timing);
  key.append(reinterpret_cast<const char*>(&ctx->timeline), sizeof ctx->timeline);
  key.append(reinterpret_cast<const char*>(&ctx->sel), sizeof ctx->sel);
  Plan* plan = nullptr;
  for (auto it = ctx->plans.begin(); it != ctx->plans.end(); ++it) {
    if (it->first == key) {
      ctx->plans.splice(ctx->plans.begin(), ctx->plans, it);
      plan = ctx->plans.front().second.get();
      break;
    }
  }
  if (!plan) {
    std::unique_ptr<Plan> np(new Plan());
    np->flags = step_flags & (LYC_STEP_S_IN | LYC_STEP_VALIDATE_S);
    np->q = q;
    np->out = out;
    np->S = S;
    np->trace = ctx->trace;
    np->timing = ctx->timing;
    np->timeline = ctx->timeline;
    np->timeline_cap = ctx->timeline_cap;
    st = build_plan(ctx, np.get(), role_mask, kv, k, step_flags);
    if (st != LYC_OK) {
      free_plan(np.get());
      return st;
    }
    ctx->plans.emplace_front(key, std::move(np));
    plan = ctx->plans.front().second.get();
    while (static_cast<int>(ctx->plans.size()) > kPlanCacheSize) {
      free_plan(ctx->plans.back().second.get());
      ctx->plans.pop_back();
    }
  }

  int set = 0;
  if (plan->timing) set = ctx->next_set++ % timing_sets();
  if (step_flags & LYC_STEP_NO_GRAPH) {
    st = enqueue_step(ctx, plan, stream, set, false);
    if (st != LYC_OK) return st;
  } else {
    if (!plan->exec) {
      st = capture_plan(ctx, plan);
      if (st != LYC_OK) return st;
    }
    if (plan->timing) {
      for (int i = 0; i < ctx->events_per_set; ++i) {
        if (!plan->ev_nodes[i]) continue;
        LYC_CUDA(cudaGraphExecEventRecordNodeSetEvent(
                     plan->exec, plan->ev_nodes[i],
                     ctx->events[static_cast<size_t>(set) * ctx->events_per_set + i]),
                 "retarget timing event");
      }
    }
    LYC_CUDA(cudaGraphLaunch(plan->exec, stream), "graph launch");
  }
  if (plan->timing) {
    auto& v = timed_steps()[ctx];
    v.push_back(TimedStep{set, plan->kernel_kind, plan->kernel_layer});
    if (static_cast<int>(v.size()) > timing_sets()) v.erase(v.begin());
  }
  ctx->last_stream = stream;
  {
    int a = 0, t = 0;
    for (int kind : plan->kernel_kind) (kind == 0 ? a : t) += 1;
    int o = 1;  // the final set copy
    if (plan->trace && plan->nfill > 0) ++o;
    if (plan->append) ++o;
    if ((plan->flags & LYC_STEP_S_IN) && (plan->flags & LYC_STEP_VALIDATE_S)) o += ctx->cfg.batch;
    ctx->last_launches[0] = a;
    ctx->last_launches[1] = t;
    ctx->last_launches[2] = o;
  }
  return LYC_OK;
}

lyc_status check_step_args(lyc_ctx* ctx, const void* q, const uint8_t* role_mask, int k, const float* out,
                           const int32_t* S, uint32_t step_flags) {
  if (!q || !role_mask || !out || !S) return fail(ctx, LYC_ERR_INVALID_ARG, "NULL tensor pointer");
  if (k < 1 || k > ctx->cfg.max_k) return fail(ctx, LYC_ERR_INVALID_ARG, "k outside [1, max_k]");
  if (step_flags & ~(LYC_STEP_S_IN | LYC_STEP_NO_GRAPH | LYC_STEP_VALIDATE_S))
    return fail(ctx, LYC_ERR_INVALID_ARG, "unknown step flag");
  return LYC_OK;
}

}  // namespace

extern "C" {

lyc_status lyc_decode_step(lyc_ctx* ctx, const void* q, const lyc_kv_cache* kv,
                           const uint8_t* role_mask, int k, float* out, int32_t* S,
                           void* stream_, uint32_t step_flags) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  lyc_status st = check_step_args(ctx, q, role_mask, k, out, S, step_flags);
  if (st == LYC_OK) st = check_kv(ctx, kv);
  if (st != LYC_OK) return st;
  return step_impl(ctx, q, view_of(kv, ctx->cfg.batch), role_mask, k, out, S, stream_, step_flags);
}

lyc_status lyc_decode_step_batch(lyc_ctx* ctx, const void* q, const lyc_kv_batch* kv,
                                 const uint8_t* role_mask, int k, float* out, int32_t* S,
                                 void* stream_, uint32_t step_flags) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  lyc_status st = check_step_args(ctx, q, role_mask, k, out, S, step_flags);
  if (st == LYC_OK) st = check_kv_batch(ctx, kv);
  if (st != LYC_OK) return st;
  return step_impl(ctx, q, view_of(kv, ctx->cfg.batch), role_mask, k, out, S, stream_, step_flags);
}

lyc_status lyc_cache_correction(lyc_ctx* ctx, const void* q, const lyc_kv_cache* kv, int T,
                                const void* k_new, const void* v_new, float* out, void* stream_) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  const lyc_config& c = ctx->cfg;
  if (!q || !kv || !kv->k || !kv->v || !out)
    return fail(ctx, LYC_ERR_INVALID_ARG, "NULL pointer");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(ctx, LYC_ERR_INVALID_ARG, "k_new and v_new go together");
  if (c.dtype != LYC_BF16 || c.head_dim != 128)
    return fail(ctx, LYC_ERR_UNSUPPORTED, "Cache Correction runs on bf16 with head_dim 128");
  const int L = c.num_layers, B = c.batch, Hq = c.num_q_heads, Hkv = c.num_kv_heads, G = ctx->G;
  const int64_t n = kv->n;
  if (T < 1 || n < T || n > c.max_ctx) return fail(ctx, LYC_ERR_INVALID_ARG, "need 1 <= T <= n <= max_ctx");
  if (static_cast<int64_t>(G) * T > 128)
    return fail(ctx, LYC_ERR_UNSUPPORTED, "G * T query rows must fit one 128-row block");
  auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (misaligned(q) || misaligned(out) || misaligned(kv->k) || misaligned(kv->v) ||
      (k_new && (misaligned(k_new) || misaligned(v_new))))
    return fail(ctx, LYC_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (kv->s_token < c.head_dim || kv->s_token % 8 || kv->s_head % 8 || kv->s_batch % 8 || kv->s_layer % 8)
    return fail(ctx, LYC_ERR_INVALID_ARG, "cache strides must be multiples of 8 elements, rows >= head_dim");
  DeviceGuard guard(c.device);
  if (!guard.ok) return fail(ctx, LYC_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (!ctx->corr_configured) {
    LYC_CUDA(correction_configure(), "correction kernel attributes");
    ctx->corr_configured = true;
  }
  // the work pool: the (l, b, g) groups' tiles cut into equal runs, one per CTA
  if (ctx->corr_n != n || ctx->corr_T != T) {
    const int64_t NT = (n + 127) / 128;
    const int64_t ngroups = static_cast<int64_t>(L) * B * Hkv;
    const int64_t TT = ngroups * NT;
    const int grid = static_cast<int>(std::min<int64_t>(TT, ctx->sms));
    std::vector<CorrPiece> pieces;
    std::vector<int32_t> cta(1, 0), group_first(ngroups + 1, 0);
    for (int cc = 0; cc < grid; ++cc) {
      const int64_t t0 = TT * cc / grid, t1 = TT * (cc + 1) / grid;
      for (int64_t x = t0; x < t1;) {
        const int64_t grp = x / NT;
        const int64_t end = std::min(t1, (grp + 1) * NT);
        CorrPiece pc;
        pc.g = static_cast<int32_t>(grp % Hkv);
        pc.b = static_cast<int32_t>((grp / Hkv) % B);
        pc.l = static_cast<int32_t>(grp / (static_cast<int64_t>(Hkv) * B));
        pc.t0 = static_cast<int32_t>(x - grp * NT);
        pc.t1 = static_cast<int32_t>(end - grp * NT);
        pc.part = static_cast<int32_t>(pieces.size());
        pieces.push_back(pc);
        group_first[grp + 1] = static_cast<int32_t>(pieces.size());
        x = end;
      }
      cta.push_back(static_cast<int32_t>(pieces.size()));
    }
    for (int64_t j = 1; j <= ngroups; ++j) group_first[j] = std::max(group_first[j], group_first[j - 1]);
    size_t bytes = pieces.size() * sizeof(CorrPiece);
    const size_t off_cta = round_up(static_cast<int64_t>(bytes), 64);
    bytes = off_cta + cta.size() * sizeof(int32_t);
    const size_t off_group = round_up(static_cast<int64_t>(bytes), 64);
    bytes = off_group + group_first.size() * sizeof(int32_t);
    std::vector<unsigned char> host(bytes, 0);
    memcpy(host.data(), pieces.data(), pieces.size() * sizeof(CorrPiece));
    memcpy(host.data() + off_cta, cta.data(), cta.size() * sizeof(int32_t));
    memcpy(host.data() + off_group, group_first.data(), group_first.size() * sizeof(int32_t));
    if (ctx->corr_dev) {
      LYC_CUDA(cudaFree(ctx->corr_dev), "cudaFree(correction pool)");
      ctx->corr_dev = nullptr;
    }
    ctx->corr_n = -1;
    LYC_CUDA(cudaMalloc(&ctx->corr_dev, bytes), "cudaMalloc(correction pool)");
    LYC_CUDA(cudaMemcpy(ctx->corr_dev, host.data(), bytes, cudaMemcpyHostToDevice), "upload correction pool");
    if (pieces.size() > ctx->corr_parts_cap) {
      if (ctx->corr_part_o) cudaFree(ctx->corr_part_o);
      if (ctx->corr_part_ml) cudaFree(ctx->corr_part_ml);
      ctx->corr_part_o = nullptr;
      ctx->corr_part_ml = nullptr;
      ctx->corr_parts_cap = 0;
      // two partial records per piece (its two key halves)
      LYC_CUDA(cudaMalloc(&ctx->corr_part_o, 2 * pieces.size() * 128 * 128 * sizeof(float)), "cudaMalloc(correction partials)");
      LYC_CUDA(cudaMalloc(&ctx->corr_part_ml, 2 * pieces.size() * 128 * sizeof(float2)), "cudaMalloc(correction partials)");
      ctx->corr_parts_cap = pieces.size();
    }
    ctx->corr_n = n;
    ctx->corr_T = T;
    ctx->corr_grid = grid;
    ctx->corr_npieces = static_cast<int>(pieces.size());
    ctx->corr_off_cta = off_cta;
    ctx->corr_off_group = off_group;
  }
  CorrParams P;
  memset(&P, 0, sizeof P);
  const KvView w = view_of(kv, B);
  lyc_status st = encode_cache_map(ctx, &P.tmk, kv->k, w, 128);
  if (st == LYC_OK) st = encode_cache_map(ctx, &P.tmv, kv->v, w, 128);
  if (st != LYC_OK) return st;
  P.q = q;
  P.out = out;
  P.pieces = reinterpret_cast<const CorrPiece*>(ctx->corr_dev);
  P.cta_begin = reinterpret_cast<const int32_t*>(ctx->corr_dev + ctx->corr_off_cta);
  P.group_first = reinterpret_cast<const int32_t*>(ctx->corr_dev + ctx->corr_off_group);
  P.part_o = ctx->corr_part_o;
  P.part_ml = ctx->corr_part_ml;
  P.status = ctx->status;
  P.L = L;
  P.B = B;
  P.Hq = Hq;
  P.Hkv = Hkv;
  P.G = G;
  P.T = T;
  P.n = static_cast<int32_t>(n);
  P.rows = G * T;
  P.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  WriteRowsParams wr{};
  if (k_new) {
    wr.k_new = static_cast<const unsigned char*>(k_new);
    wr.v_new = static_cast<const unsigned char*>(v_new);
    wr.k = static_cast<unsigned char*>(const_cast<void*>(kv->k));
    wr.v = static_cast<unsigned char*>(const_cast<void*>(kv->v));
    wr.s_layer = kv->s_layer;
    wr.s_batch = kv->s_batch;
    wr.s_head = kv->s_head;
    wr.s_token = kv->s_token;
    wr.L = L;
    wr.B = B;
    wr.Hkv = Hkv;
    wr.T = T;
    wr.n = static_cast<int32_t>(n);
    wr.row_bytes = c.head_dim * 2;
    wr.elem_bytes = 2;
  }
  LYC_CUDA(correction_launch(&P, ctx->corr_grid, k_new ? &wr : nullptr, stream), "correction launch");
  ctx->last_stream = stream;
  return LYC_OK;
}

lyc_status lyc_decode_step_host(lyc_ctx* ctx, const void* q_host, const lyc_kv_cache* kv,
                                const uint8_t* role_mask, int k, float* out_host, int32_t* S_host,
                                void* stream_, uint32_t step_flags) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  if (!q_host || !out_host || !S_host) return fail(ctx, LYC_ERR_INVALID_ARG, "NULL host pointer");
  if (k < 1 || k > ctx->cfg.max_k) return fail(ctx, LYC_ERR_INVALID_ARG, "k outside [1, max_k]");
  DeviceGuard guard(ctx->cfg.device);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const lyc_config& c = ctx->cfg;
  const size_t es = c.dtype == LYC_BF16 ? 2 : 4;
  const size_t qbytes = static_cast<size_t>(c.num_layers) * c.batch * c.num_q_heads * c.head_dim * es;
  const size_t obytes = static_cast<size_t>(c.num_layers) * c.batch * c.num_q_heads * c.head_dim * 4;
  const size_t sbytes = static_cast<size_t>(c.batch) * ctx->Hs * k * 4;
  lyc_status st = check_kv(ctx, kv);
  if (st != LYC_OK) return st;
  LYC_CUDA(cudaMemcpyAsync(ctx->q_dev, q_host, qbytes, cudaMemcpyHostToDevice, stream), "q to device");
  if (step_flags & LYC_STEP_S_IN)
    LYC_CUDA(cudaMemcpyAsync(ctx->S_dev, S_host, sbytes, cudaMemcpyHostToDevice, stream), "S to device");
  st = lyc_decode_step(ctx, ctx->q_dev, kv, role_mask, k, ctx->out_dev, ctx->S_dev, stream_, step_flags);
  if (st != LYC_OK) return st;
  LYC_CUDA(cudaMemcpyAsync(out_host, ctx->out_dev, obytes, cudaMemcpyDeviceToHost, stream), "out to host");
  LYC_CUDA(cudaMemcpyAsync(S_host, ctx->S_dev, sbytes, cudaMemcpyDeviceToHost, stream), "S to host");
  return LYC_OK;
}

lyc_status lyc_sync_status(lyc_ctx* ctx) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->cfg.device);
  LYC_CUDA(ctx->last_stream ? cudaStreamSynchronize(ctx->last_stream) : cudaDeviceSynchronize(),
           "synchronize");
  uint32_t word = 0;
  LYC_CUDA(cudaMemcpy(&word, ctx->status, sizeof word, cudaMemcpyDeviceToHost), "read status");
  LYC_CUDA(cudaMemset(ctx->status, 0, sizeof word), "clear status");
  if (word & kStatusTimeout) return fail(ctx, LYC_ERR_TIMEOUT, "a device-side wait gave up");
  if (word & kStatusScratch)
    return fail(ctx, LYC_ERR_CUDA, "a CTA ran on an SM index beyond the per-SM scratch (no work done)");
  if (word & (kStatusBadIndex | kStatusEmptySoftmax))
    return fail(ctx, LYC_ERR_BAD_INDEX, "an inherited set held an index outside [0, n)");
  return LYC_OK;
}

lyc_status lyc_set_selection(lyc_ctx* ctx, const lyc_selection* sel) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  lyc_selection s{};
  s.rule = LYC_RULE_TOPK;
  if (sel) s = *sel;
  switch (s.rule) {
    case LYC_RULE_TOPK: break;
    case LYC_RULE_RATIO:
      if (s.ratio_den < 1 || s.ratio_num < 0 || s.ratio_num > (1ll << 32) || s.ratio_den > (1ll << 32))
        return fail(ctx, LYC_ERR_INVALID_ARG, "ratio needs 0 <= num, 1 <= den (both below 2^32)");
      break;
    case LYC_RULE_BLOCK_TOPK:
      if (s.block < 1 || s.block > ctx->cfg.max_k)
        return fail(ctx, LYC_ERR_INVALID_ARG, "block selection needs 1 <= block <= max_k");
      break;
    case LYC_RULE_TOPP:
      if (!(s.p > 0.0 && s.p <= 1.0)) return fail(ctx, LYC_ERR_INVALID_ARG, "top-p needs 0 < p <= 1");
      break;
    case LYC_RULE_THRESHOLD:
      if (!(s.tau >= 0.0)) return fail(ctx, LYC_ERR_INVALID_ARG, "threshold needs tau >= 0");
      break;
    default: return fail(ctx, LYC_ERR_INVALID_ARG, "unknown selection rule");
  }
  // only the fields of the rule take part in the plan key
  lyc_selection c{};
  c.rule = s.rule;
  if (s.rule == LYC_RULE_RATIO) {
    c.ratio_num = s.ratio_num;
    c.ratio_den = s.ratio_den;
  }
  if (s.rule == LYC_RULE_BLOCK_TOPK) c.block = s.block;
  if (s.rule == LYC_RULE_TOPP) c.p = s.p;
  if (s.rule == LYC_RULE_THRESHOLD) c.tau = s.tau;
  DeviceGuard guard(ctx->cfg.device);
  if (!guard.ok) return fail(ctx, LYC_ERR_CUDA, "cudaSetDevice failed");
  // the cached plans hold the old rule's records
  for (auto& kv : ctx->plans) free_plan(kv.second.get());
  ctx->plans.clear();
  ctx->sel = c;
  return LYC_OK;
}

lyc_status lyc_set_s_trace(lyc_ctx* ctx, int32_t* trace) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  ctx->trace = trace;
  return LYC_OK;
}

lyc_status lyc_set_timeline(lyc_ctx* ctx, unsigned long long* buf, int cap) {
  if (!ctx || (buf && cap < 1)) return LYC_ERR_INVALID_ARG;
  ctx->timeline = buf;
  ctx->timeline_cap = buf ? cap : 0;
  return LYC_OK;
}

lyc_status lyc_set_timing(lyc_ctx* ctx, int mode) {
  if (!ctx || (mode != LYC_TIMING_OFF && mode != LYC_TIMING_ON)) return LYC_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->cfg.device);
  if (mode == LYC_TIMING_ON && ctx->events.empty()) {
    ctx->events_per_set = 4 * ctx->cfg.num_layers + 2;  // + the last layer's combine launch
    const size_t total = static_cast<size_t>(timing_sets()) * ctx->events_per_set;
    ctx->events.resize(total, nullptr);
    for (size_t i = 0; i < total; ++i)
      LYC_CUDA(cudaEventCreate(&ctx->events[i]), "cudaEventCreate");
  }
  ctx->timing = mode == LYC_TIMING_ON;
  return LYC_OK;
}

lyc_status lyc_kernel_times(lyc_ctx* ctx, lyc_kernel_time* times, int cap, int* count) {
  if (!ctx || !count || (cap > 0 && !times)) return LYC_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->cfg.device);
  LYC_CUDA(ctx->last_stream ? cudaStreamSynchronize(ctx->last_stream) : cudaDeviceSynchronize(),
           "synchronize");
  int nout = 0;
  auto& v = timed_steps()[ctx];
  for (const TimedStep& ts : v) {
    for (size_t i = 0; i < ts.kind.size(); ++i) {
      if (nout >= cap) break;
      float ms = 0.f;
      const size_t base = static_cast<size_t>(ts.set) * ctx->events_per_set;
      LYC_CUDA(cudaEventElapsedTime(&ms, ctx->events[base + 2 * i], ctx->events[base + 2 * i + 1]),
               "event elapsed time");
      times[nout].kind = ts.kind[i];
      times[nout].layer = ts.layer[i];
      times[nout].ms = ms;
      ++nout;
    }
  }
  v.clear();
  *count = nout;
  return LYC_OK;
}

lyc_status lyc_step_launches(const lyc_ctx* ctx, int* attention, int* selection, int* other) {
  if (!ctx || !attention || !selection || !other || ctx->last_launches[0] < 0) return LYC_ERR_INVALID_ARG;
  *attention = ctx->last_launches[0];
  *selection = ctx->last_launches[1];
  *other = ctx->last_launches[2];
  return LYC_OK;
}

lyc_status lyc_topk_f32_ex(lyc_ctx* ctx, const float* keys, int64_t n, int k, int32_t* S, int cluster,
                           int variant, void* stream) {
  if (!ctx) return LYC_ERR_INVALID_ARG;
  if (!keys || !S) return fail(ctx, LYC_ERR_INVALID_ARG, "NULL pointer");
  if (n < 1 || n > ctx->cfg.max_ctx) return fail(ctx, LYC_ERR_INVALID_ARG, "n outside [1, max_ctx]");
  if (k < 1 || k > ctx->cfg.max_k) return fail(ctx, LYC_ERR_INVALID_ARG, "k outside [1, max_k]");
  if (variant != LYC_TOPK_FIXED && variant != LYC_TOPK_RULES)
    return fail(ctx, LYC_ERR_INVALID_ARG, "unknown selection instantiation");
  const int cl = cluster == 0 ? ctx->topk_cl : cluster;
  if (cl != 4 && cl != 8 && cl != 16) return fail(ctx, LYC_ERR_INVALID_ARG, "cluster size not in {4, 8, 16}");
  if (!(ctx->topk_cls & (1u << cl)))
    return fail(ctx, LYC_ERR_UNSUPPORTED, "cluster size not configured for this context's max_ctx");
  DeviceGuard guard(ctx->cfg.device);
  TopkParams tp{};
  tp.tasks = nullptr;
  tp.single.keys = keys;
  tp.single.S = S;
  tp.n = static_cast<int>(n);
  tp.k = k;
  LYC_CUDA(topk_launch(cl, &tp, 1, static_cast<cudaStream_t>(stream), variant == LYC_TOPK_RULES),
           "top-k launch");
  ctx->last_stream = static_cast<cudaStream_t>(stream);
  return LYC_OK;
}

lyc_status lyc_topk_f32(lyc_ctx* ctx, const float* keys, int64_t n, int k, int32_t* S, void* stream) {
  return lyc_topk_f32_ex(ctx, keys, n, k, S, 0, LYC_TOPK_FIXED, stream);
}

lyc_status lyc_step_bytes(const lyc_config* cfg, const uint8_t* role_mask, int64_t n, int k, int s_in,
                          uint64_t* analytic, uint64_t* distinct) {
  if (!cfg || !role_mask || !analytic || !distinct || n < 1 || k < 1) return LYC_ERR_INVALID_ARG;
  const lyc_config& c = *cfg;
  if (c.num_kv_heads < 1 || c.num_q_heads % c.num_kv_heads != 0) return LYC_ERR_INVALID_ARG;
  const int G = c.num_q_heads / c.num_kv_heads;
  const uint64_t row = static_cast<uint64_t>(c.head_dim) * (c.dtype == LYC_BF16 ? 2 : 4) * 2;  // K + V
  const uint64_t keff = static_cast<uint64_t>(std::min<int64_t>(k, n));
  const bool kvmode = c.select_mode == LYC_SELECT_KVGROUP_MEAN;
  uint64_t a = 0, d = 0;
  for (int l = 0; l < c.num_layers; ++l) {
    for (int g = 0; g < c.num_kv_heads; ++g) {
      int nret = 0, nsp = 0;
      for (int h = g * G; h < (g + 1) * G; ++h) {
        const bool r = (l == 0 && !s_in) || role_mask[static_cast<int64_t>(l) * c.num_q_heads + h];
        nret += r;
        nsp += !r;
      }
      const uint64_t full = static_cast<uint64_t>(n) * row, part = keff * row;
      a += nret ? full : part;
      d += nret ? full : 0;
      d += kvmode ? (nsp ? part : 0) : static_cast<uint64_t>(nsp) * part;
    }
  }
  *analytic = a * c.batch;
  *distinct = d * c.batch;
  return LYC_OK;
}

}  // extern "C"
