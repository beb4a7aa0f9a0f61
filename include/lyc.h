/*
 * lyc.h -- C ABI of liblyc.so, the B200 (sm_100a) hybrid-head sparse
 * decode-attention step of LycheeDecode.
 *
 * The operation (page "LycheeDecode: Accelerating Long-Context LLM Inference
 * via Hybrid-Head Sparse Decoding", paper-graph-ui summary):
 *   for each layer l = 0..L-1, batch element b and query head h
 *   - retrieval head (section 3.4 Eq. 1; Appendix B, Algorithm 1):
 *       o = softmax(q K^T / sqrt(d)) V over all n cached rows of h's KV group,
 *       then S^(l+1) = argsTopK of its scores, k rows (section 3.4 Eq. 2);
 *   - sparse head (section 3.4 Eq. 3): o = softmax(q K[S]^T / sqrt(d)) V[S]
 *       over the k rows of the set it inherits, which it passes on unchanged;
 *   - every head of layer 0 is a retrieval head (section 3.4, initialisation
 *     of the propagation chain);
 *   - GQA: query head h uses KV head h / (Hq/Hkv).  In LYC_SELECT_KVGROUP_MEAN
 *     the group's queries are averaged before selection, one set per KV group
 *     (section 3.4, hyperparameter summary: "Q heads average-pooled").
 * Readings where the pages are silent: top-k is taken over the logits (same
 * set as over softmax scores), ties go to the lower token index, -0 == +0,
 * S is stored in ascending order and padded with -1 when k > n.
 *
 * Conventions for every entry point:
 *   - All tensors are owned by the caller and must stay valid until the work
 *     enqueued on `stream` has finished.  Device pointers live on the
 *     context's device.  The library never frees caller memory.
 *   - The library owns its scratch (partial softmax states, selection keys,
 *     set buffers, work lists) and its CUDA graphs; lyc_destroy frees them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream).  A context is not thread-safe.
 *   - Errors found on the host are returned at once and nothing is enqueued.
 *     Errors found on the device (bad inherited index, wait timeout) are
 *     latched in a device status word and returned by lyc_sync_status.
 */
#ifndef LYC_H_
#define LYC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LYC_OK = 0,
  LYC_ERR_INVALID_ARG = -1, /* bad pointer, shape, stride, alignment or k */
  LYC_ERR_UNSUPPORTED = -2, /* shape outside what the kernels are built for */
  LYC_ERR_OOM = -3,         /* a library allocation failed */
  LYC_ERR_CUDA = -4,        /* a CUDA call failed; see lyc_last_error */
  LYC_ERR_BAD_INDEX = -5,   /* an inherited set held an index outside [0, n) */
  LYC_ERR_TIMEOUT = -6,     /* a device-side wait gave up (kernel returned early) */
  LYC_ERR_SCRATCH_LIMIT = -7 /* lyc_sparse_attention_noalloc: the request exceeds its fixed scratch */
} lyc_status;

typedef enum { LYC_BF16 = 0, LYC_FP32 = 1 } lyc_dtype;

typedef enum {
  LYC_SELECT_PER_QHEAD = 0,   /* one set per query head: Hs = Hq */
  LYC_SELECT_KVGROUP_MEAN = 1 /* one set per KV head, key from the mean query: Hs = Hkv */
} lyc_select_mode;

typedef struct {
  int num_layers;   /* L >= 1 */
  int batch;        /* B >= 1 */
  int num_q_heads;  /* Hq >= 1 */
  int num_kv_heads; /* Hkv >= 1, Hq % Hkv == 0, Hq / Hkv <= 8 */
  int head_dim;     /* d in {64, 128} */
  int64_t max_ctx;  /* largest n any step will use, 1 <= max_ctx <= 655360 */
  int max_k;        /* largest k any step will use, >= 1 */
  lyc_dtype dtype;  /* element type of q, K and V */
  lyc_select_mode select_mode;
  int device;       /* CUDA device ordinal */
  uint32_t flags;   /* 0, or LYC_CFG_* bits below */
} lyc_config;

/* cfg.flags: gather the inherited K/V rows with TMA four-row gathers
 * (cp.async.bulk.tensor ... tile::gather4, one producer warp) instead of
 * 16-byte cp.async copies from eight producer warps.  Measured on B200 the
 * TMA form lands a gathered tile several times later than cp.async, so it is
 * off by default; it is kept for comparison.  It needs a flattened row view of
 * the cache (head, batch and layer strides that are whole multiples of
 * s_token, under 2^31 rows); without one the library uses cp.async anyway.
 * Results are the same either way. */
#define LYC_CFG_TMA_GATHER 0x1u
/* cfg.flags: run bf16 attention with head_dim 128 on the tcgen05 tensor-core
 * kernel (accumulators in tensor memory, 128-row tiles, one MMA-issuing
 * thread) instead of the mma.sync kernel (64-row tiles, register
 * accumulators, six consumer warps).  Measured on B200 the mma.sync kernel is
 * faster for this path (it keeps more bytes in flight per SM: six 32 KiB
 * stages consumed in parallel against three 64 KiB stages consumed in turn),
 * so it is the default; results agree within rounding. */
#define LYC_CFG_TCGEN05 0x2u

/* The KV cache of all layers.  Element (l, b, g, i, j) of K (and of V) is at
 * element offset l*s_layer + b*s_batch + g*s_head + i*s_token + j, j < d
 * contiguous.  All strides are in elements and must make every row start on a
 * 16-byte boundary (s_token*elem, s_head*elem, ... multiples of 16 bytes; base
 * pointers 16-byte aligned).  n rows are valid, the current token included
 * (it is appended before attention, Algorithm 1). */
typedef struct {
  const void* k;
  const void* v;
  int64_t n;
  int64_t s_layer, s_batch, s_head, s_token;
} lyc_kv_cache;

/* step_flags */
#define LYC_STEP_S_IN 0x1u       /* S holds S^(0) on entry; role row 0 is obeyed */
#define LYC_STEP_NO_GRAPH 0x2u   /* launch the kernels directly, no CUDA graph */
#define LYC_STEP_VALIDATE_S 0x4u /* with S_IN: check S^(0) on the device first */

typedef struct lyc_ctx lyc_ctx;

/* Create a context on cfg->device.  Allocates the library's scratch for the
 * largest step the config allows.  *out receives the context.
 * Errors: INVALID_ARG (NULL, bad sizes), UNSUPPORTED (d, dtype, group size),
 * OOM, CUDA. */
lyc_status lyc_create(const lyc_config* cfg, lyc_ctx** out);

/* One decode step of the L-layer attention stack.
 *   q         device, [L][B][Hq][d] of cfg->dtype, contiguous
 *   kv        host struct describing the device KV cache (n <= max_ctx)
 *   role_mask host, [L][Hq] uint8, 1 = retrieval head.  Row 0 is ignored
 *             (all retrieval) unless LYC_STEP_S_IN is set.
 *   k         token budget, 1 <= k <= max_k; k > n selects all n rows and
 *             pads the rest of each set with -1
 *   out       device, [L][B][Hq][d] float32, contiguous; fully written
 *   S         device, [B][Hs][k] int32, contiguous.  In: S^(0) when
 *             LYC_STEP_S_IN.  Out: S^(L), each set ascending, -1 padded.
 *   stream    cudaStream_t
 * The first step with a given (role mask, n, k, flags, pointers) builds the
 * work lists and captures a CUDA graph; later identical steps replay it.
 * Errors: INVALID_ARG, CUDA (host side); BAD_INDEX, TIMEOUT (device side,
 * via lyc_sync_status). */
lyc_status lyc_decode_step(lyc_ctx* ctx, const void* q, const lyc_kv_cache* kv,
                           const uint8_t* role_mask, int k, float* out, int32_t* S,
                           void* stream, uint32_t step_flags);

/* The same step with q, out and S in HOST memory (pinned memory gives
 * asynchronous copies).  The host-to-device copy of q (and of S with
 * LYC_STEP_S_IN) and the device-to-host copies of out and S are enqueued on
 * `stream` around the step, into library-owned device buffers.  The KV cache
 * stays on the device.  The host buffers must stay valid until the stream
 * has finished the step. */
lyc_status lyc_decode_step_host(lyc_ctx* ctx, const void* q_host, const lyc_kv_cache* kv,
                                const uint8_t* role_mask, int k, float* out_host,
                                int32_t* S_host, void* stream, uint32_t step_flags);

/* The serving form of the step: a batch whose elements have cache lengths of
 * their own, the cache either contiguous (as lyc_kv_cache) or in pages named
 * by a block table, and the current token's K and V written into the cache
 * as part of the step.  Page "LycheeDecode ..." (paper-graph-ui summary),
 * Appendix B, Algorithm 1: each decode step appends the current token's K and
 * V to the cache before the layer's attention; the attention and selection of
 * every batch element then run over its own n[b] rows exactly as in
 * lyc_decode_step (section 3.4 Eq. 1-3).
 *
 * Row i < n[b] of (layer l, batch b, KV head g), element j < d:
 *   contiguous (block_table == NULL):
 *     l*s_layer + b*s_batch + g*s_head + i*s_token + j
 *   paged (block_table != NULL): page p = block_table[b*max_blocks + i/page_rows],
 *     l*s_layer + p*s_page + (i % page_rows)*s_token + g*s_head + j
 * (s_batch is unused when paged; s_page when contiguous).  Strides are in
 * elements and must keep every row 16-byte aligned; page_rows is a multiple
 * of 64; every page a batch element uses lies in the allocation and is used
 * by that element only. */
typedef struct {
  const void* k;               /* device: K (the cache, or the page pool) */
  const void* v;               /* device: V, same layout */
  const int64_t* n;            /* host, [B]: rows of each element, its current token included */
  int64_t s_layer, s_batch, s_head, s_token, s_page;
  const int32_t* block_table;  /* device, [B][max_blocks] page indices, or NULL (contiguous) */
  int32_t page_rows;           /* rows per page (paged) */
  int32_t max_blocks;          /* block-table row length (paged) */
  int64_t num_pages;           /* pages in the pool, every block-table entry below it (paged) */
  const void* k_new;           /* device, [L][B][Hkv][d] of cfg->dtype: the current token's K,
                                  written at row n[b]-1 of every (l, b, g) before attention;
                                  or NULL (the cache already holds it) */
  const void* v_new;           /* device, the same for V (NULL iff k_new is NULL) */
} lyc_kv_batch;

/* One decode step over a lyc_kv_batch; q, role_mask, k, out, S, stream and
 * step_flags as in lyc_decode_step (LYC_STEP_S_IN: each S^(0) set of element
 * b must hold indices below n[b]).  Every n[b] is >= 1 and <= cfg->max_ctx;
 * element b's sets hold min(k, n[b]) indices, padded with -1.  The appended
 * rows are written before any layer reads the cache and stay in it after the
 * step (the caller's cache is modified).
 * Errors: INVALID_ARG (NULL pointers, n out of range, page_rows not a
 * multiple of 64, misaligned strides), UNSUPPORTED (paged layout with the
 * tcgen05 kernel or fp32), CUDA; BAD_INDEX, TIMEOUT via lyc_sync_status. */
lyc_status lyc_decode_step_batch(lyc_ctx* ctx, const void* q, const lyc_kv_batch* kv,
                                 const uint8_t* role_mask, int k, float* out, int32_t* S,
                                 void* stream, uint32_t step_flags);

/* ---- Selection rules (page "LycheeDecode: Accelerating Long-Context LLM
 * Inference via Hybrid-Head Sparse Decoding", paper-graph-ui summary: section
 * 4.4.1 with Figure 6 and Tables 5-6 compare Top-k, Top-p, Threshold and
 * Ratio; section 4.1 / Appendix F give the reasoning budget of 50 % of the
 * length, growing during decoding; the kernel section uses blocks of 64 rows).
 *
 * Every rule chooses rows from the same selection key as argsTopK (Eq. 2:
 * the retrieval head's logits, or the pooled query's in KVGROUP_MEAN mode);
 * A = softmax(key) are their probabilities.  A set never holds more than the
 * step's k rows, is written ascending and padded with -1, and holds at least
 * one row:
 *   TOPK        : the min(k, n) largest keys (ties to the lower index);
 *   RATIO       : the ceil(ratio_num * n / ratio_den) largest keys (integer
 *                 arithmetic; at least 1, at most k).  The reasoning budget is
 *                 ratio 1/2 evaluated with each step's n;
 *   BLOCK_TOPK  : rows in blocks of `block` (the last one may be shorter); a
 *                 block's score is the sum of its rows' A; the floor(k / block)
 *                 best blocks (ties to the lower block) are taken whole.  Needs
 *                 1 <= block <= k;
 *   TOPP        : the fewest largest keys whose A sum to at least p, 0 < p <= 1;
 *   THRESHOLD   : the keys with A >= tau, 0 <= tau.
 * TOPP and THRESHOLD decide on 40-bit fixed-point weights round(2^40 exp(key -
 * max key)) and BLOCK_TOPK on fp32 block scores: a row whose fp64 mass sits
 * within rounding of the boundary may fall on either side of it.
 * Sets of BLOCK_TOPK, TOPP and THRESHOLD can hold fewer rows than their
 * capacity; the sparse heads attend over their valid entries only.
 *
 * lyc_set_selection(ctx, NULL) restores TOPK.  The rule applies to the steps
 * that follow (every step entry point); changing it releases the cached step
 * plans.  Errors: INVALID_ARG (unknown rule, block < 1, ratio_den < 1,
 * ratio_num < 0, p outside (0, 1], tau < 0), OOM, CUDA.  BLOCK_TOPK with a
 * step k below `block` fails at the step with INVALID_ARG. */
typedef enum {
  LYC_RULE_TOPK = 0,
  LYC_RULE_RATIO = 1,
  LYC_RULE_BLOCK_TOPK = 2,
  LYC_RULE_TOPP = 3,
  LYC_RULE_THRESHOLD = 4
} lyc_rule;

typedef struct {
  int32_t rule;       /* lyc_rule */
  int32_t block;      /* BLOCK_TOPK: rows per block */
  int64_t ratio_num;  /* RATIO: theta = ratio_num / ratio_den */
  int64_t ratio_den;
  double p;           /* TOPP */
  double tau;         /* THRESHOLD */
} lyc_selection;

lyc_status lyc_set_selection(lyc_ctx* ctx, const lyc_selection* sel);

/* ---- Cache Correction (page "LycheeDecode: Accelerating Long-Context LLM
 * Inference via Hybrid-Head Sparse Decoding", paper-graph-ui summary: section
 * 4.2.2, and the decoding setup of section 4.1 / Appendix F).  Every 32
 * decoded tokens, the T most recent positions are prefilled again with dense
 * attention, and their K/V representations are updated.  This call runs the
 * attention part of that prefill for every layer, batch element and query
 * head: query t sits at position p = n - T + t and attends rows 0..p of the
 * cache (causal):
 *   out[l][b][h][t] = softmax(q[l][b][h][t] . K[0..p]^T / sqrt(d)) V[0..p].
 *
 *   q      device [L][B][Hq][T][d] bf16, 16-byte aligned
 *   kv     the cache as in lyc_decode_step: kv->n counts the T positions
 *   k_new, v_new  device [L][B][Hkv][T][d] bf16, or both NULL: the refreshed
 *          K/V of the T positions, written at rows n-T .. n-1 before the
 *          attention (the caller's cache is modified)
 *   out    device [L][B][Hq][T][d] fp32
 *   stream cudaStream_t (NULL: legacy stream)
 * Asynchronous like lyc_decode_step; lyc_sync_status reports device errors.
 * Needs bf16, head_dim 128, and (Hq/Hkv) * T <= 128.  The set buffers are not
 * touched: the next decode step starts its layer 0 from all retrieval heads
 * as always.  Errors: INVALID_ARG (NULL or misaligned pointers, T outside
 * [1, n], n > max_ctx, bad strides), UNSUPPORTED (fp32, head_dim 64, G*T >
 * 128), OOM, CUDA. */
lyc_status lyc_cache_correction(lyc_ctx* ctx, const void* q, const lyc_kv_cache* kv, int T,
                                const void* k_new, const void* v_new, float* out, void* stream);

/* Synchronize the stream of the last step, read and clear the device status
 * word.  Returns LYC_OK, LYC_ERR_BAD_INDEX, LYC_ERR_TIMEOUT or LYC_ERR_CUDA. */
lyc_status lyc_sync_status(lyc_ctx* ctx);

/* Record every layer's outgoing sets: trace is device [L][B][Hs][k] int32
 * (k of the steps that follow); trace[l] = the sets after layer l.  NULL turns
 * recording off.  Debug and test use.  The selection kernels write the rows of
 * the sets they refresh as they write the sets themselves, and one copy launch
 * at the end of the step fills the rows of the sets that a layer passed on
 * unchanged, so a traced step runs the same launches between its layers as an
 * untraced one. */
lyc_status lyc_set_s_trace(lyc_ctx* ctx, int32_t* trace);

/* Bytes one step must read from the KV cache (host-only arithmetic).
 *   analytic: full K+V of every KV group with a retrieval head at a layer,
 *             plus min(k, n) K+V rows for every group with sparse heads only.
 *   distinct: K+V bytes the kernels actually read: full groups as above, and
 *             for every sparse-head pass (per query head in PER_QHEAD mode, per
 *             group in KVGROUP_MEAN mode) min(k, n) rows, including the passes
 *             of sparse heads that sit in a retrieval group.
 * s_in != 0: role row 0 is obeyed (as with LYC_STEP_S_IN). */
lyc_status lyc_step_bytes(const lyc_config* cfg, const uint8_t* role_mask, int64_t n, int k,
                          int s_in, uint64_t* analytic, uint64_t* distinct);

/* Kernel launches of the most recent step enqueued on this context: its
 * attention launches (bf16: each of two, four or eight consecutive layers, the last
 * layer alone, and the launch that merges the last layer's split rows; fp32
 * and the tcgen05 kernel: one per layer and the merge launch), selection
 * launches (one per layer with retrieval heads), and the rest (the final set
 * copy, trace fill, K/V append, S^(0) check).
 * Errors: INVALID_ARG (NULL, or no step yet). */
lyc_status lyc_step_launches(const lyc_ctx* ctx, int* attention, int* selection, int* other);

/* Test hook for the selection kernel alone: S[0..k) = argsTopK(keys[0..n), k)
 * with ties to the lower index, ascending, -1 padded.  keys and S are device
 * pointers (keys float32 [n], S int32 [k]); n <= max_ctx, k <= max_k. */
lyc_status lyc_topk_f32(lyc_ctx* ctx, const float* keys, int64_t n, int k, int32_t* S,
                        void* stream);

/* The same test hook with the selection kernel's launch form chosen:
 *   cluster  4, 8 or 16 CTAs per set (the sizes the step uses: 4 for a layer
 *            with many sets, 8 beside the next layer's attention, 16 alone), or
 *            0 for the context's default (what lyc_topk_f32 uses);
 *   variant  LYC_TOPK_FIXED: the fixed-k instantiation (every top-k step);
 *            LYC_TOPK_RULES: the instantiation that carries the size rules and
 *            block selection, run here with a fixed k.
 * Both compute the same set.  Errors: INVALID_ARG (as lyc_topk_f32, or an
 * unknown cluster size or variant), UNSUPPORTED (that cluster size does not
 * fit this context's max_ctx in shared memory). */
#define LYC_TOPK_FIXED 0
#define LYC_TOPK_RULES 1
lyc_status lyc_topk_f32_ex(lyc_ctx* ctx, const float* keys, int64_t n, int k, int32_t* S,
                           int cluster, int variant, void* stream);

/* Per-kernel device time of the steps since the last call, from CUDA events
 * recorded around every launch when timing is on (LYC_TIMING_ON).  Writes up
 * to `cap` entries of {kernel kind, layer, milliseconds}; returns the count in
 * *count.  Kinds: 0 = attention (pooled dense + sparse), 1 = top-k selection,
 * 2 = block scores (BLOCK_TOPK only). */
typedef struct {
  int kind;
  int layer;
  float ms;
} lyc_kernel_time;
#define LYC_TIMING_OFF 0
#define LYC_TIMING_ON 1
lyc_status lyc_set_timing(lyc_ctx* ctx, int mode);
lyc_status lyc_kernel_times(lyc_ctx* ctx, lyc_kernel_time* times, int cap, int* count);

/* Device timeline of the steps that follow: buf is device memory of
 * 1 + 3*cap unsigned 64-bit words; the caller zeroes word 0.  Every CTA of the
 * attention and selection kernels appends (start ns, end ns, tag) read from
 * the GPU's global timer, tag = kind << 32 | layer << 16 | CTA (kind 0 =
 * attention, with the first layer of its launch; 1 = selection); word 0 counts the records (records past cap are
 * dropped).  NULL turns it off.  Profiling use. */
lyc_status lyc_set_timeline(lyc_ctx* ctx, unsigned long long* buf, int cap);

/* ---- Allocation-free sparse attention (no counterpart in the paper).
 *
 * For callers that cannot allocate device memory: code running under a
 * framework whose caching allocator owns the device memory (a raw cudaMalloc
 * fragments that pool and can fail while the pool holds the free memory), or
 * a latency-critical serving path on which cudaMalloc / cudaFree may
 * synchronize the device.  lyc_create allocates its scratch, so these callers
 * cannot hold a context; this entry point needs none and calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 * It computes the attention of sparse heads over given sets, one layer, the
 * same arithmetic as a sparse head of lyc_decode_step, bf16 inputs: for every
 * batch element b and query head h,
 *   out[b][h] = softmax(q[b][h] K[S[b][h]]^T / sqrt(d)) V[S[b][h]]
 * over the first min(k, n) entries of the set S[b][h] (entries past n are the
 * -1 padding of k > n), with query head h reading KV head h / (Hq / Hkv).
 *   q       device, [B][Hq][d] bf16, contiguous, 4-byte aligned
 *   kv      host struct; K, V bf16 [B][Hkv][n][d] with the usual strides
 *           (s_layer ignored; strides and base pointers as for lyc_decode_step)
 *   S       device, [B][Hq][k] int32, contiguous, 16-byte aligned, k % 4 == 0;
 *           indices in [0, n) (others are skipped and reported)
 *   out     device, [B][Hq][d] float32, contiguous, 16-byte aligned; fully written
 *   status  NULL, or a device or host uint32 that receives the device status
 *           word when the work completes (0 = ok, bit 0 = an index outside [0, n))
 *   stream  cudaStream_t; the work is asynchronous on it
 * Limits: B * Hq <= LYC_NOALLOC_MAX_SETS, head_dim in {64, 128}, Hq / Hkv <= 8;
 * the launch uses at most LYC_NOALLOC_MAX_CTAS CTAs.  Larger requests return
 * LYC_ERR_SCRATCH_LIMIT and enqueue nothing.
 * Scratch: one file-scope device array of LYC_NOALLOC_SCRATCH_BYTES bytes per
 * device, shared by every call; it keeps the last call's contents.  Each call
 * enqueues a small kernel that writes its work list into the array and clears
 * the parts that must start at zero (arrival counters, status word), then the
 * attention kernels and the status copy.  Calls that overlap on the GPU
 * (different streams with no ordering between them, or host threads racing)
 * race on it.
 * Set-up: the first call on a device (with that device current) looks up the
 * array's address with cudaGetSymbolAddress and sets the kernel's attributes.
 * A host mutex serializes the calls' host side.
 * Errors: INVALID_ARG (pointers, alignment, shapes, k), UNSUPPORTED (d, group
 * size), SCRATCH_LIMIT, CUDA. */
#define LYC_NOALLOC_MAX_SETS 256
#define LYC_NOALLOC_MAX_CTAS 148
#define LYC_NOALLOC_SCRATCH_BYTES (5u << 20)
lyc_status lyc_sparse_attention_noalloc(const void* q, const lyc_kv_cache* kv, int batch,
                                        int num_q_heads, int num_kv_heads, int head_dim,
                                        const int32_t* S, int k, float* out, uint32_t* status,
                                        void* stream);

const char* lyc_status_string(lyc_status s);
const char* lyc_last_error(const lyc_ctx* ctx);
void lyc_destroy(lyc_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* LYC_H_ */
