// lyc_plan.h -- work-list records shared by the host planner and the kernels.
//
// One layer of the step is a pool of segments (page "LycheeDecode ...",
// paper-graph-ui summary, Appendix C / Algorithm 2, "workload pooling"):
//   dense segment  : one (batch b, KV group g); rows 0..n-1 of the group's
//                    K/V; query rows = the group's retrieval heads (per-head
//                    selection: each row's logits are its selection key), or
//                    all of the group's heads (KV-group selection: the mean of
//                    the rows' logits is the group's key, since averaging the
//                    queries and averaging their logits give the same number;
//                    only the retrieval rows produce outputs);
//   sparse segment : one inherited set; rows = the set's list positions
//                    0..k_eff-1; query rows = the sparse heads that read that
//                    set (one head per set in per-head mode, every sparse head
//                    of the group in KV-group mode).
// The pooled rows are cut into equal runs of 64-row tiles, one run per CTA.
// A run that crosses segment boundaries becomes several pieces.  Each piece
// writes one partial softmax state (m, l, o[d]) per output row; the last piece
// of a segment to finish merges them (log-sum-exp) into `out`.
#pragma once
#include <cuda.h>
#include <stdint.h>
#include <string.h>

namespace lyc {

constexpr int kTileRows = 64;      // rows per pipeline stage (the pages' block size)
constexpr int kKeyBins = 2048;     // top 11 bits of an order-preserving key encoding
constexpr int kKeyDigitShift = 21;
constexpr int kMaxGroup = 8;       // largest Hq / Hkv supported
constexpr int kMaxQ = kMaxGroup;   // query rows per segment
constexpr int kMaxConsumerWarps = 8;
// pieces a CTA's consumer warps may run ahead of its epilogue warp: the ring
// of per-warp partial states between them has this many slots
constexpr int kPartSlots = 4;
// Pool of gathered rows that CTAs take at run time, kPoolTiles tiles at a
// time; a CTA's leader publishes the pool pieces it took into a ring of
// kPoolRing entries that every warp of the CTA reads in order.
constexpr int kPoolTiles = 8;
// Units of the sets that the selection just before a pass's layer writes
// (passes deferred to the end of a later pool, or the last layer's own:
// the only gathered rows that may wait for a selection; taken last).  Smaller units would
// spread them over more CTAs once that selection is done, but every unit is a
// piece with its own partial state (measured on B200, 128K Llama3-8B stack,
// against 8-tile units for both: KV-group sets, 4-tile units -1.2 %, 2-tile
// -3 %, 1-tile -6 %; per head, 4-tile -1.3 %).
constexpr int kPoolTilesDep = 8;
constexpr int kPoolRing = 16;

enum SegKind : int32_t { kDense = 0, kSparse = 1 };

struct Segment {
  const void* k;        // K rows of (l, b, g): row i at k + i * s_token elements
  const void* v;        // V rows, same layout
  const int32_t* idx;   // sparse: the inherited set (list positions -> token index)
  int64_t s_token;      // element stride between rows
  int64_t key_off[kMaxQ];  // per query row: element offset of its selection-key
                           // row in the key buffer, or -1
  int64_t key_mean_off;    // offset of the key row that receives the mean of all
                           // nq rows' logits (KV-group selection), or -1
  int32_t kind;         // SegKind
  int32_t l, b, g;
  int32_t rows;         // dense: n; sparse: k_eff (valid list entries)
  int32_t nq;           // query rows in use
  int32_t nout;         // rows that produce an output
  int32_t head[kMaxQ];  // query head of each row
  int32_t out_row[kMaxQ];  // output o comes from row out_row[o]
  int32_t part_base;    // first partial record of this segment
  int32_t npieces;      // pieces the segment was cut into
  int32_t cnt_base;     // first arrival counter of this segment
  int32_t row_base;     // row of (l, b, g, token 0) in the flattened row-gather map
  int32_t dep;          // sparse: the set is the previous launch's output (wait for it)
  int32_t pad_ok;       // sparse: -1 entries are padding of a shorter set (masked, not errors)
  const uint32_t* ready;  // sparse: flag word of the selection that wrote the set in
                          // this step (it holds the step's epoch + 1 once the set is
                          // complete), or NULL when the set comes from the caller
  int32_t nvalid;         // rows of (l, b): inherited indices must lie in [0, nvalid)
  int32_t page_rows;      // paged cache: rows per page; 0: contiguous rows
  const int32_t* bt;      // paged cache: the block-table row of b (row i is in page bt[i / page_rows],
                          // at k + page * s_page + (i % page_rows) * s_token); NULL: contiguous
  int64_t s_page;         // paged cache: element stride between pages
  // the segment's layer: its queries [B][Hq][d] and outputs [B][Hq][d] (a
  // launch of the mma kernel holds segments of several layers: its own
  // layers', and sparse passes deferred to it from earlier layers); NULL:
  // the launch's q and out
  const void* q;
  float* out;
};

struct Piece {
  int32_t seg;      // segment index within the launch
  int32_t r0, r1;   // row range within the segment (token or list positions)
  int32_t ordinal;  // which piece of its segment (partials at part_base + ordinal*nout + o)
};

struct AttnParams {
  const Segment* segs;
  const Piece* pieces;
  const int32_t* cta_begin;  // pieces of CTA c: [cta_begin[c], cta_begin[c+1])
  const void* q;             // the launch's first layer's queries, [B][Hq][d] (segments carry their own)
  float* out;                // the launch's first layer's outputs, [B][Hq][d] (likewise)
  float* keys;               // selection-key buffer
  float* part_o;             // [parts][d]
  float2* part_ml;           // [parts] (running max in log2 units, sum)
  int32_t* counters;         // arrival counters, left at zero after use
  float* wpart_o;            // per CTA: [kPartSlots][consumer warp][kMaxQ][d] piece states
  float2* wpart_ml;          // per CTA: [kPartSlots][consumer warp][kMaxQ] (max, sum)
  // bf16 path: the cross-piece combine of a launch runs in the next launch
  // (taken by that launch's epilogue warps)
  const Segment* prev_segs;  // the previous attention launch's segments
  const int2* prev_tasks;    // (segment, output) pairs of segments cut into > 1 piece
  int32_t prev_ntasks;
  const float* prev_part_o;  // the previous launch's piece partials
  const float2* prev_part_ml;
  float* prev_out;           // outputs of the previous launch's first layer (segments carry their own)
  int32_t wait_prev;         // 1: wait for the previous launch to complete before any
                             // work (it is not a selection launch, which would have)
  uint32_t* status;          // device status word
  unsigned long long* timeline;  // NULL, or [1 + 3*cap]: count, then (start ns, end ns, tag)
  const uint32_t* epoch;     // this step's epoch (the `ready` flags hold epoch + 1), or NULL
  // Step counters (zeroed for the next step by the step's last launch): the
  // counter of this step is at ptr + (epoch & 1) * pool_stride.
  uint32_t* done;            // NULL, or this launch's completion counter: every CTA adds 1
                             // once its work is done (release)
  const uint32_t* prev_done; // NULL, or the previous attention launch's completion
                             // counter: the epilogue waits until it reaches prev_done_expect
                             // (else on griddepcontrol.wait)
  uint32_t prev_done_expect; // CTAs of that launch
  // the pool (mma kernel): after its own pieces a CTA takes units u = 0, 1, ...
  // by an atomic cursor; unit u is the piece pool_units[u] (a row range of a
  // gathered segment, its ordinal = its partial record)
  const Piece* pool_units;
  int32_t pool_n;            // units in the pool (0: none)
  int32_t pool_stride;       // step counters per epoch parity (pool cursors, completion and
                             // key counters)
  int32_t* pool_cursors;     // [2][pool_stride]: this launch's cursor is [(epoch & 1)][layer]
  int32_t wpart_by_sm;       // 1: the piece-state ring of a CTA is the one of the SM it runs
                             // on (CTAs of consecutive launches may overlap in time); 0: of
                             // its block index
  int32_t wpart_slots;       // rings allocated
  int32_t wpart_q;           // query rows per consumer-warp record of the ring (0: kMaxQ); a
                             // caller whose segments all have one query row passes 1
  int32_t timeline_cap;
  uint32_t* keys_done;       // NULL, or the step counter of the selection keys of the launch's
                             // first layer; the counters of its later layers follow it.  Each
                             // consumer warp of a CTA with own (dense) pieces of a layer adds 1
                             // to that layer's counter once it is past them (release)
  int32_t keys_ctas;         // CTAs with own pieces of the first layer
  int32_t layer;             // the launch's first layer
  int32_t Hq, G, n;
  int32_t paged;             // 1: the segments' rows are in pages (Segment::bt)
  int32_t gather_rows;       // rows of the flattened row-gather maps (an index past
                             // the last row, used for rows that must read as zeros);
                             // 0: no such maps, gathered rows come by cp.async
  float scale_log2;          // log2(e) / sqrt(d)
  float scale;               // 1 / sqrt(d)
};

// The first piece of a CTA (mma kernel), carried in the launch parameters:
// the CTA issues its first tile copies, and starts reading its first
// segment, without first reading its piece list from global memory (three
// dependent reads, about 2 us of every CTA's start).  Only a dense piece of
// a contiguous cache is carried.
constexpr int kFirstPieces = 148;
struct FirstPiece {
  Piece pc;        // seg < 0: none (the CTA reads its pieces from the list)
  int16_t g, b;    // the piece's KV group and batch element (of the launch's layer)
};

// The launch parameters of the bf16 attention kernels (mma.sync and
// tcgen05): the tensor maps of the cache, then the work list.
struct AttnMmaParams {
  CUtensorMap tmk;  // 5-D map of K: (d, row, g, b, l), 128B swizzle; box 64 x the kernel's tile rows
  CUtensorMap tmv;  // same for V
  CUtensorMap tgk;  // 2-D map of K: (d, flattened row), box 64 x 1, 128B swizzle (row gathers)
  CUtensorMap tgv;  // same for V
  AttnParams p;
  int32_t nfirst;   // CTAs 0 .. nfirst-1 have an entry in `first` (0: none)
  FirstPiece first[kFirstPieces];
};
static_assert(sizeof(AttnMmaParams) <= 4096, "kernel parameters are at most 4 KiB");

struct TopkTask {
  const float* keys;  // n selection keys
  int32_t* S;         // the launch's k outputs
  int32_t* trace;     // NULL, or a second destination that receives the same k entries
                      // (the set trace: written by the selection itself, so that tracing
                      // adds no launch between the layers)
  uint32_t* done;     // NULL, or {arrival counter, ready flag}: the last CTA of the task
                      // to finish resets the counter and sets the flag to epoch + 1
  int32_t n;          // keys of this task (a batch element's rows; its blocks with expand > 1);
                      // 0: the launch's n
  int32_t k;          // at most this many keys are selected; 0: the launch's k
  int32_t rows;       // with expand > 1: the element's rows (the key row's length)
  int32_t pad_;
};

// How many keys a task selects (at most its k, at most n):
//  kSizeFixed     : k;
//  kSizeTopP      : the fewest largest keys whose probabilities softmax(keys)
//                   sum to at least size_x;
//  kSizeThreshold : the keys whose probability is at least size_x (at least one).
// The last two take their decision on 40-bit fixed-point weights
// round(2^40 exp(key - max)): integer sums are exact and independent of the
// order of the additions, so every CTA of a cluster reaches the same size.
enum TopkSizeRule : int32_t { kSizeFixed = 0, kSizeTopP = 1, kSizeThreshold = 2 };

struct TopkParams {
  const TopkTask* tasks;  // one per blockIdx.y; NULL: use `single`
  TopkTask single;
  const uint32_t* epoch;  // this step's epoch (for the ready flags), or NULL
  int32_t early;          // 1: let the next launch start before this one has read its keys
                          // (its readers wait on the ready flags); 0: only after
  unsigned long long* timeline;  // as in AttnParams
  const uint32_t* keys_ready;  // NULL: start on griddepcontrol.wait (the attention launch
                               // before has completed); else once this step counter (the
                               // layer's key counter, see AttnParams::keys_done) reaches
                               // keys_expect
  const uint32_t* prev_done;   // with keys_ready: the completion counter of the attention
                               // launch before the one of this layer (the last readers of the
                               // set buffers this launch writes) to wait for, up to
                               // prev_done_expect; or NULL
  uint32_t keys_expect, prev_done_expect;
  int32_t cnt_stride;          // step counters per epoch parity
  uint32_t* status;            // device status word (wait timeouts)
  int32_t timeline_cap;
  int32_t layer;
  int32_t n, k;           // k: entries of each output set
  int32_t size_rule;      // TopkSizeRule
  int32_t expand;         // > 1: block selection: the task's keys are rows, key j of the selection
                          // is the block of rows j*expand .. j*expand + expand - 1 (scored
                          // log(sum exp(key))), and the output lists the selected blocks' rows
  double size_x;          // p (top-p) or tau (threshold)
};

// Cache Correction (correction_kernel.cu): a piece is tiles [t0, t1) (128
// rows each) of KV group (l, b, g); its partial states go to record `part`.
struct CorrPiece {
  int32_t l, b, g;
  int32_t t0, t1;
  int32_t part;
};

struct CorrParams {
  CUtensorMap tmk;            // 5-D maps of K and V: (d, row, g, b, l), box 64 x 128 rows
  CUtensorMap tmv;
  const void* q;              // [L][B][Hq][T][d] bf16
  float* out;                 // [L][B][Hq][T][d]
  const CorrPiece* pieces;
  const int32_t* cta_begin;   // pieces of CTA c: [cta_begin[c], cta_begin[c+1])
  float* part_o;              // [2 * pieces][128 rows][d], unnormalised: record 2p + h is
                              // key half h (keys 64h .. 64h+63 of every tile) of piece p
  float2* part_ml;            // [2 * pieces][128 rows]: (running max in log2 units, sum)
  const int32_t* group_first; // combine: pieces of group j are [group_first[j], group_first[j+1])
  uint32_t* status;
  int32_t L, B, Hq, Hkv, G, T, n;
  int32_t rows;               // G * T query rows per group
  float scale_log2;           // log2(e) / sqrt(d)
};

// write_rows_kernel (Cache Correction's refreshed rows): k_new/v_new
// [L][B][Hkv][T][d] written at rows n - T .. n - 1 of every (l, b, g)
struct WriteRowsParams {
  const unsigned char* k_new;
  const unsigned char* v_new;
  unsigned char* k;
  unsigned char* v;
  int64_t s_layer, s_batch, s_head, s_token;
  int32_t L, B, Hkv, T, n, row_bytes, elem_bytes;
};

// Timeline tags: kind << 32 | layer << 16 | CTA
constexpr unsigned long long kTagAttention = 0ull;
constexpr unsigned long long kTagTopk = 1ull;

// copy_sets_kernel: dst[(b*Hs + s)*k + j] = src[b*Hs + s][j] for j < k, or
// with a destination list, dsts[i][j] = src[i][j]
struct CopySetsParams {
  const int32_t* const* src;
  int32_t* dst;
  int32_t nsets, k;
  uint32_t* epoch;  // the step's last launch: advance the epoch once the copy is done (or NULL)
  int32_t* pool_cursors;  // with epoch: zero the next step's pool cursors, [2][pool_stride]
  int32_t pool_stride;
  int32_t* const* dsts;  // NULL, or one destination per set (dst is then unused)
};

// append_rows_kernel: the current token's K and V ([L][B][Hkv][row_bytes]
// each, contiguous) written at row n[b]-1 of every (l, b, g) of the cache:
// element offset l*s_layer + g*s_head + b*s_batch + i*s_token (contiguous), or
// l*s_layer + g*s_head + bt[b*max_blocks + i/page_rows]*s_page +
// (i % page_rows)*s_token (paged), i = n[b] - 1; times elem_bytes
struct AppendParams {
  const unsigned char* k_new;
  const unsigned char* v_new;
  unsigned char* k;
  unsigned char* v;
  const int64_t* n;  // device, [B]
  int64_t s_layer, s_batch, s_head, s_token, s_page;
  const int32_t* bt;
  int32_t page_rows, max_blocks;
  int32_t L, B, Hkv, row_bytes, elem_bytes;
};

// validate_sets_kernel: each of nsets sets (stride `stride`) must hold
// between min_valid and k_eff ascending indices in [0, n), followed by -1 up to k
struct ValidateSetsParams {
  const int32_t* sets;
  uint32_t* status;
  int32_t nsets, stride, k, k_eff, n;
  int32_t min_valid;
};

// Order-preserving map of an fp32 selection key to an unsigned integer
// (larger key -> larger integer; -0 and +0 map to the same value).
__host__ __device__ inline uint32_t order_key(float f) {
  uint32_t b;
  memcpy(&b, &f, sizeof b);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// status word bits
constexpr uint32_t kStatusBadIndex = 1u;
constexpr uint32_t kStatusTimeout = 2u;
constexpr uint32_t kStatusEmptySoftmax = 4u;
constexpr uint32_t kStatusScratch = 8u;  // an SM index beyond the per-SM scratch

}  // namespace lyc
