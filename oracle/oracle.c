/*
 * oracle.c -- plain fp64 CPU oracle of the hybrid-head sparse decode-attention step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes (page: "LycheeDecode: Accelerating Long-Context LLM
 * Inference via Hybrid-Head Sparse Decoding", paper-graph-ui summary):
 *   - retrieval head, section 3.4 Eq. (1):  A = softmax(q K^T / sqrt(d_k)),  o = A V
 *   - token selection, section 3.4 Eq. (2): S^(l+1) = argsTopK(A, k)
 *   - sparse head, section 3.4 Eq. (3):     o = softmax(q K[S]^T / sqrt(d_k)) V[S]
 *   - propagation, section 3.4 (text after Eq. 3): a sparse head passes S on unchanged
 *   - layer 0, section 3.4 ("Initialization of the propagation chain") and the
 *     decode loop of Appendix B (Algorithm 1): every head of layer 0 is a
 *     retrieval head
 *   - GQA, section 3.4 "Hyperparameter summary": query heads are averaged per
 *     KV head before token selection (the KV-group selection mode below)
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - argsTopK is taken over the logits q.K/sqrt(d) rather than over A; softmax
 *     is strictly increasing so the chosen set is the same, and no exp underflow
 *     can create artificial ties;
 *   - ties go to the lower token index, -0 equals +0;
 *   - S is returned in ascending index order, padded with -1 when k > n;
 *   - query head h belongs to KV group h / (Hq / Hkv);
 *   - the current token is already in the cache (no causal mask).
 *
 * Selection rules other than a fixed k (section 4.4.1, Figure 6 and Tables
 * 5-6 name them; section 4.1 / Appendix F give the reasoning budget; the
 * kernel section gives the block size of 64), with the readings taken where
 * the pages give no formula:
 *   - the probabilities are A = softmax(x) of the selection key x (the
 *     logits, or the pooled query's logits in KV-group mode);
 *   - ratio: the set holds ceil(theta * n) rows (at least 1, at most k), the
 *     largest keys; theta = num / den exactly, so the budget is an integer
 *     computation.  The reasoning budget (50 % of the length, growing as the
 *     length grows) is the ratio 1/2 evaluated at each step's n;
 *   - top-p: the rows in key order (larger first, ties to the lower index)
 *     up to and including the first at which the running sum of A reaches p;
 *     all n if it never does; at most k;
 *   - threshold: the rows with A >= tau, at least the largest one (a set is
 *     never empty), at most k (then the k largest);
 *   - block top-k: rows grouped in blocks of `block` consecutive rows (the
 *     last one possibly shorter); a block's score is the sum of its rows' A;
 *     the floor(k / block) best blocks (ties to the lower block) are taken
 *     whole, so the set holds at most k rows;
 *   - every set is written in ascending row order, padded with -1 to k.
 *
 * Everything is fp64.  bf16 inputs are widened exactly (bits << 16), fp32
 * inputs are widened exactly.  Loops are plain; OpenMP only runs independent
 * heads side by side and changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_BF16 0
#define ORA_FP32 1
#define ORA_SELECT_PER_QHEAD 0
#define ORA_SELECT_KVGROUP_MEAN 1
#define ORA_RULE_TOPK 0
#define ORA_RULE_RATIO 1
#define ORA_RULE_BLOCK_TOPK 2
#define ORA_RULE_TOPP 3
#define ORA_RULE_THRESHOLD 4

typedef struct {
  int rule;                      /* ORA_RULE_* */
  int block;                     /* block top-k: rows per block */
  int64_t ratio_num, ratio_den;  /* ratio: theta = num / den */
  double p;                      /* top-p: the probability mass to reach */
  double tau;                    /* threshold: the smallest probability kept */
} ora_selection;

typedef struct {
  int L, B, Hq, Hkv, d;
  int64_t n;        /* tokens in the cache, current token included */
  int dtype;        /* ORA_BF16 (uint16 bit patterns) or ORA_FP32 */
  int select_mode;  /* ORA_SELECT_PER_QHEAD or ORA_SELECT_KVGROUP_MEAN */
  /* element strides of K and V: element (l, b, g, i, j) sits at
     l*s_layer + b*s_batch + g*s_head + i*s_token + j */
  int64_t s_layer, s_batch, s_head, s_token;
} ora_shape;

/* ---------------------------------------------------------------- inputs */

static double widen(const void* base, int dtype, int64_t idx) {
  if (dtype == ORA_BF16) {
    uint16_t h = ((const uint16_t*)base)[idx];
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float*)base)[idx];
}

static int slots_per_batch(const ora_shape* sh) {
  return sh->select_mode == ORA_SELECT_KVGROUP_MEAN ? sh->Hkv : sh->Hq;
}

/* ---------------------------------------------------------------- top-k */

typedef struct {
  double x;
  int64_t i;
} keyed;

/* order: larger value first; equal values (and -0 vs +0, which compare
   equal) keep the lower index first */
static int by_value_desc_index_asc(const void* pa, const void* pb) {
  const keyed* a = (const keyed*)pa;
  const keyed* b = (const keyed*)pb;
  if (a->x > b->x) return -1;
  if (a->x < b->x) return 1;
  return (a->i < b->i) ? -1 : (a->i > b->i) ? 1 : 0;
}

static int by_int_asc(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

/* argsTopK (section 3.4 Eq. 2) with the readings above: the min(k, n) indices
   with the largest x, ties to the lower index, written ascending, rest -1. */
int ora_topk(const double* x, int64_t n, int k, int32_t* S) {
  if (n <= 0 || k <= 0) return -1;
  keyed* all = (keyed*)malloc((size_t)n * sizeof(keyed));
  if (!all) return -3;
  for (int64_t i = 0; i < n; ++i) {
    all[i].x = x[i];
    all[i].i = i;
  }
  qsort(all, (size_t)n, sizeof(keyed), by_value_desc_index_asc);
  int64_t keff = (int64_t)k < n ? (int64_t)k : n;
  for (int64_t j = 0; j < keff; ++j) S[j] = (int32_t)all[j].i;
  qsort(S, (size_t)keff, sizeof(int32_t), by_int_asc);
  for (int64_t j = keff; j < k; ++j) S[j] = -1;
  free(all);
  return 0;
}

/* The m rows with the largest x (m <= n), ascending, padded with -1 to k. */
static int topk_into(const double* x, int64_t n, int64_t m, int k, int32_t* S) {
  int32_t* tmp = (int32_t*)malloc((size_t)m * sizeof(int32_t));
  if (!tmp) return -3;
  int rc = ora_topk(x, n, (int)m, tmp);
  if (rc == 0) {
    for (int64_t j = 0; j < m; ++j) S[j] = tmp[j];
    for (int64_t j = m; j < k; ++j) S[j] = -1;
  }
  free(tmp);
  return rc;
}

/* A = softmax(x): A_i = exp(x_i - max x) / sum_j exp(x_j - max x), in fp64. */
static double* softmax_of(const double* x, int64_t n) {
  double* a = (double*)malloc((size_t)n * sizeof(double));
  if (!a) return NULL;
  double m = -INFINITY, z = 0.0;
  for (int64_t i = 0; i < n; ++i)
    if (x[i] > m) m = x[i];
  for (int64_t i = 0; i < n; ++i) {
    a[i] = exp(x[i] - m);
    z += a[i];
  }
  for (int64_t i = 0; i < n; ++i) a[i] /= z;
  return a;
}

/* The set of one selection (Eq. 2 generalised by the rules above) from the
   selection keys x[0..n-1]; S has k entries.  sel == NULL: top-k. */
int ora_select(const double* x, int64_t n, int k, const ora_selection* sel, int32_t* S) {
  if (n <= 0 || k <= 0) return -1;
  const int rule = sel ? sel->rule : ORA_RULE_TOPK;
  if (rule == ORA_RULE_TOPK) return ora_topk(x, n, k, S);
  const int64_t cap = (int64_t)k < n ? (int64_t)k : n;
  if (rule == ORA_RULE_RATIO) {
    if (sel->ratio_num < 0 || sel->ratio_den <= 0) return -1;
    int64_t m = (sel->ratio_num * n + sel->ratio_den - 1) / sel->ratio_den;  /* ceil */
    if (m < 1) m = 1;
    if (m > cap) m = cap;
    return topk_into(x, n, m, k, S);
  }
  if (rule == ORA_RULE_TOPP || rule == ORA_RULE_THRESHOLD) {
    double* a = softmax_of(x, n);
    if (!a) return -3;
    int64_t m = 0;
    if (rule == ORA_RULE_THRESHOLD) {
      for (int64_t i = 0; i < n; ++i) m += a[i] >= sel->tau;
      if (m < 1) m = 1;
    } else {
      keyed* all = (keyed*)malloc((size_t)n * sizeof(keyed));
      if (!all) {
        free(a);
        return -3;
      }
      for (int64_t i = 0; i < n; ++i) {
        all[i].x = x[i];
        all[i].i = i;
      }
      qsort(all, (size_t)n, sizeof(keyed), by_value_desc_index_asc);
      double cum = 0.0;
      m = n;
      for (int64_t j = 0; j < n; ++j) {
        cum += a[all[j].i];
        if (cum >= sel->p) {
          m = j + 1;
          break;
        }
      }
      free(all);
    }
    free(a);
    if (m > cap) m = cap;
    return topk_into(x, n, m, k, S);
  }
  if (rule == ORA_RULE_BLOCK_TOPK) {
    const int bs = sel->block;
    if (bs <= 0 || k < bs) return -1;
    const int64_t nb = (n + bs - 1) / bs;
    int64_t kb = k / bs;
    if (kb > nb) kb = nb;
    double* a = softmax_of(x, n);
    double* score = (double*)calloc((size_t)nb, sizeof(double));
    int32_t* blocks = (int32_t*)malloc((size_t)kb * sizeof(int32_t));
    if (!a || !score || !blocks) {
      free(a);
      free(score);
      free(blocks);
      return -3;
    }
    for (int64_t i = 0; i < n; ++i) score[i / bs] += a[i];
    int rc = ora_topk(score, nb, (int)kb, blocks);
    if (rc == 0) {
      int64_t pos = 0;
      for (int64_t j = 0; j < kb; ++j)
        for (int64_t i = (int64_t)blocks[j] * bs; i < ((int64_t)blocks[j] + 1) * bs && i < n; ++i)
          S[pos++] = (int32_t)i;
      for (; pos < k; ++pos) S[pos] = -1;
    }
    free(a);
    free(score);
    free(blocks);
    return rc;
  }
  return -1;
}

/* ---------------------------------------------------------------- attention */

/* Scaled dot-product attention of one query over a list of cache rows
   (rows == NULL: all n rows in order).  Eq. (1) when the list is every row,
   Eq. (3) when it is S.  Writes o[d]; if logits != NULL also writes the
   scaled logit of each listed row, in list order. */
static void attend_rows(const ora_shape* sh, const double* q, const void* K,
                        const void* V, int64_t kv_base, const int32_t* rows,
                        int64_t count, double* o, double* logits) {
  const int d = sh->d;
  const double scale = 1.0 / sqrt((double)d);
  double* s = (double*)malloc((size_t)(count > 0 ? count : 1) * sizeof(double));
  double m = -INFINITY;
  for (int64_t r = 0; r < count; ++r) {
    int64_t i = rows ? (int64_t)rows[r] : r;
    int64_t off = kv_base + i * sh->s_token;
    double dot = 0.0;
    for (int j = 0; j < d; ++j) dot += q[j] * widen(K, sh->dtype, off + j);
    s[r] = dot * scale;
    if (s[r] > m) m = s[r];
  }
  double z = 0.0;
  for (int j = 0; j < d; ++j) o[j] = 0.0;
  for (int64_t r = 0; r < count; ++r) {
    int64_t i = rows ? (int64_t)rows[r] : r;
    int64_t off = kv_base + i * sh->s_token;
    double p = exp(s[r] - m);
    z += p;
    for (int j = 0; j < d; ++j) o[j] += p * widen(V, sh->dtype, off + j);
  }
  for (int j = 0; j < d; ++j) o[j] /= z;
  if (logits)
    for (int64_t r = 0; r < count; ++r) logits[r] = s[r];
  free(s);
}

/* ---------------------------------------------------------------- one layer */

/*
 * One layer of the step for every batch element and query head.
 *   q_all   : [L][B][Hq][d] (dtype)            K, V : see ora_shape strides
 *   role_row: [Hq] for this layer, 1 = retrieval
 *   all_retrieval: 1 forces every head to retrieval (layer 0 of a step)
 *   S_in    : [B][Hs][k] the sets this layer inherits (may be NULL only when
 *             every head is retrieval)
 *   S_out   : [B][Hs][k] the sets passed to layer l+1
 *   out_l   : [B][Hq][d] fp64
 *   keys    : [B][Hs][n] fp64 or NULL; the selection key of each refreshed slot
 *   refreshed: [Hs] or NULL; 1 where the slot was re-selected at this layer
 * Returns 0, or a negative code on a bad argument or a bad inherited index.
 */
int ora_layer_sel(const ora_shape* sh, const ora_selection* sel, int l, const void* q_all,
                  const void* K, const void* V, const uint8_t* role_row, int all_retrieval,
                  int k, const int32_t* S_in, int32_t* S_out, double* out_l, double* keys,
                  uint8_t* refreshed) {
  const int B = sh->B, Hq = sh->Hq, Hkv = sh->Hkv, d = sh->d;
  const int64_t n = sh->n;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || n <= 0 || k <= 0) return -1;
  if (Hq % Hkv != 0) return -1;
  const int G = Hq / Hkv;
  const int Hs = slots_per_batch(sh);
  const int kv_mode = sh->select_mode == ORA_SELECT_KVGROUP_MEAN;
  if (sel && sel->rule == ORA_RULE_BLOCK_TOPK && (sel->block <= 0 || k < sel->block)) return -1;
  if (sel && sel->rule == ORA_RULE_RATIO && (sel->ratio_num < 0 || sel->ratio_den <= 0)) return -1;
  if (sel && (sel->rule < ORA_RULE_TOPK || sel->rule > ORA_RULE_THRESHOLD)) return -1;

  /* which heads are retrieval, which slots are refreshed */
  int* is_ret = (int*)calloc((size_t)Hq, sizeof(int));
  int* fresh = (int*)calloc((size_t)Hs, sizeof(int));
  for (int h = 0; h < Hq; ++h) {
    is_ret[h] = all_retrieval || role_row[h] != 0;
    if (is_ret[h]) fresh[kv_mode ? h / G : h] = 1;
  }
  int need_S = 0;
  for (int h = 0; h < Hq; ++h) need_S |= !is_ret[h];
  if (need_S && !S_in) {
    free(is_ret);
    free(fresh);
    return -1;
  }
  /* inherited indices must be valid rows */
  if (need_S) {
    for (int64_t t = 0; t < (int64_t)B * Hs * k; ++t)
      if (S_in[t] >= n || S_in[t] < -1) {
        free(is_ret);
        free(fresh);
        return -5;
      }
  }

  /* selection keys of the refreshed slots, [B][Hs][n] */
  double* xk = (double*)malloc((size_t)B * Hs * n * sizeof(double));
  if (!xk) {
    free(is_ret);
    free(fresh);
    return -3;
  }

  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      const int g = h / G;
      const int64_t kv_base = (int64_t)l * sh->s_layer + (int64_t)b * sh->s_batch +
                              (int64_t)g * sh->s_head;
      double* q = (double*)malloc((size_t)d * sizeof(double));
      const int64_t q_off = (((int64_t)l * B + b) * Hq + h) * d;
      for (int j = 0; j < d; ++j) q[j] = widen(q_all, sh->dtype, q_off + j);
      double* o = out_l + ((int64_t)b * Hq + h) * d;
      if (is_ret[h]) {
        /* Eq. (1) over every row; in per-head mode its logits are the key */
        double* key = kv_mode ? NULL : xk + ((int64_t)b * Hs + h) * n;
        attend_rows(sh, q, K, V, kv_base, NULL, n, o, key);
      } else {
        /* Eq. (3) over the inherited rows (valid prefix of the slot) */
        const int slot = kv_mode ? g : h;
        const int32_t* S = S_in + ((int64_t)b * Hs + slot) * k;
        int64_t count = 0;
        while (count < k && S[count] >= 0) ++count;
        if (count == 0) {
          bad |= 1;
        } else {
          attend_rows(sh, q, K, V, kv_base, S, count, o, NULL);
        }
      }
      free(q);
    }
  }
  if (bad) {
    free(xk);
    free(is_ret);
    free(fresh);
    return -5;
  }

  /* selection keys and Eq. (2) for every refreshed slot */
  const double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    for (int s = 0; s < Hs; ++s) {
      int32_t* Sout = S_out + ((int64_t)b * Hs + s) * k;
      if (!fresh[s]) {
        /* propagation: the inherited set passes on unchanged */
        const int32_t* Sin = S_in + ((int64_t)b * Hs + s) * k;
        memcpy(Sout, Sin, (size_t)k * sizeof(int32_t));
        continue;
      }
      double* x = xk + ((int64_t)b * Hs + s) * n;
      if (kv_mode) {
        /* key = (mean of the group's G queries) . K_i / sqrt(d) */
        const int g = s;
        const int64_t kv_base = (int64_t)l * sh->s_layer + (int64_t)b * sh->s_batch +
                                (int64_t)g * sh->s_head;
        double* qbar = (double*)calloc((size_t)d, sizeof(double));
        for (int t = 0; t < G; ++t) {
          const int64_t q_off = (((int64_t)l * B + b) * Hq + (g * G + t)) * d;
          for (int j = 0; j < d; ++j) qbar[j] += widen(q_all, sh->dtype, q_off + j);
        }
        for (int j = 0; j < d; ++j) qbar[j] /= (double)G;
        for (int64_t i = 0; i < n; ++i) {
          double dot = 0.0;
          for (int j = 0; j < d; ++j)
            dot += qbar[j] * widen(K, sh->dtype, kv_base + i * sh->s_token + j);
          x[i] = dot * scale;
        }
        free(qbar);
      }
      /* per-head mode: x already holds the retrieval head's own logits */
      ora_select(x, n, k, sel, Sout);
      if (keys) memcpy(keys + ((int64_t)b * Hs + s) * n, x, (size_t)n * sizeof(double));
    }
  }
  free(xk);
  if (refreshed)
    for (int s = 0; s < Hs; ++s) refreshed[s] = (uint8_t)fresh[s];
  free(is_ret);
  free(fresh);
  return 0;
}

int ora_layer(const ora_shape* sh, int l, const void* q_all, const void* K,
              const void* V, const uint8_t* role_row, int all_retrieval, int k,
              const int32_t* S_in, int32_t* S_out, double* out_l, double* keys,
              uint8_t* refreshed) {
  return ora_layer_sel(sh, NULL, l, q_all, K, V, role_row, all_retrieval, k, S_in, S_out,
                       out_l, keys, refreshed);
}

/* ---------------------------------------------------------------- one step */

/*
 * The whole L-layer step (Algorithm 1's head loop, attention part only).
 *   s_in = 0: layer 0 is all retrieval and S is output only.
 *   s_in = 1: S holds S^(0) on entry and role row 0 is obeyed.
 *   S     : [B][Hs][k]; holds S^(L) on return.
 *   out   : [L][B][Hq][d] fp64.
 *   trace : [L][B][Hs][k] or NULL; trace[l] = the sets after layer l.
 */
int ora_decode_step_sel(const ora_shape* sh, const ora_selection* sel, const void* q,
                        const void* K, const void* V, const uint8_t* role, int k, int s_in,
                        int32_t* S, double* out, int32_t* trace) {
  const int64_t per = (int64_t)sh->B * slots_per_batch(sh) * k;
  int32_t* cur = (int32_t*)malloc((size_t)per * sizeof(int32_t));
  int32_t* nxt = (int32_t*)malloc((size_t)per * sizeof(int32_t));
  if (s_in) {
    memcpy(cur, S, (size_t)per * sizeof(int32_t));
  } else {
    for (int64_t t = 0; t < per; ++t) cur[t] = -1;
  }
  int rc = 0;
  for (int l = 0; l < sh->L && rc == 0; ++l) {
    const int all_ret = (l == 0) && !s_in;
    rc = ora_layer_sel(sh, sel, l, q, K, V, role + (int64_t)l * sh->Hq, all_ret, k,
                       (l == 0 && !s_in) ? NULL : cur, nxt,
                       out + (int64_t)l * sh->B * sh->Hq * sh->d, NULL, NULL);
    if (trace) memcpy(trace + (int64_t)l * per, nxt, (size_t)per * sizeof(int32_t));
    int32_t* t = cur;
    cur = nxt;
    nxt = t;
  }
  if (rc == 0) memcpy(S, cur, (size_t)per * sizeof(int32_t));
  free(cur);
  free(nxt);
  return rc;
}

int ora_decode_step(const ora_shape* sh, const void* q, const void* K,
                    const void* V, const uint8_t* role, int k, int s_in,
                    int32_t* S, double* out, int32_t* trace) {
  return ora_decode_step_sel(sh, NULL, q, K, V, role, k, s_in, S, out, trace);
}

/* ---------------------------------------------------------------- cache correction */

/*
 * Cache Correction (section 4.2.2; the decoding setup of section 4.1 and
 * Appendix F): after every 32 decoded tokens the T most recent positions are
 * prefilled again with dense attention.  The attention part of that prefill,
 * for every layer, batch element and query head: query t sits at position
 * p = n - T + t and attends rows 0..p of the cache (causal), whose rows
 * n - T .. n - 1 already hold the refreshed K/V of those positions.
 *   q   : [L][B][Hq][T][d] (dtype)
 *   out : [L][B][Hq][T][d] fp64
 * Returns 0, or -1 on a bad argument.
 */
int ora_correction(const ora_shape* sh, int T, const void* q_all, const void* K, const void* V,
                   double* out) {
  const int L = sh->L, B = sh->B, Hq = sh->Hq, Hkv = sh->Hkv, d = sh->d;
  const int64_t n = sh->n;
  if (L <= 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || T <= 0 || T > n)
    return -1;
  const int G = Hq / Hkv;
#pragma omp parallel for collapse(3) schedule(dynamic)
  for (int l = 0; l < L; ++l) {
    for (int b = 0; b < B; ++b) {
      for (int h = 0; h < Hq; ++h) {
        const int g = h / G;
        const int64_t kv_base = (int64_t)l * sh->s_layer + (int64_t)b * sh->s_batch +
                                (int64_t)g * sh->s_head;
        double* qv = (double*)malloc((size_t)d * sizeof(double));
        for (int t = 0; t < T; ++t) {
          const int64_t row = (((int64_t)l * B + b) * Hq + h) * T + t;
          for (int j = 0; j < d; ++j) qv[j] = widen(q_all, sh->dtype, row * d + j);
          const int64_t p = n - T + t;
          attend_rows(sh, qv, K, V, kv_base, NULL, p + 1, out + row * d, NULL);
        }
        free(qv);
      }
    }
  }
  return 0;
}
