/*
 * hs2_oracle.c -- plain fp64 CPU oracle for HySparse2's KV-Reuse hybrid block.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls this file: only
 * the tests, the graft smoke check and the benchmark's CPU-baseline leg do. It shares no code,
 * header or table with the CUDA library.
 *
 * What it computes, step by step, in the order the method states it:
 *  - "HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs" (originshq.com),
 *    section "KV Reuse and Token-Level Sparse Selection": inside a hybrid block the
 *    full-attention layer attends over the whole (causal) context and produces both the KV cache
 *    and per-token selection indices; the sparse layers that follow reuse those indices and the
 *    same KV cache. Selection is per token: 1,024 tokens over the full context plus a forced
 *    window of the 128 most recent tokens, read from the full layer's cache.
 *  - "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing" (academy.dair.ai), bullets
 *    "KV Reuse refinements" (token-level, 1,024 global + 128 forced recent) and "Inference cost"
 *    (MQA: one K/V head shared by all query heads; FP8 KV cache).
 * The pages leave the importance score open. It is read here as the head-summed softmax
 * probability s[t] = sum_h exp(l_h[t] - lse_h), l_h[t] = c * q_h . k_t, c = 1/sqrt(d), taken in a
 * second pass from the full layer's log-sum-exp. Ties go to the lower index; the window is not a
 * candidate set (top-k is over [0, p-w+1) only); the union is returned in ascending order.
 *
 * Arithmetic: every input is widened exactly to double (bf16 -> double is exact; e4m3 codes are
 * decoded through a table built from the OCP e4m3fn definition and multiplied by the fp32
 * per-token scale, which is exact in double). All sums run in double, in index order.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared hs2_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t batch, n_q, n_heads, head_dim;
  int32_t kv_dtype;          /* 0: bf16 bit patterns, 1: e4m3fn codes with fp32 per-row scale */
  const void *k, *v;         /* [rows, head_dim] */
  const float *k_scale, *v_scale;
  const int64_t *kv_start;   /* [batch] first row of sequence b */
  const int32_t *kv_len;     /* [batch] tokens of sequence b */
} hs2o_kv;

/* ---------------------------------------------------------------- formats */

static double bf16_to_double(uint16_t u) {
  uint32_t w = (uint32_t)u << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* OCP FP8 e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 encodes
 * subnormals m * 2^-9; S.1111.111 is NaN; there is no infinity. */
void hs2o_e4m3_table(double out[256]) {
  for (int c = 0; c < 256; ++c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
      v = NAN;
    else if (e == 0)
      v = ldexp((double)m, -9);
    else
      v = ldexp(1.0 + m / 8.0, e - 7);
    out[c] = s ? -v : v;
  }
}

static double g_e4m3[256];
static int g_e4m3_ready = 0;

static void widen_row(const hs2o_kv *kv, const void *base, const float *scale, int64_t row,
                      double *out) {
  int d = kv->head_dim;
  if (kv->kv_dtype == 0) {
    const uint16_t *p = (const uint16_t *)base + row * d;
    for (int j = 0; j < d; ++j) out[j] = bf16_to_double(p[j]);
  } else {
    const uint8_t *p = (const uint8_t *)base + row * d;
    double sc = (double)scale[row];
    for (int j = 0; j < d; ++j) out[j] = sc * g_e4m3[p[j]];
  }
}

static void ensure_tables(void) {
  if (!g_e4m3_ready) {
    hs2o_e4m3_table(g_e4m3);
    g_e4m3_ready = 1;
  }
}

/* ---------------------------------------------------------------- full attention + scores */

/* For each listed flat row r = b * n_q + i (query at cache position p = T_b - n_q + i):
 *   l_h[t] = c * q_h . k_t for t in [0, p]            (causal prefix, one shared K/V head)
 *   lse_h  = m_h + log sum_t exp(l_h[t] - m_h),  m_h = max_t l_h[t]
 *   O_h    = sum_t exp(l_h[t] - lse_h) v_t
 *   s[t]   = sum_h exp(l_h[t] - lse_h)                (importance score, heads in order)
 * q: bf16 bits [batch, n_q, H, d]. out: [n_rows, H, d], lse: [n_rows, H],
 * scores (optional): [n_rows, score_stride], entries t > p left untouched.
 * Returns 0, or -1 on a bad row / allocation failure. */
int hs2o_full_attn(const hs2o_kv *kv, const uint16_t *q, double c, const int64_t *rows,
                   int64_t n_rows, double *out, double *lse, double *scores,
                   int64_t score_stride) {
  ensure_tables();
  const int H = kv->n_heads, d = kv->head_dim;
  for (int64_t rr = 0; rr < n_rows; ++rr) {
    int64_t r = rows[rr];
    if (r < 0 || r >= (int64_t)kv->batch * kv->n_q) return -1;
    int64_t b = r / kv->n_q, i = r % kv->n_q;
    int64_t T = kv->kv_len[b], p = T - kv->n_q + i, n = p + 1, base = kv->kv_start[b];
    if (p < 0) return -1;
    double *qd = (double *)malloc(sizeof(double) * H * d);
    double *l = (double *)malloc(sizeof(double) * H * n);
    double *ls = (double *)malloc(sizeof(double) * H);
    if (!qd || !l || !ls) { free(qd); free(l); free(ls); return -1; }
    for (int h = 0; h < H; ++h)
      for (int j = 0; j < d; ++j) qd[h * d + j] = bf16_to_double(q[((r * H) + h) * d + j]);

    /* logits */
#pragma omp parallel
    {
      double *kt = (double *)malloc(sizeof(double) * d);
#pragma omp for schedule(static)
      for (int64_t t = 0; t < n; ++t) {
        widen_row(kv, kv->k, kv->k_scale, base + t, kt);
        for (int h = 0; h < H; ++h) {
          double acc = 0.0;
          for (int j = 0; j < d; ++j) acc += qd[h * d + j] * kt[j];
          l[h * n + t] = c * acc;
        }
      }
      free(kt);
    }
    /* log-sum-exp and output, one head per thread, sums in index order */
#pragma omp parallel
    {
      double *vt = (double *)malloc(sizeof(double) * d);
#pragma omp for schedule(static)
      for (int h = 0; h < H; ++h) {
        const double *lh = l + (int64_t)h * n;
        double m = -INFINITY;
        for (int64_t t = 0; t < n; ++t) m = lh[t] > m ? lh[t] : m;
        double z = 0.0;
        for (int64_t t = 0; t < n; ++t) z += exp(lh[t] - m);
        double L = m + log(z);
        ls[h] = L;
        double *o = out + (rr * H + h) * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
          double w = exp(lh[t] - L);
          widen_row(kv, kv->v, kv->v_scale, base + t, vt);
          for (int j = 0; j < d; ++j) o[j] += w * vt[j];
        }
      }
      free(vt);
    }
    for (int h = 0; h < H; ++h) lse[rr * H + h] = ls[h];
    if (scores) {
      double *srow = scores + rr * score_stride;
#pragma omp parallel for schedule(static)
      for (int64_t t = 0; t < n; ++t) {
        double s = 0.0;
        for (int h = 0; h < H; ++h) s += exp(l[(int64_t)h * n + t] - ls[h]);
        srow[t] = s;
      }
    }
    free(qd);
    free(l);
    free(ls);
  }
  return 0;
}

/* ---------------------------------------------------------------- selection */

typedef struct {
  double key;   /* fp64 selector: the score; fp32 selector: the uint32 bit pattern */
  int64_t t;
} cand_t;

static int cmp_cand(const void *a, const void *b) {
  const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
  if (x->key > y->key) return -1;     /* higher score first */
  if (x->key < y->key) return 1;
  return (x->t < y->t) ? -1 : (x->t > y->t);   /* ties: lower index first */
}

static int cmp_i32(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

/* Candidates C = [0, nc) with nc = max(0, p - window + 1); window W = [nc, p].
 * If nc <= topk the selection is every position [0, p]. Otherwise it is the topk candidates by
 * (key descending, index ascending), then W, in ascending order. Returns the count. */
static int64_t select_common(cand_t *cand, int64_t p, int topk, int window, int32_t *out) {
  int64_t nc = p - window + 1;
  if (nc < 0) nc = 0;
  if (nc <= topk) {
    for (int64_t t = 0; t <= p; ++t) out[t] = (int32_t)t;
    return p + 1;
  }
  qsort(cand, (size_t)nc, sizeof(cand_t), cmp_cand);
  for (int j = 0; j < topk; ++j) out[j] = (int32_t)cand[j].t;
  qsort(out, (size_t)topk, sizeof(int32_t), cmp_i32);
  int64_t cnt = topk;
  for (int64_t t = nc; t <= p; ++t) out[cnt++] = (int32_t)t;
  return cnt;
}

/* fp64 selector on the oracle's own scores s[0..p]. */
int64_t hs2o_select_f64(const double *s, int64_t p, int topk, int window, int32_t *out) {
  int64_t nc = p - window + 1;
  if (nc < 0) nc = 0;
  cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(nc > 0 ? nc : 1));
  if (!cand) return -1;
  for (int64_t t = 0; t < nc; ++t) { cand[t].key = s[t]; cand[t].t = t; }
  int64_t cnt = select_common(cand, p, topk, window, out);
  free(cand);
  return cnt;
}

/* fp32 selector on a float array (e.g. the GPU's scores), ordered by the uint32 bit pattern,
 * which for non-negative floats is the numeric order. */
int64_t hs2o_select_f32(const float *s, int64_t p, int topk, int window, int32_t *out) {
  int64_t nc = p - window + 1;
  if (nc < 0) nc = 0;
  cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(nc > 0 ? nc : 1));
  if (!cand) return -1;
  for (int64_t t = 0; t < nc; ++t) {
    uint32_t u;
    memcpy(&u, &s[t], sizeof u);
    cand[t].key = (double)u;
    cand[t].t = t;
  }
  int64_t cnt = select_common(cand, p, topk, window, out);
  free(cand);
  return cnt;
}

/* Batched selectors over listed rows; scores [*, score_stride] indexed by list position,
 * out [*, out_stride] and count [*] likewise. */
int hs2o_select_rows_f64(const hs2o_kv *kv, const int64_t *rows, int64_t n_rows,
                         const double *scores, int64_t score_stride, int topk, int window,
                         int32_t *out, int64_t out_stride, int32_t *count) {
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int64_t rr = 0; rr < n_rows; ++rr) {
    int64_t r = rows[rr], b = r / kv->n_q, i = r % kv->n_q;
    int64_t p = (int64_t)kv->kv_len[b] - kv->n_q + i;
    int64_t c = hs2o_select_f64(scores + rr * score_stride, p, topk, window,
                                out + rr * out_stride);
    if (c < 0) bad = 1;
    count[rr] = (int32_t)c;
  }
  return bad ? -1 : 0;
}

int hs2o_select_rows_f32(const hs2o_kv *kv, const int64_t *rows, int64_t n_rows,
                         const float *scores, int64_t score_stride, int topk, int window,
                         int32_t *out, int64_t out_stride, int32_t *count) {
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int64_t rr = 0; rr < n_rows; ++rr) {
    int64_t r = rows[rr], b = r / kv->n_q, i = r % kv->n_q;
    int64_t p = (int64_t)kv->kv_len[b] - kv->n_q + i;
    int64_t c = hs2o_select_f32(scores + rr * score_stride, p, topk, window,
                                out + rr * out_stride);
    if (c < 0) bad = 1;
    count[rr] = (int32_t)c;
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------- KV Bridging */

/* The cross-decoder full layer's K and V projected from a self-decoder full layer's hidden
 * states ("HySparse2: How Xiaomi Split the Transformer to Fix Agent Prefill Costs", section
 * "The Self-Decoder and Cross-Decoder Split": K_j = Proj_j^K(H_i^self), V_j = Proj_j^V(H_i^self),
 * learned projections; read here as plain linear maps, no bias). hidden: bf16 bits [m, d];
 * w: bf16 bits [256, d], rows 0..127 the K projection, 128..255 the V projection (output
 * feature x input feature). out: [m, 256] = hidden . w^T in double, summed in index order. */
void hs2o_kv_bridge(const uint16_t *hidden, const uint16_t *w, int64_t m, int d, double *out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < m; ++r) {
    double *h = (double *)malloc(sizeof(double) * (size_t)d);
    if (!h) continue;
    for (int e = 0; e < d; ++e) h[e] = bf16_to_double(hidden[r * d + e]);
    for (int c = 0; c < 256; ++c) {
      double acc = 0.0;
      for (int e = 0; e < d; ++e) acc += h[e] * bf16_to_double(w[(int64_t)c * d + e]);
      out[r * 256 + c] = acc;
    }
    free(h);
  }
}

/* ---------------------------------------------------------------- block-level selection */

/* The block-granular selection HySparse used and HySparse2 replaces ("HySparse2: How Xiaomi
 * Split the Transformer to Fix Agent Prefill Costs", section "KV Reuse and Token-Level Sparse
 * Selection": block-level selection hands the budget out 64 tokens at a time; the token-level
 * variant hands out the same 1,024 tokens one by one; "HySparse2: Hybrid Sparse Attention with
 * Two-Level KV Sharing", bullet "KV Reuse refinements": same attention budget). Read here as:
 * the candidates C = [0, nc) are cut at multiples of the block size bs into blocks
 * [j*bs, min((j+1)*bs, nc)); a block's score is the sum of its candidates' scores; the
 * topk / bs blocks with the largest score (ties: lower block index) are kept, their positions
 * in ascending order, then the window W = [nc, p]. If nc <= topk every position is kept, as
 * for tokens. bs must be a power of two that divides topk. */
static int64_t select_blocks_common(cand_t *blk, int64_t nb, int64_t nc, int64_t p, int bs,
                                    int topk, int window, int32_t *out) {
  const int kb = topk / bs;
  qsort(blk, (size_t)nb, sizeof(cand_t), cmp_cand);
  int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)kb);
  if (!ids) return -1;
  for (int j = 0; j < kb; ++j) ids[j] = (int32_t)blk[j].t;
  qsort(ids, (size_t)kb, sizeof(int32_t), cmp_i32);
  int64_t cnt = 0;
  for (int j = 0; j < kb; ++j) {
    const int64_t t0 = (int64_t)ids[j] * bs;
    const int64_t t1 = t0 + bs < nc ? t0 + bs : nc;
    for (int64_t t = t0; t < t1; ++t) out[cnt++] = (int32_t)t;
  }
  free(ids);
  for (int64_t t = nc; t <= p; ++t) out[cnt++] = (int32_t)t;
  return cnt;
}

static int blocks_args_ok(int bs, int topk) {
  return bs >= 1 && (bs & (bs - 1)) == 0 && topk >= bs && topk % bs == 0;
}

/* fp64 selector: block score = the block's candidate scores summed in double, in index order. */
int64_t hs2o_select_blocks_f64(const double *s, int64_t p, int bs, int topk, int window,
                               int32_t *out) {
  if (!blocks_args_ok(bs, topk)) return -1;
  int64_t nc = p - window + 1;
  if (nc < 0) nc = 0;
  if (nc <= topk) {
    for (int64_t t = 0; t <= p; ++t) out[t] = (int32_t)t;
    return p + 1;
  }
  const int64_t nb = (nc + bs - 1) / bs;
  cand_t *blk = (cand_t *)malloc(sizeof(cand_t) * (size_t)nb);
  if (!blk) return -1;
  for (int64_t j = 0; j < nb; ++j) {
    double acc = 0.0;
    for (int64_t t = j * bs; t < (j + 1) * bs && t < nc; ++t) acc += s[t];
    blk[j].key = acc;
    blk[j].t = j;
  }
  int64_t cnt = select_blocks_common(blk, nb, nc, p, bs, topk, window, out);
  free(blk);
  return cnt;
}

/* The float32 block score: the bs values of the block (0 for positions >= nc) summed by folding
 * the array in half until one value remains (v[i] = v[i] + v[i + n/2] for i < n/2, n = bs, bs/2,
 * ..., 2), each addition rounded to float32. This fixed order makes the score -- and so the
 * selection -- a function of the fp32 scores alone. */
float hs2o_block_score_f32(const float *s, int64_t t0, int64_t nc, int bs) {
  float v[4096];
  if (bs < 1 || bs > 4096 || (bs & (bs - 1))) return -1.0f;
  for (int i = 0; i < bs; ++i) v[i] = (t0 + i < nc) ? s[t0 + i] : 0.0f;
  for (int n = bs; n > 1; n /= 2)
    for (int i = 0; i < n / 2; ++i) v[i] = v[i] + v[i + n / 2];
  return v[0];
}

/* fp32 selector (e.g. on the GPU's scores): block scores as hs2o_block_score_f32, ordered by
 * their bit patterns (numeric order for non-negative floats). */
int64_t hs2o_select_blocks_f32(const float *s, int64_t p, int bs, int topk, int window,
                               int32_t *out) {
  if (!blocks_args_ok(bs, topk) || bs > 4096) return -1;
  int64_t nc = p - window + 1;
  if (nc < 0) nc = 0;
  if (nc <= topk) {
    for (int64_t t = 0; t <= p; ++t) out[t] = (int32_t)t;
    return p + 1;
  }
  const int64_t nb = (nc + bs - 1) / bs;
  cand_t *blk = (cand_t *)malloc(sizeof(cand_t) * (size_t)nb);
  if (!blk) return -1;
  for (int64_t j = 0; j < nb; ++j) {
    const float v = hs2o_block_score_f32(s, j * bs, nc, bs);
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    blk[j].key = (double)u;
    blk[j].t = j;
  }
  int64_t cnt = select_blocks_common(blk, nb, nc, p, bs, topk, window, out);
  free(blk);
  return cnt;
}

/* Batched block selectors over listed rows (layouts as hs2o_select_rows_*); fp32 != 0 picks the
 * float32 selector on float scores, else the fp64 one on double scores. */
int hs2o_select_blocks_rows(const hs2o_kv *kv, const int64_t *rows, int64_t n_rows,
                            const void *scores, int64_t score_stride, int fp32, int bs, int topk,
                            int window, int32_t *out, int64_t out_stride, int32_t *count) {
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int64_t rr = 0; rr < n_rows; ++rr) {
    int64_t r = rows[rr], b = r / kv->n_q, i = r % kv->n_q;
    int64_t p = (int64_t)kv->kv_len[b] - kv->n_q + i;
    int64_t c = fp32 ? hs2o_select_blocks_f32((const float *)scores + rr * score_stride, p, bs,
                                              topk, window, out + rr * out_stride)
                     : hs2o_select_blocks_f64((const double *)scores + rr * score_stride, p, bs,
                                              topk, window, out + rr * out_stride);
    if (c < 0) bad = 1;
    count[rr] = (int32_t)c;
  }
  return bad ? -1 : 0;
}

/* ---------------------------------------------------------------- sparse attention */

/* For each listed row, attention of its own queries over the selected cache positions only:
 *   l_h[j] = c * q_h . k_{S_j},  O_h = sum_j softmax_j(l_h) v_{S_j}
 * idx: [*, idx_stride] positions within the sequence (first count[*] valid), indexed by list
 * position. q: bf16 bits [batch, n_q, H, d]. out: [n_rows, H, d]. */
int hs2o_sparse_attn(const hs2o_kv *kv, const uint16_t *q, double c, const int64_t *rows,
                     int64_t n_rows, const int32_t *idx, int64_t idx_stride,
                     const int32_t *count, double *out) {
  ensure_tables();
  const int H = kv->n_heads, d = kv->head_dim;
  int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
  for (int64_t rr = 0; rr < n_rows; ++rr) {
    int64_t r = rows[rr], b = r / kv->n_q, i = r % kv->n_q;
    int64_t p = (int64_t)kv->kv_len[b] - kv->n_q + i, base = kv->kv_start[b];
    int64_t n = count[rr];
    const int32_t *S = idx + rr * idx_stride;
    double *kt = (double *)malloc(sizeof(double) * d);
    double *qd = (double *)malloc(sizeof(double) * H * d);
    double *l = (double *)malloc(sizeof(double) * (size_t)H * (size_t)(n > 0 ? n : 1));
    if (!kt || !qd || !l) { free(kt); free(qd); free(l); bad = 1; continue; }
    for (int h = 0; h < H; ++h)
      for (int e = 0; e < d; ++e) qd[h * d + e] = bf16_to_double(q[((r * H) + h) * d + e]);
    for (int64_t j = 0; j < n; ++j) {
      if (S[j] < 0 || S[j] > p) { bad = 1; break; }
      widen_row(kv, kv->k, kv->k_scale, base + S[j], kt);
      for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += qd[h * d + e] * kt[e];
        l[h * n + j] = c * acc;
      }
    }
    if (!bad) {
      for (int h = 0; h < H; ++h) {
        const double *lh = l + (int64_t)h * n;
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) m = lh[j] > m ? lh[j] : m;
        double z = 0.0;
        for (int64_t j = 0; j < n; ++j) z += exp(lh[j] - m);
        double L = m + log(z);
        double *o = out + (rr * H + h) * d;
        for (int e = 0; e < d; ++e) o[e] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
          double w = exp(lh[j] - L);
          widen_row(kv, kv->v, kv->v_scale, base + S[j], kt);
          for (int e = 0; e < d; ++e) o[e] += w * kt[e];
        }
      }
    }
    free(kt);
    free(qd);
    free(l);
  }
  return bad ? -1 : 0;
}

int hs2o_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- KV append (FP8 quantise) */

/* Round-to-nearest-even of y (|y| <= 448, already a float32 value) to the OCP e4m3fn code,
 * from the format definition: subnormals are multiples of 2^-9 below 2^-6; a normal value with
 * exponent e in [-6, 8] has mantissa steps of 2^(e-3); a carry out of the mantissa moves to the
 * next exponent; the largest finite value 448 (S.1111.110) is the saturation point. */
uint8_t hs2o_e4m3_rne(float y) {
  const int neg = signbit(y) ? 1 : 0;
  double a = fabs((double)y);
  if (a > 448.0) a = 448.0;
  int code;
  if (a < ldexp(1.0, -6)) {
    code = (int)rint(a / ldexp(1.0, -9));          /* 0..8; 8 is the smallest normal (0x08) */
  } else {
    int e;
    frexp(a, &e);                                     /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                           /* a = (1 + frac) * 2^e */
    int q = (int)rint((a / ldexp(1.0, e) - 1.0) * 8.0);
    int E = e + 7;
    if (q == 8) {
      q = 0;
      E += 1;
    }
    code = (E << 3) | q;
    if (code > 0x7e) code = 0x7e;
  }
  return (uint8_t)(code | (neg << 7));
}

/* The FP8 cache write of one appended row of d bf16 values, from the format's definition
 * value = scale * code: scale = max|x| / 448 in float32 (1 for an all-zero row), and each code is
 * the e4m3 RNE of the float32 quotient x / scale (IEEE division, correctly rounded), saturated
 * at 448. */
void hs2o_quantize_row(const uint16_t *x_bf16, int d, uint8_t *codes, float *scale) {
  float amax = 0.f;
  for (int j = 0; j < d; ++j) {
    uint32_t u = (uint32_t)x_bf16[j] << 16;
    float v;
    memcpy(&v, &u, 4);
    if (fabsf(v) > amax) amax = fabsf(v);
  }
  const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
  for (int j = 0; j < d; ++j) {
    uint32_t u = (uint32_t)x_bf16[j] << 16;
    float v;
    memcpy(&v, &u, 4);
    const float y = v / sc;
    codes[j] = hs2o_e4m3_rne(y);
  }
  *scale = sc;
}
