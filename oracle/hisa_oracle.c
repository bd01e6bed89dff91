/*
 * hisa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, step-by-step CPU statement of the two-level (block -> token)
 * indexer and of the sparse attention that consumes its output.  Only the
 * tests, the smoke check and the bench's CPU-baseline leg may load it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources (cited by short key below):
 *   [IP]  "北大HISA稀疏注意力机制：长文本处理效率提升3倍" (intelliparadigm.com),
 *         section 1.2.1 "块级粗过滤" (coarse block filtering) and section
 *         1.2.2 "块内精筛选" (fine token selection).
 *   [QB]  QbitAI article on HISA (m.digipub.cc, KPSAJS2O0511DSSR), sections
 *         "塊級粗過濾", "塊內精挑字符" and the complexity / drop-in paragraph
 *         "HISA的關鍵優勢在於".
 *
 * Arithmetic: inputs are bf16 bit patterns; everything is computed in fp64.
 * On the integer-valued indexer inputs every block mean, block score and token
 * score is exact, so the selections below are exact.
 *
 * Readings of points the pages leave open (each one is listed with its reason
 * in the design notes):
 *   - the indexer score is a single-head dot product q.k, or, when the
 *     indexer has H >= 1 query heads, sum_j w_j * max(0, q_j . k) with the
 *     query's head weights w_j (the original indexer's own score function,
 *     which [IP] 1.3 item 4 asks to keep; the form is the multi-head indexer
 *     of DeepSeek-V3.2);
 *   - "first and last block" = block 0 and the query's own block
 *     c = floor(p / B), the newest block the query can see;
 *   - the two forced blocks count toward m;
 *   - the final k tokens are a global top-k over the union of the selected
 *     blocks' causally visible tokens;
 *   - ties go to the lower index (score descending, index ascending);
 *   - index lists are written in ascending order, padded with -1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_value(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

typedef struct {
  double score;
  int64_t index;
} scored_t;

/* Total order of the selection: higher score first, then lower index. */
static int by_score_desc_index_asc(const void *a, const void *b) {
  const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

static int by_index_asc(const void *a, const void *b) {
  const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
  return (x->index > y->index) - (x->index < y->index);
}

static double dot_bf16_bf16(const uint16_t *a, const uint16_t *b, int32_t n) {
  double s = 0.0;
  for (int32_t e = 0; e < n; ++e) s += bf16_value(a[e]) * bf16_value(b[e]);
  return s;
}

static double dot_bf16_f64(const uint16_t *a, const double *b, int32_t n) {
  double s = 0.0;
  for (int32_t e = 0; e < n; ++e) s += bf16_value(a[e]) * b[e];
  return s;
}

/* The indexer's score of one key -- [IP] 1.2.1 item 2 and 1.2.2 item 1 (the
 * original indexer's score function), 1.3 item 4 (the same score function as
 * the original model).  n_idx_heads = 0: the dot product q . key.
 * n_idx_heads = H >= 1: sum over the query's H heads q_j ([H][d_idx]) of
 * w_j * max(0, q_j . key).  One version per key type: block keys are fp64
 * means, token keys bf16. */
static double relu(double x) { return x > 0.0 ? x : 0.0; }

static double score_block_key(const uint16_t *q, const double *w, int32_t n_idx_heads, const double *key,
                              int32_t d_idx) {
  if (n_idx_heads == 0) return dot_bf16_f64(q, key, d_idx);
  double s = 0.0;
  for (int32_t j = 0; j < n_idx_heads; ++j) s += w[j] * relu(dot_bf16_f64(q + (int64_t)j * d_idx, key, d_idx));
  return s;
}

static double score_token_key(const uint16_t *q, const double *w, int32_t n_idx_heads, const uint16_t *key,
                              int32_t d_idx) {
  if (n_idx_heads == 0) return dot_bf16_bf16(q, key, d_idx);
  double s = 0.0;
  for (int32_t j = 0; j < n_idx_heads; ++j) s += w[j] * relu(dot_bf16_bf16(q + (int64_t)j * d_idx, key, d_idx));
  return s;
}

/* Step 1 -- [IP] 1.2.1 item 1, [QB] "塊級粗過濾" first bullet: cut the keys into
 * fixed blocks of B tokens and mean-pool each block into one block key.  The
 * last block may be partial; its mean is over the tokens it holds.
 * k_idx: [n_kv][d_idx] of one sequence; block_keys: [ceil(n_kv/B)][d_idx]. */
void hisa_oracle_block_pool(const uint16_t *k_idx, int64_t n_kv, int32_t d_idx, int32_t block,
                            double *block_keys) {
  int64_t n_blk = (n_kv + block - 1) / block;
  for (int64_t j = 0; j < n_blk; ++j) {
    int64_t t0 = j * block;
    int64_t cnt = n_kv - t0 < block ? n_kv - t0 : block;
    for (int32_t e = 0; e < d_idx; ++e) {
      double sum = 0.0;
      for (int64_t t = t0; t < t0 + cnt; ++t) sum += bf16_value(k_idx[t * d_idx + e]);
      block_keys[j * d_idx + e] = sum / (double)cnt;
    }
  }
}

/* Steps 2-3 -- [IP] 1.2.1 items 2-3, [QB] "塊級粗過濾" bullets 2-3 and the
 * forced-block remark of "塊內精挑字符": score the query against the block keys
 * it can see with the indexer's score and keep m blocks, always
 * including the first block and the query's own block.
 * Returns s = min(m, c+1), the number of selected blocks.  sel[0..m) receives
 * the selected block ids in ascending order, -1 padded.  sel_scores (may be
 * NULL) receives the score of each selected block (NAN for padding).  q_row:
 * [max(1, n_idx_heads)][d_idx]; w: [n_idx_heads] (unused when 0). */
int32_t hisa_oracle_block_topm(const uint16_t *q_row, const double *w, int32_t n_idx_heads, const double *block_keys,
                               int32_t d_idx, int32_t block, int64_t p, int32_t top_m, int32_t *sel,
                               double *sel_scores) {
  int64_t c = p / block; /* the query's own block */
  int64_t n_vis = c + 1;
  int64_t s = top_m < n_vis ? top_m : n_vis;
  int64_t n = 0;
  if (s == n_vis) {
    /* every visible block fits: nothing is filtered */
    for (int64_t j = 0; j <= c; ++j) sel[n++] = (int32_t)j;
  } else {
    /* s < n_vis implies c >= 2 and s >= 2: the forced pair plus the best s-2 of blocks 1..c-1 */
    int64_t n_mid = c - 1;
    scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)n_mid);
    for (int64_t j = 1; j <= c - 1; ++j) {
      cand[j - 1].score = score_block_key(q_row, w, n_idx_heads, block_keys + j * d_idx, d_idx);
      cand[j - 1].index = j;
    }
    qsort(cand, (size_t)n_mid, sizeof(scored_t), by_score_desc_index_asc);
    qsort(cand, (size_t)(s - 2), sizeof(scored_t), by_index_asc);
    sel[n++] = 0;
    for (int64_t r = 0; r < s - 2; ++r) sel[n++] = (int32_t)cand[r].index;
    sel[n++] = (int32_t)c;
    free(cand);
  }
  for (int64_t r = n; r < top_m; ++r) sel[r] = -1;
  if (sel_scores) {
    for (int64_t r = 0; r < top_m; ++r)
      sel_scores[r] =
          sel[r] >= 0 ? score_block_key(q_row, w, n_idx_heads, block_keys + (int64_t)sel[r] * d_idx, d_idx) : NAN;
  }
  return (int32_t)s;
}

/* Keep the best k of n scored candidates (score desc, index asc); write their
 * indices ascending, -1 padded to top_k.  Returns k_eff. */
static int32_t keep_top_k(scored_t *cand, int64_t n, int32_t top_k, int32_t *tok, double *tok_scores) {
  int64_t k_eff = n < top_k ? n : top_k;
  qsort(cand, (size_t)n, sizeof(scored_t), by_score_desc_index_asc);
  qsort(cand, (size_t)k_eff, sizeof(scored_t), by_index_asc);
  for (int64_t r = 0; r < top_k; ++r) {
    tok[r] = r < k_eff ? (int32_t)cand[r].index : -1;
    if (tok_scores) tok_scores[r] = r < k_eff ? cand[r].score : NAN;
  }
  return (int32_t)k_eff;
}

/* Steps 4-5 -- [IP] 1.2.2 items 1-2, [QB] "塊內精挑字符": run the token-level
 * indexer only on the tokens of the selected blocks that the query can see
 * (t <= p), and keep the top k of their union.  The output has the flat
 * indexer's format (ascending token ids, -1 padded), so attention is unchanged.
 * k_idx: [n_kv][d_idx] of the query's sequence.  Returns k_eff; *n_cand gets
 * the number of candidates scanned. */
int32_t hisa_oracle_token_topk(const uint16_t *q_row, const double *w, int32_t n_idx_heads, const uint16_t *k_idx,
                               int32_t d_idx, int32_t block, int64_t n_kv, int64_t p, const int32_t *sel,
                               int32_t top_m, int32_t top_k, int32_t *tok, double *tok_scores, int64_t *n_cand) {
  int64_t cap = (int64_t)top_m * block, n = 0;
  scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)(cap > 0 ? cap : 1));
  for (int32_t r = 0; r < top_m; ++r) {
    if (sel[r] < 0) continue;
    int64_t t0 = (int64_t)sel[r] * block;
    int64_t t1 = t0 + block;
    if (t1 > n_kv) t1 = n_kv;
    if (t1 > p + 1) t1 = p + 1;
    for (int64_t t = t0; t < t1; ++t) {
      cand[n].score = score_token_key(q_row, w, n_idx_heads, k_idx + t * d_idx, d_idx);
      cand[n].index = t;
      ++n;
    }
  }
  if (n_cand) *n_cand = n;
  int32_t k_eff = keep_top_k(cand, n, top_k, tok, tok_scores);
  free(cand);
  return k_eff;
}

/* The flat token indexer the two-level one replaces ([IP] 1.1 item 1, [QB]
 * "兩步消除上下文索引瓶頸"): score every token t <= p and keep the top k. */
int32_t hisa_oracle_flat_topk(const uint16_t *q_row, const double *w, int32_t n_idx_heads, const uint16_t *k_idx,
                              int32_t d_idx, int64_t p, int32_t top_k, int32_t *tok, double *tok_scores) {
  scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)(p + 1));
  for (int64_t t = 0; t <= p; ++t) {
    cand[t].score = score_token_key(q_row, w, n_idx_heads, k_idx + t * d_idx, d_idx);
    cand[t].index = t;
  }
  int32_t k_eff = keep_top_k(cand, p + 1, top_k, tok, tok_scores);
  free(cand);
  return k_eff;
}

/* Step 6 -- [QB] "HISA的關鍵優勢在於" (downstream attention unchanged): per
 * head h, softmax attention of Q[h] over the selected tokens' K and V:
 *   w_t = exp(scale * Q[h].K[t][g] - max),  O[h] = sum_t w_t V[t][g] / sum_t w_t,
 *   LSE[h] = max + ln sum_t w_t,   g = h / (n_heads / n_kv_heads).
 * q_row: [n_heads][d]; k, v: [*][n_kv_heads][d] addressed by token id; tok:
 * top_k ids, -1 entries skipped.  o: [n_heads][d], lse: [n_heads]. */
void hisa_oracle_sparse_attn(const uint16_t *q_row, const uint16_t *k, const uint16_t *v, int32_t n_heads,
                             int32_t n_kv_heads, int32_t d_head, double scale, const int32_t *tok, int32_t top_k,
                             double *o, double *lse) {
  int32_t group = n_heads / n_kv_heads;
  double *w = (double *)malloc(sizeof(double) * (size_t)(top_k > 0 ? top_k : 1));
  for (int32_t h = 0; h < n_heads; ++h) {
    int32_t g = h / group;
    const uint16_t *qh = q_row + (int64_t)h * d_head;
    double mx = -INFINITY;
    for (int32_t r = 0; r < top_k; ++r) {
      if (tok[r] < 0) continue;
      const uint16_t *kr = k + ((int64_t)tok[r] * n_kv_heads + g) * d_head;
      w[r] = scale * dot_bf16_bf16(qh, kr, d_head);
      if (w[r] > mx) mx = w[r];
    }
    double sum = 0.0;
    for (int32_t r = 0; r < top_k; ++r) {
      if (tok[r] < 0) continue;
      w[r] = exp(w[r] - mx);
      sum += w[r];
    }
    for (int32_t e = 0; e < d_head; ++e) {
      double acc = 0.0;
      for (int32_t r = 0; r < top_k; ++r) {
        if (tok[r] < 0) continue;
        acc += w[r] * bf16_value(v[((int64_t)tok[r] * n_kv_heads + g) * d_head + e]);
      }
      o[(int64_t)h * d_head + e] = acc / sum;
    }
    lse[h] = mx + log(sum);
  }
  free(w);
}

/* The whole path for a list of queries (ids seq * n_q + i; position
 * p = n_kv - n_q + i), in parallel over queries.  block_keys comes from
 * hisa_oracle_block_pool of every sequence ([batch][n_blk][d_idx]).  Outputs
 * are one row per listed query.  q_idx: [batch][n_q][max(1, n_idx_heads)][d_idx];
 * idx_w: [batch][n_q][n_idx_heads] (NULL when n_idx_heads is 0).  With flat != 0 the token list comes from the
 * flat indexer and block_idx is left untouched.  q, k, v may be NULL (indexer
 * only).  n_cand (may be NULL) gets the candidates each query scanned. */
int32_t hisa_oracle_run(int32_t batch, int64_t n_q, int64_t n_kv, int32_t d_idx, int32_t block, int32_t top_m,
                        int32_t top_k, int32_t n_heads, int32_t n_kv_heads, int32_t d_head, double scale,
                        int32_t n_idx_heads, const double *idx_w,
                        const uint16_t *q_idx, const uint16_t *k_idx, const double *block_keys, const uint16_t *q,
                        const uint16_t *k, const uint16_t *v, const int64_t *query_ids, int64_t n_queries,
                        int32_t *block_idx, int32_t *token_idx, double *o, double *lse, int64_t *n_cand,
                        int32_t flat) {
  int64_t n_blk = (n_kv + block - 1) / block;
  int64_t bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
#endif
  for (int64_t r = 0; r < n_queries; ++r) {
    int64_t id = query_ids[r];
    int64_t seq = id / n_q, i = id % n_q;
    if (seq < 0 || seq >= batch) {
      ++bad;
      continue;
    }
    int64_t p = n_kv - n_q + i;
    const int32_t qh = n_idx_heads > 0 ? n_idx_heads : 1;
    const uint16_t *qi = q_idx + id * qh * d_idx;
    const double *wi = n_idx_heads > 0 ? idx_w + id * n_idx_heads : NULL;
    const uint16_t *ks = k_idx + seq * n_kv * d_idx;
    int32_t *tok = token_idx + r * top_k;
    int64_t nc = 0;
    if (flat) {
      hisa_oracle_flat_topk(qi, wi, n_idx_heads, ks, d_idx, p, top_k, tok, NULL);
      nc = p + 1;
    } else {
      int32_t *sel = block_idx + r * top_m;
      hisa_oracle_block_topm(qi, wi, n_idx_heads, block_keys + seq * n_blk * d_idx, d_idx, block, p, top_m, sel,
                             NULL);
      hisa_oracle_token_topk(qi, wi, n_idx_heads, ks, d_idx, block, n_kv, p, sel, top_m, top_k, tok, NULL, &nc);
    }
    if (n_cand) n_cand[r] = nc;
    if (q && k && v && o && lse) {
      int64_t per_kv = (int64_t)n_kv_heads * d_head;
      hisa_oracle_sparse_attn(q + id * (int64_t)n_heads * d_head, k + seq * n_kv * per_kv,
                              v + seq * n_kv * per_kv, n_heads, n_kv_heads, d_head, scale, tok, top_k,
                              o + r * (int64_t)n_heads * d_head, lse + r * n_heads);
    }
  }
  return bad ? -1 : 0;
}

int32_t hisa_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void hisa_oracle_set_threads(int32_t n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
