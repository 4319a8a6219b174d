/*
 * fp64 CPU oracle for vertical-slash sparse prefill attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may call this code; the product path
 * never does.  It shares no code with the CUDA kernels.
 *
 * What it computes follows the VSPrefill summary pages:
 *   - vertical lines are key columns j, slash lines are diagonals at a fixed
 *     relative offset o = i - j ("VSPrefill ..." Technical Summary, section 2
 *     Methodology, "Core Concept: Vertical-Slash Pattern");
 *   - attention for query i runs over the union of the selected columns and
 *     the keys at the selected offsets behind it, with no n x n matrix
 *     (section 2, "Adaptive Inference Pipeline", fused kernel);
 *   - budgets come from a fixed top-k or from a cumulative-mass threshold on
 *     the predicted scores (section 2, "Dynamic Budgeting");
 *   - scores may come from a shared-weight two-layer linear map on
 *     concat(K with RoPE, V) (section 2, "VSIndexer").
 * The precise readings taken where the pages are silent are listed beside
 * each function.
 *
 * Every function is plain fp64 arithmetic in the order of its definition.
 * OpenMP parallelises independent rows only; it never changes the order of a
 * sum.
 *
 * Parity status: every function here is pinned by tests against closed
 * forms, brute force or library routines (see the oracle tests).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BF16 0
#define OR_FP32 1

#define OR_TOPK 0
#define OR_THRESHOLD 1
#define OR_MAXFRAC 2

static double load_elem(const void* base, int dtype, int64_t off) {
  if (dtype == OR_BF16) {
    uint32_t b = ((uint32_t)((const uint16_t*)base)[off]) << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
  }
  return (double)((const float*)base)[off];
}

/* ---------------------------------------------------------------- select
 * Order: score descending, NaN after everything (also after -inf), ties by
 * smaller index.  -0.0 and +0.0 compare equal (plain float comparison).
 *
 * TOPK: the first k entries in that order.
 * THRESHOLD ("cumulative-threshold strategy" on the predicted scores read as
 * logits): p_r = exp(s_r - s_max) in fp64, with p_r = 1 for entries equal to
 * s_max and p_r = 0 for NaN; Z = sum of p_r in the sorted order; k is the
 * smallest k >= 1 whose prefix sum reaches tau*Z (>=); tau == 1 keeps every
 * entry with p_r > 0; Z == 0 gives k = 1; then k = min(k, cap).
 * MAXFRAC (FlashPrefill summary page, section 2B, "max-based dynamic
 * thresholding": an entry survives when its score is at least alpha times
 * the largest score; no sort, no cumulative sum).  The score of an entry is
 * its softmax mass, so the rule is p_r / Z >= alpha * p_max / Z, i.e.
 * exp(s_r - s_max) >= alpha, taken in the log domain as
 *     keep r  iff  s_r == s_max  or  (double)s_r - (double)s_max >= log(alpha)
 * with `tau` carrying alpha in (0, 1]; NaN is never kept; when every score
 * is NaN, k = 1; then k = min(k, cap).  The kept entries are a prefix of the
 * order above, so the output is that prefix.
 * Output: the k indices in ascending order, padded with -1 up to k_or_cap.
 * `margin` receives min(|prefix(k-1) - tau Z|, |prefix(k) - tau Z|) / Z for
 * the threshold decision (+inf for TOPK, and +inf when the uncapped k exceeds
 * the cap, since then a +-1 change of k does not change the output), so
 * callers can flag heads whose output sits within rounding of a boundary.
 */
typedef struct {
  float s;
  int32_t i;
} or_pair;

static int cmp_pair(const void* a, const void* b) {
  const or_pair* x = (const or_pair*)a;
  const or_pair* y = (const or_pair*)b;
  int xn = isnan(x->s), yn = isnan(y->s);
  if (xn != yn) return xn ? 1 : -1; /* NaN last */
  if (!xn) {
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
  }
  return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

int or_select(const float* s, int N, int mode, int k_or_cap, double tau, int32_t* idx,
              int32_t* count, double* margin) {
  if (N < 1 || k_or_cap < 1 || k_or_cap > N) return -1;
  if (mode != OR_TOPK && mode != OR_THRESHOLD && mode != OR_MAXFRAC) return -1;
  if (mode != OR_TOPK && !(tau > 0.0 && tau <= 1.0)) return -1;
  or_pair* v = (or_pair*)malloc(sizeof(or_pair) * (size_t)N);
  for (int r = 0; r < N; ++r) {
    v[r].s = s[r];
    v[r].i = r;
  }
  qsort(v, (size_t)N, sizeof(or_pair), cmp_pair);
  int k;
  *margin = INFINITY;
  if (mode == OR_TOPK) {
    k = k_or_cap;
  } else if (mode == OR_MAXFRAC) {
    const double smax = (double)v[0].s, lna = log(tau);
    k = 0;
    for (int r = 0; r < N; ++r) {
      const double x = (double)v[r].s;
      if (isnan(x)) continue;
      if (x == smax || x - smax >= lna) ++k;
    }
    if (k < 1) k = 1;
    if (k > k_or_cap) k = k_or_cap;
  } else {
    double smax = (double)v[0].s;
    double* p = (double*)malloc(sizeof(double) * (size_t)N);
    for (int r = 0; r < N; ++r) {
      double x = (double)v[r].s;
      if (isnan(x)) p[r] = 0.0;
      else if (x == smax) p[r] = 1.0;
      else p[r] = exp(x - smax);
    }
    double Z = 0.0;
    for (int r = 0; r < N; ++r) Z += p[r];
    if (Z == 0.0) {
      k = 1;
    } else if (tau == 1.0) {
      k = 0;
      for (int r = 0; r < N; ++r) k += (p[r] > 0.0);
      if (k < 1) k = 1;
    } else {
      double target = tau * Z, prefix = 0.0, prev = 0.0;
      k = N;
      for (int r = 0; r < N; ++r) {
        prev = prefix;
        prefix += p[r];
        if (prefix >= target) {
          k = r + 1;
          break;
        }
      }
      double m1 = fabs(prev - target) / Z, m2 = fabs(prefix - target) / Z;
      *margin = m1 < m2 ? m1 : m2;
    }
    free(p);
    /* a +-1 change of an uncapped k above the cap leaves min(k, cap) unchanged */
    if (k > k_or_cap) *margin = INFINITY;
    if (k > k_or_cap) k = k_or_cap;
  }
  for (int r = 0; r < k; ++r) idx[r] = v[r].i;
  qsort(idx, (size_t)k, sizeof(int32_t), cmp_i32);
  for (int r = k; r < k_or_cap; ++r) idx[r] = -1;
  *count = k;
  free(v);
  return 0;
}

/* ------------------------------------------------------------- attention
 * Key set of query i in query head h:
 *   K_i = {j in V_h : j <= i}  union  {i - o : o in S_h, o <= i}
 * each key counted once (set union).  Query head h reads KV head
 * h / (Hq/Hkv) and index-set head h * H_sel / Hq.
 * s_ij = scale * q_i . k_j in fp64 (inputs upcast exactly);
 * O_i = sum_j exp(s_ij - m) v_j / sum_j exp(s_ij - m), m = max_j s_ij;
 * LSE_i = m + log(sum_j exp(s_ij - m)).  An empty key set gives O_i = 0 and
 * LSE_i = -inf.  `dense` != 0 ignores the index sets and uses K_i = [0, i].
 */
typedef struct {
  const void *Q, *K, *V;
  int dtype, N, Hq, Hkv, d;
  int64_t q_stride_tok, kv_stride_tok;
  double scale;
  int H_sel;
  const int32_t* v_idx;
  int64_t v_ld;
  const int32_t* v_cnt;
  const int32_t* s_idx;
  int64_t s_ld;
  const int32_t* s_cnt;
  int dense;
} or_attn_args;

static void softmax_row(const or_attn_args* a, int h, int64_t i, const int32_t* keys, int nk,
                        double* o, double* lse) {
  const int d = a->d;
  const int kvh = h / (a->Hq / a->Hkv);
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (nk == 0) {
    *lse = -INFINITY;
    return;
  }
  double* sc = (double*)malloc(sizeof(double) * (size_t)nk);
  const int64_t qoff = i * a->q_stride_tok + (int64_t)h * d;
  double m = -INFINITY;
  for (int t = 0; t < nk; ++t) {
    const int64_t koff = (int64_t)keys[t] * a->kv_stride_tok + (int64_t)kvh * d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += load_elem(a->Q, a->dtype, qoff + c) * load_elem(a->K, a->dtype, koff + c);
    sc[t] = acc * a->scale;
    if (sc[t] > m) m = sc[t];
  }
  double l = 0.0;
  for (int t = 0; t < nk; ++t) {
    double p = exp(sc[t] - m);
    l += p;
    const int64_t voff = (int64_t)keys[t] * a->kv_stride_tok + (int64_t)kvh * d;
    for (int c = 0; c < d; ++c) o[c] += p * load_elem(a->V, a->dtype, voff + c);
  }
  for (int c = 0; c < d; ++c) o[c] /= l;
  *lse = m + log(l);
  free(sc);
}

/* Row form: builds K_i by merging the ascending column list (prefix j <= i)
 * with the ascending list {i - o} (offsets walked from the largest o <= i
 * down), skipping duplicates.  Works for any N.  Index lists must be
 * ascending. */
static int row_keys(const or_attn_args* a, int h, int64_t i, int32_t* keys) {
  if (a->dense) {
    for (int64_t j = 0; j <= i; ++j) keys[j] = (int32_t)j;
    return (int)(i + 1);
  }
  const int hs = (int)(((int64_t)h * a->H_sel) / a->Hq);
  const int32_t* vv = a->v_idx + (int64_t)hs * a->v_ld;
  const int32_t* ss = a->s_idx + (int64_t)hs * a->s_ld;
  const int nv = a->v_cnt[hs], ns = a->s_cnt[hs];
  int pv = 0, ps = ns - 1, n = 0;
  while (ps >= 0 && ss[ps] > i) --ps; /* largest offset o <= i */
  int32_t last = -1;
  for (;;) {
    int32_t jv = (pv < nv && vv[pv] <= i) ? vv[pv] : INT32_MAX;
    int32_t js = (ps >= 0) ? (int32_t)(i - ss[ps]) : INT32_MAX;
    int32_t j = jv < js ? jv : js;
    if (j == INT32_MAX) break;
    if (jv == j) ++pv;
    if (js == j) --ps;
    if (j != last) keys[n++] = j;
    last = j;
  }
  return n;
}

void or_attn_rows(const void* Q, const void* K, const void* V, int dtype, int N, int Hq, int Hkv,
                  int d, int64_t q_stride_tok, int64_t kv_stride_tok, double scale, int H_sel,
                  const int32_t* v_idx, int64_t v_ld, const int32_t* v_cnt, const int32_t* s_idx,
                  int64_t s_ld, const int32_t* s_cnt, int dense, int h, const int64_t* rows,
                  int nrows, double* O, double* lse) {
  or_attn_args a = {Q, K, V, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok, scale, H_sel,
                    v_idx, v_ld, v_cnt, s_idx, s_ld, s_cnt, dense};
#pragma omp parallel
  {
    int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
      int nk = row_keys(&a, h, rows[r], keys);
      softmax_row(&a, h, rows[r], keys, nk, O + (int64_t)r * d, lse + r);
    }
    free(keys);
  }
}

/* Explicit-mask form (small N): builds the N x N boolean mask
 *   M[i][j] = (j <= i) && (j in V || (i - j) in S)
 * from membership tables, then runs masked softmax over each full row. */
void or_attn_mask(const void* Q, const void* K, const void* V, int dtype, int N, int Hq, int Hkv,
                  int d, int64_t q_stride_tok, int64_t kv_stride_tok, double scale, int H_sel,
                  const int32_t* v_idx, int64_t v_ld, const int32_t* v_cnt, const int32_t* s_idx,
                  int64_t s_ld, const int32_t* s_cnt, int h, double* O, double* lse,
                  uint8_t* mask_out) {
  or_attn_args a = {Q, K, V, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok, scale, H_sel,
                    v_idx, v_ld, v_cnt, s_idx, s_ld, s_cnt, 0};
  const int hs = (int)(((int64_t)h * H_sel) / Hq);
  uint8_t* inV = (uint8_t*)calloc((size_t)N, 1);
  uint8_t* inS = (uint8_t*)calloc((size_t)N, 1);
  for (int t = 0; t < v_cnt[hs]; ++t) inV[v_idx[(int64_t)hs * v_ld + t]] = 1;
  for (int t = 0; t < s_cnt[hs]; ++t) inS[s_idx[(int64_t)hs * s_ld + t]] = 1;
  uint8_t* M = mask_out ? mask_out : (uint8_t*)malloc((size_t)N * (size_t)N);
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j) M[i * N + j] = (j <= i) && (inV[j] || inS[i - j]);
#pragma omp parallel
  {
    int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
    for (int64_t i = 0; i < N; ++i) {
      int nk = 0;
      for (int64_t j = 0; j < N; ++j)
        if (M[i * N + j]) keys[nk++] = (int32_t)j;
      softmax_row(&a, h, i, keys, nk, O + i * d, lse + i);
    }
    free(keys);
  }
  if (!mask_out) free(M);
  free(inV);
  free(inS);
}

/* Number of (i, j) pairs in the key sets of index-set head hs, by brute force
 * over rows (row form). */
int64_t or_count_pairs(int N, const int32_t* v_idx, int nv, const int32_t* s_idx, int ns) {
  int32_t one = 0;
  or_attn_args a = {0};
  a.N = N;
  a.Hq = 1;
  a.H_sel = 1;
  a.v_idx = v_idx;
  a.v_ld = nv;
  a.v_cnt = &nv;
  a.s_idx = s_idx;
  a.s_ld = ns;
  a.s_cnt = &ns;
  (void)one;
  int64_t total = 0;
#pragma omp parallel reduction(+ : total)
  {
    int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
#pragma omp for schedule(dynamic, 64)
    for (int64_t i = 0; i < N; ++i) total += row_keys(&a, 0, i, keys);
    free(keys);
  }
  return total;
}

/* ---------------------------------------------------------------- indexer
 * Per token t and KV head g: x = [k_t ; v_t] (2d values, k first),
 * h_u = max(0, sum_c W1[u][c] x_c) for u < hidden, then
 * logit_v[g][t] = sum_u W2[0][u] h_u and logit_s[g][t] = sum_u W2[1][u] h_u.
 * No biases.  One weight set shared by all heads. */
void or_index_scores(const void* K, const void* V, int dtype, int N, int Hkv, int d,
                     int64_t stride_tok, int64_t stride_head, const float* W1, const float* W2,
                     int hidden, const int64_t* toks, int ntok, double* lv, double* ls) {
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)(2 * d));
    double* hh = (double*)malloc(sizeof(double) * (size_t)hidden);
#pragma omp for schedule(static)
    for (int64_t r = 0; r < (int64_t)ntok * Hkv; ++r) {
      const int64_t t = toks[r / Hkv];
      const int g = (int)(r % Hkv);
      const int64_t off = t * stride_tok + (int64_t)g * stride_head;
      for (int c = 0; c < d; ++c) {
        x[c] = load_elem(K, dtype, off + c);
        x[d + c] = load_elem(V, dtype, off + c);
      }
      for (int u = 0; u < hidden; ++u) {
        double acc = 0.0;
        for (int c = 0; c < 2 * d; ++c) acc += (double)W1[(int64_t)u * 2 * d + c] * x[c];
        hh[u] = acc > 0.0 ? acc : 0.0;
      }
      double a0 = 0.0, a1 = 0.0;
      for (int u = 0; u < hidden; ++u) {
        a0 += (double)W2[u] * hh[u];
        a1 += (double)W2[hidden + u] * hh[u];
      }
      lv[(int64_t)g * ntok + r / Hkv] = a0;
      ls[(int64_t)g * ntok + r / Hkv] = a1;
    }
    free(x);
    free(hh);
  }
}

/* ------------------------------------------------- ground-truth aggregation
 * The distillation target of the VSIndexer ("VSPrefill ..." Technical
 * Summary, section 2, "Distillation Training": a kernel aggregates the full
 * attention weights along vertical columns and slash diagonals during the
 * block-wise computation, without materialising the n x n matrix).  For query
 * head h with full causal softmax weights p_ij (j <= i):
 *     A_v[j] = sum_{i >= j} p_ij          (column sums)
 *     A_s[o] = sum_{i >= o} p_{i, i - o}  (sums along the diagonal at offset o)
 * so that sum_j A_v[j] = sum_o A_s[o] = N.  Scores s_ij = scale * q_i . k_j in
 * fp64 (inputs upcast exactly); p_ij = exp(s_ij - m_i) / sum_j exp(s_ij - m_i).
 * Only rows i in [row_lo, row_hi) contribute (the full result for
 * [0, N)); A_v[j] for j >= row_lo and A_s[o] for o >= row_lo are then exact
 * when row_hi = N, since no other row reaches them.  Rows are added in
 * ascending order; OpenMP runs heads in parallel, never one sum.
 * Av, As: [nheads][N], zeroed here; heads[] lists the query heads. */
void or_aggregate(const void* Q, const void* K, int dtype, int N, int Hq, int Hkv, int d,
                  int64_t q_stride_tok, int64_t kv_stride_tok, double scale, const int* heads,
                  int nheads, int64_t row_lo, int64_t row_hi, double* Av, double* As) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int x = 0; x < nheads; ++x) {
    const int h = heads[x];
    const int kvh = h / (Hq / Hkv);
    double* av = Av + (int64_t)x * N;
    double* as = As + (int64_t)x * N;
    for (int64_t j = 0; j < N; ++j) av[j] = as[j] = 0.0;
    double* q = (double*)malloc(sizeof(double) * (size_t)d);
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    for (int64_t i = row_lo; i < row_hi; ++i) {
      for (int c = 0; c < d; ++c) q[c] = load_elem(Q, dtype, i * q_stride_tok + (int64_t)h * d + c);
      double m = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        const int64_t off = j * kv_stride_tok + (int64_t)kvh * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * load_elem(K, dtype, off + c);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
      }
      double z = 0.0;
      for (int64_t j = 0; j <= i; ++j) z += exp(s[j] - m);
      for (int64_t j = 0; j <= i; ++j) {
        const double p = exp(s[j] - m) / z;
        av[j] += p;
        as[i - j] += p;
      }
    }
    free(q);
    free(s);
  }
}

/* ------------------------------------------------ FlashPrefill block pattern
 * FlashPrefill summary page, section 2A (block approximation: a skeleton of
 * uniformly spaced queries probes the key blocks, with each key block's mean
 * key as its proxy -- the geometric mean of the block's attention weights,
 * a monotone proxy of their sum) and section 2B (max-based threshold: for
 * query block I keep key block J when its score is at least alpha times the
 * best block's score).  Read here as, with blocks of 128 and B_I the probes
 * of query block I (rows 128 I + 8 m, m = 0..15, below N):
 *   kbar_J = mean of the keys of block J (rows below N);
 *   for J < I:  Score(I, J) = mean over q in B_I of
 *               softmax_{J' < I}(scale * q . kbar_J')[J];
 *   keep J < I  iff  Score(I, J) >= alpha * max_{J' < I} Score(I, J');
 *   the diagonal block J = I is always kept (causal coverage);
 * all in fp64.  Output: mask [nheads][T][W] words (W = (T + 31) / 32), bit J
 * of row I set iff block J is kept for query block I.  `margin` receives,
 * per head, the smallest |Score - alpha max| / (alpha max) over the
 * decisions other than the best block's (kept for any alpha <= 1), so callers
 * can flag decisions within rounding of the boundary.
 */
void or_block_select(const void* Q, const void* K, int dtype, int N, int Hq, int Hkv, int d,
                     int64_t q_stride_tok, int64_t kv_stride_tok, double scale, double alpha,
                     const int* heads, int nheads, uint32_t* mask, double* margin) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  const int T = (N + 127) / 128, W = (T + 31) / 32;
#pragma omp parallel for schedule(dynamic, 1)
  for (int x = 0; x < nheads; ++x) {
    const int h = heads[x];
    const int kvh = h / (Hq / Hkv);
    double* kbar = (double*)calloc((size_t)T * d, sizeof(double));
    for (int J = 0; J < T; ++J) {
      int n = 0;
      for (int64_t j = 128 * (int64_t)J; j < 128 * (int64_t)J + 128 && j < N; ++j, ++n)
        for (int c = 0; c < d; ++c)
          kbar[(int64_t)J * d + c] += load_elem(K, dtype, j * kv_stride_tok + (int64_t)kvh * d + c);
      for (int c = 0; c < d; ++c) kbar[(int64_t)J * d + c] /= (double)n;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)T);
    double* score = (double*)malloc(sizeof(double) * (size_t)T);
    double* q = (double*)malloc(sizeof(double) * (size_t)d);
    double mg = INFINITY;
    uint32_t* mrow = mask + (int64_t)x * T * W;
    memset(mrow, 0, sizeof(uint32_t) * (size_t)T * W);
    for (int I = 0; I < T; ++I) {
      uint32_t* m = mrow + (int64_t)I * W;
      m[I >> 5] |= 1u << (I & 31);
      if (I == 0) continue;
      for (int J = 0; J < I; ++J) score[J] = 0.0;
      int np = 0;
      for (int pm = 0; pm < 16; ++pm) {
        const int64_t i = 128 * (int64_t)I + 8 * pm;
        if (i >= N) break;
        ++np;
        for (int c = 0; c < d; ++c) q[c] = load_elem(Q, dtype, i * q_stride_tok + (int64_t)h * d + c);
        double mx = -INFINITY;
        for (int J = 0; J < I; ++J) {
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += q[c] * kbar[(int64_t)J * d + c];
          s[J] = scale * dot;
          if (s[J] > mx) mx = s[J];
        }
        double z = 0.0;
        for (int J = 0; J < I; ++J) z += exp(s[J] - mx);
        for (int J = 0; J < I; ++J) score[J] += exp(s[J] - mx) / z;
      }
      double best = 0.0;
      for (int J = 0; J < I; ++J) {
        score[J] /= (double)np;
        if (score[J] > best) best = score[J];
      }
      const double thr = alpha * best;
      for (int J = 0; J < I; ++J) {
        if (score[J] >= thr) m[J >> 5] |= 1u << (J & 31);
        if (score[J] == best) continue;  /* the best block is kept for any alpha <= 1 */
        const double r = fabs(score[J] - thr) / thr;
        if (r < mg) mg = r;
      }
    }
    margin[x] = mg;
    free(kbar);
    free(s);
    free(score);
    free(q);
  }
}

/* Block-sparse causal attention rows: query i (block I = i / 128) attends
 * to every key j <= i of every block kept in row I of `mask` (as written by
 * or_block_select, [Hq][T][W]); softmax and LSE as in or_attn_rows. */
void or_attn_block_rows(const void* Q, const void* K, const void* V, int dtype, int N, int Hq,
                        int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok, double scale,
                        const uint32_t* mask, int h, const int64_t* rows, int nrows, double* O,
                        double* lse) {
  or_attn_args a = {0};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.dtype = dtype;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.q_stride_tok = q_stride_tok;
  a.kv_stride_tok = kv_stride_tok;
  a.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
  const int T = (N + 127) / 128, W = (T + 31) / 32;
#pragma omp parallel
  {
    int32_t* keys = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
    for (int r = 0; r < nrows; ++r) {
      const int64_t i = rows[r];
      const uint32_t* m = mask + ((int64_t)h * T + i / 128) * W;
      int nk = 0;
      for (int64_t j = 0; j <= i; ++j) {
        const int J = (int)(j / 128);
        if ((m[J >> 5] >> (J & 31)) & 1u) keys[nk++] = (int32_t)j;
      }
      softmax_row(&a, h, i, keys, nk, O + (int64_t)r * d, lse + r);
    }
    free(keys);
  }
}
