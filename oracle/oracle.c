/*
 * oracle.c - plain, slow, obviously correct CPU oracle of the MoE-layer
 * forward (router -> top-k gates -> dispatch layout -> experts -> combine).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header or constant with the CUDA library.
 *
 * Arithmetic: every floating-point input is widened exactly (bf16 -> float ->
 * double, or float -> double) and all sums run in double, in the natural
 * index order, with no blocking or reordering.  OpenMP only splits the outer
 * loop over tokens / rows; each output value is computed by one thread in a
 * fixed order, so results do not depend on the thread count.
 *
 * Sources (page title, then section / table):
 *  [MoE-Layout]   "MoE Pretraining: Parallelism Layout Changes the Model, Not
 *                 Quality": Methodology / Models and Data (16 SwiGLU experts,
 *                 top-4); Finding 3 (routing margin, near-ties).
 *  [Coupling]     "Expert Coupling in MoE Pretraining: Reducing All-to-All
 *                 Overhead with Correlated Placement and Token Shuffling":
 *                 Abstract (each token sent to each GPU once), Table I
 *                 (GPUs per token, deduplication; tokens split evenly
 *                 over the GPUs),
 *                 Table III (notation S_l(t), W[e,e']).
 *  [Revisiting]   "Revisiting MoE and Dense Speed-Accuracy Comparisons for
 *                 LLM Training": 2.1 Architecture (SwiGLU; Top-K routing),
 *                 Table 1 (router "ME", FFN1 "EMH", FFN2 "EHM" layouts).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_F32 0
#define OR_BF16 1

/* exact widening of one stored element */
static double ld(const void* p, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)((const float*)p)[i];
  uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * Router logits l[t,e] = sum_i x[t,i] * W_r[i,e] + bias[e]   ([Revisiting]
 * Table 1: router weights "ME" = [model, experts]).  tokens==NULL means all
 * T tokens; otherwise the n listed tokens, in that order.
 */
void oracle_router_logits(int64_t T, int32_t d, int32_t E, int32_t dtype,
                          const void* x, const void* w_r, const float* bias,
                          const int64_t* tokens, int64_t n, double* logits) {
  if (!tokens) n = T;
#pragma omp parallel for schedule(static)
  for (int64_t q = 0; q < n; ++q) {
    int64_t t = tokens ? tokens[q] : q;
    for (int32_t e = 0; e < E; ++e) {
      double s = 0.0;
      for (int32_t i = 0; i < d; ++i)
        s += ld(x, dtype, (size_t)t * d + i) * ld(w_r, dtype, (size_t)i * E + e);
      if (bias) s += (double)bias[e];
      logits[q * E + e] = s;
    }
  }
}

/* expert a beats expert b: larger logit, equal logits -> lower index.
 * (-0.0 == +0.0 under IEEE comparison, so they tie.) */
static int beats(double la, int a, double lb, int b) {
  return la > lb || (la == lb && a < b);
}

/*
 * Top-k with softmax gates over the k ([MoE-Layout] Models and Data: top-4
 * routing; [Revisiting] 2.1: Top-K routing).  The experts are ordered by the
 * key (logit desc, index asc) and the first k are taken, in that order:
 * repeated selection of the best not yet chosen expert.  Gates are the
 * softmax of the chosen k logits, g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0),
 * which equals the softmax over all E renormalised over the chosen k.
 */
void oracle_topk(int64_t n, int32_t E, int32_t k, const double* logits,
                 int32_t* idx, double* gate) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    const double* l = logits + t * E;
    char taken[1024];
    memset(taken, 0, (size_t)E);
    for (int32_t j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || beats(l[e], e, l[best], best))) best = e;
      taken[best] = 1;
      idx[t * k + j] = best;
    }
    double l0 = l[idx[t * k]];
    double z = 0.0;
    for (int32_t j = 0; j < k; ++j) z += exp(l[idx[t * k + j]] - l0);
    for (int32_t j = 0; j < k; ++j) gate[t * k + j] = exp(l[idx[t * k + j]] - l0) / z;
  }
}

/*
 * Routing margin ([MoE-Layout] Finding 3): the gap between the k-th and the
 * (k+1)-th largest scores of a token divided by the spread (max - min) of its
 * scores.  k == E has no unchosen expert: margin = +inf.  A zero spread (all
 * scores equal) gives margin 0.
 */
void oracle_margin(int64_t n, int32_t E, int32_t k, const double* logits, double* m) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    const double* l = logits + t * E;
    if (k >= E) { m[t] = INFINITY; continue; }
    /* k-th and (k+1)-th order statistics by counting */
    double mx = l[0], mn = l[0];
    for (int e = 1; e < E; ++e) { if (l[e] > mx) mx = l[e]; if (l[e] < mn) mn = l[e]; }
    double sk = 0, sk1 = 0;
    /* value v is the r-th largest (1-based) if #{> v} < r <= #{>= v} */
    for (int e = 0; e < E; ++e) {
      int gt = 0, ge = 0;
      for (int q = 0; q < E; ++q) { gt += l[q] > l[e]; ge += l[q] >= l[e]; }
      if (gt < k && k <= ge) sk = l[e];
      if (gt < k + 1 && k + 1 <= ge) sk1 = l[e];
    }
    double spread = mx - mn;
    m[t] = spread > 0 ? (sk - sk1) / spread : 0.0;
  }
}

/*
 * Expert-grouped dispatch layout and the deduplicated per-rank send layout.
 *
 *  counts[e]   = #assignments a = t*k+j with idx[a] == e
 *  offsets     = exclusive prefix sum of counts, offsets[E] = T*k
 *  rows of expert e hold its assignments in ascending flat index a (a stable
 *  counting sort): row_token[row] = t, slot_row[a] = row.
 *
 * Deduplicated send layout ([Coupling] Abstract: each token is sent to each
 * GPU once; Table I: "GPUs" = distinct destinations per token,
 * "Deduplication" = rows removed as duplicates):
 *  R(t) = the distinct ranks map[idx[t,j]]; one send row per (t, r in R(t)),
 *  grouped by rank ascending and, within a rank, by token ascending.
 *  rank_counts[r], rank_offsets (exclusive scan), send_token[row] = t,
 *  slot_send_row[a] = the send row of (t, map[idx[a]]).
 *  With ep == 1 there is no dispatch: the send layout is not built (its
 *  arrays are left untouched and may be NULL).
 *
 * stats[0] rows_sent          = sum_t |R(t)|           (0 when ep == 1)
 * stats[1] dup_removed        = T*k - rows_sent        (0 when ep == 1)
 * stats[2] tokens_single_rank = #t with |R(t)| == 1
 * stats[3] home_rank_rows     = #a with map[idx[a]] == home(t),
 *                               home(t) = floor(t*ep/T) ([Coupling] Table I:
 *                               tokens split evenly over the GPUs)
 * stats[4] max expert count, stats[5] min expert count.
 *
 * Returns 0, or -1 if an index is out of range.
 */
int oracle_dispatch_layout(int64_t T, int32_t E, int32_t k, int32_t ep,
                           const int32_t* idx, const int32_t* map,
                           int32_t* counts, int32_t* offsets,
                           int32_t* row_token, int32_t* slot_row,
                           int32_t* rank_counts, int32_t* rank_offsets,
                           int32_t* send_token, int32_t* slot_send_row,
                           int64_t* stats) {
  int64_t R = T * k;
  for (int64_t a = 0; a < R; ++a)
    if (idx[a] < 0 || idx[a] >= E) return -1;
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < R; ++a) counts[idx[a]]++;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > ep ? E : ep));
  for (int32_t e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int64_t a = 0; a < R; ++a) {
    int32_t row = cursor[idx[a]]++;
    row_token[row] = (int32_t)(a / k);
    slot_row[a] = row;
  }
  int32_t mx = 0, mn = (int32_t)R;
  for (int32_t e = 0; e < E; ++e) {
    if (counts[e] > mx) mx = counts[e];
    if (counts[e] < mn) mn = counts[e];
  }
  if (E == 0) mn = 0;
  int64_t rows_sent = 0, single = 0, home_rows = 0;
  /* distinct ranks of each token, as a sorted list */
  int32_t rs[256];
  for (int64_t t = 0; t < T; ++t) {
    int nr = 0;
    int64_t home = (t * ep) / (T > 0 ? T : 1);
    for (int32_t j = 0; j < k; ++j) {
      int32_t r = map[idx[t * k + j]];
      if (r == home) home_rows++;
      int seen = 0;
      for (int q = 0; q < nr; ++q) seen |= rs[q] == r;
      if (!seen) rs[nr++] = r;
    }
    rows_sent += nr;
    single += nr == 1;
  }
  if (ep > 1) {
    for (int32_t r = 0; r < ep; ++r) rank_counts[r] = 0;
    for (int64_t t = 0; t < T; ++t) {
      /* one row per distinct rank of t */
      for (int32_t r = 0; r < ep; ++r) {
        int hit = 0;
        for (int32_t j = 0; j < k; ++j) hit |= map[idx[t * k + j]] == r;
        rank_counts[r] += hit;
      }
    }
    rank_offsets[0] = 0;
    for (int32_t r = 0; r < ep; ++r) rank_offsets[r + 1] = rank_offsets[r] + rank_counts[r];
    for (int32_t r = 0; r < ep; ++r) cursor[r] = rank_offsets[r];
    for (int64_t t = 0; t < T; ++t) {
      for (int32_t r = 0; r < ep; ++r) {
        int hit = 0;
        for (int32_t j = 0; j < k; ++j) hit |= map[idx[t * k + j]] == r;
        if (!hit) continue;
        int32_t srow = cursor[r]++;
        send_token[srow] = (int32_t)t;
        for (int32_t j = 0; j < k; ++j)
          if (map[idx[t * k + j]] == r) slot_send_row[t * k + j] = srow;
      }
    }
    stats[0] = rows_sent;
    stats[1] = R - rows_sent;
  } else {
    stats[0] = 0;
    stats[1] = 0;
  }
  stats[2] = single;
  stats[3] = home_rows;
  stats[4] = mx;
  stats[5] = mn;
  free(cursor);
  return 0;
}

/*
 * One SwiGLU expert on one input row ([Revisiting] 2.1 Architecture: SwiGLU;
 * [MoE-Layout] Models and Data: SwiGLU experts):
 *   a = x W_g[e], b = x W_u[e]  (W_g, W_u [E,d,f], "EMH")
 *   h = silu(a) * b = a / (1 + exp(-a)) * b      (no intermediate rounding)
 *   out = h W_d[e]              (W_d [E,f,d], "EHM")
 * xrow: d doubles.  out: d doubles.  scratch: 3*f doubles.
 */
static void swiglu_expert(int32_t d, int32_t f, int32_t dtype, int32_t e,
                          const double* xrow, const void* w_g, const void* w_u,
                          const void* w_d, double* out, double* scratch) {
  double* a = scratch;
  double* b = scratch + f;
  double* h = scratch + 2 * (size_t)f;
  size_t base_gu = (size_t)e * d * f;
  for (int32_t i = 0; i < f; ++i) { a[i] = 0.0; b[i] = 0.0; }
  for (int32_t c = 0; c < d; ++c) {
    double xc = xrow[c];
    for (int32_t i = 0; i < f; ++i) {
      a[i] += xc * ld(w_g, dtype, base_gu + (size_t)c * f + i);
      b[i] += xc * ld(w_u, dtype, base_gu + (size_t)c * f + i);
    }
  }
  for (int32_t i = 0; i < f; ++i) h[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
  size_t base_d = (size_t)e * f * d;
  for (int32_t o = 0; o < d; ++o) out[o] = 0.0;
  for (int32_t i = 0; i < f; ++i) {
    double hi = h[i];
    for (int32_t o = 0; o < d; ++o) out[o] += hi * ld(w_d, dtype, base_d + (size_t)i * d + o);
  }
}

/*
 * Grouped experts over a permuted activation matrix: row r of x_perm belongs
 * to the expert e with offsets[e] <= r < offsets[e+1]; y_perm[r] = expert_e(
 * x_perm[r]).  rows==NULL: all offsets[E] rows; else the n listed rows.
 */
void oracle_grouped_swiglu(int32_t d, int32_t E, int32_t f, int32_t dtype,
                           const void* x_perm, const int32_t* offsets,
                           const void* w_g, const void* w_u, const void* w_d,
                           const int64_t* rows, int64_t n, double* y_perm) {
  if (!rows) n = offsets[E];
#pragma omp parallel
  {
    double* xr = (double*)malloc(sizeof(double) * ((size_t)d + 3 * (size_t)f));
    double* sc = xr + d;
#pragma omp for schedule(dynamic, 16)
    for (int64_t q = 0; q < n; ++q) {
      int64_t r = rows ? rows[q] : q;
      int32_t e = 0;
      while (e < E && offsets[e + 1] <= r) ++e;
      for (int32_t c = 0; c < d; ++c) xr[c] = ld(x_perm, dtype, (size_t)r * d + c);
      swiglu_expert(d, f, dtype, e, xr, w_g, w_u, w_d, y_perm + q * (size_t)d, sc);
    }
    free(xr);
  }
}

/*
 * Gate-weighted combine: y[t] = sum_{j<k} gate[t,j] * y_perm[slot_row[t*k+j]],
 * j ascending, in double.  y_perm is typed (dtype) when y_perm_d is NULL, else
 * y_perm_d (double) is used.  gate==NULL means unit gates.
 */
void oracle_combine(int64_t T, int32_t d, int32_t k, int32_t dtype,
                    const void* y_perm, const double* y_perm_d,
                    const int32_t* slot_row, const double* gate, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t c = 0; c < d; ++c) {
      double s = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        size_t src = (size_t)slot_row[t * k + j] * d + c;
        double v = y_perm_d ? y_perm_d[src] : ld(y_perm, dtype, src);
        s += (gate ? gate[t * k + j] : 1.0) * v;
      }
      y[t * (size_t)d + c] = s;
    }
  }
}

/*
 * Layer output of listed tokens given their routing (idx, gate), straight
 * from the definition: y[t] = sum_j gate[t,j] * expert_{idx[t,j]}(x[t]).
 * The dispatch permutation is a pure data movement and does not appear.
 * tokens==NULL: all T tokens.  idx/gate are indexed by position q in the
 * token list (n rows of k).
 */
void oracle_moe_output(int64_t T, int32_t d, int32_t k, int32_t f, int32_t dtype,
                       const void* x, const int32_t* idx, const double* gate,
                       const void* w_g, const void* w_u, const void* w_d,
                       const int64_t* tokens, int64_t n, double* y) {
  if (!tokens) n = T;
#pragma omp parallel
  {
    double* xr = (double*)malloc(sizeof(double) * (2 * (size_t)d + 3 * (size_t)f));
    double* out = xr + d;
    double* sc = out + d;
#pragma omp for schedule(dynamic, 4)
    for (int64_t q = 0; q < n; ++q) {
      int64_t t = tokens ? tokens[q] : q;
      for (int32_t c = 0; c < d; ++c) xr[c] = ld(x, dtype, (size_t)t * d + c);
      double* yq = y + q * (size_t)d;
      for (int32_t c = 0; c < d; ++c) yq[c] = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        swiglu_expert(d, f, dtype, idx[q * k + j], xr, w_g, w_u, w_d, out, sc);
        double g = gate[q * k + j];
        for (int32_t c = 0; c < d; ++c) yq[c] += g * out[c];
      }
    }
    free(xr);
  }
}

/* number of threads OpenMP uses for the parallel loops above */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
