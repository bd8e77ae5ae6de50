/*
 * HSTU jagged pointwise attention: plain, slow fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the bench's CPU
 * baseline leg load this library.  It shares no code, header, table or helper
 * with the CUDA library; the two only ever see the same seeded inputs.
 *
 * What it computes (plain definition, no tiling, no skipping, no reordering):
 *
 *   For a user u with n tokens of which the last c are candidates (h = n - c):
 *     position        p(i) = min(i, h)
 *     allowed set     M(i,j) = (j <= i)              if i <  h   (causal history)
 *                              (j <  h) or (j == i)  if i >= h   (M-FALCON candidate)
 *     time bucket     b(i,j) = clamp(floor(ln(|t_i - t_j| + 1) / 0.301), 0, NB-1)
 *     score           s(i,j) = alpha * <q_i, k_j> + rab_pos[p(i) - p(j) + N_max - 1] + rab_ts[b(i,j)]
 *     weight          a(i,j) = SiLU(s(i,j)) / N_max  on M(i,j), else 0;  SiLU(x) = x / (1 + e^-x)
 *     per head        o_i = sum_j a(i,j) v_j
 *     output          y_i = ((o_i - mean) / sqrt(var + eps) * gamma + beta) * u_i
 *                     (mean and biased var over the H*d concatenated head features)
 *
 * Sources: "Generative Recommenders at Scale" (Inside NVIDIA's GPU-native stack; FAQ):
 * HSTU replaces softmax by SiLU weighting with relative attention bias and
 * elementwise gating.  "How Generative Recommenders Are Redefining RecSys at
 * Scale" (Summary; Takeaways): timestamp-ordered interleaved items and actions,
 * gating applied before the output projection.  "HSTU Generative Recommenders:
 * Deploy on GPU Cloud" (M-FALCON: Microbatched Attention ...): candidates are
 * scored in one pass with the mask and relative bias modified so they share
 * the history computation.  The formula itself, the bucket rule and the
 * normalisation by N_max come from the problem statement these pages are read
 * with; readings of the points the pages leave open are:
 *   - candidates all sit at position h (p(i) = min(i, h));
 *   - the mask is applied after SiLU (masked pairs contribute exactly 0);
 *   - 0.301 is the decimal 0.301; the bucket uses |dt|;
 *   - LayerNorm is over the H*d features, biased variance, gamma=1/beta=0 if absent.
 *
 * The time bucket is evaluated in binary128 (libquadmath): floor(logq(x)/0.301Q)
 * is exact for every integer x <= 2^63 because every bucket edge e^(0.301 b),
 * b = 1..127, is at least 0.0045 away from the nearest integer, i.e. more than
 * 1e-19 relative, far above binary128's 1e-34 rounding (the tests check the
 * edges and the buckets against an exact 60-digit decimal evaluation).
 */
#include <math.h>
#include <quadmath.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)

/* ---- time bucket ------------------------------------------------------- */

int32_t oracle_ts_bucket(int64_t dt, int32_t num_buckets) {
  /* |dt| without overflow for INT64_MIN */
  uint64_t mag = dt < 0 ? (uint64_t)0 - (uint64_t)dt : (uint64_t)dt;
  __float128 x = (__float128)mag + 1.0Q;
  __float128 b = floorq(logq(x) / 0.301Q);
  if (b < 0) b = 0;
  if (b > (__float128)(num_buckets - 1)) b = (__float128)(num_buckets - 1);
  return (int32_t)b;
}

void oracle_ts_bucket_array(const int64_t* dt, int64_t n, int32_t num_buckets, int32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_ts_bucket(dt[i], num_buckets);
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

/* ---- one user's sequence ------------------------------------------------ */

/* A view of one user's full sequence: token j's key/value for head h are at
 * key(j,h) / val(j,h).  In the jagged case all tokens are rows of q/k/v; in
 * the paged case the first `cached` tokens come from the page pool. */
typedef struct {
  int64_t n;          /* tokens in the sequence                          */
  int64_t hist;       /* n - candidates                                  */
  int64_t cached;     /* paged prefix length (0 when not paged)          */
  const int64_t* ts;  /* [n] timestamps                                  */
  /* jagged rows of the new (or all) tokens: row of token j is row0 + j - cached */
  const double* k;
  const double* v;
  int64_t row0;
  /* paged prefix */
  const double* k_pool;
  const double* v_pool;
  const int32_t* page_row; /* this user's page-table row */
  int32_t page_size;
} seq_view;

typedef struct {
  int32_t H, d, n_max, nb;
  double alpha;
  const double* rab_pos;
  const double* rab_ts;
} attn_cfg;

static const double* key_at(const seq_view* s, const attn_cfg* c, int64_t j, int h) {
  if (j < s->cached) {
    int64_t page = s->page_row[j / s->page_size];
    int64_t slot = j % s->page_size;
    return s->k_pool + (((page * c->H + h) * (int64_t)s->page_size + slot) * c->d);
  }
  return s->k + ((s->row0 + j - s->cached) * c->H + h) * (int64_t)c->d;
}

static const double* val_at(const seq_view* s, const attn_cfg* c, int64_t j, int h) {
  if (j < s->cached) {
    int64_t page = s->page_row[j / s->page_size];
    int64_t slot = j % s->page_size;
    return s->v_pool + (((page * c->H + h) * (int64_t)s->page_size + slot) * c->d);
  }
  return s->v + ((s->row0 + j - s->cached) * c->H + h) * (int64_t)c->d;
}

static int allowed(int64_t i, int64_t j, int64_t hist) {
  if (i < hist) return j <= i;
  return j < hist || j == i;
}

static int64_t position(int64_t i, int64_t hist) { return i < hist ? i : hist; }

/* o (length d) = sum_j a(i,j) v_j for query token i of the sequence, head h. */
static void attend(const seq_view* s, const attn_cfg* c, const double* qi, int64_t i, int h,
                   double* o) {
  for (int e = 0; e < c->d; ++e) o[e] = 0.0;
  for (int64_t j = 0; j < s->n; ++j) {
    if (!allowed(i, j, s->hist)) continue;
    const double* kj = key_at(s, c, j, h);
    double dot = 0.0;
    for (int e = 0; e < c->d; ++e) dot += qi[e] * kj[e];
    int64_t rel = position(i, s->hist) - position(j, s->hist);
    double score = c->alpha * dot + c->rab_pos[rel + c->n_max - 1] +
                   c->rab_ts[oracle_ts_bucket(s->ts[i] - s->ts[j], c->nb)];
    double a = silu(score) / (double)c->n_max;
    const double* vj = val_at(s, c, j, h);
    for (int e = 0; e < c->d; ++e) o[e] += a * vj[e];
  }
}

/* y = ((o - mean)/sqrt(var + eps) * gamma + beta) * u over D features */
static void layer_norm_gate(const double* o, const double* u, const double* gamma,
                            const double* beta, double eps, int D, double* y) {
  double mean = 0.0;
  for (int e = 0; e < D; ++e) mean += o[e];
  mean /= D;
  double var = 0.0;
  for (int e = 0; e < D; ++e) var += (o[e] - mean) * (o[e] - mean);
  var /= D;
  double rstd = 1.0 / sqrt(var + eps);
  for (int e = 0; e < D; ++e) {
    double g = gamma ? gamma[e] : 1.0;
    double b = beta ? beta[e] : 0.0;
    y[e] = ((o[e] - mean) * rstd * g + b) * u[e];
  }
}

static int check_cfg(int32_t H, int32_t d, int32_t n_max, int32_t nb) {
  return (H > 0 && d > 0 && n_max > 0 && nb > 0) ? ORACLE_OK : ORACLE_BAD_ARG;
}

/* Find the user of jagged row `row` (linear scan: plain and obviously right). */
static int64_t user_of(const int32_t* offsets, int32_t B, int64_t row) {
  for (int32_t b = 0; b < B; ++b)
    if (row >= offsets[b] && row < offsets[b + 1]) return b;
  return -1;
}

/*
 * Jagged attention over whole users, or over a subset of rows.
 *   q,k,v [T,H,d]; u [T,H*d]; seq_offsets [B+1]; timestamps [T];
 *   num_candidates [B] or NULL; rab_pos [2*n_max-1]; rab_ts [nb];
 *   gamma/beta [H*d] or NULL.
 *   rows: NULL = every row 0..T-1, else `nrows` row indices; outputs are
 *   written in that order: o_out [nrows,H,d] (may be NULL), y_out [nrows,H*d].
 * Returns 0, or -1 on a bad argument (lengths above n_max, bad offsets).
 */
int oracle_attn_jagged(const double* q, const double* k, const double* v, const double* u,
                       const int32_t* seq_offsets, int32_t B, const int64_t* timestamps,
                       const int32_t* num_candidates, const double* rab_pos,
                       const double* rab_ts, int32_t nb, double alpha, int32_t n_max,
                       int32_t H, int32_t d, const double* gamma, const double* beta,
                       double eps, const int64_t* rows, int64_t nrows, double* o_out,
                       double* y_out) {
  if (check_cfg(H, d, n_max, nb) != ORACLE_OK || seq_offsets[0] != 0) return ORACLE_BAD_ARG;
  for (int32_t b = 0; b < B; ++b) {
    int64_t n = (int64_t)seq_offsets[b + 1] - seq_offsets[b];
    int64_t cnd = num_candidates ? num_candidates[b] : 0;
    if (n < 0 || n > n_max || cnd < 0 || cnd > n) return ORACLE_BAD_ARG;
  }
  int64_t T = seq_offsets[B];
  if (!rows) nrows = T;
  attn_cfg cfg = {H, d, n_max, nb, alpha, rab_pos, rab_ts};
  const int D = H * d;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t row = rows ? rows[r] : r;
    int64_t b = user_of(seq_offsets, B, row);
    if (b < 0) { bad = 1; continue; }
    seq_view s;
    memset(&s, 0, sizeof s);
    s.n = (int64_t)seq_offsets[b + 1] - seq_offsets[b];
    s.hist = s.n - (num_candidates ? num_candidates[b] : 0);
    s.ts = timestamps + seq_offsets[b];
    s.k = k;
    s.v = v;
    s.row0 = seq_offsets[b];
    int64_t i = row - seq_offsets[b];
    double* o = (double*)malloc(sizeof(double) * D);
    for (int h = 0; h < H; ++h) attend(&s, &cfg, q + (row * H + h) * (int64_t)d, i, h, o + h * d);
    if (o_out) memcpy(o_out + r * D, o, sizeof(double) * D);
    layer_norm_gate(o, u + row * (int64_t)D, gamma, beta, eps, D, y_out + r * D);
    free(o);
  }
  return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/*
 * Incremental attention: new tokens of each user attend to a cached prefix
 * held in a paged pool plus to the new tokens themselves; the result is the
 * full-recompute result for the new tokens.
 *   q,k,v [T_new,H,d]; u [T_new,H*d]; new_offsets [B+1];
 *   timestamps: jagged over prefix+new tokens by ts_offsets [B+1];
 *   num_candidates [B]: the last new tokens of a user are candidates;
 *   k_pool, v_pool [num_pages,H,page_size,d]; page_table [B,max_pages];
 *   cached_lens [B].  rows: NULL = every new row, else a subset of new rows.
 */
int oracle_attn_paged(const double* q, const double* k, const double* v, const double* u,
                      const int32_t* new_offsets, int32_t B, const int64_t* timestamps,
                      const int32_t* ts_offsets, const int32_t* num_candidates,
                      const double* rab_pos, const double* rab_ts, int32_t nb, double alpha,
                      int32_t n_max, int32_t H, int32_t d, const double* gamma,
                      const double* beta, double eps, const double* k_pool,
                      const double* v_pool, const int32_t* page_table, int32_t max_pages,
                      int32_t page_size, const int32_t* cached_lens, const int64_t* rows,
                      int64_t nrows, double* o_out, double* y_out) {
  if (check_cfg(H, d, n_max, nb) != ORACLE_OK || page_size <= 0) return ORACLE_BAD_ARG;
  for (int32_t b = 0; b < B; ++b) {
    int64_t nn = (int64_t)new_offsets[b + 1] - new_offsets[b];
    int64_t n = cached_lens[b] + nn;
    int64_t cnd = num_candidates ? num_candidates[b] : 0;
    if (nn < 0 || n > n_max || cnd < 0 || cnd > nn) return ORACLE_BAD_ARG;
    if ((int64_t)ts_offsets[b + 1] - ts_offsets[b] != n) return ORACLE_BAD_ARG;
    if ((cached_lens[b] + page_size - 1) / page_size > max_pages) return ORACLE_BAD_ARG;
  }
  int64_t T = new_offsets[B];
  if (!rows) nrows = T;
  attn_cfg cfg = {H, d, n_max, nb, alpha, rab_pos, rab_ts};
  const int D = H * d;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t row = rows ? rows[r] : r;
    int64_t b = user_of(new_offsets, B, row);
    if (b < 0) { bad = 1; continue; }
    seq_view s;
    s.cached = cached_lens[b];
    s.n = s.cached + ((int64_t)new_offsets[b + 1] - new_offsets[b]);
    s.hist = s.n - (num_candidates ? num_candidates[b] : 0);
    s.ts = timestamps + ts_offsets[b];
    s.k = k;
    s.v = v;
    s.row0 = new_offsets[b];
    s.k_pool = k_pool;
    s.v_pool = v_pool;
    s.page_row = page_table + (int64_t)b * max_pages;
    s.page_size = page_size;
    int64_t i = s.cached + (row - new_offsets[b]);
    double* o = (double*)malloc(sizeof(double) * D);
    for (int h = 0; h < H; ++h) attend(&s, &cfg, q + (row * H + h) * (int64_t)d, i, h, o + h * d);
    if (o_out) memcpy(o_out + r * D, o, sizeof(double) * D);
    layer_norm_gate(o, u + row * (int64_t)D, gamma, beta, eps, D, y_out + r * D);
    free(o);
  }
  return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

/* Number of allowed (i,j) pairs per head: the algorithmic work unit. */
int64_t oracle_allowed_pairs(const int32_t* seq_offsets, int32_t B, const int32_t* num_candidates) {
  int64_t total = 0;
  for (int32_t b = 0; b < B; ++b) {
    int64_t n = (int64_t)seq_offsets[b + 1] - seq_offsets[b];
    int64_t hist = n - (num_candidates ? num_candidates[b] : 0);
    for (int64_t i = 0; i < n; ++i)
      for (int64_t j = 0; j < n; ++j) total += allowed(i, j, hist);
  }
  return total;
}
