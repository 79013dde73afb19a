/*
 * beam_oracle.c -- plain, slow fp64 CPU oracle of the Beam 1.0 attention core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this library.  It shares no code with the CUDA path and
 * includes none of its headers.
 *
 * Source: "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax"
 * (flozi.net, English page; the German page is its twin).  Each function
 * names the section it follows.  The page's display equations did not survive
 * extraction, so the attention and gate formulas are rebuilt from its prose;
 * the readings taken are listed beside each function.
 *
 * Everything is double precision.  Inputs arrive as bf16 bit patterns (exactly
 * representable in double) or float32 weights (also exact).  No intermediate is
 * rounded.  Work is spread over POSIX threads by whole output rows; each row is
 * computed by the same sequential loops, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t n_q_heads;   /* 48 */
  int32_t n_kv_heads;  /* 8 */
  int32_t head_dim;    /* 128 */
  int32_t window;      /* 512: keys t-window+1 .. t are visible in a local layer */
  double rope_theta;   /* 10000 */
  double rms_eps;      /* 1e-6 */
  double ssmax_base;   /* 2048 */
  double ssmax_exp;    /* 0.1 */
  double softmax_scale;/* 1/sqrt(128) */
} oracle_params;

enum { ORACLE_LOCAL = 0, ORACLE_GLOBAL = 1 };

/* FP8 E4M3 codes (defined with the FP8 cache functions below) */
double oracle_e4m3_decode(uint8_t code);
uint8_t oracle_e4m3_encode(double x);

/* ---------------------------------------------------------------- scalars */

double oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Nearest bf16 (ties to even) of a double, via the nearest float first is NOT
 * used: the double is rounded once, directly, to 8 significand bits. */
uint16_t oracle_double_to_bf16(double x) {
  if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
  int e;
  double m = frexp(fabs(x), &e);          /* |x| = m * 2^e, m in [0.5, 1) */
  double scaled = ldexp(m, 8);            /* 8 significand bits incl. the leading one */
  double r = nearbyint(scaled);           /* default rounding: to nearest, ties to even */
  double y = ldexp(r, e - 8);
  float f = (float)y;                     /* exact: y has 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t b = (uint16_t)(u >> 16);
  if (signbit(x)) b |= 0x8000u;
  return b;
}

/* Scalable-softmax query factor a(p) = (1 + p/2048)^0.1, p = t + 1 the
 * one-based absolute query position (section "Follow the tensors": only Q of a
 * global layer receives a(p); section "What scalable softmax changes
 * mathematically" prints a at 2,048 / 65,536 / 1,048,576). */
double oracle_ssmax_factor(int64_t p, double base, double expo) {
  return pow(1.0 + (double)p / base, expo);
}

double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------- vector ops */

/* RMSNorm along the head axis (section "Follow the tensors": Q and K are
 * normalised along their 128-coordinate head axis with epsilon 1e-6; V is
 * not).  Reading: the learned weight multiplies directly (y = x/rms * w). */
void oracle_rms_norm(const double *x, const double *w, int d, double eps, double *y) {
  double ss = 0.0;
  for (int i = 0; i < d; ++i) ss += x[i] * x[i];
  double inv_rms = 1.0 / sqrt(ss / (double)d + eps);
  for (int i = 0; i < d; ++i) y[i] = x[i] * inv_rms * w[i];
}

/* RoPE of a local layer (section "Follow the tensors": RoPE rotates the
 * normalised Q and K).  The page gives neither theta nor the convention; the
 * reading taken is theta = 10000 and the rotate-half pairing of coordinate i
 * with i + d/2, frequency theta^(-2i/d), angle t * frequency with t the 0-based
 * position.  The angle is formed in double; cos and sin take it unreduced. */
void oracle_rope(double *x, int d, int64_t t, double theta) {
  int half = d / 2;
  for (int i = 0; i < half; ++i) {
    double freq = pow(theta, -2.0 * (double)i / (double)d);
    double phi = (double)t * freq;
    double c = cos(phi), s = sin(phi);
    double a = x[i], b = x[i + half];
    x[i] = a * c - b * s;
    x[i + half] = b * c + a * s;
  }
}

/* Softmax over n scores: prob_j = exp(s_j - max) / sum_k exp(s_k - max). */
void oracle_softmax(const double *s, int64_t n, double *prob) {
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) if (s[j] > m) m = s[j];
  double z = 0.0;
  for (int64_t j = 0; j < n; ++j) { prob[j] = exp(s[j] - m); z += prob[j]; }
  for (int64_t j = 0; j < n; ++j) prob[j] /= z;
}

/* Visibility of key position j to query position t (sections "Two attention
 * paths in one decoder" and "Follow the tensors"): a local layer sees the
 * current token and the window-1 before it; a global layer sees every j <= t. */
int oracle_visible(int kind, int64_t t, int64_t j, int64_t window) {
  if (j > t || j < 0) return 0;
  if (kind == ORACLE_LOCAL) return t - j <= window - 1;
  return 1;
}

/* Cache slot of position j: a global cache appends (slot j); a local ring of
 * `slots` entries reuses slot j mod slots. */
int64_t oracle_cache_slot(int kind, int64_t j, int64_t slots) {
  return kind == ORACLE_LOCAL ? j % slots : j;
}

/* Query of one head after normalisation and the layer's position operation:
 * local -> RoPE at t; global -> no rotation, times a(t+1). */
static void prepare_query(int kind, const oracle_params *P, const uint16_t *q_raw,
                          const double *w, int64_t t, double *out) {
  int d = P->head_dim;
  double *x = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) x[i] = oracle_bf16_to_double(q_raw[i]);
  oracle_rms_norm(x, w, d, P->rms_eps, out);
  if (kind == ORACLE_LOCAL) {
    oracle_rope(out, d, t, P->rope_theta);
  } else {
    double a = oracle_ssmax_factor(t + 1, P->ssmax_base, P->ssmax_exp);
    for (int i = 0; i < d; ++i) out[i] *= a;
  }
  free(x);
}

/* Key after normalisation: local -> RoPE at its own position j; global -> K
 * stays unrotated and unscaled. */
static void prepare_key(int kind, const oracle_params *P, const uint16_t *k_raw,
                        const double *w, int64_t j, double *out) {
  int d = P->head_dim;
  double *x = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) x[i] = oracle_bf16_to_double(k_raw[i]);
  oracle_rms_norm(x, w, d, P->rms_eps, out);
  if (kind == ORACLE_LOCAL) oracle_rope(out, d, j, P->rope_theta);
  free(x);
}

/* Exported so tests can pin the two position operations in isolation. */
void oracle_prepare_query(int kind, const oracle_params *P, const uint16_t *q_raw,
                          const float *w32, int64_t t, double *out) {
  double *w = (double *)malloc(sizeof(double) * P->head_dim);
  for (int i = 0; i < P->head_dim; ++i) w[i] = (double)w32[i];
  prepare_query(kind, P, q_raw, w, t, out);
  free(w);
}

void oracle_prepare_key(int kind, const oracle_params *P, const uint16_t *k_raw,
                        const float *w32, int64_t j, double *out) {
  double *w = (double *)malloc(sizeof(double) * P->head_dim);
  for (int i = 0; i < P->head_dim; ++i) w[i] = (double)w32[i];
  prepare_key(kind, P, k_raw, w, j, out);
  free(w);
}

/* Row accessor: writes key row j and value row j (d doubles each) of the
 * visible sequence, j = 0 .. n-1. */
typedef void (*row_fn)(const void *ctx, int64_t j, double *k_row, double *v_row);

/* One gated attention output for one query head (section "Follow the
 * tensors"): s_j = scale * <q~, k^_j> over the n visible keys, P = softmax(s),
 * O = sum_j P_j v_j, then Y_c = O_c * sigmoid(G_c + b_h): the gate acts on every
 * coordinate, the bias is one value per head.  Rows are fetched through `row`
 * twice (once for the scores, once for the weighted sum) so that long
 * contexts need no copy of the cache. */
static void attend_one(const oracle_params *P, const double *q, int64_t n, row_fn row,
                       const void *rctx, const uint16_t *gate_raw, double bias,
                       double *scores, double *y) {
  int d = P->head_dim;
  double *kr = (double *)malloc(sizeof(double) * 2 * d), *vr = kr + d;
  for (int64_t j = 0; j < n; ++j) {
    row(rctx, j, kr, vr);
    double dot = 0.0;
    for (int i = 0; i < d; ++i) dot += q[i] * kr[i];
    scores[j] = P->softmax_scale * dot;
  }
  oracle_softmax(scores, n, scores);
  for (int i = 0; i < d; ++i) y[i] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    row(rctx, j, kr, vr);
    for (int i = 0; i < d; ++i) y[i] += scores[j] * vr[i];
  }
  for (int i = 0; i < d; ++i)
    y[i] *= oracle_sigmoid(oracle_bf16_to_double(gate_raw[i]) + bias);
  free(kr);
}

/* ------------------------------------------------------------ threading */

typedef void (*job_fn)(void *ctx, int64_t item);
typedef struct { job_fn fn; void *ctx; int64_t n_items; int64_t next; pthread_mutex_t mu; } pool_t;

static void *pool_worker(void *arg) {
  pool_t *p = (pool_t *)arg;
  for (;;) {
    pthread_mutex_lock(&p->mu);
    int64_t item = p->next++;
    pthread_mutex_unlock(&p->mu);
    if (item >= p->n_items) return NULL;
    p->fn(p->ctx, item);
  }
}

static void run_parallel(job_fn fn, void *ctx, int64_t n_items, int n_threads) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  pool_t p;
  p.fn = fn; p.ctx = ctx; p.n_items = n_items; p.next = 0;
  pthread_mutex_init(&p.mu, NULL);
  pthread_t th[256];
  for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
  for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&p.mu);
}

/* --------------------------------------------------------------- prefill */

/* Prefill of one layer for B sequences of T tokens at positions 0..T-1.
 * Inputs are the post-projection tensors, token-major:
 *   q, gate [B][T][Hq][d]; k, v [B][T][Hkv][d] (bf16 bits);
 *   q_norm_w, k_norm_w [d] and gate_bias [Hq] (float32).
 * Only the listed rows (b = rows_b[r], t = rows_t[r]) are computed; out is
 * [n_rows][Hq][d] doubles.  Query head h reads KV head h / (Hq/Hkv)
 * (section "Follow the tensors": six query heads share each KV head). */
typedef struct {
  int kind;
  const oracle_params *P;
  int B, T;
  const uint16_t *q, *k, *v, *gate;
  const double *qw, *kw;
  const float *bias;
  const int64_t *rows_b, *rows_t;
  const int64_t *rows_h;   /* oracle_prefill_row_heads: the one query head of each item */
  double *out;
  double **khat;   /* per sequence: [T][Hkv][d] prepared keys (NULL if unused) */
  double **vd;     /* per sequence: [T][Hkv][d] values as doubles */
  int64_t key_b;   /* sequence whose keys prefill_key_job prepares */
} prefill_ctx;

static void prefill_key_job(void *vctx, int64_t j) {
  prefill_ctx *c = (prefill_ctx *)vctx;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hkv = P->n_kv_heads;
  int64_t b = c->key_b;
  for (int g = 0; g < Hkv; ++g) {
    size_t in_off = (((size_t)b * c->T + j) * Hkv + g) * d;
    size_t out_off = ((size_t)j * Hkv + g) * d;
    prepare_key(c->kind, P, c->k + in_off, c->kw, j, c->khat[b] + out_off);
    for (int i = 0; i < d; ++i) c->vd[b][out_off + i] = oracle_bf16_to_double(c->v[in_off + i]);
  }
}

typedef struct { const double *k0, *v0; int64_t row_stride; int d; } kv_view;

static void kv_view_row(const void *vctx, int64_t j, double *k_row, double *v_row) {
  const kv_view *r = (const kv_view *)vctx;
  memcpy(k_row, r->k0 + (size_t)j * r->row_stride, sizeof(double) * r->d);
  memcpy(v_row, r->v0 + (size_t)j * r->row_stride, sizeof(double) * r->d);
}

static void prefill_row_job(void *vctx, int64_t r) {
  prefill_ctx *c = (prefill_ctx *)vctx;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hq = P->n_q_heads, Hkv = P->n_kv_heads, G = Hq / Hkv;
  int64_t b = c->rows_b[r], t = c->rows_t[r];
  int64_t lo = 0;
  while (!oracle_visible(c->kind, t, lo, P->window)) ++lo;  /* first visible key */
  int64_t n = t - lo + 1;
  double *q = (double *)malloc(sizeof(double) * d);
  double *scores = (double *)malloc(sizeof(double) * n);
  for (int h = 0; h < Hq; ++h) {
    int g = h / G;
    kv_view view = {c->khat[b] + ((size_t)lo * Hkv + g) * d, c->vd[b] + ((size_t)lo * Hkv + g) * d,
                    (int64_t)Hkv * d, d};
    size_t q_off = (((size_t)b * c->T + t) * Hq + h) * d;
    prepare_query(c->kind, P, c->q + q_off, c->qw, t, q);
    attend_one(P, q, n, kv_view_row, &view, c->gate + q_off, (double)c->bias[h], scores,
               c->out + ((size_t)r * Hq + h) * d);
  }
  free(q); free(scores);
}

int oracle_prefill_rows(int kind, const oracle_params *P, int B, int T,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const uint16_t *gate, const float *q_norm_w, const float *k_norm_w,
                        const float *gate_bias, int64_t n_rows, const int64_t *rows_b,
                        const int64_t *rows_t, double *out, int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows_b[r] < 0 || rows_b[r] >= B || rows_t[r] < 0 || rows_t[r] >= T) return -1;
  int d = P->head_dim, Hkv = P->n_kv_heads;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  prefill_ctx c;
  memset(&c, 0, sizeof c);
  c.kind = kind; c.P = P; c.B = B; c.T = T;
  c.q = q; c.k = k; c.v = v; c.gate = gate; c.qw = qw; c.kw = kw; c.bias = gate_bias;
  c.rows_b = rows_b; c.rows_t = rows_t; c.out = out;
  c.khat = (double **)calloc(B, sizeof(double *));
  c.vd = (double **)calloc(B, sizeof(double *));
  for (int b = 0; b < B; ++b) {
    int used = 0;
    for (int64_t r = 0; r < n_rows && !used; ++r) used = rows_b[r] == b;
    if (!used) continue;
    c.khat[b] = (double *)malloc(sizeof(double) * (size_t)T * Hkv * d);
    c.vd[b] = (double *)malloc(sizeof(double) * (size_t)T * Hkv * d);
    c.key_b = b;
    run_parallel(prefill_key_job, &c, T, n_threads);
  }
  run_parallel(prefill_row_job, &c, n_rows, n_threads);
  for (int b = 0; b < B; ++b) { free(c.khat[b]); free(c.vd[b]); }
  free(c.khat); free(c.vd); free(qw); free(kw);
  return 0;
}

/* The same output as oracle_prefill_rows for single (row, head) items: item r is
 * query head rows_h[r] of row (rows_b[r], rows_t[r]); out is [n_items][d].  Long
 * rows then cost one head instead of 48, so a parity sample can reach deep into a
 * 131,072-token sequence and still spread over every head. */
static void prefill_row_head_job(void *vctx, int64_t r) {
  prefill_ctx *c = (prefill_ctx *)vctx;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hq = P->n_q_heads, Hkv = P->n_kv_heads, G = Hq / Hkv;
  int64_t b = c->rows_b[r], t = c->rows_t[r];
  int h = (int)c->rows_h[r], g = h / G;
  int64_t lo = 0;
  while (!oracle_visible(c->kind, t, lo, P->window)) ++lo;  /* first visible key */
  int64_t n = t - lo + 1;
  double *q = (double *)malloc(sizeof(double) * d);
  double *scores = (double *)malloc(sizeof(double) * n);
  kv_view view = {c->khat[b] + ((size_t)lo * Hkv + g) * d, c->vd[b] + ((size_t)lo * Hkv + g) * d,
                  (int64_t)Hkv * d, d};
  size_t q_off = (((size_t)b * c->T + t) * Hq + h) * d;
  prepare_query(c->kind, P, c->q + q_off, c->qw, t, q);
  attend_one(P, q, n, kv_view_row, &view, c->gate + q_off, (double)c->bias[h], scores,
             c->out + (size_t)r * d);
  free(q); free(scores);
}

int oracle_prefill_row_heads(int kind, const oracle_params *P, int B, int T,
                             const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const uint16_t *gate, const float *q_norm_w, const float *k_norm_w,
                             const float *gate_bias, int64_t n_items, const int64_t *rows_b,
                             const int64_t *rows_t, const int64_t *rows_h, double *out,
                             int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  for (int64_t r = 0; r < n_items; ++r)
    if (rows_b[r] < 0 || rows_b[r] >= B || rows_t[r] < 0 || rows_t[r] >= T || rows_h[r] < 0 ||
        rows_h[r] >= P->n_q_heads)
      return -1;
  int d = P->head_dim, Hkv = P->n_kv_heads;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  prefill_ctx c;
  memset(&c, 0, sizeof c);
  c.kind = kind; c.P = P; c.B = B; c.T = T;
  c.q = q; c.k = k; c.v = v; c.gate = gate; c.qw = qw; c.kw = kw; c.bias = gate_bias;
  c.rows_b = rows_b; c.rows_t = rows_t; c.rows_h = rows_h; c.out = out;
  c.khat = (double **)calloc(B, sizeof(double *));
  c.vd = (double **)calloc(B, sizeof(double *));
  for (int b = 0; b < B; ++b) {
    int used = 0;
    for (int64_t r = 0; r < n_items && !used; ++r) used = rows_b[r] == b;
    if (!used) continue;
    c.khat[b] = (double *)malloc(sizeof(double) * (size_t)T * Hkv * d);
    c.vd[b] = (double *)malloc(sizeof(double) * (size_t)T * Hkv * d);
    c.key_b = b;
    run_parallel(prefill_key_job, &c, T, n_threads);
  }
  run_parallel(prefill_row_head_job, &c, n_items, n_threads);
  for (int b = 0; b < B; ++b) { free(c.khat[b]); free(c.vd[b]); }
  free(c.khat); free(c.vd); free(qw); free(kw);
  return 0;
}

/* ---------------------------------------------------------------- decode */

/* One decode step for B sequences, each adding one token at 0-based position
 * pos[b] (so p = pos[b] + 1).  The caches hold the rows written before this
 * step, head-major [B][Hkv][slots][d] (bf16 bits): keys already normalised
 * and, in a local ring, already rotated.  The new token's own key and value
 * are prepared here exactly and take part in the attention (append first,
 * then attend).  Visible earlier positions j are read from slot
 * oracle_cache_slot(kind, j, slots).  out is [B][Hq][d] doubles. */
typedef struct {
  int kind;
  const oracle_params *P;
  int B;
  const uint16_t *q, *k, *v, *gate;
  const double *qw, *kw;
  const float *bias;
  const int64_t *pos;
  const uint16_t *k_cache, *v_cache;
  int64_t slots;
  double *out;
} decode_ctx;

typedef struct {
  const decode_ctx *c;
  int64_t b, g, lo, t;
  const double *k_new, *v_new;  /* the new token's prepared key and value */
} decode_view;

static void decode_row(const void *vctx, int64_t idx, double *k_row, double *v_row) {
  const decode_view *r = (const decode_view *)vctx;
  const decode_ctx *c = r->c;
  int d = c->P->head_dim;
  int64_t j = r->lo + idx;
  if (j == r->t) {
    memcpy(k_row, r->k_new, sizeof(double) * d);
    memcpy(v_row, r->v_new, sizeof(double) * d);
    return;
  }
  int64_t s = oracle_cache_slot(c->kind, j, c->slots);
  size_t off = (((size_t)r->b * c->P->n_kv_heads + r->g) * c->slots + s) * d;
  for (int i = 0; i < d; ++i) {
    k_row[i] = oracle_bf16_to_double(c->k_cache[off + i]);
    v_row[i] = oracle_bf16_to_double(c->v_cache[off + i]);
  }
}

static void decode_job(void *vctx, int64_t item) {
  decode_ctx *c = (decode_ctx *)vctx;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hq = P->n_q_heads, Hkv = P->n_kv_heads, G = Hq / Hkv;
  int64_t b = item / Hq;
  int h = (int)(item % Hq), g = h / G;
  int64_t t = c->pos[b];
  int64_t lo = 0;
  while (!oracle_visible(c->kind, t, lo, P->window)) ++lo;
  int64_t n = t - lo + 1;
  double *scores = (double *)malloc(sizeof(double) * n);
  double *q = (double *)malloc(sizeof(double) * d);
  double *kv_new = (double *)malloc(sizeof(double) * 2 * d);
  size_t kv_off = ((size_t)b * Hkv + g) * d;
  prepare_key(c->kind, P, c->k + kv_off, c->kw, t, kv_new);
  for (int i = 0; i < d; ++i) kv_new[d + i] = oracle_bf16_to_double(c->v[kv_off + i]);
  decode_view view = {c, b, g, lo, t, kv_new, kv_new + d};
  size_t q_off = ((size_t)b * Hq + h) * d;
  prepare_query(c->kind, P, c->q + q_off, c->qw, t, q);
  attend_one(P, q, n, decode_row, &view, c->gate + q_off, (double)c->bias[h], scores,
             c->out + q_off);
  free(scores); free(q); free(kv_new);
}

int oracle_decode(int kind, const oracle_params *P, int B, const uint16_t *q, const uint16_t *k,
                  const uint16_t *v, const uint16_t *gate, const float *q_norm_w,
                  const float *k_norm_w, const float *gate_bias, const int64_t *pos,
                  const uint16_t *k_cache, const uint16_t *v_cache, int64_t slots, double *out,
                  int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return -1;
    if (kind == ORACLE_GLOBAL && pos[b] >= slots) return -1;
    if (kind == ORACLE_LOCAL && slots < P->window) return -1;
  }
  int d = P->head_dim;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  decode_ctx c = {kind, P, B, q, k, v, gate, qw, kw, gate_bias, pos, k_cache, v_cache, slots, out};
  run_parallel(decode_job, &c, (int64_t)B * P->n_q_heads, n_threads);
  free(qw); free(kw);
  return 0;
}

/* --------------------------------------------------------- chunked prefill */

/* Prefill of one chunk against an existing cache: sequence b adds T new
 * tokens at 0-based positions pos0[b] .. pos0[b] + T - 1 after pos0[b] earlier
 * tokens (section "KV memory": a call that continues a sequence reads the
 * earlier keys from the global cache or the local ring).  New token i of
 * sequence b is the query at t = pos0[b] + i.  Its visible keys j
 * (oracle_visible) come from two places: j < pos0[b] from the cache as it was
 * before the call (slot oracle_cache_slot(kind, j, slots), keys already
 * prepared), j >= pos0[b] from the chunk's own new token j - pos0[b], prepared
 * here exactly, the way decode treats its one new token.  q, k, v, gate are
 * token-major [B][T][heads][d] as in oracle_prefill_rows; the caches are
 * head-major [B][Hkv][slots][d].  Only the listed rows (b = rows_b[r], new
 * token i = rows_i[r]) are computed; out is [n_rows][Hq][d] doubles. */
typedef struct {
  int kind;
  const oracle_params *P;
  int B, T;
  const uint16_t *q, *k, *v, *gate;
  const double *qw, *kw;
  const float *bias;
  const int64_t *pos0;
  const uint16_t *k_cache, *v_cache;
  int64_t slots;
  const int64_t *rows_b, *rows_i;
  double *out;
  /* FP8 E4M3 caches (oracle_prefill_chunk_rows_fp8): cached rows are
   * E4M3^-1(code) * scale, and the chunk's own keys and values are first
   * written as codes, so the queries see them read back from the cache too */
  int fp8;
  const uint8_t *k_codes, *v_codes;
  double k_scale, v_scale;
} chunk_ctx;

typedef struct {
  const chunk_ctx *c;
  int64_t b, g, lo;
  const double *k_new, *v_new;  /* [T][d]: the chunk's prepared keys and values, head g */
} chunk_view;

static void chunk_row(const void *vctx, int64_t idx, double *k_row, double *v_row) {
  const chunk_view *r = (const chunk_view *)vctx;
  const chunk_ctx *c = r->c;
  int d = c->P->head_dim;
  int64_t j = r->lo + idx, p0 = c->pos0[r->b];
  if (j >= p0) {
    memcpy(k_row, r->k_new + (size_t)(j - p0) * d, sizeof(double) * d);
    memcpy(v_row, r->v_new + (size_t)(j - p0) * d, sizeof(double) * d);
    return;
  }
  int64_t s = oracle_cache_slot(c->kind, j, c->slots);
  size_t off = (((size_t)r->b * c->P->n_kv_heads + r->g) * c->slots + s) * d;
  for (int i = 0; i < d; ++i) {
    if (c->fp8) {
      k_row[i] = oracle_e4m3_decode(c->k_codes[off + i]) * c->k_scale;
      v_row[i] = oracle_e4m3_decode(c->v_codes[off + i]) * c->v_scale;
    } else {
      k_row[i] = oracle_bf16_to_double(c->k_cache[off + i]);
      v_row[i] = oracle_bf16_to_double(c->v_cache[off + i]);
    }
  }
}

static void chunk_job(void *vctx, int64_t r) {
  chunk_ctx *c = (chunk_ctx *)vctx;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hq = P->n_q_heads, Hkv = P->n_kv_heads, G = Hq / Hkv;
  int64_t b = c->rows_b[r], i = c->rows_i[r];
  int64_t t = c->pos0[b] + i;
  int64_t lo = 0;
  while (!oracle_visible(c->kind, t, lo, P->window)) ++lo;
  int64_t n = t - lo + 1;
  /* the new tokens m0 .. i of this sequence that are visible, prepared at their own
   * positions (rows below m0 are never read) */
  int64_t m0 = lo > c->pos0[b] ? lo - c->pos0[b] : 0;
  double *kv_new = (double *)malloc(sizeof(double) * 2 * (size_t)(i + 1) * d);
  double *scores = (double *)malloc(sizeof(double) * n);
  double *q = (double *)malloc(sizeof(double) * d);
  for (int h = 0; h < Hq; ++h) {
    int g = h / G;
    if (h % G == 0) {
      for (int64_t m = m0; m <= i; ++m) {
        size_t in_off = (((size_t)b * c->T + m) * Hkv + g) * d;
        double *kn = kv_new + (size_t)m * d, *vn = kv_new + (size_t)(i + 1) * d + (size_t)m * d;
        prepare_key(c->kind, P, c->k + in_off, c->kw, c->pos0[b] + m, kn);
        for (int e = 0; e < d; ++e) vn[e] = oracle_bf16_to_double(c->v[in_off + e]);
        if (c->fp8)   /* written as codes first, read back from the cache */
          for (int e = 0; e < d; ++e) {
            kn[e] = oracle_e4m3_decode(oracle_e4m3_encode(kn[e] / c->k_scale)) * c->k_scale;
            vn[e] = oracle_e4m3_decode(oracle_e4m3_encode(vn[e] / c->v_scale)) * c->v_scale;
          }
      }
    }
    chunk_view view = {c, b, g, lo, kv_new, kv_new + (size_t)(i + 1) * d};
    size_t q_off = (((size_t)b * c->T + i) * Hq + h) * d;
    prepare_query(c->kind, P, c->q + q_off, c->qw, t, q);
    attend_one(P, q, n, chunk_row, &view, c->gate + q_off, (double)c->bias[h], scores,
               c->out + ((size_t)r * Hq + h) * d);
  }
  free(kv_new); free(scores); free(q);
}

int oracle_prefill_chunk_rows(int kind, const oracle_params *P, int B, int T,
                              const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const uint16_t *gate, const float *q_norm_w, const float *k_norm_w,
                              const float *gate_bias, const int64_t *pos0,
                              const uint16_t *k_cache, const uint16_t *v_cache, int64_t slots,
                              int64_t n_rows, const int64_t *rows_b, const int64_t *rows_i,
                              double *out, int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  for (int b = 0; b < B; ++b) {
    if (pos0[b] < 0) return -1;
    if (kind == ORACLE_GLOBAL && pos0[b] + T > slots) return -1;
    if (kind == ORACLE_LOCAL && slots < P->window) return -1;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows_b[r] < 0 || rows_b[r] >= B || rows_i[r] < 0 || rows_i[r] >= T) return -1;
  int d = P->head_dim;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  chunk_ctx c = {kind, P, B, T, q, k, v, gate, qw, kw, gate_bias, pos0, k_cache, v_cache, slots,
                 rows_b, rows_i, out, 0, NULL, NULL, 1.0, 1.0};
  run_parallel(chunk_job, &c, n_rows, n_threads);
  free(qw); free(kw);
  return 0;
}

/* ------------------------------------------------------------ FP8 cache */

/* FP8 E4M3 as the KV-cache element (section "KV memory": 18 KiB per token
 * over the nine global layers instead of 36 KiB in BF16).  The page names the
 * format only; its definition here is the OCP 8-bit floating-point E4M3 one
 * without infinities: sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent 0 holds the subnormals m * 2^-9; S.1111.111 is NaN, so the largest
 * finite magnitude is 1.75 * 2^8 = 448.  A cache element stores
 * code = E4M3(x / scale) with one float scale per cache tensor of a layer, and
 * reads back as E4M3^-1(code) * scale. */
double oracle_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Nearest code, ties to the even mantissa; magnitudes past 448 saturate to
 * +-448 (the conversion the cache write uses), NaN stays NaN. */
uint8_t oracle_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t s = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a >= 448.0) return s | 0x7E;
  int e2;
  frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
  int e = e2 - 1;         /* a in [2^e, 2^(e+1)) */
  if (a == 0.0 || e < -6) {
    double m = nearbyint(ldexp(a, 9));   /* subnormal steps of 2^-9; 8 -> smallest normal */
    return s | (uint8_t)m;
  }
  double m = nearbyint((ldexp(a, -e) - 1.0) * 8.0);   /* 0 .. 8 */
  if (m == 8.0) { m = 0.0; ++e; }
  if (e > 8 || (e == 8 && m > 6.0)) return s | 0x7E;
  return s | (uint8_t)(((e + 7) << 3) | (int)m);
}

/* One decode step over FP8 caches: as oracle_decode, but every cached row is
 * E4M3^-1(code) * scale, and the new token's key and value are first written
 * as codes (append first, then attend), so the query sees them read back from
 * the cache too.  Caches are head-major [B][Hkv][slots][d] codes. */
typedef struct {
  decode_ctx base;
  const uint8_t *k_codes, *v_codes;
  double k_scale, v_scale;
} decode8_ctx;

typedef struct {
  const decode8_ctx *c;
  int64_t b, g, lo, t;
  const double *k_new, *v_new;
} decode8_view;

static void decode8_row(const void *vctx, int64_t idx, double *k_row, double *v_row) {
  const decode8_view *r = (const decode8_view *)vctx;
  const decode8_ctx *c = r->c;
  int d = c->base.P->head_dim;
  int64_t j = r->lo + idx;
  if (j == r->t) {
    memcpy(k_row, r->k_new, sizeof(double) * d);
    memcpy(v_row, r->v_new, sizeof(double) * d);
    return;
  }
  int64_t s = oracle_cache_slot(c->base.kind, j, c->base.slots);
  size_t off = (((size_t)r->b * c->base.P->n_kv_heads + r->g) * c->base.slots + s) * d;
  for (int i = 0; i < d; ++i) {
    k_row[i] = oracle_e4m3_decode(c->k_codes[off + i]) * c->k_scale;
    v_row[i] = oracle_e4m3_decode(c->v_codes[off + i]) * c->v_scale;
  }
}

static void decode8_job(void *vctx, int64_t item) {
  decode8_ctx *c8 = (decode8_ctx *)vctx;
  const decode_ctx *c = &c8->base;
  const oracle_params *P = c->P;
  int d = P->head_dim, Hq = P->n_q_heads, Hkv = P->n_kv_heads, G = Hq / Hkv;
  int64_t b = item / Hq;
  int h = (int)(item % Hq), g = h / G;
  int64_t t = c->pos[b];
  int64_t lo = 0;
  while (!oracle_visible(c->kind, t, lo, P->window)) ++lo;
  int64_t n = t - lo + 1;
  double *scores = (double *)malloc(sizeof(double) * n);
  double *q = (double *)malloc(sizeof(double) * d);
  double *kv_new = (double *)malloc(sizeof(double) * 2 * d);
  size_t kv_off = ((size_t)b * Hkv + g) * d;
  prepare_key(c->kind, P, c->k + kv_off, c->kw, t, kv_new);
  for (int i = 0; i < d; ++i) {
    kv_new[i] = oracle_e4m3_decode(oracle_e4m3_encode(kv_new[i] / c8->k_scale)) * c8->k_scale;
    double v = oracle_bf16_to_double(c->v[kv_off + i]);
    kv_new[d + i] = oracle_e4m3_decode(oracle_e4m3_encode(v / c8->v_scale)) * c8->v_scale;
  }
  decode8_view view = {c8, b, g, lo, t, kv_new, kv_new + d};
  size_t q_off = ((size_t)b * Hq + h) * d;
  prepare_query(c->kind, P, c->q + q_off, c->qw, t, q);
  attend_one(P, q, n, decode8_row, &view, c->gate + q_off, (double)c->bias[h], scores,
             c->out + q_off);
  free(scores); free(q); free(kv_new);
}

int oracle_decode_fp8(int kind, const oracle_params *P, int B, const uint16_t *q,
                      const uint16_t *k, const uint16_t *v, const uint16_t *gate,
                      const float *q_norm_w, const float *k_norm_w, const float *gate_bias,
                      const int64_t *pos, const uint8_t *k_codes, const uint8_t *v_codes,
                      int64_t slots, double k_scale, double v_scale, double *out, int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  if (!(k_scale > 0.0) || !(v_scale > 0.0)) return -1;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) return -1;
    if (kind == ORACLE_GLOBAL && pos[b] >= slots) return -1;
    if (kind == ORACLE_LOCAL && slots < P->window) return -1;
  }
  int d = P->head_dim;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  decode8_ctx c = {{kind, P, B, q, k, v, gate, qw, kw, gate_bias, pos, NULL, NULL, slots, out},
                   k_codes, v_codes, k_scale, v_scale};
  run_parallel(decode8_job, &c, (int64_t)B * P->n_q_heads, n_threads);
  free(qw); free(kw);
  return 0;
}

/* Chunked prefill over FP8 E4M3 caches (section "KV memory": the FP8 cache, and a
 * call that continues a sequence reads its earlier keys from the cache): as
 * oracle_prefill_chunk_rows, but a cached row is E4M3^-1(code) * scale and the
 * chunk's own keys and values are written as codes first (code = E4M3(x / scale)
 * of the exact prepared key and of the raw value), so the queries see them read
 * back from the cache -- the order oracle_decode_fp8 takes for one new token.
 * Caches are head-major [B][Hkv][slots][d] codes as they were before the call. */
int oracle_prefill_chunk_rows_fp8(int kind, const oracle_params *P, int B, int T,
                                  const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  const uint16_t *gate, const float *q_norm_w,
                                  const float *k_norm_w, const float *gate_bias,
                                  const int64_t *pos0, const uint8_t *k_codes,
                                  const uint8_t *v_codes, int64_t slots, double k_scale,
                                  double v_scale, int64_t n_rows, const int64_t *rows_b,
                                  const int64_t *rows_i, double *out, int n_threads) {
  if (!P || P->n_kv_heads <= 0 || P->n_q_heads % P->n_kv_heads) return -1;
  if (!(k_scale > 0.0) || !(v_scale > 0.0)) return -1;
  for (int b = 0; b < B; ++b) {
    if (pos0[b] < 0) return -1;
    if (kind == ORACLE_GLOBAL && pos0[b] + T > slots) return -1;
    if (kind == ORACLE_LOCAL && slots < P->window) return -1;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows_b[r] < 0 || rows_b[r] >= B || rows_i[r] < 0 || rows_i[r] >= T) return -1;
  int d = P->head_dim;
  double *qw = (double *)malloc(sizeof(double) * d), *kw = (double *)malloc(sizeof(double) * d);
  for (int i = 0; i < d; ++i) { qw[i] = q_norm_w[i]; kw[i] = k_norm_w[i]; }
  chunk_ctx c = {kind, P, B, T, q, k, v, gate, qw, kw, gate_bias, pos0, NULL, NULL, slots,
                 rows_b, rows_i, out, 1, k_codes, v_codes, k_scale, v_scale};
  run_parallel(chunk_job, &c, n_rows, n_threads);
  free(qw); free(kw);
  return 0;
}

/* Expected FP8 cache rows for one token at position j: codes of the exact
 * prepared key and of the raw value, each divided by its scale. */
void oracle_kv_row_fp8(int kind, const oracle_params *P, const uint16_t *k_raw_token,
                       const uint16_t *v_raw_token, const float *k_norm_w, int64_t j,
                       double k_scale, double v_scale, uint8_t *k_row, uint8_t *v_row) {
  int d = P->head_dim;
  double *tmp = (double *)malloc(sizeof(double) * d);
  for (int g = 0; g < P->n_kv_heads; ++g) {
    oracle_prepare_key(kind, P, k_raw_token + (size_t)g * d, k_norm_w, j, tmp);
    for (int i = 0; i < d; ++i) {
      k_row[(size_t)g * d + i] = oracle_e4m3_encode(tmp[i] / k_scale);
      v_row[(size_t)g * d + i] =
          oracle_e4m3_encode(oracle_bf16_to_double(v_raw_token[(size_t)g * d + i]) / v_scale);
    }
  }
  free(tmp);
}

/* Expected cache rows written for one token at position j: the prepared key
 * rounded to the nearest bf16 and the raw value bits, one row per KV head
 * ([Hkv][d] each).  Tests compare these with what the device wrote at slot
 * oracle_cache_slot(kind, j, slots). */
void oracle_kv_row(int kind, const oracle_params *P, const uint16_t *k_raw_token,
                   const uint16_t *v_raw_token, const float *k_norm_w, int64_t j,
                   uint16_t *k_row, uint16_t *v_row) {
  int d = P->head_dim;
  double *tmp = (double *)malloc(sizeof(double) * d);
  for (int g = 0; g < P->n_kv_heads; ++g) {
    oracle_prepare_key(kind, P, k_raw_token + (size_t)g * d, k_norm_w, j, tmp);
    for (int i = 0; i < d; ++i) {
      k_row[(size_t)g * d + i] = oracle_double_to_bf16(tmp[i]);
      v_row[(size_t)g * d + i] = v_raw_token[(size_t)g * d + i];
    }
  }
  free(tmp);
}
