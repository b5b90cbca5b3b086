/*
 * ssd_oracle.c -- fp64 CPU oracle for the Mamba-2 SSD layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this
 * file: only the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (all arrays row-major, contiguous, float64):
 *   x  [b, L, H, P]     dt [b, L, H]     A [H]     D [H]
 *   B  [b, L, G, N]     C  [b, L, G, N]  state [b, H, P, N]     y [b, L, H, P]
 * Head h reads group g = h / (H / G) (contiguous head groups).
 *
 * Three independent formulations of one layer:
 *
 *  1. ssd_oracle_recurrence -- the sequential recurrence.  "Engineering Hybrid
 *     State-Space Models" (section 2, "Mathematical Formalization") writes the diagonal
 *     recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t with Abar_t =
 *     exp(dt_t A); "Compiler-First State Space Duality ..." (abstract) fixes the
 *     dynamics as one scalar per head; the skip term D x_t is the feedthrough of
 *     "Mamba and Selective State Space Models" (section 2).  The input matrix is taken in
 *     the Euler form Bbar_t = dt_t B_t (the same page's code section applies
 *     bBar = delta * x), so per head
 *        h[p][n] <- exp(dt_t A_h) h[p][n] + dt_t x_t[p] B_t[n]
 *        y_t[p]   = sum_n C_t[n] h[p][n] + D_h x_t[p]     (h after the update).
 *     This is the definition the GPU path is checked against.
 *
 *  2. ssd_oracle_quadratic -- the semiseparable ("attention") form of the same page's
 *     section 2: Y = (M o C B^T) X with M[j][k] = prod_{i=k+1..j} a_i for k <= j
 *     (empty product = 1 on the diagonal) and 0 for k > j, applied per head to the
 *     dt-scaled inputs, plus the decayed contribution of an initial state.
 *
 *  3. ssd_oracle_chunked -- the same layer split into fixed-size chunks (section 2 of
 *     the same page, chunks of Q tokens; "Compiler-First ..." abstract, fixed-size
 *     chunking): within a chunk the quadratic form, across chunks a state carried by
 *     the first-order linear recurrence h_c = (prod of the chunk's a_i) h_{c-1} + S_c
 *     (the associative combine of "Mamba and Selective State Space Models", section 5).
 *
 * Forms 2 and 3 exist to pin form 1: their agreement is the duality claim of section 2.
 * Parallelism: pthreads over independent (batch, head) pairs; every pair is computed by
 * exactly one thread in the same order, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

typedef struct {
  int64_t b, L, H, P, N, G;
} dims_t;

static int check_dims(const dims_t *d) {
  if (d->b < 0 || d->L < 0 || d->H < 1 || d->P < 1 || d->N < 1 || d->G < 1) return 0;
  if (d->H % d->G != 0) return 0;
  return 1;
}

/* ---------------------------------------------------------------- index helpers */
static inline int64_t ix_x(const dims_t *d, int64_t bi, int64_t t, int64_t h, int64_t p) {
  return ((bi * d->L + t) * d->H + h) * d->P + p;
}
static inline int64_t ix_dt(const dims_t *d, int64_t bi, int64_t t, int64_t h) {
  return (bi * d->L + t) * d->H + h;
}
static inline int64_t ix_bc(const dims_t *d, int64_t bi, int64_t t, int64_t g, int64_t n) {
  return ((bi * d->L + t) * d->G + g) * d->N + n;
}
static inline int64_t ix_state(const dims_t *d, int64_t bi, int64_t h, int64_t p, int64_t n) {
  return ((bi * d->H + h) * d->P + p) * d->N + n;
}

/* ---------------------------------------------------------------- thread fan-out */
typedef void (*head_fn)(void *ctx, int64_t bi, int64_t h);
typedef struct {
  head_fn fn;
  void *ctx;
  int64_t nb, nh, next;
  pthread_mutex_t lock;
} pool_t;

static void *pool_worker(void *arg) {
  pool_t *pl = (pool_t *)arg;
  for (;;) {
    pthread_mutex_lock(&pl->lock);
    int64_t job = pl->next++;
    pthread_mutex_unlock(&pl->lock);
    if (job >= pl->nb * pl->nh) break;
    pl->fn(pl->ctx, job / pl->nh, job % pl->nh);
  }
  return NULL;
}

static void run_heads(head_fn fn, void *ctx, int64_t nb, int64_t nh, int nthreads) {
  int64_t jobs = nb * nh;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > jobs) nthreads = (int)(jobs > 0 ? jobs : 1);
  pool_t pl;
  pl.fn = fn;
  pl.ctx = ctx;
  pl.nb = nb;
  pl.nh = nh;
  pl.next = 0;
  pthread_mutex_init(&pl.lock, NULL);
  if (nthreads == 1) {
    pool_worker(&pl);
  } else {
    pthread_t th[256];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
      if (pthread_create(&th[i], NULL, pool_worker, &pl) == 0) ++started;
    }
    if (started == 0) pool_worker(&pl);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  }
  pthread_mutex_destroy(&pl.lock);
}

/* ============================================================ 1. recurrence */
typedef struct {
  const dims_t *d;
  const double *x, *dt, *A, *B, *C, *D;
  double *state, *y;
} rec_ctx;

static void rec_head(void *vctx, int64_t bi, int64_t h) {
  const rec_ctx *c = (const rec_ctx *)vctx;
  const dims_t *d = c->d;
  const int64_t g = h / (d->H / d->G);
  double *hs = c->state + ix_state(d, bi, h, 0, 0); /* [P][N] for this head */
  for (int64_t t = 0; t < d->L; ++t) {
    const double dtv = c->dt[ix_dt(d, bi, t, h)];
    const double abar = exp(dtv * c->A[h]); /* Abar_t = exp(dt_t A_h) */
    const double *Bt = c->B + ix_bc(d, bi, t, g, 0);
    const double *Ct = c->C + ix_bc(d, bi, t, g, 0);
    for (int64_t p = 0; p < d->P; ++p) {
      const double xv = c->x[ix_x(d, bi, t, h, p)];
      double *row = hs + p * d->N;
      double acc = 0.0;
      for (int64_t n = 0; n < d->N; ++n) {
        row[n] = abar * row[n] + dtv * xv * Bt[n]; /* h_t = Abar h_{t-1} + dt B x */
        acc += Ct[n] * row[n];                       /* C_t h_t */
      }
      c->y[ix_x(d, bi, t, h, p)] = acc + c->D[h] * xv; /* + D x_t */
    }
  }
}

/* state: in = initial state, out = state after the last token (updated in place). */
int ssd_oracle_recurrence(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                          const double *x, const double *dt, const double *A,
                          const double *B, const double *C, const double *D,
                          double *state, double *y, int nthreads) {
  dims_t d = {b, L, H, P, N, G};
  if (!check_dims(&d)) return ORACLE_EINVAL;
  rec_ctx c = {&d, x, dt, A, B, C, D, state, y};
  run_heads(rec_head, &c, b, H, nthreads);
  return ORACLE_OK;
}

/* ============================================================ 2. quadratic form */
typedef struct {
  const dims_t *d;
  const double *x, *dt, *A, *B, *C, *D, *init;
  double *y, *final_state;
} quad_ctx;

static void quad_head(void *vctx, int64_t bi, int64_t h) {
  const quad_ctx *c = (const quad_ctx *)vctx;
  const dims_t *d = c->d;
  const int64_t L = d->L, P = d->P, N = d->N;
  const int64_t g = h / (d->H / d->G);
  double *a = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double *Mrow = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  if (!a || !Mrow) {
    free(a);
    free(Mrow);
    return;
  }
  for (int64_t t = 0; t < L; ++t) a[t] = exp(c->dt[ix_dt(d, bi, t, h)] * c->A[h]);

  for (int64_t t = 0; t < L; ++t) {
    /* Row t of the 1-semiseparable mask: M[t][s] = prod_{i=s+1..t} a_i, s <= t. */
    Mrow[t] = 1.0;
    for (int64_t s = t - 1; s >= 0; --s) Mrow[s] = Mrow[s + 1] * a[s + 1];
    /* Decay of the initial state seen by token t: prod_{i=0..t} a_i. */
    const double init_decay = Mrow[0] * a[0];
    const double *Ct = c->C + ix_bc(d, bi, t, g, 0);
    for (int64_t p = 0; p < P; ++p) {
      double acc = 0.0;
      for (int64_t s = 0; s <= t; ++s) {
        const double *Bs = c->B + ix_bc(d, bi, s, g, 0);
        double cb = 0.0; /* (C B^T)[t][s] */
        for (int64_t n = 0; n < N; ++n) cb += Ct[n] * Bs[n];
        acc += Mrow[s] * cb * c->dt[ix_dt(d, bi, s, h)] * c->x[ix_x(d, bi, s, h, p)];
      }
      if (c->init) {
        double ch = 0.0;
        for (int64_t n = 0; n < N; ++n) ch += Ct[n] * c->init[ix_state(d, bi, h, p, n)];
        acc += init_decay * ch;
      }
      c->y[ix_x(d, bi, t, h, p)] = acc + c->D[h] * c->x[ix_x(d, bi, t, h, p)];
    }
  }

  /* Final state: h_{L-1}[p][n] = sum_s M[L-1][s] dt_s x_s[p] B_s[n] + prod(a) h_init. */
  if (c->final_state) {
    if (L > 0) {
      Mrow[L - 1] = 1.0;
      for (int64_t s = L - 2; s >= 0; --s) Mrow[s] = Mrow[s + 1] * a[s + 1];
    }
    const double total_decay = (L > 0) ? Mrow[0] * a[0] : 1.0;
    for (int64_t p = 0; p < P; ++p) {
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t s = 0; s < L; ++s)
          acc += Mrow[s] * c->dt[ix_dt(d, bi, s, h)] * c->x[ix_x(d, bi, s, h, p)] *
                 c->B[ix_bc(d, bi, s, g, n)];
        if (c->init) acc += total_decay * c->init[ix_state(d, bi, h, p, n)];
        c->final_state[ix_state(d, bi, h, p, n)] = acc;
      }
    }
  }
  free(a);
  free(Mrow);
}

/* init_state may be NULL (zero initial state); final_state may be NULL. */
int ssd_oracle_quadratic(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                         const double *x, const double *dt, const double *A,
                         const double *B, const double *C, const double *D,
                         const double *init_state, double *y, double *final_state,
                         int nthreads) {
  dims_t d = {b, L, H, P, N, G};
  if (!check_dims(&d)) return ORACLE_EINVAL;
  quad_ctx c = {&d, x, dt, A, B, C, D, init_state, y, final_state};
  run_heads(quad_head, &c, b, H, nthreads);
  return ORACLE_OK;
}

/* ============================================================ 3. chunked form */
typedef struct {
  const dims_t *d;
  int64_t Q;
  const double *x, *dt, *A, *B, *C, *D, *init;
  double *y, *final_state;
} chunk_ctx;

static void chunk_head(void *vctx, int64_t bi, int64_t h) {
  const chunk_ctx *c = (const chunk_ctx *)vctx;
  const dims_t *d = c->d;
  const int64_t L = d->L, P = d->P, N = d->N, Q = c->Q;
  const int64_t g = h / (d->H / d->G);
  double *hprev = (double *)calloc((size_t)(P * N), sizeof(double)); /* state entering chunk */
  double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));    /* chunk contribution */
  double *lcum = (double *)malloc(sizeof(double) * (size_t)Q);       /* log of in-chunk decay */
  if (!hprev || !S || !lcum) {
    free(hprev);
    free(S);
    free(lcum);
    return;
  }
  if (c->init) memcpy(hprev, c->init + ix_state(d, bi, h, 0, 0), sizeof(double) * (size_t)(P * N));

  for (int64_t t0 = 0; t0 < L; t0 += Q) {
    const int64_t len = (L - t0 < Q) ? (L - t0) : Q;
    /* (a) lcum[j] = sum_{i=0..j} dt_i A_h over the chunk: exp(lcum[j] - lcum[k]) is the
     *     product of a_i for i = k+1..j, and exp(lcum[j]) the decay since the chunk start. */
    double run = 0.0;
    for (int64_t j = 0; j < len; ++j) {
      run += c->dt[ix_dt(d, bi, t0 + j, h)] * c->A[h];
      lcum[j] = run;
    }
    const double lend = lcum[len - 1];
    /* (b) chunk contribution S[p][n] = sum_k exp(lend - lcum[k]) dt_k x_k[p] B_k[n]. */
    for (int64_t p = 0; p < P; ++p)
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t k = 0; k < len; ++k)
          acc += exp(lend - lcum[k]) * c->dt[ix_dt(d, bi, t0 + k, h)] *
                 c->x[ix_x(d, bi, t0 + k, h, p)] * c->B[ix_bc(d, bi, t0 + k, g, n)];
        S[p * N + n] = acc;
      }
    /* (d) outputs: intra-chunk quadratic form + decayed state entering the chunk + D x. */
    for (int64_t j = 0; j < len; ++j) {
      const double *Cj = c->C + ix_bc(d, bi, t0 + j, g, 0);
      for (int64_t p = 0; p < P; ++p) {
        double acc = 0.0;
        for (int64_t k = 0; k <= j; ++k) {
          const double *Bk = c->B + ix_bc(d, bi, t0 + k, g, 0);
          double cb = 0.0;
          for (int64_t n = 0; n < N; ++n) cb += Cj[n] * Bk[n];
          acc += exp(lcum[j] - lcum[k]) * cb * c->dt[ix_dt(d, bi, t0 + k, h)] *
                 c->x[ix_x(d, bi, t0 + k, h, p)];
        }
        double ch = 0.0;
        for (int64_t n = 0; n < N; ++n) ch += Cj[n] * hprev[p * N + n];
        acc += exp(lcum[j]) * ch;
        c->y[ix_x(d, bi, t0 + j, h, p)] = acc + c->D[h] * c->x[ix_x(d, bi, t0 + j, h, p)];
      }
    }
    /* (c) carry: h_c = exp(lend) h_{c-1} + S_c. */
    const double dec = exp(lend);
    for (int64_t e = 0; e < P * N; ++e) hprev[e] = dec * hprev[e] + S[e];
  }
  if (c->final_state)
    memcpy(c->final_state + ix_state(d, bi, h, 0, 0), hprev, sizeof(double) * (size_t)(P * N));
  free(hprev);
  free(S);
  free(lcum);
}

int ssd_oracle_chunked(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                       int64_t chunk, const double *x, const double *dt, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *init_state, double *y, double *final_state,
                       int nthreads) {
  dims_t d = {b, L, H, P, N, G};
  if (!check_dims(&d) || chunk < 1) return ORACLE_EINVAL;
  chunk_ctx c = {&d, chunk, x, dt, A, B, C, D, init_state, y, final_state};
  run_heads(chunk_head, &c, b, H, nthreads);
  return ORACLE_OK;
}
