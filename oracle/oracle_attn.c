/*
 * CPU oracle for structured sparse causal attention with depth-staggered
 * Fibonacci offsets.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg call it; the product path never does.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * Source of the method: "Depth-Staggered Fibonacci Spacing for Sparse
 * Attention: Static Schedules Beat Learned Dilation and Extrapolate Where Dense
 * Attention Fails" (C. A. Capps), technical summary, section "Methodology":
 *   - "Attended set": query i attends a dense local window of W keys plus the
 *     sparse Fibonacci offsets f = 1, 2, 3, 5, ..., 987;
 *   - "Scaling": each offset becomes a distance d_k = alpha * f_k, one alpha
 *     per layer;
 *   - "Implementation": non-integer distances linearly interpolate between
 *     adjacent key/value rows (so gradients reach alpha), and RoPE is applied
 *     before the gather.
 * Readings where the page is silent (each one is listed in the design notes):
 *   window = keys i-W+1 .. i (self included); an offset is dropped for query
 *   i when i - ceil(d_k) < 0; d_k is one IEEE fp32 product alpha*f_k, then
 *   lo = floor(d_k), w = d_k - lo; the interpolated row is
 *   (1-w)*X[i-lo] + w*X[i-lo-1] for X in {RoPE(K), V}; sinks are keys
 *   0..S-1, attended when j <= i; duplicates stay separate softmax members;
 *   one softmax over all members with scale 1/sqrt(D); RoPE is rotate-half
 *   (pairs (j, j+D/2), theta_j = base^(-2j/D)) on Q and K, not V.
 *   An offset with d_k outside [0, 2^24) (alpha negative, NaN, or huge) has
 *   no defined row: its score is NaN, so the query's outputs become NaN.
 *
 * Optional additive log-prior on the offset members.  "pi-Attention: Periodic
 * Sparse Transformers for Efficient Long-Context Modeling" (Core components,
 * dynamic adaptive fusion) merges its local and skip logits into one softmax
 * by adding a log-prior in the log domain.  Softmax ignores a shift common to
 * all of a query's members, so the two per-query priors act only through
 * their difference: here one value beta[i] per query is added to the score
 * of every offset member of query i.  The window and the sinks get 0.  The
 * gradient is dbeta[i] = sum over those offset members of dLoss/dscore.
 * beta is [L][B][H][T] and may be NULL, meaning zero.
 *
 * This file is compiled twice: with ORACLE_REAL=double / ORACLE_SUFFIX=_f64
 * (parity reference and finite differences) and with ORACLE_REAL=float /
 * ORACLE_SUFFIX=_f32 (the plain fp32 CPU baseline).  RoPE angles and their
 * sine/cosine are always taken in double precision, then rounded to REAL.
 *
 * Layout of every [L][B][H][T][D] tensor: contiguous, D innermost.
 * The work is split over independent (layer, batch, head) units with OpenMP;
 * each unit writes disjoint outputs, and the per-layer d-alpha partials are
 * summed afterwards in a fixed order, so results do not depend on threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_REAL
#error "compile with -DORACLE_REAL=double or float"
#endif
typedef ORACLE_REAL real;
#define CAT2(a, b) a##b
#define CAT(a, b) CAT2(a, b)
#define FN(name) CAT(name, ORACLE_SUFFIX)

#define ORACLE_MAX_OFFSETS 64

/* Offset geometry for one (alpha, f) pair ("Scaling"; interpolation reading).
 * d is a single fp32 multiply; floor/ceil are taken on that float. */
typedef struct {
  int ok;        /* 0: d outside [0, 2^24) or NaN -> the member's score is NaN */
  int64_t lo;    /* floor(d)                                                  */
  int64_t c;     /* ceil(d): the member exists for query i iff i - c >= 0     */
  double w;      /* d - lo, exact in fp32                                     */
  int32_t f;
} geom_t;

static geom_t geometry(float alpha, int32_t f) {
  geom_t g;
  volatile float d = alpha * (float)f; /* volatile: keep it one fp32 product */
  g.f = f;
  if (!(d >= 0.0f && d < 16777216.0f)) {
    g.ok = 0; g.lo = 0; g.c = 0; g.w = 0.0;
    return g;
  }
  float fl = floorf(d);
  g.ok = 1;
  g.lo = (int64_t)fl;
  g.c = (int64_t)ceilf(d);
  g.w = (double)(d - fl);
  return g;
}

/* Rotate-half RoPE of one row at integer position pos ("RoPE before the
 * gather").  out may not alias x. */
static void rope_row(const real* x, int64_t pos, int D, double base, real* out) {
  int half = D / 2;
  for (int j = 0; j < half; ++j) {
    double theta = pow(base, -2.0 * (double)j / (double)D);
    double ang = (double)pos * theta;
    real cs = (real)cos(ang), sn = (real)sin(ang);
    real a = x[j], b = x[j + half];
    out[j] = a * cs - b * sn;
    out[j + half] = b * cs + a * sn;
  }
}

/* Transpose of rope_row (the inverse rotation), used to carry gradients from
 * rotated coordinates back to the raw Q/K rows. */
static void rope_row_t(const real* x, int64_t pos, int D, double base, real* out) {
  int half = D / 2;
  for (int j = 0; j < half; ++j) {
    double theta = pow(base, -2.0 * (double)j / (double)D);
    double ang = (double)pos * theta;
    real cs = (real)cos(ang), sn = (real)sin(ang);
    real a = x[j], b = x[j + half];
    out[j] = a * cs + b * sn;
    out[j + half] = b * cs - a * sn;
  }
}

/* One member of a query's attended set. */
typedef struct {
  int kind;      /* 0 window, 1 sink, 2 offset */
  int slot;      /* position in the fixed per-query slot list (window, sinks, offsets) */
  int k;         /* offset index for kind 2 */
  int nan_score; /* geometry outside its domain */
  int64_t a, b;  /* rows; b < 0 means "no second row" */
  real wa, wb;   /* interpolation weights: (1-w), w */
} member_t;

/* Enumerate the attended set of query i ("Attended set"). Returns count. */
static int members_of(int64_t i, int W, int S, int n_off, const geom_t* g, member_t* m) {
  int n = 0;
  for (int t = 0; t < W; ++t) {            /* window keys i, i-1, ..., i-W+1 */
    int64_t j = i - t;
    if (j < 0) continue;
    member_t x = {0, t, -1, 0, j, -1, (real)1, (real)0};
    m[n++] = x;
  }
  for (int s = 0; s < S; ++s) {            /* sinks 0..S-1, causal */
    if ((int64_t)s > i) continue;
    member_t x = {1, W + s, -1, 0, (int64_t)s, -1, (real)1, (real)0};
    m[n++] = x;
  }
  for (int k = 0; k < n_off; ++k) {        /* scaled, interpolated offsets */
    member_t x = {2, W + S + k, k, 0, -1, -1, (real)1, (real)0};
    if (!g[k].ok) {
      x.nan_score = 1;
      m[n++] = x;
      continue;
    }
    if (i - g[k].c < 0) continue;          /* drop rule */
    x.a = i - g[k].lo;
    x.wa = (real)(1.0 - g[k].w);
    if (g[k].w != 0.0) {
      x.b = i - g[k].lo - 1;
      x.wb = (real)g[k].w;
    }
    m[n++] = x;
  }
  return n;
}

static real dot(const real* x, const real* y, int D) {
  real s = 0;
  for (int d = 0; d < D; ++d) s += x[d] * y[d];
  return s;
}

/* Interpolated row: wa * X[a] + wb * X[b] ("Implementation"). */
static void gather_row(const real* X, const member_t* mb, int D, real* out) {
  for (int d = 0; d < D; ++d) {
    real v = mb->wa * X[mb->a * D + d];
    if (mb->b >= 0) v += mb->wb * X[mb->b * D + d];
    out[d] = v;
  }
}

typedef struct {
  int L, B, H, T, D, W, n_off, S;
  double base, scale;
  const int32_t* offsets;
  const float* alpha;
} prob_t;

static int check(const prob_t* p) {
  if (p->L < 1 || p->B < 1 || p->H < 1 || p->T < 1 || p->D < 2 || (p->D & 1)) return -1;
  if (p->W < 1 || p->S < 0 || p->n_off < 0 || p->n_off > ORACLE_MAX_OFFSETS) return -1;
  for (int k = 0; k < p->n_off; ++k)
    if (p->offsets[k] < 1) return -1;
  return 0;
}

/* Rotated keys of one unit: Kr[j] = RoPE(K[j], j). */
static void rotate_unit(const real* K, int64_t T, int D, double base, real* Kr) {
  for (int64_t j = 0; j < T; ++j) rope_row(K + j * D, j, D, base, Kr + j * D);
}

/*
 * Forward.  O[L][B][H][T][D], LSE[L][B][H][T] (may be NULL), and optionally
 * P[L][B][H][T][W+S+n_off]: each member's softmax weight in its fixed slot
 * (window t, then sink s, then offset k), 0 for members that do not exist.
 * beta (may be NULL): the per-query log-prior on the offset members.
 */
int FN(oracle_fwd)(int L, int B, int H, int T, int D, int W, int n_off,
                   const int32_t* offsets, int S, double rope_base, double scale,
                   const float* alpha, const real* Q, const real* K, const real* V,
                   real* O, real* LSE, real* P, const real* beta) {
  prob_t p = {L, B, H, T, D, W, n_off, S, rope_base, scale, offsets, alpha};
  if (check(&p)) return -1;
  const double s = scale > 0 ? scale : 1.0 / sqrt((double)D);
  const int n_slots = W + S + n_off;
  const int64_t units = (int64_t)L * B * H;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
  for (int64_t u = 0; u < units; ++u) {
    const int l = (int)(u / ((int64_t)B * H));
    geom_t g[ORACLE_MAX_OFFSETS];
    for (int k = 0; k < n_off; ++k) g[k] = geometry(alpha[l], offsets[k]);
    const int64_t base_off = u * (int64_t)T * D;
    real* Kr = (real*)malloc(sizeof(real) * (size_t)T * D);
    real* qh = (real*)malloc(sizeof(real) * D);
    real* row = (real*)malloc(sizeof(real) * D);
    member_t* mb = (member_t*)malloc(sizeof(member_t) * (size_t)n_slots);
    real* sc = (real*)malloc(sizeof(real) * (size_t)n_slots);
    if (!Kr || !qh || !row || !mb || !sc) { err |= 1; goto done; }
    rotate_unit(K + base_off, T, D, rope_base, Kr);
    const real* Vu = V + base_off;
    for (int64_t i = 0; i < T; ++i) {
      rope_row(Q + base_off + i * D, i, D, rope_base, qh);
      for (int d = 0; d < D; ++d) qh[d] = (real)s * qh[d];
      int n = members_of(i, W, S, n_off, g, mb);
      real mx = -INFINITY;
      int any_nan = 0;
      for (int m = 0; m < n; ++m) {
        if (mb[m].nan_score) { sc[m] = (real)NAN; any_nan = 1; continue; }
        gather_row(Kr, &mb[m], D, row);
        sc[m] = dot(qh, row, D);
        if (beta && mb[m].kind == 2) sc[m] += beta[u * T + i];   /* log-prior */
        if (sc[m] > mx) mx = sc[m];
      }
      real sum = 0;
      for (int m = 0; m < n; ++m) {
        sc[m] = any_nan ? (real)NAN : (real)exp((double)(sc[m] - mx));
        sum += sc[m];
      }
      real* o = O + base_off + i * D;
      for (int d = 0; d < D; ++d) o[d] = 0;
      for (int m = 0; m < n; ++m) {
        real pm = sc[m] / sum;
        sc[m] = pm;
        if (mb[m].nan_score) { for (int d = 0; d < D; ++d) o[d] = (real)NAN; continue; }
        gather_row(Vu, &mb[m], D, row);
        for (int d = 0; d < D; ++d) o[d] += pm * row[d];
      }
      if (LSE) LSE[u * T + i] = any_nan ? (real)NAN : mx + (real)log((double)sum);
      if (P) {
        real* pr = P + (u * T + i) * n_slots;
        for (int m = 0; m < n_slots; ++m) pr[m] = 0;
        for (int m = 0; m < n; ++m) pr[mb[m].slot] = sc[m];
      }
    }
  done:
    free(Kr); free(qh); free(row); free(mb); free(sc);
  }
  return err ? -2 : 0;
}

/*
 * Backward of the forward above for an upstream gradient dO, by the chain
 * rule written out member by member and scattered onto the rows each member
 * read.  Outputs dQ, dK, dV ([L][B][H][T][D], overwritten) and dalpha[L]
 * (overwritten): the gradient to each layer's alpha through the interpolation
 * weight w = alpha*f - floor(alpha*f), dw/dalpha = f ("Implementation": the
 * interpolation exists so that gradients reach alpha).  floor() is held fixed
 * (the right derivative at integer d); a second row i-lo-1 < 0 contributes 0.
 * beta (may be NULL): the forward's log-prior; dbeta (may be NULL) receives
 * its gradient [L][B][H][T].  dalpha_units (may be NULL) receives each
 * (layer, batch, head) unit's own share of dalpha, [L][B][H]: the terms that
 * dalpha[l] sums in fixed order.
 */
int FN(oracle_bwd)(int L, int B, int H, int T, int D, int W, int n_off,
                   const int32_t* offsets, int S, double rope_base, double scale,
                   const float* alpha, const real* Q, const real* K, const real* V,
                   const real* dO, real* dQ, real* dK, real* dV, real* dalpha,
                   const real* beta, real* dbeta, real* dalpha_units) {
  prob_t p = {L, B, H, T, D, W, n_off, S, rope_base, scale, offsets, alpha};
  if (check(&p)) return -1;
  const double s = scale > 0 ? scale : 1.0 / sqrt((double)D);
  const int n_slots = W + S + n_off;
  const int64_t units = (int64_t)L * B * H;
  real* dal_unit = (real*)calloc((size_t)units, sizeof(real));
  if (!dal_unit) return -2;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
  for (int64_t u = 0; u < units; ++u) {
    const int l = (int)(u / ((int64_t)B * H));
    geom_t g[ORACLE_MAX_OFFSETS];
    for (int k = 0; k < n_off; ++k) g[k] = geometry(alpha[l], offsets[k]);
    const int64_t base_off = u * (int64_t)T * D;
    const real* Vu = V + base_off;
    real* Kr = (real*)malloc(sizeof(real) * (size_t)T * D);
    real* dKr = (real*)calloc((size_t)T * D, sizeof(real));
    real* qh = (real*)malloc(sizeof(real) * D);
    real* dqh = (real*)malloc(sizeof(real) * D);
    real* krow = (real*)malloc(sizeof(real) * (size_t)n_slots * D);
    real* vrow = (real*)malloc(sizeof(real) * (size_t)n_slots * D);
    member_t* mb = (member_t*)malloc(sizeof(member_t) * (size_t)n_slots);
    real* sc = (real*)malloc(sizeof(real) * (size_t)n_slots);
    real* dp = (real*)malloc(sizeof(real) * (size_t)n_slots);
    real dal = 0;
    if (!Kr || !dKr || !qh || !dqh || !krow || !vrow || !mb || !sc || !dp) { err |= 1; goto done; }
    real* dVu = dV + base_off;
    {
      int bad = 0;
      for (int k = 0; k < n_off; ++k) bad |= !g[k].ok;
      if (bad) { /* every query of this layer has a NaN member */
        for (int64_t e = 0; e < (int64_t)T * D; ++e)
          dQ[base_off + e] = dK[base_off + e] = dVu[e] = (real)NAN;
        dal_unit[u] = (real)NAN;
        if (dbeta)
          for (int64_t i = 0; i < T; ++i) dbeta[u * T + i] = (real)NAN;
        goto done;
      }
    }
    rotate_unit(K + base_off, T, D, rope_base, Kr);
    for (int64_t e = 0; e < (int64_t)T * D; ++e) dVu[e] = 0;
    for (int64_t i = 0; i < T; ++i) {
      const real* go = dO + base_off + i * D;
      rope_row(Q + base_off + i * D, i, D, rope_base, qh);
      for (int d = 0; d < D; ++d) qh[d] = (real)s * qh[d];
      int n = members_of(i, W, S, n_off, g, mb);
      /* forward recomputation: interpolated key/value rows, scores, softmax */
      real mx = -INFINITY;
      for (int m = 0; m < n; ++m) {
        gather_row(Kr, &mb[m], D, krow + m * D);
        gather_row(Vu, &mb[m], D, vrow + m * D);
        sc[m] = dot(qh, krow + m * D, D);
        if (beta && mb[m].kind == 2) sc[m] += beta[u * T + i];   /* log-prior */
        if (sc[m] > mx) mx = sc[m];
      }
      real sum = 0;
      for (int m = 0; m < n; ++m) { sc[m] = (real)exp((double)(sc[m] - mx)); sum += sc[m]; }
      for (int m = 0; m < n; ++m) sc[m] /= sum;             /* sc = p */
      /* dp_m = dO . v_m ; Dsum = sum_m p_m dp_m ; dsigma_m = p_m (dp_m - Dsum) */
      real Dsum = 0;
      for (int m = 0; m < n; ++m) { dp[m] = dot(go, vrow + m * D, D); Dsum += sc[m] * dp[m]; }
      for (int d = 0; d < D; ++d) dqh[d] = 0;
      real dbet = 0;    /* d score of each offset member, summed: d beta_i */
      for (int m = 0; m < n; ++m) {
        const real pm = sc[m];
        const real gs = pm * (dp[m] - Dsum);
        if (mb[m].kind == 2) dbet += gs;
        const real* kr = krow + m * D;
        for (int d = 0; d < D; ++d) dqh[d] += gs * kr[d];
        /* scatter onto the rows the member read */
        for (int d = 0; d < D; ++d) {
          dKr[mb[m].a * D + d] += mb[m].wa * gs * qh[d];
          dVu[mb[m].a * D + d] += mb[m].wa * pm * go[d];
          if (mb[m].b >= 0) {
            dKr[mb[m].b * D + d] += mb[m].wb * gs * qh[d];
            dVu[mb[m].b * D + d] += mb[m].wb * pm * go[d];
          }
        }
        /* d alpha through w: d sigma/dw = q.(K[b]-K[a]); d v/dw = V[b]-V[a] */
        if (mb[m].kind == 2) {
          const int64_t rb = i - g[mb[m].k].lo - 1;
          if (rb >= 0) {
            const real* ka = Kr + mb[m].a * D;
            const real* kb = Kr + rb * D;
            const real* va = Vu + mb[m].a * D;
            const real* vb = Vu + rb * D;
            real t = 0;
            for (int d = 0; d < D; ++d)
              t += gs * qh[d] * (kb[d] - ka[d]) + pm * go[d] * (vb[d] - va[d]);
            dal += (real)g[mb[m].k].f * t;
          }
        }
      }
      /* q_hat = s * R_i Q_i  ->  dQ_i = s * R_i^T dq_hat */
      rope_row_t(dqh, i, D, rope_base, dQ + base_off + i * D);
      for (int d = 0; d < D; ++d) dQ[base_off + i * D + d] *= (real)s;
      if (dbeta) dbeta[u * T + i] = dbet;
    }
    for (int64_t j = 0; j < T; ++j) rope_row_t(dKr + j * D, j, D, rope_base, dK + base_off + j * D);
    dal_unit[u] = dal;
  done:
    free(Kr); free(dKr); free(qh); free(dqh); free(krow); free(vrow);
    free(mb); free(sc); free(dp);
  }
  for (int l = 0; l < L; ++l) {
    real acc = 0;
    for (int64_t r = 0; r < (int64_t)B * H; ++r) acc += dal_unit[(int64_t)l * B * H + r];
    dalpha[l] = acc;
  }
  if (dalpha_units)
    for (int64_t u = 0; u < units; ++u) dalpha_units[u] = dal_unit[u];
  free(dal_unit);
  return err ? -2 : 0;
}

/*
 * Single-token decode: for every unit, the output of one query q1 at
 * position pos against K/V rows 0..pos (the attended set of query pos,
 * "Attended set"; rows after pos are never touched).  Q1 and O1 are
 * [L][B][H][D]; K and V are [L][B][H][T][D] with pos < T; LSE1 is
 * [L][B][H] (may be NULL).  Each key row a member reads is rotated at its own
 * position, one member at a time.  beta1 (may be NULL): the new query's
 * log-prior on its offset members, [L][B][H].
 */
int FN(oracle_decode)(int L, int B, int H, int T, int D, int W, int n_off,
                      const int32_t* offsets, int S, double rope_base, double scale,
                      const float* alpha, int64_t pos, const real* Q1, const real* K,
                      const real* V, real* O1, real* LSE1, const real* beta1) {
  prob_t p = {L, B, H, T, D, W, n_off, S, rope_base, scale, offsets, alpha};
  if (check(&p) || pos < 0 || pos >= T) return -1;
  const double s = scale > 0 ? scale : 1.0 / sqrt((double)D);
  const int n_slots = W + S + n_off;
  const int64_t units = (int64_t)L * B * H;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
  for (int64_t u = 0; u < units; ++u) {
    const int l = (int)(u / ((int64_t)B * H));
    geom_t g[ORACLE_MAX_OFFSETS];
    for (int k = 0; k < n_off; ++k) g[k] = geometry(alpha[l], offsets[k]);
    const real* Ku = K + u * (int64_t)T * D;
    const real* Vu = V + u * (int64_t)T * D;
    real* qh = (real*)malloc(sizeof(real) * D);
    real* ka = (real*)malloc(sizeof(real) * D);
    real* kb = (real*)malloc(sizeof(real) * D);
    member_t* mb = (member_t*)malloc(sizeof(member_t) * (size_t)n_slots);
    real* sc = (real*)malloc(sizeof(real) * (size_t)n_slots);
    if (!qh || !ka || !kb || !mb || !sc) { err |= 1; goto done; }
    rope_row(Q1 + u * D, pos, D, rope_base, qh);
    for (int d = 0; d < D; ++d) qh[d] = (real)s * qh[d];
    int n = members_of(pos, W, S, n_off, g, mb);
    real mx = -INFINITY;
    int any_nan = 0;
    for (int m = 0; m < n; ++m) {
      if (mb[m].nan_score) { sc[m] = (real)NAN; any_nan = 1; continue; }
      rope_row(Ku + mb[m].a * D, mb[m].a, D, rope_base, ka);
      real v = mb[m].wa * dot(qh, ka, D);
      if (mb[m].b >= 0) {
        rope_row(Ku + mb[m].b * D, mb[m].b, D, rope_base, kb);
        v += mb[m].wb * dot(qh, kb, D);
      }
      if (beta1 && mb[m].kind == 2) v += beta1[u];   /* log-prior */
      sc[m] = v;
      if (v > mx) mx = v;
    }
    real sum = 0;
    for (int m = 0; m < n; ++m) {
      sc[m] = any_nan ? (real)NAN : (real)exp((double)(sc[m] - mx));
      sum += sc[m];
    }
    real* o = O1 + u * D;
    for (int d = 0; d < D; ++d) o[d] = 0;
    for (int m = 0; m < n; ++m) {
      if (mb[m].nan_score) { for (int d = 0; d < D; ++d) o[d] = (real)NAN; continue; }
      const real pm = sc[m] / sum;
      gather_row(Vu, &mb[m], D, ka);
      for (int d = 0; d < D; ++d) o[d] += pm * ka[d];
    }
    if (LSE1) LSE1[u] = any_nan ? (real)NAN : mx + (real)log((double)sum);
  done:
    free(qh); free(ka); free(kb); free(mb); free(sc);
  }
  return err ? -2 : 0;
}

/*
 * Learned-alpha parametrisation ("Scaling": alpha is constrained to
 * [0.5, 1.5]; "Experimental variables": the learned schedule has one free
 * parameter theta per layer, initialised at alpha = 1).  The page gives no
 * map; the reading taken is alpha = 0.5 + sigmoid(theta), and the gradient
 * follows by the chain rule: dtheta = dalpha * sigmoid(theta) (1 - sigmoid(theta)).
 */
void FN(oracle_alpha_from_theta)(int L, const real* theta, real* alpha) {
  for (int l = 0; l < L; ++l) alpha[l] = (real)(0.5 + 1.0 / (1.0 + exp(-(double)theta[l])));
}

void FN(oracle_dtheta)(int L, const real* theta, const real* dalpha, real* dtheta) {
  for (int l = 0; l < L; ++l) {
    const double s = 1.0 / (1.0 + exp(-(double)theta[l]));
    dtheta[l] = (real)((double)dalpha[l] * s * (1.0 - s));
  }
}

/* Exposed for the pins: the geometry of one (alpha, f) and RoPE of one row. */
int FN(oracle_geometry)(float alpha, int32_t f, int64_t* lo, double* w, int64_t* c) {
  geom_t g = geometry(alpha, f);
  *lo = g.lo; *w = g.w; *c = g.c;
  return g.ok;
}

void FN(oracle_rope)(const real* x, int64_t pos, int D, double base, real* out) {
  rope_row(x, pos, D, base, out);
}
