/*
 * s2attn_oracle.c -- plain fp64 CPU oracle for shifted short attention (S^2-Attn)
 * and for RoPE with position interpolation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, __graft_entry__.smoke() and bench.py's CPU-baseline
 * leg do.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (sources are the LongLoRA pages):
 *   - "LongLoRA paper notes" (smallflyingpig blog), section 3.3 S^2-Attn: the
 *     length-L sequence is cut into groups of L/g tokens and attention runs only
 *     inside a group; the shift-by-half-a-group drawing (groups 1-4, 5-8, 9-12
 *     become 3-6, 7-10, 11-14).
 *   - "LLaMA2 context to 100k" (nearauto.com), section "shift short attention":
 *     the two steps (1) shift the tokens of half of the attention heads,
 *     (2) move the features from the token dimension to the batch dimension.
 *   - python88.com article, mechanism paragraph: heads are split into two halves,
 *     and the shifted half gives the exchange between neighbouring groups.
 *   - "LongLoRA paper notes", section 3.4: position interpolation maps positions
 *     [0, L) onto [0, L0).
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - heads h >= H - shift_heads are shifted by s = G/2, the others by 0;
 *   - the roll is cyclic: rolled row r holds original token (r + s) mod N;
 *   - attention is causal inside a group, in rolled order; scale 1/sqrt(D);
 *   - lse = natural log of sum_j exp(scale * q.k_j) over the unmasked keys,
 *     stored at the ORIGINAL token index;
 *   - RoPE pairs element i with element i + D/2, theta_i = base^(-2i/D), and the
 *     interpolated position of token t is t * pos_scale.
 *
 * Everything is written out step by step: explicit gather of the rolled rows,
 * explicit causal loop, explicit softmax, explicit un-roll (scatter).  The
 * backward pass is the analytic gradient of softmax attention:
 *   P = softmax(S), dV = P^T dO, dP = dO V^T, dS = P o (dP - rowsum(P o dP)),
 *   dQ = scale dS K, dK = scale dS^T Q.
 * Loops over rows are split across OpenMP threads; each row's arithmetic is the
 * plain sequential sum.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (see oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F64 = 0, ORACLE_F32 = 1, ORACLE_BF16 = 2 };

/* ---- element access ------------------------------------------------------ */

static double widen(const void *p, size_t i, int dtype) {
  if (dtype == ORACLE_F64) return ((const double *)p)[i];
  if (dtype == ORACLE_F32) return (double)((const float *)p)[i];
  /* bf16: the upper 16 bits of an IEEE binary32 */
  uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ---- the head partition and the roll ------------------------------------- */

/* Shift of head h: the last `shift_heads` heads are shifted by half a group. */
static long head_shift(int h, int H, int G, int shift_heads) {
  return (h >= H - shift_heads) ? (long)(G / 2) : 0L;
}

/* Rolled row r of a head with shift s holds original token (r + s) mod N. */
static long rolled_to_token(long r, long s, long N) { return (r + s) % N; }

static size_t idx_bnhd(long b, long t, long h, long d, long N, long H, long D) {
  return (size_t)(((b * N + t) * H + h) * D + d);
}

/* Step (1)+(2): gather the G rows of group j of head h, in rolled order, into a
 * dense G x D fp64 block (the group becomes its own "batch" entry).  tok[i]
 * receives the original token index of local row i. */
static void gather_group(const void *X, int dtype, int N, int H, int D, int G,
                         long s, int b, int h, int j, double *out, long long *tok) {
  for (int i = 0; i < G; ++i) {
    long r = (long)j * G + i;
    long t = rolled_to_token(r, s, N);
    if (tok) tok[i] = t;
    for (int d = 0; d < D; ++d) out[(size_t)i * D + d] = widen(X, idx_bnhd(b, t, h, d, N, H, D), dtype);
  }
}

static double dot(const double *a, const double *b, int D) {
  double acc = 0.0;
  for (int d = 0; d < D; ++d) acc += a[d] * b[d];
  return acc;
}

/* ---- forward: one query row of one group ---------------------------------- */

/* Row i of the group (rolled-local index).  Keys i' <= i are visible (causal in
 * rolled order); keys i' > i are masked out.  Writes o_row (D), returns lse. */
static double fwd_row(const double *Qr, const double *Kr, const double *Vr, int D, int i,
                      double scale, double *S, double *o_row) {
  double m = -INFINITY;
  for (int kk = 0; kk <= i; ++kk) {
    S[kk] = scale * dot(Qr + (size_t)i * D, Kr + (size_t)kk * D, D);
    if (S[kk] > m) m = S[kk];
  }
  double l = 0.0;
  for (int kk = 0; kk <= i; ++kk) l += exp(S[kk] - m);
  for (int d = 0; d < D; ++d) o_row[d] = 0.0;
  for (int kk = 0; kk <= i; ++kk) {
    double p = exp(S[kk] - m) / l;
    for (int d = 0; d < D; ++d) o_row[d] += p * Vr[(size_t)kk * D + d];
  }
  return m + log(l);
}

/* ---- backward pieces ------------------------------------------------------ */

/* For query row i: P_i = exp(S_i - lse_i), dP_i = dO_i V^T, delta_i = sum P dP,
 * dS_i = P (dP - delta_i), dQ_i = scale * dS_i K.  Returns delta_i. */
static double bwd_query_row(const double *Qr, const double *Kr, const double *Vr,
                            const double *dOr, int D, int i, double scale, double lse_i,
                            double *P, double *dP, double *dq_row) {
  double delta = 0.0;
  for (int kk = 0; kk <= i; ++kk) {
    P[kk] = exp(scale * dot(Qr + (size_t)i * D, Kr + (size_t)kk * D, D) - lse_i);
    dP[kk] = dot(dOr + (size_t)i * D, Vr + (size_t)kk * D, D);
    delta += P[kk] * dP[kk];
  }
  if (dq_row) {
    for (int d = 0; d < D; ++d) dq_row[d] = 0.0;
    for (int kk = 0; kk <= i; ++kk) {
      double ds = P[kk] * (dP[kk] - delta);
      for (int d = 0; d < D; ++d) dq_row[d] += scale * ds * Kr[(size_t)kk * D + d];
    }
  }
  return delta;
}

/* For key row kk: the queries that see it are i = kk .. G-1.
 * dV_kk = sum_i P[i,kk] dO_i ;  dK_kk = scale * sum_i dS[i,kk] Q_i. */
static void bwd_key_row(const double *Qr, const double *Kr, const double *Vr,
                        const double *dOr, int D, int G, int kk, double scale,
                        const double *lse, const double *delta, double *dk_row, double *dv_row) {
  for (int d = 0; d < D; ++d) { dk_row[d] = 0.0; dv_row[d] = 0.0; }
  for (int i = kk; i < G; ++i) {
    double p = exp(scale * dot(Qr + (size_t)i * D, Kr + (size_t)kk * D, D) - lse[i]);
    double dp = dot(dOr + (size_t)i * D, Vr + (size_t)kk * D, D);
    double ds = p * (dp - delta[i]);
    for (int d = 0; d < D; ++d) {
      dv_row[d] += p * dOr[(size_t)i * D + d];
      dk_row[d] += scale * ds * Qr[(size_t)i * D + d];
    }
  }
}

static int check_shape(int B, int N, int H, int D, int G, int shift_heads) {
  if (B < 1 || N < 1 || H < 1 || D < 1 || G < 1) return -1;
  if (N % G != 0) return -1;
  if (shift_heads < 0 || shift_heads > H) return -1;
  if (shift_heads > 0 && (G % 2) != 0) return -1;
  return 0;
}

/* ---- public: one group, selected rows -------------------------------------- */

/*
 * Computes, for group j of head h in batch b:
 *   for each rolled-local query row qrows[a]:  o[a][:], lse[a], and (if dout) dq[a][:]
 *   for each rolled-local key row krows[a] (needs dout): dk[a][:], dv[a][:]
 * qtok / ktok receive the original token index of each row (the un-roll map).
 * Inputs are [B,N,H,D] arrays of the given dtype.  Returns 0, or -1 on bad args.
 */
int oracle_s2attn_unit(int dtype, const void *q, const void *k, const void *v, const void *dout,
                       int B, int N, int H, int D, int G, int shift_heads, int b, int h, int j,
                       const int *qrows, int nq, const int *krows, int nk,
                       double *o, double *lse, double *dq, double *dk, double *dv,
                       long long *qtok, long long *ktok) {
  if (check_shape(B, N, H, D, G, shift_heads)) return -1;
  if (b < 0 || b >= B || h < 0 || h >= H || j < 0 || j >= N / G) return -1;
  if (nk > 0 && !dout) return -1;
  const double scale = 1.0 / sqrt((double)D);
  const long s = head_shift(h, H, G, shift_heads);
  double *Qr = malloc(sizeof(double) * (size_t)G * D);
  double *Kr = malloc(sizeof(double) * (size_t)G * D);
  double *Vr = malloc(sizeof(double) * (size_t)G * D);
  double *dOr = dout ? malloc(sizeof(double) * (size_t)G * D) : NULL;
  long long *tok = malloc(sizeof(long long) * (size_t)G);
  gather_group(q, dtype, N, H, D, G, s, b, h, j, Qr, tok);
  gather_group(k, dtype, N, H, D, G, s, b, h, j, Kr, NULL);
  gather_group(v, dtype, N, H, D, G, s, b, h, j, Vr, NULL);
  if (dout) gather_group(dout, dtype, N, H, D, G, s, b, h, j, dOr, NULL);

  int bad = 0;
  for (int a = 0; a < nq; ++a) if (qrows[a] < 0 || qrows[a] >= G) bad = 1;
  for (int a = 0; a < nk; ++a) if (krows[a] < 0 || krows[a] >= G) bad = 1;
  if (bad) { free(Qr); free(Kr); free(Vr); free(dOr); free(tok); return -1; }

#pragma omp parallel
  {
    double *S = malloc(sizeof(double) * (size_t)G);
    double *P = malloc(sizeof(double) * (size_t)G);
    double *dP = malloc(sizeof(double) * (size_t)G);
    double *tmp = malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
    for (int a = 0; a < nq; ++a) {
      int i = qrows[a];
      lse[a] = fwd_row(Qr, Kr, Vr, D, i, scale, S, o + (size_t)a * D);
      if (qtok) qtok[a] = tok[i];
      if (dout && dq) bwd_query_row(Qr, Kr, Vr, dOr, D, i, scale, lse[a], P, dP, dq + (size_t)a * D);
    }
    free(S); free(P); free(dP); free(tmp);
  }

  if (nk > 0) {
    /* dK/dV of key row kk need lse_i and delta_i of every query i >= kk. */
    int kmin = G;
    for (int a = 0; a < nk; ++a) if (krows[a] < kmin) kmin = krows[a];
    double *lse_all = calloc((size_t)G, sizeof(double));
    double *delta_all = calloc((size_t)G, sizeof(double));
#pragma omp parallel
    {
      double *S = malloc(sizeof(double) * (size_t)G);
      double *P = malloc(sizeof(double) * (size_t)G);
      double *dP = malloc(sizeof(double) * (size_t)G);
      double *orow = malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
      for (int i = kmin; i < G; ++i) {
        lse_all[i] = fwd_row(Qr, Kr, Vr, D, i, scale, S, orow);
        delta_all[i] = bwd_query_row(Qr, Kr, Vr, dOr, D, i, scale, lse_all[i], P, dP, NULL);
      }
      free(S); free(P); free(dP); free(orow);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int a = 0; a < nk; ++a) {
      int kk = krows[a];
      if (ktok) ktok[a] = tok[kk];
      bwd_key_row(Qr, Kr, Vr, dOr, D, G, kk, scale, lse_all, delta_all,
                  dk + (size_t)a * D, dv + (size_t)a * D);
    }
    free(lse_all); free(delta_all);
  }
  free(Qr); free(Kr); free(Vr); free(dOr); free(tok);
  return 0;
}

/* ---- public: whole tensors ------------------------------------------------ */

/* Forward over every group of every head; outputs are un-rolled back to the
 * original token order: o [B,N,H,D], lse [B,H,N]. */
int oracle_s2attn_fwd_full(int dtype, const void *q, const void *k, const void *v,
                           int B, int N, int H, int D, int G, int shift_heads,
                           double *o, double *lse) {
  if (check_shape(B, N, H, D, G, shift_heads)) return -1;
  int *rows = malloc(sizeof(int) * (size_t)G);
  for (int i = 0; i < G; ++i) rows[i] = i;
  double *ou = malloc(sizeof(double) * (size_t)G * D);
  double *lu = malloc(sizeof(double) * (size_t)G);
  long long *tok = malloc(sizeof(long long) * (size_t)G);
  int rc = 0;
  for (int b = 0; b < B && !rc; ++b)
    for (int h = 0; h < H && !rc; ++h)
      for (int j = 0; j < N / G && !rc; ++j) {
        rc = oracle_s2attn_unit(dtype, q, k, v, NULL, B, N, H, D, G, shift_heads, b, h, j,
                                rows, G, NULL, 0, ou, lu, NULL, NULL, NULL, tok, NULL);
        /* un-roll: row i of the group goes back to its original token */
        for (int i = 0; i < G; ++i) {
          long t = (long)tok[i];
          lse[((size_t)b * H + h) * N + t] = lu[i];
          for (int d = 0; d < D; ++d) o[idx_bnhd(b, t, h, d, N, H, D)] = ou[(size_t)i * D + d];
        }
      }
  free(rows); free(ou); free(lu); free(tok);
  return rc;
}

/* Backward over every group of every head: dq, dk, dv [B,N,H,D] in original order. */
int oracle_s2attn_bwd_full(int dtype, const void *q, const void *k, const void *v, const void *dout,
                           int B, int N, int H, int D, int G, int shift_heads,
                           double *dq, double *dk, double *dv) {
  if (check_shape(B, N, H, D, G, shift_heads)) return -1;
  int *rows = malloc(sizeof(int) * (size_t)G);
  for (int i = 0; i < G; ++i) rows[i] = i;
  size_t gd = (size_t)G * D;
  double *ou = malloc(sizeof(double) * gd), *lu = malloc(sizeof(double) * (size_t)G);
  double *dqu = malloc(sizeof(double) * gd), *dku = malloc(sizeof(double) * gd);
  double *dvu = malloc(sizeof(double) * gd);
  long long *qt = malloc(sizeof(long long) * (size_t)G), *kt = malloc(sizeof(long long) * (size_t)G);
  int rc = 0;
  for (int b = 0; b < B && !rc; ++b)
    for (int h = 0; h < H && !rc; ++h)
      for (int j = 0; j < N / G && !rc; ++j) {
        rc = oracle_s2attn_unit(dtype, q, k, v, dout, B, N, H, D, G, shift_heads, b, h, j,
                                rows, G, rows, G, ou, lu, dqu, dku, dvu, qt, kt);
        for (int i = 0; i < G; ++i)
          for (int d = 0; d < D; ++d) {
            dq[idx_bnhd(b, qt[i], h, d, N, H, D)] = dqu[(size_t)i * D + d];
            dk[idx_bnhd(b, kt[i], h, d, N, H, D)] = dku[(size_t)i * D + d];
            dv[idx_bnhd(b, kt[i], h, d, N, H, D)] = dvu[(size_t)i * D + d];
          }
      }
  free(rows); free(ou); free(lu); free(dqu); free(dku); free(dvu); free(qt); free(kt);
  return rc;
}

/* ---- decoding: full causal attention for the last M positions ------------- */

/*
 * Inference runs ordinary full attention, not S^2-Attn ("LongLoRA paper notes",
 * section 3.1; model.aibase.cn, features list).  A decoding step appends M new
 * tokens to a sequence of N positions: k, v [B,N,H,D] hold all N positions
 * (the new ones included), q [B,M,H,D] holds the M new queries, query m sits at
 * position N - M + m and sees the keys at positions 0 .. N - M + m.
 * Writes o [B,M,H,D] and lse [B,H,M] (natural log of sum_t exp(scale*q.k_t)).
 * Returns 0, or -1 on bad sizes (M < 1, M > N, ...).
 */
int oracle_decode(int dtype, const void *q, const void *k, const void *v,
                  int B, int M, int N, int H, int D, double *o, double *lse) {
  if (B < 1 || M < 1 || N < 1 || H < 1 || D < 1 || M > N) return -1;
  const double scale = 1.0 / sqrt((double)D);
#pragma omp parallel
  {
    double *qrow = malloc(sizeof(double) * (size_t)D);
    double *krow = malloc(sizeof(double) * (size_t)D);
    double *S = malloc(sizeof(double) * (size_t)N);
#pragma omp for collapse(3) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h)
        for (int m = 0; m < M; ++m) {
          const long pos = (long)N - M + m; /* last visible key */
          for (int d = 0; d < D; ++d) qrow[d] = widen(q, idx_bnhd(b, m, h, d, M, H, D), dtype);
          double mx = -INFINITY;
          for (long t = 0; t <= pos; ++t) {
            for (int d = 0; d < D; ++d) krow[d] = widen(k, idx_bnhd(b, t, h, d, N, H, D), dtype);
            S[t] = scale * dot(qrow, krow, D);
            if (S[t] > mx) mx = S[t];
          }
          double l = 0.0;
          for (long t = 0; t <= pos; ++t) l += exp(S[t] - mx);
          double *orow = o + idx_bnhd(b, m, h, 0, M, H, D);
          for (int d = 0; d < D; ++d) orow[d] = 0.0;
          for (long t = 0; t <= pos; ++t) {
            double p = exp(S[t] - mx) / l;
            for (int d = 0; d < D; ++d) orow[d] += p * widen(v, idx_bnhd(b, t, h, d, N, H, D), dtype);
          }
          lse[((size_t)b * H + h) * M + m] = mx + log(l);
        }
    free(qrow); free(krow); free(S);
  }
  return 0;
}

/* ---- RoPE with position interpolation ------------------------------------ */

/* fp64 reference.  Token t sits at interpolated position t * pos_scale; pair
 * (x_i, x_{i+D/2}) is rotated by angle pos * base^(-2i/D). */
void oracle_rope_pi_f64(const double *x, double *y, int B, int N, int H, int D,
                        double pos_scale, double base) {
  int half = D / 2;
#pragma omp parallel for collapse(2)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < N; ++t)
      for (int h = 0; h < H; ++h)
        for (int i = 0; i < half; ++i) {
          double theta = pow(base, -2.0 * (double)i / (double)D);
          double ang = ((double)t * pos_scale) * theta;
          double c = cos(ang), s = sin(ang);
          size_t i1 = idx_bnhd(b, t, h, i, N, H, D), i2 = idx_bnhd(b, t, h, i + half, N, H, D);
          double x1 = x[i1], x2 = x[i2];
          y[i1] = x1 * c - x2 * s;
          y[i2] = x2 * c + x1 * s;
        }
}

/* Round a binary32 to bfloat16, round-to-nearest-even (finite inputs). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/*
 * fp32 version, in this exact operation order (every step rounded to binary32):
 *   theta_i = (float) base^(-2i/D)            [pow in fp64, then rounded]
 *   a       = ((float)t * pos_scale) * theta_i
 *   c, s    = (float) cos((double)a), (float) sin((double)a)
 *   y1      = x1*c - x2*s ;  y2 = x2*c + x1*s  (products rounded before the sum)
 * then rounded to bf16 (nearest-even).  x and y are bf16 bit patterns [B,N,H,D];
 * in-place (x == y) is allowed.
 */
void oracle_rope_pi_f32_bf16_at(const uint16_t *x, uint16_t *y, int B, int N, int H, int D, int pos0,
                                float pos_scale, float base);

void oracle_rope_pi_f32_bf16(const uint16_t *x, uint16_t *y, int B, int N, int H, int D,
                             float pos_scale, float base) {
  oracle_rope_pi_f32_bf16_at(x, y, B, N, H, D, 0, pos_scale, base);
}

/* The same, for a tensor whose row t holds the token at position pos0 + t (the new tokens
 * of a decoding step): the position index is pos0 + t, everything else as above. */
void oracle_rope_pi_f32_bf16_at(const uint16_t *x, uint16_t *y, int B, int N, int H, int D, int pos0,
                                float pos_scale, float base) {
  int half = D / 2;
#pragma omp parallel for collapse(2)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < N; ++t) {
      float pos = (float)(pos0 + t) * pos_scale;
      for (int i = 0; i < half; ++i) {
        float theta = (float)pow((double)base, -2.0 * (double)i / (double)D);
        float a = pos * theta;
        float c = (float)cos((double)a);
        float s = (float)sin((double)a);
        for (int h = 0; h < H; ++h) {
          size_t i1 = idx_bnhd(b, t, h, i, N, H, D), i2 = idx_bnhd(b, t, h, i + half, N, H, D);
          float x1 = bf16_to_f32(x[i1]), x2 = bf16_to_f32(x[i2]);
          float p1 = x1 * c, p2 = x2 * s, p3 = x2 * c, p4 = x1 * s;
          float y1 = p1 - p2, y2 = p3 + p4;
          y[i1] = f32_to_bf16_rne(y1);
          y[i2] = f32_to_bf16_rne(y2);
        }
      }
    }
}
