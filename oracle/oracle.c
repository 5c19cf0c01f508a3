/*
 * oracle.c -- plain, slow, fp64 CPU model of the ReplaySSM SSM-layer decode
 * step.  TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
 * benchmark).  The product path never includes, links or calls it, and it
 * shares no source with the CUDA library.
 *
 * Source tags ([sitech], [hamidun], [felizola], [Dao & Gu 2024],
 * [Yang et al. 2025], [OCP MX v1.0]) are expanded in oracle.h.
 *
 * What the pages fix, and what this file does with it:
 *   - The state of every (sequence, head) is a checkpoint plus a buffer of the
 *     most recent input records; a non-flush step appends the current record
 *     and produces the output from checkpoint + buffer without writing the
 *     state; when the 16-record buffer is full, a flush step folds the
 *     buffered inputs into a new checkpoint, written once, and empties the
 *     buffer.  Outputs equal conventional decoding up to rounding.
 *     [sitech §How ReplaySSM works], [felizola ¶2]
 *   - Conventional decoding reads and writes the whole state at every step;
 *     over a 16-token window that is 16 reads and 16 writes, against one
 *     checkpoint write for ReplaySSM.  [sitech §How ReplaySSM works,
 *     §Reducing state traffic and simplifying rollback]
 *   - Speculative drafts are appended to the buffer and evaluated output-only;
 *     the accepted prefix is committed with no snapshot/restore of state.
 *     [sitech §Reducing state traffic...], [felizola ¶3]
 *   - A high-precision checkpoint feeds the recurrence while a low-precision
 *     copy serves reads, so read error does not enter the recurrence.
 *     [sitech §Bounding quantisation error]
 *   - Layer types: Mamba-2, Gated DeltaNet (KDA not modelled).
 *     [hamidun §Why hybrid models became the norm]
 *
 * The recurrences themselves are not on the pages; the standard published
 * forms are used: Mamba-2 [Dao & Gu 2024], gated delta rule [Yang et al. 2025].
 * The replay output formulas below are obtained by unrolling those recurrences
 * from the checkpoint; the fold is done by literally stepping the recurrence
 * record by record.  Decay products are formed as running products of the
 * per-step factors.  Nothing is blocked, fused or reordered beyond that.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define MAXCAP 256

static size_t ix2(size_t a, size_t na, size_t b) { (void)na; return a * na + b; }

/* ===================================================================== */
/*                               Mamba-2                                  */
/* ===================================================================== */

/* One token of the Mamba-2 selective state update on one head, as in
 * [Dao & Gu 2024]:  dA = exp(dt*A);  S[p][n] <- dA*S[p][n] + dt*x[p]*B[n].
 * dt is already post-softplus; A is the scalar decay rate of the head. */
static void m2_step(int P, int N, double *s, const double *x, double dt,
                    const double *Bv, double A) {
  const double dA = exp(dt * A);
  for (int p = 0; p < P; ++p)
    for (int n = 0; n < N; ++n)
      s[(size_t)p * N + n] = dA * s[(size_t)p * N + n] + dt * x[p] * Bv[n];
}

/* Mamba-2 output read from a state:  y[p] = sum_n S[p][n]*C[n] + D*x[p]. */
static void m2_out(int P, int N, const double *s, const double *Cv,
                   const double *x, double D, double *y) {
  for (int p = 0; p < P; ++p) {
    double acc = 0.0;
    for (int n = 0; n < N; ++n) acc += s[(size_t)p * N + n] * Cv[n];
    y[p] = acc + D * x[p];
  }
}

/* Output of a replay step from the checkpoint read view and k >= 1 buffered
 * records (record k-1 is the current token).  Unrolling the recurrence from
 * the checkpoint h0 gives, with dA_i = exp(dt_i*A):
 *   S_k = (prod_{m<=k} dA_m) h0 + sum_{i<=k} (prod_{i<m<=k} dA_m) dt_i x_i B_i^T
 * hence
 *   y_k = (prod_{m<=k} dA_m) (h0 C_k) + sum_i (prod_{i<m<=k} dA_m) dt_i (B_i.C_k) x_i
 *         + D x_k.
 * The decay products are running products built from the newest record back.
 * [sitech §How ReplaySSM works]: output from checkpoint + buffer, no state write. */
static void m2_replay_out(int P, int N, int k, const double *view,
                          const double *rx, const double *rdt,
                          const double *rB, const double *rC, double A,
                          double D, double *y) {
  double coef[MAXCAP], bc[MAXCAP];
  const double *Ck = rC + (size_t)(k - 1) * N;
  const double *xk = rx + (size_t)(k - 1) * P;
  coef[k - 1] = 1.0;
  for (int i = k - 2; i >= 0; --i) coef[i] = coef[i + 1] * exp(rdt[i + 1] * A);
  const double lam = coef[0] * exp(rdt[0] * A);
  for (int i = 0; i < k; ++i) {
    double acc = 0.0;
    for (int n = 0; n < N; ++n) acc += rB[(size_t)i * N + n] * Ck[n];
    bc[i] = acc;
  }
  for (int p = 0; p < P; ++p) {
    double hc = 0.0;
    for (int n = 0; n < N; ++n) hc += view[(size_t)p * N + n] * Ck[n];
    double acc = lam * hc;
    for (int i = 0; i < k; ++i) acc += coef[i] * rdt[i] * bc[i] * rx[(size_t)i * P + p];
    y[p] = acc + D * xk[p];
  }
}

/* Flush fold: the new checkpoint is the state reached by stepping the
 * recurrence through the k buffered records from h0.  [sitech §How ReplaySSM
 * works]: the buffered inputs are folded into a new checkpoint. */
static void m2_fold(int P, int N, double *h0, int k, const double *rx,
                    const double *rdt, const double *rB, double A) {
  for (int i = 0; i < k; ++i)
    m2_step(P, N, h0, rx + (size_t)i * P, rdt[i], rB + (size_t)i * N, A);
}

/* Read view of a checkpoint (see make_view below). */
static void make_view(int fmt, int rows, int cols, const double *h, double *view);
static void quant_ckpt_tile(int fmt, int rows, int cols, double *h);

int oracle_m2_conventional(int T, int B, int H, int P, int N, int G, double *S,
                           const double *x, const double *dt, const double *Bm,
                           const double *Cm, const double *A, const double *D,
                           double *y, long long *reads, long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
  const int hpg = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const int g = h / hpg;
      const size_t bh = ix2(b, H, h);
      double *s = S + bh * P * N;
      for (int t = 0; t < T; ++t) {
        const size_t tbh = (size_t)t * B * H + bh;
        const size_t tbg = ((size_t)t * B + b) * G + g;
        /* conventional decode: the whole state is read, updated and written
         * back at every step [sitech §How ReplaySSM works] */
        reads[bh] += 1;
        m2_step(P, N, s, x + tbh * P, dt[tbh], Bm + tbg * N, A[h]);
        writes[bh] += 1;
        m2_out(P, N, s, Cm + tbg * N, x + tbh * P, D[h], y + tbh * P);
      }
    }
  return 0;
}

int oracle_m2_replay(int T, int B, int H, int P, int N, int G, int L, int cap,
                     int read_fmt, int ckpt_fmt, double *h0, double *rec_x,
                     double *rec_dt, double *rec_B, double *rec_C, int *len,
                     const double *x, const double *dt, const double *Bm,
                     const double *Cm, const double *A, const double *D,
                     double *y, int *len_trace, int *flush_trace,
                     long long *reads, long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
  if (L <= 0 || cap < L || cap > MAXCAP) return -1;
  if (read_fmt && ckpt_fmt) return -1;
  const int hpg = H / G;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const int g = h / hpg;
      const size_t bh = ix2(b, H, h);
      double *hh = h0 + bh * P * N;
      double *rx = rec_x + bh * cap * P, *rdt = rec_dt + bh * cap;
      double *rB = rec_B + bh * cap * N, *rC = rec_C + bh * cap * N;
      double *view = hh;
      double *vbuf = NULL;
      if (read_fmt) {
        vbuf = (double *)malloc(sizeof(double) * P * N);
        make_view(read_fmt, P, N, hh, vbuf);
        view = vbuf;
      }
      int n = len[bh];
      if (n < 0 || n >= L) { bad |= 1; free(vbuf); continue; }
      for (int t = 0; t < T; ++t) {
        const size_t tbh = (size_t)t * B * H + bh;
        const size_t tbg = ((size_t)t * B + b) * G + g;
        /* append the current input record at slot n [sitech §How ReplaySSM works] */
        memcpy(rx + (size_t)n * P, x + tbh * P, sizeof(double) * P);
        rdt[n] = dt[tbh];
        memcpy(rB + (size_t)n * N, Bm + tbg * N, sizeof(double) * N);
        memcpy(rC + (size_t)n * N, Cm + tbg * N, sizeof(double) * N);
        n += 1;
        /* output from checkpoint view + buffer; the checkpoint is read once */
        reads[bh] += 1;
        m2_replay_out(P, N, n, view, rx, rdt, rB, rC, A[h], D[h], y + tbh * P);
        int flushed = 0;
        if (n == L) {
          /* the buffer is full: fold, write the checkpoint once, clear */
          m2_fold(P, N, hh, n, rx, rdt, rB, A[h]);
          if (ckpt_fmt) quant_ckpt_tile(ckpt_fmt, P, N, hh);
          if (read_fmt) make_view(read_fmt, P, N, hh, vbuf);
          writes[bh] += 1;
          n = 0;
          flushed = 1;
        }
        if (len_trace) len_trace[tbh] = n;
        if (flush_trace) flush_trace[tbh] = flushed;
      }
      len[bh] = n;
      free(vbuf);
    }
  return bad ? -1 : 0;
}

int oracle_m2_flush(int B, int H, int P, int N, int L, int cap, int force,
                    int ckpt_fmt, double *h0, const double *rec_x,
                    const double *rec_dt, const double *rec_B, int *len,
                    const double *A) {
  if (B < 0 || H <= 0 || P <= 0 || N <= 0 || L <= 0 || cap < L || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) { bad |= 1; continue; }
      if (n >= L || (force && n > 0)) {
        double *hh = h0 + bh * P * N;
        m2_fold(P, N, hh, n, rec_x + bh * cap * P, rec_dt + bh * cap,
                rec_B + bh * cap * N, A[h]);
        if (ckpt_fmt) quant_ckpt_tile(ckpt_fmt, P, N, hh);
        len[bh] = 0;
      }
    }
  return bad ? -1 : 0;
}

int oracle_m2_materialize(int B, int H, int P, int N, int cap, const double *h0,
                          const double *rec_x, const double *rec_dt,
                          const double *rec_B, const int *len, const double *A,
                          double *S_out) {
  if (B < 0 || H <= 0 || P <= 0 || N <= 0 || cap <= 0 || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) { bad |= 1; continue; }
      double *so = S_out + bh * P * N;
      memcpy(so, h0 + bh * P * N, sizeof(double) * P * N);
      m2_fold(P, N, so, n, rec_x + bh * cap * P, rec_dt + bh * cap,
              rec_B + bh * cap * N, A[h]);
    }
  return bad ? -1 : 0;
}

int oracle_m2_verify_replay(int R, int B, int H, int P, int N, int G, int L,
                            int cap, int Dn, double *h0, double *rec_x,
                            double *rec_dt, double *rec_B, double *rec_C,
                            int *len, const double *x, const double *dt,
                            const double *Bm, const double *Cm,
                            const double *A, const double *D, const int *acc,
                            double *y, int *len_trace) {
  if (R < 0 || B < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
  if (L <= 0 || Dn <= 0 || cap < L + Dn - 1 || cap > MAXCAP) return -1;
  const int hpg = H / G;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const int g = h / hpg;
      const size_t bh = ix2(b, H, h);
      double *hh = h0 + bh * P * N;
      double *rx = rec_x + bh * cap * P, *rdt = rec_dt + bh * cap;
      double *rB = rec_B + bh * cap * N, *rC = rec_C + bh * cap * N;
      int n = len[bh];
      for (int r = 0; r < R && !bad; ++r) {
        const int a = acc[(size_t)r * B + b];
        if (n < 0 || n >= L || n + Dn > cap || a < 0 || a > Dn) { bad |= 1; break; }
        /* drafts are appended to the buffer, after the committed records
         * [sitech §Reducing state traffic...] */
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          const size_t rbdg = (((size_t)r * B + b) * Dn + d) * G + g;
          memcpy(rx + (size_t)(n + d) * P, x + rbdh * P, sizeof(double) * P);
          rdt[n + d] = dt[rbdh];
          memcpy(rB + (size_t)(n + d) * N, Bm + rbdg * N, sizeof(double) * N);
          memcpy(rC + (size_t)(n + d) * N, Cm + rbdg * N, sizeof(double) * N);
        }
        /* output-only evaluation of every draft from checkpoint + buffer */
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          m2_replay_out(P, N, n + d + 1, hh, rx, rdt, rB, rC, A[h], D[h], y + rbdh * P);
        }
        /* commit the accepted prefix: the records are already in place, so
         * the buffer length simply advances; rejected drafts are left behind
         * to be overwritten [felizola ¶3] */
        n += a;
        if (n >= L) {
          m2_fold(P, N, hh, n, rx, rdt, rB, A[h]);
          n = 0;
        }
        if (len_trace) len_trace[(size_t)r * B * H + bh] = n;
      }
      len[bh] = n;
    }
  return bad ? -1 : 0;
}

int oracle_m2_verify_snapshot(int R, int B, int H, int P, int N, int G, int Dn,
                              double *S, const double *x, const double *dt,
                              const double *Bm, const double *Cm,
                              const double *A, const double *D, const int *acc,
                              double *y, long long *state_copies) {
  if (R < 0 || B < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G || Dn <= 0) return -1;
  const int hpg = H / G;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const int g = h / hpg;
      const size_t bh = ix2(b, H, h);
      double *s = S + bh * P * N;
      double *snap = (double *)malloc(sizeof(double) * P * N);
      for (int r = 0; r < R; ++r) {
        const int a = acc[(size_t)r * B + b];
        if (a < 0 || a > Dn) { bad |= 1; break; }
        /* conventional speculative decoding: snapshot the state, step through
         * the drafts, restore, then replay the accepted ones
         * [hamidun §Where the state problem appears] */
        memcpy(snap, s, sizeof(double) * P * N);
        state_copies[bh] += 1;
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          const size_t rbdg = (((size_t)r * B + b) * Dn + d) * G + g;
          m2_step(P, N, s, x + rbdh * P, dt[rbdh], Bm + rbdg * N, A[h]);
          m2_out(P, N, s, Cm + rbdg * N, x + rbdh * P, D[h], y + rbdh * P);
        }
        memcpy(s, snap, sizeof(double) * P * N);
        state_copies[bh] += 1;
        for (int d = 0; d < a; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          const size_t rbdg = (((size_t)r * B + b) * Dn + d) * G + g;
          m2_step(P, N, s, x + rbdh * P, dt[rbdh], Bm + rbdg * N, A[h]);
        }
      }
      free(snap);
    }
  return bad ? -1 : 0;
}

/* ===================================================================== */
/*                            Gated DeltaNet                              */
/* ===================================================================== */

/* One token of the gated delta rule on one head [Yang et al. 2025], with the
 * state S laid out [DK][DV] (key index = row):
 *   S <- alpha * (I - beta k k^T) S + beta k v^T,
 * evaluated through w = k^T S  (so (I - beta k k^T) S = S - beta k w^T). */
static void gdn_step(int DK, int DV, double *s, const double *kv,
                     const double *vv, double alpha, double beta, double *w) {
  for (int j = 0; j < DV; ++j) {
    double acc = 0.0;
    for (int r = 0; r < DK; ++r) acc += kv[r] * s[(size_t)r * DV + j];
    w[j] = acc;
  }
  for (int r = 0; r < DK; ++r)
    for (int j = 0; j < DV; ++j)
      s[(size_t)r * DV + j] =
          alpha * (s[(size_t)r * DV + j] - beta * kv[r] * w[j]) + beta * kv[r] * vv[j];
}

/* Output read from a state: o = scale * S^T q. */
static void gdn_out(int DK, int DV, const double *s, const double *qv,
                    double scale, double *o) {
  for (int j = 0; j < DV; ++j) {
    double acc = 0.0;
    for (int r = 0; r < DK; ++r) acc += s[(size_t)r * DV + j] * qv[r];
    o[j] = scale * acc;
  }
}

/* Output of a replay step from the checkpoint and k >= 1 buffered records
 * (record k-1 is the current token).  Unrolling the gated delta rule from h0,
 * with gamma_i = prod_{m<=i} alpha_m, the state after record i is
 *   S_i = gamma_i h0 + sum_{j<=i} (gamma_i/gamma_j) k_j u_j^T,
 *   u_i = beta_i ( v_i - gamma_i h0^T k_i - sum_{j<i} (gamma_i/gamma_j)(k_j.k_i) u_j ),
 * so the output needs only h0 and the records:
 *   o_k = scale * ( gamma_k h0^T q_k + sum_{i<=k} (gamma_k/gamma_i)(k_i.q_k) u_i ).
 * No intermediate state is formed (output-only evaluation, [sitech §Reducing
 * state traffic...]).  The ratios gamma_i/gamma_j are running products of the
 * alphas strictly after j up to i. */
static void gdn_replay_out(int DK, int DV, int kc, double scale,
                           const double *h0, const double *rq, const double *rk,
                           const double *rv, const double *ra, const double *rb,
                           double *o, double *u, double *z) {
  for (int i = 0; i < kc; ++i) {
    const double *ki = rk + (size_t)i * DK;
    double gi = 1.0;
    for (int m = 0; m <= i; ++m) gi *= ra[m];
    for (int j = 0; j < DV; ++j) {
      double acc = 0.0;
      for (int r = 0; r < DK; ++r) acc += h0[(size_t)r * DV + j] * ki[r];
      z[j] = acc;
    }
    double *ui = u + (size_t)i * DV;
    for (int j = 0; j < DV; ++j) ui[j] = rv[(size_t)i * DV + j] - gi * z[j];
    for (int jj = 0; jj < i; ++jj) {
      double ratio = 1.0;
      for (int m = jj + 1; m <= i; ++m) ratio *= ra[m];
      double kk = 0.0;
      for (int r = 0; r < DK; ++r) kk += rk[(size_t)jj * DK + r] * ki[r];
      for (int j = 0; j < DV; ++j) ui[j] -= ratio * kk * u[(size_t)jj * DV + j];
    }
    for (int j = 0; j < DV; ++j) ui[j] *= rb[i];
  }
  const double *qk = rq + (size_t)(kc - 1) * DK;
  double gk = 1.0;
  for (int m = 0; m < kc; ++m) gk *= ra[m];
  for (int j = 0; j < DV; ++j) {
    double acc = 0.0;
    for (int r = 0; r < DK; ++r) acc += h0[(size_t)r * DV + j] * qk[r];
    o[j] = gk * acc;
  }
  for (int i = 0; i < kc; ++i) {
    double ratio = 1.0;
    for (int m = i + 1; m < kc; ++m) ratio *= ra[m];
    double kq = 0.0;
    for (int r = 0; r < DK; ++r) kq += rk[(size_t)i * DK + r] * qk[r];
    for (int j = 0; j < DV; ++j) o[j] += ratio * kq * u[(size_t)i * DV + j];
  }
  for (int j = 0; j < DV; ++j) o[j] *= scale;
}

static void gdn_fold(int DK, int DV, double *h0, int kc, const double *rk,
                     const double *rv, const double *ra, const double *rb,
                     double *w) {
  for (int i = 0; i < kc; ++i)
    gdn_step(DK, DV, h0, rk + (size_t)i * DK, rv + (size_t)i * DV, ra[i], rb[i], w);
}

int oracle_gdn_conventional(int T, int B, int H, int DK, int DV, double scale,
                            double *S, const double *q, const double *k,
                            const double *v, const double *alpha,
                            const double *beta, double *o, long long *reads,
                            long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *s = S + bh * DK * DV;
      double *w = (double *)malloc(sizeof(double) * DV);
      for (int t = 0; t < T; ++t) {
        const size_t tbh = (size_t)t * B * H + bh;
        reads[bh] += 1;
        gdn_step(DK, DV, s, k + tbh * DK, v + tbh * DV, alpha[tbh], beta[tbh], w);
        writes[bh] += 1;
        gdn_out(DK, DV, s, q + tbh * DK, scale, o + tbh * DV);
      }
      free(w);
    }
  return 0;
}

int oracle_gdn_replay(int T, int B, int H, int DK, int DV, int L, int cap,
                      double scale, double *h0, double *rec_q, double *rec_k,
                      double *rec_v, double *rec_alpha, double *rec_beta,
                      int *len, const double *q, const double *k,
                      const double *v, const double *alpha, const double *beta,
                      double *o, int *len_trace, int *flush_trace,
                      long long *reads, long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0) return -1;
  if (L <= 0 || cap < L || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *hh = h0 + bh * DK * DV;
      double *rq = rec_q + bh * cap * DK, *rk = rec_k + bh * cap * DK;
      double *rv = rec_v + bh * cap * DV;
      double *ra = rec_alpha + bh * cap, *rb = rec_beta + bh * cap;
      double *u = (double *)malloc(sizeof(double) * cap * DV);
      double *z = (double *)malloc(sizeof(double) * DV);
      int n = len[bh];
      if (n < 0 || n >= L) { bad |= 1; free(u); free(z); continue; }
      for (int t = 0; t < T; ++t) {
        const size_t tbh = (size_t)t * B * H + bh;
        memcpy(rq + (size_t)n * DK, q + tbh * DK, sizeof(double) * DK);
        memcpy(rk + (size_t)n * DK, k + tbh * DK, sizeof(double) * DK);
        memcpy(rv + (size_t)n * DV, v + tbh * DV, sizeof(double) * DV);
        ra[n] = alpha[tbh];
        rb[n] = beta[tbh];
        n += 1;
        reads[bh] += 1;
        gdn_replay_out(DK, DV, n, scale, hh, rq, rk, rv, ra, rb, o + tbh * DV, u, z);
        int flushed = 0;
        if (n == L) {
          gdn_fold(DK, DV, hh, n, rk, rv, ra, rb, z);
          writes[bh] += 1;
          n = 0;
          flushed = 1;
        }
        if (len_trace) len_trace[tbh] = n;
        if (flush_trace) flush_trace[tbh] = flushed;
      }
      len[bh] = n;
      free(u);
      free(z);
    }
  return bad ? -1 : 0;
}

/* Speculative verify for Gated DeltaNet, replay form (the Mamba-2 round
 * carried over to the delta rule, [sitech §Reducing state traffic...]): per
 * round the Dn drafts are appended after the committed records, each draft's
 * output is evaluated from h0 and records 0..len+d with no intermediate
 * state, then the accepted prefix is committed by advancing len (rejected
 * drafts stay behind, to be overwritten), folding when len reaches L.
 * Drafts: q, k [R][B][Dn][H][DK], v [R][B][Dn][H][DV], alpha, beta
 * [R][B][Dn][H]; acc [R][B]; o [R][B][Dn][H][DV]; len_trace [R][B][H]. */
int oracle_gdn_verify_replay(int R, int B, int H, int DK, int DV, int L, int cap,
                             int Dn, double scale, double *h0, double *rec_q,
                             double *rec_k, double *rec_v, double *rec_alpha,
                             double *rec_beta, int *len, const double *q,
                             const double *k, const double *v,
                             const double *alpha, const double *beta,
                             const int *acc, double *o, int *len_trace) {
  if (R < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0) return -1;
  if (L <= 0 || Dn <= 0 || cap < L + Dn - 1 || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *hh = h0 + bh * DK * DV;
      double *rq = rec_q + bh * cap * DK, *rk = rec_k + bh * cap * DK;
      double *rv = rec_v + bh * cap * DV;
      double *ra = rec_alpha + bh * cap, *rb = rec_beta + bh * cap;
      double *u = (double *)malloc(sizeof(double) * cap * DV);
      double *z = (double *)malloc(sizeof(double) * DV);
      int n = len[bh];
      for (int r = 0; r < R && !bad; ++r) {
        const int a = acc[(size_t)r * B + b];
        if (n < 0 || n >= L || n + Dn > cap || a < 0 || a > Dn) { bad |= 1; break; }
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          memcpy(rq + (size_t)(n + d) * DK, q + rbdh * DK, sizeof(double) * DK);
          memcpy(rk + (size_t)(n + d) * DK, k + rbdh * DK, sizeof(double) * DK);
          memcpy(rv + (size_t)(n + d) * DV, v + rbdh * DV, sizeof(double) * DV);
          ra[n + d] = alpha[rbdh];
          rb[n + d] = beta[rbdh];
        }
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          gdn_replay_out(DK, DV, n + d + 1, scale, hh, rq, rk, rv, ra, rb, o + rbdh * DV, u, z);
        }
        n += a;
        if (n >= L) {
          gdn_fold(DK, DV, hh, n, rk, rv, ra, rb, z);
          n = 0;
        }
        if (len_trace) len_trace[(size_t)r * B * H + bh] = n;
      }
      len[bh] = n;
      free(u);
      free(z);
    }
  return bad ? -1 : 0;
}

/* The conventional comparison: snapshot the full state, step through the
 * drafts, restore, step through the accepted ones again
 * [hamidun §Where the state problem appears]. */
int oracle_gdn_verify_snapshot(int R, int B, int H, int DK, int DV, int Dn, double scale,
                               double *S, const double *q, const double *k,
                               const double *v, const double *alpha,
                               const double *beta, const int *acc, double *o,
                               long long *state_copies) {
  if (R < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0 || Dn <= 0) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *s = S + bh * DK * DV;
      double *snap = (double *)malloc(sizeof(double) * DK * DV);
      double *w = (double *)malloc(sizeof(double) * DV);
      for (int r = 0; r < R; ++r) {
        const int a = acc[(size_t)r * B + b];
        if (a < 0 || a > Dn) { bad |= 1; break; }
        memcpy(snap, s, sizeof(double) * DK * DV);
        state_copies[bh] += 1;
        for (int d = 0; d < Dn; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          gdn_step(DK, DV, s, k + rbdh * DK, v + rbdh * DV, alpha[rbdh], beta[rbdh], w);
          gdn_out(DK, DV, s, q + rbdh * DK, scale, o + rbdh * DV);
        }
        memcpy(s, snap, sizeof(double) * DK * DV);
        state_copies[bh] += 1;
        for (int d = 0; d < a; ++d) {
          const size_t rbdh = (((size_t)r * B + b) * Dn + d) * H + h;
          gdn_step(DK, DV, s, k + rbdh * DK, v + rbdh * DV, alpha[rbdh], beta[rbdh], w);
        }
      }
      free(snap);
      free(w);
    }
  return bad ? -1 : 0;
}

int oracle_gdn_flush(int B, int H, int DK, int DV, int L, int cap, int force,
                     double *h0, const double *rec_k, const double *rec_v,
                     const double *rec_alpha, const double *rec_beta, int *len) {
  if (B < 0 || H <= 0 || DK <= 0 || DV <= 0 || L <= 0 || cap < L || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) { bad |= 1; continue; }
      if (n >= L || (force && n > 0)) {
        double *w = (double *)malloc(sizeof(double) * DV);
        gdn_fold(DK, DV, h0 + bh * DK * DV, n, rec_k + bh * cap * DK,
                 rec_v + bh * cap * DV, rec_alpha + bh * cap, rec_beta + bh * cap, w);
        free(w);
        len[bh] = 0;
      }
    }
  return bad ? -1 : 0;
}

int oracle_gdn_materialize(int B, int H, int DK, int DV, int cap,
                           const double *h0, const double *rec_k,
                           const double *rec_v, const double *rec_alpha,
                           const double *rec_beta, const int *len,
                           double *S_out) {
  if (B < 0 || H <= 0 || DK <= 0 || DV <= 0 || cap <= 0 || cap > MAXCAP) return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) { bad |= 1; continue; }
      double *so = S_out + bh * DK * DV;
      double *w = (double *)malloc(sizeof(double) * DV);
      memcpy(so, h0 + bh * DK * DV, sizeof(double) * DK * DV);
      gdn_fold(DK, DV, so, n, rec_k + bh * cap * DK, rec_v + bh * cap * DV,
               rec_alpha + bh * cap, rec_beta + bh * cap, w);
      free(w);
    }
  return bad ? -1 : 0;
}

/* ===================================================================== */
/*                    Low-precision formats [OCP MX v1.0]                 */
/* ===================================================================== */


/* ----------------------------------------------------- Kimi Delta Attention
 * The third layer type the pages name [hamidun §Why hybrid models became the
 * norm]: the gated delta rule with a decay per key channel instead of one
 * scalar (Kimi Linear, Moonshot AI 2025).  State S [DK][DV], alpha_t in
 * (0,1)^DK:
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = scale S_t^T q_t.
 * Replay form, written out here step by step from h0 (Gamma_i = the running
 * elementwise product alpha_0 .. alpha_i, formed directly):
 *   u_i = beta_i (v_i - h0^T (Gamma_i o k_i)
 *                 - sum_{j<i} [sum_r k_j[r] (prod_{j<m<=i} alpha_m[r]) k_i[r]] u_j)
 *   o   = scale (h0^T (Gamma_t o q) + sum_{i<=t} [sum_r k_i[r] (prod_{i<m<=t} alpha_m[r]) q[r]] u_i)
 * and the fold steps the recurrence through the records. */
static void kda_step(int DK, int DV, double *s, const double *kv, const double *vv,
                     const double *av, double beta, double *w) {
  for (int r = 0; r < DK; ++r)
    for (int j = 0; j < DV; ++j) s[(size_t)r * DV + j] *= av[r];
  for (int j = 0; j < DV; ++j) {
    double acc = 0.0;
    for (int r = 0; r < DK; ++r) acc += kv[r] * s[(size_t)r * DV + j];
    w[j] = acc;
  }
  for (int r = 0; r < DK; ++r)
    for (int j = 0; j < DV; ++j)
      s[(size_t)r * DV + j] += beta * kv[r] * (vv[j] - w[j]);
}

/* prod_{a < m <= b} alpha_m[r] over records (a = -1: from the first) */
static double kda_ratio(int DK, const double *ra, int a, int b, int r) {
  double p = 1.0;
  for (int m = a + 1; m <= b; ++m) p *= ra[(size_t)m * DK + r];
  return p;
}

static void kda_replay_out(int DK, int DV, int kc, double scale, const double *h0,
                           const double *rq, const double *rk, const double *rv,
                           const double *ra, const double *rb, double *o, double *u,
                           double *z) {
  for (int i = 0; i < kc; ++i) {
    const double *ki = rk + (size_t)i * DK;
    for (int j = 0; j < DV; ++j) {
      double acc = 0.0;
      for (int r = 0; r < DK; ++r) acc += h0[(size_t)r * DV + j] * kda_ratio(DK, ra, -1, i, r) * ki[r];
      z[j] = acc;
    }
    double *ui = u + (size_t)i * DV;
    for (int j = 0; j < DV; ++j) ui[j] = rv[(size_t)i * DV + j] - z[j];
    for (int jj = 0; jj < i; ++jj) {
      double kk = 0.0;
      for (int r = 0; r < DK; ++r)
        kk += rk[(size_t)jj * DK + r] * kda_ratio(DK, ra, jj, i, r) * ki[r];
      for (int j = 0; j < DV; ++j) ui[j] -= kk * u[(size_t)jj * DV + j];
    }
    for (int j = 0; j < DV; ++j) ui[j] *= rb[i];
  }
  const double *qk = rq + (size_t)(kc - 1) * DK;
  for (int j = 0; j < DV; ++j) {
    double acc = 0.0;
    for (int r = 0; r < DK; ++r) acc += h0[(size_t)r * DV + j] * kda_ratio(DK, ra, -1, kc - 1, r) * qk[r];
    o[j] = acc;
  }
  for (int i = 0; i < kc; ++i) {
    double kq = 0.0;
    for (int r = 0; r < DK; ++r)
      kq += rk[(size_t)i * DK + r] * kda_ratio(DK, ra, i, kc - 1, r) * qk[r];
    for (int j = 0; j < DV; ++j) o[j] += kq * u[(size_t)i * DV + j];
  }
  for (int j = 0; j < DV; ++j) o[j] *= scale;
}

static void kda_fold(int DK, int DV, double *h0, int kc, const double *rk, const double *rv,
                     const double *ra, const double *rb, double *w) {
  for (int i = 0; i < kc; ++i)
    kda_step(DK, DV, h0, rk + (size_t)i * DK, rv + (size_t)i * DV, ra + (size_t)i * DK, rb[i], w);
}

int oracle_kda_conventional(int T, int B, int H, int DK, int DV, double scale, double *S,
                            const double *q, const double *k, const double *v,
                            const double *alpha, const double *beta, double *o,
                            long long *reads, long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0) return -1;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *s = S + bh * DK * DV;
      double *w = (double *)malloc(sizeof(double) * DV);
      for (int t = 0; t < T; ++t) {
        const size_t tbh = ((size_t)t * B + b) * H + h;
        kda_step(DK, DV, s, k + tbh * DK, v + tbh * DV, alpha + tbh * DK, beta[tbh], w);
        for (int j = 0; j < DV; ++j) {
          double acc = 0.0;
          for (int r = 0; r < DK; ++r) acc += s[(size_t)r * DV + j] * q[tbh * DK + r];
          o[tbh * DV + j] = scale * acc;
        }
        if (reads) reads[bh] += 1;
        if (writes) writes[bh] += 1;
      }
      free(w);
    }
  return 0;
}

int oracle_kda_replay(int T, int B, int H, int DK, int DV, int L, int cap, double scale,
                      double *h0, double *rec_q, double *rec_k, double *rec_v,
                      double *rec_alpha, double *rec_beta, int *len, const double *q,
                      const double *k, const double *v, const double *alpha,
                      const double *beta, double *o, int *len_trace, int *flush_trace,
                      long long *reads, long long *writes) {
  if (T < 0 || B < 0 || H <= 0 || DK <= 0 || DV <= 0 || L <= 0 || cap < L || cap > MAXCAP)
    return -1;
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : bad)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      double *hh = h0 + bh * DK * DV;
      double *rq = rec_q + bh * cap * DK, *rk = rec_k + bh * cap * DK;
      double *rv = rec_v + bh * cap * DV, *ra = rec_alpha + bh * cap * DK;
      double *rb = rec_beta + bh * cap;
      double *u = (double *)malloc(sizeof(double) * cap * DV);
      double *z = (double *)malloc(sizeof(double) * DV);
      int n = len[bh];
      for (int t = 0; t < T && !bad; ++t) {
        if (n < 0 || n >= L) { bad |= 1; break; }
        const size_t tbh = ((size_t)t * B + b) * H + h;
        /* append the step's record [sitech §How ReplaySSM works] */
        memcpy(rq + (size_t)n * DK, q + tbh * DK, sizeof(double) * DK);
        memcpy(rk + (size_t)n * DK, k + tbh * DK, sizeof(double) * DK);
        memcpy(rv + (size_t)n * DV, v + tbh * DV, sizeof(double) * DV);
        memcpy(ra + (size_t)n * DK, alpha + tbh * DK, sizeof(double) * DK);
        rb[n] = beta[tbh];
        ++n;
        kda_replay_out(DK, DV, n, scale, hh, rq, rk, rv, ra, rb, o + tbh * DV, u, z);
        if (reads) reads[bh] += 1;
        int flushed = 0;
        if (n == L) {
          kda_fold(DK, DV, hh, n, rk, rv, ra, rb, z);
          n = 0;
          flushed = 1;
          if (writes) writes[bh] += 1;
        }
        if (len_trace) len_trace[tbh] = n;
        if (flush_trace) flush_trace[tbh] = flushed;
      }
      len[bh] = n;
      free(u);
      free(z);
    }
  return bad ? -1 : 0;
}

int oracle_kda_flush(int B, int H, int DK, int DV, int L, int cap, int force, double *h0,
                     const double *rec_k, const double *rec_v, const double *rec_alpha,
                     const double *rec_beta, int *len) {
  if (B < 0 || H <= 0 || DK <= 0 || DV <= 0 || cap > MAXCAP) return -1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) return -1;
      if (!(n >= L || (force && n > 0))) continue;
      double *w = (double *)malloc(sizeof(double) * DV);
      kda_fold(DK, DV, h0 + bh * DK * DV, n, rec_k + bh * cap * DK, rec_v + bh * cap * DV,
               rec_alpha + bh * cap * DK, rec_beta + bh * cap, w);
      free(w);
      len[bh] = 0;
    }
  return 0;
}

int oracle_kda_materialize(int B, int H, int DK, int DV, int cap, const double *h0,
                           const double *rec_k, const double *rec_v, const double *rec_alpha,
                           const double *rec_beta, const int *len, double *S_out) {
  if (B < 0 || H <= 0 || DK <= 0 || DV <= 0 || cap > MAXCAP) return -1;
  memcpy(S_out, h0, sizeof(double) * (size_t)B * H * DK * DV);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const size_t bh = ix2(b, H, h);
      const int n = len[bh];
      if (n < 0 || n > cap) return -1;
      double *w = (double *)malloc(sizeof(double) * DV);
      kda_fold(DK, DV, S_out + bh * DK * DV, n, rec_k + bh * cap * DK, rec_v + bh * cap * DV,
               rec_alpha + bh * cap * DK, rec_beta + bh * cap, w);
      free(w);
    }
  return 0;
}


/* FP8 E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0
 * holds subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities; the largest
 * finite magnitude is 1.75 * 2^8 = 448 (code 0x7E). */
static double e4m3_mag(int c) {
  const int e = (c >> 3) & 0xF, m = c & 7;
  if (e == 0) return ldexp((double)m / 8.0, -6);
  return ldexp(1.0 + (double)m / 8.0, e - 7);
}

double oracle_e4m3_decode(uint8_t c) {
  const int mag = c & 0x7F;
  if (mag == 0x7F) return NAN;
  const double v = e4m3_mag(mag);
  return (c & 0x80) ? -v : v;
}

/* Round to nearest, ties to the even code, saturating to +-448, found by a
 * search over the ascending table of magnitudes. */
uint8_t oracle_e4m3_encode(float vf) {
  const double v = (double)vf;
  if (isnan(v)) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs(v);
  if (a >= 448.0) return sign | 0x7E;
  int lo = 0;
  for (int c = 0; c <= 0x7E; ++c)
    if (e4m3_mag(c) <= a) lo = c;
  if (e4m3_mag(lo) == a) return sign | (uint8_t)lo;
  const int hi = lo + 1;
  const double dl = a - e4m3_mag(lo), dh = e4m3_mag(hi) - a;
  int c;
  if (dl < dh) c = lo;
  else if (dh < dl) c = hi;
  else c = (lo % 2 == 0) ? lo : hi;
  return sign | (uint8_t)c;
}

/* FP4 E2M1: sign bit 3, 2 exponent bits (bias 1), 1 mantissa bit; exponent
 * field 0 holds the subnormal 0.5; magnitudes 0,0.5,1,1.5,2,3,4,6. */
static double e2m1_mag(int c) {
  const int e = (c >> 1) & 3, m = c & 1;
  if (e == 0) return 0.5 * m;
  return ldexp(1.0 + 0.5 * m, e - 1);
}

double oracle_e2m1_decode(uint8_t c) {
  const double v = e2m1_mag(c & 7);
  return (c & 8) ? -v : v;
}

uint8_t oracle_e2m1_encode(float vf) {
  const double v = (double)vf;
  if (isnan(v)) return 0x7;
  const uint8_t sign = signbit(v) ? 0x8 : 0x0;
  const double a = fabs(v);
  if (a >= 6.0) return sign | 0x7;
  int lo = 0;
  for (int c = 0; c <= 7; ++c)
    if (e2m1_mag(c) <= a) lo = c;
  if (e2m1_mag(lo) == a) return sign | (uint8_t)lo;
  const int hi = lo + 1;
  const double dl = a - e2m1_mag(lo), dh = e2m1_mag(hi) - a;
  int c;
  if (dl < dh) c = lo;
  else if (dh < dl) c = hi;
  else c = (lo % 2 == 0) ? lo : hi;
  return sign | (uint8_t)c;
}

int oracle_fp8_quant(long long n, const float *x, uint8_t *codes) {
  if (n < 0) return -1;
  for (long long i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode(x[i]);
  return 0;
}

int oracle_fp8_dequant(long long n, const uint8_t *codes, float *out) {
  if (n < 0) return -1;
  for (long long i = 0; i < n; ++i) out[i] = (float)oracle_e4m3_decode(codes[i]);
  return 0;
}

/* NVFP4 tile quantisation, decided in fp32 (the precision the kernel uses):
 *   s_g  = amax(tile) / (6*448)        (1 when the tile is all zeros)
 *   s_b  = E4M3( amax(block of 16) / (6*s_g) )
 *   code = E2M1( x / (s_b*s_g) )        (0 when s_b*s_g == 0)
 * Each '/' and '*' is one correctly rounded fp32 operation. */
int oracle_nvfp4_quant(int ntile, int rows, int cols, const float *x,
                       uint8_t *codes, uint8_t *scales, float *gscale) {
  if (ntile < 0 || rows <= 0 || cols <= 0 || cols % 16) return -1;
  const int nb = cols / 16;
  for (int t = 0; t < ntile; ++t) {
    const float *xt = x + (size_t)t * rows * cols;
    float amax = 0.0f;
    for (size_t i = 0; i < (size_t)rows * cols; ++i) {
      const float a = fabsf(xt[i]);
      if (a > amax) amax = a;
    }
    const float sg = amax > 0.0f ? amax / 2688.0f : 1.0f;
    gscale[t] = sg;
    const float six_sg = 6.0f * sg;
    for (int r = 0; r < rows; ++r)
      for (int blk = 0; blk < nb; ++blk) {
        const float *xb = xt + (size_t)r * cols + blk * 16;
        float bmax = 0.0f;
        for (int j = 0; j < 16; ++j) {
          const float a = fabsf(xb[j]);
          if (a > bmax) bmax = a;
        }
        const float qs = bmax / six_sg;
        const uint8_t sc = oracle_e4m3_encode(qs);
        scales[((size_t)t * rows + r) * nb + blk] = sc;
        const float sb = (float)oracle_e4m3_decode(sc);
        const float d = sb * sg;
        for (int j = 0; j < 16; j += 2) {
          const uint8_t c0 = d > 0.0f ? oracle_e2m1_encode(xb[j] / d) : 0;
          const uint8_t c1 = d > 0.0f ? oracle_e2m1_encode(xb[j + 1] / d) : 0;
          codes[((size_t)t * rows + r) * (cols / 2) + (blk * 16 + j) / 2] =
              (uint8_t)(c0 | (c1 << 4));
        }
      }
  }
  return 0;
}

int oracle_nvfp4_dequant(int ntile, int rows, int cols, const uint8_t *codes,
                         const uint8_t *scales, const float *gscale,
                         float *out) {
  if (ntile < 0 || rows <= 0 || cols <= 0 || cols % 16) return -1;
  const int nb = cols / 16;
  for (int t = 0; t < ntile; ++t)
    for (int r = 0; r < rows; ++r)
      for (int c = 0; c < cols; ++c) {
        const uint8_t byte = codes[((size_t)t * rows + r) * (cols / 2) + c / 2];
        const uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        const float sb = (float)oracle_e4m3_decode(scales[((size_t)t * rows + r) * nb + c / 16]);
        const float v = (float)oracle_e2m1_decode(code) * sb; /* exact */
        out[((size_t)t * rows + r) * cols + c] = v * gscale[t];
      }
  return 0;
}

/* Read view of a checkpoint tile: the values a reader sees when reads go
 * through a low-precision copy, deq(Q(fp32(h))).  [sitech §Bounding
 * quantisation error]: the copy serves reads only; the recurrence keeps the
 * high-precision checkpoint. */
static void make_view(int fmt, int rows, int cols, const double *h, double *view) {
  const size_t n = (size_t)rows * cols;
  float *f = (float *)malloc(sizeof(float) * n);
  for (size_t i = 0; i < n; ++i) f[i] = (float)h[i];
  if (fmt == ORACLE_FMT_FP8) {
    uint8_t *c = (uint8_t *)malloc(n);
    oracle_fp8_quant((long long)n, f, c);
    oracle_fp8_dequant((long long)n, c, f);
    free(c);
  } else if (fmt == ORACLE_FMT_NVFP4) {
    uint8_t *c = (uint8_t *)malloc(n / 2);
    uint8_t *s = (uint8_t *)malloc(n / 16);
    float g;
    oracle_nvfp4_quant(1, rows, cols, f, c, s, &g);
    oracle_nvfp4_dequant(1, rows, cols, c, s, &g, f);
    free(c);
    free(s);
  }
  for (size_t i = 0; i < n; ++i) view[i] = (double)f[i];
  free(f);
}

/* The "quantised checkpoint" baseline: the checkpoint itself is stored in the
 * low-precision format, so every fold starts from deq(Q(.)). */
static void quant_ckpt_tile(int fmt, int rows, int cols, double *h) {
  make_view(fmt, rows, cols, h, h);
}

int oracle_quantize_ckpt(int fmt, int ntile, int rows, int cols, double *h) {
  if (fmt != ORACLE_FMT_FP8 && fmt != ORACLE_FMT_NVFP4) return -1;
  if (ntile < 0 || rows <= 0 || cols <= 0 || cols % 16) return -1;
#pragma omp parallel for schedule(dynamic)
  for (int t = 0; t < ntile; ++t) quant_ckpt_tile(fmt, rows, cols, h + (size_t)t * rows * cols);
  return 0;
}
