/*
 * Interdomain Attention (IA) -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, __graft_entry__.smoke() and
 * bench.py's CPU legs, never by the product path.  Independent of the CUDA
 * path: no shared code, headers, tables or helpers.
 *
 * Every routine here follows the plain definitions of the method as the paper
 * "Interdomain Attention: Beyond Token-Level Key-Value Memory" states them
 * (paperlayer.ai summary, sec. 3.1-3.2; formula extract on the AI-radio page,
 * "Key Components and Derivation"):
 *   - one complex-diagonal S4D recurrence with a shared basis drives the key
 *     features xi(k_t), the values v_t and the constant 1 (states U, Gamma, eta);
 *   - each query reads out O = F_q U^T Gamma / F_q U^T eta, taken here as
 *     num_t = Re(a_t^H Gamma_t), den_t = Re(a_t^H eta_t), a_t = U_t xi(q_t).
 * Readings where the pages are silent: xi = elu + 1 (alpha = 1); S4D-Lin
 * A_m = -1/2 + i*pi*m, m = 0..M-1; zero-order-hold b = (lambda - 1)/A; one
 * Delta per head shared by all modes, or (flag dpm) one Delta per head and
 * mode, Delta[h][m]; the state is updated with token t before query t reads
 * it (inclusive causality); no epsilon in o = num/den.
 *
 * All arithmetic is IEEE fp64 in the order written; no blocking or fusion.
 */
#define _GNU_SOURCE
#include "ia_oracle.h"

#include <complex.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef double complex cd;

/* elu(x) + 1 with alpha = 1: x + 1 above zero, exp(x) at or below zero. */
static double feat(double x) { return x > 0.0 ? x + 1.0 : exp(x); }
/* Its derivative: 1 above zero, exp(x) at or below (both sides meet at 1). */
static double dfeat(double x) { return x > 0.0 ? 1.0 : exp(x); }

static const double kPi = 3.14159265358979323846;

static cd mode_A(const double* A, int m) {
  if (A) return A[2 * m] + I * A[2 * m + 1];
  return -0.5 + I * (kPi * (double)m);          /* S4D-Lin */
}

/* Delta of head h and mode m: one per head, or one per (head, mode) with dpm. */
static double delta_hm(const double* delta, int dpm, int M, int h, int m) {
  return dpm ? delta[(long)h * M + m] : delta[h];
}

static cd ld_c(const double* p) { return p[0] + I * p[1]; }
static void st_c(double* p, cd z) { p[0] = creal(z); p[1] = cimag(z); }

long iao_state_len(int B, int H, int M, int d_xi, int d_v) {
  return 2L * B * H * M * ((long)d_xi + d_v + 1);
}

int iao_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Zero-order hold of dx/dt = A x + u over a step Delta:
 * lambda = exp(Delta A), b = (lambda - 1) / A. */
static void zoh(double delta, cd a, cd* l, cd* bm) {
  *l = cexp(delta * a);
  *bm = (*l - 1.0) / a;
}

int iao_params(int M, double delta, const double* A, double* lam, double* b) {
  if (M <= 0 || !(delta > 0.0) || !lam || !b) return -1;
  for (int m = 0; m < M; ++m) {
    cd l, bm;
    zoh(delta, mode_A(A, m), &l, &bm);
    st_c(lam + 2 * m, l);
    st_c(b + 2 * m, bm);
  }
  return 0;
}

static int bad_dims(int B, int H, int N, int d_xi, int d_v, int M) {
  return B <= 0 || H <= 0 || N < 0 || d_xi <= 0 || d_v <= 0 || M <= 0;
}

/* Per-(b,h) state views inside one state buffer. */
typedef struct {
  long u_off, g_off, e_off;   /* offsets (in doubles) of this (b,h)'s U, Gamma, eta */
} state_ofs;

static state_ofs state_offsets(int B, int H, int M, int d_xi, int d_v, int bh) {
  state_ofs s;
  long BH = (long)B * H;
  s.u_off = 2L * bh * M * d_xi;
  s.g_off = 2L * BH * M * d_xi + 2L * bh * M * d_v;
  s.e_off = 2L * BH * M * ((long)d_xi + d_v) + 2L * bh * M;
  return s;
}

/*
 * The recurrence and readout for one (b,h) sequence.  fq, fk are already
 * mapped features [N,d_xi]; v is [N,d_v]; U, G, eta are the running state
 * (updated in place).  lam, bb are this head's [M] tables.
 */
static void run_sequence(int N, int d_xi, int d_v, int M,
                         const double* fq, const double* fk, const double* v,
                         const cd* lam, const cd* bb, cd* U, cd* G, cd* eta,
                         double* o, double* num, double* den, cd* a) {
  for (int t = 0; t < N; ++t) {
    const double* fkt = fk + (long)t * d_xi;
    const double* fqt = fq + (long)t * d_xi;
    const double* vt = v + (long)t * d_v;
    for (int m = 0; m < M; ++m) {
      cd* Um = U + (long)m * d_xi;
      cd* Gm = G + (long)m * d_v;
      cd am = 0.0;
      for (int f = 0; f < d_xi; ++f) {
        Um[f] = lam[m] * Um[f] + bb[m] * fkt[f];
        am += Um[f] * fqt[f];
      }
      for (int f = 0; f < d_v; ++f) Gm[f] = lam[m] * Gm[f] + bb[m] * vt[f];
      eta[m] = lam[m] * eta[m] + bb[m];
      a[m] = am;
    }
    double dn = 0.0;
    for (int m = 0; m < M; ++m) dn += creal(conj(a[m]) * eta[m]);
    for (int f = 0; f < d_v; ++f) {
      double nf = 0.0;
      for (int m = 0; m < M; ++m) nf += creal(conj(a[m]) * G[(long)m * d_v + f]);
      if (num) num[(long)t * d_v + f] = nf;
      o[(long)t * d_v + f] = nf / dn;
    }
    if (den) den[t] = dn;
  }
}

static void load_state(const double* st, int B, int H, int M, int d_xi, int d_v, int bh,
                       cd* U, cd* G, cd* eta) {
  if (!st) {
    for (long i = 0; i < (long)M * d_xi; ++i) U[i] = 0.0;
    for (long i = 0; i < (long)M * d_v; ++i) G[i] = 0.0;
    for (int m = 0; m < M; ++m) eta[m] = 0.0;
    return;
  }
  state_ofs s = state_offsets(B, H, M, d_xi, d_v, bh);
  for (long i = 0; i < (long)M * d_xi; ++i) U[i] = ld_c(st + s.u_off + 2 * i);
  for (long i = 0; i < (long)M * d_v; ++i) G[i] = ld_c(st + s.g_off + 2 * i);
  for (int m = 0; m < M; ++m) eta[m] = ld_c(st + s.e_off + 2 * m);
}

static void store_state(double* st, int B, int H, int M, int d_xi, int d_v, int bh,
                        const cd* U, const cd* G, const cd* eta) {
  state_ofs s = state_offsets(B, H, M, d_xi, d_v, bh);
  for (long i = 0; i < (long)M * d_xi; ++i) st_c(st + s.u_off + 2 * i, U[i]);
  for (long i = 0; i < (long)M * d_v; ++i) st_c(st + s.g_off + 2 * i, G[i]);
  for (int m = 0; m < M; ++m) st_c(st + s.e_off + 2 * m, eta[m]);
}

/* Shared driver: features given, tables given per head as [H,M] complex. */
static int forward_impl(int B, int H, int N, int d_xi, int d_v, int M,
                        const double* q, const double* k, int map_features,
                        const double* v, const double* lamtab, const double* btab,
                        const double* state_in, double* o, double* num, double* den,
                        double* state_out) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !q || !k || !v || !o || !lamtab || !btab) return -1;
  long BH = (long)B * H;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    int h = (int)(bh % H);
    cd* lam = malloc(sizeof(cd) * M);
    cd* bb = malloc(sizeof(cd) * M);
    cd* U = malloc(sizeof(cd) * (size_t)M * d_xi);
    cd* G = malloc(sizeof(cd) * (size_t)M * d_v);
    cd* eta = malloc(sizeof(cd) * M);
    cd* a = malloc(sizeof(cd) * M);
    double* fq = malloc(sizeof(double) * ((size_t)N * d_xi + 1));
    double* fk = malloc(sizeof(double) * ((size_t)N * d_xi + 1));
    if (!lam || !bb || !U || !G || !eta || !a || !fq || !fk) {
#pragma omp atomic write
      err = -2;
    } else {
      for (int m = 0; m < M; ++m) {
        lam[m] = ld_c(lamtab + 2L * ((long)h * M + m));
        bb[m] = ld_c(btab + 2L * ((long)h * M + m));
      }
      const double* qb = q + bh * (long)N * d_xi;
      const double* kb = k + bh * (long)N * d_xi;
      for (long i = 0; i < (long)N * d_xi; ++i) {
        fq[i] = map_features ? feat(qb[i]) : qb[i];
        fk[i] = map_features ? feat(kb[i]) : kb[i];
      }
      load_state(state_in, B, H, M, d_xi, d_v, (int)bh, U, G, eta);
      run_sequence(N, d_xi, d_v, M, fq, fk, v + bh * (long)N * d_v, lam, bb, U, G, eta,
                   o + bh * (long)N * d_v, num ? num + bh * (long)N * d_v : NULL,
                   den ? den + bh * (long)N : NULL, a);
      if (state_out) store_state(state_out, B, H, M, d_xi, d_v, (int)bh, U, G, eta);
    }
    free(lam); free(bb); free(U); free(G); free(eta); free(a); free(fq); free(fk);
  }
  return err;
}

static int head_tables(int H, int M, const double* delta, int dpm, const double* A,
                       double** lamtab, double** btab) {
  *lamtab = malloc(sizeof(double) * 2 * (size_t)H * M);
  *btab = malloc(sizeof(double) * 2 * (size_t)H * M);
  if (!*lamtab || !*btab) return -2;
  for (int h = 0; h < H; ++h) {
    for (int m = 0; m < M; ++m) {
      double dl = delta_hm(delta, dpm, M, h, m);
      if (!(dl > 0.0)) return -1;
      cd l, bm;
      zoh(dl, mode_A(A, m), &l, &bm);
      st_c(*lamtab + 2L * ((long)h * M + m), l);
      st_c(*btab + 2L * ((long)h * M + m), bm);
    }
  }
  return 0;
}

int iao_forward(int B, int H, int N, int d_xi, int d_v, int M,
                const double* q, const double* k, const double* v,
                const double* delta, int dpm, const double* A, const double* state_in,
                double* o, double* num, double* den, double* state_out) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !delta) return -1;
  double *lt = NULL, *bt = NULL;
  int err = head_tables(H, M, delta, dpm, A, &lt, &bt);
  if (!err)
    err = forward_impl(B, H, N, d_xi, d_v, M, q, k, 1, v, lt, bt, state_in, o, num, den,
                       state_out);
  free(lt); free(bt);
  return err;
}

int iao_forward_features(int B, int H, int N, int d_xi, int d_v, int M,
                         const double* fq, const double* fk, const double* v,
                         const double* lam, const double* b, const double* state_in,
                         double* o, double* num, double* den, double* state_out) {
  return forward_impl(B, H, N, d_xi, d_v, M, fq, fk, 0, v, lam, b, state_in, o, num, den,
                      state_out);
}

int iao_decode_step(int B, int H, int d_xi, int d_v, int M,
                    const double* q, const double* k, const double* v,
                    const double* delta, int dpm, const double* A, double* state,
                    double* o, double* num, double* den) {
  if (!state) return -1;
  /* One iteration of the loop body, reading and writing the same state. */
  long n = iao_state_len(B, H, M, d_xi, d_v);
  double* tmp = malloc(sizeof(double) * (size_t)n);
  if (!tmp) return -2;
  memcpy(tmp, state, sizeof(double) * (size_t)n);
  int err = iao_forward(B, H, 1, d_xi, d_v, M, q, k, v, delta, dpm, A, tmp, o, num, den, state);
  free(tmp);
  return err;
}

/*
 * Extended layer forward: the optional parts of the layer, each off when its
 * argument is NULL (with all of them off this is iao_forward).
 *
 *   Input stabilisation (AI-radio page, "Implementation Details": the SSM
 *   input z_t = (xi(k_t), v_t) passes an RMSNorm with a learnable per-head
 *   bias before the SSM): with gain or bias given,
 *       z_t <- z_t / sqrt(mean_f z_t[f]^2 + eps) * gain_h + bias_h,
 *   over the d_xi + d_v entries of z_t; gain, bias [H, d_xi + d_v] (NULL gain
 *   = 1, NULL bias = 0).  The query features are not normalised.
 *
 *   Selective writing and memory decay (summary sec. 3.3 and sec. 5.3): with
 *   delta_t [B,H,N] given, token t of sequence (b,h) uses its own step,
 *   lambda_t = exp(delta_t A), b_t = (lambda_t - 1)/A, for all modes: a small
 *   step writes little and forgets little.
 *
 *   Full complex readout matrix (summary sec. A.3, and the M^2 term of the
 *   decode cost in sec. 3.2): with W [H,M,M] complex given (W[h][m][m'],
 *   row m, column m'), the query's mode coefficients are mixed before the
 *   readout: a~_t = W_h a_t, num_t = Re(a~_t^H Gamma_t), den_t = Re(a~_t^H eta_t).
 *
 * map_features = 0 takes q and k as already-mapped features (xi is then
 * skipped), which lets a pin scale the SSM input directly.
 */
int iao_forward_ex(int B, int H, int N, int d_xi, int d_v, int M,
                   const double* q, const double* k, const double* v, int map_features,
                   const double* delta, int dpm, const double* A, const double* delta_t,
                   const double* gain, const double* bias, double eps, const double* W,
                   const double* state_in, double* o, double* num, double* den,
                   double* state_out) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !q || !k || !v || !o || (!delta && !delta_t)) return -1;
  long BH = (long)B * H;
  int D = d_xi + d_v;
  int norm = gain || bias;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    int h = (int)(bh % H);
    cd* Am = malloc(sizeof(cd) * M);
    cd* lam = malloc(sizeof(cd) * M);
    cd* bb = malloc(sizeof(cd) * M);
    cd* U = malloc(sizeof(cd) * (size_t)M * d_xi);
    cd* G = malloc(sizeof(cd) * (size_t)M * d_v);
    cd* eta = malloc(sizeof(cd) * M);
    cd* a = malloc(sizeof(cd) * M);
    cd* at = malloc(sizeof(cd) * M);
    double* z = malloc(sizeof(double) * (size_t)D);
    double* fq = malloc(sizeof(double) * (size_t)d_xi);
    if (!Am || !lam || !bb || !U || !G || !eta || !a || !at || !z || !fq) {
#pragma omp atomic write
      err = -2;
    } else {
      for (int m = 0; m < M; ++m) {
        Am[m] = mode_A(A, m);
        if (!delta_t) zoh(delta_hm(delta, dpm, M, h, m), Am[m], &lam[m], &bb[m]);
      }
      load_state(state_in, B, H, M, d_xi, d_v, (int)bh, U, G, eta);
      for (int t = 0; t < N; ++t) {
        long rq = (bh * N + t) * (long)d_xi, rv = (bh * N + t) * (long)d_v;
        /* the SSM input z_t = (xi(k_t), v_t), normalised if asked */
        for (int f = 0; f < d_xi; ++f) {
          z[f] = map_features ? feat(k[rq + f]) : k[rq + f];
          fq[f] = map_features ? feat(q[rq + f]) : q[rq + f];
        }
        for (int f = 0; f < d_v; ++f) z[d_xi + f] = v[rv + f];
        if (norm) {
          double ss = 0.0;
          for (int f = 0; f < D; ++f) ss += z[f] * z[f];
          double r = 1.0 / sqrt(ss / (double)D + eps);
          for (int f = 0; f < D; ++f) {
            double g = gain ? gain[(long)h * D + f] : 1.0;
            double c = bias ? bias[(long)h * D + f] : 0.0;
            z[f] = z[f] * r * g + c;
          }
        }
        /* this token's step */
        if (delta_t)
          for (int m = 0; m < M; ++m) zoh(delta_t[bh * N + t], Am[m], &lam[m], &bb[m]);
        /* recurrence, then the query's mode coefficients */
        for (int m = 0; m < M; ++m) {
          cd am = 0.0;
          for (int f = 0; f < d_xi; ++f) {
            U[(long)m * d_xi + f] = lam[m] * U[(long)m * d_xi + f] + bb[m] * z[f];
            am += U[(long)m * d_xi + f] * fq[f];
          }
          for (int f = 0; f < d_v; ++f)
            G[(long)m * d_v + f] = lam[m] * G[(long)m * d_v + f] + bb[m] * z[d_xi + f];
          eta[m] = lam[m] * eta[m] + bb[m];
          a[m] = am;
        }
        /* readout matrix */
        for (int m = 0; m < M; ++m) {
          if (!W) { at[m] = a[m]; continue; }
          cd acc = 0.0;
          for (int mp = 0; mp < M; ++mp) acc += ld_c(W + 2 * (((long)h * M + m) * M + mp)) * a[mp];
          at[m] = acc;
        }
        double dn = 0.0;
        for (int m = 0; m < M; ++m) dn += creal(conj(at[m]) * eta[m]);
        for (int f = 0; f < d_v; ++f) {
          double nf = 0.0;
          for (int m = 0; m < M; ++m) nf += creal(conj(at[m]) * G[(long)m * d_v + f]);
          if (num) num[rv + f] = nf;
          o[rv + f] = nf / dn;
        }
        if (den) den[bh * N + t] = dn;
      }
      if (state_out) store_state(state_out, B, H, M, d_xi, d_v, (int)bh, U, G, eta);
    }
    free(Am); free(lam); free(bb); free(U); free(G); free(eta); free(a); free(at); free(z); free(fq);
  }
  return err;
}

/*
 * Brute force from a zero state.  Unrolling the recurrence gives
 *   a_tm  = b_m sum_{n<=t} lambda_m^(t-n) s_tn,     s_tn = xi(q_t).xi(k_n)
 *   w_tn  = Re sum_m conj(a_tm) b_m lambda_m^(t-n)
 *   num_t = sum_{n<=t} w_tn v_n,   den_t = sum_{n<=t} w_tn
 * with every power evaluated as exp((t-n) Delta A_m).
 */
int iao_brute(int B, int H, int N, int d_xi, int d_v, int M,
              const double* q, const double* k, const double* v,
              const double* delta, int dpm, const double* A,
              double* o, double* num, double* den) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !q || !k || !v || !delta || !o) return -1;
  long BH = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    int h = (int)(bh % H);
    const double* qb = q + bh * (long)N * d_xi;
    const double* kb = k + bh * (long)N * d_xi;
    const double* vb = v + bh * (long)N * d_v;
    cd* a = malloc(sizeof(cd) * M);
    double* w = malloc(sizeof(double) * ((size_t)N + 1));
    for (int t = 0; t < N; ++t) {
      for (int m = 0; m < M; ++m) {
        cd Am = mode_A(A, m);
        double dl = delta_hm(delta, dpm, M, h, m);
        cd bm = (cexp(dl * Am) - 1.0) / Am;
        cd acc = 0.0;
        for (int n = 0; n <= t; ++n) {
          double s = 0.0;
          for (int f = 0; f < d_xi; ++f)
            s += feat(qb[(long)t * d_xi + f]) * feat(kb[(long)n * d_xi + f]);
          acc += cexp((double)(t - n) * dl * Am) * s;
        }
        a[m] = bm * acc;
      }
      double dn = 0.0;
      for (int n = 0; n <= t; ++n) {
        double wt = 0.0;
        for (int m = 0; m < M; ++m) {
          cd Am = mode_A(A, m);
          double dl = delta_hm(delta, dpm, M, h, m);
          cd bm = (cexp(dl * Am) - 1.0) / Am;
          wt += creal(conj(a[m]) * bm * cexp((double)(t - n) * dl * Am));
        }
        w[n] = wt;
        dn += wt;
      }
      for (int f = 0; f < d_v; ++f) {
        double nf = 0.0;
        for (int n = 0; n <= t; ++n) nf += w[n] * vb[(long)n * d_v + f];
        if (num) num[(bh * N + t) * (long)d_v + f] = nf;
        o[(bh * N + t) * (long)d_v + f] = nf / dn;
      }
      if (den) den[bh * N + t] = dn;
    }
    free(a); free(w);
  }
  return 0;
}

/*
 * Reverse mode of the recurrence (zero initial state).  With upstream dO_t:
 *   dnum_t = dO_t / den_t,  dden_t = -(dO_t . o_t) / den_t
 *   gbar_a_t[m]   = sum_f Gamma_t[m,f] dnum_t[f] + eta_t[m] dden_t
 *   dxi(q_t)[f]   = Re sum_m conj(gbar_a_t[m]) U_t[m,f]
 *   local adjoints: gU_t = gbar_a_t xi(q_t)^T, gGamma_t = a_t dnum_t^T,
 *                   geta_t = a_t dden_t
 *   reverse scans:  G_t = g_t + conj(lambda) G_{t+1}   (U, Gamma, eta alike)
 *   dxi(k_t)[f] = Re sum_m conj(b_m) G^U_t[m,f],  dv_t[f] likewise with G^Gamma
 *   gbar_lambda_m = sum_t G_t . conj(S_{t-1}),  gbar_b_m = sum_t G_t . x_t
 *   dDelta_hm = Re(conj(gbar_lambda_m) A_m lambda_m + conj(gbar_b_m) lambda_m)
 *     (summed over the batch, and over m when one Delta serves all modes)
 *   dA_m = sum over batch and heads of conj(dlambda/dA) gbar_lambda_m
 *          + conj(db/dA) gbar_b_m,  dlambda/dA = Delta lambda,
 *          db/dA = (Delta lambda - b) / A     (lambda = exp(Delta A), b = (lambda - 1)/A)
 *   dq = dxi(q) * xi'(q),  dk = dxi(k) * xi'(k).
 * Complex adjoints use the convention g = dL/dRe + i dL/dIm (so dA_m holds
 * dL/dRe A_m and dL/dIm A_m).  States are recomputed forward from
 * checkpoints every CK steps.
 */
#define CK 64

int iao_backward(int B, int H, int N, int d_xi, int d_v, int M,
                 const double* q, const double* k, const double* v,
                 const double* delta, int dpm, const double* A, const double* dO,
                 double* o_out, double* dq, double* dk, double* dv, double* dDelta,
                 double* dA) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !q || !k || !v || !delta || !dO || !dq || !dk ||
      !dv || !dDelta)
    return -1;
  long BH = (long)B * H;
  long S1 = (long)M * d_xi, S2 = (long)M * d_v;
  long SL = S1 + S2 + M;                       /* complex entries per state */
  /* per (b,h,m): dL/dDelta_hm and the complex dL/dA_m of that sequence */
  double* part = calloc((size_t)BH * M, sizeof(double));
  cd* partA = calloc((size_t)BH * M, sizeof(cd));
  if (!part || !partA) { free(part); free(partA); return -2; }
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    int h = (int)(bh % H);
    const double* qb = q + bh * (long)N * d_xi;
    const double* kb = k + bh * (long)N * d_xi;
    const double* vb = v + bh * (long)N * d_v;
    const double* gb = dO + bh * (long)N * d_v;
    int nck = (N + CK - 1) / CK;
    cd* lam = malloc(sizeof(cd) * M);
    cd* bb = malloc(sizeof(cd) * M);
    cd* Am = malloc(sizeof(cd) * M);
    cd* ck = malloc(sizeof(cd) * (size_t)SL * (nck + 1));   /* state before each block */
    cd* blk = malloc(sizeof(cd) * (size_t)SL * (CK + 1));   /* states inside a block */
    cd* G = calloc((size_t)SL, sizeof(cd));                 /* running adjoint */
    cd* ga = malloc(sizeof(cd) * M);
    cd* a = malloc(sizeof(cd) * M);
    cd* glam = calloc((size_t)M, sizeof(cd));
    cd* gb_ = calloc((size_t)M, sizeof(cd));
    double* fq = malloc(sizeof(double) * ((size_t)N * d_xi + 1));
    double* fk = malloc(sizeof(double) * ((size_t)N * d_xi + 1));
    double* o = malloc(sizeof(double) * ((size_t)N * d_v + 1));
    double* den = malloc(sizeof(double) * ((size_t)N + 1));
    if (!lam || !bb || !Am || !ck || !blk || !G || !ga || !a || !glam || !gb_ || !fq || !fk ||
        !o || !den) {
#pragma omp atomic write
      err = -2;
    } else {
      for (int m = 0; m < M; ++m) {
        Am[m] = mode_A(A, m);
        lam[m] = cexp(delta_hm(delta, dpm, M, h, m) * Am[m]);
        bb[m] = (lam[m] - 1.0) / Am[m];
      }
      for (long i = 0; i < (long)N * d_xi; ++i) { fq[i] = feat(qb[i]); fk[i] = feat(kb[i]); }
      /* Forward sweep: outputs, den and the checkpoints. */
      cd* cur = blk;                                  /* scratch state */
      for (long i = 0; i < SL; ++i) cur[i] = 0.0;
      for (int t = 0; t < N; ++t) {
        if (t % CK == 0) memcpy(ck + (size_t)(t / CK) * SL, cur, sizeof(cd) * SL);
        run_sequence(1, d_xi, d_v, M, fq + (long)t * d_xi, fk + (long)t * d_xi,
                     vb + (long)t * d_v, lam, bb, cur, cur + S1, cur + S1 + S2,
                     o + (long)t * d_v, NULL, den + t, a);
      }
      if (o_out) memcpy(o_out + bh * (long)N * d_v, o, sizeof(double) * (size_t)N * d_v);
      /* Reverse sweep, one checkpoint block at a time. */
      for (int c = nck - 1; c >= 0; --c) {
        int t0 = c * CK, t1 = (t0 + CK < N) ? t0 + CK : N;
        /* blk[j] = state after token t0 + j - 1 (blk[0] = checkpoint). */
        memcpy(blk, ck + (size_t)c * SL, sizeof(cd) * SL);
        for (int t = t0; t < t1; ++t) {
          cd* prev = blk + (size_t)(t - t0) * SL;
          cd* nxt = prev + SL;
          for (int m = 0; m < M; ++m) {
            for (int f = 0; f < d_xi; ++f)
              nxt[m * d_xi + f] = lam[m] * prev[m * d_xi + f] + bb[m] * fk[(long)t * d_xi + f];
            for (int f = 0; f < d_v; ++f)
              nxt[S1 + m * d_v + f] = lam[m] * prev[S1 + m * d_v + f] + bb[m] * vb[(long)t * d_v + f];
            nxt[S1 + S2 + m] = lam[m] * prev[S1 + S2 + m] + bb[m];
          }
        }
        for (int t = t1 - 1; t >= t0; --t) {
          const cd* St = blk + (size_t)(t - t0 + 1) * SL;   /* S_t */
          const cd* Sp = blk + (size_t)(t - t0) * SL;       /* S_{t-1} */
          const cd* Ut = St;
          const cd* Gt = St + S1;
          const cd* et = St + S1 + S2;
          const double* fqt = fq + (long)t * d_xi;
          const double* fkt = fk + (long)t * d_xi;
          const double* vt = vb + (long)t * d_v;
          const double* dOt = gb + (long)t * d_v;
          const double* ot = o + (long)t * d_v;
          double dden = 0.0;
          for (int f = 0; f < d_v; ++f) dden -= dOt[f] * ot[f];
          dden /= den[t];
          for (int m = 0; m < M; ++m) {
            cd am = 0.0, gam = 0.0;
            for (int f = 0; f < d_xi; ++f) am += Ut[m * d_xi + f] * fqt[f];
            for (int f = 0; f < d_v; ++f) gam += Gt[m * d_v + f] * (dOt[f] / den[t]);
            gam += et[m] * dden;
            a[m] = am;
            ga[m] = gam;
          }
          long base = (bh * N + t);
          for (int f = 0; f < d_xi; ++f) {
            double s = 0.0;
            for (int m = 0; m < M; ++m) s += creal(conj(ga[m]) * Ut[m * d_xi + f]);
            dq[base * d_xi + f] = s * dfeat(qb[(long)t * d_xi + f]);
          }
          /* Add the local adjoints: G now holds the full adjoint of S_t. */
          for (int m = 0; m < M; ++m) {
            for (int f = 0; f < d_xi; ++f) G[m * d_xi + f] += ga[m] * fqt[f];
            for (int f = 0; f < d_v; ++f) G[S1 + m * d_v + f] += a[m] * (dOt[f] / den[t]);
            G[S1 + S2 + m] += a[m] * dden;
          }
          for (int f = 0; f < d_xi; ++f) {
            double s = 0.0;
            for (int m = 0; m < M; ++m) s += creal(conj(bb[m]) * G[m * d_xi + f]);
            dk[base * d_xi + f] = s * dfeat(kb[(long)t * d_xi + f]);
          }
          for (int f = 0; f < d_v; ++f) {
            double s = 0.0;
            for (int m = 0; m < M; ++m) s += creal(conj(bb[m]) * G[S1 + m * d_v + f]);
            dv[base * d_v + f] = s;
          }
          for (int m = 0; m < M; ++m) {
            cd sl = 0.0, sb = 0.0;
            for (int f = 0; f < d_xi; ++f) {
              sl += G[m * d_xi + f] * conj(Sp[m * d_xi + f]);
              sb += G[m * d_xi + f] * fkt[f];
            }
            for (int f = 0; f < d_v; ++f) {
              sl += G[S1 + m * d_v + f] * conj(Sp[S1 + m * d_v + f]);
              sb += G[S1 + m * d_v + f] * vt[f];
            }
            sl += G[S1 + S2 + m] * conj(Sp[S1 + S2 + m]);
            sb += G[S1 + S2 + m];
            glam[m] += sl;
            gb_[m] += sb;
          }
          /* Carry the adjoint one step back: multiply by conj(lambda). */
          for (int m = 0; m < M; ++m) {
            cd cl = conj(lam[m]);
            for (int f = 0; f < d_xi; ++f) G[m * d_xi + f] *= cl;
            for (int f = 0; f < d_v; ++f) G[S1 + m * d_v + f] *= cl;
            G[S1 + S2 + m] *= cl;
          }
        }
      }
      for (int m = 0; m < M; ++m) {
        double dl = delta_hm(delta, dpm, M, h, m);
        part[bh * M + m] = creal(conj(glam[m]) * Am[m] * lam[m] + conj(gb_[m]) * lam[m]);
        partA[bh * M + m] = conj(dl * lam[m]) * glam[m] + conj((dl * lam[m] - bb[m]) / Am[m]) * gb_[m];
      }
    }
    free(lam); free(bb); free(Am); free(ck); free(blk); free(G); free(ga); free(a);
    free(glam); free(gb_); free(fq); free(fk); free(o); free(den);
  }
  long nD = dpm ? (long)H * M : H;
  for (long i = 0; i < nD; ++i) dDelta[i] = 0.0;
  for (long bh = 0; bh < BH; ++bh)
    for (int m = 0; m < M; ++m)
      dDelta[dpm ? (bh % H) * M + m : bh % H] += part[bh * M + m];
  if (dA) {
    for (int m = 0; m < M; ++m) {
      cd acc = 0.0;
      for (long bh = 0; bh < BH; ++bh) acc += partA[bh * M + m];
      st_c(dA + 2 * m, acc);
    }
  }
  free(part); free(partA);
  return err;
}

/*
 * Tangent (forward-mode) recurrence along (tq, tk, tv, tdelta, tA):
 *   lambda' = lambda (A delta' + Delta A'),  b' = lambda delta' + (Delta lambda - b)/A A'
 *   U'_t = lambda U'_{t-1} + lambda' U_{t-1} + b' xi(k_t) + b xi'(k_t) tk_t   (Gamma, eta alike)
 *   a'_t = U'_t xi(q_t) + U_t (xi'(q_t) tq_t)
 *   num' = Re(conj(a') Gamma + conj(a) Gamma'),  den' likewise with eta
 *   o'   = (num' - o den') / den
 */
int iao_jvp(int B, int H, int N, int d_xi, int d_v, int M,
            const double* q, const double* k, const double* v,
            const double* delta, int dpm, const double* A,
            const double* tq, const double* tk, const double* tv, const double* tdelta,
            const double* tA, double* to_) {
  if (bad_dims(B, H, N, d_xi, d_v, M) || !q || !k || !v || !delta || !tq || !tk || !tv ||
      !tdelta || !to_)
    return -1;
  long BH = (long)B * H;
  long S1 = (long)M * d_xi, S2 = (long)M * d_v, SL = S1 + S2 + M;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    int h = (int)(bh % H);
    cd* lam = malloc(sizeof(cd) * M);
    cd* bb = malloc(sizeof(cd) * M);
    cd* dl = malloc(sizeof(cd) * M);
    cd* dbb = malloc(sizeof(cd) * M);
    cd* S = calloc((size_t)SL, sizeof(cd));
    cd* T = calloc((size_t)SL, sizeof(cd));
    cd* a = malloc(sizeof(cd) * M);
    cd* ta = malloc(sizeof(cd) * M);
    for (int m = 0; m < M; ++m) {
      cd Am = mode_A(A, m);
      double de = delta_hm(delta, dpm, M, h, m), tde = delta_hm(tdelta, dpm, M, h, m);
      lam[m] = cexp(de * Am);
      bb[m] = (lam[m] - 1.0) / Am;
      dl[m] = Am * lam[m] * tde;
      dbb[m] = lam[m] * tde;
      if (tA) {
        cd ta = ld_c(tA + 2 * m);
        dl[m] += de * lam[m] * ta;
        dbb[m] += (de * lam[m] - bb[m]) / Am * ta;
      }
    }
    for (int t = 0; t < N; ++t) {
      long rq = (bh * N + t) * (long)d_xi, rv = (bh * N + t) * (long)d_v;
      for (int m = 0; m < M; ++m) {
        cd am = 0.0, tam = 0.0;
        for (int f = 0; f < d_xi; ++f) {
          double x = feat(k[rq + f]), tx = dfeat(k[rq + f]) * tk[rq + f];
          cd u = S[m * d_xi + f];
          T[m * d_xi + f] = lam[m] * T[m * d_xi + f] + dl[m] * u + dbb[m] * x + bb[m] * tx;
          S[m * d_xi + f] = lam[m] * u + bb[m] * x;
          am += S[m * d_xi + f] * feat(q[rq + f]);
          tam += T[m * d_xi + f] * feat(q[rq + f]) + S[m * d_xi + f] * dfeat(q[rq + f]) * tq[rq + f];
        }
        for (int f = 0; f < d_v; ++f) {
          cd g = S[S1 + m * d_v + f];
          T[S1 + m * d_v + f] = lam[m] * T[S1 + m * d_v + f] + dl[m] * g + dbb[m] * v[rv + f] +
                                bb[m] * tv[rv + f];
          S[S1 + m * d_v + f] = lam[m] * g + bb[m] * v[rv + f];
        }
        cd e = S[S1 + S2 + m];
        T[S1 + S2 + m] = lam[m] * T[S1 + S2 + m] + dl[m] * e + dbb[m];
        S[S1 + S2 + m] = lam[m] * e + bb[m];
        a[m] = am;
        ta[m] = tam;
      }
      double dn = 0.0, tdn = 0.0;
      for (int m = 0; m < M; ++m) {
        dn += creal(conj(a[m]) * S[S1 + S2 + m]);
        tdn += creal(conj(ta[m]) * S[S1 + S2 + m] + conj(a[m]) * T[S1 + S2 + m]);
      }
      for (int f = 0; f < d_v; ++f) {
        double nf = 0.0, tnf = 0.0;
        for (int m = 0; m < M; ++m) {
          nf += creal(conj(a[m]) * S[S1 + m * d_v + f]);
          tnf += creal(conj(ta[m]) * S[S1 + m * d_v + f] + conj(a[m]) * T[S1 + m * d_v + f]);
        }
        double of = nf / dn;
        to_[rv + f] = (tnf - of * tdn) / dn;
      }
    }
    free(lam); free(bb); free(dl); free(dbb); free(S); free(T); free(a); free(ta);
  }
  return 0;
}
