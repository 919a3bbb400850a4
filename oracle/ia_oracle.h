/*
 * Interdomain Attention (IA) -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path under
 * ssm_token_mixer_b200/csrc.
 *
 * What it computes (paper "Interdomain Attention: Beyond Token-Level
 * Key-Value Memory", Kiyohara et al.; the paperlayer.ai summary, section 3.2
 * "A practical implementation", and the formula extract on the AI-radio page,
 * "Key Components and Derivation"):
 *
 *   xi(x)   = elu(x) + 1            (positive finite feature map)
 *   lambda_m = exp(Delta_h * A_m),  b_m = (lambda_m - 1) / A_m      (ZOH of S4D;
 *              Delta_hm per mode when the caller asks for it)
 *   A_m     = -1/2 + i*pi*m  (S4D-Lin) unless the caller passes A
 *   U_t     = lambda U_{t-1} + b xi(k_t)^T      (M x d_xi, complex)
 *   Gamma_t = lambda Gamma_{t-1} + b v_t^T      (M x d_v,  complex)
 *   eta_t   = lambda eta_{t-1} + b              (M,        complex)
 *   a_t     = U_t xi(q_t)                       (M, complex)
 *   num_t   = Re(a_t^H Gamma_t),  den_t = Re(a_t^H eta_t),  o_t = num_t / den_t
 *
 * which is the pages' matrix form O = F_q U^T Gamma / F_q U^T eta with the
 * query-side conjugate and real part made explicit.
 *
 * Layout conventions (all host memory, row-major, fp64):
 *   q, k : [B,H,N,d_xi]     v, o, num : [B,H,N,d_v]     den : [B,H,N]
 *   delta: [H], or [H,M] with dpm = 1 (one Delta per head and mode)
 *   A    : [M] complex as (re,im) pairs, or NULL (S4D-Lin)
 *   state: one buffer  U [B,H,M,d_xi] | Gamma [B,H,M,d_v] | eta [B,H,M],
 *          each complex entry stored as (re,im); NULL state_in = zero state.
 * Every function returns 0 on success and a negative value on bad arguments.
 */
#ifndef IA_ORACLE_H
#define IA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* Number of doubles in one state buffer. */
long iao_state_len(int B, int H, int M, int d_xi, int d_v);

/* lambda_m and b_m for one head: lam, b are [M] complex (re,im) pairs. */
int iao_params(int M, double delta, const double* A, double* lam, double* b);

/* Causal layer forward over N tokens (sequential recurrence).
 * num, den, state_out may be NULL. */
int iao_forward(int B, int H, int N, int d_xi, int d_v, int M,
                const double* q, const double* k, const double* v,
                const double* delta, int dpm, const double* A, const double* state_in,
                double* o, double* num, double* den, double* state_out);

/* Same recurrence, but on features that are already mapped (fq = xi(q),
 * fk = xi(k)) and on explicit per-head lambda/b tables [H,M] complex.
 * Lets the pins scale features and split mode sets. */
int iao_forward_features(int B, int H, int N, int d_xi, int d_v, int M,
                         const double* fq, const double* fk, const double* v,
                         const double* lam, const double* b, const double* state_in,
                         double* o, double* num, double* den, double* state_out);

/* One recurrent decode step: q,k [B,H,d_xi], v [B,H,d_v]; state in place. */
int iao_decode_step(int B, int H, int d_xi, int d_v, int M,
                    const double* q, const double* k, const double* v,
                    const double* delta, int dpm, const double* A, double* state,
                    double* o, double* num, double* den);

/* O(N^2 M) quadratic-form evaluation from a zero state, with every decay
 * power taken as exp(n * Delta * A_m) directly (no recurrence). */
int iao_brute(int B, int H, int N, int d_xi, int d_v, int M,
              const double* q, const double* k, const double* v,
              const double* delta, int dpm, const double* A,
              double* o, double* num, double* den);

/* Reverse mode of iao_forward from a zero state.  dO [B,H,N,d_v] -> dq, dk
 * [B,H,N,d_xi], dv [B,H,N,d_v], dDelta [H] or [H,M] (as delta; summed over
 * batch and time) and dA [M] complex (dL/dRe A_m, dL/dIm A_m; summed over
 * batch, heads and time).  o and dA may be NULL. */
int iao_backward(int B, int H, int N, int d_xi, int d_v, int M,
                 const double* q, const double* k, const double* v,
                 const double* delta, int dpm, const double* A, const double* dO,
                 double* o, double* dq, double* dk, double* dv, double* dDelta, double* dA);

/* Forward-mode tangent of iao_forward from a zero state along the direction
 * (tq, tk, tv, tdelta[, tA]): writes the output tangent to_ [B,H,N,d_v].
 * tdelta has delta's shape; tA [M] complex or NULL. */
int iao_jvp(int B, int H, int N, int d_xi, int d_v, int M,
            const double* q, const double* k, const double* v,
            const double* delta, int dpm, const double* A,
            const double* tq, const double* tk, const double* tv, const double* tdelta,
            const double* tA, double* to_);

/* Extended forward: the layer with its optional parts, each off when its
 * argument is NULL (all off = iao_forward): RMSNorm with per-head gain and
 * bias [H, d_xi+d_v] on the SSM input (xi(k_t), v_t); a step per token
 * delta_t [B,H,N] (selective writing and memory decay; delta then unused);
 * a complex readout matrix W [H,M,M] mixing the query's mode coefficients.
 * map_features = 0 takes q, k as already-mapped features. */
int iao_forward_ex(int B, int H, int N, int d_xi, int d_v, int M,
                   const double* q, const double* k, const double* v, int map_features,
                   const double* delta, int dpm, const double* A, const double* delta_t,
                   const double* gain, const double* bias, double eps, const double* W,
                   const double* state_in, double* o, double* num, double* den,
                   double* state_out);

/* Threads the OpenMP loops will use (for reporting). */
int iao_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
