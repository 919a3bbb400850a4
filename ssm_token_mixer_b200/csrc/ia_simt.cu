// IA layer on CUDA cores in fp32: per-head parameter tables of the chunked
// tensor-core path, the sequential recurrence (forward) and its reverse-mode
// adjoint (backward).
//
// The recurrence and readout follow the paper 'Interdomain Attention: Beyond
// Token-Level Key-Value Memory' (paperlayer.ai summary sec. 3.1-3.2; AI-radio
// page formula extract): one complex-diagonal S4D recurrence drives xi(k_t),
// v_t and 1; o_t = Re(a_t^H Gamma_t) / Re(a_t^H eta_t), a_t = U_t xi(q_t).
// These kernels carry any shape whose state fits in shared memory and serve
// fp32 inputs (parity at 1e-4) and shapes outside the tensor-core kernel.
#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"
#include "ia_simt_common.cuh"

namespace ia {


// ------------------------------------------------------------------------
// Parameter prologue for the tensor-core path: one block per head, four
// threads per mode.  Each thread covers 16 consecutive j: the powers
// lambda^(c-j) come from an fp64 recurrence started at a directly computed
// power (relative error ~16 * 2^-53); the sum of E' over the chunk is reduced
// across the four threads, and the remaining per-mode powers are shared out
// among them.  The E' table is staged in shared memory and written out with
// coalesced 16-byte stores.  With dtab, also the derivative tables of the
// reverse pass, [3][H][128][64] fp32 followed by their row sums [3][H][128]:
// table w, row k = 2m + comp, column j holds component comp of
//   w = 0: dE'[j,m]/dDelta_hm = lambda^n (lambda + n A b)
//   w = 1: dE'[j,m]/dA_m      = lambda^n ((Delta lambda - b)/A + n Delta b)
//   w = 2: i dE'[j,m]/dA_m    (the derivative along Im A_m)
// with n = c - j, so that the reverse pass contracts its adjoint of E' with
// each table to get dL/dDelta, dL/dRe A and dL/dIm A.
// The tensor-core operands carry factors up to |lambda_m|^(-C/2) =
// exp(Delta |Re A_m| C/2) in fp16 (the centred decay table and the readout
// scale); a head whose factor exceeds kMaxHalfChunkGrowth, or whose Delta is
// not positive, raises kErrParamRange in *err instead of returning numbers
// that may have overflowed.
constexpr double kMaxHalfChunkGrowth = 64.0;

__global__ void __launch_bounds__(4 * kModesTC) param_tables_kernel(int H, const float* __restrict__ delta,
                                                                    const float* __restrict__ A,
                                                                    HeadTables* __restrict__ tabs,
                                                                    float* __restrict__ dtab,
                                                                    int* __restrict__ err,
                                                                    int* __restrict__ flags, int nflags,
                                                                    int dpm) {
  __shared__ __align__(16) __half Es[2 * kModesTC * kChunk];
  griddep_launch_dependents();   // the chunk pass may start its table-free prologue now
  const int h = blockIdx.x;
  if (h == 0)   // the chunk pass's look-back flags start at zero
    for (int i = threadIdx.x; i < nflags; i += blockDim.x) flags[i] = 0;
  HeadTables* T = tabs + h;
  constexpr int C = kChunk, c = kChunk / 2, JS = kChunk / 4;
  const int m = threadIdx.x >> 2, part = threadIdx.x & 3;   // four threads per mode, adjacent lanes
  const float dl = delta_hm(delta, dpm, kModesTC, h, m);
  ModeD md = mode_consts(dl, A, m);
  const double rdA = dl * md.ar, idA = dl * md.ai;
  if (part == 0 && !(dl > 0.f && fabs(rdA) * (C / 2) <= log(kMaxHalfChunkGrowth))) atomicOr(err, kErrParamRange);
  // The powers of lambda the tables need, from lambda itself by complex
  // squarings, products and inverses in fp64 (relative error about n eps for
  // lambda^n, far below the fp16 and fp32 the tables store).
  auto cm = [](double ar, double ai, double br, double bi, double* r, double* i) {
    *r = ar * br - ai * bi;
    *i = ar * bi + ai * br;
  };
  auto cinv = [](double ar, double ai, double* r, double* i) {   // 1 / a = conj(a) / |a|^2
    const double n = ar * ar + ai * ai;
    *r = ar / n;
    *i = -ai / n;
  };
  double l16r = md.lr, l16i = md.li;
  for (int sq = 0; sq < 4; ++sq) cm(l16r, l16i, l16r, l16i, &l16r, &l16i);   // lambda^16
  double l32r, l32i, ir, ii;
  cm(l16r, l16i, l16r, l16i, &l32r, &l32i);                                 // lambda^32
  cinv(md.lr, md.li, &ir, &ii);                                              // lambda^-1
  static_assert(c == 32 && JS == 16, "the first powers below are lambda^32, ^16, ^0, ^-16");
  double pr, pi;   // lambda^(c-j) at this thread's first j
  if (part == 0) {
    pr = l32r;
    pi = l32i;
  } else if (part == 1) {
    pr = l16r;
    pi = l16i;
  } else if (part == 2) {
    pr = 1.0;
    pi = 0.0;
  } else {
    cinv(l16r, l16i, &pr, &pi);
  }
  double sr = 0.0, si = 0.0;
  double dsr[3] = {0.0, 0.0, 0.0}, dsi[3] = {0.0, 0.0, 0.0};
  char* base = reinterpret_cast<char*>(Es);
  const size_t tab_stride = static_cast<size_t>(H) * 2 * kModesTC * C;   // floats per derivative table
  // (Delta lambda - b) / A: the A-derivative of b, less its n Delta b part
  const double cr = dl * md.lr - md.br, ci = dl * md.li - md.bi, aa = md.ar * md.ar + md.ai * md.ai;
  const double gr = (cr * md.ar + ci * md.ai) / aa, gi = (ci * md.ar - cr * md.ai) / aa;
  for (int j = JS * part; j < JS * (part + 1); ++j) {   // E'[j] = b lambda^(c-j)
    const double er = md.br * pr - md.bi * pi, ei = md.br * pi + md.bi * pr;
    *reinterpret_cast<__half*>(base + etab_offset(2 * m, j)) = __double2half(er);
    *reinterpret_cast<__half*>(base + etab_offset(2 * m + 1, j)) = __double2half(ei);
    sr += er;
    si += ei;
    if (dtab) {
      const double n = c - j;
      // dDelta: lambda^n (lambda + n A b)
      const double fr = md.lr + n * (md.ar * md.br - md.ai * md.bi), fi = md.li + n * (md.ar * md.bi + md.ai * md.br);
      // dA: lambda^n ((Delta lambda - b)/A + n Delta b)
      const double hr = gr + n * dl * md.br, hi = gi + n * dl * md.bi;
      const double d0r = pr * fr - pi * fi, d0i = pr * fi + pi * fr;
      const double d1r = pr * hr - pi * hi, d1i = pr * hi + pi * hr;
      const double comp[3][2] = {{d0r, d0i}, {d1r, d1i}, {-d1i, d1r}};   // rows 2m, 2m+1 of each table
      for (int w = 0; w < 3; ++w) {
        float* row = dtab + w * tab_stride + (static_cast<size_t>(h) * 2 * kModesTC + 2 * m) * C;
        row[j] = static_cast<float>(comp[w][0]);
        row[C + j] = static_cast<float>(comp[w][1]);
        dsr[w] += comp[w][0];
        dsi[w] += comp[w][1];
      }
    }
    const double nr = pr * ir - pi * ii;
    pi = pr * ii + pi * ir;
    pr = nr;
  }
  // sums over the chunk: the four partial sums of this mode
  for (int off = 1; off < 4; off <<= 1) {
    sr += __shfl_xor_sync(0xffffffffu, sr, off);
    si += __shfl_xor_sync(0xffffffffu, si, off);
    for (int w = 0; w < 3; ++w) {
      dsr[w] += __shfl_xor_sync(0xffffffffu, dsr[w], off);
      dsi[w] += __shfl_xor_sync(0xffffffffu, dsi[w], off);
    }
  }
  if (dtab && part == 0) {   // row sums after the three tables
    for (int w = 0; w < 3; ++w) {
      float* dsum = dtab + 3 * tab_stride + (static_cast<size_t>(w) * H + h) * 2 * kModesTC;
      dsum[2 * m] = static_cast<float>(dsr[w]);
      dsum[2 * m + 1] = static_cast<float>(dsi[w]);
    }
  }
  if (part == 0) {
    T->lam[m] = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
    T->b[m] = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
    T->esum[m] = make_float2(static_cast<float>(sr), static_cast<float>(si));
    T->re_dA[m] = rdA;
    T->im_dA[m] = idA;
  } else if (part == 1) {
    static_assert(C == 64, "lambda^C is lambda^32 squared");
    cm(l32r, l32i, l32r, l32i, &pr, &pi);
    T->lamC[m] = make_float2(static_cast<float>(pr), static_cast<float>(pi));
    T->r2[m] = static_cast<float>(md.lr * md.lr + md.li * md.li);   // |lambda|^2
  } else if (part == 2) {
    cm(l32r, l32i, ir, ii, &pr, &pi);   // lambda^(C-c-1) = lambda^31
    T->sc[m] = make_float2(static_cast<float>(pr), static_cast<float>(pi));
    T->s0[m] = static_cast<float>(1.0 / (l32r * l32r + l32i * l32i));   // |lambda|^(-2c)
  } else {
    double tr, ti;
    cm(l32r, l32i, ir, ii, &tr, &ti);
    cinv(tr, ti, &pr, &pi);   // lambda^-(C-c-1)
    T->sc_inv[m] = make_float2(static_cast<float>(pr), static_cast<float>(pi));
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(Es);
  uint4* dst = reinterpret_cast<uint4*>(T->E);
  for (int i = threadIdx.x; i < 2 * kModesTC * kChunk * 2 / 16; i += blockDim.x) dst[i] = src[i];
}

// ------------------------------------------------------------------------
// Sequential forward: one block per (b,h); state in shared memory.
// Shared layout (float2): U [M*DX] | G [M*DV] | eta [M] | lam [M] | b [M] | a [M]
// followed by floats fq [DX] | fk [DX] | vv [DV].
template <typename T>
__global__ void seq_fwd_kernel(int H, int N, int DX, int DV, int M, const T* __restrict__ q,
                               const T* __restrict__ k, const T* __restrict__ v,
                               const float* __restrict__ delta, int dpm, const float* __restrict__ A,
                               const float2* __restrict__ state_in, float* __restrict__ o,
                               float* __restrict__ num, float* __restrict__ den,
                               float2* __restrict__ state_out, long long BH) {
  extern __shared__ float4 smem_f4[];
  float2* U = reinterpret_cast<float2*>(smem_f4);
  float2* G = U + M * DX;
  float2* eta = G + M * DV;
  float2* lam = eta + M;
  float2* bb = lam + M;
  float2* a = bb + M;
  float* fq = reinterpret_cast<float*>(a + M);
  float* fk = fq + DX;
  float* vv = fk + DX;

  const long long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nwarp = nthr >> 5;

  for (int m = tid; m < M; m += nthr) {
    ModeD md = mode_consts(delta_hm(delta, dpm, M, h, m), A, m);
    lam[m] = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
    bb[m] = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
  }
  const long long u0 = bh * M * DX, g0 = BH * M * DX + bh * M * DV, e0 = BH * M * (DX + DV) + bh * M;
  for (int i = tid; i < M * DX; i += nthr) U[i] = state_in ? state_in[u0 + i] : make_float2(0.f, 0.f);
  for (int i = tid; i < M * DV; i += nthr) G[i] = state_in ? state_in[g0 + i] : make_float2(0.f, 0.f);
  for (int i = tid; i < M; i += nthr) eta[i] = state_in ? state_in[e0 + i] : make_float2(0.f, 0.f);
  __syncthreads();

  const T* qb = q + bh * N * DX;
  const T* kb = k + bh * N * DX;
  const T* vb = v + bh * N * DV;
  for (int t = 0; t < N; ++t) {
    for (int f = tid; f < DX; f += nthr) {
      fq[f] = feat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
      fk[f] = feat_acc(ldf(kb + static_cast<long long>(t) * DX + f));
    }
    for (int f = tid; f < DV; f += nthr) vv[f] = ldf(vb + static_cast<long long>(t) * DV + f);
    __syncthreads();
    for (int m = warp; m < M; m += nwarp) {
      const float2 L = lam[m], Bm = bb[m];
      float ar = 0.f, ai = 0.f;
      for (int f = lane; f < DX; f += 32) {
        float2 u = cfma(L, U[m * DX + f], make_float2(Bm.x * fk[f], Bm.y * fk[f]));
        U[m * DX + f] = u;
        ar = fmaf(u.x, fq[f], ar);
        ai = fmaf(u.y, fq[f], ai);
      }
      for (int f = lane; f < DV; f += 32)
        G[m * DV + f] = cfma(L, G[m * DV + f], make_float2(Bm.x * vv[f], Bm.y * vv[f]));
      ar = warp_sum(ar);
      ai = warp_sum(ai);
      if (lane == 0) {
        a[m] = make_float2(ar, ai);
        eta[m] = cfma(L, eta[m], Bm);
      }
    }
    __syncthreads();
    float dn = 0.f;
    for (int m = 0; m < M; ++m) dn += re_conj_mul(a[m], eta[m]);
    const long long row = (bh * N + t);
    for (int f = tid; f < DV; f += nthr) {
      float nf = 0.f;
      for (int m = 0; m < M; ++m) nf += re_conj_mul(a[m], G[m * DV + f]);
      o[row * DV + f] = nf / dn;
      if (num) num[row * DV + f] = nf;
    }
    if (den && tid == 0) den[row] = dn;
    __syncthreads();
  }
  if (state_out) {
    for (int i = tid; i < M * DX; i += nthr) state_out[u0 + i] = U[i];
    for (int i = tid; i < M * DV; i += nthr) state_out[g0 + i] = G[i];
    for (int i = tid; i < M; i += nthr) state_out[e0 + i] = eta[i];
  }
}

// ------------------------------------------------------------------------
// Sequential reverse mode from a zero state.  One block per (b,h).  The
// forward sweep stores the state before every block of kCk tokens, o and
// den; the reverse sweep recomputes each block's states into global scratch
// and runs the adjoint recurrence G_t = g_t + conj(lambda) G_{t+1} with the
// adjoint G in shared memory:
//   dnum = dO/den, dden = -(dO . o)/den
//   gbar_a = Gamma_t dnum + eta_t dden;     dxi(q_t) = Re(U_t^H gbar_a)
//   G^U += gbar_a xi(q_t)^T, G^Gamma += a_t dnum^T, G^eta += a_t dden
//   dxi(k_t) = Re(b^H G^U),  dv_t = Re(b^H G^Gamma)
//   gbar_lambda += G . conj(S_{t-1}),  gbar_b += G . x_t
//   dDelta_h += sum_m Re(conj(gbar_lambda) A lambda + conj(gbar_b) lambda)
constexpr int kCk = 64;

template <typename T>
__global__ void seq_bwd_kernel(int H, int N, int DX, int DV, int M, const T* __restrict__ q,
                               const T* __restrict__ k, const T* __restrict__ v,
                               const T* __restrict__ dO, const float* __restrict__ delta, int dpm,
                               const float* __restrict__ A, float* __restrict__ o,
                               float* __restrict__ dq, float* __restrict__ dk,
                               float* __restrict__ dv, float* __restrict__ gpart,
                               float2* __restrict__ ws, long long per_bh) {
  extern __shared__ float4 smem_f4[];
  const int SL = M * (DX + DV + 1);
  float2* Gs = reinterpret_cast<float2*>(smem_f4);  // adjoint [SL]
  float2* lam = Gs + SL;
  float2* bb = lam + M;
  float2* a = bb + M;
  float2* ga = a + M;
  float2* glam = ga + M;
  float2* gbs = glam + M;
  float2* Am = gbs + M;
  float* fq = reinterpret_cast<float*>(Am + M);
  float* fk = fq + DX;
  float* vv = fk + DX;
  float* dn = vv + DV;   // dnum [DV]
  float* red = dn + DV;  // [32] reduction scratch

  const long long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nwarp = nthr >> 5;
  const int nck = (N + kCk - 1) / kCk;
  float2* ck = ws + bh * per_bh;                 // [nck][SL]
  float2* blk = ck + static_cast<long long>(nck) * SL;      // [kCk+1][SL]
  float* den_ws = reinterpret_cast<float*>(blk + static_cast<long long>(kCk + 1) * SL);  // [N]

  for (int m = tid; m < M; m += nthr) {
    ModeD md = mode_consts(delta_hm(delta, dpm, M, h, m), A, m);
    lam[m] = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
    bb[m] = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
    Am[m] = make_float2(static_cast<float>(md.ar), static_cast<float>(md.ai));
    glam[m] = make_float2(0.f, 0.f);
    gbs[m] = make_float2(0.f, 0.f);
  }
  // Forward sweep in global scratch (blk[0] is the running state).
  float2* cur = blk;
  for (int i = tid; i < SL; i += nthr) cur[i] = make_float2(0.f, 0.f);
  __syncthreads();
  const T* qb = q + bh * N * DX;
  const T* kb = k + bh * N * DX;
  const T* vb = v + bh * N * DV;
  const T* gb = dO + bh * N * DV;
  for (int t = 0; t < N; ++t) {
    if (t % kCk == 0) {
      float2* dst = ck + static_cast<long long>(t / kCk) * SL;
      for (int i = tid; i < SL; i += nthr) dst[i] = cur[i];
    }
    for (int f = tid; f < DX; f += nthr) {
      fq[f] = feat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
      fk[f] = feat_acc(ldf(kb + static_cast<long long>(t) * DX + f));
    }
    for (int f = tid; f < DV; f += nthr) vv[f] = ldf(vb + static_cast<long long>(t) * DV + f);
    __syncthreads();
    for (int m = warp; m < M; m += nwarp) {
      const float2 L = lam[m], Bm = bb[m];
      float ar = 0.f, ai = 0.f;
      for (int f = lane; f < DX; f += 32) {
        float2 u = cfma(L, cur[m * DX + f], make_float2(Bm.x * fk[f], Bm.y * fk[f]));
        cur[m * DX + f] = u;
        ar = fmaf(u.x, fq[f], ar);
        ai = fmaf(u.y, fq[f], ai);
      }
      for (int f = lane; f < DV; f += 32)
        cur[M * DX + m * DV + f] =
            cfma(L, cur[M * DX + m * DV + f], make_float2(Bm.x * vv[f], Bm.y * vv[f]));
      ar = warp_sum(ar);
      ai = warp_sum(ai);
      if (lane == 0) {
        a[m] = make_float2(ar, ai);
        cur[M * (DX + DV) + m] = cfma(L, cur[M * (DX + DV) + m], Bm);
      }
    }
    __syncthreads();
    float d_ = 0.f;
    for (int m = 0; m < M; ++m) d_ += re_conj_mul(a[m], cur[M * (DX + DV) + m]);
    const long long row = bh * N + t;
    for (int f = tid; f < DV; f += nthr) {
      float nf = 0.f;
      for (int m = 0; m < M; ++m) nf += re_conj_mul(a[m], cur[M * DX + m * DV + f]);
      o[row * DV + f] = nf / d_;
    }
    if (tid == 0) den_ws[t] = d_;
    __syncthreads();
  }

  // Reverse sweep.
  for (int i = tid; i < SL; i += nthr) Gs[i] = make_float2(0.f, 0.f);
  __syncthreads();
  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * kCk, t1 = min(t0 + kCk, N);
    const float2* src = ck + static_cast<long long>(c) * SL;
    for (int i = tid; i < SL; i += nthr) blk[i] = src[i];
    __syncthreads();
    for (int t = t0; t < t1; ++t) {   // blk[t - t0 + 1] = S_t
      const float2* prev = blk + static_cast<long long>(t - t0) * SL;
      float2* nxt = blk + static_cast<long long>(t - t0 + 1) * SL;
      for (int f = tid; f < DX; f += nthr) fk[f] = feat_acc(ldf(kb + static_cast<long long>(t) * DX + f));
      for (int f = tid; f < DV; f += nthr) vv[f] = ldf(vb + static_cast<long long>(t) * DV + f);
      __syncthreads();
      for (int i = tid; i < SL; i += nthr) {
        int m, f;
        float x;
        if (i < M * DX) { m = i / DX; f = i % DX; x = fk[f]; }
        else if (i < M * (DX + DV)) { m = (i - M * DX) / DV; f = (i - M * DX) % DV; x = vv[f]; }
        else { m = i - M * (DX + DV); x = 1.f; }
        nxt[i] = cfma(lam[m], prev[i], make_float2(bb[m].x * x, bb[m].y * x));
      }
      __syncthreads();
    }
    for (int t = t1 - 1; t >= t0; --t) {
      const float2* St = blk + static_cast<long long>(t - t0 + 1) * SL;
      const float2* Sp = blk + static_cast<long long>(t - t0) * SL;
      const long long row = bh * N + t;
      const float dent = den_ws[t];
      for (int f = tid; f < DX; f += nthr) {
        fq[f] = feat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
        fk[f] = feat_acc(ldf(kb + static_cast<long long>(t) * DX + f));
      }
      float part = 0.f;
      for (int f = tid; f < DV; f += nthr) {
        float g = ldf(gb + static_cast<long long>(t) * DV + f);
        vv[f] = ldf(vb + static_cast<long long>(t) * DV + f);
        dn[f] = g / dent;
        part += g * o[row * DV + f];
      }
      part = warp_sum(part);
      if (lane == 0) red[warp] = part;
      __syncthreads();
      float dden = 0.f;
      for (int w = 0; w < nwarp; ++w) dden += red[w];
      dden = -dden / dent;
      // a_t and gbar_a (warp per mode)
      for (int m = warp; m < M; m += nwarp) {
        float ar = 0.f, ai = 0.f, gr = 0.f, gi = 0.f;
        for (int f = lane; f < DX; f += 32) {
          float2 u = St[m * DX + f];
          ar = fmaf(u.x, fq[f], ar);
          ai = fmaf(u.y, fq[f], ai);
        }
        for (int f = lane; f < DV; f += 32) {
          float2 g = St[M * DX + m * DV + f];
          gr = fmaf(g.x, dn[f], gr);
          gi = fmaf(g.y, dn[f], gi);
        }
        ar = warp_sum(ar); ai = warp_sum(ai); gr = warp_sum(gr); gi = warp_sum(gi);
        if (lane == 0) {
          float2 e = St[M * (DX + DV) + m];
          a[m] = make_float2(ar, ai);
          ga[m] = make_float2(fmaf(e.x, dden, gr), fmaf(e.y, dden, gi));
        }
      }
      __syncthreads();
      for (int f = tid; f < DX; f += nthr) {
        float s = 0.f;
        for (int m = 0; m < M; ++m) s += re_conj_mul(ga[m], St[m * DX + f]);
        dq[row * DX + f] = s * dfeat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
      }
      // add local adjoints, accumulate gbar_lambda / gbar_b (warp per mode)
      for (int m = warp; m < M; m += nwarp) {
        const float2 gam = ga[m], am = a[m];
        float lr = 0.f, li = 0.f, br_ = 0.f, bi_ = 0.f;
        for (int f = lane; f < DX; f += 32) {
          float2 g = Gs[m * DX + f];
          g.x = fmaf(gam.x, fq[f], g.x);
          g.y = fmaf(gam.y, fq[f], g.y);
          Gs[m * DX + f] = g;
          float2 p = Sp[m * DX + f];   // G * conj(p)
          lr += g.x * p.x + g.y * p.y;
          li += g.y * p.x - g.x * p.y;
          br_ = fmaf(g.x, fk[f], br_);
          bi_ = fmaf(g.y, fk[f], bi_);
        }
        for (int f = lane; f < DV; f += 32) {
          float2 g = Gs[M * DX + m * DV + f];
          g.x = fmaf(am.x, dn[f], g.x);
          g.y = fmaf(am.y, dn[f], g.y);
          Gs[M * DX + m * DV + f] = g;
          float2 p = Sp[M * DX + m * DV + f];
          lr += g.x * p.x + g.y * p.y;
          li += g.y * p.x - g.x * p.y;
          br_ = fmaf(g.x, vv[f], br_);
          bi_ = fmaf(g.y, vv[f], bi_);
        }
        lr = warp_sum(lr); li = warp_sum(li); br_ = warp_sum(br_); bi_ = warp_sum(bi_);
        if (lane == 0) {
          float2 g = Gs[M * (DX + DV) + m];
          g.x = fmaf(am.x, dden, g.x);
          g.y = fmaf(am.y, dden, g.y);
          Gs[M * (DX + DV) + m] = g;
          float2 p = Sp[M * (DX + DV) + m];
          lr += g.x * p.x + g.y * p.y;
          li += g.y * p.x - g.x * p.y;
          br_ += g.x;
          bi_ += g.y;
          glam[m] = make_float2(glam[m].x + lr, glam[m].y + li);
          gbs[m] = make_float2(gbs[m].x + br_, gbs[m].y + bi_);
        }
      }
      __syncthreads();
      for (int f = tid; f < DX; f += nthr) {
        float s = 0.f;
        for (int m = 0; m < M; ++m) s += re_conj_mul(bb[m], Gs[m * DX + f]);
        dk[row * DX + f] = s * dfeat_acc(ldf(kb + static_cast<long long>(t) * DX + f));
      }
      for (int f = tid; f < DV; f += nthr) {
        float s = 0.f;
        for (int m = 0; m < M; ++m) s += re_conj_mul(bb[m], Gs[M * DX + m * DV + f]);
        dv[row * DV + f] = s;
      }
      __syncthreads();
      for (int i = tid; i < SL; i += nthr) {
        int m = i < M * DX ? i / DX : (i < M * (DX + DV) ? (i - M * DX) / DV : i - M * (DX + DV));
        float2 L = lam[m];
        Gs[i] = cmul(make_float2(L.x, -L.y), Gs[i]);
      }
      __syncthreads();
    }
  }
  // this sequence's share of the parameter gradients, per mode:
  //   dL/dDelta_hm = Re(conj(gbar_lambda) A lambda + conj(gbar_b) lambda)
  //   dL/dA_m      = conj(Delta lambda) gbar_lambda + conj((Delta lambda - b)/A) gbar_b
  for (int m = tid; m < M; m += nthr) {
    const float dl = delta_hm(delta, dpm, M, h, m);
    const float2 Al = cmul(Am[m], lam[m]);
    const float2 dlam = make_float2(dl * lam[m].x, dl * lam[m].y);
    const float2 num_ = make_float2(dlam.x - bb[m].x, dlam.y - bb[m].y);
    const float aa = fmaf(Am[m].x, Am[m].x, Am[m].y * Am[m].y);
    const float2 dbdA = make_float2(fmaf(num_.x, Am[m].x, num_.y * Am[m].y) / aa,
                                    fmaf(num_.y, Am[m].x, -num_.x * Am[m].y) / aa);
    float* out = gpart + (bh * M + m) * 3;
    out[0] = re_conj_mul(glam[m], Al) + re_conj_mul(gbs[m], lam[m]);
    // conj(x) g summed: real part Re(conj(x) g), imaginary part Im(conj(x) g)
    out[1] = re_conj_mul(dlam, glam[m]) + re_conj_mul(dbdA, gbs[m]);
    out[2] = (dlam.x * glam[m].y - dlam.y * glam[m].x) + (dbdA.x * gbs[m].y - dbdA.y * gbs[m].x);
  }
}

// ------------------------------------------------------------------------
// host-side launchers
cudaError_t launch_param_tables(int H, const float* delta, int dpm, const float* A, HeadTables* tabs,
                                cudaStream_t st, float* dtab, int* flags, int nflags) {
  int* err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  param_tables_kernel<<<H, 4 * kModesTC, 0, st>>>(H, delta, A, tabs, dtab, err, flags, nflags, dpm);
  return cudaGetLastError();
}

size_t seq_fwd_smem(int DX, int DV, int M) {
  return sizeof(float2) * (static_cast<size_t>(M) * (DX + DV) + 4 * M) + sizeof(float) * (2 * DX + DV) + 16;
}

template <typename T>
static cudaError_t seq_fwd_impl(const ia_shape_t& s, const void* q, const void* k, const void* v,
                                const float* delta, const float* A, const void* state_in,
                                float* o, float* num, float* den, void* state_out,
                                cudaStream_t st) {
  size_t smem = seq_fwd_smem(s.d_xi, s.d_v, s.M);
  auto kern = seq_fwd_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  long long BH = static_cast<long long>(s.B) * s.H;
  mark_launch_begin(st);
  kern<<<static_cast<unsigned>(BH), 256, smem, st>>>(
      s.H, s.N, s.d_xi, s.d_v, s.M, static_cast<const T*>(q), static_cast<const T*>(k),
      static_cast<const T*>(v), delta, s.delta_per_mode, A, static_cast<const float2*>(state_in), o, num, den,
      static_cast<float2*>(state_out), BH);
  e = cudaGetLastError();
  mark_launch_end(st);
  return e;
}

cudaError_t launch_seq_fwd(const ia_shape_t& s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, const void* state_in, float* o,
                           float* num, float* den, void* state_out, cudaStream_t st) {
  if (s.in_dtype == IA_F32)
    return seq_fwd_impl<float>(s, q, k, v, delta, A, state_in, o, num, den, state_out, st);
  return seq_fwd_impl<__nv_bfloat16>(s, q, k, v, delta, A, state_in, o, num, den, state_out, st);
}

size_t seq_bwd_smem(int DX, int DV, int M) {
  size_t SL = static_cast<size_t>(M) * (DX + DV + 1);
  return sizeof(float2) * (SL + 7 * static_cast<size_t>(M)) + sizeof(float) * (2 * DX + 2 * DV + 32) + 16;
}

size_t seq_bwd_ws_per_bh(int N, int DX, int DV, int M) {   // in float2 units
  size_t SL = static_cast<size_t>(M) * (DX + DV + 1);
  size_t nck = (N + kCk - 1) / kCk;
  size_t n = nck * SL + (kCk + 1) * SL + (N + 1) / 2 + 1;
  return (n + 31) & ~static_cast<size_t>(31);
}

size_t seq_bwd_workspace_bytes(const ia_shape_t& s) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  return sizeof(float2) * BH * seq_bwd_ws_per_bh(s.N, s.d_xi, s.d_v, s.M) + 256 +
         grad_partials_bytes(s) + 256;
}

template <typename T>
static cudaError_t seq_bwd_impl(const ia_shape_t& s, const void* q, const void* k, const void* v,
                                const float* delta, const float* A, const void* dO, float* o,
                                float* dq, float* dk, float* dv, float* dDelta, float* dA, void* ws,
                                cudaStream_t st) {
  size_t smem = seq_bwd_smem(s.d_xi, s.d_v, s.M);
  auto kern = seq_bwd_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  long long BH = static_cast<long long>(s.B) * s.H;
  const long long per_bh = static_cast<long long>(seq_bwd_ws_per_bh(s.N, s.d_xi, s.d_v, s.M));
  float2* scratch = static_cast<float2*>(ws);
  uintptr_t gp = reinterpret_cast<uintptr_t>(scratch + BH * per_bh);
  float* gpart = reinterpret_cast<float*>((gp + 255) & ~static_cast<uintptr_t>(255));
  mark_launch_begin(st);
  kern<<<static_cast<unsigned>(BH), 256, smem, st>>>(
      s.H, s.N, s.d_xi, s.d_v, s.M, static_cast<const T*>(q), static_cast<const T*>(k),
      static_cast<const T*>(v), static_cast<const T*>(dO), delta, s.delta_per_mode, A, o, dq, dk, dv, gpart,
      scratch, per_bh);
  e = cudaGetLastError();
  mark_launch_end(st);
  if (e != cudaSuccess) return e;
  return launch_grad_reduce(s, gpart, dDelta, dA, st);
}

cudaError_t launch_seq_bwd(const ia_shape_t& s, const void* q, const void* k, const void* v,
                           const float* delta, const float* A, const void* dO, float* o, float* dq,
                           float* dk, float* dv, float* dDelta, float* dA, void* ws, cudaStream_t st) {
  if (s.in_dtype == IA_F32)
    return seq_bwd_impl<float>(s, q, k, v, delta, A, dO, o, dq, dk, dv, dDelta, dA, ws, st);
  return seq_bwd_impl<__nv_bfloat16>(s, q, k, v, delta, A, dO, o, dq, dk, dv, dDelta, dA, ws, st);
}

// ------------------------------------------------------------------------
// dDelta and dA from the per-(b,h,m) partials of a reverse pass, summed in a
// fixed order (b, then h, then m), so that the result is the same on every
// run.  One thread per output: dDelta[h] or dDelta[h][m], then dA[m].
__global__ void grad_reduce_kernel(int B, int H, int M, int dpm, const float* __restrict__ gpart,
                                   float* __restrict__ dDelta, float* __restrict__ dA) {
  const int nD = dpm ? H * M : H;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < nD) {
    const int h = dpm ? idx / M : idx;
    const int m0 = dpm ? idx % M : 0, m1 = dpm ? m0 + 1 : M;
    float acc = 0.f;
    for (int b = 0; b < B; ++b)
      for (int m = m0; m < m1; ++m) acc += gpart[((static_cast<long long>(b) * H + h) * M + m) * 3];
    dDelta[idx] = acc;
  } else if (dA && idx < nD + M) {
    const int m = idx - nD;
    float re = 0.f, im = 0.f;
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h) {
        const float* p = gpart + ((static_cast<long long>(b) * H + h) * M + m) * 3;
        re += p[1];
        im += p[2];
      }
    dA[2 * m] = re;
    dA[2 * m + 1] = im;
  }
}

size_t grad_partials_bytes(const ia_shape_t& s) {
  return sizeof(float) * 3 * static_cast<size_t>(s.B) * s.H * s.M;
}

cudaError_t launch_grad_reduce(const ia_shape_t& s, const float* gpart, float* dDelta, float* dA,
                               cudaStream_t st) {
  const int n = (s.delta_per_mode ? s.H * s.M : s.H) + s.M;
  grad_reduce_kernel<<<(n + 127) / 128, 128, 0, st>>>(s.B, s.H, s.M, s.delta_per_mode, gpart, dDelta, dA);
  return cudaGetLastError();
}

}  // namespace ia
