// The layer with its optional parts, on CUDA cores in fp32 (one CTA per
// segment of a (b,h), token after token), behind ia_prefill_fwd_ex where its
// tensor-core form does not apply, and behind ia_decode_step_ex.
//
// The optional parts are the ones the pages name beside the plain layer
// (paper 'Interdomain Attention: Beyond Token-Level Key-Value Memory'):
//   - input stabilisation (AI-radio page, "Implementation Details"): the SSM
//     input z_t = (xi(k_t), v_t) passes an RMSNorm with a learnable per-head
//     bias, z <- z / sqrt(mean(z^2) + eps) * gain_h + bias_h;
//   - selective writing and memory decay (paperlayer.ai summary, sec. 3.3 and
//     sec. 5.3): a step per token, lambda_t = exp(Delta_t A), b_t = (lambda_t - 1)/A;
//   - the full complex readout matrix (summary sec. A.3; the M^2 term of the
//     decode cost, sec. 3.2): a~_t = W_h a_t before num = Re(a~^H Gamma),
//     den = Re(a~^H eta);
//   - the bidirectional pass (summary sec. 5.2, Caduceus-IA keeps Caduceus'
//     bidirectional handling): o = f(x) + flip(f(flip x)), the second term a
//     second launch that reads and writes the sequence back to front and adds
//     its output to the first.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_simt_common.cuh"

namespace ia {
namespace {

// shared (float2): U [M*DX] | G [M*DV] | eta [M] | lam [M] | b [M] | a [M] | a~ [M]
// then floats: fq [DX] | z [DX + DV] | red [32]; then, when it fits, the
// head's readout matrix W_h [M*M] (float2)
size_t ex_smem(int DX, int DV, int M) {
  return sizeof(float2) * (static_cast<size_t>(M) * (DX + DV) + 5 * M) + sizeof(float) * (2 * DX + DV + 32) + 16;
}
size_t ex_smem_w(int M) { return sizeof(float2) * static_cast<size_t>(M) * M; }

struct ExArgs {
  const float* delta;     // [H] or [H,M] (unused with delta_t)
  int dpm;
  const float* A;
  const float* delta_t;   // [B,H,N] or null
  const float* gain;      // [H, DX+DV] or null
  const float* bias;      // [H, DX+DV] or null
  float eps;
  const float* W;         // [H,M,M] complex or null
  const float2* state_in;
  float2* state_out;
  float* o;
  float* num;
  float* den;
  int reverse;            // read and write tokens back to front
  int accumulate;         // add o to what is there instead of overwriting it
  int w_smem;             // W_h is staged in shared memory
  // The sequence may be cut into nseg segments of seg_len steps, one CTA
  // each, in two passes around a carry composition (the summary's sec. A.2):
  // pass 1 runs segments 0 .. nseg-2 for their end states only (segment 0
  // from state_in, the others from zero) into seg, and the step sums of
  // delta into dsum; ex_carry_kernel turns slot s of seg into the state
  // entering segment s+1; pass 2 (or the single pass, nseg = 1) runs every
  // segment from its entering state with the readout.
  int nseg, seg_len, pass;
  float2* seg;            // [BH][nseg-1][M (DX + DV + 1)]
  double* dsum;           // [BH][nseg]: sum of delta_t over the segment's tokens
};

template <typename T>
__global__ void __launch_bounds__(256, 3) seq_fwd_ex_kernel(int H, int N, int DX, int DV, int M, const T* __restrict__ q,
                                                         const T* __restrict__ k, const T* __restrict__ v,
                                                         const ExArgs a, long long BH) {
  extern __shared__ float4 smem_f4[];
  float2* U = reinterpret_cast<float2*>(smem_f4);
  float2* G = U + M * DX;
  float2* eta = G + M * DV;
  float2* lam = eta + M;
  float2* bb = lam + M;
  float2* av = bb + M;
  float2* at = av + M;
  float* fq = reinterpret_cast<float*>(at + M);
  float* z = fq + DX;            // [DX + DV]: xi(k) then v, normalised when asked
  float* red = z + DX + DV;      // [32]
  // W_h after the floats, on a 16-byte boundary
  float2* Ws = reinterpret_cast<float2*>((reinterpret_cast<uintptr_t>(red + 32) + 15) & ~static_cast<uintptr_t>(15));

  const long long bh = blockIdx.x / a.nseg;
  const int sg = static_cast<int>(blockIdx.x - bh * a.nseg);
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int step0 = sg * a.seg_len, step1 = min(N, step0 + a.seg_len);
  const bool readout = a.pass != 1;
  if (!readout && sg == a.nseg - 1) return;   // pass 1: the last segment's end state is not needed
  const int SW = M * (DX + DV + 1);   // complex entries of one (b,h) state
  float2* slot_in = sg > 0 ? a.seg + (bh * (a.nseg - 1) + (sg - 1)) * SW : nullptr;
  const int warp = tid >> 5, lane = tid & 31, nwarp = nthr >> 5;
  const int D = DX + DV;
  const bool norm = a.gain || a.bias;

  if (!a.delta_t) {
    for (int m = tid; m < M; m += nthr) {
      const ModeD md = mode_consts(delta_hm(a.delta, a.dpm, M, h, m), a.A, m);
      lam[m] = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
      bb[m] = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
    }
  }
  const long long u0 = bh * M * DX, g0 = BH * M * DX + bh * M * DV, e0 = BH * M * (DX + DV) + bh * M;
  if (sg == 0) {   // the caller's state (public layout), or zero
    for (int i = tid; i < M * DX; i += nthr) U[i] = a.state_in ? a.state_in[u0 + i] : make_float2(0.f, 0.f);
    for (int i = tid; i < M * DV; i += nthr) G[i] = a.state_in ? a.state_in[g0 + i] : make_float2(0.f, 0.f);
    for (int i = tid; i < M; i += nthr) eta[i] = a.state_in ? a.state_in[e0 + i] : make_float2(0.f, 0.f);
  } else {         // pass 2: the composed carry; pass 1: zero
    for (int i = tid; i < SW; i += nthr) U[i] = readout ? slot_in[i] : make_float2(0.f, 0.f);
  }
  if (a.W && a.w_smem && readout) {
    const float2* Wg = reinterpret_cast<const float2*>(a.W) + static_cast<long long>(h) * M * M;
    for (int i = tid; i < M * M; i += nthr) Ws[i] = Wg[i];
  }
  __syncthreads();

  const T* qb = q + bh * N * DX;
  const T* kb = k + bh * N * DX;
  const T* vb = v + bh * N * DV;
  // A step per token: this thread's mode's A (tid < M), and lambda_t, b_t in
  // fp32 in the decode step's form (lambda - 1 = expm1(x) cos(y) - 2 sin^2(y/2)
  // + i e^x sin(y), so that b keeps its relative accuracy at small Delta_t).
  float m_ar = -0.5f, m_ai = 0.f;
  if (a.delta_t && tid < M) {
    m_ar = a.A ? a.A[2 * tid] : -0.5f;
    m_ai = a.A ? a.A[2 * tid + 1] : 3.14159265358979323846f * static_cast<float>(tid);
  }
  auto step_params = [&](float dt) {
    const float x = dt * m_ar, y = dt * m_ai;
    float sy, cy, sh, ch;
    sincosf(y, &sy, &cy);
    sincosf(0.5f * y, &sh, &ch);
    const float ex = expf(x), em1 = expm1f(x);
    const float nr = fmaf(em1, cy, -2.f * sh * sh), ni = ex * sy;
    const float dd = fmaf(m_ar, m_ar, m_ai * m_ai);
    lam[tid] = make_float2(ex * cy, ex * sy);
    bb[tid] = make_float2(fmaf(nr, m_ar, ni * m_ai) / dd, fmaf(ni, m_ar, -nr * m_ai) / dd);
  };
  // The next token's inputs are loaded while this one is processed: each
  // thread holds entries f = tid and tid + 256 of k|v and of q.
  constexpr int kPre = 2;
  const bool pre = D <= kPre * nthr && DX <= kPre * nthr;
  float rz[kPre] = {0.f, 0.f}, rq[kPre] = {0.f, 0.f}, rdt = 0.f;
  auto fetch = [&](int tt) {
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
      const int f = tid + i * nthr;
      if (f < DX) {
        rz[i] = ldf(kb + static_cast<long long>(tt) * DX + f);
        rq[i] = ldf(qb + static_cast<long long>(tt) * DX + f);
      } else if (f < D) {
        rz[i] = ldf(vb + static_cast<long long>(tt) * DV + (f - DX));
      }
    }
    if (a.delta_t && tid < M) rdt = a.delta_t[bh * N + tt];
  };
  double dt_sum = 0.0;   // pass 1, thread 0: the segment's sum of delta_t
  if (pre && step1 > step0) fetch(a.reverse ? N - 1 - step0 : step0);
  for (int step = step0; step < step1; ++step) {
    const int t = a.reverse ? N - 1 - step : step;
    // the SSM input z = (xi(k_t), v_t) and the query features
    float ss = 0.f;
    if (pre) {
#pragma unroll
      for (int i = 0; i < kPre; ++i) {
        const int f = tid + i * nthr;
        if (f < D) {
          const float x = f < DX ? feat_acc(rz[i]) : rz[i];
          z[f] = x;
          ss = fmaf(x, x, ss);
        }
        if (f < DX) fq[f] = feat_acc(rq[i]);
      }
      if (a.delta_t && tid < M) step_params(rdt);
      if (a.delta_t && tid == 0) dt_sum += rdt;
      if (step + 1 < step1) fetch(a.reverse ? N - 2 - step : step + 1);
    } else {
      for (int f = tid; f < D; f += nthr) {
        const float x = f < DX ? feat_acc(ldf(kb + static_cast<long long>(t) * DX + f))
                               : ldf(vb + static_cast<long long>(t) * DV + (f - DX));
        z[f] = x;
        ss = fmaf(x, x, ss);
      }
      for (int f = tid; f < DX; f += nthr) fq[f] = feat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
      if (a.delta_t && tid < M) step_params(a.delta_t[bh * N + t]);
      if (a.delta_t && tid == 0) dt_sum += a.delta_t[bh * N + t];
    }
    if (a.delta_t && M > nthr) {   // modes past the block's threads
      const float dt = a.delta_t[bh * N + t];
      for (int m = tid + nthr; m < M; m += nthr) {
        const ModeD md = mode_consts(dt, a.A, m);
        lam[m] = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
        bb[m] = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
      }
    }
    if (norm) {   // RMSNorm over the d_xi + d_v entries, then gain and bias
      ss = warp_sum(ss);
      if (lane == 0) red[warp] = ss;
      __syncthreads();
      float tot = 0.f;
      for (int w = 0; w < nwarp; ++w) tot += red[w];
      const float r = rsqrtf(tot / static_cast<float>(D) + a.eps);
      for (int f = tid; f < D; f += nthr) {
        const float g = a.gain ? a.gain[static_cast<long long>(h) * D + f] : 1.f;
        const float c = a.bias ? a.bias[static_cast<long long>(h) * D + f] : 0.f;
        z[f] = fmaf(z[f] * r, g, c);
      }
    }
    __syncthreads();
    // state update and a = U xi(q): four modes per warp at a time, their
    // eight warp sums reduced together
    constexpr int MB = 4;
    for (int mb = warp * MB; mb < M; mb += nwarp * MB) {
      float pr[MB], pi[MB];
      float2 L[MB], Bm[MB];
#pragma unroll
      for (int u = 0; u < MB; ++u) {
        pr[u] = pi[u] = 0.f;
        const int m = min(mb + u, M - 1);   // a mode past M repeats the last one and is not stored
        L[u] = lam[m];
        Bm[u] = bb[m];
      }
      const int nu = min(MB, M - mb);
      // each column's z and xi(q) are read once for the warp's modes
      for (int f = lane; f < DX; f += 32) {
        const float zf = z[f], qf = fq[f];
#pragma unroll
        for (int u = 0; u < MB; ++u) {
          if (u >= nu) break;
          float2* up = U + (mb + u) * DX + f;
          const float2 uu = cfma(L[u], *up, make_float2(Bm[u].x * zf, Bm[u].y * zf));
          *up = uu;
          if (readout) {
            pr[u] = fmaf(uu.x, qf, pr[u]);
            pi[u] = fmaf(uu.y, qf, pi[u]);
          }
        }
      }
      for (int f = lane; f < DV; f += 32) {
        const float zv = z[DX + f];
#pragma unroll
        for (int u = 0; u < MB; ++u) {
          if (u >= nu) break;
          float2* gp = G + (mb + u) * DV + f;
          *gp = cfma(L[u], *gp, make_float2(Bm[u].x * zv, Bm[u].y * zv));
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < MB; ++u) {
          pr[u] += __shfl_xor_sync(0xffffffffu, pr[u], off);
          pi[u] += __shfl_xor_sync(0xffffffffu, pi[u], off);
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int u = 0; u < MB; ++u) {
          const int m = mb + u;
          if (m < M) {
            av[m] = make_float2(pr[u], pi[u]);
            eta[m] = cfma(L[u], eta[m], Bm[u]);
          }
        }
      }
    }
    __syncthreads();
    if (!readout) continue;   // pass 1: the state only (uniform over the block)
    // readout matrix: a~ = W_h a (row m of W dotted with a), four rows per
    // warp at a time
    if (a.W) {
      const float2* Wh = a.w_smem ? Ws : reinterpret_cast<const float2*>(a.W) + static_cast<long long>(h) * M * M;
      for (int mb = warp * MB; mb < M; mb += nwarp * MB) {
        float sr[MB], si[MB];
#pragma unroll
        for (int u = 0; u < MB; ++u) {
          sr[u] = si[u] = 0.f;
          const int m = mb + u;
          if (m >= M) continue;
          for (int mp = lane; mp < M; mp += 32) {
            const float2 w = Wh[static_cast<long long>(m) * M + mp], x = av[mp];
            sr[u] = fmaf(w.x, x.x, fmaf(-w.y, x.y, sr[u]));
            si[u] = fmaf(w.x, x.y, fmaf(w.y, x.x, si[u]));
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
          for (int u = 0; u < MB; ++u) {
            sr[u] += __shfl_xor_sync(0xffffffffu, sr[u], off);
            si[u] += __shfl_xor_sync(0xffffffffu, si[u], off);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int u = 0; u < MB; ++u)
            if (mb + u < M) at[mb + u] = make_float2(sr[u], si[u]);
        }
      }
      __syncthreads();
    }
    // num and den: P threads per value column, each summing every P-th mode
    // (four interleaved partial sums), then a shuffle sum over the P lanes
    const float2* rd = a.W ? at : av;
    int P = 1;
    while (P < 8 && 2 * P * DV <= nthr) P *= 2;
    const int part = tid % P, S = nthr / P;
    const long long row = bh * N + t;
    const int rounds = (DV + S - 1) / S;   // the same for every thread: the shuffles below see whole warps
    for (int rr = 0; rr < rounds; ++rr) {
      const int f0 = rr * S + tid / P;
      const int f = f0 < DV ? f0 : DV - 1;
      float n0 = 0.f, n1 = 0.f, e0 = 0.f, e1 = 0.f;
      int m = part;
      for (; m + P < M; m += 2 * P) {
        n0 += re_conj_mul(rd[m], G[m * DV + f]);
        e0 += re_conj_mul(rd[m], eta[m]);
        n1 += re_conj_mul(rd[m + P], G[(m + P) * DV + f]);
        e1 += re_conj_mul(rd[m + P], eta[m + P]);
      }
      if (m < M) {
        n0 += re_conj_mul(rd[m], G[m * DV + f]);
        e0 += re_conj_mul(rd[m], eta[m]);
      }
      float nf = n0 + n1, dn = e0 + e1;
      for (int off = 1; off < P; off <<= 1) {
        nf += __shfl_xor_sync(0xffffffffu, nf, off);
        dn += __shfl_xor_sync(0xffffffffu, dn, off);
      }
      if (part == 0 && f0 < DV) {
        const float of = nf / dn;
        a.o[row * DV + f] = a.accumulate ? a.o[row * DV + f] + of : of;
        if (a.num) a.num[row * DV + f] = nf;
        if (a.den && f == 0) a.den[row] = dn;
      }
    }
    __syncthreads();
  }
  if (!readout) {   // pass 1: this segment's end state into its slot
    float2* slot = a.seg + (bh * (a.nseg - 1) + sg) * SW;
    for (int i = tid; i < SW; i += nthr) slot[i] = U[i];
    if (tid == 0 && a.dsum) a.dsum[bh * a.nseg + sg] = dt_sum;
  } else if (a.state_out && sg == a.nseg - 1) {
    for (int i = tid; i < M * DX; i += nthr) a.state_out[u0 + i] = U[i];
    for (int i = tid; i < M * DV; i += nthr) a.state_out[g0 + i] = G[i];
    for (int i = tid; i < M; i += nthr) a.state_out[e0 + i] = eta[i];
  }
}

// Register-resident form for d_xi = d_v = M = 64 (the same arithmetic, the
// same segments and passes): 16 warps, warp w owning modes 4w .. 4w+3 and
// lane l the state columns 2l, 2l+1 of U and Gamma in registers (every lane
// keeps its warp's four eta), so that the state does not pass through shared
// memory every token.  Warps 0-3 stage the token's z and xi(q), warps 4-5 its
// lambda_t, b_t, in shared memory, double-buffered by token parity, and so are
// a and the warps' partial num and den: one block barrier per token orders
// the update, warps 14-15 sum the previous token's partials right after it,
// and with W a token's readout (which needs every warp's a) is formed after
// the next token's barrier, from its a and the state before that update.
constexpr int kRegWarps = 16, kRegModes = 4, kRegD = 64, kRegM = 64;

bool ex_reg_form(const ia_shape_t& s) { return s.d_xi == kRegD && s.d_v == kRegD && s.M == kRegM; }

template <typename T>
__global__ void __launch_bounds__(kRegWarps * 32, 1) seq_ex_reg_kernel(int H, int N, const T* __restrict__ q,
                                                                        const T* __restrict__ k,
                                                                        const T* __restrict__ v, const ExArgs a,
                                                                        long long BH) {
  constexpr int DX = kRegD, DV = kRegD, M = kRegM, D = DX + DV;
  __shared__ __align__(16) float zs[2][D];     // xi(k) | v, normalised when asked
  __shared__ __align__(16) float qs[2][DX];    // xi(q)
  __shared__ float2 lamS[2][M], bS[2][M];
  __shared__ float2 aS[2][M];                  // a, for the readout matrix
  __shared__ __align__(16) float part[2][kRegWarps][DV];
  __shared__ float dpart[2][kRegWarps];
  __shared__ float red[4];
  extern __shared__ float4 wsm[];              // W_h [M*M] (float2), when given and reading out
  float2* Ws = reinterpret_cast<float2*>(wsm);

  const long long bh = blockIdx.x / a.nseg;
  const int sg = static_cast<int>(blockIdx.x - bh * a.nseg);
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int step0 = sg * a.seg_len, step1 = min(N, step0 + a.seg_len);
  const bool readout = a.pass != 1;
  if (!readout && sg == a.nseg - 1) return;   // pass 1: the last segment's end state is not needed
  constexpr int SW = M * (DX + DV + 1);
  const int m0 = warp * kRegModes, f0 = 2 * lane;
  const bool norm = a.gain || a.bias;

  // this thread's state entries: (public layout for segment 0, else the slot)
  float2 U[kRegModes][2], G[kRegModes][2], E[kRegModes];
  {
    const float2* su = nullptr;
    const float2* sgm = nullptr;
    const float2* se = nullptr;
    if (sg == 0 && a.state_in) {
      su = a.state_in + bh * M * DX;
      sgm = a.state_in + BH * M * DX + bh * M * DV;
      se = a.state_in + BH * M * (DX + DV) + bh * M;
    } else if (sg > 0 && readout) {
      const float2* slot = a.seg + (bh * (a.nseg - 1) + (sg - 1)) * SW;
      su = slot;
      sgm = slot + M * DX;
      se = slot + M * (DX + DV);
    }
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const int m = m0 + u;
      float4 x = su ? *reinterpret_cast<const float4*>(su + m * DX + f0) : make_float4(0.f, 0.f, 0.f, 0.f);
      U[u][0] = make_float2(x.x, x.y);
      U[u][1] = make_float2(x.z, x.w);
      x = sgm ? *reinterpret_cast<const float4*>(sgm + m * DV + f0) : make_float4(0.f, 0.f, 0.f, 0.f);
      G[u][0] = make_float2(x.x, x.y);
      G[u][1] = make_float2(x.z, x.w);
      E[u] = se ? se[m] : make_float2(0.f, 0.f);
    }
  }
  if (a.W && readout) {
    const float2* Wg = reinterpret_cast<const float2*>(a.W) + static_cast<long long>(h) * M * M;
    for (int i = tid; i < M * M; i += kRegWarps * 32) Ws[i] = Wg[i];
  }
  // warps 4-5 (mode pm = tid - 128): its A; lambda, b once for a constant step
  constexpr int kParamT0 = 4 * 32, kSumT0 = kRegWarps * 32 - DV;
  const int pm = tid - kParamT0;
  const bool param_thread = pm >= 0 && pm < M;
  float m_ar = -0.5f, m_ai = 0.f;
  if (param_thread) {
    m_ar = a.A ? a.A[2 * pm] : -0.5f;
    m_ai = a.A ? a.A[2 * pm + 1] : 3.14159265358979323846f * static_cast<float>(pm);
    if (!a.delta_t) {
      const ModeD md = mode_consts(delta_hm(a.delta, a.dpm, M, h, pm), a.A, pm);
      const float2 l = make_float2(static_cast<float>(md.lr), static_cast<float>(md.li));
      const float2 b = make_float2(static_cast<float>(md.br), static_cast<float>(md.bi));
      lamS[0][pm] = lamS[1][pm] = l;
      bS[0][pm] = bS[1][pm] = b;
    }
  }
  const T* qb = q + bh * N * DX;
  const T* kb = k + bh * N * DX;
  const T* vb = v + bh * N * DV;
  // the next token's inputs, loaded while this one is processed
  float rz = 0.f, rq = 0.f, rdt = 0.f;
  auto fetch = [&](int tt) {
    if (tid < DX) {
      rz = ldf(kb + static_cast<long long>(tt) * DX + tid);
      rq = ldf(qb + static_cast<long long>(tt) * DX + tid);
    } else if (tid < D) {
      rz = ldf(vb + static_cast<long long>(tt) * DV + (tid - DX));
    }
    if (a.delta_t && param_thread) rdt = a.delta_t[bh * N + tt];
  };
  // warps 14-15: column f of num, den and o of token tt from the partials in
  // buffer pp (written before the block barrier that precedes this call)
  auto finish = [&](int pp, int tt) {
    const int f = tid - kSumT0;
    float nf = 0.f, d = 0.f;
#pragma unroll
    for (int w = 0; w < kRegWarps; ++w) {
      nf += part[pp][w][f];
      d += dpart[pp][w];
    }
    const long long row = bh * N + tt;
    const float of = nf / d;
    a.o[row * DV + f] = a.accumulate ? a.o[row * DV + f] + of : of;
    if (a.num) a.num[row * DV + f] = nf;
    if (a.den && f == 0) a.den[row] = d;
  };
  // W: this warp's rows of a~ = W_h a from buffer pp, then its partial num
  // and den with the current state, into the partial buffer pp
  auto w_partials = [&](int pp) {
    const float2 a0 = aS[pp][f0], a1 = aS[pp][f0 + 1];
    float sr[kRegModes], si[kRegModes];
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const float4 w = *reinterpret_cast<const float4*>(Ws + (m0 + u) * M + f0);   // W[m][2l], W[m][2l+1]
      sr[u] = fmaf(w.x, a0.x, fmaf(-w.y, a0.y, fmaf(w.z, a1.x, -w.w * a1.y)));
      si[u] = fmaf(w.x, a0.y, fmaf(w.y, a0.x, fmaf(w.z, a1.y, w.w * a1.x)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < kRegModes; ++u) {
        sr[u] += __shfl_xor_sync(0xffffffffu, sr[u], off);
        si[u] += __shfl_xor_sync(0xffffffffu, si[u], off);
      }
    }
    float n0 = 0.f, n1 = 0.f, dn = 0.f;
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const float2 at = make_float2(sr[u], si[u]);
      n0 += re_conj_mul(at, G[u][0]);
      n1 += re_conj_mul(at, G[u][1]);
      dn += re_conj_mul(at, E[u]);
    }
    *reinterpret_cast<float2*>(&part[pp][warp][f0]) = make_float2(n0, n1);
    if (lane == 0) dpart[pp][warp] = dn;
  };
  double dt_sum = 0.0;
  int prev_t = -1, prev_p = 0;   // the token whose partials are written, not yet summed
  int wpend_t = -1, wpend_p = 0;  // W: the token whose a is staged, its readout not yet formed
  if (step1 > step0) fetch(a.reverse ? N - 1 - step0 : step0);
  for (int step = step0; step < step1; ++step) {
    const int t = a.reverse ? N - 1 - step : step;
    const int p = (step - step0) & 1;
    if (tid < D) {   // warps 0-3: z_t and xi(q_t)
      float x = tid < DX ? feat_acc(rz) : rz;
      if (norm) {
        const float ss = warp_sum(x * x);
        if (lane == 0) red[warp] = ss;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const float r = rsqrtf((red[0] + red[1] + red[2] + red[3]) / static_cast<float>(D) + a.eps);
        const float g = a.gain ? a.gain[static_cast<long long>(h) * D + tid] : 1.f;
        const float c = a.bias ? a.bias[static_cast<long long>(h) * D + tid] : 0.f;
        x = fmaf(x * r, g, c);
      }
      zs[p][tid] = x;
      if (tid < DX) qs[p][tid] = feat_acc(rq);
    }
    if (a.delta_t && param_thread) {   // lambda_t, b_t as in the decode step (b through expm1)
      const float x = rdt * m_ar, y = rdt * m_ai;
      float sy, cy, sh, ch;
      sincosf(y, &sy, &cy);
      sincosf(0.5f * y, &sh, &ch);
      const float ex = expf(x), em1 = expm1f(x);
      const float nr = fmaf(em1, cy, -2.f * sh * sh), ni = ex * sy;
      const float dd = fmaf(m_ar, m_ar, m_ai * m_ai);
      lamS[p][pm] = make_float2(ex * cy, ex * sy);
      bS[p][pm] = make_float2(fmaf(nr, m_ar, ni * m_ai) / dd, fmaf(ni, m_ar, -nr * m_ai) / dd);
      if (pm == 0) dt_sum += rdt;
    }
    if (step + 1 < step1) fetch(a.reverse ? N - 2 - step : step + 1);
    __syncthreads();
    if (prev_t >= 0 && tid >= kSumT0) finish(prev_p, prev_t);
    if (wpend_t >= 0) {   // W: the previous token's readout, with the state before this update
      w_partials(wpend_p);
      prev_t = wpend_t;
      prev_p = wpend_p;
      wpend_t = -1;
    }
    // the update, and this lane's part of a = U xi(q) for the warp's modes
    const float2 zk = *reinterpret_cast<const float2*>(&zs[p][f0]);
    const float2 zv = *reinterpret_cast<const float2*>(&zs[p][DX + f0]);
    const float2 zq = *reinterpret_cast<const float2*>(&qs[p][f0]);
    float ar[kRegModes], ai[kRegModes];
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const float2 L = lamS[p][m0 + u], B = bS[p][m0 + u];
      U[u][0] = cfma(L, U[u][0], make_float2(B.x * zk.x, B.y * zk.x));
      U[u][1] = cfma(L, U[u][1], make_float2(B.x * zk.y, B.y * zk.y));
      G[u][0] = cfma(L, G[u][0], make_float2(B.x * zv.x, B.y * zv.x));
      G[u][1] = cfma(L, G[u][1], make_float2(B.x * zv.y, B.y * zv.y));
      E[u] = cfma(L, E[u], B);
      ar[u] = fmaf(U[u][0].x, zq.x, U[u][1].x * zq.y);
      ai[u] = fmaf(U[u][0].y, zq.x, U[u][1].y * zq.y);
    }
    if (!readout) continue;   // pass 1: the state only (uniform over the block)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < kRegModes; ++u) {
        ar[u] += __shfl_xor_sync(0xffffffffu, ar[u], off);
        ai[u] += __shfl_xor_sync(0xffffffffu, ai[u], off);
      }
    }
    if (a.W) {   // a~ = W_h a needs every warp's a: staged, formed after the next barrier
      if (lane == 0) {
#pragma unroll
        for (int u = 0; u < kRegModes; ++u) aS[p][m0 + u] = make_float2(ar[u], ai[u]);
      }
      wpend_t = t;
      wpend_p = p;
      continue;
    }
    // this lane's two columns of num over the warp's modes, and den
    float n0 = 0.f, n1 = 0.f, dn = 0.f;
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const float2 at = make_float2(ar[u], ai[u]);
      n0 += re_conj_mul(at, G[u][0]);
      n1 += re_conj_mul(at, G[u][1]);
      dn += re_conj_mul(at, E[u]);
    }
    *reinterpret_cast<float2*>(&part[p][warp][f0]) = make_float2(n0, n1);
    if (lane == 0) dpart[p][warp] = dn;
    prev_t = t;
    prev_p = p;
  }
  if (prev_t >= 0 || wpend_t >= 0) {   // the pending sums (uniform: readout and a non-empty range)
    __syncthreads();
    if (prev_t >= 0 && tid >= kSumT0) finish(prev_p, prev_t);
    if (wpend_t >= 0) {   // the last token's readout with W (the other partial buffer)
      w_partials(wpend_p);
      __syncthreads();
      if (tid >= kSumT0) finish(wpend_p, wpend_t);
    }
  }
  // end state: pass 1 into this segment's slot, else the last segment's state_out
  float2* du = nullptr;
  float2* dg = nullptr;
  float2* de = nullptr;
  if (!readout) {
    float2* slot = a.seg + (bh * (a.nseg - 1) + sg) * SW;
    du = slot;
    dg = slot + M * DX;
    de = slot + M * (DX + DV);
    if (pm == 0 && a.dsum) a.dsum[bh * a.nseg + sg] = dt_sum;
  } else if (a.state_out && sg == a.nseg - 1) {
    du = a.state_out + bh * M * DX;
    dg = a.state_out + BH * M * DX + bh * M * DV;
    de = a.state_out + BH * M * (DX + DV) + bh * M;
  }
  if (du) {
#pragma unroll
    for (int u = 0; u < kRegModes; ++u) {
      const int m = m0 + u;
      *reinterpret_cast<float4*>(du + m * DX + f0) = make_float4(U[u][0].x, U[u][0].y, U[u][1].x, U[u][1].y);
      *reinterpret_cast<float4*>(dg + m * DV + f0) = make_float4(G[u][0].x, G[u][0].y, G[u][1].x, G[u][1].y);
      if (lane == 0) de[m] = E[u];
    }
  }
}

// Turns the pass-1 end states into the states entering each segment, per
// (b,h) and mode: slot 0 already is the state entering segment 1 (segment 0
// started from state_in); slot s (s >= 1) becomes Lambda_s slot(s-1) +
// slot s, Lambda_s the decay over segment s, exp(A_m D_s) with D_s its sum of
// steps (delta_t summed in pass 1, or Delta_hm times its length), in fp64.
__global__ void __launch_bounds__(128) ex_carry_kernel(int H, int N, int DX, int DV, int M, const float* delta,
                                                       int dpm, const float* A, const double* dsum, int nseg,
                                                       int seg_len, float2* seg) {
  extern __shared__ double2 lamS[];   // [nseg]
  const long long bh = blockIdx.x / M;
  const int m = static_cast<int>(blockIdx.x - bh * M);
  const int h = static_cast<int>(bh % H);
  const double ar = A ? A[2 * m] : -0.5;
  const double ai = A ? A[2 * m + 1] : 3.14159265358979323846 * m;
  for (int sgi = threadIdx.x + 1; sgi < nseg - 1; sgi += blockDim.x) {
    const int len = min(N, (sgi + 1) * seg_len) - sgi * seg_len;
    const double D = dsum ? dsum[bh * nseg + sgi] : static_cast<double>(delta_hm(delta, dpm, M, h, m)) * len;
    const double e = exp(D * ar);
    double sn, cs;
    sincos(fmod(D * ai, 6.283185307179586476925), &sn, &cs);
    lamS[sgi] = make_double2(e * cs, e * sn);
  }
  __syncthreads();
  const int SW = M * (DX + DV + 1);
  float2* base = seg + bh * (nseg - 1) * SW;
  auto walk = [&](int e) {   // one state entry through the segments
    double cr = base[e].x, ci = base[e].y;
    for (int sgi = 1; sgi < nseg - 1; ++sgi) {
      const double2 L = lamS[sgi];
      const float2 loc = base[sgi * SW + e];
      const double nr = L.x * cr - L.y * ci + loc.x;
      ci = L.x * ci + L.y * cr + loc.y;
      cr = nr;
      base[sgi * SW + e] = make_float2(static_cast<float>(cr), static_cast<float>(ci));
    }
  };
  for (int f = threadIdx.x; f < DX; f += blockDim.x) walk(m * DX + f);
  for (int f = threadIdx.x; f < DV; f += blockDim.x) walk(M * DX + m * DV + f);
  if (threadIdx.x == 0) walk(M * (DX + DV) + m);
}

constexpr int kExThreads = 256;

// dynamic shared memory of one launch: W_h is staged when it fits and the
// launch reads out (pass 1 keeps the state only)
size_t ex_launch_smem(const ia_shape_t& s, bool with_w, bool* w_smem) {
  size_t smem = ex_smem(s.d_xi, s.d_v, s.M);
  *w_smem = with_w && smem + 16 + ex_smem_w(s.M) <= 232448;
  return *w_smem ? smem + 16 + ex_smem_w(s.M) : smem;
}

template <typename T>
cudaError_t launch_ex(const ia_shape_t& s, int N, const void* q, const void* k, const void* v, const ExArgs& a,
                      cudaStream_t st) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  if (ex_reg_form(s)) {
    const size_t wsm = a.W && a.pass != 1 ? sizeof(float2) * kRegM * kRegM : 0;
    auto kern = seq_ex_reg_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(wsm));
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(BH * a.nseg), kRegWarps * 32, wsm, st>>>(
        s.H, N, static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), a, BH);
    return cudaGetLastError();
  }
  ExArgs args = a;
  bool ws = false;
  const size_t smem = ex_launch_smem(s, a.W && a.pass != 1, &ws);
  args.w_smem = ws ? 1 : 0;
  auto kern = seq_fwd_ex_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(BH * args.nseg), kExThreads, smem, st>>>(
      s.H, N, s.d_xi, s.d_v, s.M, static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), args,
      BH);
  return cudaGetLastError();
}

cudaError_t launch_ex_any(const ia_shape_t& s, int N, const void* q, const void* k, const void* v,
                          const ExArgs& a, cudaStream_t st) {
  if (s.in_dtype == IA_F32) return launch_ex<float>(s, N, q, k, v, a, st);
  return launch_ex<__nv_bfloat16>(s, N, q, k, v, a, st);
}

// CTAs of the reading-out launch resident per SM (1 when no device answers)
int ex_resident(const ia_shape_t& s, bool with_w) {
  if (ex_reg_form(s)) return 1;   // 512 threads of up to 128 registers
  bool ws = false;
  const size_t smem = ex_launch_smem(s, with_w, &ws);
  const void* fn = s.in_dtype == IA_F32 ? reinterpret_cast<const void*>(seq_fwd_ex_kernel<float>)
                                        : reinterpret_cast<const void*>(seq_fwd_ex_kernel<__nv_bfloat16>);
  int n = 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kExThreads, smem) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 1;
  }
  return n;
}

// Segments per sequence of the token-serial form: enough that the grid of
// B H nseg CTAs fills the SMs' resident slots once, each segment at least
// kMinSegment tokens, at most kMaxSegments (the carry walks them in turn).
constexpr int kMinSegment = 64, kMaxSegments = 64;

int ex_segments(const ia_shape_t& s, const ia_options_t* opt) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  const long long by_len = std::min<long long>(s.N / kMinSegment, kMaxSegments);
  if (by_len < 2) return 1;
  const long long slots = static_cast<long long>(num_sms()) * ex_resident(s, opt && opt->W);
  return static_cast<int>(std::max<long long>(1, std::min(by_len, slots / BH)));
}

// workspace of nseg segments: the end-state slots, then the delta_t sums, with
// 16 bytes of slack to align the caller's pointer
size_t ex_seg_bytes(const ia_shape_t& s, const ia_options_t* opt, int nseg) {
  if (nseg <= 1) return 0;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t SW = static_cast<size_t>(s.M) * (s.d_xi + s.d_v + 1);
  return 16 + BH * (nseg - 1) * SW * sizeof(float2) + (opt && opt->delta_t ? BH * nseg * sizeof(double) : 0);
}

// the planned count, lowered until the caller's workspace holds it
int ex_fit_segments(const ia_shape_t& s, const ia_options_t* opt, const void* workspace, size_t workspace_bytes) {
  int nseg = ex_segments(s, opt);
  while (nseg > 1 && (!workspace || ex_seg_bytes(s, opt, nseg) > workspace_bytes)) --nseg;
  return nseg;
}

cudaError_t launch_ex_carry(const ia_shape_t& s, const ExArgs& a, cudaStream_t st) {
  const long long rows = static_cast<long long>(s.B) * s.H * s.M;
  ex_carry_kernel<<<static_cast<unsigned>(rows), 128, sizeof(double2) * a.nseg, st>>>(
      s.H, s.N, s.d_xi, s.d_v, s.M, a.delta, a.dpm, a.A, a.dsum, a.nseg, a.seg_len, a.seg);
  return cudaGetLastError();
}

// one direction of the token-serial form: a single pass, or pass 1, the carry
// and pass 2 over the segments
cudaError_t run_ex_direction(const ia_shape_t& s, const void* q, const void* k, const void* v, ExArgs a,
                             cudaStream_t st) {
  if (a.nseg <= 1) {
    a.pass = 0;
    return launch_ex_any(s, s.N, q, k, v, a, st);
  }
  a.pass = 1;
  cudaError_t e = launch_ex_any(s, s.N, q, k, v, a, st);
  if (e == cudaSuccess && a.nseg > 2) e = launch_ex_carry(s, a, st);
  if (e != cudaSuccess) return e;
  a.pass = 2;
  return launch_ex_any(s, s.N, q, k, v, a, st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kMaxSmem = 232448;

ExArgs make_args(const ia_shape_t* s, const ia_options_t* opt, const float* delta, const float* A) {
  ExArgs a = {};
  a.nseg = 1;
  a.seg_len = 1 << 30;
  a.delta = delta;
  a.dpm = s->delta_per_mode;
  a.A = A;
  if (opt) {
    a.delta_t = opt->delta_t;
    a.gain = opt->gain;
    a.bias = opt->bias;
    a.eps = opt->eps;
    a.W = opt->W;
  }
  return a;
}

// The tensor-core form (ia_layer_tc.cu) serves bf16 shapes of the chunk pass
// without a per-token step (the input stabilisation, the bidirectional layer
// and, at d_xi = 64, the readout matrix); IA_PREFILL_SIMT forces the
// token-serial kernel, as for the plain layer.
bool ex_use_tc(const ia_shape_t& s, const ia_options_t* opt) {
  const char* env = std::getenv("IA_PREFILL_SIMT");
  if (env && env[0] && std::strcmp(env, "0") != 0) return false;
  return ex_tc_supported(s, opt);
}

bool valid_options(const ia_options_t* opt) {
  if (!opt) return true;
  const void* ptrs[] = {opt->delta_t, opt->gain, opt->bias, opt->W};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return false;
  if ((opt->gain || opt->bias) && !(opt->eps >= 0.f)) return false;
  return opt->bidirectional == 0 || opt->bidirectional == 1;
}

}  // namespace
}  // namespace ia

using namespace ia;

extern "C" {

IA_API size_t ia_prefill_ex_workspace_bytes(const ia_shape_t* s, const ia_options_t* opt) {
  if (!valid_dims(s, true) || !valid_options(opt)) return 0;
  if (!ex_use_tc(*s, opt)) return ex_seg_bytes(*s, opt, ex_segments(*s, opt));
  return ex_tc_workspace_bytes(*s, opt, tc_plan(*s, num_sms()));
}

IA_API int ia_prefill_ex_segments(const ia_shape_t* s, const ia_options_t* opt, const void* workspace,
                                  size_t workspace_bytes) {
  if (!valid_dims(s, true) || !valid_options(opt)) return 0;
  if (ex_use_tc(*s, opt)) return 1;
  return ex_fit_segments(*s, opt, workspace, workspace_bytes);
}

IA_API int ia_prefill_ex_path(const ia_shape_t* s, const ia_options_t* opt) {
  if (!valid_dims(s, true) || !valid_options(opt)) return IA_PATH_NONE;
  return ex_use_tc(*s, opt) ? IA_PATH_TENSOR_CORE : IA_PATH_SEQUENTIAL;
}

IA_API ia_status_t ia_prefill_fwd_ex(const ia_shape_t* s, const ia_options_t* opt, const void* q,
                                     const void* k, const void* v, const float* delta, const float* A,
                                     const void* state_in, float* o, float* num, float* den,
                                     void* state_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dims(s, true) || !valid_options(opt)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || (!delta && !(opt && opt->delta_t))) return IA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, delta, A, state_in, o, num, den, state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (state_in && state_in == state_out) return IA_ERR_INVALID_ARG;
  const bool bidir = opt && opt->bidirectional;
  // the two directions of the bidirectional layer have no single state, and
  // their num / den do not combine into o
  if (bidir && (state_in || state_out || num || den)) return IA_ERR_INVALID_ARG;
  const bool tc = ex_use_tc(*s, opt);
  if (!tc && ex_smem(s->d_xi, s->d_v, s->M) > kMaxSmem) return IA_ERR_UNSUPPORTED;
  TcPlan plan{1};
  if (tc) {
    plan = tc_plan(*s, num_sms());
    if (!workspace || workspace_bytes < ex_tc_workspace_bytes(*s, opt, plan)) return IA_ERR_WORKSPACE;
  }
  if (inject_launch_failure()) return IA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc) {   // the marks bracket every pass of the call
    mark_launch_begin(st);
    hold_launch_marks(true);
    const cudaError_t e = launch_ex_tc(*s, opt, plan, q, k, v, delta, A, state_in, o, num, den, state_out,
                                       workspace, st);
    hold_launch_marks(false);
    mark_launch_end(st);
    return map_cuda(e);
  }
  ExArgs a = make_args(s, opt, delta, A);
  a.state_in = static_cast<const float2*>(state_in);
  a.state_out = static_cast<float2*>(state_out);
  a.o = o;
  a.num = num;
  a.den = den;
  const int nseg = ex_fit_segments(*s, opt, workspace, workspace_bytes);
  if (nseg > 1) {
    const uintptr_t base = (reinterpret_cast<uintptr_t>(workspace) + 15) & ~static_cast<uintptr_t>(15);
    const size_t BH = static_cast<size_t>(s->B) * s->H;
    const size_t slots = BH * (nseg - 1) * s->M * (s->d_xi + s->d_v + 1) * sizeof(float2);
    a.nseg = nseg;
    a.seg_len = (s->N + nseg - 1) / nseg;
    a.seg = reinterpret_cast<float2*>(base);
    a.dsum = a.delta_t ? reinterpret_cast<double*>(base + slots) : nullptr;
  }
  mark_launch_begin(st);
  cudaError_t e = run_ex_direction(*s, q, k, v, a, st);
  if (e == cudaSuccess && bidir) {
    a.reverse = 1;
    a.accumulate = 1;
    e = run_ex_direction(*s, q, k, v, a, st);
  }
  mark_launch_end(st);
  return map_cuda(e);
}

IA_API ia_status_t ia_decode_step_ex(const ia_shape_t* s, const ia_options_t* opt, const void* q,
                                     const void* k, const void* v, const float* delta, const float* A,
                                     void* state, float* o, float* num, float* den, void* stream) {
  if (!valid_dims(s, false) || !valid_options(opt)) return IA_ERR_INVALID_ARG;
  if (!q || !k || !v || !state || !o || (!delta && !(opt && opt->delta_t))) return IA_ERR_INVALID_ARG;
  if (opt && opt->bidirectional) return IA_ERR_INVALID_ARG;   // not causal: no step-by-step form
  const void* ptrs[] = {q, k, v, delta, A, state, o, num, den};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return IA_ERR_INVALID_ARG;
  if (ex_smem(s->d_xi, s->d_v, s->M) > kMaxSmem) return IA_ERR_UNSUPPORTED;
  if (inject_launch_failure()) return IA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // one token on the state in place: each CTA reads its whole state into
  // shared memory before it writes it back
  ExArgs a = make_args(s, opt, delta, A);
  a.state_in = static_cast<const float2*>(state);
  a.state_out = static_cast<float2*>(state);
  a.o = o;
  a.num = num;
  a.den = den;
  mark_launch_begin(st);
  const cudaError_t e = launch_ex_any(*s, 1, q, k, v, a, st);
  mark_launch_end(st);
  return map_cuda(e);
}

}  // extern "C"
