// The layer with its optional parts, on CUDA cores in fp32 (one CTA per (b,h),
// token after token), behind ia_prefill_fwd_ex and ia_decode_step_ex.
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
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_simt_common.cuh"

namespace ia {
namespace {

// shared (float2): U [M*DX] | G [M*DV] | eta [M] | lam [M] | b [M] | a [M] | a~ [M]
// then floats: fq [DX] | z [DX + DV] | red [32]
size_t ex_smem(int DX, int DV, int M) {
  return sizeof(float2) * (static_cast<size_t>(M) * (DX + DV) + 5 * M) + sizeof(float) * (2 * DX + DV + 32) + 16;
}

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
};

template <typename T>
__global__ void __launch_bounds__(256) seq_fwd_ex_kernel(int H, int N, int DX, int DV, int M, const T* __restrict__ q,
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

  const long long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, nthr = blockDim.x;
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
  for (int i = tid; i < M * DX; i += nthr) U[i] = a.state_in ? a.state_in[u0 + i] : make_float2(0.f, 0.f);
  for (int i = tid; i < M * DV; i += nthr) G[i] = a.state_in ? a.state_in[g0 + i] : make_float2(0.f, 0.f);
  for (int i = tid; i < M; i += nthr) eta[i] = a.state_in ? a.state_in[e0 + i] : make_float2(0.f, 0.f);
  __syncthreads();

  const T* qb = q + bh * N * DX;
  const T* kb = k + bh * N * DX;
  const T* vb = v + bh * N * DV;
  for (int step = 0; step < N; ++step) {
    const int t = a.reverse ? N - 1 - step : step;
    // the SSM input z = (xi(k_t), v_t) and the query features
    float ss = 0.f;
    for (int f = tid; f < D; f += nthr) {
      const float x = f < DX ? feat_acc(ldf(kb + static_cast<long long>(t) * DX + f))
                             : ldf(vb + static_cast<long long>(t) * DV + (f - DX));
      z[f] = x;
      ss = fmaf(x, x, ss);
    }
    for (int f = tid; f < DX; f += nthr) fq[f] = feat_acc(ldf(qb + static_cast<long long>(t) * DX + f));
    if (a.delta_t) {   // this token's step for every mode
      const float dt = a.delta_t[bh * N + t];
      for (int m = tid; m < M; m += nthr) {
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
    for (int m = warp; m < M; m += nwarp) {
      const float2 L = lam[m], Bm = bb[m];
      float ar = 0.f, ai = 0.f;
      for (int f = lane; f < DX; f += 32) {
        const float2 u = cfma(L, U[m * DX + f], make_float2(Bm.x * z[f], Bm.y * z[f]));
        U[m * DX + f] = u;
        ar = fmaf(u.x, fq[f], ar);
        ai = fmaf(u.y, fq[f], ai);
      }
      for (int f = lane; f < DV; f += 32)
        G[m * DV + f] = cfma(L, G[m * DV + f], make_float2(Bm.x * z[DX + f], Bm.y * z[DX + f]));
      ar = warp_sum(ar);
      ai = warp_sum(ai);
      if (lane == 0) {
        av[m] = make_float2(ar, ai);
        eta[m] = cfma(L, eta[m], Bm);
      }
    }
    __syncthreads();
    // readout matrix: a~ = W_h a (row m of W dotted with a, one warp per row)
    if (a.W) {
      const float2* Wh = reinterpret_cast<const float2*>(a.W) + static_cast<long long>(h) * M * M;
      for (int m = warp; m < M; m += nwarp) {
        float sr = 0.f, si = 0.f;
        for (int mp = lane; mp < M; mp += 32) {
          const float2 w = Wh[static_cast<long long>(m) * M + mp], x = av[mp];
          sr = fmaf(w.x, x.x, fmaf(-w.y, x.y, sr));
          si = fmaf(w.x, x.y, fmaf(w.y, x.x, si));
        }
        sr = warp_sum(sr);
        si = warp_sum(si);
        if (lane == 0) at[m] = make_float2(sr, si);
      }
      __syncthreads();
    }
    const float2* rd = a.W ? at : av;
    float dn = 0.f;
    for (int m = 0; m < M; ++m) dn += re_conj_mul(rd[m], eta[m]);
    const long long row = bh * N + t;
    for (int f = tid; f < DV; f += nthr) {
      float nf = 0.f;
      for (int m = 0; m < M; ++m) nf += re_conj_mul(rd[m], G[m * DV + f]);
      const float of = nf / dn;
      a.o[row * DV + f] = a.accumulate ? a.o[row * DV + f] + of : of;
      if (a.num) a.num[row * DV + f] = nf;
    }
    if (a.den && tid == 0) a.den[row] = dn;
    __syncthreads();
  }
  if (a.state_out) {
    for (int i = tid; i < M * DX; i += nthr) a.state_out[u0 + i] = U[i];
    for (int i = tid; i < M * DV; i += nthr) a.state_out[g0 + i] = G[i];
    for (int i = tid; i < M; i += nthr) a.state_out[e0 + i] = eta[i];
  }
}

template <typename T>
cudaError_t launch_ex(const ia_shape_t& s, int N, const void* q, const void* k, const void* v, const ExArgs& a,
                      cudaStream_t st) {
  const size_t smem = ex_smem(s.d_xi, s.d_v, s.M);
  auto kern = seq_fwd_ex_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long BH = static_cast<long long>(s.B) * s.H;
  kern<<<static_cast<unsigned>(BH), 256, smem, st>>>(s.H, N, s.d_xi, s.d_v, s.M, static_cast<const T*>(q),
                                                     static_cast<const T*>(k), static_cast<const T*>(v), a, BH);
  return cudaGetLastError();
}

cudaError_t launch_ex_any(const ia_shape_t& s, int N, const void* q, const void* k, const void* v,
                          const ExArgs& a, cudaStream_t st) {
  if (s.in_dtype == IA_F32) return launch_ex<float>(s, N, q, k, v, a, st);
  return launch_ex<__nv_bfloat16>(s, N, q, k, v, a, st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kMaxSmem = 232448;

ExArgs make_args(const ia_shape_t* s, const ia_options_t* opt, const float* delta, const float* A) {
  ExArgs a = {};
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
// whose options are only the input stabilisation and / or the bidirectional
// layer; IA_PREFILL_SIMT forces the token-serial kernel, as for the plain layer.
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
  if (!valid_dims(s, true) || !valid_options(opt) || !ex_use_tc(*s, opt)) return 0;
  return ex_tc_workspace_bytes(*s, opt, tc_plan(*s, num_sms()));
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
  mark_launch_begin(st);
  cudaError_t e = launch_ex_any(*s, s->N, q, k, v, a, st);
  if (e == cudaSuccess && bidir) {
    a.reverse = 1;
    a.accumulate = 1;
    e = launch_ex_any(*s, s->N, q, k, v, a, st);
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
