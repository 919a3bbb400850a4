// Two optional parts of the layer on the tensor-core chunk pass, for bf16
// inputs and the shapes that pass runs (M = 64, d_xi and d_v in {64, 128}):
//   - input stabilisation (AI-radio page, "Implementation Details"): the SSM
//     input z_t = (xi(k_t), v_t) passes an RMSNorm with a per-head gain and
//     bias, z <- z / sqrt(mean(z^2) + eps) * gain_h + bias_h, before the
//     recurrence.  A prologue kernel writes the normalised z as the fp16
//     k and v operands, and the chunk pass takes them as they are;
//   - the bidirectional layer (summary sec. 5.2): o = f(x) + flip(f(flip x)).
//     The prologue also writes the time-reversed q (bf16) and z (fp16), a
//     second chunk pass runs the causal layer on them, and an epilogue adds
//     its output, reversed back, to the first pass's.
//   - the complex readout matrix (summary sec. A.3), d_xi = 64: a~_t = W_h a_t
//     before the readout.  wprime_kernel writes W_h as the real fp16 matrix W'
//     (ia_tables.cuh) and the chunk pass runs one more contraction per chunk,
//     G_W: a~~ = W' a, between its key-state read and its score matrix (the
//     readout factor then is a complex rotation per entry instead of a real
//     row scale).  W' and a are fp16 operands, one rounding more than the
//     plain layer's.
// The per-token step (selective writing) changes the chunk decay itself and
// stays on the token-serial kernel (ia_layer_ex.cu).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_simt_common.cuh"
#include "ia_tables.cuh"

namespace ia {
namespace {

constexpr int kPrepWarps = 8;

// One warp per token (b,h,t).  NORM: z normalised with gain and bias, written
// at t to kz, vz.  FLIP: q copied to qr at N-1-t, z (normalised if NORM) to
// kr, vr at N-1-t.
template <bool NORM, bool FLIP>
__global__ void __launch_bounds__(kPrepWarps * 32) ex_prep_kernel(
    int H, int N, int DX, int DV, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ gain, const float* __restrict__ bias, float eps,
    __half* __restrict__ kz, __half* __restrict__ vz, __nv_bfloat16* __restrict__ qr, __half* __restrict__ kr,
    __half* __restrict__ vr, long long tokens) {
  const int lane = threadIdx.x & 31;
  const long long tok = static_cast<long long>(blockIdx.x) * kPrepWarps + (threadIdx.x >> 5);
  if (tok >= tokens) return;
  const long long bh = tok / N;
  const int t = static_cast<int>(tok - bh * N);
  const int h = static_cast<int>(bh % H);
  const int D = DX + DV;
  constexpr int kMaxPerLane = 8;   // D <= 256
  float z[kMaxPerLane];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxPerLane; ++u) {
    const int f = lane + 32 * u;
    float x = 0.f;
    if (f < DX) x = simt::feat_acc(__bfloat162float(k[tok * DX + f]));
    else if (f < D) x = __bfloat162float(v[tok * DV + (f - DX)]);
    z[u] = x;
    ss = fmaf(x, x, ss);
  }
  if (NORM) {
    ss = simt::warp_sum(ss);
    const float r = rsqrtf(ss / static_cast<float>(D) + eps);
#pragma unroll
    for (int u = 0; u < kMaxPerLane; ++u) {
      const int f = lane + 32 * u;
      if (f < D) {
        const float g = gain ? gain[static_cast<long long>(h) * D + f] : 1.f;
        const float c = bias ? bias[static_cast<long long>(h) * D + f] : 0.f;
        z[u] = fmaf(z[u] * r, g, c);
      }
    }
  }
  const long long rt = bh * N + (N - 1 - t);   // the token's place in the reversed sequence
#pragma unroll
  for (int u = 0; u < kMaxPerLane; ++u) {
    const int f = lane + 32 * u;
    if (f >= D) continue;
    const __half zh = __float2half_rn(z[u]);
    if (f < DX) {
      if (NORM) kz[tok * DX + f] = zh;
      if (FLIP) {
        kr[rt * DX + f] = zh;
        qr[rt * DX + f] = q[tok * DX + f];
      }
    } else {
      if (NORM) vz[tok * DV + (f - DX)] = zh;
      if (FLIP) vr[rt * DV + (f - DX)] = zh;
    }
  }
}

// W [H][M][M] complex (re, im pairs) -> W' per head (wprime_offset layout):
// one block per (h, row k of W'), one thread per column k'.
__global__ void __launch_bounds__(2 * kModesTC) wprime_kernel(const float* __restrict__ W, __half* __restrict__ Wt) {
  const int h = blockIdx.x / (2 * kModesTC), k = blockIdx.x % (2 * kModesTC), kp = threadIdx.x;
  const int m = k >> 1, mp = kp >> 1;
  const float2 w = reinterpret_cast<const float2*>(W)[(static_cast<long long>(h) * kModesTC + m) * kModesTC + mp];
  // [re -im; im re] in the (k, k') parities
  const float x = (k & 1) == (kp & 1) ? w.x : ((k & 1) ? w.y : -w.y);
  *reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(Wt) + static_cast<size_t>(h) * kWprimeBytes +
                             wprime_offset(k, kp)) = __float2half_rn(x);
}

// o[bh][t] += orv[bh][N-1-t], four floats per thread (DV a multiple of 4)
__global__ void __launch_bounds__(256) add_reversed_kernel(int N, int DV, float* __restrict__ o,
                                                          const float* __restrict__ orv, long long n4) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const int per = DV / 4;
  const long long row = i / per;   // bh * N + t
  const int c = static_cast<int>(i - row * per);
  const long long bh = row / N;
  const int t = static_cast<int>(row - bh * N);
  const float4 a = reinterpret_cast<const float4*>(o)[i];
  const float4 b = reinterpret_cast<const float4*>(orv)[(bh * N + (N - 1 - t)) * per + c];
  reinterpret_cast<float4*>(o)[i] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

struct ExLayout {   // byte offsets inside the workspace (after the chunk pass's own)
  size_t tc, kz, vz, qr, kr, vr, orv, wt, total;
};

ExLayout ex_layout(const ia_shape_t& s, const ia_options_t& opt, const TcPlan& p) {
  const size_t tokens = static_cast<size_t>(s.B) * s.H * s.N;
  const bool norm = opt.gain || opt.bias, flip = opt.bidirectional != 0;
  ExLayout L = {};
  size_t at = round256(tc_workspace_bytes(s, p));
  L.tc = 0;
  auto take = [&](bool need, size_t bytes) -> size_t {
    if (!need) return 0;
    const size_t here = at;
    at = round256(at + bytes);
    return here;
  };
  L.kz = take(norm, tokens * s.d_xi * 2);
  L.vz = take(norm, tokens * s.d_v * 2);
  L.qr = take(flip, tokens * s.d_xi * 2);
  L.kr = take(flip, tokens * s.d_xi * 2);
  L.vr = take(flip, tokens * s.d_v * 2);
  L.orv = take(flip, tokens * s.d_v * 4);
  L.wt = take(opt.W != nullptr, static_cast<size_t>(s.H) * kWprimeBytes);
  L.total = at + 256;   // the caller's pointer may need rounding up to 256
  return L;
}

}  // namespace

bool ex_tc_supported(const ia_shape_t& s, const ia_options_t* opt) {
  if (!tc_prefill_supported(s)) return false;
  if (opt && opt->delta_t) return false;
  if (opt && opt->W && s.d_xi != 64) return false;   // W' takes the shared memory of d_xi = 128's tiles
  return s.d_xi + s.d_v <= 256;
}

size_t ex_tc_workspace_bytes(const ia_shape_t& s, const ia_options_t* opt, const TcPlan& p) {
  const ia_options_t none = {};
  return ex_layout(s, opt ? *opt : none, p).total;
}

cudaError_t launch_ex_tc(const ia_shape_t& s, const ia_options_t* opt, const TcPlan& p, const void* q,
                         const void* k, const void* v, const float* delta, const float* A,
                         const void* state_in, float* o, float* num, float* den, void* state_out, void* ws,
                         cudaStream_t st) {
  const ia_options_t none = {};
  const ia_options_t& op = opt ? *opt : none;
  const bool norm = op.gain || op.bias, flip = op.bidirectional != 0;
  const ExLayout L = ex_layout(s, op, p);
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255));
  auto at = [&](size_t off) { return base + off; };
  const long long tokens = static_cast<long long>(s.B) * s.H * s.N;
  __half* kz = reinterpret_cast<__half*>(at(L.kz));
  __half* vz = reinterpret_cast<__half*>(at(L.vz));
  __nv_bfloat16* qr = reinterpret_cast<__nv_bfloat16*>(at(L.qr));
  __half* kr = reinterpret_cast<__half*>(at(L.kr));
  __half* vr = reinterpret_cast<__half*>(at(L.vr));
  float* orv = reinterpret_cast<float*>(at(L.orv));
  __half* wt = op.W ? reinterpret_cast<__half*>(at(L.wt)) : nullptr;
  if (wt) {
    wprime_kernel<<<static_cast<unsigned>(s.H * 2 * kModesTC), 2 * kModesTC, 0, st>>>(op.W, wt);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (norm || flip) {
    const unsigned grid = static_cast<unsigned>((tokens + kPrepWarps - 1) / kPrepWarps);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    if (norm && flip)
      ex_prep_kernel<true, true><<<grid, kPrepWarps * 32, 0, st>>>(s.H, s.N, s.d_xi, s.d_v, qb, kb, vb, op.gain,
                                                                 op.bias, op.eps, kz, vz, qr, kr, vr, tokens);
    else if (norm)
      ex_prep_kernel<true, false><<<grid, kPrepWarps * 32, 0, st>>>(s.H, s.N, s.d_xi, s.d_v, qb, kb, vb, op.gain,
                                                                  op.bias, op.eps, kz, vz, qr, kr, vr, tokens);
    else
      ex_prep_kernel<false, true><<<grid, kPrepWarps * 32, 0, st>>>(s.H, s.N, s.d_xi, s.d_v, qb, kb, vb, op.gain,
                                                                  op.bias, op.eps, kz, vz, qr, kr, vr, tokens);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the causal pass over the sequence as given (z normalised when asked)
  cudaError_t e = launch_tc_prefill(s, p, q, norm ? static_cast<const void*>(kz) : k,
                                    norm ? static_cast<const void*>(vz) : v, delta, A, state_in, o, num, den,
                                    state_out, ws, st, nullptr, nullptr, nullptr, norm, wt);
  if (e != cudaSuccess || !flip) return e;
  // the causal pass over the reversed sequence, added back in forward order
  e = launch_tc_prefill(s, p, qr, kr, vr, delta, A, nullptr, orv, nullptr, nullptr, nullptr, ws, st, nullptr,
                        nullptr, nullptr, true, wt);
  if (e != cudaSuccess) return e;
  const long long n4 = tokens * s.d_v / 4;
  add_reversed_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(s.N, s.d_v, o, orv, n4);
  return cudaGetLastError();
}

}  // namespace ia
