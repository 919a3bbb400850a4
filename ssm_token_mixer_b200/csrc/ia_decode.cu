// One recurrent decode step of the IA layer (paperlayer.ai summary of
// 'Interdomain Attention', sec. 3.2: a fixed state of size O(M(R + d)) and
// constant work per generated token; sec. F.3: graphed decode whose latency
// does not depend on the prefix length).  For every (b,h):
//   U <- lambda U + b xi(k)^T,  Gamma <- lambda Gamma + b v^T,  eta <- lambda eta + b
//   a = U xi(q),  o = Re(a^H Gamma) / Re(a^H eta)
//
// The step is bound by state bytes: every state entry is read and written
// once in fp32.  A thread-block cluster serves one (b,h); each CTA of the
// cluster streams a group of modes with 16-byte loads and stores, keeps its
// partial num/den in shared memory, and the cluster's rank-0 CTA sums the
// partials over distributed shared memory and writes o.
#include <cstdlib>
#include <cooperative_groups.h>

#include "ia_device.cuh"
#include "ia_internal.h"

namespace cg = cooperative_groups;

namespace ia {
namespace {

constexpr int kDecThreads = 256;
constexpr int kVecPerLane = 4;   // rows up to 256 complex entries (d <= 256)
constexpr int kModesPerWarp = 2;  // up to 16 modes per CTA

template <typename T>
__device__ __forceinline__ float ldx(const T* p);
template <>
__device__ __forceinline__ float ldx<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float xi_acc(float x) { return x > 0.f ? x + 1.f : expf(x); }

// shared: fq [DX] | fk [DX] | vv [DV] | part [8 warps][DV] | pden [8] | lam,b [MG] float2
template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(
    int H, int DX, int DV, int M, int MG, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const float* __restrict__ delta, int dpm, const float* __restrict__ A,
    float2* __restrict__ state, float* __restrict__ o, float* __restrict__ num,
    float* __restrict__ den, long long BH) {
  extern __shared__ float4 dsm[];
  float* fq = reinterpret_cast<float*>(dsm);
  float* fk = fq + DX;
  float* vv = fk + DX;
  float* part = vv + DV;                    // [8][DV]
  float* pden = part + 8 * DV;              // [8]
  float2* lamb = reinterpret_cast<float2*>(pden + 8);   // [MG] lambda, [MG] b
  float2* bb = lamb + MG;

  cg::cluster_group cluster = cg::this_cluster();
  const int g = static_cast<int>(cluster.block_rank());
  const int G = static_cast<int>(cluster.num_blocks());
  const long long bh = blockIdx.x / G;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = g * MG;
  const int nu = DX / 2, ng = DV / 2;   // 16-byte vectors (two complex entries) per row

  float2* Ub = state + bh * M * DX;
  float2* Gb = state + BH * M * DX + bh * M * DV;
  float2* Eb = state + BH * M * (DX + DV) + bh * M;

  // Issue every state load of this warp's modes first, so that HBM latency
  // overlaps the parameter and feature set-up below.
  float4 uv[kModesPerWarp][kVecPerLane], gv[kModesPerWarp][kVecPerLane];
  float2 ev[kModesPerWarp];
#pragma unroll
  for (int r = 0; r < kModesPerWarp; ++r) {
    const int mi = warp + 8 * r, m = m0 + mi;
    const bool ok = mi < MG && m < M;
    const float4* Ur = reinterpret_cast<const float4*>(Ub + static_cast<long long>(m) * DX);
    const float4* Gr = reinterpret_cast<const float4*>(Gb + static_cast<long long>(m) * DV);
#pragma unroll
    for (int i = 0; i < kVecPerLane; ++i) {
      const int p = lane + 32 * i;
      if (ok && p < nu) uv[r][i] = Ur[p];
      if (ok && p < ng) gv[r][i] = Gr[p];
    }
    ev[r] = (ok && lane == 0) ? Eb[m] : make_float2(0.f, 0.f);
  }

  for (int f = tid; f < DX; f += kDecThreads) {
    fq[f] = xi_acc(ldx(q + bh * DX + f));
    fk[f] = xi_acc(ldx(k + bh * DX + f));
  }
  for (int f = tid; f < DV; f += kDecThreads) vv[f] = ldx(v + bh * DV + f);
  for (int i = tid; i < MG; i += kDecThreads) {
    // lambda = exp(Delta A), b = (lambda - 1)/A in fp32; lambda - 1 is formed
    // as expm1(x) cos(y) - 2 sin^2(y/2) + i e^x sin(y) so it keeps its
    // relative accuracy for small Delta.
    const int m = m0 + i;
    const float ar = A ? A[2 * m] : -0.5f;
    const float ai = A ? A[2 * m + 1] : 3.14159265358979f * static_cast<float>(m);
    const float d = delta_hm(delta, dpm, M, h, m);
    const float x = d * ar, y = d * ai;
    float sy, cy, sh, ch;
    sincosf(y, &sy, &cy);
    sincosf(0.5f * y, &sh, &ch);
    const float ex = expf(x), em1 = expm1f(x);
    const float nr = fmaf(em1, cy, -2.f * sh * sh), ni = ex * sy;   // lambda - 1
    const float dd = fmaf(ar, ar, ai * ai);
    lamb[i] = make_float2(ex * cy, ex * sy);
    bb[i] = make_float2(fmaf(nr, ar, ni * ai) / dd, fmaf(ni, ar, -nr * ai) / dd);
  }
  for (int i = tid; i < 8 * DV + 8; i += kDecThreads) part[i] = 0.f;
  __syncthreads();

  float* mypart = part + warp * DV;
  float dpart = 0.f;
#pragma unroll
  for (int r = 0; r < kModesPerWarp; ++r) {
    const int mi = warp + 8 * r, m = m0 + mi;
    if (mi >= MG || m >= M) break;
    const float2 L = lamb[mi], Bm = bb[mi];
    float4* Ur = reinterpret_cast<float4*>(Ub + static_cast<long long>(m) * DX);
    float4* Gr = reinterpret_cast<float4*>(Gb + static_cast<long long>(m) * DV);
    float ar = 0.f, ai = 0.f;
#pragma unroll
    for (int i = 0; i < kVecPerLane; ++i) {
      const int p = lane + 32 * i;
      if (p < nu) {
        const float4 u = uv[r][i];
        const float x0 = fk[2 * p], x1 = fk[2 * p + 1];
        float4 w;
        w.x = fmaf(L.x, u.x, fmaf(-L.y, u.y, Bm.x * x0));
        w.y = fmaf(L.x, u.y, fmaf(L.y, u.x, Bm.y * x0));
        w.z = fmaf(L.x, u.z, fmaf(-L.y, u.w, Bm.x * x1));
        w.w = fmaf(L.x, u.w, fmaf(L.y, u.z, Bm.y * x1));
        Ur[p] = w;
        ar = fmaf(w.x, fq[2 * p], fmaf(w.z, fq[2 * p + 1], ar));
        ai = fmaf(w.y, fq[2 * p], fmaf(w.w, fq[2 * p + 1], ai));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ar += __shfl_xor_sync(0xffffffffu, ar, off);
      ai += __shfl_xor_sync(0xffffffffu, ai, off);
    }
#pragma unroll
    for (int i = 0; i < kVecPerLane; ++i) {
      const int p = lane + 32 * i;
      if (p < ng) {
        const float4 gq = gv[r][i];
        const float x0 = vv[2 * p], x1 = vv[2 * p + 1];
        float4 w;
        w.x = fmaf(L.x, gq.x, fmaf(-L.y, gq.y, Bm.x * x0));
        w.y = fmaf(L.x, gq.y, fmaf(L.y, gq.x, Bm.y * x0));
        w.z = fmaf(L.x, gq.z, fmaf(-L.y, gq.w, Bm.x * x1));
        w.w = fmaf(L.x, gq.w, fmaf(L.y, gq.z, Bm.y * x1));
        Gr[p] = w;
        mypart[2 * p] += fmaf(ar, w.x, ai * w.y);       // Re(conj(a) Gamma)
        mypart[2 * p + 1] += fmaf(ar, w.z, ai * w.w);
      }
    }
    if (lane == 0) {
      const float2 e = ev[r];
      const float2 w = make_float2(fmaf(L.x, e.x, fmaf(-L.y, e.y, Bm.x)), fmaf(L.x, e.y, fmaf(L.y, e.x, Bm.y)));
      Eb[m] = w;
      dpart += fmaf(ar, w.x, ai * w.y);
    }
  }
  if (lane == 0) pden[warp] = dpart;
  __syncthreads();
  // CTA partial: fold the 8 warp rows into row 0
  for (int f = tid; f < DV; f += kDecThreads) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += part[w * DV + f];
    part[f] = s;
  }
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += pden[w];
    pden[0] = s;
  }
  cluster.sync();
  if (g == 0) {
    float dn = 0.f;
    for (int r = 0; r < G; ++r) dn += cluster.map_shared_rank(pden, r)[0];
    for (int f = tid; f < DV; f += kDecThreads) {
      float s = 0.f;
      for (int r = 0; r < G; ++r) s += cluster.map_shared_rank(part, r)[f];
      o[bh * DV + f] = s / dn;
      if (num) num[bh * DV + f] = s;
    }
    if (den && tid == 0) den[bh] = dn;
  }
  cluster.sync();   // keep every CTA's shared memory alive until rank 0 has read it
}

// Large-batch variant: one CTA per (b,h) covers all modes, so no cluster and
// no cross-CTA reduction is needed.  Each warp walks its modes (warp, warp+8,
// ...) through a ring of D shared-memory slots: bulk copies bring the U and
// Gamma rows of the next D modes while it updates the current one, so each SM
// keeps enough bytes in flight to cover the memory latency; the updated rows
// go straight back to HBM and the partial Re(a^H Gamma) stays in registers.
constexpr int kBhWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kBhWarps * 32, 3) decode_bh_kernel(
    int H, int DX, int DV, int M, int D, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const float* __restrict__ delta, int dpm, const float* __restrict__ A,
    float2* __restrict__ state, float* __restrict__ o, float* __restrict__ num,
    float* __restrict__ den, long long BH, int* err) {
  extern __shared__ float4 dsm[];
  const uint32_t rowU = static_cast<uint32_t>(DX) * 8, rowG = static_cast<uint32_t>(DV) * 8, slot = rowU + rowG;
  // ring of D mode rows (U row then Gamma row) per warp, then its mbarriers
  uint8_t* ring = reinterpret_cast<uint8_t*>(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kBhWarps * D * slot);
  float* fq = reinterpret_cast<float*>(bars + kBhWarps * D);
  float* fk = fq + DX;
  float* vv = fk + DX;
  float* part = vv + DV;                    // [8][DV]
  float* pden = part + kBhWarps * DV;       // [8]
  float2* lamb = reinterpret_cast<float2*>(pden + kBhWarps);   // [M]
  float2* bb = lamb + M;
  float2* eta = bb + M;
  const long long bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nu = DX / 2, ng = DV / 2;
  float2* Ub = state + bh * M * DX;
  float2* Gb = state + BH * M * DX + bh * M * DV;
  float2* Eb = state + BH * M * (DX + DV) + bh * M;
  uint8_t* myring = ring + warp * D * slot;
  uint64_t* mybar = bars + warp * D;
  const int nj = warp < M ? (M - warp + kBhWarps - 1) / kBhWarps : 0;   // modes warp, warp + 8, ...

  // each warp streams its own modes' state rows through its ring, D rows ahead
  auto issue = [&](int j) {
    const int m = warp + kBhWarps * j, s = j % D;
    mbar_arrive_expect_tx(mybar + s, slot);
    bulk_g2s(myring + s * slot, Ub + static_cast<long long>(m) * DX, rowU, mybar + s);
    bulk_g2s(myring + s * slot + rowU, Gb + static_cast<long long>(m) * DV, rowG, mybar + s);
  };
  int issued = 0;
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(mybar + s, 1);
    fence_barrier_init();
    for (; issued < D && issued < nj; ++issued) issue(issued);
  }
  __syncwarp();

  for (int f = tid; f < DX; f += kBhWarps * 32) {
    fq[f] = xi_acc(ldx(q + bh * DX + f));
    fk[f] = xi_acc(ldx(k + bh * DX + f));
  }
  for (int f = tid; f < DV; f += kBhWarps * 32) vv[f] = ldx(v + bh * DV + f);
  for (int m = tid; m < M; m += kBhWarps * 32) {
    const float ar = A ? A[2 * m] : -0.5f;
    const float ai = A ? A[2 * m + 1] : 3.14159265358979f * static_cast<float>(m);
    const float d = delta_hm(delta, dpm, M, h, m);
    const float x = d * ar, y = d * ai;
    float sy, cy, sh, ch;
    sincosf(y, &sy, &cy);
    sincosf(0.5f * y, &sh, &ch);
    const float ex = expf(x), em1 = expm1f(x);
    const float nr = fmaf(em1, cy, -2.f * sh * sh), ni = ex * sy;
    const float dd = fmaf(ar, ar, ai * ai);
    lamb[m] = make_float2(ex * cy, ex * sy);
    bb[m] = make_float2(fmaf(nr, ar, ni * ai) / dd, fmaf(ni, ar, -nr * ai) / dd);
    eta[m] = Eb[m];
  }
  __syncthreads();

  float acc[2 * kVecPerLane];
#pragma unroll
  for (int i = 0; i < 2 * kVecPerLane; ++i) acc[i] = 0.f;
  float dpart = 0.f;
  bool ok = true;
  for (int j = 0; j < nj; ++j) {
    const int m = warp + kBhWarps * j, s = j % D;
    if (!mbar_wait(mybar + s, static_cast<uint32_t>((j / D) & 1), err)) {
      ok = false;
      break;
    }
    const float4* us = reinterpret_cast<const float4*>(myring + s * slot);
    const float4* gs = reinterpret_cast<const float4*>(myring + s * slot + rowU);
    const float2 L = lamb[m], Bm = bb[m];
    float4* Ur = reinterpret_cast<float4*>(Ub + static_cast<long long>(m) * DX);
    float4* Gr = reinterpret_cast<float4*>(Gb + static_cast<long long>(m) * DV);
    float ar = 0.f, ai = 0.f;
#pragma unroll
    for (int i = 0; i < kVecPerLane; ++i) {
      const int p = lane + 32 * i;
      if (p < nu) {
        const float4 u = us[p];
        const float x0 = fk[2 * p], x1 = fk[2 * p + 1];
        float4 w;
        w.x = fmaf(L.x, u.x, fmaf(-L.y, u.y, Bm.x * x0));
        w.y = fmaf(L.x, u.y, fmaf(L.y, u.x, Bm.y * x0));
        w.z = fmaf(L.x, u.z, fmaf(-L.y, u.w, Bm.x * x1));
        w.w = fmaf(L.x, u.w, fmaf(L.y, u.z, Bm.y * x1));
        Ur[p] = w;
        ar = fmaf(w.x, fq[2 * p], fmaf(w.z, fq[2 * p + 1], ar));
        ai = fmaf(w.y, fq[2 * p], fmaf(w.w, fq[2 * p + 1], ai));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ar += __shfl_xor_sync(0xffffffffu, ar, off);
      ai += __shfl_xor_sync(0xffffffffu, ai, off);
    }
#pragma unroll
    for (int i = 0; i < kVecPerLane; ++i) {
      const int p = lane + 32 * i;
      if (p < ng) {
        const float4 g = gs[p];
        const float x0 = vv[2 * p], x1 = vv[2 * p + 1];
        float4 w;
        w.x = fmaf(L.x, g.x, fmaf(-L.y, g.y, Bm.x * x0));
        w.y = fmaf(L.x, g.y, fmaf(L.y, g.x, Bm.y * x0));
        w.z = fmaf(L.x, g.z, fmaf(-L.y, g.w, Bm.x * x1));
        w.w = fmaf(L.x, g.w, fmaf(L.y, g.z, Bm.y * x1));
        Gr[p] = w;
        acc[2 * i] = fmaf(ar, w.x, fmaf(ai, w.y, acc[2 * i]));        // Re(conj(a) Gamma)
        acc[2 * i + 1] = fmaf(ar, w.z, fmaf(ai, w.w, acc[2 * i + 1]));
      }
    }
    if (lane == 0) {
      const float2 e = eta[m];
      const float2 w = make_float2(fmaf(L.x, e.x, fmaf(-L.y, e.y, Bm.x)), fmaf(L.x, e.y, fmaf(L.y, e.x, Bm.y)));
      Eb[m] = w;
      dpart = fmaf(ar, w.x, fmaf(ai, w.y, dpart));
    }
    __syncwarp();   // every lane has read slot s
    if (lane == 0 && issued < nj) {
      fence_async_smem();   // the generic reads of the slot come before the copy that refills it
      issue(issued++);
    }
  }
  if (!ok) {   // let this warp's copies in flight land (bounded) before the block exits
    if (lane == 0)
      for (int j = 0; j < issued; ++j) mbar_wait(mybar + j % D, static_cast<uint32_t>((j / D) & 1), err);
    __syncwarp();
  }
#pragma unroll
  for (int i = 0; i < kVecPerLane; ++i) {
    const int p = lane + 32 * i;
    if (p < ng) {
      part[warp * DV + 2 * p] = acc[2 * i];
      part[warp * DV + 2 * p + 1] = acc[2 * i + 1];
    }
  }
  if (lane == 0) pden[warp] = dpart;
  __syncthreads();
  float dn = 0.f;
  for (int w = 0; w < kBhWarps; ++w) dn += pden[w];
  for (int f = tid; f < DV; f += kBhWarps * 32) {
    float s = 0.f;
    for (int w = 0; w < kBhWarps; ++w) s += part[w * DV + f];
    o[bh * DV + f] = s / dn;
    if (num) num[bh * DV + f] = s;
  }
  if (den && tid == 0) den[bh] = dn;
}

template <typename T>
cudaError_t decode_impl(const ia_shape_t& s, const void* q, const void* k, const void* v,
                        const float* delta, const float* A, void* state, float* o, float* num,
                        float* den, cudaStream_t st) {
  const long long BHc = static_cast<long long>(s.B) * s.H;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // tuning switch: the smallest B*H that takes the one-CTA-per-(b,h) kernel
  const char* thr_env = std::getenv("IA_DECODE_BH_MIN");
  const long long thr = thr_env ? std::atoll(thr_env) : static_cast<long long>(sms);
  if (BHc >= thr) {   // at least one (b,h) per SM: no need to split the modes across CTAs
    // ring depth: four mode rows per warp while several CTAs still fit on an SM
    const size_t row = static_cast<size_t>(s.d_xi + s.d_v) * 8;
    const int D = kBhWarps * 4 * row <= 96 * 1024 ? 4 : 2;
    const size_t smem = kBhWarps * D * (row + 8) + sizeof(float) * (2 * s.d_xi + s.d_v + kBhWarps * s.d_v + kBhWarps) +
                        sizeof(float2) * 3 * s.M + 16;
    int* err = device_error_ptr();
    if (!err) return cudaErrorInvalidSymbol;
    auto kern = decode_bh_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mark_launch_begin(st);
    kern<<<static_cast<unsigned>(BHc), kBhWarps * 32, smem, st>>>(
        s.H, s.d_xi, s.d_v, s.M, D, static_cast<const T*>(q), static_cast<const T*>(k),
        static_cast<const T*>(v), delta, s.delta_per_mode, A, static_cast<float2*>(state), o, num, den, BHc, err);
    e = cudaGetLastError();
    mark_launch_end(st);
    return e;
  }
  // 16 modes (two per warp) per CTA, up to 8 CTAs per cluster
  const int G = (s.M + 15) / 16;
  const int MG = (s.M + G - 1) / G;
  const long long BH = static_cast<long long>(s.B) * s.H;
  const size_t smem = sizeof(float) * (2 * s.d_xi + s.d_v + 8 * s.d_v + 8) + sizeof(float2) * 2 * MG + 16;
  auto kern = decode_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G * BH), 1, 1);
  cfg.blockDim = dim3(kDecThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  mark_launch_begin(st);
  e = cudaLaunchKernelEx(&cfg, kern, s.H, s.d_xi, s.d_v, s.M, MG, static_cast<const T*>(q),
                         static_cast<const T*>(k), static_cast<const T*>(v), delta, s.delta_per_mode, A,
                         static_cast<float2*>(state), o, num, den, BH);
  mark_launch_end(st);
  return e;
}

}  // namespace

cudaError_t launch_decode(const ia_shape_t& s, const void* q, const void* k, const void* v,
                          const float* delta, const float* A, void* state, float* o, float* num,
                          float* den, cudaStream_t st) {
  if (s.in_dtype == IA_F32) return decode_impl<float>(s, q, k, v, delta, A, state, o, num, den, st);
  return decode_impl<__nv_bfloat16>(s, q, k, v, delta, A, state, o, num, den, st);
}

}  // namespace ia
