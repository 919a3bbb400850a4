// One recurrent decode step of the IA layer (paperlayer.ai summary of
// 'Interdomain Attention', sec. 3.2: a fixed state of size O(M(R + d)) and
// constant work per generated token; sec. F.3: graphed decode whose latency
// does not depend on the prefix length).  For every (b,h):
//   U <- lambda U + b xi(k)^T,  Gamma <- lambda Gamma + b v^T,  eta <- lambda eta + b
//   a = U xi(q),  o = Re(a^H Gamma) / Re(a^H eta)
//
// The step is bound by state bytes: every state entry is read and written
// once in fp32.  A cluster of 1-8 CTAs serves one (b,h); each CTA streams a
// group of modes through shared memory with bulk copies and writes them back
// with 16-byte stores, and the cluster's rank-0 CTA sums the partial num/den
// over distributed shared memory and writes o.
#include <algorithm>
#include <cstdlib>
#include <cooperative_groups.h>

#include "ia_device.cuh"
#include "ia_internal.h"

namespace cg = cooperative_groups;

namespace ia {
namespace {

constexpr int kVecPerLane = 4;   // rows up to 256 complex entries (d <= 256)

template <typename T>
__device__ __forceinline__ float ldx(const T* p);
template <>
__device__ __forceinline__ float ldx<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float xi_acc(float x) { return x > 0.f ? x + 1.f : expf(x); }

// Streaming variant: a cluster of S CTAs (S = 1, 2, 4 or 8) serves one
// (b,h), CTA r taking modes [r M/S, (r+1) M/S).  Each warp walks its modes
// (warp, warp+8, ... of that range) through a ring of D shared-memory slots:
// bulk copies bring the U and Gamma rows of the next D modes while it
// updates the current one, so each SM keeps enough bytes in flight to cover
// the memory latency; the updated rows go straight back to HBM and the
// partial Re(a^H Gamma) stays in registers.  Small batches take S > 1 so
// that every SM holds several CTAs and each warp's rows are all in flight at
// once; the cluster's rank-0 CTA then adds the partials of the others over
// distributed shared memory, in rank order.
// NW warps per CTA (8).  Smaller CTAs (4 warps, each (b,h) split over 2, 4
// or 8 of them so that every SM gets an even share of mode rows) measured
// slower on a B200 at every batch of the 1.3B shape: at B = 16 the 256 whole
// (b,h) already stream at about 0.9 of HBM in the main phase, and the split
// repeats the per-(b,h) set-up.
template <typename T, int NW>
__global__ void __launch_bounds__(NW * 32, NW == 8 ? 4 : 8) decode_bh_kernel(
    int H, int DX, int DV, int M, int D, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const float* __restrict__ delta, int dpm, const float* __restrict__ A,
    float2* __restrict__ state, float* __restrict__ o, float* __restrict__ num,
    float* __restrict__ den, long long BH, int* err) {
  constexpr int kBhWarps = NW;
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
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int S = static_cast<int>(cluster.num_blocks());
  const long long bh = blockIdx.x / S;
  const int h = static_cast<int>(bh % H);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nu = DX / 2, ng = DV / 2;
  const int MS = M / S, m_lo = rank * MS;   // this CTA's modes
  float2* Ub = state + bh * M * DX;
  float2* Gb = state + BH * M * DX + bh * M * DV;
  float2* Eb = state + BH * M * (DX + DV) + bh * M;
  uint8_t* myring = ring + warp * D * slot;
  uint64_t* mybar = bars + warp * D;
  const int nj = warp < MS ? (MS - warp + kBhWarps - 1) / kBhWarps : 0;   // modes m_lo + warp, + 8, ...
  // Programmatic dependent launch: this grid may have become resident while
  // the previous kernel in the stream finished; nothing global is read before
  // that kernel has completed and its writes are visible.
  griddep_wait();

  // each warp streams its own modes' state rows through its ring, D rows ahead
  auto issue = [&](int j) {
    const int m = m_lo + warp + kBhWarps * j, s = j % D;
    mbar_arrive_expect_tx(mybar + s, slot);
    bulk_g2s(myring + s * slot, Ub + static_cast<long long>(m) * DX, rowU, mybar + s);
    bulk_g2s(myring + s * slot + rowU, Gb + static_cast<long long>(m) * DV, rowG, mybar + s);
  };
  // The per-(b,h) inputs (q, k, v, Delta, A, eta) are loaded first, in one
  // round trip, ahead of the ring's bulk copies: behind them, each of these
  // small dependent loads would wait out the copies' queue.
  constexpr int NT = kBhWarps * 32;
  constexpr int R = (2 * 32 * kVecPerLane + NT - 1) / NT;   // features per thread (d <= 256)
  float xq[R], xk[R], xv[R], pd = 0.f, par = -0.5f, pai = 0.f;
  float2 pe = make_float2(0.f, 0.f);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int f = tid + r * NT;
    xq[r] = f < DX ? ldx(q + bh * DX + f) : 0.f;
    xk[r] = f < DX ? ldx(k + bh * DX + f) : 0.f;
    xv[r] = f < DV ? ldx(v + bh * DV + f) : 0.f;
  }
  if (tid < MS) {
    const int m = m_lo + tid;
    if (A) {
      par = A[2 * m];
      pai = A[2 * m + 1];
    } else {
      pai = 3.14159265358979f * static_cast<float>(m);
    }
    pd = delta_hm(delta, dpm, M, h, m);
    pe = Eb[m];
  }
  int issued = 0;
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(mybar + s, 1);
    fence_barrier_init();
    for (; issued < D && issued < nj; ++issued) issue(issued);
  }
  __syncwarp();

  // lambda = exp(Delta A), b = (lambda - 1)/A in fp32; lambda - 1 is formed as
  // expm1(x) cos(y) - 2 sin^2(y/2) + i e^x sin(y), keeping its relative
  // accuracy for small Delta
  auto params = [&](int mi, float ar, float ai, float d, float2 e) {
    const float x = d * ar, y = d * ai;
    float sy, cy, sh, ch;
    sincosf(y, &sy, &cy);
    sincosf(0.5f * y, &sh, &ch);
    const float ex = expf(x), em1 = expm1f(x);
    const float nr = fmaf(em1, cy, -2.f * sh * sh), ni = ex * sy;
    const float dd = fmaf(ar, ar, ai * ai);
    lamb[mi] = make_float2(ex * cy, ex * sy);
    bb[mi] = make_float2(fmaf(nr, ar, ni * ai) / dd, fmaf(ni, ar, -nr * ai) / dd);
    eta[mi] = e;
  };
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int f = tid + r * NT;
    if (f < DX) {
      fq[f] = xi_acc(xq[r]);
      fk[f] = xi_acc(xk[r]);
    }
    if (f < DV) vv[f] = xv[r];
  }
  if (tid < MS) params(tid, par, pai, pd, pe);
  for (int mi = tid + NT; mi < MS; mi += NT) {   // more modes per CTA than threads
    const int m = m_lo + mi;
    params(mi, A ? A[2 * m] : -0.5f, A ? A[2 * m + 1] : 3.14159265358979f * static_cast<float>(m),
           delta_hm(delta, dpm, M, h, m), Eb[m]);
  }
  __syncthreads();

  float acc[2 * kVecPerLane];
#pragma unroll
  for (int i = 0; i < 2 * kVecPerLane; ++i) acc[i] = 0.f;
  float dpart = 0.f;
  bool ok = true;
  for (int j = 0; j < nj; ++j) {
    const int mi = warp + kBhWarps * j, m = m_lo + mi, s = j % D;
    if (!mbar_wait(mybar + s, static_cast<uint32_t>((j / D) & 1), err)) {
      ok = false;
      break;
    }
    const float4* us = reinterpret_cast<const float4*>(myring + s * slot);
    const float4* gs = reinterpret_cast<const float4*>(myring + s * slot + rowU);
    const float2 L = lamb[mi], Bm = bb[mi];
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
      const float2 e = eta[mi];
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
  // the next kernel in the stream may launch once every CTA has streamed its
  // rows (it still waits for this grid's completion before reading memory)
  griddep_launch_dependents();
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
  if (S == 1) {
    float dn = 0.f;
    for (int w = 0; w < kBhWarps; ++w) dn += pden[w];
    for (int f = tid; f < DV; f += kBhWarps * 32) {
      float s = 0.f;
      for (int w = 0; w < kBhWarps; ++w) s += part[w * DV + f];
      o[bh * DV + f] = s / dn;
      if (num) num[bh * DV + f] = s;
    }
    if (den && tid == 0) den[bh] = dn;
    return;
  }
  // fold this CTA's warps into row 0, then rank 0 adds the ranks in order
  for (int f = tid; f < DV; f += kBhWarps * 32) {
    float s = 0.f;
    for (int w = 0; w < kBhWarps; ++w) s += part[w * DV + f];
    part[f] = s;
  }
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < kBhWarps; ++w) s += pden[w];
    pden[0] = s;
  }
  cluster.sync();
  if (rank == 0) {
    float dn = 0.f;
    for (int r = 0; r < S; ++r) dn += cluster.map_shared_rank(pden, r)[0];
    for (int f = tid; f < DV; f += kBhWarps * 32) {
      float s = 0.f;
      for (int r = 0; r < S; ++r) s += cluster.map_shared_rank(part, r)[f];
      o[bh * DV + f] = s / dn;
      if (num) num[bh * DV + f] = s;
    }
    if (den && tid == 0) den[bh] = dn;
  }
  cluster.sync();   // keep every CTA's shared memory alive until rank 0 has read it
}

// shared memory besides the ring: features, partial sums, mode parameters
size_t decode_fixed_smem(const ia_shape_t& s, int nw) {
  return sizeof(float) * (2 * s.d_xi + s.d_v + nw * s.d_v + nw) + sizeof(float2) * 3 * s.M + 16;
}

template <typename T, int NW>
cudaError_t decode_launch(const ia_shape_t& s, int S, const void* q, const void* k, const void* v,
                          const float* delta, const float* A, void* state, float* o, float* num, float* den,
                          cudaStream_t st) {
  const long long BHc = static_cast<long long>(s.B) * s.H;
  // ring depth: up to four mode rows per warp, within a quarter of an SM's
  // shared memory per CTA so that four fit (a deeper ring for fewer CTAs per
  // SM measured slower on a B200)
  const size_t row = static_cast<size_t>(s.d_xi + s.d_v) * 8;
  const size_t fixed = decode_fixed_smem(s, NW);
  const int per_warp = (s.M / S + NW - 1) / NW;
  const size_t budget = 56 * 1024;
  int D = 4;
  while (D > 1 && NW * D * (row + 8) + fixed > budget) --D;
  D = std::max(1, std::min(D, per_warp));
  const size_t smem = NW * D * (row + 8) + fixed;
  int* err = device_error_ptr();
  if (!err) return cudaErrorInvalidSymbol;
  auto kern = decode_bh_kernel<T, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BHc * S), 1, 1);
  cfg.blockDim = dim3(NW * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  mark_launch_begin(st);
  e = cudaLaunchKernelEx(&cfg, kern, s.H, s.d_xi, s.d_v, s.M, D, static_cast<const T*>(q), static_cast<const T*>(k),
                         static_cast<const T*>(v), delta, s.delta_per_mode, A, static_cast<float2*>(state), o, num,
                         den, BHc, err);
  mark_launch_end(st);
  return e;
}

template <typename T>
cudaError_t decode_impl(const ia_shape_t& s, const void* q, const void* k, const void* v,
                        const float* delta, const float* A, void* state, float* o, float* num,
                        float* den, cudaStream_t st) {
  const long long BHc = static_cast<long long>(s.B) * s.H;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Cluster size S: one CTA per (b,h) once there is a (b,h) for every SM,
  // else the fewest CTAs per (b,h) that give every SM one (S divides M; on a
  // B200 splitting the 256 (b,h) of a 16 x 16-head batch measured slower, each
  // CTA repeating the per-(b,h) set-up).  IA_DECODE_SPLIT=n forces S.
  int S = 1;
  while (S < 8 && BHc * S < sms && s.M % (2 * S) == 0) S *= 2;
  if (const char* env = std::getenv("IA_DECODE_SPLIT")) {
    const int f = std::atoi(env);
    if ((f == 1 || f == 2 || f == 4 || f == 8) && s.M % f == 0) S = f;
  }
  return decode_launch<T, 8>(s, S, q, k, v, delta, A, state, o, num, den, st);
}

}  // namespace

size_t decode_smem_bytes(const ia_shape_t& s) {   // the larger CTA's least ring
  return 8 * (static_cast<size_t>(s.d_xi + s.d_v) * 8 + 8) + decode_fixed_smem(s, 8);
}

cudaError_t launch_decode(const ia_shape_t& s, const void* q, const void* k, const void* v,
                          const float* delta, const float* A, void* state, float* o, float* num,
                          float* den, cudaStream_t st) {
  if (s.in_dtype == IA_F32) return decode_impl<float>(s, q, k, v, delta, A, state, o, num, den, st);
  return decode_impl<__nv_bfloat16>(s, q, k, v, delta, A, state, o, num, den, st);
}

}  // namespace ia
