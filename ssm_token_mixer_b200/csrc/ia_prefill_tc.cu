// Chunked IA prefill on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// What it computes is the causal IA layer (paper 'Interdomain Attention:
// Beyond Token-Level Key-Value Memory'; paperlayer.ai summary sec. 3.1-3.2;
// AI-radio page formula extract "O = Fq U^T Gamma / Fq U^T eta"), run
// chunkwise with chunk length C = 64 and state passing between chunks as the
// summary's sec. A.2 describes.  Per (b,h) and chunk, with positions i, j in
// [0, C), centre c = C/2 and the per-head table E'[j,m] = b_m lambda_m^(c-j):
//
//   S^T   = xi(K) xi(Q)^T                         GEMM1  (masked j <= i)
//   a~^T  = E'^T S^T + R_U xi(Q)^T                GEMM2 + GEMM3   (a_i = lambda^(i-c) a~_i)
//   X     = |lambda|^(2(i-c)) a~                  (rows re/im; = conj(a) lambda^(i-c))
//   P     = X E'^T                                GEMM4  (masked j <= i)
//   num   = P V + X R_Gamma,  den = P 1 + X R_eta GEMM5,5b + GEMM6,6b
//   o     = num / den
//   S_hat <- R + E'^T [xi(K) | V]                 GEMM7  (accumulated onto R in TMEM)
//
// where the running state is kept scaled, S_hat = lambda^-(C-c-1) S, so that
// R = lambda^C S_hat is both the decayed state the chunk adds to and the
// carried state its queries read (lambda^(c+1) S0).  Complex numbers are
// split into real rows k = 2m (re) and 2m+1 (im), so every contraction is a
// real fp16 x fp16 -> fp32 tcgen05 MMA with M = 64 or 128.
//
// Layouts: every shared-memory operand is in the no-swizzle canonical layout
// (core matrices of 8 rows x 16 bytes, 128 contiguous bytes).  A tile with
// rows r and columns x (x contiguous) of width W stores element (r, x) at
//   (r/8)*(W*16) + (x/8)*128 + (r%8)*16 + (x%8)*2,
// which serves as K-major (rows = M/N, lbo 128, sbo W*16) or as MN-major
// (columns = M/N, lbo W*16, sbo 128) depending on the contraction.
//
// TMEM columns: [0,F) scaled state rows k; [F,F+64) a~^T (den aliases its
// first 16 columns later in the chunk); [F+64,F+128) S^T then P (M=64
// layout); [F+128, F+128+DV) num (M=64 layout).  F = d_xi + d_v.
//
// Sequences are split into segments when (b,h) pairs alone cannot fill the
// GPU: a state-only pass produces each segment's local end state, a scan
// combines them (S_in(s+1) = lambda^L S_in(s) + S_local(s)), and the full
// pass recomputes every segment from its carried-in state -- the two
// parallel passes around a sequential carry pass of the summary's sec. A.2.
#include <cuda.h>

#include <cmath>
#include <cstdlib>

#include "ia_device.cuh"
#include "ia_internal.h"
#include "ia_tables.cuh"
#include "ia_tc_common.cuh"

namespace ia {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links no driver stub).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// q, k or v [BH][N][64] bf16: one box is 64 rows x 64 columns (128 bytes) of
// one (b,h), 128-byte swizzled in shared memory.  Rows >= N lie outside the
// map and read as zero.
bool encode_input_map(CUtensorMap* m, const void* x, long long BH, int N) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {64 * 2, static_cast<cuuint64_t>(N) * 64 * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kChunk), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An fp32 [BH][N][64] array (o, dq, dk, dv) seen as boxes of 32 columns x 64
// rows of one (b,h), 128-byte swizzled in shared memory; rows >= N lie
// outside the map (TMA stores skip them).
bool encode_rows64_f32_map(CUtensorMap* m, float* o, long long BH, int N) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {64 * sizeof(float), static_cast<cuuint64_t>(N) * 64 * sizeof(float)};
  const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(kChunk), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, o, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using namespace tc;

constexpr int NT = 512;            // 16 warps: warp w owns TMEM lane quadrant w%4, column quarter w/4
constexpr int NWARP = NT / 32;

template <int DX, int DV>
struct Cfg {
  static constexpr int F = DX + DV;
  // den rides along the value contractions as an extra column when TMEM has room
  static constexpr bool MERGE = F + 128 + DV + 16 <= 512;
  static constexpr int WV = MERGE ? DV + 16 : DV;   // width of the V and R_Gamma tiles
  static constexpr int NV = MERGE ? DV + 16 : DV;   // N of the value contractions
  static constexpr uint32_t RSX = DX * 16;          // row-group stride of an [r][DX] fp16 tile
  static constexpr uint32_t RSV = WV * 16;
  static constexpr uint32_t T_STATE = 0, T_A = F, T_SP = F + 64, T_NUM = F + 128;
  static constexpr uint32_t T_DEN = MERGE ? T_NUM + DV : F;
  static_assert(F + 128 + NV <= 512, "TMEM budget");
  static_assert(DX % 64 == 0 && DV % 64 == 0, "feature widths must be multiples of 64");
  static constexpr uint32_t STG_Q = 0;
  static constexpr uint32_t STG_K = STG_Q + C * DX * 2;
  static constexpr uint32_t STG_V = STG_K + C * DX * 2;
  static constexpr uint32_t S_Q = STG_V + C * DV * 2;
  static constexpr uint32_t S_K = S_Q + C * DX * 2;
  static constexpr uint32_t S_V = S_K + C * DX * 2;
  static constexpr uint32_t S_E = S_V + C * WV * 2;
  static constexpr uint32_t S_SP = S_E + KR * C * 2;
  static constexpr uint32_t S_X = S_SP + C * C * 2;
  static constexpr uint32_t S_RU = S_X + KR * C * 2;
  static constexpr uint32_t S_RG = S_RU + KR * DX * 2;
  static constexpr uint32_t S_RE = S_RG + KR * WV * 2;
  static constexpr uint32_t S_ONES = S_RE + (MERGE ? 0 : KR * 16 * 2);
  static constexpr uint32_t S_BAR = S_ONES + (MERGE ? 0 : C * 16 * 2);
  static constexpr uint32_t S_TMEMH = S_BAR + 32;
  static constexpr uint32_t SMEM = S_TMEMH + 16;
  // o of one chunk is staged (fp32, swizzled) over the sX and sRU tiles, both
  // free while the output is written
  static constexpr uint32_t S_OUT = S_X;
  static_assert(KR * C * 2 + KR * DX * 2 >= C * DV * 4, "output staging fits");
};

struct TcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const HeadTables* tabs;
  const float2* state_in;   // public layout, unscaled; seeds segment 0 of the full pass
  float* seg_state;         // [BH][nseg-1][128][F] scaled: local end states, then carries
  float* seg_eta;           // [BH][nseg-1][128]
  float* o;
  float* num;
  float* den;
  float2* state_out;
  int* err;                 // device error flag
  uint8_t* dump_R;          // optional: R = lambda^C S_hat at every chunk start, fp16 tiles (dump_r16)
  float* dump_Re;           // optional: the eta part, [BH][nch][128] fp32
  int H, N, nseg, seg_chunks;
  long long BH;
};

// bf16 staging rows [C][W] (row-major) -> fp16 canonical tile of row width WD,
// applying xi when FEAT; rows >= nv become zero.  Work is split into warp
// iterations of 8 rows x 4 column groups, the column group rotated by the row
// so that staging reads and tile writes are bank-conflict free; all loads of
// a thread are issued before any conversion.
template <int W, int WD, bool FEAT, int NW = NWARP>
__device__ __forceinline__ void convert_all(const uint8_t* stg, uint8_t* dst, int nv, int warp, int lane) {
  constexpr int NCG = W / 8;
  constexpr int ITERS = (C / 8) * (NCG / 4);
  constexpr int PER = (ITERS + NW - 1) / NW;
  const int r8 = lane & 7, slot = lane >> 3;
  uint4 in[PER];
  int rr[PER], cc[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int it = warp + u * NW;
    const int rb = it & 7, rest = it >> 3;
    rr[u] = rb * 8 + r8;
    cc[u] = (rest >> 1) * 8 + ((slot + 4 * (rest & 1) + r8) & 7);
    in[u] = make_uint4(0u, 0u, 0u, 0u);
    if (it < ITERS && rr[u] < nv) in[u] = *reinterpret_cast<const uint4*>(stg + rr[u] * (W * 2) + cc[u] * 16);
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int it = warp + u * NW;
    if (it >= ITERS) break;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (rr[u] < nv) {
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&in[u]);
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        if (FEAT) { f.x = feat(f.x); f.y = feat(f.y); }
        w[e] = pack_half2(f.x, f.y);
      }
      out = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(dst + tile_off(rr[u], cc[u] * 8, WD * 16)) = out;
  }
}

__device__ __forceinline__ uint4 pack8f(const uint32_t* r, float scale) {
  return make_uint4(pack_half2(__uint_as_float(r[0]) * scale, __uint_as_float(r[1]) * scale),
                    pack_half2(__uint_as_float(r[2]) * scale, __uint_as_float(r[3]) * scale),
                    pack_half2(__uint_as_float(r[4]) * scale, __uint_as_float(r[5]) * scale),
                    pack_half2(__uint_as_float(r[6]) * scale, __uint_as_float(r[7]) * scale));
}

// R for the reverse pass: per chunk two fp16 tiles, R_U then R_Gamma, each
// 128 rows (k) x 64 columns in the 128-byte swizzled layout (16-byte chunk c
// of row k at byte k * 128 + (c ^ (k % 8)) * 16), 32 KB per chunk, so that a
// plain bulk copy lands them ready to serve as tensor-core operands.  Stores
// columns col0..col0+15 (col0 a multiple of 16) of row k of chunk `chunk`.
constexpr uint32_t kDumpTile = KR * 64 * 2;
__device__ __forceinline__ void dump_r16(uint8_t* base, long long chunk, int k, int col0, const uint32_t* w) {
  uint8_t* row = base + (chunk * 2 + (col0 >= 64 ? 1 : 0)) * kDumpTile + k * 128;
  const int c0 = (col0 & 63) >> 3;
#pragma unroll
  for (int g = 0; g < 2; ++g)
    *reinterpret_cast<uint4*>(row + (((c0 + g) ^ (k & 7)) << 4)) = pack8f(w + 8 * g, 1.f);
}

template <int DX, int DV, bool FULL>
__global__ void __launch_bounds__(NT, 1) tc_prefill_kernel(const TcArgs a) {
  using K = Cfg<DX, DV>;
  constexpr int F = K::F;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, part = warp >> 2;   // lane quadrant, column quarter
  const int nrun = FULL ? a.nseg : a.nseg - 1;
  const long long bh = blockIdx.x / nrun;
  const int seg = static_cast<int>(blockIdx.x % nrun);
  const int h = static_cast<int>(bh % a.H);
  const HeadTables* T = a.tabs + h;
  const int nch_total = (a.N + C - 1) / C;
  const int ch0 = seg * a.seg_chunks;
  const int ch1 = min(ch0 + a.seg_chunks, nch_total);

  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + K::S_TMEMH);
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  {  // E' table -> shared (already in canonical layout), constant tiles
    const uint4* src = reinterpret_cast<const uint4*>(T->E);
    uint4* dst = reinterpret_cast<uint4*>(smem + K::S_E);
    for (int i = tid; i < KR * C * 2 / 16; i += NT) dst[i] = src[i];
    if (FULL) {
      const uint32_t one2 = 0x3C003C00u;   // two fp16 ones
      if (K::MERGE) {
        // V's extra column DV is 1 (gives den = P 1), R_Gamma's extra columns
        // start at zero (column DV receives R_eta every chunk)
        for (int r = tid; r < C; r += NT) {
          *reinterpret_cast<uint4*>(smem + K::S_V + tile_off(r, DV, K::RSV)) = make_uint4(0x00003C00u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(smem + K::S_V + tile_off(r, DV + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
        }
        for (int r = tid; r < KR; r += NT) {
          *reinterpret_cast<uint4*>(smem + K::S_RG + tile_off(r, DV, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(smem + K::S_RG + tile_off(r, DV + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        uint4* ones = reinterpret_cast<uint4*>(smem + K::S_ONES);
        for (int i = tid; i < C * 16 * 2 / 16; i += NT) ones[i] = make_uint4(one2, one2, one2, one2);
        uint4* re = reinterpret_cast<uint4*>(smem + K::S_RE);
        for (int i = tid; i < KR * 16 * 2 / 16; i += NT) re[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Per-thread row constants: TMEM lane / state row k = 2m + comp.
  const int k = 32 * quad + lane;
  const int m = k >> 1, comp = k & 1;
  const float2 lamC = T->lamC[m];
  const float sgnLi = comp ? lamC.y : -lamC.y;
  const float r2 = T->r2[m];
  const float s_start = static_cast<float>(exp(2.0 * T->re_dA[m] * (16.0 * part - C / 2)));
  const float esum_c = comp ? T->esum[m].y : T->esum[m].x;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
  constexpr int FQ = F / 4;    // state columns per thread

  // Initial (scaled) state into TMEM rows.
  float eta_c = 0.f;
  {
    const float* carry = nullptr;
    const float* carry_eta = nullptr;
    if (FULL && seg > 0) {
      carry = a.seg_state + ((bh * (a.nseg - 1) + (seg - 1)) * KR + k) * F;
      carry_eta = a.seg_eta + (bh * (a.nseg - 1) + (seg - 1)) * KR + k;
    }
    const bool from_in = FULL && seg == 0 && a.state_in != nullptr;
    const float2 si = T->sc_inv[m];
#pragma unroll
    for (int cb = 0; cb < FQ; cb += 16) {
      const int col0 = part * FQ + cb;
      uint32_t r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float val = 0.f;
        const int f = col0 + e;
        if (carry) {
          val = carry[f];
        } else if (from_in) {
          float2 x = f < DX ? a.state_in[(bh * 64 + m) * DX + f]
                            : a.state_in[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)];
          val = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
        }
        r[e] = __float_as_uint(val);
      }
      tmem_st16(trow + K::T_STATE + col0, r);
    }
    if (carry_eta) {
      eta_c = *carry_eta;
    } else if (from_in) {
      float2 x = a.state_in[a.BH * 64 * F + bh * 64 + m];
      eta_c = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
    }
    tmem_st_wait();
  }

  auto issue_load = [&](int ch) {
    const int n0 = ch * C;
    const int nv = min(C, a.N - n0);
    const uint32_t bq = static_cast<uint32_t>(nv * DX * 2), bv = static_cast<uint32_t>(nv * DV * 2);
    mbar_arrive_expect_tx(bar_tma, FULL ? 2 * bq + bv : bq + bv);
    const long long row = bh * a.N + n0;
    if (FULL) bulk_g2s(smem + K::STG_Q, a.q + row * DX, bq, bar_tma);
    bulk_g2s(smem + K::STG_K, a.k + row * DX, bq, bar_tma);
    bulk_g2s(smem + K::STG_V, a.v + row * DV, bv, bar_tma);
  };

  if (tid == 0 && ch0 < ch1) issue_load(ch0);
  bool tma_pending = ch0 < ch1;
  uint32_t ph_tma = 0, ph_mma = 0;
  bool aborted = false;

  auto mma_sync = [&](void) -> bool {   // wait for the last commit; uniform result
    bool ok = mbar_wait(bar_mma, ph_mma, a.err);
    ph_mma ^= 1u;
    tc_fence_after();
    return !__syncthreads_or(!ok);
  };
  auto to_tensor_core = [&]() {   // make thread smem / TMEM writes visible to the MMA issuer
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  };

  int nv = C;
  for (int ch = ch0; ch < ch1; ++ch) {
    const int n0 = ch * C;
    nv = min(C, a.N - n0);
    {
      bool ok = mbar_wait(bar_tma, ph_tma, a.err);
      ph_tma ^= 1u;
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      tma_pending = false;
    }
    if (FULL) convert_all<DX, DX, true>(smem + K::STG_Q, smem + K::S_Q, nv, warp, lane);
    convert_all<DX, DX, true>(smem + K::STG_K, smem + K::S_K, nv, warp, lane);
    convert_all<DV, K::WV, false>(smem + K::STG_V, smem + K::S_V, nv, warp, lane);
    __syncthreads();   // staging consumed
    if (tid == 0 && ch + 1 < ch1) issue_load(ch + 1);
    tma_pending = ch + 1 < ch1;

    // ---- state: R = lambda^C S_hat -> TMEM (for GEMM7) and fp16 operands
#pragma unroll
    for (int cb = 0; cb < FQ; cb += 16) {
      const int col0 = part * FQ + cb;
      uint32_t r[16];
      tmem_ld16(trow + K::T_STATE + col0, r);
      tmem_ld_wait16(r);
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x = __uint_as_float(r[e]);
        const float y = __shfl_xor_sync(kFull, x, 1);
        w[e] = __float_as_uint(fmaf(lamC.x, x, sgnLi * y));
      }
      tmem_st16(trow + K::T_STATE + col0, w);
      if (FULL && a.dump_R) dump_r16(a.dump_R, bh * nch_total + ch, k, col0, w);
      if (FULL) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint4 pk = pack8f(w + 8 * g, 1.f);
          const int f = col0 + 8 * g;
          if (f < DX)
            *reinterpret_cast<uint4*>(smem + K::S_RU + tile_off(k, f, K::RSX)) = pk;
          else
            *reinterpret_cast<uint4*>(smem + K::S_RG + tile_off(k, f - DX, K::RSV)) = pk;
        }
      }
    }
    tmem_st_wait();
    {  // eta: R_eta = lambda^C eta_hat;  eta_hat <- R_eta + sum_{j<nv} E'[j]
      const float y = __shfl_xor_sync(kFull, eta_c, 1);
      const float Re = fmaf(lamC.x, eta_c, sgnLi * y);
      if (FULL && part == 0) {
        if (a.dump_Re) a.dump_Re[(bh * nch_total + ch) * KR + k] = Re;
        const uint4 pk = make_uint4(pack_half2(Re, 0.f), 0u, 0u, 0u);
        if (K::MERGE)
          *reinterpret_cast<uint4*>(smem + K::S_RG + tile_off(k, DV, K::RSV)) = pk;
        else
          *reinterpret_cast<uint4*>(smem + K::S_RE + tile_off(k, 0, 256)) = pk;
      }
      float add = esum_c;
      if (nv < C) {   // ragged last chunk: partial sum of E' over the valid keys
        double sr = 0.0, si = 0.0;
        const double br = T->b[m].x, bi = T->b[m].y;
        for (int j = 0; j < nv; ++j) {
          const double e = exp((C / 2 - j) * T->re_dA[m]);
          const double ph = fmod((C / 2 - j) * T->im_dA[m], 6.283185307179586476925);
          double sn, cs;
          sincos(ph, &sn, &cs);
          const double pr = e * cs, pi = e * sn;
          sr += br * pr - bi * pi;
          si += br * pi + bi * pr;
        }
        add = static_cast<float>(comp ? si : sr);
      }
      eta_c = Re + add;
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sE = sbase + K::S_E, sK = sbase + K::S_K, sV = sbase + K::S_V;
      if (FULL) {
        const uint32_t sQ = sbase + K::S_Q;
        gemm(tmem + K::T_SP, sK, 128, K::RSX, 256, sQ, 128, K::RSX, 256, idesc_f16(64, 64, 0, 0),
             DX / 16, false);   // GEMM1: S^T
      }
      gemm(tmem + K::T_STATE, sE, 128, 1024, 256, sK, K::RSX, 128, 2 * K::RSX,
           idesc_f16(128, DX, 0, 1), C / 16, true);   // GEMM7: U carry
      gemm(tmem + K::T_STATE + DX, sE, 128, 1024, 256, sV, K::RSV, 128, 2 * K::RSV,
           idesc_f16(128, DV, 0, 1), C / 16, true);   // GEMM7: Gamma carry
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }
    if (!FULL) continue;

    const int i0 = 16 * part;     // this warp's 16 columns of the 64-wide tiles
    // The M = 64 accumulators (S^T, P, num) fill lanes 0-15 of each quadrant:
    // thread t takes row 16 * quad + t % 16, the two half-warps splitting the
    // warp's columns.
    const int r16 = 16 * quad + (lane & 15), hb = lane >> 4;
    const int c8 = i0 + 8 * hb;   // this thread's 8 columns
    // ---- E1: S^T (M=64 rows j) -> masked fp16, MN-major B of GEMM2
    {
      const int j = r16;
      uint32_t r[8];
      tmem_ld8_halves<8>(trow + K::T_SP + i0, r);
      tmem_ld_wait8(r);
      const bool keep = j < nv;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!(keep && c8 + e >= j)) r[e] = 0u;
      *reinterpret_cast<uint4*>(smem + K::S_SP + tile_off(j, c8, 1024)) = pack8f(r, 1.f);
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sE = sbase + K::S_E, sSP = sbase + K::S_SP, sQ = sbase + K::S_Q,
                     sRU = sbase + K::S_RU;
      gemm(tmem + K::T_A, sE, 128, 1024, 256, sSP, 1024, 128, 2048, idesc_f16(128, 64, 0, 1),
           C / 16, false);   // GEMM2
      gemm(tmem + K::T_A, sRU, 128, K::RSX, 256, sQ, 128, K::RSX, 256, idesc_f16(128, 64, 0, 0),
           DX / 16, true);   // GEMM3
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E2: X = |lambda|^(2(i-c)) a~  (rows k, columns i) -> MN-major A of GEMM4/6
    {
      uint32_t r[16];
      tmem_ld16(trow + K::T_A + i0, r);
      tmem_ld_wait16(r);
      float s = s_start;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        r[e] = __float_as_uint(__uint_as_float(r[e]) * s);
        s *= r2;
      }
      *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0, 1024)) = pack8f(r, 1.f);
      *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 8, 1024)) = pack8f(r + 8, 1.f);
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      gemm(tmem + K::T_SP, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
           idesc_f16(64, 64, 1, 1), KR / 16, false);   // GEMM4: P
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E3: P (M=64 rows i) -> masked fp16, K-major A of GEMM5
    {
      const int i = r16;
      uint32_t r[8];
      tmem_ld8_halves<8>(trow + K::T_SP + i0, r);
      tmem_ld_wait8(r);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (c8 + e > i) r[e] = 0u;
      *reinterpret_cast<uint4*>(smem + K::S_SP + tile_off(i, c8, 1024)) = pack8f(r, 1.f);
    }
    to_tensor_core();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sSP = sbase + K::S_SP, sX = sbase + K::S_X;
      gemm(tmem + K::T_NUM, sSP, 128, 1024, 256, sbase + K::S_V, K::RSV, 128, 2 * K::RSV,
           idesc_f16(64, K::NV, 0, 1), C / 16, false);   // GEMM5: P [V | 1]
      gemm(tmem + K::T_NUM, sX, 1024, 128, 2048, sbase + K::S_RG, K::RSV, 128, 2 * K::RSV,
           idesc_f16(64, K::NV, 1, 1), KR / 16, true);   // GEMM6: X [R_Gamma | R_eta]
      if (!K::MERGE) {
        gemm(tmem + K::T_DEN, sSP, 128, 1024, 256, sbase + K::S_ONES, 256, 128, 512,
             idesc_f16(64, 16, 0, 1), C / 16, false);   // GEMM5b: P 1
        gemm(tmem + K::T_DEN, sX, 1024, 128, 2048, sbase + K::S_RE, 256, 128, 512,
             idesc_f16(64, 16, 1, 1), KR / 16, true);   // GEMM6b: X R_eta
      }
      mma_commit(bar_mma);
    }
    if (!mma_sync()) { aborted = true; break; }

    // ---- E4: o = num / den, staged in shared memory, then written coalesced
    {
      const int i = r16;
      uint32_t rd;
      tmem_ld1(trow + K::T_DEN, rd);   // one column of all 32 lanes: rows in lanes 0-15
      tmem_ld_wait1(rd);
      const float dn = __shfl_sync(kFull, __uint_as_float(rd), lane & 15);
      const float rdn = 1.0f / dn;
      const long long row = bh * a.N + n0 + i;
      const bool valid = i < nv;
      if (valid && a.den && part == 0 && hb == 0) a.den[row] = dn;
      constexpr int DQ = DV / 4;   // value columns per warp
      static_assert(DQ == 16 || DQ == 32, "a warp's value columns split into two halves of 8 or 16");
      constexpr int PH = DQ / 2;   // value columns per thread
      const int f0 = part * DQ + PH * hb;
      uint32_t r[PH];
      if constexpr (PH == 16) {
        tmem_ld16_halves<16>(trow + K::T_NUM + part * DQ, r);
        tmem_ld_wait16(r);
      } else {
        tmem_ld8_halves<8>(trow + K::T_NUM + part * DQ, r);
        tmem_ld_wait8(r);
      }
#pragma unroll
      for (int g = 0; g < PH / 4; ++g) {
        const int chunk = (f0 >> 2) + g;
        *reinterpret_cast<float4*>(smem + K::S_OUT + i * DV * 4 + ((chunk ^ (i & 7)) << 4)) =
            make_float4(__uint_as_float(r[4 * g]) * rdn, __uint_as_float(r[4 * g + 1]) * rdn,
                        __uint_as_float(r[4 * g + 2]) * rdn, __uint_as_float(r[4 * g + 3]) * rdn);
      }
      if (valid && a.num) {
        float4* np = reinterpret_cast<float4*>(a.num + row * DV + f0);
#pragma unroll
        for (int g = 0; g < PH / 4; ++g)
          np[g] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                              __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
      }
      __syncthreads();
      constexpr int CPR = DV / 4;  // 16-byte chunks per row
      float* obase = a.o + (bh * a.N + n0) * DV;
      for (int c = tid; c < nv * CPR; c += NT) {
        const int rr = c / CPR, g = c % CPR;
        const float4 x = *reinterpret_cast<const float4*>(smem + K::S_OUT + rr * DV * 4 + ((g ^ (rr & 7)) << 4));
        *reinterpret_cast<float4*>(obase + rr * DV + 4 * g) = x;
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted) {
    if (FULL) {
      if (a.state_out && seg == a.nseg - 1) {
        // state after the last token: sc * lambda^(nv - C) * S_hat = lambda^(nv-c-1) S_hat
        const double ex = exp((nv - C / 2 - 1) * T->re_dA[m]);
        const double ph = fmod((nv - C / 2 - 1) * T->im_dA[m], 6.283185307179586476925);
        double sn, cs;
        sincos(ph, &sn, &cs);
        const float fr = static_cast<float>(ex * cs), fi = static_cast<float>(ex * sn);
#pragma unroll
        for (int cb = 0; cb < FQ; cb += 16) {
          const int col0 = part * FQ + cb;
          uint32_t r[16];
          tmem_ld16(trow + K::T_STATE + col0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float x = __uint_as_float(r[e2]);
            const float y = __shfl_xor_sync(kFull, x, 1);
            if (comp == 0) {   // x = re, y = im
              const float2 z = make_float2(fr * x - fi * y, fr * y + fi * x);
              const int f = col0 + e2;
              if (f < DX) a.state_out[(bh * 64 + m) * DX + f] = z;
              else a.state_out[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)] = z;
            }
          }
        }
        const float y = __shfl_xor_sync(kFull, eta_c, 1);
        if (comp == 0 && part == 0)
          a.state_out[a.BH * 64 * F + bh * 64 + m] =
              make_float2(fr * eta_c - fi * y, fr * y + fi * eta_c);
      }
    } else {
      float* dst = a.seg_state + ((bh * (a.nseg - 1) + seg) * KR + k) * F;
#pragma unroll
      for (int cb = 0; cb < FQ; cb += 16) {
        const int col0 = part * FQ + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_STATE + col0, r);
        tmem_ld_wait16(r);
        float4* d4 = reinterpret_cast<float4*>(dst + col0);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          d4[g] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                              __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
      }
      if (part == 0) a.seg_eta[(bh * (a.nseg - 1) + seg) * KR + k] = eta_c;
    }
  } else if (tma_pending) {
    mbar_wait(bar_tma, ph_tma, a.err);   // bounded: let our own copy land before exiting
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Warp-specialized full pass for d_xi = d_v = 64.  tcgen05.mma issue blocks
// the issuing thread for about as long as the tensor core works, so the
// contractions are issued by a dedicated warp (warp 16, which also issues the
// bulk copies) while 16 epilogue warps do the elementwise phases.  The two
// sides hand over through mbarriers: "ready" barriers (512 epilogue-thread
// arrivals after their shared/TMEM writes) and "done" barriers (one
// tcgen05.commit).  Chunks are software-pipelined: the tail of chunk t-1
// (mask P, value contractions, output) is interleaved with the head of chunk
// t (Gram, decay contractions, readout scale), so the tensor core works on
// one chunk while the epilogue warps work on the other.  V, R_Gamma and R_eta
// are double-buffered; S, P, a~, num have their own TMEM tiles.
constexpr int WS_EW = 16;                   // epilogue warps
constexpr int WS_ET = WS_EW * 32;           // epilogue threads
constexpr int WS_NT = WS_ET + 32;           // + one MMA / copy warp

struct WCfg {
  static constexpr int DX = 64, DV = 64, F = 128, WV = 80, NV = 80;
  static constexpr uint32_t RSX = DX * 16, RSV = WV * 16;
  static constexpr uint32_t T_STATE = 0, T_A = 128, T_S = 192, T_P = 256, T_NUM = 320,
                            T_DEN = 320 + 64;
  static constexpr uint32_t STG_Q = 0;
  static constexpr uint32_t STG_K = STG_Q + C * DX * 2;
  static constexpr uint32_t STG_V = STG_K + C * DX * 2;
  static constexpr uint32_t S_Q = STG_V + C * DV * 2;
  static constexpr uint32_t S_K = S_Q + C * DX * 2;
  static constexpr uint32_t S_V0 = S_K + C * DX * 2;
  static constexpr uint32_t S_V1 = S_V0 + C * WV * 2;
  static constexpr uint32_t S_E = S_V1 + C * WV * 2;
  static constexpr uint32_t S_S = S_E + KR * C * 2;
  static constexpr uint32_t S_P = S_S + C * C * 2;
  static constexpr uint32_t S_X = S_P + C * C * 2;
  static constexpr uint32_t S_RU = S_X + KR * C * 2;
  static constexpr uint32_t S_RG0 = S_RU + KR * DX * 2;
  static constexpr uint32_t S_RG1 = S_RG0 + KR * WV * 2;
  static constexpr uint32_t S_BAR = S_RG1 + KR * WV * 2;    // 10 mbarriers
  static constexpr uint32_t S_FLAG = S_BAR + 80;
  static constexpr uint32_t S_TMEMH = S_FLAG + 16;
  static constexpr uint32_t SMEM = S_TMEMH + 16;
  static constexpr uint32_t S_OUT = S_X;   // o of chunk t-1 is staged while sX is free
  static_assert(KR * C * 2 >= C * DV * 4, "output staging fits in sX");
};

__global__ void __launch_bounds__(WS_NT, 1) tc_prefill_ws_kernel(const TcArgs a) {
  using K = WCfg;
  constexpr int DX = K::DX, DV = K::DV, F = K::F;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool mma_warp = warp == WS_EW;
  const int quad = warp & 3, part = (warp >> 2) & 3;
  const long long bh = blockIdx.x / a.nseg;
  const int seg = static_cast<int>(blockIdx.x % a.nseg);
  const int h = static_cast<int>(bh % a.H);
  const HeadTables* T = a.tabs + h;
  const int nch_total = (a.N + C - 1) / C;
  const int ch0 = seg * a.seg_chunks;
  const int ch1 = min(ch0 + a.seg_chunks, nch_total);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* bar_tma = bars + 0;
  uint64_t* rdy = bars + 1;     // rdy[0..3]: ready for G1+G7, G2+G3, G4, G5+G6
  uint64_t* dne = bars + 5;     // dne[0..3]: done   "
  uint64_t* bar_drain = bars + 9;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + K::S_TMEMH);
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(rdy + i, WS_ET);
      mbar_init(dne + i, 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    const uint4* src = reinterpret_cast<const uint4*>(T->E);
    uint4* dst = reinterpret_cast<uint4*>(smem + K::S_E);
    for (int i = tid; i < KR * C * 2 / 16; i += WS_NT) dst[i] = src[i];
    // V's extra column DV is 1 (den = P 1); R_Gamma's extra columns start at 0
    for (int r = tid; r < C; r += WS_NT) {
      for (int p = 0; p < 2; ++p) {
        const uint32_t sv = p ? K::S_V1 : K::S_V0;
        *reinterpret_cast<uint4*>(smem + sv + tile_off(r, DV, K::RSV)) = make_uint4(0x00003C00u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + sv + tile_off(r, DV + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    for (int r = tid; r < KR; r += WS_NT) {
      for (int p = 0; p < 2; ++p) {
        const uint32_t sr = p ? K::S_RG1 : K::S_RG0;
        *reinterpret_cast<uint4*>(smem + sr + tile_off(r, DV, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + sr + tile_off(r, DV + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (mma_warp) {
    // ------------------------------------------------ MMA and copy issuer
    if (lane == 0) {
      uint32_t pr[4] = {0u, 0u, 0u, 0u};
      int issued = 0;
      bool ok = true;
      auto issue_load = [&](int ch) {
        const int n0 = ch * C;
        const int nv = min(C, a.N - n0);
        const uint32_t bq = static_cast<uint32_t>(nv * DX * 2), bv = static_cast<uint32_t>(nv * DV * 2);
        mbar_arrive_expect_tx(bar_tma, 2 * bq + bv);
        const long long row = bh * a.N + n0;
        bulk_g2s(smem + K::STG_Q, a.q + row * DX, bq, bar_tma);
        bulk_g2s(smem + K::STG_K, a.k + row * DX, bq, bar_tma);
        bulk_g2s(smem + K::STG_V, a.v + row * DV, bv, bar_tma);
        ++issued;
      };
      auto wait_rdy = [&](int i) -> bool {
        const bool r = mbar_wait_or_abort(rdy + i, pr[i], a.err, abort_flag);
        pr[i] ^= 1u;
        tc_fence_after();
        return r;
      };
      auto g5g6 = [&](int pp) {
        const uint32_t sv = sbase + (pp ? K::S_V1 : K::S_V0), srg = sbase + (pp ? K::S_RG1 : K::S_RG0);
        gemm(tmem + K::T_NUM, sbase + K::S_P, 128, 1024, 256, sv, K::RSV, 128, 2 * K::RSV,
             idesc_f16(64, K::NV, 0, 1), C / 16, false);   // G5: P [V | 1]
        gemm(tmem + K::T_NUM, sbase + K::S_X, 1024, 128, 2048, srg, K::RSV, 128, 2 * K::RSV,
             idesc_f16(64, K::NV, 1, 1), KR / 16, true);   // G6: X [R_Gamma | R_eta]
        mma_commit(dne + 3);
      };
      if (ch0 < ch1) issue_load(ch0);
      for (int t = ch0; t < ch1; ++t) {
        const int p = (t - ch0) & 1;
        if (!(ok = wait_rdy(0))) break;
        if (t + 1 < ch1) issue_load(t + 1);   // staging was consumed before ready(0)
        const uint32_t sv = sbase + (p ? K::S_V1 : K::S_V0);
        gemm(tmem + K::T_S, sbase + K::S_K, 128, K::RSX, 256, sbase + K::S_Q, 128, K::RSX, 256,
             idesc_f16(64, 64, 0, 0), DX / 16, false);   // G1: S^T
        gemm(tmem + K::T_STATE, sbase + K::S_E, 128, 1024, 256, sbase + K::S_K, K::RSX, 128,
             2 * K::RSX, idesc_f16(128, DX, 0, 1), C / 16, true);   // G7: U carry
        gemm(tmem + K::T_STATE + DX, sbase + K::S_E, 128, 1024, 256, sv, K::RSV, 128, 2 * K::RSV,
             idesc_f16(128, DV, 0, 1), C / 16, true);   // G7: Gamma carry
        mma_commit(dne + 0);
        if (t > ch0) {
          if (!(ok = wait_rdy(3))) break;
          g5g6(p ^ 1);
        }
        if (!(ok = wait_rdy(1))) break;
        gemm(tmem + K::T_A, sbase + K::S_E, 128, 1024, 256, sbase + K::S_S, 1024, 128, 2048,
             idesc_f16(128, 64, 0, 1), C / 16, false);   // G2
        gemm(tmem + K::T_A, sbase + K::S_RU, 128, K::RSX, 256, sbase + K::S_Q, 128, K::RSX, 256,
             idesc_f16(128, 64, 0, 0), DX / 16, true);   // G3
        mma_commit(dne + 1);
        if (!(ok = wait_rdy(2))) break;
        gemm(tmem + K::T_P, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
             idesc_f16(64, 64, 1, 1), KR / 16, false);   // G4: P
        mma_commit(dne + 2);
      }
      if (ok && ch0 < ch1) {
        if ((ok = wait_rdy(3))) g5g6((ch1 - 1 - ch0) & 1);
      }
      if (!ok) {
        // drain: every tensor-core group issued so far, and the last copy
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0u, a.err);
        if (issued > 0) mbar_wait(bar_tma, static_cast<uint32_t>((issued - 1) & 1), a.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue warps
    const int k = 32 * quad + lane;
    const int m = k >> 1, comp = k & 1;
    const float2 lamC = T->lamC[m];
    const float sgnLi = comp ? lamC.y : -lamC.y;
    const float r2 = T->r2[m];
    const float s_start = static_cast<float>(exp(2.0 * T->re_dA[m] * (16.0 * part - C / 2)));
    const float esum_c = comp ? T->esum[m].y : T->esum[m].x;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    constexpr int FQ = F / 4;
    const int i0 = 16 * part;
    uint32_t pd[4] = {0u, 0u, 0u, 0u};
    uint32_t ptma = 0u;
    auto wait_dne = [&](int i) -> bool {   // outcome made uniform across the epilogue warps
      const bool r = mbar_wait_or_abort(dne + i, pd[i], a.err, abort_flag);
      pd[i] ^= 1u;
      tc_fence_after();
      return !named_sync_or(2, WS_ET, !r);
    };
    auto signal = [&](int i) {   // my shared / TMEM writes are done: ready(i)
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(rdy + i);
    };

    float eta_c = 0.f;
    {  // initial (scaled) state
      const float* carry = nullptr;
      const float* carry_eta = nullptr;
      if (seg > 0) {
        carry = a.seg_state + ((bh * (a.nseg - 1) + (seg - 1)) * KR + k) * F;
        carry_eta = a.seg_eta + (bh * (a.nseg - 1) + (seg - 1)) * KR + k;
      }
      const bool from_in = seg == 0 && a.state_in != nullptr;
      const float2 si = T->sc_inv[m];
#pragma unroll
      for (int cb = 0; cb < FQ; cb += 16) {
        const int col0 = part * FQ + cb;
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float val = 0.f;
          const int f = col0 + e;
          if (carry) {
            val = carry[f];
          } else if (from_in) {
            float2 x = f < DX ? a.state_in[(bh * 64 + m) * DX + f]
                              : a.state_in[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)];
            val = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
          }
          r[e] = __float_as_uint(val);
        }
        tmem_st16(trow + K::T_STATE + col0, r);
      }
      if (carry_eta) {
        eta_c = *carry_eta;
      } else if (from_in) {
        float2 x = a.state_in[a.BH * 64 * F + bh * 64 + m];
        eta_c = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
      }
      tmem_st_wait();
    }

    int nv_last = C;
    // chunk ch, buffer parity p: convert inputs, rotate the state, signal ready(0)
    auto prepare = [&](int ch, int p) -> bool {
      const int nv = min(C, a.N - ch * C);
      nv_last = nv;
      const bool r = mbar_wait_or_abort(bar_tma, ptma, a.err, abort_flag);
      ptma ^= 1u;
      if (named_sync_or(2, WS_ET, !r)) return false;
      const uint32_t sv = p ? K::S_V1 : K::S_V0, srg = p ? K::S_RG1 : K::S_RG0;
      convert_all<DX, DX, true>(smem + K::STG_Q, smem + K::S_Q, nv, warp, lane);
      convert_all<DX, DX, true>(smem + K::STG_K, smem + K::S_K, nv, warp, lane);
      convert_all<DV, K::WV, false>(smem + K::STG_V, smem + sv, nv, warp, lane);
      static_assert(FQ == 32, "two 16-column blocks per thread");
      uint32_t rs[2][16];
      tmem_ld16(trow + K::T_STATE + part * FQ, rs[0]);
      tmem_ld16(trow + K::T_STATE + part * FQ + 16, rs[1]);
      tmem_ld_wait16(rs[0]);
      tmem_ld_wait16(rs[1]);
#pragma unroll
      for (int cb = 0; cb < FQ; cb += 16) {
        const int col0 = part * FQ + cb;
        uint32_t (&rr)[16] = rs[cb / 16];
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x = __uint_as_float(rr[e]);
          const float y = __shfl_xor_sync(kFull, x, 1);
          w[e] = __float_as_uint(fmaf(lamC.x, x, sgnLi * y));
        }
        tmem_st16(trow + K::T_STATE + col0, w);
        if (a.dump_R) dump_r16(a.dump_R, bh * nch_total + ch, k, col0, w);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint4 pk = pack8f(w + 8 * g, 1.f);
          const int f = col0 + 8 * g;
          if (f < DX)
            *reinterpret_cast<uint4*>(smem + K::S_RU + tile_off(k, f, K::RSX)) = pk;
          else
            *reinterpret_cast<uint4*>(smem + srg + tile_off(k, f - DX, K::RSV)) = pk;
        }
      }
      tmem_st_wait();
      {
        const float y = __shfl_xor_sync(kFull, eta_c, 1);
        const float Re = fmaf(lamC.x, eta_c, sgnLi * y);
        if (part == 0) {
          if (a.dump_Re) a.dump_Re[(bh * nch_total + ch) * KR + k] = Re;
          *reinterpret_cast<uint4*>(smem + srg + tile_off(k, DV, K::RSV)) =
              make_uint4(pack_half2(Re, 0.f), 0u, 0u, 0u);
        }
        float add = esum_c;
        if (nv < C) {
          double sr = 0.0, si = 0.0;
          const double br = T->b[m].x, bi = T->b[m].y;
          for (int j = 0; j < nv; ++j) {
            const double e = exp((C / 2 - j) * T->re_dA[m]);
            const double ph = fmod((C / 2 - j) * T->im_dA[m], 6.283185307179586476925);
            double sn, cs;
            sincos(ph, &sn, &cs);
            const double pr = e * cs, pi = e * sn;
            sr += br * pr - bi * pi;
            si += br * pi + bi * pr;
          }
          add = static_cast<float>(comp ? si : sr);
        }
        eta_c = Re + add;
      }
      signal(0);
      return true;
    };
    auto e3 = [&]() {   // masked P -> [i][j]
      const int i = 16 * quad + lane;
      uint32_t r[16];
      tmem_ld16(trow + K::T_P + i0, r);
      tmem_ld_wait16(r);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (i0 + e > i) r[e] = 0u;
        *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(i, i0, 1024)) = pack8f(r, 1.f);
        *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(i, i0 + 8, 1024)) = pack8f(r + 8, 1.f);
      }
      signal(3);
    };
    auto e4 = [&](int ch, int nv) {   // o = num / den, staged then written coalesced
      const int n0 = ch * C;
      const int i = 16 * quad + lane;
      uint32_t rd[16], r[16];
      tmem_ld16(trow + K::T_DEN, rd);
      tmem_ld16(trow + K::T_NUM + i0, r);
      tmem_ld_wait16(rd);
      tmem_ld_wait16(r);
      const float dn = __uint_as_float(rd[0]);
      const float rdn = 1.0f / dn;
      const long long row = bh * a.N + n0 + i;
      if (lane < 16) {
        if (i < nv && a.den && part == 0) a.den[row] = dn;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int chunk = (i0 >> 2) + g;
          *reinterpret_cast<float4*>(smem + K::S_OUT + i * DV * 4 + ((chunk ^ (i & 7)) << 4)) =
              make_float4(__uint_as_float(r[4 * g]) * rdn, __uint_as_float(r[4 * g + 1]) * rdn,
                          __uint_as_float(r[4 * g + 2]) * rdn, __uint_as_float(r[4 * g + 3]) * rdn);
        }
        if (i < nv && a.num) {
          float4* np = reinterpret_cast<float4*>(a.num + row * DV + i0);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            np[g] = make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
        }
      }
      named_sync(1, WS_ET);
      constexpr int CPR = DV / 4;
      float* obase = a.o + (bh * a.N + n0) * DV;
      for (int c = tid; c < nv * CPR; c += WS_ET) {
        const int rr = c / CPR, g = c % CPR;
        const float4 x = *reinterpret_cast<const float4*>(smem + K::S_OUT + rr * DV * 4 + ((g ^ (rr & 7)) << 4));
        *reinterpret_cast<float4*>(obase + rr * DV + 4 * g) = x;
      }
      named_sync(1, WS_ET);   // staging (sX) is read before E2 of the next chunk writes it
    };

    bool ok = true;
    int prev = -1, prev_nv = C;
    if (ch0 < ch1) ok = prepare(ch0, 0);
    for (int t = ch0; ok && t < ch1; ++t) {
      const int nv = min(C, a.N - t * C);
      if (prev >= 0) {
        if (!(ok = wait_dne(2))) break;   // G4(t-1)
        e3();
      }
      if (!(ok = wait_dne(0))) break;     // G1 + G7(t)
      {  // E1(t): masked S^T -> [j][i]
        const int j = 16 * quad + lane;
        uint32_t r[16];
        tmem_ld16(trow + K::T_S + i0, r);
        tmem_ld_wait16(r);
        if (lane < 16) {
          const bool keep = j < nv;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (!(keep && i0 + e >= j)) r[e] = 0u;
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, i0, 1024)) = pack8f(r, 1.f);
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, i0 + 8, 1024)) = pack8f(r + 8, 1.f);
        }
        signal(1);
      }
      if (prev >= 0) {
        if (!(ok = wait_dne(3))) break;   // G5 + G6(t-1)
        e4(prev, prev_nv);
      }
      if (!(ok = wait_dne(1))) break;     // G2 + G3(t)
      {  // E2(t): X = |lambda|^(2(i-c)) a~
        uint32_t r[16];
        tmem_ld16(trow + K::T_A + i0, r);
        tmem_ld_wait16(r);
        float s = s_start;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          r[e] = __float_as_uint(__uint_as_float(r[e]) * s);
          s *= r2;
        }
        *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0, 1024)) = pack8f(r, 1.f);
        *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 8, 1024)) = pack8f(r + 8, 1.f);
        signal(2);
      }
      prev = t;
      prev_nv = nv;
      if (t + 1 < ch1) ok = prepare(t + 1, (t + 1 - ch0) & 1);
    }
    if (ok && prev >= 0) {
      if ((ok = wait_dne(2))) e3();
      if (ok && (ok = wait_dne(3))) e4(prev, prev_nv);
    }
    if (ok && a.state_out && seg == a.nseg - 1) {
      const int nv = nv_last;
      const double ex = exp((nv - C / 2 - 1) * T->re_dA[m]);
      const double ph = fmod((nv - C / 2 - 1) * T->im_dA[m], 6.283185307179586476925);
      double sn, cs;
      sincos(ph, &sn, &cs);
      const float fr = static_cast<float>(ex * cs), fi = static_cast<float>(ex * sn);
#pragma unroll
      for (int cb = 0; cb < FQ; cb += 16) {
        const int col0 = part * FQ + cb;
        uint32_t r[16];
        tmem_ld16(trow + K::T_STATE + col0, r);
        tmem_ld_wait16(r);
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const float x = __uint_as_float(r[e2]);
          const float y = __shfl_xor_sync(kFull, x, 1);
          if (comp == 0) {
            const float2 z = make_float2(fr * x - fi * y, fr * y + fi * x);
            const int f = col0 + e2;
            if (f < DX) a.state_out[(bh * 64 + m) * DX + f] = z;
            else a.state_out[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)] = z;
          }
        }
      }
      const float y = __shfl_xor_sync(kFull, eta_c, 1);
      if (comp == 0 && part == 0)
        a.state_out[a.BH * 64 * F + bh * 64 + m] = make_float2(fr * eta_c - fi * y, fr * y + fi * eta_c);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Two-group warp-specialized full pass for d_xi = d_v = 64.  Four roles run
// concurrently: 8 "prepare" warps (0-7) convert the inputs and rotate the
// carried state into R(t); 8 "output" warps (8-15) run the masks, readout
// scale and o = num/den of chunks t and t-1; warp 16 issues every
// tensor-core contraction; warp 17 brings q, k, v in with TMA tensor loads
// that land directly in the operand layout, where the prepare warps convert
// them in place, so there is no staging area.  A 64-row box arrives as 64
// rows of 128 bytes in the 128-byte swizzled layout, which the tensor core
// reads as a K-major (features along K) or an MN-major (tokens along K)
// operand alike.  Rows past the sequence arrive as zeros.
// R_U, the A operand of G3, is written to tensor memory as fp16 pairs, and o
// leaves through TMA tensor stores from a double-buffered staging area, so
// neither waits on the other side.  q, k, v and R_Gamma have three buffer sets and
// R_U two: the fetch warp refills a set as soon as the contractions of the
// chunk it held are done, about two chunks ahead of its use.  Handover is by
// mbarriers: loaded(set) from the copies, ready(0) from the prepare warps,
// ready(1..3) from the output warps, done(0..3) and the buffer releases
// (freeQK after G2+G3, freeVR after G5+G6) from tcgen05.commit.
constexpr int W2_GW = 8;                       // warps per epilogue group
constexpr int W2_GT = W2_GW * 32;              // threads per epilogue group
constexpr int W2_NT = 2 * W2_GT + 64;          // + the MMA warp and the fetch warp

struct W2Cfg {
  static constexpr int DX = 64, DV = 64, F = 128, WV = 80, NV = 80;
  static constexpr uint32_t RSV = WV * 16;
  static constexpr uint32_t T_STATE = 0, T_A = 128, T_S = 192, T_P = 256, T_NUM = 320,
                            T_DEN = 320 + 64, T_RU = 400;   // T_RU: [2] x 32 columns of fp16 pairs
  static constexpr uint32_t TQ = C * DX * 2, TV = C * DV * 2, TRG = KR * WV * 2;
  static constexpr uint32_t TO = C * DV * 4;               // o of one chunk: two 64 x 128-byte boxes
  static constexpr int NB = 3;                             // q, k, v and R_Gamma buffer sets
  static constexpr uint32_t TIN = C * 64 * 2;              // bytes of one TMA box (64 rows x 64 bf16)
  static constexpr uint32_t SW = 1024;                     // one swizzle atom: 8 rows x 128 bytes
  static constexpr uint32_t S_Q = 0;                       // [NB]
  static constexpr uint32_t S_K = S_Q + NB * TQ;           // [NB]
  static constexpr uint32_t S_V = S_K + NB * TQ;           // [NB]
  static constexpr uint32_t S_ONES = S_V + NB * TV;        // [V | 1]: MN-block 64..127 of G5's B operand
  static constexpr uint32_t S_E = S_ONES + TV;
  static constexpr uint32_t S_S = S_E + KR * C * 2;
  static constexpr uint32_t S_P = S_S + C * C * 2;
  static constexpr uint32_t S_X = S_P + C * C * 2;
  static constexpr uint32_t S_O = S_X + KR * C * 2;        // [2] o staging, 128-byte swizzled
  static constexpr uint32_t S_RG = S_O + 2 * TO;           // [NB]
  static constexpr uint32_t S_BAR = S_RG + NB * TRG;       // 18 mbarriers
  static constexpr uint32_t S_FLAG = S_BAR + 256;
  static constexpr uint32_t S_TMEMH = S_FLAG + 16;
  static constexpr uint32_t SMEM = S_TMEMH + 16;
  static_assert(SMEM <= 232448, "fits one CTA's opt-in shared memory");
  static_assert(S_O % 1024 == 0 && S_K % 1024 == 0 && S_V % 1024 == 0 && S_ONES % 1024 == 0,
                "swizzled tiles start on the 128-byte swizzle period");
};

__global__ void __launch_bounds__(W2_NT, 1)
    tc_prefill_ws2_kernel(const __grid_constant__ TcArgs a, const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o) {
  using K = W2Cfg;
  constexpr int DX = K::DX, DV = K::DV, F = K::F, NB = K::NB;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int role = warp < 2 * W2_GW ? warp / W2_GW : warp - 2 * W2_GW + 2;   // prepare, output, mma, fetch
  const int gw = warp & (W2_GW - 1);          // warp index within its epilogue group
  const int quad = warp & 3, half = gw >> 2;
  const long long bh = blockIdx.x / a.nseg;
  const int seg = static_cast<int>(blockIdx.x % a.nseg);
  const int h = static_cast<int>(bh % a.H);
  const HeadTables* T = a.tabs + h;
  const int nch_total = (a.N + C - 1) / C;
  const int ch0 = seg * a.seg_chunks;
  const int ch1 = min(ch0 + a.seg_chunks, nch_total);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::S_BAR);
  uint64_t* rdy = bars + 0;       // [4]
  uint64_t* dne = bars + 4;       // [4]
  uint64_t* freeQK = bars + 8;    // [NB]: sQ, sK of that set (and the sR_U it was read with) reusable
  uint64_t* freeVR = bars + 11;   // [NB]: sV, sR_Gamma of that set reusable
  uint64_t* bar_drain = bars + 14;
  uint64_t* loaded = bars + 15;   // [NB]: that set's q, k, v rows have landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::S_FLAG);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + K::S_TMEMH);
  const uint32_t sbase = smem_u32(smem);
  auto sQ = [&](int b) { return K::S_Q + b * K::TQ; };
  auto sK = [&](int b) { return K::S_K + b * K::TQ; };
  auto sV = [&](int b) { return K::S_V + b * K::TV; };
  auto sRG = [&](int b) { return K::S_RG + b * K::TRG; };

  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(rdy + i, W2_GT);
      mbar_init(dne + i, 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(freeQK + i, 1);
      mbar_init(freeVR + i, 1);
      mbar_init(loaded + i, 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    // V's extra column DV is 1 (den = P 1); R_Gamma's extra columns start at 0
    // the ones column after V: MN element 64 (first of the second 64-block)
    // is 1 in every row, the rest 0, in the swizzled layout
    for (int i = tid; i < C * 8; i += W2_NT) {
      const int r = i >> 3, c = i & 7;
      *reinterpret_cast<uint4*>(smem + K::S_ONES + r * 128 + c * 16) =
          make_uint4((c == (r & 7)) ? 0x00003C00u : 0u, 0u, 0u, 0u);
    }
    for (int r = tid; r < KR; r += W2_NT) {
      for (int b = 0; b < NB; ++b) {
        *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(r, DV, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(r, DV + 8, K::RSV)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // Everything above touches only this CTA's own resources.  The kernel may
    // have been launched while the previous kernel of the stream (the table
    // prologue, or the segment carry scan) still runs: every global read of
    // the tables, carries and inputs comes after this wait, and nothing global
    // is written before it.
    griddep_wait();
    const uint4* src = reinterpret_cast<const uint4*>(T->E);
    uint4* dst = reinterpret_cast<uint4*>(smem + K::S_E);
    for (int i = tid; i < KR * C * 2 / 16; i += W2_NT) dst[i] = src[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (role == 2) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t pr[4] = {0u, 0u, 0u, 0u};
      bool ok = true;
      auto wait_rdy = [&](int i) -> bool {
        const bool r = mbar_wait_or_abort(rdy + i, pr[i], a.err, abort_flag);
        pr[i] ^= 1u;
        tc_fence_after();
        return r;
      };
      // contraction over ksteps K-steps of 16 with prebuilt descriptors; the
      // start addresses advance by astep / bstep bytes per step
      auto gemm_d = [&](uint32_t d, uint64_t ad, uint32_t astep, uint64_t bd, uint32_t bstep, uint32_t idesc,
                        int ksteps, bool acc) {
        for (int kk = 0; kk < ksteps; ++kk)
          mma_f16(d, ad + ((kk * astep) >> 4), bd + ((kk * bstep) >> 4), idesc, (kk > 0 || acc) ? 1u : 0u);
      };
      auto g5g6 = [&](int bb) {
        gemm_d(tmem + K::T_NUM, smem_desc(sbase + K::S_P, 128, 1024), 256,
               smem_desc_sw128(sbase + sV(bb), K::S_ONES - sV(bb), K::SW), 2 * K::SW,
               idesc_f16(64, K::NV, 0, 1), C / 16, false);   // G5: P [V | 1]
        gemm(tmem + K::T_NUM, sbase + K::S_X, 1024, 128, 2048, sbase + sRG(bb), K::RSV, 128, 2 * K::RSV,
             idesc_f16(64, K::NV, 1, 1), KR / 16, true);   // G6: X [R_Gamma | R_eta]
        mma_commit(dne + 3);
        mma_commit(freeVR + bb);
      };
      for (int t = ch0; t < ch1; ++t) {
        const int rel = t - ch0, b = rel % NB, p = rel & 1;
        if (!(ok = wait_rdy(0))) break;
        gemm_d(tmem + K::T_S, smem_desc_sw128(sbase + sK(b), 16, K::SW), 32,
               smem_desc_sw128(sbase + sQ(b), 16, K::SW), 32, idesc_f16(64, 64, 0, 0), DX / 16,
               false);   // G1: S^T
        gemm_d(tmem + K::T_STATE, smem_desc(sbase + K::S_E, 128, 1024), 256,
               smem_desc_sw128(sbase + sK(b), K::TQ, K::SW), 2 * K::SW, idesc_f16(128, DX, 0, 1), C / 16,
               true);   // G7: U carry
        gemm_d(tmem + K::T_STATE + DX, smem_desc(sbase + K::S_E, 128, 1024), 256,
               smem_desc_sw128(sbase + sV(b), K::S_ONES - sV(b), K::SW), 2 * K::SW, idesc_f16(128, DV, 0, 1),
               C / 16, true);   // G7: Gamma carry
        mma_commit(dne + 0);
        if (t > ch0) {
          if (!(ok = wait_rdy(3))) break;
          g5g6((rel + NB - 1) % NB);
        }
        if (!(ok = wait_rdy(1))) break;
        gemm(tmem + K::T_A, sbase + K::S_E, 128, 1024, 256, sbase + K::S_S, 1024, 128, 2048,
             idesc_f16(128, 64, 0, 1), C / 16, false);   // G2
        for (int kk = 0; kk < DX / 16; ++kk)   // G3: A = R_U from tensor memory
          mma_f16_ts(tmem + K::T_A, tmem + K::T_RU + 32 * p + 8 * kk,
                     smem_desc_sw128(sbase + sQ(b) + 32 * kk, 16, K::SW), idesc_f16(128, 64, 0, 0), 1u);
        mma_commit(dne + 1);
        mma_commit(freeQK + b);
        if (!(ok = wait_rdy(2))) break;
        gemm(tmem + K::T_P, sbase + K::S_X, 1024, 128, 2048, sbase + K::S_E, 1024, 128, 2048,
             idesc_f16(64, 64, 1, 1), KR / 16, false);   // G4: P
        mma_commit(dne + 2);
      }
      if (ok && ch0 < ch1) {
        if ((ok = wait_rdy(3))) g5g6((ch1 - 1 - ch0) % NB);
      }
      if (!ok) {   // drain every tensor-core group issued so far
        mma_commit(bar_drain);
        mbar_wait(bar_drain, 0u, a.err);
      }
    }
    __syncwarp();
  } else if (role == 0) {
    // ------------------------------------------------ prepare warps
    const int k = 32 * quad + lane;
    const int m = k >> 1, comp = k & 1;
    const float2 lamC = T->lamC[m];
    const float sgnLi = comp ? lamC.y : -lamC.y;
    const uint64_t lamC2 = f2_pack(lamC.x, lamC.x), sgnLi2 = f2_pack(sgnLi, sgnLi);
    const float esum_c = comp ? T->esum[m].y : T->esum[m].x;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    constexpr int FH = F / 2;   // state columns per thread
    uint32_t pd0 = 0u, pld[NB] = {0u, 0u, 0u};
    auto waitA = [&](uint64_t* bar, uint32_t& ph) -> bool {   // uniform over the prepare group
      const bool r = mbar_wait_or_abort(bar, ph, a.err, abort_flag);
      ph ^= 1u;
      tc_fence_after();
      return !named_sync_or(2, W2_GT, !r);
    };
    // 16-byte pieces of a 64 x 64 input tile in address order (piece =
    // row * 8 + slot); the map is elementwise, so the swizzle does not matter
    auto piece = [](int pc, int& r, int& slot) {
      r = pc >> 3;
      slot = pc & 7;
    };
    // bf16 -> fp16 in place (q, k through the feature map); rows past the
    // sequence become 0
    auto convert = [&](int nv, int b) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        int r, slot;
        piece(tid + u * W2_GT, r, slot);   // this thread converts pieces tid, tid + 256
        const uint32_t off = r * 128 + slot * 16;
        uint4* ptr[3] = {reinterpret_cast<uint4*>(smem + sQ(b) + off),
                         reinterpret_cast<uint4*>(smem + sK(b) + off),
                         reinterpret_cast<uint4*>(smem + sV(b) + off)};
        uint4 in[3] = {*ptr[0], *ptr[1], *ptr[2]};
#pragma unroll
        for (int tsel = 0; tsel < 3; ++tsel) {
          uint4 out = make_uint4(0u, 0u, 0u, 0u);
          if (r < nv) {
            const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&in[tsel]);
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(x2[e]);
              w[e] = tsel < 2 ? feat_h2(f.x, f.y) : pack_half2(f.x, f.y);
            }
            out = make_uint4(w[0], w[1], w[2], w[3]);
          }
          *ptr[tsel] = out;
        }
      }
    };
    float eta_c = 0.f;
    {  // initial (scaled) state
      const float* carry = nullptr;
      const float* carry_eta = nullptr;
      if (seg > 0) {
        carry = a.seg_state + ((bh * (a.nseg - 1) + (seg - 1)) * KR + k) * F;
        carry_eta = a.seg_eta + (bh * (a.nseg - 1) + (seg - 1)) * KR + k;
      }
      const bool from_in = seg == 0 && a.state_in != nullptr;
      const float2 si = T->sc_inv[m];
#pragma unroll
      for (int cb = 0; cb < FH; cb += 16) {
        const int col0 = half * FH + cb;
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float val = 0.f;
          const int f = col0 + e;
          if (carry) {
            val = carry[f];
          } else if (from_in) {
            float2 x = f < DX ? a.state_in[(bh * 64 + m) * DX + f]
                              : a.state_in[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)];
            val = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
          }
          r[e] = __float_as_uint(val);
        }
        tmem_st16(trow + K::T_STATE + col0, r);
      }
      if (carry_eta) {
        eta_c = *carry_eta;
      } else if (from_in) {
        float2 x = a.state_in[a.BH * 64 * F + bh * 64 + m];
        eta_c = comp ? fmaf(si.x, x.y, si.y * x.x) : fmaf(si.x, x.x, -si.y * x.y);
      }
      tmem_st_wait();
    }
    bool ok = true;
    int nv_last = C;
    for (int t = ch0; t < ch1; ++t) {
      const int rel = t - ch0, b = rel % NB, p = rel & 1;
      const int nv = min(C, a.N - t * C);
      nv_last = nv;
      if (!(ok = waitA(loaded + b, pld[b]))) break;
      convert(nv, b);
      if (rel >= 1 && !(ok = waitA(dne + 0, pd0))) break;   // G7(t-1): the state is current
      uint32_t ru[16];
#pragma unroll
      for (int blk = 0; blk < FH / 16; ++blk) {
        const int col0 = half * FH + 16 * blk;
        uint32_t rs[16], w[16];
        tmem_ld16(trow + K::T_STATE + col0, rs);
        tmem_ld_wait16(rs);
#pragma unroll
        for (int e = 0; e < 16; e += 2) {   // w = Re/Im of lambda^C times the partner row, two columns at once
          const float x0 = __uint_as_float(rs[e]), x1 = __uint_as_float(rs[e + 1]);
          const uint64_t y = f2_pack(__shfl_xor_sync(kFull, x0, 1), __shfl_xor_sync(kFull, x1, 1));
          float w0, w1;
          f2_unpack(f2_fma(lamC2, f2_pack(x0, x1), f2_mul(sgnLi2, y)), w0, w1);
          w[e] = __float_as_uint(w0);
          w[e + 1] = __float_as_uint(w1);
        }
        tmem_st16(trow + K::T_STATE + col0, w);
        if (a.dump_R) dump_r16(a.dump_R, bh * nch_total + t, k, col0, w);
        if (half == 0) {   // R_U: fp16 pairs into tensor memory, 16 columns per two blocks
#pragma unroll
          for (int e = 0; e < 8; ++e)
            ru[(blk & 1) * 8 + e] = pack_half2(__uint_as_float(w[2 * e]), __uint_as_float(w[2 * e + 1]));
          if (blk & 1) tmem_st16(trow + K::T_RU + 32 * p + 16 * (blk >> 1), ru);
        } else {           // R_Gamma: shared memory, B operand of G6
#pragma unroll
          for (int g = 0; g < 2; ++g)
            *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(k, col0 - DX + 8 * g, K::RSV)) =
                pack8f(w + 8 * g, 1.f);
        }
      }
      tmem_st_wait();
      {
        const float y = __shfl_xor_sync(kFull, eta_c, 1);
        const float Re = fmaf(lamC.x, eta_c, sgnLi * y);
        if (half == 0) {
          if (a.dump_Re) a.dump_Re[(bh * nch_total + t) * KR + k] = Re;
          *reinterpret_cast<uint4*>(smem + sRG(b) + tile_off(k, DV, K::RSV)) =
              make_uint4(pack_half2(Re, 0.f), 0u, 0u, 0u);
        }
        float add = esum_c;
        if (nv < C) {
          double sr = 0.0, si = 0.0;
          const double br = T->b[m].x, bi = T->b[m].y;
          for (int j = 0; j < nv; ++j) {
            const double e = exp((C / 2 - j) * T->re_dA[m]);
            const double ph = fmod((C / 2 - j) * T->im_dA[m], 6.283185307179586476925);
            double sn, cs;
            sincos(ph, &sn, &cs);
            const double pr = e * cs, pi = e * sn;
            sr += br * pr - bi * pi;
            si += br * pi + bi * pr;
          }
          add = static_cast<float>(comp ? si : sr);
        }
        eta_c = Re + add;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(rdy + 0);
    }
    if (ok && ch0 < ch1 && a.state_out && seg == a.nseg - 1) {
      ok = waitA(dne + 0, pd0);   // G7 of the last chunk
      if (ok) {
        const int nv = nv_last;
        const double ex = exp((nv - C / 2 - 1) * T->re_dA[m]);
        const double ph = fmod((nv - C / 2 - 1) * T->im_dA[m], 6.283185307179586476925);
        double sn, cs;
        sincos(ph, &sn, &cs);
        const float fr = static_cast<float>(ex * cs), fi = static_cast<float>(ex * sn);
#pragma unroll
        for (int cb = 0; cb < FH; cb += 16) {
          const int col0 = half * FH + cb;
          uint32_t r[16];
          tmem_ld16(trow + K::T_STATE + col0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float x = __uint_as_float(r[e2]);
            const float y = __shfl_xor_sync(kFull, x, 1);
            if (comp == 0) {
              const float2 z = make_float2(fr * x - fi * y, fr * y + fi * x);
              const int f = col0 + e2;
              if (f < DX) a.state_out[(bh * 64 + m) * DX + f] = z;
              else a.state_out[a.BH * 64 * DX + (bh * 64 + m) * DV + (f - DX)] = z;
            }
          }
        }
        const float y = __shfl_xor_sync(kFull, eta_c, 1);
        if (comp == 0 && half == 0)
          a.state_out[a.BH * 64 * F + bh * 64 + m] = make_float2(fr * eta_c - fi * y, fr * y + fi * eta_c);
      }
    }
  } else if (role == 1) {
    // ------------------------------------------------ output warps
    const int k = 32 * quad + lane;
    const int m = k >> 1;
    const float r2 = T->r2[m];
    const float s_start = static_cast<float>(exp(2.0 * T->re_dA[m] * (32.0 * half - C / 2)));
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    const int i0 = 32 * half;     // this thread's 32 columns of the 64-wide tiles
    uint32_t pd[4] = {0u, 0u, 0u, 0u};
    auto waitB = [&](int i) -> bool {
      const bool r = mbar_wait_or_abort(dne + i, pd[i], a.err, abort_flag);
      pd[i] ^= 1u;
      tc_fence_after();
      return !named_sync_or(3, W2_GT, !r);
    };
    auto signalB = [&](int i) {
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(rdy + i);
    };
    // The M = 64 accumulators (S^T, P, num) fill lanes 0-15 of each quadrant:
    // thread t takes row 16 * quad + t % 16 and columns c0 .. c0 + 15 of the
    // warp's 32, the two half-warps splitting them.
    const int r16 = 16 * quad + (lane & 15);
    const int c0 = i0 + 16 * (lane >> 4);
    auto e3 = [&]() {   // masked P -> [i][j]
      uint32_t r[16];
      tmem_ld16_halves<16>(trow + K::T_P + i0, r);
      tmem_ld_wait16(r);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c0 + e > r16) r[e] = 0u;
      *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(r16, c0, 1024)) = pack8f(r, 1.f);
      *reinterpret_cast<uint4*>(smem + K::S_P + tile_off(r16, c0 + 8, 1024)) = pack8f(r + 8, 1.f);
      signalB(3);
    };
    // o = num / den, staged as two boxes of 64 rows x 128 bytes (columns 0-31
    // and 32-63) in the 128-byte swizzled layout, which keeps the row-per-lane
    // writes free of bank conflicts, then written by one TMA store per box.
    // Rows past the sequence lie outside the tensor map and are not written.
    // Staging alternates between two buffers.  Before the barrier that
    // precedes each store, the issuing thread waits until the store before it
    // has finished reading its buffer; every thread passes that barrier before
    // it writes that buffer again one chunk later.
    auto e4 = [&](int ch, int nv) {
      const int i = r16, hb = lane >> 4;
      uint32_t rd, rr[16];
      tmem_ld1(trow + K::T_DEN, rd);   // one column of all 32 lanes: rows in lanes 0-15
      tmem_ld16_halves<16>(trow + K::T_NUM + i0, rr);
      tmem_ld_wait1(rd);
      tmem_ld_wait16(rr);
      const float dn = __shfl_sync(kFull, __uint_as_float(rd), lane & 15);
      const float rdn = 1.0f / dn;
      const uint64_t rdn2 = f2_pack(rdn, rdn);
      const long long row = bh * a.N + ch * C + i;
      const uint32_t stage = K::S_O + ((ch - ch0) & 1) * K::TO;
      if (i < nv && a.den && half == 0 && hb == 0) a.den[row] = dn;
      uint8_t* box = smem + stage + half * (K::TO / 2) + i * 128;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t* r = rr + 4 * g;
        float4 q;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(r[0]), __uint_as_float(r[1])), rdn2), q.x, q.y);
        f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2]), __uint_as_float(r[3])), rdn2), q.z, q.w);
        *reinterpret_cast<float4*>(box + (((4 * hb + g) ^ (i & 7)) << 4)) = q;
      }
      if (i < nv && a.num) {
        float4* np = reinterpret_cast<float4*>(a.num + row * DV + c0);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          np[g] = make_float4(__uint_as_float(rr[4 * g]), __uint_as_float(rr[4 * g + 1]),
                              __uint_as_float(rr[4 * g + 2]), __uint_as_float(rr[4 * g + 3]));
      }
      fence_async_smem();
      if (tid == W2_GT) bulk_wait_read_0();
      named_sync(1, W2_GT);
      if (tid == W2_GT) {
        tma_store_3d(&tm_o, sbase + stage, 0, ch * C, static_cast<int>(bh));
        tma_store_3d(&tm_o, sbase + stage + K::TO / 2, 32, ch * C, static_cast<int>(bh));
        bulk_commit();
      }
    };
    bool ok = true;
    int prev = -1, prev_nv = C;
    // E2(t) comes before E4(t-1) so that G4(t) can start while E4 runs;
    // t == ch1 runs only the tail (E3, E4) of the last chunk
    for (int t = ch0; ok && t <= ch1 && ch0 < ch1; ++t) {
      const bool head = t < ch1;
      const int nv = head ? min(C, a.N - t * C) : 0;
      if (prev >= 0) {
        if (!(ok = waitB(2))) break;   // G4(t-1)
        e3();
      }
      if (head) {
        if (!(ok = waitB(0))) break;   // G1 + G7(t)
        {  // E1(t): masked S^T -> [j][i]
          const int j = r16;
          const bool keep = j < nv;
          uint32_t r[16];
          tmem_ld16_halves<16>(trow + K::T_S + i0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (!(keep && c0 + e >= j)) r[e] = 0u;
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, c0, 1024)) = pack8f(r, 1.f);
          *reinterpret_cast<uint4*>(smem + K::S_S + tile_off(j, c0 + 8, 1024)) = pack8f(r + 8, 1.f);
          signalB(1);
        }
      }
      if (head) {
        if (!(ok = waitB(1))) break;   // G2 + G3(t)
        {  // E2(t): X = |lambda|^(2(i-c)) a~
          uint64_t s2 = f2_pack(s_start, s_start * r2);   // scales of two adjacent columns
          const uint64_t r4 = f2_pack(r2 * r2, r2 * r2);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            uint32_t r[16];
            tmem_ld16(trow + K::T_A + i0 + 16 * b, r);
            tmem_ld_wait16(r);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float x0, x1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), s2), x0, x1);
              r[e] = __float_as_uint(x0);
              r[e + 1] = __float_as_uint(x1);
              s2 = f2_mul(s2, r4);
            }
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * b, 1024)) = pack8f(r, 1.f);
            *reinterpret_cast<uint4*>(smem + K::S_X + tile_off(k, i0 + 16 * b + 8, 1024)) = pack8f(r + 8, 1.f);
          }
          signalB(2);
        }
      }
      if (prev >= 0) {
        if (!(ok = waitB(3))) break;   // G5 + G6(t-1)
        e4(prev, prev_nv);
      }
      prev = t;
      prev_nv = nv;
    }
    if (tid == W2_GT) bulk_wait_all();   // o is in global memory before the block exits
  }
  if (role == 3) {
    // ------------------------------------------------ fetch warp
    if (lane == 0) {
      uint32_t pfq[NB] = {0u, 0u, 0u}, pfv[NB] = {0u, 0u, 0u};
      int issued[NB] = {0, 0, 0};
      for (int t = ch0; t < ch1; ++t) {
        const int rel = t - ch0, b = rel % NB;
        if (rel >= NB) {   // set b last held chunk t-3: wait until its contractions are done
          bool ok = mbar_wait_or_abort(freeQK + b, pfq[b], a.err, abort_flag);
          pfq[b] ^= 1u;
          if (ok) ok = mbar_wait_or_abort(freeVR + b, pfv[b], a.err, abort_flag);
          pfv[b] ^= 1u;
          if (!ok) break;
        }
        mbar_arrive_expect_tx(loaded + b, 3 * K::TIN);
        tma_load_3d(sbase + sQ(b), &tm_q, 0, t * C, static_cast<int>(bh), loaded + b);
        tma_load_3d(sbase + sK(b), &tm_k, 0, t * C, static_cast<int>(bh), loaded + b);
        tma_load_3d(sbase + sV(b), &tm_v, 0, t * C, static_cast<int>(bh), loaded + b);
        ++issued[b];
      }
      for (int b = 0; b < NB; ++b)   // no copy of ours lands after the block exits
        if (issued[b] > 0) mbar_wait(loaded + b, static_cast<uint32_t>((issued[b] - 1) & 1), a.err);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Tuning switch IA_PREFILL_WS for d = 64: 0 the one-role loop, 1 one epilogue
// group, unset or 2 the four-role kernel.
bool ws2_selected() {
  const char* ws = std::getenv("IA_PREFILL_WS");
  return !ws || std::atoi(ws) >= 2;
}

template <int DX, int DV>
cudaError_t launch_impl(const TcArgs& args, const ia_shape_t& s, const TcPlan& p, cudaStream_t st) {
  using K = Cfg<DX, DV>;
  cudaError_t e;
  if (p.nseg > 1) {
    auto k1 = tc_prefill_kernel<DX, DV, false>;
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
    if (e != cudaSuccess) return e;
    k1<<<static_cast<unsigned>(args.BH * (p.nseg - 1)), NT, K::SMEM, st>>>(args);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = launch_segment_scan(s.B, s.H, DX, DV, p.nseg, p.seg_chunks * C, args.tabs, args.state_in,
                            args.seg_state, args.seg_eta, st);
    if (e != cudaSuccess) return e;
  }
  if constexpr (DX == 64 && DV == 64) {
    if (ws2_selected()) {
      CUtensorMap tm_q, tm_k, tm_v, tm_o;
      if (!encode_input_map(&tm_q, args.q, args.BH, args.N) || !encode_input_map(&tm_k, args.k, args.BH, args.N) ||
          !encode_input_map(&tm_v, args.v, args.BH, args.N) || !encode_rows64_f32_map(&tm_o, args.o, args.BH, args.N))
        return cudaErrorNotSupported;
      e = cudaFuncSetAttribute(tc_prefill_ws2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, W2Cfg::SMEM);
      if (e != cudaSuccess) return e;
      // Programmatic dependent launch: the CTAs set up barriers, TMEM and
      // constant tiles while the previous kernel finishes (see griddep_wait).
      // Straight after the table kernel, the timing mark was set before it.
      if (p.nseg > 1) mark_launch_begin(st);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(args.BH * p.nseg));
      cfg.blockDim = dim3(W2_NT);
      cfg.dynamicSmemBytes = W2Cfg::SMEM;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, tc_prefill_ws2_kernel, args, tm_q, tm_k, tm_v, tm_o);
      mark_launch_end(st);
      return e;
    }
    const char* ws = std::getenv("IA_PREFILL_WS");
    if (std::atoi(ws) == 1) {
      e = cudaFuncSetAttribute(tc_prefill_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, WCfg::SMEM);
      if (e != cudaSuccess) return e;
      mark_launch_begin(st);
      tc_prefill_ws_kernel<<<static_cast<unsigned>(args.BH * p.nseg), WS_NT, WCfg::SMEM, st>>>(args);
      e = cudaGetLastError();
      mark_launch_end(st);
      return e;
    }
  }
  auto k3 = tc_prefill_kernel<DX, DV, true>;
  e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
  if (e != cudaSuccess) return e;
  mark_launch_begin(st);
  k3<<<static_cast<unsigned>(args.BH * p.nseg), NT, K::SMEM, st>>>(args);
  e = cudaGetLastError();
  mark_launch_end(st);
  return e;
}

}  // namespace

bool tc_prefill_supported(const ia_shape_t& s) {
  const bool dx = s.d_xi == 64 || s.d_xi == 128;
  const bool dv = s.d_v == 64 || s.d_v == 128;
  return s.in_dtype == IA_BF16 && s.M == kModesTC && dx && dv;
}

TcPlan tc_plan(const ia_shape_t& s, int num_sms) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  const int nch = (s.N + C - 1) / C;
  // Forced segment count (tuning and tests): IA_PREFILL_SEGMENTS=n.
  if (const char* env = std::getenv("IA_PREFILL_SEGMENTS")) {
    const int n = std::atoi(env);
    if (n >= 1 && n <= nch) {
      const int L = (nch + n - 1) / n;
      return TcPlan{(nch + L - 1) / L, L};
    }
  }
  // Cost in units of one full chunk pass: waves x (chunks per CTA + per-CTA
  // prologue/epilogue), a state-only chunk costing alpha, plus the scan.
  const double alpha = 0.35, cta_overhead = 1.0, scan = 1.0;
  const int min_len = 4;   // shorter segments spend more on state round trips than they save
  TcPlan best{1, nch};
  double best_t = 1e300;
  for (int nseg = 1; nseg <= 32 && nseg <= nch; ++nseg) {
    const int L = (nch + nseg - 1) / nseg;
    if ((nch + L - 1) / L != nseg) continue;
    if (nseg > 1 && L < min_len) continue;
    const double w1 = nseg > 1 ? std::ceil(static_cast<double>(BH * (nseg - 1)) / num_sms) : 0.0;
    const double w3 = std::ceil(static_cast<double>(BH * nseg) / num_sms);
    const double t = w1 * (L * alpha + cta_overhead) + w3 * (L + cta_overhead) + (nseg > 1 ? scan : 0.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = TcPlan{nseg, L};
    }
  }
  return best;
}

size_t tc_workspace_bytes(const ia_shape_t& s, const TcPlan& p) {
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  size_t bytes = sizeof(HeadTables) * static_cast<size_t>(s.H);
  if (p.nseg > 1) {
    bytes += BH * (p.nseg - 1) * (static_cast<size_t>(KR) * (s.d_xi + s.d_v) + KR) * sizeof(float);
  }
  return bytes + 256;
}

HeadTables* tc_tables(void* ws) {
  return reinterpret_cast<HeadTables*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255));
}

cudaError_t launch_tc_prefill(const ia_shape_t& s, const TcPlan& p, const void* q, const void* k,
                              const void* v, const float* delta, const float* A,
                              const void* state_in, float* o, float* num, float* den,
                              void* state_out, void* ws, cudaStream_t st, void* dump_R,
                              float* dump_Re, float* dtab) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  w = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(w) + 255) & ~static_cast<uintptr_t>(255));
  HeadTables* tabs = reinterpret_cast<HeadTables*>(w);
  float* seg_state = reinterpret_cast<float*>(w + sizeof(HeadTables) * s.H);
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  float* seg_eta = seg_state + BH * (p.nseg > 1 ? p.nseg - 1 : 0) * KR * (s.d_xi + s.d_v);
  // the four-role d = 64 kernel directly after the tables overlaps them, so
  // its timing mark goes before the table kernel
  if (s.d_xi == 64 && s.d_v == 64 && p.nseg == 1 && ws2_selected()) mark_launch_begin(st);
  cudaError_t e = launch_param_tables(s.H, delta, A, tabs, st, dtab);
  if (e != cudaSuccess) return e;
  TcArgs args;
  args.q = static_cast<const __nv_bfloat16*>(q);
  args.k = static_cast<const __nv_bfloat16*>(k);
  args.v = static_cast<const __nv_bfloat16*>(v);
  args.tabs = tabs;
  args.state_in = static_cast<const float2*>(state_in);
  args.seg_state = seg_state;
  args.seg_eta = seg_eta;
  args.o = o;
  args.num = num;
  args.den = den;
  args.state_out = static_cast<float2*>(state_out);
  args.err = device_error_ptr();
  args.dump_R = static_cast<uint8_t*>(dump_R);
  args.dump_Re = dump_Re;
  if (!args.err) return cudaErrorInvalidSymbol;
  args.H = s.H;
  args.N = s.N;
  args.nseg = p.nseg;
  args.seg_chunks = p.seg_chunks;
  args.BH = static_cast<long long>(BH);
  if (s.d_xi == 64 && s.d_v == 64) return launch_impl<64, 64>(args, s, p, st);
  if (s.d_xi == 128 && s.d_v == 128) return launch_impl<128, 128>(args, s, p, st);
  if (s.d_xi == 64 && s.d_v == 128) return launch_impl<64, 128>(args, s, p, st);
  if (s.d_xi == 128 && s.d_v == 64) return launch_impl<128, 64>(args, s, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace ia
