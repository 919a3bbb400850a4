// Shared pieces of the tcgen05 chunk kernels (forward and reverse mode):
// chunk constants, the no-swizzle canonical tile layout, MMA issue over K
// steps, and the bf16 -> fp16 tile conversion that applies the feature map.
//
// Tile layout: a tile with rows r and columns x (x contiguous) of width W
// stores element (r, x) at byte (r/8)*(W*16) + (x/8)*128 + (r%8)*16 + (x%8)*2.
// Used with rows as the M/N dimension it is K-major (lbo 128, sbo 16W, 256
// bytes per K step of 16); with columns as M/N it is MN-major (lbo 16W,
// sbo 128, 32W bytes per K step).
#pragma once

#include "ia_device.cuh"
#include "ia_tables.cuh"

namespace ia {
namespace tc {

constexpr int C = kChunk;          // 64 tokens per chunk
constexpr int KR = 2 * kModesTC;   // 128 real rows (mode, re/im)
constexpr int NTHR = 256;          // 8 warps: warp w owns TMEM lane quadrant w%4, column half w/4
constexpr uint32_t kFull = 0xffffffffu;

__host__ __device__ constexpr uint32_t kmaj_lbo() { return 128; }
__host__ __device__ constexpr uint32_t kmaj_sbo(int W) { return static_cast<uint32_t>(W * 16); }
__host__ __device__ constexpr uint32_t kmaj_step() { return 256; }
__host__ __device__ constexpr uint32_t mn_lbo(int W) { return static_cast<uint32_t>(W * 16); }
__host__ __device__ constexpr uint32_t mn_sbo() { return 128; }
__host__ __device__ constexpr uint32_t mn_step(int W) { return static_cast<uint32_t>(W * 32); }

__device__ __forceinline__ uint32_t tile_off(int r, int x, uint32_t rs) {
  return static_cast<uint32_t>((r >> 3) * rs + (x >> 3) * 128 + (r & 7) * 16 + (x & 7) * 2);
}

// D (+)= A * B^T over ksteps of K = 16; A and B described by (addr, lbo, sbo,
// byte advance per K step).
__device__ __forceinline__ void gemm(uint32_t dtm, uint32_t a, uint32_t alb, uint32_t asb,
                                     uint32_t ast, uint32_t b, uint32_t blb, uint32_t bsb,
                                     uint32_t bst, uint32_t idesc, int ksteps, bool acc) {
  for (int kk = 0; kk < ksteps; ++kk) {
    mma_f16(dtm, smem_desc(a + kk * ast, alb, asb), smem_desc(b + kk * bst, blb, bsb), idesc,
            (kk > 0 || acc) ? 1u : 0u);
  }
}

// Same with prebuilt descriptors (e.g. swizzled tiles): the start addresses
// advance by astep / bstep bytes per K-step of 16.
__device__ __forceinline__ void gemm_dd(uint32_t dtm, uint64_t adesc, uint32_t astep, uint64_t bdesc,
                                        uint32_t bstep, uint32_t idesc, int ksteps, bool acc) {
  for (int kk = 0; kk < ksteps; ++kk)
    mma_f16(dtm, adesc + ((kk * astep) >> 4), bdesc + ((kk * bstep) >> 4), idesc, (kk > 0 || acc) ? 1u : 0u);
}

// bf16 staging rows [C][W] (row-major, contiguous) -> fp16 canonical tile,
// applying xi (on fp16 pairs, as the forward does) when FEAT; rows >= nv
// become zero.  One warp iteration moves 8 rows x 4 column groups; the column
// group is rotated by the row so that both the staging reads and the tile
// writes are bank-conflict free.
template <int W, bool FEAT>
__device__ __forceinline__ void convert_tile(const uint8_t* stg, uint8_t* dst, int nv, int warp,
                                             int lane) {
  constexpr int NCG = W / 8;            // 16-byte column groups per row
  constexpr int ITERS = (C / 8) * (NCG / 4);
  const int r8 = lane & 7, slot = lane >> 3;
  for (int it = warp; it < ITERS; it += NTHR / 32) {
    const int rb = it & 7, rest = it >> 3;
    const int cb8 = rest >> 1, sub = rest & 1;
    const int r = rb * 8 + r8;
    const int cg = cb8 * 8 + ((slot + 4 * sub + r8) & 7);
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (r < nv) {
      uint4 in = *reinterpret_cast<const uint4*>(stg + r * (W * 2) + cg * 16);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&in);
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        w[e] = FEAT ? feat_h2(f.x, f.y) : pack_half2(f.x, f.y);
      }
      out = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(dst + tile_off(r, cg * 8, W * 16)) = out;
  }
}

}  // namespace tc
}  // namespace ia
