// wy_common.cuh -- fp32 operands on the bf16 warp-level tensor cores (hi + lo
// splits) and the blocked inverse (I + L)^-1, shared by the chunk preparation
// kernels of the WY chunk form.
#pragma once

#include <stdint.h>

#include "warp_mma.cuh"

namespace gdn {
namespace wy {

using namespace wm;

constexpr int LDX = 64 + 8;  // f32 row stride of the 64 x 64 L and X (conflict-free float2)
constexpr int LDB = 20;      // f32 row stride of a 16 x 16 block product

// x = hi + lo with hi = rn_bf16(x), lo = rn_bf16(x - hi), for a pair of values.
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack2(x, y);
  const float2 h = unpack2(hi);
  lo = pack2(x - h.x, y - h.y);
}

// A fragment (16 x 16, row-major) of an fp32 matrix M (row stride ld) at
// (r0, c0), as bf16 hi + lo parts.
__device__ __forceinline__ void frag_a_split(const float* M, int ld, int r0, int c0, int g8, int t4,
                                             uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  const float2 x00 = *reinterpret_cast<const float2*>(M + (r0 + g8) * ld + c0 + 2 * t4);
  const float2 x10 = *reinterpret_cast<const float2*>(M + (r0 + g8 + 8) * ld + c0 + 2 * t4);
  const float2 x01 = *reinterpret_cast<const float2*>(M + (r0 + g8) * ld + c0 + 2 * t4 + 8);
  const float2 x11 = *reinterpret_cast<const float2*>(M + (r0 + g8 + 8) * ld + c0 + 2 * t4 + 8);
  split2(x00.x, x00.y, hi[0], lo[0]);
  split2(x10.x, x10.y, hi[1], lo[1]);
  split2(x01.x, x01.y, hi[2], lo[2]);
  split2(x11.x, x11.y, hi[3], lo[3]);
}
// B fragment (16 x 8, k x n) of an fp32 matrix M (row = k) at (k0, n0), split.
__device__ __forceinline__ void frag_b_split(const float* M, int ld, int k0, int n0, int g8, int t4,
                                             uint32_t (&hi)[2], uint32_t (&lo)[2]) {
  const float* p = M + (k0 + 2 * t4) * ld + n0 + g8;
  split2(p[0], p[ld], hi[0], lo[0]);
  split2(p[8 * ld], p[9 * ld], hi[1], lo[1]);
}
// D += A B for split operands, the lo x lo term dropped (about 2^-16 relative).
__device__ __forceinline__ void mma_split3(float (&d)[4], const uint32_t (&ah)[4],
                                           const uint32_t (&al)[4], const uint32_t (&bh)[2],
                                           const uint32_t (&bl)[2]) {
  mma_bf16(d, ah, bh[0], bh[1]);
  mma_bf16(d, ah, bl[0], bl[1]);
  mma_bf16(d, al, bh[0], bh[1]);
}

// Exponent e with (max |row|) * 2^-e in [1, 2) (e = 0 for a zero row).
__device__ __forceinline__ int row_exponent(float m) { return m > 0.f ? ilogbf(m) : 0; }

// One 16 x 8 tile (columns n0 .. n0 + 7) of sum_i A_i B_i over nk pairs of 16 x 16
// fp32 blocks, A_i at (ar, ac[i]) of A (row stride lda) and B_i at (br[i], n0) of
// B (row stride ldb), on the warp tensor cores with the operands as bf16 hi + lo.
__device__ __forceinline__ void block_prod(const float* A, int lda, int ar, const int* ac,
                                           const float* Bm, int ldb, const int* br, int nk, int n0,
                                           int g8, int t4, float (&d)[4]) {
  for (int i = 0; i < nk; ++i) {
    uint32_t ah[4], al[4], bh[2], bl[2];
    frag_a_split(A, lda, ar, ac[i], g8, t4, ah, al);
    frag_b_split(Bm, ldb, br[i], n0, g8, t4, bh, bl);
    mma_split3(d, ah, al, bh, bl);
  }
}
// The 16 x 8 tile d to rows r0 .. r0 + 15, columns c0 .. c0 + 7 of M (row stride ld), scaled by s.
__device__ __forceinline__ void store_tile(float* M, int ld, int r0, int c0, int g8, int t4,
                                           const float (&d)[4], float s) {
  *reinterpret_cast<float2*>(M + (r0 + g8) * ld + c0 + 2 * t4) = make_float2(s * d[0], s * d[1]);
  *reinterpret_cast<float2*>(M + (r0 + g8 + 8) * ld + c0 + 2 * t4) = make_float2(s * d[2], s * d[3]);
}

// X = (I + L)^-1 in place for a strictly lower 64 x 64 fp32 L (row stride LDX,
// zero upper triangle), by the whole CTA (products on warps 0-7, every warp at the
// barriers), by recursive doubling over 16 x 16 blocks (L_ij, X_ij):
//   X_ii       : forward substitution, one thread per column of a diagonal block;
//   32 x 32    : X_10 = -X_11 (L_10 X_00),  X_32 = -X_33 (L_32 X_22);
//   64 x 64    : X_[2:4][0:2] = -X_[2:4][2:4] (L_[2:4][0:2] X_[0:2][0:2]),
// each product stage one 16 x 8 output tile per warp, the intermediate products in Tm
// (four [16][LDB] fp32 tiles).  Every write of a block waits at a barrier until the
// reads of the L block it replaces are done.
__device__ inline void invert_in_place(float* M, float* Tm, int tid, int warp, int g8, int t4) {
  float x[16];
  const int base = 16 * (tid >> 4), cc = tid & 15;
  if (tid < 64) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float s = 0.f;
#pragma unroll
      for (int jj = 0; jj < r; ++jj) s = fmaf(M[(base + r) * LDX + base + jj], x[jj], s);
      x[r] = r == cc ? 1.f : -s;  // rows above cc come out as zero
    }
  }
  __syncthreads();
  if (tid < 64) {
#pragma unroll
    for (int r = 0; r < 16; ++r) M[(base + r) * LDX + base + cc] = x[r];
  }
  __syncthreads();
  const int nt = warp & 1, n8 = 8 * nt;
  // 32 x 32 blocks: T_0 = L_10 X_00, T_1 = L_32 X_22 (warps 0-3), then X_10, X_32
  if (warp < 4) {
    const int b = warp >> 1, o = 32 * b;  // block pair (0, 1) or (2, 3)
    float d[4] = {};
    const int ac[1] = {o}, br[1] = {o};
    block_prod(M, LDX, o + 16, ac, M, LDX, br, 1, o + n8, g8, t4, d);
    store_tile(Tm + b * 16 * LDB, LDB, 0, n8, g8, t4, d, 1.f);
  }
  __syncthreads();
  if (warp < 4) {
    const int b = warp >> 1, o = 32 * b;
    float d[4] = {};
    const int ac[1] = {o + 16}, br[1] = {0};
    block_prod(M, LDX, o + 16, ac, Tm + b * 16 * LDB, LDB, br, 1, n8, g8, t4, d);
    store_tile(M, LDX, o + 16, o + n8, g8, t4, d, -1.f);
  }
  __syncthreads();
  // 64 x 64: T_(ri, cj) = sum_{k=cj}^{1} L_(ri, k) X_(k, cj) for ri = 2, 3 and cj = 0, 1
  // (warps 0-7; the warps past them only keep the barriers)
  const int t = warp >> 1, ri = 2 + (t >> 1), cj = t & 1;
  if (warp < 8) {
    float d[4] = {};
    const int ac[2] = {16 * cj, 16}, br[2] = {16 * cj, 16};
    block_prod(M, LDX, 16 * ri, ac, M, LDX, br, 2 - cj, 16 * cj + n8, g8, t4, d);
    store_tile(Tm + t * 16 * LDB, LDB, 0, n8, g8, t4, d, 1.f);
  }
  __syncthreads();
  //         X_(ri, cj) = -sum_{k=2}^{ri} X_(ri, k) T_(k, cj)
  if (warp < 8) {
    float d[4] = {};
    for (int k = 2; k <= ri; ++k) {
      const int ac[1] = {16 * k}, br[1] = {0};
      block_prod(M, LDX, 16 * ri, ac, Tm + (2 * (k - 2) + cj) * 16 * LDB, LDB, br, 1, n8, g8, t4, d);
    }
    store_tile(M, LDX, 16 * ri, 16 * cj + n8, g8, t4, d, -1.f);
  }
  __syncthreads();
}

}  // namespace wy
}  // namespace gdn
