// wy_common.cuh -- fp32 operands on the bf16 warp-level tensor cores (hi + lo
// splits), shared by the chunk preparation kernels of the WY chunk form.
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

}  // namespace wy
}  // namespace gdn
