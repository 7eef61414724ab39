// rmsnorm_gated.cu -- the gated RMSNorm of the core output,
//   y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z),
// per (token, value head) over its d_v channels ("gated-deltanet-qwen3.5"
// section 输出门控与 RMSNorm: RMSNormGated(core_attn_out, z), the norm and then
// the SwiGLU-like z gate; the "Qwen3.5" module skeleton applies it per head after
// the recurrence).
//
// HBM-bound: o and z are read once and y written once.  One warp per row: each
// lane holds DV / 32 consecutive channels (8 bytes of bf16 at d_v = 128), so a
// warp reads and writes whole 256-byte rows; the sum of squares is a warp
// reduction.  Every lane reads its own o and z entries before it writes y, so y
// may be o or z (in place).
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kRT = 256;  // threads per CTA (8 rows at a time)

template <typename T, int PER>
__device__ __forceinline__ void load_per(const T* p, float* f) {
#pragma unroll
  for (int i = 0; i < PER; ++i) f[i] = to_f32(p[i]);
}
template <typename T, int PER>
__device__ __forceinline__ void store_per(T* p, const float* f) {
#pragma unroll
  for (int i = 0; i < PER; ++i) p[i] = from_f32<T>(f[i]);
}

// o and y of type T, the gate z of type TZ (float32 cores gated by bf16 z on the
// float32-output path of gdn_chunk_fwd_gated_norm).
template <typename T, typename TZ, int DV>
__global__ void __launch_bounds__(kRT)
rmsnorm_gated_kernel(const T* o, const TZ* z, const float* __restrict__ weight, T* y, long rows,
                     float eps) {
  constexpr int PER = DV / 32;
  const int lane = threadIdx.x & 31;
  const long row = (blockIdx.x * (long)kRT + threadIdx.x) >> 5;
  if (row >= rows) return;  // whole warps: rows are per warp, no barrier below
  const size_t off = (size_t)row * DV + lane * PER;
  float ov[PER], zv[PER], wv[PER];
  load_per<T, PER>(o + off, ov);
  load_per<TZ, PER>(z + off, zv);
#pragma unroll
  for (int i = 0; i < PER; ++i) wv[i] = weight[lane * PER + i];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) ss = fmaf(ov[i], ov[i], ss);
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss * (1.f / DV) + eps);
  float yv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float g = __fdividef(zv[i], 1.f + __expf(-zv[i]));  // SiLU(z)
    yv[i] = ov[i] * inv * wv[i] * g;
  }
  store_per<T, PER>(y + off, yv);
}

template <typename T, typename TZ, int DV>
cudaError_t launch_typed(const void* o, const void* z, const float* w, void* y, long rows,
                         float eps, cudaStream_t s) {
  const long blocks = (rows + kRT / 32 - 1) / (kRT / 32);
  rmsnorm_gated_kernel<T, TZ, DV><<<(unsigned)blocks, kRT, 0, s>>>(
      static_cast<const T*>(o), static_cast<const TZ*>(z), w, static_cast<T*>(y), rows, eps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rmsnorm_gated(const void* o, const void* z, const float* weight, void* y,
                                 long rows, int dv, int dtype, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if ((rows + kRT / 32 - 1) / (kRT / 32) > 0x7fffffffL) return cudaErrorInvalidValue;
  using bf16 = __nv_bfloat16;
  if (dtype == GDN_BF16)
    return dv == 128 ? launch_typed<bf16, bf16, 128>(o, z, weight, y, rows, eps, s)
                     : launch_typed<bf16, bf16, 64>(o, z, weight, y, rows, eps, s);
  return dv == 128 ? launch_typed<float, float, 128>(o, z, weight, y, rows, eps, s)
                   : launch_typed<float, float, 64>(o, z, weight, y, rows, eps, s);
}

cudaError_t launch_rmsnorm_gated_f32_bf16z(const float* o, const void* z, const float* weight,
                                           float* y, long rows, int dv, float eps,
                                           cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if ((rows + kRT / 32 - 1) / (kRT / 32) > 0x7fffffffL) return cudaErrorInvalidValue;
  using bf16 = __nv_bfloat16;
  return dv == 128 ? launch_typed<float, bf16, 128>(o, z, weight, y, rows, eps, s)
                   : launch_typed<float, bf16, 64>(o, z, weight, y, rows, eps, s);
}

}  // namespace gdn
