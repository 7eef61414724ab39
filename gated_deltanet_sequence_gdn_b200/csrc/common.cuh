// common.cuh -- small device helpers shared by the kernels of libgdn.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Element access for the two input types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// softplus(x) = log(1 + e^x), evaluated as max(x,0) + log1p(exp(-|x|)) (the same
// number without overflow).  "从 Full Attention 到 Gated DeltaNet", section 9.
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// Log-decay of one (token, value head): g = -exp(A_log) * softplus(a + dt_bias).
__device__ __forceinline__ float gdn_log_decay(float a, float A_log, float dt_bias) {
  return -expf(A_log) * softplus_f(a + dt_bias);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Device status word (its address is passed to kernels with bounded waits):
// an expired wait records where it gave up; gdn_check_status reads and clears it.
__device__ __forceinline__ void report_timeout(int* status, int where) {
  atomicCAS(status, 0, where);
}
// Bit of the status word set when an intermediate left the range of its
// reduced-precision operand format (the outputs of that call are not valid).
constexpr int kStatusRange = 1 << 30;
__device__ __forceinline__ void report_range(int* status) {
  if (status) atomicOr(status, kStatusRange);
}

}  // namespace gdn
