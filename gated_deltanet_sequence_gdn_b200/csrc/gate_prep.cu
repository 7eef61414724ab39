// gate_prep.cu -- the gate and L2-norm prologue as one elementwise kernel.
//
// "Qwen3.5" (rainlin-net), module skeleton: beta = sigmoid(b) and
// g = -exp(A_log) * softplus(a + dt_bias) in float32.  The per-head L2 norm of
// q and k (x / sqrt(|x|^2 + 1e-6)) and the query scale applied after it are
// this library's reading of the pages.
//
// HBM-bound: one read of q, k, a, b and one write of the outputs.  One CTA per
// group of token rows; a group of lanes per (row, head) vector of q or k, each
// lane moving 16-byte pieces, several vectors in flight per lane; the gates are
// spread over the CTA's threads.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;

template <typename T>
struct Vec16;  // 16 bytes of T
template <> struct Vec16<float> { using type = float4; static constexpr int n = 4; };
template <> struct Vec16<__nv_bfloat16> { using type = uint4; static constexpr int n = 8; };

template <typename T>
__device__ __forceinline__ void unpack(const typename Vec16<T>::type& v, float* f);
template <> __device__ __forceinline__ void unpack<float>(const float4& v, float* f) {
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <> __device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& v, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x; f[2 * i + 1] = t.y;
  }
}
template <typename T>
__device__ __forceinline__ typename Vec16<T>::type pack(const float* f);
template <> __device__ __forceinline__ float4 pack<float>(const float* f) {
  return make_float4(f[0], f[1], f[2], f[3]);
}
template <> __device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float* f) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return v;
}

// Sum over the `width` lanes of an aligned lane group (width a power of 2 <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// rows_per_cta token rows per CTA; d in {64, 128}.  A q / k vector of one (row,
// head) is d / E lanes of 16 bytes (a lane group); a warp holds 32 / (d / E) such
// groups, and each group takes kU vectors per pass, all loads issued before the
// first reduction, so that every lane has kU 16-byte loads in flight.
template <typename T>
__global__ void __launch_bounds__(kThreads)
gate_prep_kernel(const T* q, const T* k,
                 const T* __restrict__ a, const T* __restrict__ b,
                 const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                 long rows, int Hk, int Hv, int d, float scale, int rows_per_cta,
                 T* q_out, T* k_out, float* __restrict__ g_out,
                 float* __restrict__ beta_out) {
  using V = typename Vec16<T>::type;
  constexpr int E = Vec16<T>::n;
  constexpr int kU = 4;
  const long row0 = (long)blockIdx.x * rows_per_cta;
  const long row1 = min(rows, row0 + rows_per_cta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int width = d / E;                 // lanes per vector: 8, 16 or 32
  const int groups = 32 / width;           // vectors per warp and pass step
  const int gl = lane % width, grp = lane / width;
  // vectors: item = (row, head, which), q and k of a head adjacent
  const long n_items = (row1 - row0) * Hk * 2;
  const long step = (long)(kThreads / 32) * groups;
  // the loop bound is the same for every lane of the warp (the shuffles below take
  // all 32 lanes); a group past the end just has nothing to load
  for (long wbase = (long)warp * groups; wbase < n_items; wbase += step * kU) {
    const long base = wbase + grp;
    V vin[kU];
    bool have[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long it = base + u * step;
      have[u] = it < n_items;
      if (have[u]) {
        const long r = row0 + it / (2 * Hk);
        const int rem = (int)(it % (2 * Hk));
        const size_t off = ((size_t)r * Hk + (rem >> 1)) * d;
        vin[u] = reinterpret_cast<const V*>(((rem & 1) == 0 ? q : k) + off)[gl];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long it = base + u * step;
      float f[E];
      float ss = 0.f;
      if (have[u]) {
        unpack<T>(vin[u], f);
#pragma unroll
        for (int i = 0; i < E; ++i) ss += f[i] * f[i];
      }
      ss = group_sum(ss, width);  // every lane takes part (no divergent shuffles)
      if (have[u]) {
        const long r = row0 + it / (2 * Hk);
        const int rem = (int)(it % (2 * Hk));
        const bool is_q = (rem & 1) == 0;
        const size_t off = ((size_t)r * Hk + (rem >> 1)) * d;
        const float mul = rsqrtf(ss + 1e-6f) * (is_q ? scale : 1.f);
#pragma unroll
        for (int i = 0; i < E; ++i) f[i] *= mul;
        reinterpret_cast<V*>((is_q ? q_out : k_out) + off)[gl] = pack<T>(f);
      }
    }
  }
  // gates: item = (row, value head)
  const long n_gates = (row1 - row0) * Hv;
  for (long it = threadIdx.x; it < n_gates; it += kThreads) {
    const long r = row0 + it / Hv;
    const int h = (int)(it % Hv);
    const size_t idx = (size_t)r * Hv + h;
    g_out[idx] = gdn_log_decay(to_f32(a[idx]), A_log[h], dt_bias[h]);
    beta_out[idx] = sigmoid_f(to_f32(b[idx]));
  }
}

}  // namespace

cudaError_t launch_gate_prep(const void* q, const void* k, int dtype, const void* a,
                             const void* b, const float* A_log, const float* dt_bias,
                             int B, int T, int Hk, int Hv, int d, float scale,
                             void* q_out, void* k_out, float* g_out, float* beta_out,
                             cudaStream_t s) {
  const long rows = (long)B * T;
  if (rows == 0) return cudaSuccess;
  const int rows_per_cta = 8;
  const long grid = (rows + rows_per_cta - 1) / rows_per_cta;
  if (dtype == GDN_BF16) {
    gate_prep_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)a,
        (const __nv_bfloat16*)b, A_log, dt_bias, rows, Hk, Hv, d, scale, rows_per_cta,
        (__nv_bfloat16*)q_out, (__nv_bfloat16*)k_out, g_out, beta_out);
  } else {
    gate_prep_kernel<float><<<(unsigned)grid, kThreads, 0, s>>>(
        (const float*)q, (const float*)k, (const float*)a, (const float*)b, A_log,
        dt_bias, rows, Hk, Hv, d, scale, rows_per_cta, (float*)q_out, (float*)k_out,
        g_out, beta_out);
  }
  return cudaGetLastError();
}

}  // namespace gdn
