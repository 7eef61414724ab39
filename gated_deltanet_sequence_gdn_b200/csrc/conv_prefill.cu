// conv_prefill.cu -- the causal depthwise conv1d (kernel 4) + SiLU over a whole
// prefill of the mixed [q | k | v] channel stream, written as the contiguous q,
// k and v the chunk path reads, with the conv window (the last three inputs of
// every channel) carried in and out for the decode steps that follow.
//
// Pages: "从 Full Attention 到 Gated DeltaNet" section 10 (x -> CausalConv1D ->
// SiLU -> q, k, v); "gated-deltanet-qwen3.5" section 因果卷积 (kernel 4,
// depthwise, causal) and its architecture diagram (conv_states handed to the
// inference branch).  The L2 norm of q and k is left to the chunk path's
// prologue (gdn_chunk_fwd with GDN_QK_L2NORM), which fuses it.
//
// HBM-bound: every input and every output element crosses HBM once.  A thread
// takes 8 channels (16 bytes of bf16) of 16 consecutive tokens; consecutive
// threads take consecutive channel groups, so each warp reads and writes whole
// 512-byte runs of a token row.  A thread stages its input rows in shared memory
// with asynchronous copies issued all at once (the three inputs before the tile
// and its first 8 tokens, then the other 8), and works on the first 8 while the
// rest arrive; it reads back only the rows it copied itself, so no barrier is
// needed.  The three inputs before a token tile are re-read (from L2) by the
// tile's threads.  The conv window in conv_state is read and rewritten only by the
// threads of the first token tile, so an in-place update has no race between
// CTAs.
#include "common.cuh"
#include "launch.h"
#include "warp_mma.cuh"

namespace gdn {
namespace {

constexpr int kCT = 128;  // threads per CTA (five CTAs per SM: their load and SiLU phases stagger)
constexpr int kTT = 16;   // tokens per thread

// SiLU(x) = x / (1 + e^-x) with the hardware exp2 and reciprocal approximations
// (relative error ~1e-7; the accurate expf and division would make this
// HBM-bound kernel issue-bound).  For x below about -88, e^-x is +inf and the
// quotient is 0, the limit of SiLU there.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// 8 channels of one token as loaded (16 bytes of bf16, 32 of fp32), and their
// float32 values.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = *reinterpret_cast<const uint4*>(p);
  }
  __device__ __forceinline__ void get(float* f) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ void get(float* f) const {
    f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w;
    f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
  }
};
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* f) {
  Raw8<T> r;
  r.load(p);
  r.get(f);
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float* f);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* p, const float* f) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// x [B, T, Cc] with Cc = 2 QK + V (channel order q | k | v); conv_w [Cc, 4]
// (tap 3 multiplies the newest input); conv_state [B, Cc, 3] (index 2 newest) or
// null (a zero window, nothing written back); q, k [B, T, QK]; v [B, T, V].
// Shared memory: rows r = 0 .. kTT + 2 (input t0 - 3 + r) of kCT threads x 8 channels.
template <typename T>
constexpr int conv_stage_bytes() { return (kTT + 3) * kCT * 8 * (int)sizeof(T); }

template <typename T>
__global__ void __launch_bounds__(kCT)
conv_prefill_kernel(const T* __restrict__ x, const float* __restrict__ conv_w, T* conv_state,
                    T* __restrict__ q, T* __restrict__ k, T* __restrict__ v, int Tn, int Cc,
                    int QK, int V) {
  extern __shared__ __align__(16) uint8_t stage[];
  constexpr int EB = 8 * (int)sizeof(T);  // bytes of 8 channels
  const int cg = blockIdx.x * kCT + threadIdx.x;
  if (cg >= Cc / 8) return;  // no barrier in this kernel
  const int c0 = 8 * cg, t0 = blockIdx.y * kTT, bb = blockIdx.z;
  const int tn = min(kTT, Tn - t0);
  const T* xb = x + (size_t)bb * Tn * Cc + c0;
  uint8_t* my = stage + threadIdx.x * EB;  // row r of this thread at my + r * kCT * EB
  {
    const int r_end[2] = {3 + min(tn, 8), 3 + tn};
    int r = t0 > 0 ? 0 : 3;
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
      for (; r < r_end[grp]; ++r) {
        const T* src = xb + (size_t)(t0 - 3 + r) * Cc;
#pragma unroll
        for (int h = 0; h < EB / 16; ++h)
          wm::cp16(my + (size_t)r * kCT * EB + 16 * h, src + h * (16 / (int)sizeof(T)), 16);
      }
      wm::cp_commit();
    }
  }
  float w[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 t = *reinterpret_cast<const float4*>(conv_w + (size_t)(c0 + u) * 4);
    w[u][0] = t.x, w[u][1] = t.y, w[u][2] = t.z, w[u][3] = t.w;
  }
  T* cs = conv_state == nullptr ? nullptr : conv_state + ((size_t)bb * Cc + c0) * 3;
  auto srow = [&](int r) { return reinterpret_cast<const T*>(my + (size_t)r * kCT * EB); };
  // the window before t0: inputs t0 - 3, t0 - 2, t0 - 1 (from the carried window at t0 = 0)
  float h0[8], h1[8], h2[8];
  wm::cp_wait<1>();  // the first group: the window rows and tokens 0 .. 7
  if (t0 > 0) {
    load8(srow(0), h0);
    load8(srow(1), h1);
    load8(srow(2), h2);
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      h0[u] = cs ? to_f32(cs[3 * u + 0]) : 0.f;
      h1[u] = cs ? to_f32(cs[3 * u + 1]) : 0.f;
      h2[u] = cs ? to_f32(cs[3 * u + 2]) : 0.f;
    }
  }
  T* dst;
  size_t ld;
  if (c0 < QK) dst = q + c0, ld = QK;
  else if (c0 < 2 * QK) dst = k + (c0 - QK), ld = QK;
  else dst = v + (c0 - 2 * QK), ld = V;
  dst += ((size_t)bb * Tn + t0) * ld;
#pragma unroll 1
  for (int i = 0; i < tn; ++i) {
    if (i == 8) wm::cp_wait<0>();  // the second group: tokens 8 .. 15
    float xn[8], y[8];
    load8(srow(3 + i), xn);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float acc = w[u][0] * h0[u] + w[u][1] * h1[u] + w[u][2] * h2[u] + w[u][3] * xn[u];
      y[u] = silu_fast(acc);
      h0[u] = h1[u], h1[u] = h2[u], h2[u] = xn[u];
    }
    store8(dst + (size_t)i * ld, y);
  }
  // the window after the last token (inputs Tn - 3 .. Tn - 1; for Tn < 3 partly
  // the carried window), all read before any is written
  if (t0 == 0 && cs != nullptr) {
    float s[3][8];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int tj = Tn - 3 + j;
      if (tj >= 0) {
        load8(xb + (size_t)tj * Cc, s[j]);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) s[j][u] = to_f32(cs[3 * u + Tn + j]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cs[3 * u + 0] = from_f32<T>(s[0][u]);
      cs[3 * u + 1] = from_f32<T>(s[1][u]);
      cs[3 * u + 2] = from_f32<T>(s[2][u]);
    }
  }
}

}  // namespace

cudaError_t launch_conv_prefill(const void* x, const float* conv_w, void* conv_state, void* q,
                                void* k, void* v, int B, int T, int Hk, int Hv, int dk, int dv,
                                int dtype, cudaStream_t s) {
  const int QK = Hk * dk, V = Hv * dv, Cc = 2 * QK + V;
  if (B <= 0 || T <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((Cc / 8 + kCT - 1) / kCT), (unsigned)((T + kTT - 1) / kTT),
                  (unsigned)B);
  if (grid.y > 65535u || grid.z > 65535u) return cudaErrorInvalidValue;
  if (dtype == GDN_BF16) {
    using bf16 = __nv_bfloat16;
    constexpr int smem = conv_stage_bytes<bf16>();
    cudaError_t e = cudaFuncSetAttribute(conv_prefill_kernel<bf16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    conv_prefill_kernel<bf16><<<grid, kCT, smem, s>>>(
        static_cast<const bf16*>(x), conv_w, static_cast<bf16*>(conv_state),
        static_cast<bf16*>(q), static_cast<bf16*>(k), static_cast<bf16*>(v), T, Cc, QK, V);
  } else {
    constexpr int smem = conv_stage_bytes<float>();
    cudaError_t e = cudaFuncSetAttribute(conv_prefill_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    conv_prefill_kernel<float><<<grid, kCT, smem, s>>>(
        static_cast<const float*>(x), conv_w, static_cast<float*>(conv_state),
        static_cast<float*>(q), static_cast<float*>(k), static_cast<float*>(v), T, Cc, QK, V);
  }
  return cudaGetLastError();
}

}  // namespace gdn
