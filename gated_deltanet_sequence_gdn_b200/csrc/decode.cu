// decode.cu -- one-token GDN decode step fused with the causal conv1d update.
//
// Pages: "gated-deltanet-qwen3.5" (architecture diagram, inference branch:
// recurrent_gated_delta_rule reads and updates conv_states and
// recurrent_states); "从 Full Attention 到 Gated DeltaNet" section 10
// (x -> CausalConv1D -> SiLU -> q, k, v); "Qwen3.5" GDN详解 (five-step update:
// decay, read, delta, write, read-out).
//
// HBM-bound: every [dk, dv] float32 state is read once and written once with
// 16-byte coalesced accesses; everything else (conv window, x, gates, o) is a
// few percent of the traffic.  One CTA per (sequence, key-head group): the
// group's query/key conv channels are shared by its Hv/Hk value heads, so the
// CTA that owns them is the only one that shifts their conv window (no race
// between CTAs on the in-place conv state).
//
// With NORM each output row leaves through the gated RMSNorm of the pages' output
// stage ("gated-deltanet-qwen3.5", 输出门控与 RMSNorm): y = o / sqrt(mean(o^2) + eps)
// * w * SiLU(z) over the dv columns of the (sequence, value head); the CTA holds
// the whole row, so the mean is a block reduction.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;

template <typename T, typename TO, int DK, int DV, bool NORM>
__global__ void __launch_bounds__(kThreads, 2)
decode_step_kernel(const T* __restrict__ x, const float* __restrict__ conv_w,
                   T* __restrict__ conv_state, const T* __restrict__ a,
                   const T* __restrict__ b, const float* __restrict__ A_log,
                   const float* __restrict__ dt_bias, float* __restrict__ state,
                   TO* __restrict__ o, int Hk, int Hv, float scale, const T* __restrict__ nz,
                   const float* __restrict__ nw, float neps) {
  constexpr int TPR = DV / 4;               // threads per state row (float4 each)
  constexpr int RPP = kThreads / TPR;       // rows covered per pass
  constexpr int PASSES = DK / RPP;          // rows per thread
  static_assert(DK % RPP == 0, "tile");
  const int G = Hv / Hk;
  const int n = blockIdx.x / Hk;
  const int hk = blockIdx.x % Hk;
  const int Cc = 2 * Hk * DK + Hv * DV;
  const int tid = threadIdx.x;

  extern __shared__ float smem[];
  float* qv = smem;                 // [DK]  normalised, scaled query
  float* kvec = qv + DK;            // [DK]  normalised key
  float* vv = kvec + DK;            // [G*DV] values of the group's heads
  float* red = vv + G * DV;         // [RPP][DV] partial sums
  float* gates = red + RPP * DV;    // [G][2] alpha, beta
  __shared__ float norm_ss[2];
  __shared__ float row_ss[DV / 32];

  // ---- 1. conv1d + SiLU over the group's channels, window shifted in place
  const int n_ch = 2 * DK + G * DV;
  for (int i = tid; i < n_ch; i += kThreads) {
    int c;  // global channel
    if (i < DK) c = hk * DK + i;
    else if (i < 2 * DK) c = Hk * DK + hk * DK + (i - DK);
    else c = 2 * Hk * DK + hk * G * DV + (i - 2 * DK);
    const float xn = to_f32(x[(size_t)n * Cc + c]);
    float y;
    if (conv_w != nullptr) {
      T* cs = conv_state + ((size_t)n * Cc + c) * 3;
      const float c0 = to_f32(cs[0]), c1 = to_f32(cs[1]), c2 = to_f32(cs[2]);
      const float4 w = *reinterpret_cast<const float4*>(conv_w + (size_t)c * 4);
      const float acc = w.x * c0 + w.y * c1 + w.z * c2 + w.w * xn;
      y = acc * sigmoid_f(acc);
      cs[0] = cs[1];
      cs[1] = cs[2];
      cs[2] = x[(size_t)n * Cc + c];
    } else {
      y = xn;
    }
    smem[i] = y;  // qv | kvec | vv are contiguous in that order
  }
  if (tid < 2 * G) {
    const int h = hk * G + (tid >> 1);
    const size_t idx = (size_t)n * Hv + h;
    if ((tid & 1) == 0)
      gates[tid] = expf(gdn_log_decay(to_f32(a[idx]), A_log[h], dt_bias[h]));
    else
      gates[tid] = sigmoid_f(to_f32(b[idx]));
  }
  __syncthreads();
  // ---- 2. L2 norm of q and k (warps 0 and 1)
  if (tid < 64) {
    const float* src = tid < 32 ? qv : kvec;
    const int lane = tid & 31;
    float ss = 0.f;
    for (int i = lane; i < DK; i += 32) ss += src[i] * src[i];
    ss = warp_sum(ss);
    if (lane == 0) norm_ss[tid >> 5] = ss;
  }
  __syncthreads();
  {
    const float mq = rsqrtf(norm_ss[0] + 1e-6f) * scale;
    const float mk = rsqrtf(norm_ss[1] + 1e-6f);
    __syncthreads();
    for (int i = tid; i < DK; i += kThreads) {
      qv[i] *= mq;
      kvec[i] *= mk;
    }
  }
  __syncthreads();

  // ---- 3. state update per value head of the group
  const int col4 = tid % TPR;   // this thread's 4 columns: 4*col4 .. 4*col4+3
  const int rsub = tid / TPR;   // rows rsub, rsub+RPP, ...
  for (int g = 0; g < G; ++g) {
    const int hv = hk * G + g;
    float4* S = reinterpret_cast<float4*>(state + ((size_t)n * Hv + hv) * DK * DV);
    const float alpha = gates[2 * g], beta = gates[2 * g + 1];
    float4 s[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) s[p] = S[(size_t)(p * RPP + rsub) * TPR + col4];
    float4 kv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const float kr = kvec[p * RPP + rsub];
      s[p].x *= alpha; s[p].y *= alpha; s[p].z *= alpha; s[p].w *= alpha;
      kv.x += s[p].x * kr; kv.y += s[p].y * kr; kv.z += s[p].z * kr; kv.w += s[p].w * kr;
    }
    reinterpret_cast<float4*>(red + rsub * DV)[col4] = kv;
    __syncthreads();
    // every thread sums the RPP partials of its own 4 columns
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int r = 0; r < RPP; ++r) {
      const float4 t = reinterpret_cast<const float4*>(red + r * DV)[col4];
      tot.x += t.x; tot.y += t.y; tot.z += t.z; tot.w += t.w;
    }
    const float4 vj = reinterpret_cast<const float4*>(vv + g * DV)[col4];
    const float4 dl = make_float4(beta * (vj.x - tot.x), beta * (vj.y - tot.y),
                                  beta * (vj.z - tot.z), beta * (vj.w - tot.w));
    float4 oo = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int r = p * RPP + rsub;
      const float kr = kvec[r], qr = qv[r];
      s[p].x += kr * dl.x; s[p].y += kr * dl.y; s[p].z += kr * dl.z; s[p].w += kr * dl.w;
      S[(size_t)r * TPR + col4] = s[p];
      oo.x += s[p].x * qr; oo.y += s[p].y * qr; oo.z += s[p].z * qr; oo.w += s[p].w * qr;
    }
    __syncthreads();  // everyone has read `red`
    reinterpret_cast<float4*>(red + rsub * DV)[col4] = oo;
    __syncthreads();
    float acc = 0.f;
    if (tid < DV) {
#pragma unroll 4
      for (int r = 0; r < RPP; ++r) acc += red[r * DV + tid];
    }
    if (NORM) {  // sum of squares of the row over its DV columns (warps 0 .. DV/32-1)
      if (tid < DV) {
        const float ss = warp_sum(acc * acc);
        if ((tid & 31) == 0) row_ss[tid >> 5] = ss;
      }
      __syncthreads();
      if (tid < DV) {
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < DV / 32; ++w) ss += row_ss[w];
        const float zz = to_f32(nz[((size_t)n * Hv + hv) * DV + tid]);
        acc *= rsqrtf(ss * (1.f / DV) + neps) * nw[tid] * (zz * sigmoid_f(zz));
      }
    }
    if (tid < DV) o[((size_t)n * Hv + hv) * DV + tid] = from_f32<TO>(acc);
    __syncthreads();
  }
}

template <typename T, typename TO, int DK, int DV>
cudaError_t launch_t(const void* x, const float* conv_w, void* conv_state, const void* a,
                     const void* b, const float* A_log, const float* dt_bias, float* state,
                     void* o, int N, int Hk, int Hv, float scale, const DecodeNorm& nm,
                     cudaStream_t s) {
  const int G = Hv / Hk;
  constexpr int RPP = kThreads / (DV / 4);
  const size_t smem = sizeof(float) * (2 * DK + G * DV + RPP * DV + 2 * G);
  auto kern = nm.z ? decode_step_kernel<T, TO, DK, DV, true>
                   : decode_step_kernel<T, TO, DK, DV, false>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<(unsigned)(N * Hk), kThreads, smem, s>>>(
      (const T*)x, conv_w, (T*)conv_state, (const T*)a, (const T*)b, A_log, dt_bias, state,
      (TO*)o, Hk, Hv, scale, static_cast<const T*>(nm.z), nm.w, nm.eps);
  return cudaGetLastError();
}

template <typename T, typename TO>
cudaError_t launch_dt(int dk, int dv, const void* x, const float* conv_w, void* conv_state,
                      const void* a, const void* b, const float* A_log, const float* dt_bias,
                      float* state, void* o, int N, int Hk, int Hv, float scale,
                      const DecodeNorm& nm, cudaStream_t s) {
#define GDN_DEC(DK_, DV_)                                                               \
  if (dk == DK_ && dv == DV_)                                                           \
    return launch_t<T, TO, DK_, DV_>(x, conv_w, conv_state, a, b, A_log, dt_bias, state, o, \
                                 N, Hk, Hv, scale, nm, s);
  GDN_DEC(64, 64) GDN_DEC(64, 128) GDN_DEC(128, 64) GDN_DEC(128, 128)
#undef GDN_DEC
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent_step(const void* x, const float* conv_w, void* conv_state,
                                  const void* a, const void* b, const float* A_log,
                                  const float* dt_bias, float* state, void* o, int N,
                                  int Hk, int Hv, int dk, int dv, int dtype, float scale,
                                  bool out_f32, const DecodeNorm& nm, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  if (dtype == GDN_BF16)
    return out_f32 ? launch_dt<__nv_bfloat16, float>(dk, dv, x, conv_w, conv_state, a, b, A_log,
                                                     dt_bias, state, o, N, Hk, Hv, scale, nm, s)
                   : launch_dt<__nv_bfloat16, __nv_bfloat16>(dk, dv, x, conv_w, conv_state, a,
                                                             b, A_log, dt_bias, state, o, N, Hk,
                                                             Hv, scale, nm, s);
  return launch_dt<float, float>(dk, dv, x, conv_w, conv_state, a, b, A_log, dt_bias, state, o,
                                 N, Hk, Hv, scale, nm, s);
}

}  // namespace gdn
