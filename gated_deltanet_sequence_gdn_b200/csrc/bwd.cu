// bwd.cu -- the backward pass of the GDN chunk forward (gdn_chunk_bwd), in fp32
// on the CUDA cores.
//
// The gradients of sum(o * do) + sum(ht * dht) with respect to q, k, v, the gate
// inputs, A_log, dt_bias and h0, by reverse-mode differentiation of the WY chunk
// form ("Gated DeltaNet-2", sections 高效训练：WY 算法依然成立 and Gate-aware 反向传播;
// GDN is its scalar-decay case).  Per chunk of C = 64 tokens and value head, with
// G the in-chunk prefix sum of the log-decays g, gamma = e^G, gamma_C its last
// entry, Gamma_rj = e^{G_r - G_j} (j <= r), the forward is
//   L = tril(diag(beta) (K K^T o Gamma), -1),  A = (I + L)^-1,
//   W = A diag(beta gamma) K,  U = A diag(beta) V,  A_qk = tril(Q K^T o Gamma),
//   U~ = U - W S0,  O = diag(gamma) Q S0 + A_qk U~,
//   S1 = gamma_C S0 + K~^T U~,  K~ = diag(gamma_C / gamma) K,
// and the backward runs it in reverse:
//   - a forward scan over the chunks recomputes every chunk's start state S0 and
//     U~ (the state is not stored by the forward call);
//   - a reverse scan carries the state gradient dS from the last chunk to the
//     first: dU~ = K~ dS1 + A_qk^T dO,  dS0 = gamma_C dS1 + (diag(gamma) Q)^T dO
//     - W^T dU~ (its final value is dh0);
//   - per chunk, independent of the others: dQ = diag(gamma) dO S0^T + dQK K,
//     dW = -dU~ S0^T, dA = dU~ (diag(beta) V)^T + dW (diag(beta gamma) K)^T,
//     dV = diag(beta) A^T dU~, dK from A^T dW, from dL = tril(-A^T dA A^T, -1)
//     through K K^T, from dQK = dA_qk o Gamma through Q K^T and from K~, dbeta, and
//     the gradient of G collected from every place it enters and summed back to
//     the log-decays by a reverse cumulative sum;
//   - last, the chain rule through the L2 norms of q and k (summed over the value
//     heads of a key head) and through the gates.
// The in-chunk products run through one batched kernel (bmm_kernel) over all
// (value head, chunk) pairs; the scans hold a 64-column slice of the d_k x d_v
// state per CTA in shared memory.  All arithmetic is fp32 whatever the input
// type (the fp32 bar of 1e-4 holds for both).
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kC = 64;
constexpr int kNS = 64;  // state columns per scan CTA

struct Dims {
  int B, T, Hk, Hv, D, Tp, Nc;
};

// A matrix operand of the batched products, one per (value head h, chunk c):
//  kTV: token rows of a value head, [B*Hv][Tp][D] (64 rows x D from row 64 c)
//  kTK: token rows of the key head of h, [B*Hk][Tp][D]
//  kDD: one D x D matrix per (h, c), [B*Hv*Nc][D][D]
//  kCC: one 64 x 64 matrix per (h, c), [B*Hv*Nc][64][64]
enum { kTV = 0, kTK = 1, kDD = 2, kCC = 3 };
struct Opnd {
  const float* p;
  int kind;
  int t;  // 1: the operand enters transposed
};

__device__ __forceinline__ size_t opnd_off(int kind, int z, const Dims& d) {
  const int h = z / d.Nc, c = z % d.Nc;
  switch (kind) {
    case kTV:
      return ((size_t)h * d.Tp + (size_t)c * kC) * d.D;
    case kTK: {
      const int b = h / d.Hv, hv = h % d.Hv;
      const int kh = b * d.Hk + hv / (d.Hv / d.Hk);
      return ((size_t)kh * d.Tp + (size_t)c * kC) * d.D;
    }
    case kDD:
      return (size_t)z * d.D * d.D;
    default:
      return (size_t)z * kC * kC;
  }
}
__device__ __forceinline__ int opnd_ld(int kind, const Dims& d) { return kind == kCC ? kC : d.D; }

// Scale vectors taken from the chunk's (G, beta): none, beta, beta gamma, gamma.
enum { kScNone = 0, kScBeta = 1, kScBetaGamma = 2, kScGamma = 3 };
// Output masks: none, j <= r, j < r.
enum { kMaskNone = 0, kMaskLower = 1, kMaskStrict = 2 };

struct BmmArgs {
  Opnd x, y;          // out[M x N] = alpha op(x)[M x K] diag(ks) op(y)[K x N]
  float* out;
  int out_kind;       // kTV (M = 64, N = D), kCC (M = N = 64) or kDD (M = N = D)
  int M, N, K;
  float alpha;
  int kscale, rscale, cscale, mask;  // kscale needs K = 64, rscale M = 64, cscale N = 64
  int accumulate;
  const float2* gb;   // (G, beta) per [B*Hv][Tp]
};

// Batched product, one 64 x 64 output tile per CTA (blockIdx.x: (h, c),
// blockIdx.y: column tile, blockIdx.z: row tile); 256 threads with 4 x 4 outputs
// each; K in steps of 32 through shared memory.
template <bool XT, bool YT>
__global__ void __launch_bounds__(256, 3) bmm_kernel(BmmArgs P, Dims d) {
  __shared__ __align__(16) float Xs[32][68];
  __shared__ __align__(16) float Ys[32][68];
  __shared__ float sv[3][kC];
  const int z = blockIdx.x, n0 = blockIdx.y * 64, m0 = blockIdx.z * 64, tid = threadIdx.x;
  const int h = z / d.Nc, c = z % d.Nc;
  const float* X = P.x.p + opnd_off(P.x.kind, z, d);
  const float* Y = P.y.p + opnd_off(P.y.kind, z, d);
  const int ldx = opnd_ld(P.x.kind, d), ldy = opnd_ld(P.y.kind, d);
  if (tid < kC) {
    const float2 gb = P.gb[(size_t)h * d.Tp + (size_t)c * kC + tid];
    const int modes[3] = {P.kscale, P.rscale, P.cscale};
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int m = modes[i];
      sv[i][tid] = m == kScNone ? 1.f
                   : m == kScBeta ? gb.y
                   : m == kScBetaGamma ? gb.y * expf(gb.x)
                                       : expf(gb.x);
    }
  }
  const int tm = tid >> 4, tn = tid & 15;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < P.K; k0 += 32) {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = tid + 256 * u;
      if (!XT) Xs[i & 31][i >> 5] = X[(size_t)(m0 + (i >> 5)) * ldx + k0 + (i & 31)];
      else Xs[i >> 6][i & 63] = X[(size_t)(k0 + (i >> 6)) * ldx + m0 + (i & 63)];
      if (!YT) Ys[i >> 6][i & 63] = Y[(size_t)(k0 + (i >> 6)) * ldy + n0 + (i & 63)];
      else Ys[i & 31][i >> 5] = Y[(size_t)(n0 + (i >> 5)) * ldy + k0 + (i & 31)];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const float ks = P.kscale != kScNone ? sv[0][k0 + k] : 1.f;
      const float4 a = *reinterpret_cast<const float4*>(&Xs[k][4 * tm]);
      float4 b = *reinterpret_cast<const float4*>(&Ys[k][4 * tn]);
      b.x *= ks, b.y *= ks, b.z *= ks, b.w *= ks;
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  float* out = P.out + (P.out_kind == kCC   ? (size_t)z * kC * kC
                        : P.out_kind == kDD ? (size_t)z * d.D * d.D + (size_t)m0 * d.D
                                            : ((size_t)h * d.Tp + (size_t)c * kC) * d.D);
  const int ldo = P.out_kind == kCC ? kC : d.D;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 4 * tm + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + 4 * tn + j;
      float v = P.alpha * acc[i][j] * (P.rscale != kScNone ? sv[1][r] : 1.f);
      if (P.cscale != kScNone) v *= sv[2][col];
      if ((P.mask == kMaskLower && col > r) || (P.mask == kMaskStrict && col >= r)) v = 0.f;
      float* o = out + (size_t)r * ldo + col;
      *o = P.accumulate ? *o + v : v;
    }
  }
}

// ------------------------------------------------------------------ token prep
// q^ = scale q / sqrt(sum q^2 + 1e-6) (or scale q), k^ likewise with scale 1, as
// fp32 rows [B*Hk][Tp][D]; rows past T are zero.  One warp per (b, t, key head).
template <typename T>
__global__ void qk_prep_kernel(const T* __restrict__ q, const T* __restrict__ k, float* QN,
                               float* KN, Dims d, float scale, int l2) {
  const long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long rows = (long)d.B * d.Hk * d.Tp;
  if (row >= rows) return;
  const int t = (int)(row % d.Tp);
  const long kh = row / d.Tp;  // b * Hk + hk
  const int b = (int)(kh / d.Hk), hk = (int)(kh % d.Hk);
  float* qo = QN + row * d.D;
  float* ko = KN + row * d.D;
  if (t >= d.T) {
    for (int i = lane; i < d.D; i += 32) qo[i] = 0.f, ko[i] = 0.f;
    return;
  }
  const size_t in = (((size_t)b * d.T + t) * d.Hk + hk) * d.D;
  float sq = 0.f, sk = 0.f;
  for (int i = lane; i < d.D; i += 32) {
    const float a = to_f32(q[in + i]), c = to_f32(k[in + i]);
    sq = fmaf(a, a, sq), sk = fmaf(c, c, sk);
  }
  sq = warp_sum(sq), sk = warp_sum(sk);
  const float fq = (l2 ? rsqrtf(sq + 1e-6f) : 1.f) * scale, fk = l2 ? rsqrtf(sk + 1e-6f) : 1.f;
  for (int i = lane; i < d.D; i += 32) {
    qo[i] = to_f32(q[in + i]) * fq;
    ko[i] = to_f32(k[in + i]) * fk;
  }
}

// v and do as fp32 rows [B*Hv][Tp][D] (zero past T).
template <typename T>
__global__ void tok_prep_kernel(const T* __restrict__ v, const T* __restrict__ dout, float* V32,
                                float* dO32, Dims d) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long n = (long)d.B * d.Hv * d.Tp * d.D;
  if (i >= n) return;
  const int col = (int)(i % d.D);
  const long row = i / d.D;
  const int t = (int)(row % d.Tp);
  const long h = row / d.Tp;
  const int b = (int)(h / d.Hv), hv = (int)(h % d.Hv);
  float vv = 0.f, dd = 0.f;
  if (t < d.T) {
    const size_t in = (((size_t)b * d.T + t) * d.Hv + hv) * d.D + col;
    vv = to_f32(v[in]);
    dd = to_f32(dout[in]);
  }
  V32[i] = vv;
  dO32[i] = dd;
}

// (G, beta) per token: g from the gate logits (or given), its inclusive prefix
// sum inside the chunk; tokens past T carry g = 0, beta = 0.  One CTA of 64
// threads per (h, chunk).
template <typename T>
__global__ void gates_prep_kernel(const void* a_, const void* b_, const float* A_log,
                                  const float* dt_bias, float2* GB, Dims d, int pre) {
  __shared__ float part[2];
  const int c = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int b = h / d.Hv, hv = h % d.Hv;
  const int t = c * kC + tid;
  float g = 0.f, be = 0.f;
  if (t < d.T) {
    const size_t idx = ((size_t)b * d.T + t) * d.Hv + hv;
    if (pre) {
      g = static_cast<const float*>(a_)[idx];
      be = static_cast<const float*>(b_)[idx];
    } else {
      g = gdn_log_decay(to_f32(static_cast<const T*>(a_)[idx]), A_log[hv], dt_bias[hv]);
      be = sigmoid_f(to_f32(static_cast<const T*>(b_)[idx]));
    }
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, g, o);
    if (lane >= o) g += y;
  }
  if (lane == 31) part[tid >> 5] = g;
  __syncthreads();
  if (tid >= 32) g += part[0];
  GB[(size_t)h * d.Tp + t] = make_float2(g, be);
}

// ------------------------------------------------------------------ chunk prep
// From the raw Gram products KK = K K^T and QK = Q K^T: L = tril(beta_r KK o
// Gamma, -1) into Lb and A_qk = tril(QK o Gamma) into Aq.  One CTA per (h, c).
__global__ void __launch_bounds__(256) gram_gates_kernel(const float* KK, const float* QK,
                                                         const float2* GB, float* Lb, float* Aq,
                                                         Dims d) {
  __shared__ float G[kC], be[kC];
  const int z = blockIdx.x, h = z / d.Nc, c = z % d.Nc, tid = threadIdx.x;
  if (tid < kC) {
    const float2 gb = GB[(size_t)h * d.Tp + (size_t)c * kC + tid];
    G[tid] = gb.x, be[tid] = gb.y;
  }
  __syncthreads();
  const size_t base = (size_t)z * kC * kC;
  for (int i = tid; i < kC * kC; i += 256) {
    const int r = i >> 6, j = i & 63;
    const float gam = j <= r ? expf(G[r] - G[j]) : 0.f;
    Lb[base + i] = j < r ? be[r] * KK[base + i] * gam : 0.f;
    Aq[base + i] = QK[base + i] * gam;
  }
}

// A = (I + L)^-1 in place for one strictly lower L per CTA, by forward
// substitution down each column (64 threads, one column each).
__global__ void __launch_bounds__(64) tri_inverse_kernel(float* Lb) {
  __shared__ float L[kC][kC + 1], X[kC][kC + 1];
  const int z = blockIdx.x, c = threadIdx.x;
  float* M = Lb + (size_t)z * kC * kC;
  for (int r = 0; r < kC; ++r) L[r][c] = M[r * kC + c];
  __syncthreads();
  for (int r = 0; r < kC; ++r) {
    float s = r == c ? 1.f : 0.f;
    for (int j = c; j < r; ++j) s = fmaf(-L[r][j], X[j][c], s);
    X[r][c] = r < c ? 0.f : s;
  }
  __syncthreads();
  for (int r = 0; r < kC; ++r) M[r * kC + c] = X[r][c];
}

// ------------------------------------------------------------------ the scans
// 16-byte asynchronous copies of a [64][D] fp32 tile into shared rows of D + 4.
template <int D>
__device__ __forceinline__ void tile_async(float* dst, const float* src, int tid) {
#pragma unroll
  for (int u = 0; u < kC * D / 4 / 256; ++u) {
    const int i = tid + 256 * u, r = i / (D / 4), q4 = i % (D / 4);
    const uint32_t sa = (uint32_t)__cvta_generic_to_shared(dst + r * (D + 4) + 4 * q4);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa),
                 "l"(src + (size_t)r * D + 4 * q4)
                 : "memory");
  }
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void async_wait_prev() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Shared memory of the scans: W and K tiles twice (the next chunk's land while
// the current one is used), the state (or its gradient) slice and a 64 x kNS
// row block.
template <int D>
constexpr size_t scan_smem_bytes() {
  return (size_t)(4 * kC * (D + 4) + D * (kNS + 4) + kC * (kNS + 4) + kC) * 4;
}

// Forward: S0 of every chunk (the state before it, slice of kNS columns) and
// U~ = U - W S0 (in place over U).  One CTA per (slice, h); 256 threads.
template <int D>
__global__ void __launch_bounds__(256) fwd_state_scan_kernel(const float* Wm, float* Um,
                                                             const float* KN, const float2* GB,
                                                             const float* h0, float* S0, Dims d) {
  extern __shared__ __align__(16) float sm[];
  float* Wb = sm;                          // [2][64][D + 4]
  float* Kb = Wb + 2 * kC * (D + 4);       // [2][64][D + 4]
  float* S = Kb + 2 * kC * (D + 4);        // [D][kNS + 4]
  float* Us = S + D * (kNS + 4);           // [64][kNS + 4]
  float* ratio = Us + kC * (kNS + 4);      // [64]
  const int n0 = blockIdx.x * kNS, h = blockIdx.y, tid = threadIdx.x;
  const int b = h / d.Hv, hv = h % d.Hv, kh = b * d.Hk + hv / (d.Hv / d.Hk);
  for (int i = tid; i < D * kNS; i += 256) {
    const int k = i / kNS, n = i % kNS;
    S[k * (kNS + 4) + n] = h0 ? h0[((size_t)h * D + k) * D + n0 + n] : 0.f;
  }
  auto rowv = [&](int c) { return ((size_t)h * d.Tp + (size_t)c * kC) * D; };
  auto rowk = [&](int c) { return ((size_t)kh * d.Tp + (size_t)c * kC) * D; };
  tile_async<D>(Wb, Wm + rowv(0), tid);
  tile_async<D>(Kb, KN + rowk(0), tid);
  async_commit();
  const int tm = tid >> 4, tn = tid & 15;
  for (int c = 0; c < d.Nc; ++c) {
    const size_t z = (size_t)h * d.Nc + c, rv = rowv(c);
    const float* Ws = Wb + (c & 1) * kC * (D + 4);
    const float* Ks = Kb + (c & 1) * kC * (D + 4);
    if (c + 1 < d.Nc) {  // the next chunk's tiles, into the other buffers
      tile_async<D>(Wb + ((c + 1) & 1) * kC * (D + 4), Wm + rowv(c + 1), tid);
      tile_async<D>(Kb + ((c + 1) & 1) * kC * (D + 4), KN + rowk(c + 1), tid);
    }
    async_commit();
    async_wait_prev();  // this chunk's tiles have landed (this thread's copies)
    if (tid < kC) {
      const float G = GB[(size_t)h * d.Tp + (size_t)c * kC + tid].x;
      const float GC = GB[(size_t)h * d.Tp + (size_t)c * kC + kC - 1].x;
      ratio[tid] = expf(GC - G);
    }
    for (int i = tid; i < D * kNS; i += 256) {
      const int k = i / kNS, n = i % kNS;
      S0[z * D * D + (size_t)k * D + n0 + n] = S[k * (kNS + 4) + n];
    }
    __syncthreads();  // every thread's copies, S and ratio are visible
    // U~ = U - W S0: rows 4 tm .. 4 tm + 3, columns 4 tn .. 4 tn + 3
    {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float4 s4 = *reinterpret_cast<const float4*>(&S[k * (kNS + 4) + 4 * tn]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float w = Ws[(4 * tm + i) * (D + 4) + k];
          acc[i][0] = fmaf(w, s4.x, acc[i][0]);
          acc[i][1] = fmaf(w, s4.y, acc[i][1]);
          acc[i][2] = fmaf(w, s4.z, acc[i][2]);
          acc[i][3] = fmaf(w, s4.w, acc[i][3]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * tm + i;
        const float4 u4 = *reinterpret_cast<const float4*>(&Um[rv + (size_t)r * D + n0 + 4 * tn]);
        const float4 o4 = make_float4(u4.x - acc[i][0], u4.y - acc[i][1], u4.z - acc[i][2],
                                      u4.w - acc[i][3]);
        *reinterpret_cast<float4*>(&Um[rv + (size_t)r * D + n0 + 4 * tn]) = o4;
        *reinterpret_cast<float4*>(&Us[r * (kNS + 4) + 4 * tn]) = o4;
      }
    }
    __syncthreads();
    // S <- gamma_C S + K~^T U~: rows (d_k) k0 .. k0 + 7 with k0 = 8 tm (+ 128),
    // columns 4 tn .. + 3
    {
      const float gC = expf(GB[(size_t)h * d.Tp + (size_t)c * kC + kC - 1].x);
      for (int k0 = 8 * tm; k0 < D; k0 += 128) {
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int r = 0; r < kC; ++r) {
          const float4 u4 = *reinterpret_cast<const float4*>(&Us[r * (kNS + 4) + 4 * tn]);
          const float rr = ratio[r];
          const float4 ka = *reinterpret_cast<const float4*>(&Ks[r * (D + 4) + k0]);
          const float4 kb = *reinterpret_cast<const float4*>(&Ks[r * (D + 4) + k0 + 4]);
          const float kv[8] = {ka.x * rr, ka.y * rr, ka.z * rr, ka.w * rr,
                               kb.x * rr, kb.y * rr, kb.z * rr, kb.w * rr};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[i][0] = fmaf(kv[i], u4.x, acc[i][0]);
            acc[i][1] = fmaf(kv[i], u4.y, acc[i][1]);
            acc[i][2] = fmaf(kv[i], u4.z, acc[i][2]);
            acc[i][3] = fmaf(kv[i], u4.w, acc[i][3]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float* s = &S[(k0 + i) * (kNS + 4) + 4 * tn + j];
            *s = fmaf(gC, *s, acc[i][j]);
          }
      }
    }
    __syncthreads();  // the buffers of this chunk are free for the chunk after next
  }
}

// Reverse: dS1 of every chunk (the state gradient after it) and dU~; the final dS
// is dh0.  The terms that do not depend on dS come precomputed: P1 = A_qk^T dO in
// dUt (replaced by dU~ in place) and P2 = (diag(gamma) Q)^T dO per chunk.  One
// CTA per (slice, h); 256 threads.
template <int D>
__global__ void __launch_bounds__(256) rev_state_scan_kernel(const float* Wm, const float* KN,
                                                             const float* P2, const float2* GB,
                                                             const float* dht, float* dS1,
                                                             float* dUt, float* dh0, Dims d) {
  extern __shared__ __align__(16) float sm[];
  float* Wb = sm;                          // [2][64][D + 4]
  float* Kb = Wb + 2 * kC * (D + 4);       // [2][64][D + 4]
  float* dS = Kb + 2 * kC * (D + 4);       // [D][kNS + 4]
  float* dUs = dS + D * (kNS + 4);         // [64][kNS + 4]
  float* ratio = dUs + kC * (kNS + 4);     // [64]
  const int n0 = blockIdx.x * kNS, h = blockIdx.y, tid = threadIdx.x;
  const int b = h / d.Hv, hv = h % d.Hv, kh = b * d.Hk + hv / (d.Hv / d.Hk);
  for (int i = tid; i < D * kNS; i += 256) {
    const int k = i / kNS, n = i % kNS;
    dS[k * (kNS + 4) + n] = dht ? dht[((size_t)h * D + k) * D + n0 + n] : 0.f;
  }
  auto rowv = [&](int c) { return ((size_t)h * d.Tp + (size_t)c * kC) * D; };
  auto rowk = [&](int c) { return ((size_t)kh * d.Tp + (size_t)c * kC) * D; };
  const int last = d.Nc - 1;
  tile_async<D>(Wb + (last & 1) * kC * (D + 4), Wm + rowv(last), tid);
  tile_async<D>(Kb + (last & 1) * kC * (D + 4), KN + rowk(last), tid);
  async_commit();
  const int tm = tid >> 4, tn = tid & 15;
  for (int c = last; c >= 0; --c) {
    const size_t z = (size_t)h * d.Nc + c, rv = rowv(c);
    const float* Ws = Wb + (c & 1) * kC * (D + 4);
    const float* Ks = Kb + (c & 1) * kC * (D + 4);
    if (c > 0) {  // the previous chunk's tiles, into the other buffers
      tile_async<D>(Wb + ((c - 1) & 1) * kC * (D + 4), Wm + rowv(c - 1), tid);
      tile_async<D>(Kb + ((c - 1) & 1) * kC * (D + 4), KN + rowk(c - 1), tid);
    }
    async_commit();
    async_wait_prev();
    if (tid < kC) {
      const float G = GB[(size_t)h * d.Tp + (size_t)c * kC + tid].x;
      const float GC = GB[(size_t)h * d.Tp + (size_t)c * kC + kC - 1].x;
      ratio[tid] = expf(GC - G);
    }
    for (int i = tid; i < D * kNS; i += 256) {
      const int k = i / kNS, n = i % kNS;
      dS1[z * D * D + (size_t)k * D + n0 + n] = dS[k * (kNS + 4) + n];
    }
    __syncthreads();
    // dU~ = K~ dS1 + P1
    {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float4 s4 = *reinterpret_cast<const float4*>(&dS[k * (kNS + 4) + 4 * tn]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float kv = Ks[(4 * tm + i) * (D + 4) + k];
          acc[i][0] = fmaf(kv, s4.x, acc[i][0]);
          acc[i][1] = fmaf(kv, s4.y, acc[i][1]);
          acc[i][2] = fmaf(kv, s4.z, acc[i][2]);
          acc[i][3] = fmaf(kv, s4.w, acc[i][3]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * tm + i;
        const float rr = ratio[r];
        float* g = &dUt[rv + (size_t)r * D + n0 + 4 * tn];
        const float4 p4 = *reinterpret_cast<const float4*>(g);
        const float4 o4 = make_float4(fmaf(rr, acc[i][0], p4.x), fmaf(rr, acc[i][1], p4.y),
                                      fmaf(rr, acc[i][2], p4.z), fmaf(rr, acc[i][3], p4.w));
        *reinterpret_cast<float4*>(g) = o4;
        *reinterpret_cast<float4*>(&dUs[r * (kNS + 4) + 4 * tn]) = o4;
      }
    }
    __syncthreads();
    // dS <- gamma_C dS + P2 - W^T dU~
    {
      const float gC = expf(GB[(size_t)h * d.Tp + (size_t)c * kC + kC - 1].x);
      for (int k0 = 8 * tm; k0 < D; k0 += 128) {
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int r = 0; r < kC; ++r) {
          const float4 u4 = *reinterpret_cast<const float4*>(&dUs[r * (kNS + 4) + 4 * tn]);
          const float4 wa = *reinterpret_cast<const float4*>(&Ws[r * (D + 4) + k0]);
          const float4 wb = *reinterpret_cast<const float4*>(&Ws[r * (D + 4) + k0 + 4]);
          const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[i][0] = fmaf(wv[i], u4.x, acc[i][0]);
            acc[i][1] = fmaf(wv[i], u4.y, acc[i][1]);
            acc[i][2] = fmaf(wv[i], u4.z, acc[i][2]);
            acc[i][3] = fmaf(wv[i], u4.w, acc[i][3]);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 p4 =
              *reinterpret_cast<const float4*>(&P2[z * D * D + (size_t)(k0 + i) * D + n0 + 4 * tn]);
          const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float* s = &dS[(k0 + i) * (kNS + 4) + 4 * tn + j];
            *s = fmaf(gC, *s, pv[j] - acc[i][j]);
          }
        }
      }
    }
    __syncthreads();
  }
  if (dh0)
    for (int i = tid; i < D * kNS; i += 256) {
      const int k = i / kNS, n = i % kNS;
      dh0[((size_t)h * D + k) * D + n0 + n] = dS[k * (kNS + 4) + n];
    }
}

// ------------------------------------------------------------------ chunk-local
// Per chunk scalars and rows (float4 per row of (h, c)): x = dgam, y = dbeta,
// z = dG collected from the Gamma masks, w unused.  dgam starts as
// rowsum(dO o Q S0); dgC = <dS1, S0> per chunk.
// The row kernels below take one warp per token row (8 rows per warp), the lanes
// over the row's D columns, so every access is a coalesced row segment.
__global__ void __launch_bounds__(256) dgam_kernel(const float* dO32, const float* QS,
                                                   float4* VB, Dims d) {
  const int z = blockIdx.x, h = z / d.Nc, c = z % d.Nc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t rv = ((size_t)h * d.Tp + (size_t)c * kC) * d.D;
  for (int r = warp; r < kC; r += 8) {
    float s = 0.f;
    for (int i = lane; i < d.D; i += 32) {
      const size_t e = rv + (size_t)r * d.D + i;
      s = fmaf(dO32[e], QS[e], s);
    }
    s = warp_sum(s);
    if (lane == 0) VB[(size_t)z * kC + r] = make_float4(s, 0.f, 0.f, 0.f);
  }
}

__global__ void __launch_bounds__(256) dgc_kernel(const float* dS1, const float* S0, float* SC,
                                                  Dims d) {
  __shared__ float red[8];
  const int z = blockIdx.x, tid = threadIdx.x;
  const size_t n = (size_t)d.D * d.D, base = (size_t)z * n;
  float s = 0.f;
  for (size_t i = tid; i < n; i += 256) s = fmaf(dS1[base + i], S0[base + i], s);
  s = warp_sum(s);
  if ((tid & 31) == 0) red[tid >> 5] = s;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i];
    SC[z] = t;
  }
}

// After dVb = A^T dU~ and dKb = A^T dW: dv = beta dVb (to the output), dK = beta
// gamma dKb (starts the dK buffer), dbeta = rowsum(dVb o V) + gamma rowsum(dKb o
// K), dgam += beta rowsum(dKb o K).
__global__ void __launch_bounds__(256) vb_kernel(const float* dVb, const float* dKb,
                                                 const float* V32, const float* KN,
                                                 const float2* GB, float* dK, float4* VB,
                                                 float* dv_out, Dims d) {
  const int z = blockIdx.x, h = z / d.Nc, c = z % d.Nc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = h / d.Hv, hv = h % d.Hv, kh = b * d.Hk + hv / (d.Hv / d.Hk);
  const size_t rv = ((size_t)h * d.Tp + (size_t)c * kC) * d.D;
  const size_t rk = ((size_t)kh * d.Tp + (size_t)c * kC) * d.D;
  for (int r = warp; r < kC; r += 8) {
    const float2 gb = GB[(size_t)h * d.Tp + (size_t)c * kC + r];
    const float be = gb.y, gm = expf(gb.x);
    const int t = c * kC + r;
    float s1 = 0.f, s2 = 0.f;
    for (int i = lane; i < d.D; i += 32) {
      const size_t e = rv + (size_t)r * d.D + i;
      const float vb = dVb[e], kb = dKb[e];
      s1 = fmaf(vb, V32[e], s1);
      s2 = fmaf(kb, KN[rk + (size_t)r * d.D + i], s2);
      dK[e] = be * gm * kb;
      if (t < d.T) dv_out[(((size_t)b * d.T + t) * d.Hv + hv) * d.D + i] = be * vb;
    }
    s1 = warp_sum(s1), s2 = warp_sum(s2);
    if (lane == 0) {
      float4 v = VB[(size_t)z * kC + r];
      v.x += be * s2;
      v.y = s1 + gm * s2;
      VB[(size_t)z * kC + r] = v;
    }
  }
}

// After dL = tril(-A^T dA A^T, -1): with M = KK o Gamma, dbeta += rowsum(dL o
// M), dM = beta dL, dKK = dM o Gamma (in place of KK), dQK = dA_qk o Gamma (in
// place of QK), and the Gamma gradient tG = (dM o KK + dA_qk o QK) o Gamma
// reduced to rowsum - colsum (into VB.z).
__global__ void __launch_bounds__(256) dl_kernel(const float* dL, const float* dAqk, float* KK,
                                                 float* QK, const float2* GB, float4* VB,
                                                 Dims d) {
  __shared__ float tG[kC][kC + 1];
  __shared__ float G[kC], be[kC], dbl[kC][4];
  const int z = blockIdx.x, h = z / d.Nc, c = z % d.Nc, tid = threadIdx.x;
  if (tid < kC) {
    const float2 gb = GB[(size_t)h * d.Tp + (size_t)c * kC + tid];
    G[tid] = gb.x, be[tid] = gb.y;
  }
  __syncthreads();
  const size_t base = (size_t)z * kC * kC;
  // row r = tid / 4, columns j = part, part + 4, ...
  const int r = tid >> 2, part = tid & 3;
  float db = 0.f;
  for (int j = part; j < kC; j += 4) {
    const size_t e = base + (size_t)r * kC + j;
    const float gam = j <= r ? expf(G[r] - G[j]) : 0.f;
    const float kk = KK[e], qk = QK[e], dl = dL[e], da = dAqk[e];
    db = fmaf(dl, kk * gam, db);
    const float dM = be[r] * dl;
    KK[e] = dM * gam;
    QK[e] = da * gam;
    tG[r][j] = (dM * kk + da * qk) * gam;
  }
  dbl[r][part] = db;
  __syncthreads();
  if (tid < kC) {
    float rs = 0.f, cs = 0.f;
    for (int j = 0; j < kC; ++j) rs += tG[tid][j];
    for (int i = 0; i < kC; ++i) cs += tG[i][tid];
    float4 v = VB[(size_t)z * kC + tid];
    v.y += dbl[tid][0] + dbl[tid][1] + dbl[tid][2] + dbl[tid][3];
    v.z = rs - cs;
    VB[(size_t)z * kC + tid] = v;
  }
}

// Last per-chunk step: dK += ratio dK~ (K~ = diag(ratio) K, ratio = gamma_C /
// gamma), the G gradient dG = (rowsum - colsum of tG) + dgam gamma - dratio ratio
// with the gamma_C terms on the last row, then dg = the reverse cumulative sum
// of dG inside the chunk.  Writes (dg, dbeta) per token into DG.
__global__ void __launch_bounds__(256) dg_kernel(const float* dKt, const float* KN,
                                                 const float2* GB, const float4* VB,
                                                 const float* SC, float* dK, float2* DG,
                                                 Dims d) {
  __shared__ float dG[kC], rrat[kC];
  const int z = blockIdx.x, h = z / d.Nc, c = z % d.Nc, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int b = h / d.Hv, hv = h % d.Hv, kh = b * d.Hk + hv / (d.Hv / d.Hk);
  const size_t rv = ((size_t)h * d.Tp + (size_t)c * kC) * d.D;
  const size_t rk = ((size_t)kh * d.Tp + (size_t)c * kC) * d.D;
  const float GC = GB[(size_t)h * d.Tp + (size_t)c * kC + kC - 1].x;
  for (int r = warp; r < kC; r += 8) {
    const float G = GB[(size_t)h * d.Tp + (size_t)c * kC + r].x;
    const float ratio = expf(GC - G), gm = expf(G);
    float dratio = 0.f;
    for (int i = lane; i < d.D; i += 32) {
      const size_t e = rv + (size_t)r * d.D + i;
      const float kt = dKt[e];
      dratio = fmaf(kt, KN[rk + (size_t)r * d.D + i], dratio);
      dK[e] = fmaf(ratio, kt, dK[e]);
    }
    dratio = warp_sum(dratio);
    if (lane == 0) {
      const float4 v = VB[(size_t)z * kC + r];
      dG[r] = v.z + v.x * gm - dratio * ratio;
      rrat[r] = dratio * ratio;
    }
  }
  __syncthreads();
  if (tid < 32) {  // the last row's gamma_C terms, then the reverse cumulative sum
    float s = rrat[tid] + rrat[tid + 32];
    s = warp_sum(s);
    if (tid == 0) dG[kC - 1] += s + SC[z] * expf(GC);
  }
  __syncthreads();
  if (tid == 0) {
    float run = 0.f;
    for (int i = kC - 1; i >= 0; --i) {
      run += dG[i];
      dG[i] = run;
    }
  }
  __syncthreads();
  if (tid < kC) {
    const int t = c * kC + tid;
    if (t < d.T) DG[(size_t)h * d.Tp + t] = make_float2(dG[tid], VB[(size_t)z * kC + tid].y);
  }
}

// ------------------------------------------------------------------ the chain rule
// dq, dk [B,T,Hk,D]: the gradients of the normalised rows summed over the value
// heads of the key head, through x -> scale x / sqrt(sum x^2 + 1e-6).
template <typename T>
__global__ void finish_qk_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                 const float* dQ, const float* dK, float* dq, float* dk,
                                 Dims d, float scale, int l2) {
  const long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= (long)d.B * d.T * d.Hk) return;
  const int hk = (int)(row % d.Hk);
  const long bt = row / d.Hk;
  const int t = (int)(bt % d.T), b = (int)(bt / d.T);
  const int G = d.Hv / d.Hk;
  const size_t in = (size_t)row * d.D;
  for (int which = 0; which < 2; ++which) {
    const T* x = which ? k : q;
    const float* g = which ? dK : dQ;
    const float sc = which ? 1.f : scale;
    float ss = 0.f, xg = 0.f;
    for (int i = lane; i < d.D; i += 32) {
      float gy = 0.f;
      for (int j = 0; j < G; ++j) {
        const size_t h = (size_t)b * d.Hv + (size_t)hk * G + j;
        gy += g[(h * d.Tp + t) * d.D + i];
      }
      const float xv = to_f32(x[in + i]);
      ss = fmaf(xv, xv, ss);
      xg = fmaf(xv, gy, xg);
    }
    ss = warp_sum(ss), xg = warp_sum(xg);
    const float inv = l2 ? rsqrtf(ss + 1e-6f) : 1.f;
    float* out = which ? dk : dq;
    for (int i = lane; i < d.D; i += 32) {
      float gy = 0.f;
      for (int j = 0; j < G; ++j) {
        const size_t h = (size_t)b * d.Hv + (size_t)hk * G + j;
        gy += g[(h * d.Tp + t) * d.D + i];
      }
      const float xv = to_f32(x[in + i]);
      out[in + i] = l2 ? sc * (gy * inv - xv * xg * inv * inv * inv) : sc * gy;
    }
  }
}

// da, db [B,T,Hv] from (dg, dbeta): given gates pass through; from logits,
// g = -e^{A_log} softplus(a + dt_bias) and beta = sigmoid(b).  Also, per token, the
// contributions to ddt_bias (dg d g / d dt_bias) and dA_log (dg g) in R.
template <typename T>
__global__ void finish_gates_kernel(const void* a_, const void* b_, const float* A_log,
                                    const float* dt_bias, const float2* DG, float* da,
                                    float* db, float2* R, Dims d, int pre) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)d.B * d.T * d.Hv) return;
  const int hv = (int)(i % d.Hv);
  const long bt = i / d.Hv;
  const int t = (int)(bt % d.T), b = (int)(bt / d.T);
  const float2 g2 = DG[((size_t)b * d.Hv + hv) * d.Tp + t];
  if (pre) {
    da[i] = g2.x;
    db[i] = g2.y;
    return;
  }
  const float x = to_f32(static_cast<const T*>(a_)[i]) + dt_bias[hv];
  const float na = -expf(A_log[hv]);
  const float g = na * softplus_f(x);
  const float dx = g2.x * na * sigmoid_f(x);
  const float be = sigmoid_f(to_f32(static_cast<const T*>(b_)[i]));
  da[i] = dx;
  db[i] = g2.y * be * (1.f - be);
  R[i] = make_float2(dx, g2.x * g);
}

// dA_log[hv] = sum over (b, t) of dg g; ddt_bias[hv] = sum of dg dg/d dt_bias.
__global__ void __launch_bounds__(256) reduce_gates_kernel(const float2* R, float* dA_log,
                                                           float* ddt_bias, Dims d) {
  __shared__ float r1[8], r2[8];
  const int hv = blockIdx.x, tid = threadIdx.x;
  float s1 = 0.f, s2 = 0.f;
  const long n = (long)d.B * d.T;
  for (long i = tid; i < n; i += 256) {
    const float2 v = R[i * d.Hv + hv];
    s1 += v.x, s2 += v.y;
  }
  s1 = warp_sum(s1), s2 = warp_sum(s2);
  if ((tid & 31) == 0) r1[tid >> 5] = s1, r2[tid >> 5] = s2;
  __syncthreads();
  if (tid == 0) {
    float a = 0.f, c = 0.f;
    for (int i = 0; i < 8; ++i) a += r1[i], c += r2[i];
    ddt_bias[hv] = a;
    dA_log[hv] = c;
  }
}

// ------------------------------------------------------------------ host side
struct BwdLayout {
  size_t QN, KN, V32, dO32, Wm, Um, dUt, dQ, dW, dKt, QS, dVb, dKb, dK;  // token rows
  size_t S0, dS1, P2;                                                      // D x D per chunk
  size_t KK, QK, Am, Aq, dAqk, dA, T1, dL;                                 // 64 x 64 per chunk
  size_t GB, DG, VB, SC, R;
  size_t total;
};

BwdLayout bwd_layout(int B, int T, int Hk, int Hv, int D) {
  BwdLayout L{};
  const size_t Tp = (size_t)((T + kC - 1) / kC) * kC, Nc = Tp / kC;
  const size_t tk = (size_t)B * Hk * Tp * D * 4, tv = (size_t)B * Hv * Tp * D * 4;
  const size_t dd = (size_t)B * Hv * Nc * D * D * 4, cc = (size_t)B * Hv * Nc * kC * kC * 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  L.QN = take(tk), L.KN = take(tk);
  L.V32 = take(tv), L.dO32 = take(tv), L.Wm = take(tv), L.Um = take(tv), L.dUt = take(tv);
  L.dQ = take(tv), L.dW = take(tv), L.dKt = take(tv), L.QS = take(tv), L.dVb = take(tv);
  L.dKb = take(tv), L.dK = take(tv);
  L.S0 = take(dd), L.dS1 = take(dd), L.P2 = take(dd);
  L.KK = take(cc), L.QK = take(cc), L.Am = take(cc), L.Aq = take(cc), L.dAqk = take(cc);
  L.dA = take(cc), L.T1 = take(cc), L.dL = take(cc);
  L.GB = take((size_t)B * Hv * Tp * 8), L.DG = take((size_t)B * Hv * Tp * 8);
  L.VB = take((size_t)B * Hv * Nc * kC * 16), L.SC = take((size_t)B * Hv * Nc * 4);
  L.R = take((size_t)B * T * Hv * 8);
  L.total = off;
  return L;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int Hk, int Hv, int D) {
  return bwd_layout(B, T, Hk, Hv, D).total;
}

template <typename T>
static cudaError_t run_bwd(const BwdArgs& a, uint8_t* ws, cudaStream_t s) {
  const BwdLayout L = bwd_layout(a.B, a.T, a.Hk, a.Hv, a.D);
  Dims d{a.B, a.T, a.Hk, a.Hv, a.D, 0, 0};
  d.Tp = ((a.T + kC - 1) / kC) * kC;
  d.Nc = d.Tp / kC;
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  float2* GB = reinterpret_cast<float2*>(ws + L.GB);
  float2* DG = reinterpret_cast<float2*>(ws + L.DG);
  float4* VB = reinterpret_cast<float4*>(ws + L.VB);
  float2* R = reinterpret_cast<float2*>(ws + L.R);
  const int Z = a.B * a.Hv * d.Nc;
  const int l2 = (a.flags & GDN_QK_L2NORM) ? 1 : 0;
  const int pre = (a.flags & GDN_GATES_PRECOMPUTED) ? 1 : 0;
  cudaError_t e;
#define GDN_BWD_CHECK()                     \
  do {                                      \
    if ((e = cudaGetLastError()) != cudaSuccess) return e; \
  } while (0)

  {
    const long rows = (long)a.B * a.Hk * d.Tp;
    qk_prep_kernel<T><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), F(L.QN), F(L.KN), d, a.scale,
        l2);
    GDN_BWD_CHECK();
    const long n = (long)a.B * a.Hv * d.Tp * a.D;
    tok_prep_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        static_cast<const T*>(a.v), static_cast<const T*>(a.dout), F(L.V32), F(L.dO32), d);
    GDN_BWD_CHECK();
    gates_prep_kernel<T><<<dim3(d.Nc, a.B * a.Hv), kC, 0, s>>>(a.a, a.b, a.A_log, a.dt_bias,
                                                                 GB, d, pre);
    GDN_BWD_CHECK();
  }
  auto bmm = [&](Opnd x, Opnd y, size_t out, int out_kind, int K, float alpha, int ks, int rs,
                 int cs, int mask, int accumulate) -> cudaError_t {
    const int M = out_kind == kDD ? a.D : kC, N = out_kind == kCC ? kC : a.D;
    BmmArgs P{x, y, F(out), out_kind, M, N, K, alpha, ks, rs, cs, mask, accumulate, GB};
    const dim3 grid(Z, N / 64, M / 64);
    if (x.t && y.t) bmm_kernel<true, true><<<grid, 256, 0, s>>>(P, d);
    else if (x.t) bmm_kernel<true, false><<<grid, 256, 0, s>>>(P, d);
    else if (y.t) bmm_kernel<false, true><<<grid, 256, 0, s>>>(P, d);
    else bmm_kernel<false, false><<<grid, 256, 0, s>>>(P, d);
    return cudaGetLastError();
  };
  const float* QN = F(L.QN);
  const float* KN = F(L.KN);
  auto O = [&](size_t off, int kind, int t) { return Opnd{F(off), kind, t}; };
  // chunk prep: Gram products, the masks, A = (I + L)^-1, W, U
  if ((e = bmm(Opnd{KN, kTK, 0}, Opnd{KN, kTK, 1}, L.KK, kCC, a.D, 1.f, 0, 0, 0, 0, 0))) return e;
  if ((e = bmm(Opnd{QN, kTK, 0}, Opnd{KN, kTK, 1}, L.QK, kCC, a.D, 1.f, 0, 0, 0, 0, 0))) return e;
  gram_gates_kernel<<<Z, 256, 0, s>>>(F(L.KK), F(L.QK), GB, F(L.Am), F(L.Aq), d);
  GDN_BWD_CHECK();
  tri_inverse_kernel<<<Z, kC, 0, s>>>(F(L.Am));
  GDN_BWD_CHECK();
  if ((e = bmm(O(L.Am, kCC, 0), Opnd{KN, kTK, 0}, L.Wm, kTV, kC, 1.f, kScBetaGamma, 0, 0, 0, 0)))
    return e;
  if ((e = bmm(O(L.Am, kCC, 0), O(L.V32, kTV, 0), L.Um, kTV, kC, 1.f, kScBeta, 0, 0, 0, 0)))
    return e;
  // the two scans; the reverse one takes its dS-independent terms precomputed:
  // P1 = A_qk^T dO (into dUt) and P2 = (diag(gamma) Q)^T dO
  if ((e = bmm(O(L.Aq, kCC, 1), O(L.dO32, kTV, 0), L.dUt, kTV, kC, 1.f, 0, 0, 0, 0, 0)))
    return e;
  if ((e = bmm(Opnd{QN, kTK, 1}, O(L.dO32, kTV, 0), L.P2, kDD, kC, 1.f, kScGamma, 0, 0, 0, 0)))
    return e;
  {
    const dim3 grid(a.D / kNS, a.B * a.Hv);
    if (a.D == 128) {
      constexpr size_t sm = scan_smem_bytes<128>();
      e = cudaFuncSetAttribute(fwd_state_scan_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e) return e;
      fwd_state_scan_kernel<128><<<grid, 256, sm, s>>>(F(L.Wm), F(L.Um), KN, GB, a.h0, F(L.S0),
                                                         d);
      GDN_BWD_CHECK();
      e = cudaFuncSetAttribute(rev_state_scan_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e) return e;
      rev_state_scan_kernel<128><<<grid, 256, sm, s>>>(F(L.Wm), KN, F(L.P2), GB, a.dht, F(L.dS1),
                                                         F(L.dUt), a.dh0, d);
      GDN_BWD_CHECK();
    } else {
      constexpr size_t sm = scan_smem_bytes<64>();
      e = cudaFuncSetAttribute(fwd_state_scan_kernel<64>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e) return e;
      fwd_state_scan_kernel<64><<<grid, 256, sm, s>>>(F(L.Wm), F(L.Um), KN, GB, a.h0, F(L.S0), d);
      GDN_BWD_CHECK();
      e = cudaFuncSetAttribute(rev_state_scan_kernel<64>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e) return e;
      rev_state_scan_kernel<64><<<grid, 256, sm, s>>>(F(L.Wm), KN, F(L.P2), GB, a.dht, F(L.dS1),
                                                        F(L.dUt), a.dh0, d);
      GDN_BWD_CHECK();
    }
  }
  // per-chunk gradients (the order of the derivation; Um now holds U~)
  if ((e = bmm(O(L.dO32, kTV, 0), O(L.S0, kDD, 1), L.dQ, kTV, a.D, 1.f, 0, kScGamma, 0, 0, 0)))
    return e;  // dQ = diag(gamma) dO S0^T
  if ((e = bmm(O(L.dUt, kTV, 0), O(L.S0, kDD, 1), L.dW, kTV, a.D, -1.f, 0, 0, 0, 0, 0)))
    return e;  // dW = -dU~ S0^T
  if ((e = bmm(O(L.Um, kTV, 0), O(L.dS1, kDD, 1), L.dKt, kTV, a.D, 1.f, 0, 0, 0, 0, 0)))
    return e;  // dK~ = U~ dS1^T
  if ((e = bmm(Opnd{QN, kTK, 0}, O(L.S0, kDD, 0), L.QS, kTV, a.D, 1.f, 0, 0, 0, 0, 0)))
    return e;  // Q S0
  dgam_kernel<<<Z, 256, 0, s>>>(F(L.dO32), F(L.QS), VB, d);
  GDN_BWD_CHECK();
  dgc_kernel<<<Z, 256, 0, s>>>(F(L.dS1), F(L.S0), F(L.SC), d);
  GDN_BWD_CHECK();
  if ((e = bmm(O(L.dO32, kTV, 0), O(L.Um, kTV, 1), L.dAqk, kCC, a.D, 1.f, 0, 0, 0, kMaskLower,
               0)))
    return e;  // dA_qk = tril(dO U~^T)
  if ((e = bmm(O(L.dUt, kTV, 0), O(L.V32, kTV, 1), L.dA, kCC, a.D, 1.f, 0, 0, kScBeta, 0, 0)))
    return e;  // dA = dU~ (diag(beta) V)^T
  if ((e = bmm(O(L.dW, kTV, 0), Opnd{KN, kTK, 1}, L.dA, kCC, a.D, 1.f, 0, 0, kScBetaGamma, 0,
               1)))
    return e;  //    + dW (diag(beta gamma) K)^T
  if ((e = bmm(O(L.Am, kCC, 1), O(L.dUt, kTV, 0), L.dVb, kTV, kC, 1.f, 0, 0, 0, 0, 0)))
    return e;  // dVb = A^T dU~
  if ((e = bmm(O(L.Am, kCC, 1), O(L.dW, kTV, 0), L.dKb, kTV, kC, 1.f, 0, 0, 0, 0, 0)))
    return e;  // dKb = A^T dW
  vb_kernel<<<Z, 256, 0, s>>>(F(L.dVb), F(L.dKb), F(L.V32), KN, GB, F(L.dK), VB, a.dv, d);
  GDN_BWD_CHECK();
  if ((e = bmm(O(L.dA, kCC, 0), O(L.Am, kCC, 1), L.T1, kCC, kC, 1.f, 0, 0, 0, 0, 0)))
    return e;  // dA A^T
  if ((e = bmm(O(L.Am, kCC, 1), O(L.T1, kCC, 0), L.dL, kCC, kC, -1.f, 0, 0, 0, kMaskStrict, 0)))
    return e;  // dL = tril(-A^T dA A^T, -1)
  dl_kernel<<<Z, 256, 0, s>>>(F(L.dL), F(L.dAqk), F(L.KK), F(L.QK), GB, VB, d);
  GDN_BWD_CHECK();
  // KK now holds dKK = beta dL o Gamma, QK holds dQK = dA_qk o Gamma
  if ((e = bmm(O(L.KK, kCC, 0), Opnd{KN, kTK, 0}, L.dK, kTV, kC, 1.f, 0, 0, 0, 0, 1))) return e;
  if ((e = bmm(O(L.KK, kCC, 1), Opnd{KN, kTK, 0}, L.dK, kTV, kC, 1.f, 0, 0, 0, 0, 1))) return e;
  if ((e = bmm(O(L.QK, kCC, 0), Opnd{KN, kTK, 0}, L.dQ, kTV, kC, 1.f, 0, 0, 0, 0, 1))) return e;
  if ((e = bmm(O(L.QK, kCC, 1), Opnd{QN, kTK, 0}, L.dK, kTV, kC, 1.f, 0, 0, 0, 0, 1))) return e;
  dg_kernel<<<Z, 256, 0, s>>>(F(L.dKt), KN, GB, VB, F(L.SC), F(L.dK), DG, d);
  GDN_BWD_CHECK();
  // the chain rule through the norms and the gates
  {
    const long rows = (long)a.B * a.T * a.Hk;
    finish_qk_kernel<T><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), F(L.dQ), F(L.dK), a.dq, a.dk, d,
        a.scale, l2);
    GDN_BWD_CHECK();
    const long n = (long)a.B * a.T * a.Hv;
    finish_gates_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        a.a, a.b, a.A_log, a.dt_bias, DG, a.da, a.db, R, d, pre);
    GDN_BWD_CHECK();
    if (!pre) {
      reduce_gates_kernel<<<a.Hv, 256, 0, s>>>(R, a.dA_log, a.ddt_bias, d);
      GDN_BWD_CHECK();
    }
  }
#undef GDN_BWD_CHECK
  return cudaSuccess;
}

cudaError_t launch_chunk_bwd(const BwdArgs& a, void* workspace, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return a.dtype == GDN_BF16 ? run_bwd<__nv_bfloat16>(a, ws, s) : run_bwd<float>(a, ws, s);
}

}  // namespace gdn
