// chunk_simt.cu -- chunkwise GDN / Gated DeltaNet-2 forward on the CUDA cores
// in float32 (the float32 path of gdn_chunk_fwd and gdn2_chunk_fwd).
//
// Algebra ("Gated DeltaNet-2" page, 高效训练 / WY 形式; scalar decay for GDN):
// for a chunk of C = 64 tokens with cumulative log-decay G_r and start state S,
//   L   = tril(E K^T (.) exp(G_r - G_j), -1)      E = beta K (GDN), b (.) K (GDN-2)
//   A   = (I + L)^-1                              forward substitution
//   W   = A (gamma (.) E),  U = A Z               Z = beta V (GDN), w (.) V (GDN-2)
//   U~  = U - W S
//   O   = (gamma (.) Q) S + tril(Q K^T (.) exp(G_r - G_j)) U~
//   S  <- Diag(gamma_C) S + ((gamma_C / gamma) (.) K)^T U~
// Only exponents of non-positive numbers are formed.  The state slice stays in
// shared memory across the chunks of one (batch, value head, 64 value columns):
// state columns evolve independently, so the value dimension is split across
// CTAs for parallelism.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kC = 64;        // chunk length
constexpr int kThreads = 256;

// out(m, n, acc) for m < M, n < N of sum_k A(m,k) B(k,n); 16x16 thread grid,
// rows ty + 16 i and columns tx + 16 j per thread.
template <int M, int N, typename FA, typename FB, typename FO>
__device__ __forceinline__ void block_gemm(int K, FA A, FB B, FO out) {
  constexpr int TM = M / 16, TN = N / 16;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
  for (int kk = 0; kk < K; ++kk) {
    float av[TM], bv[TN];
#pragma unroll
    for (int i = 0; i < TM; ++i) av[i] = A(ty + 16 * i, kk);
#pragma unroll
    for (int j = 0; j < TN; ++j) bv[j] = B(kk, tx + 16 * j);
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) out(ty + 16 * i, tx + 16 * j, acc[i][j]);
}

// Value columns per CTA: 64 for GDN, 32 for GDN-2 (which also keeps the
// per-channel erase directions in shared memory).
template <bool GDN2> struct Cols { static constexpr int value = GDN2 ? 32 : 64; };

template <int DK, bool GDN2>
struct Smem {
  static constexpr int kDVS = Cols<GDN2>::value;
  static constexpr int LDK = DK + 1, LDC = kC + 1, LDV = kDVS + 1;
  float K[kC * LDK];      // k_hat rows; later (gamma_C/gamma) (.) k
  float Q[kC * LDK];      // q_hat rows; later gamma (.) q
  float E[GDN2 ? kC * LDK : 1];  // GDN-2 erase directions b (.) k_hat
  float GW[kC * LDK];     // GDN-2 cumulative log-decay; then W (both kinds)
  float S[DK * LDV];      // state slice [DK][kDVS]
  float V[kC * LDV];      // Z (gated values); later U~
  float L[kC * LDC];      // L; later U
  float A[kC * LDC];      // (I + L)^-1
  float P[kC * LDC];      // tril(Q K^T ...)
  float g[kC], beta[kC], G[kC];   // GDN scalar gates, cumulative log-decay
  float gC[DK];           // per-channel total log-decay of the chunk
  float rn_q[kC], rn_k[kC];       // row scales (norm * scale)
};

template <typename T, typename TO, int DK, bool GDN2>
__global__ void __launch_bounds__(kThreads, 1)
chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const void* __restrict__ a_, const void* __restrict__ b_,
                  const void* __restrict__ w_, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, const float* h0, int T_len, int Hk,
                  int Hv, int dv, float scale, int flags, TO* __restrict__ o, float* ht) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  using SM = Smem<DK, GDN2>;
  SM& sm = *reinterpret_cast<SM*>(smem_raw);
  constexpr int LDK = SM::LDK, LDC = SM::LDC, LDV = SM::LDV, kDVS = SM::kDVS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;               // b * Hv + hv
  const int bi = bh / Hv, hv = bh % Hv;
  const int hk = hv / (Hv / Hk);
  const int c0v = blockIdx.y * kDVS;       // first value column of this CTA
  const bool l2 = (flags & GDN_QK_L2NORM) != 0;
  const bool pre = (flags & GDN_GATES_PRECOMPUTED) != 0;
  const int Hq = GDN2 ? Hv : Hk;           // heads of q/k tensors

  // initial state slice
  for (int x = tid; x < DK * kDVS; x += kThreads) {
    const int i = x / kDVS, c = x % kDVS;
    sm.S[i * LDV + c] = h0 ? h0[((size_t)bh * DK + i) * dv + c0v + c] : 0.f;
  }

  for (int t0 = 0; t0 < T_len; t0 += kC) {
    const int n = min(kC, T_len - t0);
    __syncthreads();
    // ---- load the chunk: raw q, k rows; v slice; gates
    for (int x = tid; x < kC * DK; x += kThreads) {
      const int r = x / DK, i = x % DK;
      float qq = 0.f, kk = 0.f;
      if (r < n) {
        const size_t off = (((size_t)bi * T_len + t0 + r) * Hq + (GDN2 ? hv : hk)) * DK + i;
        qq = to_f32(q[off]);
        kk = to_f32(k[off]);
      }
      sm.Q[r * LDK + i] = qq;
      sm.K[r * LDK + i] = kk;
    }
    for (int x = tid; x < kC * kDVS; x += kThreads) {
      const int r = x / kDVS, c = x % kDVS;
      float vv = 0.f;
      if (r < n) {
        const size_t off = (((size_t)bi * T_len + t0 + r) * Hv + hv) * dv + c0v + c;
        vv = to_f32(v[off]);
        if (GDN2) {
          const float wl = pre ? reinterpret_cast<const float*>(w_)[off]
                               : to_f32(reinterpret_cast<const T*>(w_)[off]);
          vv *= pre ? wl : sigmoid_f(wl);
        }
      }
      sm.V[r * LDV + c] = vv;
    }
    if (!GDN2 && tid < kC) {
      float g = 0.f, be = 0.f;
      if (tid < n) {
        const size_t idx = ((size_t)bi * T_len + t0 + tid) * Hv + hv;
        if (pre) {
          g = reinterpret_cast<const float*>(a_)[idx];
          be = reinterpret_cast<const float*>(b_)[idx];
        } else {
          g = gdn_log_decay(to_f32(reinterpret_cast<const T*>(a_)[idx]), A_log[hv], dt_bias[hv]);
          be = sigmoid_f(to_f32(reinterpret_cast<const T*>(b_)[idx]));
        }
      }
      sm.g[tid] = g;
      sm.beta[tid] = be;
    }
    if (GDN2) {
      // per-channel log-decay and erase gate (padded rows: g = 0, b = 0)
      for (int x = tid; x < kC * DK; x += kThreads) {
        const int r = x / DK, i = x % DK;
        float g = 0.f, be = 0.f;
        if (r < n) {
          const size_t off = (((size_t)bi * T_len + t0 + r) * Hv + hv) * DK + i;
          if (pre) {
            g = reinterpret_cast<const float*>(a_)[off];
            be = reinterpret_cast<const float*>(b_)[off];
          } else {
            g = gdn_log_decay(to_f32(reinterpret_cast<const T*>(a_)[off]),
                              A_log[hv * DK + i], dt_bias[hv * DK + i]);
            be = sigmoid_f(to_f32(reinterpret_cast<const T*>(b_)[off]));
          }
        }
        sm.GW[r * LDK + i] = g;
        sm.E[r * LDK + i] = be;  // times k_hat below
      }
    }
    __syncthreads();
    // ---- row norms (one warp per row) and cumulative decay
    for (int r = warp; r < kC; r += kThreads / 32) {
      float sq = 0.f, sk = 0.f;
      for (int i = lane; i < DK; i += 32) {
        sq += sm.Q[r * LDK + i] * sm.Q[r * LDK + i];
        sk += sm.K[r * LDK + i] * sm.K[r * LDK + i];
      }
      sq = warp_sum(sq);
      sk = warp_sum(sk);
      if (lane == 0) {
        sm.rn_q[r] = (l2 ? rsqrtf(sq + 1e-6f) : 1.f) * scale;
        sm.rn_k[r] = l2 ? rsqrtf(sk + 1e-6f) : 1.f;
      }
    }
    if (!GDN2 && tid == 0) {
      float acc = 0.f;
      for (int r = 0; r < kC; ++r) { acc += sm.g[r]; sm.G[r] = acc; }
    }
    if (GDN2 && tid < DK) {  // cumulative sum down each channel
      float acc = 0.f;
      for (int r = 0; r < kC; ++r) { acc += sm.GW[r * LDK + tid]; sm.GW[r * LDK + tid] = acc; }
      sm.gC[tid] = acc;
    }
    __syncthreads();
    for (int x = tid; x < kC * DK; x += kThreads) {
      const int r = x / DK, i = x % DK;
      sm.Q[r * LDK + i] *= sm.rn_q[r];
      sm.K[r * LDK + i] *= sm.rn_k[r];
      if (GDN2) sm.E[r * LDK + i] *= sm.K[r * LDK + i];
    }
    __syncthreads();

    // ---- phase A: L and the masked Q K^T, both with exp(G_r - G_j) <= 1
    if (!GDN2) {
      block_gemm<kC, kC>(DK, [&](int m, int kk) { return sm.K[m * LDK + kk]; },
                         [&](int kk, int j) { return sm.K[j * LDK + kk]; },
                         [&](int m, int j, float acc) {
                           sm.L[m * LDC + j] =
                               j < m ? sm.beta[m] * acc * __expf(sm.G[m] - sm.G[j]) : 0.f;
                         });
      block_gemm<kC, kC>(DK, [&](int m, int kk) { return sm.Q[m * LDK + kk]; },
                         [&](int kk, int j) { return sm.K[j * LDK + kk]; },
                         [&](int m, int j, float acc) {
                           sm.P[m * LDC + j] = j <= m ? acc * __expf(sm.G[m] - sm.G[j]) : 0.f;
                         });
    } else {
      for (int x = tid; x < kC * kC; x += kThreads) {
        const int m = x / kC, j = x % kC;
        float l = 0.f, p = 0.f;
        if (j <= m) {
          for (int i = 0; i < DK; ++i) {
            const float f = __expf(sm.GW[m * LDK + i] - sm.GW[j * LDK + i]);
            const float kf = sm.K[j * LDK + i] * f;
            l = fmaf(sm.E[m * LDK + i], kf, l);
            p = fmaf(sm.Q[m * LDK + i], kf, p);
          }
        }
        sm.L[m * LDC + j] = j < m ? l : 0.f;
        sm.P[m * LDC + j] = p;
      }
    }
    __syncthreads();
    // ---- A = (I + L)^-1, one row at a time (column c by thread c)
    if (tid < kC) sm.A[0 * LDC + tid] = tid == 0 ? 1.f : 0.f;
    for (int r = 1; r < kC; ++r) {
      __syncthreads();
      if (tid < kC) {
        const int c = tid;
        float acc = 0.f;
        for (int j = c; j < r; ++j) acc = fmaf(sm.L[r * LDC + j], sm.A[j * LDC + c], acc);
        sm.A[r * LDC + c] = c < r ? -acc : (c == r ? 1.f : 0.f);
      }
    }
    __syncthreads();
    // ---- phase B: W = A (gamma (.) E) into GW; U = A Z into L
    if (!GDN2) {
      block_gemm<kC, DK>(kC, [&](int m, int j) { return sm.A[m * LDC + j]; },
                         [&](int j, int i) {
                           return sm.beta[j] * __expf(sm.G[j]) * sm.K[j * LDK + i];
                         },
                         [&](int m, int i, float acc) { sm.GW[m * LDK + i] = acc; });
      block_gemm<kC, kDVS>(kC, [&](int m, int j) { return sm.A[m * LDC + j]; },
                           [&](int j, int c) { return sm.beta[j] * sm.V[j * LDV + c]; },
                           [&](int m, int c, float acc) { sm.L[m * LDC + c] = acc; });
    } else {
      // gamma (.) E in place (E is not needed afterwards); GW still holds G
      for (int x = tid; x < kC * DK; x += kThreads) {
        const int r = x / DK, i = x % DK;
        sm.E[r * LDK + i] *= __expf(sm.GW[r * LDK + i]);
        sm.Q[r * LDK + i] *= __expf(sm.GW[r * LDK + i]);
        sm.K[r * LDK + i] *= __expf(sm.gC[i] - sm.GW[r * LDK + i]);
      }
      __syncthreads();
      block_gemm<kC, DK>(kC, [&](int m, int j) { return sm.A[m * LDC + j]; },
                         [&](int j, int i) { return sm.E[j * LDK + i]; },
                         [&](int m, int i, float acc) { sm.GW[m * LDK + i] = acc; });
      block_gemm<kC, kDVS>(kC, [&](int m, int j) { return sm.A[m * LDC + j]; },
                           [&](int j, int c) { return sm.V[j * LDV + c]; },
                           [&](int m, int c, float acc) { sm.L[m * LDC + c] = acc; });
    }
    __syncthreads();
    if (!GDN2) {  // gamma (.) Q and (gamma_C / gamma) (.) K
      const float GC = sm.G[kC - 1];
      for (int x = tid; x < kC * DK; x += kThreads) {
        const int r = x / DK, i = x % DK;
        sm.Q[r * LDK + i] *= __expf(sm.G[r]);
        sm.K[r * LDK + i] *= __expf(GC - sm.G[r]);
      }
      if (tid < DK) sm.gC[tid] = GC;
    }
    // ---- phase C: U~ = U - W S (into V)
    block_gemm<kC, kDVS>(DK, [&](int m, int i) { return sm.GW[m * LDK + i]; },
                         [&](int i, int c) { return sm.S[i * LDV + c]; },
                         [&](int m, int c, float acc) {
                           sm.V[m * LDV + c] = sm.L[m * LDC + c] - acc;
                         });
    __syncthreads();
    // O = (gamma (.) Q) S + P U~
    block_gemm<kC, kDVS>(DK + kC,
                         [&](int m, int kk) {
                           return kk < DK ? sm.Q[m * LDK + kk] : sm.P[m * LDC + kk - DK];
                         },
                         [&](int kk, int c) {
                           return kk < DK ? sm.S[kk * LDV + c] : sm.V[(kk - DK) * LDV + c];
                         },
                         [&](int m, int c, float acc) {
                           if (m < n)
                             o[(((size_t)bi * T_len + t0 + m) * Hv + hv) * dv + c0v + c] =
                                 from_f32<TO>(acc);
                         });
    __syncthreads();
    // S <- Diag(gamma_C) S + K_tail^T U~
    block_gemm<DK, kDVS>(kC, [&](int i, int r) { return sm.K[r * LDK + i]; },
                         [&](int r, int c) { return sm.V[r * LDV + c]; },
                         [&](int i, int c, float acc) {
                           sm.S[i * LDV + c] = __expf(sm.gC[i]) * sm.S[i * LDV + c] + acc;
                         });
  }
  __syncthreads();
  if (ht) {
    for (int x = tid; x < DK * kDVS; x += kThreads) {
      const int i = x / kDVS, c = x % kDVS;
      ht[((size_t)bh * DK + i) * dv + c0v + c] = sm.S[i * LDV + c];
    }
  }
}

template <typename T, typename TO, int DK, bool GDN2>
cudaError_t launch_t(const ChunkArgs& a, cudaStream_t s) {
  auto kern = chunk_simt_kernel<T, TO, DK, GDN2>;
  const int smem = (int)sizeof(Smem<DK, GDN2>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.B * a.Hv, a.dv / Smem<DK, GDN2>::kDVS);
  kern<<<grid, kThreads, smem, s>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, a.a, a.b, a.w,
                                    a.A_log, a.dt_bias, a.h0, a.T, a.Hk, a.Hv, a.dv, a.scale,
                                    a.flags, (TO*)a.o, a.ht);
  return cudaGetLastError();
}

template <typename T, bool GDN2>
cudaError_t launch_dk(const ChunkArgs& a, cudaStream_t s) {
  const bool of32 = (a.flags & GDN_OUT_F32) != 0 || sizeof(T) == 4;
  if (a.dk == 64)
    return of32 ? launch_t<T, float, 64, GDN2>(a, s) : launch_t<T, __nv_bfloat16, 64, GDN2>(a, s);
  if (a.dk == 128)
    return of32 ? launch_t<T, float, 128, GDN2>(a, s)
                : launch_t<T, __nv_bfloat16, 128, GDN2>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a, bool gdn2, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  if (a.dtype == GDN_BF16)
    return gdn2 ? launch_dk<__nv_bfloat16, true>(a, s) : launch_dk<__nv_bfloat16, false>(a, s);
  return gdn2 ? launch_dk<float, true>(a, s) : launch_dk<float, false>(a, s);
}

}  // namespace gdn
