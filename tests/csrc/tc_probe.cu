// tc_probe.cu -- single-CTA probes of the sm_100a building blocks the chunk
// kernel is made of (tensor-memory round trip, TMA 4-D tile load with the
// 128-byte swizzle, tcgen05.mma with K-major / MN-major operands at M = 64 and
// M = 128).  Each probe copies its result to global memory for the host to
// compare with torch; every wait is bounded and reports through *status.
// Test infrastructure: built by tests/test_tc_primitives_gpu.py only.
#include <cuda.h>
#include <string.h>
#include <cudaTypedefs.h>

#include "../../gated_deltanet_sequence_gdn_b200/csrc/tc_ptx.cuh"

using namespace gdn;
using namespace gdn::tc;

namespace {

struct ProbeSmem {
  uint64_t bar;
  uint32_t tmem;
};

// ---------------------------------------------------------------- TMEM
__global__ void tmem_roundtrip_kernel(float* out, int* status) {
  __shared__ ProbeSmem ps;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) tmem_alloc(&ps.tmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ps.tmem;
  const uint32_t lb = (uint32_t)(warp * 32) << 16;
  float v[16];
  for (int blk = 0; blk < 4; ++blk) {  // columns 0,128,256,384 (+16)
    for (int c = 0; c < 16; ++c) v[c] = (float)(tid * 1000 + blk * 100 + c);
    tmem_st16(tmem + lb + 128 * blk, v);
  }
  tmem_st_wait();
  for (int blk = 0; blk < 4; ++blk) {
    tmem_ld16(tmem + lb + 128 * blk, v);
    tmem_ld_wait();
    for (int c = 0; c < 16; ++c) out[(tid * 4 + blk) * 16 + c] = v[c];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- TMA
// src: bf16 [B=1][T][H][128]; loads the box (c0 in {0,64}, head h, token t0)
// and writes it un-swizzled to out [64][64] (float).
// nbox boxes (box b: channel half b % 2 of head h, into sm + 8192 b) on one
// barrier; optionally prefetches the tensor map first.
__global__ void tma_load_kernel(const __grid_constant__ CUtensorMap tm, int c0, int h, int t0,
                                int nbox, int prefetch, float* out, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 8192 * nbox);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (prefetch) prefetch_tmap(&tm);
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, 8192 * nbox);
    for (int b = 0; b < nbox; ++b)
      tma_load_4d(sm + 8192 * b, &tm, bar, nbox == 1 ? c0 : 64 * (b % 2), h, t0, 0);
  }
  const bool ok = mbar_wait(bar, 0, status, 11);
  if (!__syncthreads_or(!ok)) {
    for (int x = tid; x < nbox * 64 * 64; x += blockDim.x) {
      const int b = x / 4096, r = (x / 64) % 64, c = x % 64;
      const __nv_bfloat16 e =
          *reinterpret_cast<const __nv_bfloat16*>(sm + 8192 * b + sw128_offset(r, c));
      out[x] = __bfloat162float(e);
    }
  }
}

// ---------------------------------------------------------------- MMA
// D[M][N] = sum_k A[m][k] B[k][n], K = 64, bf16 inputs given row-major
// (A [M][64], B [64][N]); staged into shared memory as K-major or MN-major
// 128-byte-swizzled tiles exactly as the chunk kernel lays them out.
// M in {64,128}, N in {64,128}; output float [M][N].
__global__ void mma_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B, float* D, int M, int N,
                           int a_mn, int b_mn, int dcol, int base_off, int atom, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~uintptr_t(1023));
  // operands at sm + base_off: A region 2 * atom bytes, then B region 2 * atom bytes
  uint8_t* sa = sm + base_off;
  uint8_t* sb = sm + base_off + 2 * atom;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int K = 64;
  // A: K-major -> row m at m*128 (one 64-wide K atom column);
  //    MN-major -> atom (m/64) at 8192*(m/64), row k at k*128, col m%64
  for (int x = tid; x < M * K; x += blockDim.x) {
    const int m = x / K, k = x % K;
    const uint32_t off = a_mn ? (uint32_t)(m / 64) * (uint32_t)atom + sw128_offset(k, m % 64)
                              : sw128_offset(m, k);
    *reinterpret_cast<__nv_bfloat16*>(sa + off) = A[x];
  }
  // B: K-major -> row n at n*128; MN-major -> atom (n/64) at 8192*(n/64), row k
  for (int x = tid; x < K * N; x += blockDim.x) {
    const int k = x / N, n = x % N;
    const uint32_t off = b_mn ? (uint32_t)(n / 64) * (uint32_t)atom + sw128_offset(k, n % 64)
                              : sw128_offset(n, k);
    *reinterpret_cast<__nv_bfloat16*>(sb + off) = B[x];
  }
  fence_proxy_async_smem();
  if (warp == 0) tmem_alloc(slot, 512);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t sa_u = smem_u32(sa), sb_u = smem_u32(sb);
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16(M, N, a_mn != 0, b_mn != 0);
    for (int k16 = 0; k16 < K / 16; ++k16) {
      const uint64_t ad = a_mn ? sw128_desc(sa_u + k16 * 2048, atom, 1024)
                               : sw128_desc(sa_u + k16 * 32, 16, 1024);
      const uint64_t bd = b_mn ? sw128_desc(sb_u + k16 * 2048, atom, 1024)
                               : sw128_desc(sb_u + k16 * 32, 16, 1024);
      mma_bf16(tmem + dcol, ad, bd, idesc, k16 > 0);
    }
    mma_commit(bar);
  }
  const bool ok = mbar_wait(bar, 0, status, 21);
  const bool bad = __syncthreads_or(!ok);
  tc_fence_after();
  if (!bad) {
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    float v[16];
    for (int c0 = 0; c0 < N; c0 += 16) {
      tmem_ld16(tmem + lb + dcol + c0, v);
      int row = -1;
      if (M == 128) row = tid;
      else if (lane < 16) row = 16 * warp + lane;  // M = 64 layout
      if (row >= 0)
        for (int c = 0; c < 16; ++c) D[row * N + c0 + c] = v[c];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- choreography
// The chunk kernel's MMA / tensor-memory schedule with synthetic operands at its
// shared-memory offsets: four commit/wait rounds on one barrier, interleaved
// MMAs of different shapes, tile stores while the tensor cores run.  Operand
// tiles come in already swizzled (bf16 images of the kernel's tiles); every
// accumulator is dumped to `out` (float) for the host to check:
//   out[0      : 8192 )  KQ  [128][64]   = [K;Q] K^T
//   out[8192   : 16384)  W   [64][128]   = A1 K
//   out[16384  : 20480)  U   [64][64]    = A2 V
//   out[20480  : 24576)  P   [64][64]    = Wt S      (Wt = given W tile)
//   out[24576  : 28672)  OQ  [64][64]    = Q S
//   out[28672  : 32768)  OA  [64][64]    = Aqk Ut
//   out[32768  : 40960)  DS  [128][64]   = K^T Us
namespace sk {
constexpr uint32_t KQ = 0, V = 32768, AQK = 40960, A1 = 49152, A2 = 57344, W = 65536, SB = 81920,
                   UT = 98304, US = 106496, BAR = 149056, SMEM = 150144;
}

__device__ void dump_tmem(uint32_t taddr_col, int M, int N, float* dst) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t lb = (uint32_t)(warp * 32) << 16;
  float v[16];
  for (int c0 = 0; c0 < N; c0 += 16) {
    tmem_ld16(taddr_col + lb + c0, v);
    int row = -1;
    if (M == 128) row = tid;
    else if (lane < 16) row = 16 * warp + lane;
    if (row >= 0)
      for (int c = 0; c < 16; ++c) dst[row * N + c0 + c] = v[c];
  }
}

// mode bits: 1 = threads 64-127 read the Q tile with generic loads while the
// first MMA reads it; 2 = a ~100 us CUDA-core phase between the first and the
// second round; 4 = fp32 traffic through shared bytes [114688, 147968) between
// those rounds; 8 = the TMA and MMA barriers adjacent (8 bytes apart); 16 = the
// S tile stored row per thread from registers; 32 = everything repeated 3 times in
// a runtime loop (the chunk loop's shape).
__global__ void skeleton_kernel(const uint8_t* tiles, float* out, int* status,
                                const __grid_constant__ CUtensorMap tq,
                                const __grid_constant__ CUtensorMap tk,
                                const __grid_constant__ CUtensorMap tv, int use_tma, int mode,
                                float* sink) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + sk::BAR + ((mode & 8) ? 8 : 0));
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + sk::BAR + 32);
  const int tid = threadIdx.x, warp = tid >> 5;
  out += (size_t)blockIdx.y * 40960;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + sk::BAR + ((mode & 8) ? 0 : 16));
  float acc_sink = 0.f;
  // operand tiles except SB / W / UT / US (those are stored mid-way, as the kernel does);
  // with use_tma the K, Q, V tiles come from TMA instead
  for (int x = tid * 16 + (use_tma ? (int)sk::AQK : 0); x < (int)sk::W; x += 128 * 16)
    *reinterpret_cast<uint4*>(sm + x) = *reinterpret_cast<const uint4*>(tiles + x);
  fence_proxy_async_smem();
  if (warp == 0) tmem_alloc(slot, 512);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_tma, 1);
    fence_mbar_init();
    if (use_tma) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t sb = smem_u32(sm);
  uint32_t ph = 0;
  bool ok;
  const int iters = (mode & 32) ? 3 : 1;
  for (int it = 0; it < iters; ++it) {
  if (use_tma) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_tma, 5 * 8192);
      tma_load_4d(sm + sk::KQ + 0, &tk, bar_tma, 0, 0, 0, 0);
      tma_load_4d(sm + sk::KQ + 16384, &tk, bar_tma, 64, 0, 0, 0);
      tma_load_4d(sm + sk::KQ + 8192, &tq, bar_tma, 0, 0, 0, 0);
      tma_load_4d(sm + sk::KQ + 24576, &tq, bar_tma, 64, 0, 0, 0);
      tma_load_4d(sm + sk::V, &tv, bar_tma, 64 * blockIdx.y, 0, 0, 0);
    }
    ok = mbar_wait(bar_tma, it & 1, status, 30);
    if (__syncthreads_or(!ok)) goto done;
  }
  // round 1: [K;Q] K^T
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 8; ++k16) {
      const uint32_t off = (uint32_t)(k16 >> 2) * 16384u + (uint32_t)(k16 & 3) * 32u;
      mma_bf16(tmem + 64, sw128_desc(sb + sk::KQ + off, 16, 1024),
               sw128_desc(sb + sk::KQ + off, 16, 1024), idesc_bf16(128, 64, false, false), k16 > 0);
    }
    mma_commit(bar);
  }
  if ((mode & 1) && tid >= 64) {
    const int r = tid - 64;
    for (int h = 0; h < 2; ++h)
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(sm + sk::KQ + 8192 + h * 16384 + r * 128 +
                                                        16 * c);
        acc_sink += __uint_as_float(u.x & 0x3fffffffu) + __uint_as_float(u.w & 0x3fffffffu);
      }
  }
  ok = mbar_wait(bar, ph, status, 31); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  dump_tmem(tmem + 64, 128, 64, out + 0);
  if (mode & 4) {
    float* scratch = reinterpret_cast<float*>(sm + 114688);
    for (int x = tid; x < (147968 - 114688) / 4; x += 128) scratch[x] = (float)(x + blockIdx.y);
    __syncthreads();
    for (int x = tid; x < (147968 - 114688) / 4; x += 128) acc_sink += scratch[(x * 7) % 8320];
    __syncthreads();
  }
  if (mode & 2) {
    const long long t_end = clock64() + 200000;  // ~100 us at 1.9 GHz
    float a = acc_sink;
    while (clock64() < t_end) a = fmaf(a, 0.999f, 1e-3f);
    acc_sink = a;
    __syncthreads();
  }
  // round 2: W = A1 K, U = A2 V interleaved; SB stored meanwhile
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 4; ++k16) {
      mma_bf16(tmem + 128, sw128_desc(sb + sk::A1 + k16 * 32, 16, 1024),
               sw128_desc(sb + sk::KQ + k16 * 2048, 16384, 1024), idesc_bf16(64, 128, false, true),
               k16 > 0);
      mma_bf16(tmem + 256, sw128_desc(sb + sk::A2 + k16 * 32, 16, 1024),
               sw128_desc(sb + sk::V + k16 * 2048, 8192, 1024), idesc_bf16(64, 64, false, true),
               k16 > 0);
    }
    mma_commit(bar);
  }
  if (mode & 16) {
    // the chunk kernel's pattern: thread t owns row t, values in registers
    float rowv[64];
    for (int c = 0; c < 64; ++c)
      rowv[c] = __bfloat162float(
          *reinterpret_cast<const __nv_bfloat16*>(tiles + sk::SB + sw128_offset(tid, c)));
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 16) st_row16_bf16(sm + sk::SB, tid, c0, rowv + c0);
  } else {
    for (int x = tid * 16; x < 16384; x += 128 * 16)
      *reinterpret_cast<uint4*>(sm + sk::SB + x) =
          *reinterpret_cast<const uint4*>(tiles + sk::SB + x);
  }
  ok = mbar_wait(bar, ph, status, 32); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  dump_tmem(tmem + 128, 64, 128, out + 8192);
  dump_tmem(tmem + 256, 64, 64, out + 16384);
  for (int x = tid * 16; x < 16384; x += 128 * 16)
    *reinterpret_cast<uint4*>(sm + sk::W + x) = *reinterpret_cast<const uint4*>(tiles + sk::W + x);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // round 3: P = Wt S, OQ = Q S interleaved
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 8; ++k16) {
      const uint32_t kin = (uint32_t)(k16 & 3) * 32u;
      const uint64_t bd = sw128_desc(sb + sk::SB + k16 * 2048, 8192, 1024);
      mma_bf16(tmem + 320, sw128_desc(sb + sk::W + (k16 >> 2) * 8192 + kin, 16, 1024), bd,
               idesc_bf16(64, 64, false, true), k16 > 0);
      mma_bf16(tmem + 384, sw128_desc(sb + sk::KQ + 8192 + (k16 >> 2) * 16384 + kin, 16, 1024),
               bd, idesc_bf16(64, 64, false, true), k16 > 0);
    }
    mma_commit(bar);
  }
  ok = mbar_wait(bar, ph, status, 33); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  dump_tmem(tmem + 320, 64, 64, out + 20480);
  dump_tmem(tmem + 384, 64, 64, out + 24576);
  for (int x = tid * 16; x < 16384; x += 128 * 16)
    *reinterpret_cast<uint4*>(sm + sk::UT + x) = *reinterpret_cast<const uint4*>(tiles + sk::UT + x);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // round 4: OA = Aqk Ut, DS = K^T Us interleaved
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 4; ++k16) {
      mma_bf16(tmem + 448, sw128_desc(sb + sk::AQK + k16 * 32, 16, 1024),
               sw128_desc(sb + sk::UT + k16 * 2048, 8192, 1024), idesc_bf16(64, 64, false, true),
               k16 > 0);
      mma_bf16(tmem + 0, sw128_desc(sb + sk::KQ + k16 * 2048, 16384, 1024),
               sw128_desc(sb + sk::US + k16 * 2048, 8192, 1024), idesc_bf16(128, 64, true, true),
               k16 > 0);
    }
    mma_commit(bar);
  }
  ok = mbar_wait(bar, ph, status, 34); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  dump_tmem(tmem + 448, 64, 64, out + 28672);
  dump_tmem(tmem + 0, 128, 64, out + 32768);
  tc_fence_before();
  __syncthreads();
  }  // iterations
done:
  if (acc_sink == 1234.5f) sink[0] = acc_sink;  // keeps the probe reads alive
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The chunk kernel's own prologue (gates from real gate tensors, q norms, the
// KK / QK epilogue, forward substitution, A1 / A2), run on the validated
// skeleton, followed by the W / U round that consumes the computed tiles.  The
// launch mirrors the chunk kernel's: tensor maps first, __launch_bounds__(128, 1),
// a template instantiation, the state rows live in registers.
// out (per CTA, floats): [0, 4096) A1, [4096, 8192) A2 (dense [64][64]),
// [8192, 16384) W [64][128], [16384, 20480) U [64][64], [20480, 28672) SB as read back;
// stages >= 1 adds phase 6 and phase 8: [28672, 32768) P = W S, [32768, 36864) Q S;
// stages >= 2 adds phases 9-10: [36864, 40960) Aqk, [40960, 45056) U~, [45056, 49152) U~s,
// [49152, 53248) Aqk U~, [53248, 61440) K^T U~s; stages >= 3 adds phase 11 (o written) and
// the updated state rows [61440, 69632).
namespace pk {
constexpr uint32_t OFF_LF = 114688, OFF_XF = OFF_LF + 64 * 65 * 4, OFF_VEC = OFF_XF + 64 * 65 * 4;
}
template <typename TO, int PRESSURE = 0>
__global__ void __launch_bounds__(128, 1)
prologue_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const void* __restrict__ a_,
                const void* __restrict__ b_, const float* __restrict__ A_log,
                const float* __restrict__ dt_bias, const float* h0, int T, int Hk, int Hv,
                float scale, int flags, TO* __restrict__ o, float* out, int* status,
                int stages) {
  float hold[PRESSURE > 0 ? PRESSURE : 1];
#pragma unroll
  for (int i = 0; i < (PRESSURE > 0 ? PRESSURE : 1); ++i) hold[i] = __int_as_float(threadIdx.x * 131 + i);
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~uintptr_t(1023));
  float* Lf = reinterpret_cast<float*>(sm + pk::OFF_LF);
  float* Xf = reinterpret_cast<float*>(sm + pk::OFF_XF);
  float* Gs = reinterpret_cast<float*>(sm + pk::OFF_VEC);
  float* betas = Gs + 64;
  float* rks = betas + 64;
  float* sqs = rks + 64;
  float* misc = sqs + 64;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + sk::BAR);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, bi = bh / Hv, hv = bh % Hv, hk = hv / (Hv / Hk);
  const int c0v = blockIdx.y * 64;
  const bool l2 = (flags & 1) != 0;
  const uint32_t sbase = smem_u32(sm);
  out += (size_t)blockIdx.y * 69632;
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int r64 = 16 * warp + lane;
  float S[64];
  {
    const float* src = h0 ? h0 + ((size_t)bh * 128 + tid) * 128 + c0v : nullptr;
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
      const float4 t = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0, 0, 0, 0);
      S[c] = t.x; S[c + 1] = t.y; S[c + 2] = t.z; S[c + 3] = t.w;
    }
  }
  uint32_t ph = 0;
  bool ok;
  const int t0 = 0, n = min(64, T);
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_tma, 5 * 8192);
    tma_load_4d(sm + 0, &tm_k, bar_tma, 0, hk, t0, bi);
    tma_load_4d(sm + 16384, &tm_k, bar_tma, 64, hk, t0, bi);
    tma_load_4d(sm + 8192, &tm_q, bar_tma, 0, hk, t0, bi);
    tma_load_4d(sm + 24576, &tm_q, bar_tma, 64, hk, t0, bi);
    tma_load_4d(sm + sk::V, &tm_v, bar_tma, c0v, hv, t0, bi);
  }
  if (tid < 64) {
    float g = 0.f, be = 0.f;
    if (tid < n) {
      const size_t idx = ((size_t)bi * T + t0 + tid) * Hv + hv;
      g = gdn_log_decay(__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a_)[idx]),
                        A_log[hv], dt_bias[hv]);
      be = sigmoid_f(__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(b_)[idx]));
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, g, off);
      if (lane >= off) g += y;
    }
    if (tid == 31) misc[0] = g;
    Gs[tid] = g;
    betas[tid] = be;
  }
  __syncthreads();
  if (tid >= 32 && tid < 64) Gs[tid] += misc[0];
  ok = mbar_wait(bar_tma, 0, status, 40);
  if (__syncthreads_or(!ok)) goto done;
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 8; ++k16) {
      const uint32_t off = (uint32_t)(k16 >> 2) * 16384u + (uint32_t)(k16 & 3) * 32u;
      mma_bf16(tmem + 64, sw128_desc(sbase + off, 16, 1024), sw128_desc(sbase + off, 16, 1024),
               idesc_bf16(128, 64, false, false), k16 > 0);
    }
    mma_commit(bar_mma);
  }
  if (tid >= 64) {
    const int r = tid - 64;
    float ss = 0.f;
    for (int h = 0; h < 2; ++h) {
      const uint8_t* row = sm + 8192 + h * 16384 + r * 128;
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(row + 16 * c);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
          ss += f.x * f.x + f.y * f.y;
        }
      }
    }
    sqs[r] = (l2 ? rsqrtf(ss + 1e-6f) : 1.f) * scale;
  }
  ok = mbar_wait(bar_mma, ph, status, 41); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  {
    float* dst = tid < 64 ? Lf + tid * 65 : Xf + (tid - 64) * 65;
    float v[16];
    for (int j = 0; j < 4; ++j) {
      tmem_ld16(tmem + lane_base + 64 + 16 * j, v);
#pragma unroll
      for (int c = 0; c < 16; ++c) dst[16 * j + c] = v[c];
    }
  }
  __syncthreads();
  if (tid < 64) rks[tid] = l2 ? rsqrtf(Lf[tid * 65 + tid] + 1e-6f) : 1.f;
  __syncthreads();
  if (tid < 64) {
    const int r = tid;
    const float br = betas[r] * rks[r], Gr = Gs[r];
    for (int j = 0; j < 64; ++j) {
      const float kk = Lf[r * 65 + j];
      Lf[r * 65 + j] = j < r ? br * kk * rks[j] * __expf(Gr - Gs[j]) : 0.f;
    }
  } else {
    const int r = tid - 64;
    const float sr = sqs[r], Gr = Gs[r];
    for (int j0 = 0; j0 < 64; j0 += 16) {
      float a[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int j = j0 + c;
        a[c] = j <= r ? Xf[r * 65 + j] * sr * rks[j] * __expf(Gr - Gs[j]) : 0.f;
      }
      st_row16_bf16(sm + sk::AQK, r, j0, a);
    }
  }
  __syncthreads();
  if (tid < 64) {
    const int c = tid;
    for (int r = 0; r < 64; ++r) {
      float acc = 0.f;
      for (int j = c; j < r; ++j) acc = fmaf(Lf[r * 65 + j], Xf[j * 65 + c], acc);
      Xf[r * 65 + c] = c < r ? -acc : (c == r ? 1.f : 0.f);
    }
  }
  __syncthreads();
  {
    const int r = tid & 63;
    const bool first = tid < 64;
    for (int j0 = 0; j0 < 64; j0 += 16) {
      float a[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int j = j0 + c;
        a[c] = Xf[r * 65 + j] * betas[j] * (first ? __expf(Gs[j]) * rks[j] : 1.f);
        out[(first ? 0 : 4096) + r * 64 + j] = __bfloat162float(__float2bfloat16_rn(a[c]));
      }
      st_row16_bf16(sm + (first ? sk::A1 : sk::A2), r, j0, a);
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    for (int k16 = 0; k16 < 4; ++k16) {
      mma_bf16(tmem + 128, sw128_desc(sbase + sk::A1 + k16 * 32, 16, 1024),
               sw128_desc(sbase + k16 * 2048, 16384, 1024), idesc_bf16(64, 128, false, true),
               k16 > 0);
      mma_bf16(tmem + 256, sw128_desc(sbase + sk::A2 + k16 * 32, 16, 1024),
               sw128_desc(sbase + sk::V + k16 * 2048, 8192, 1024), idesc_bf16(64, 64, false, true),
               k16 > 0);
    }
    mma_commit(bar_mma);
  }
#pragma unroll
  for (int c0 = 0; c0 < 64; c0 += 16) st_row16_bf16(sm + sk::SB, tid, c0, S + c0);
  ok = mbar_wait(bar_mma, ph, status, 42); ph ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  dump_tmem(tmem + 128, 64, 128, out + 8192);
  dump_tmem(tmem + 256, 64, 64, out + 16384);
  for (int c = 0; c < 64; ++c)
    out[20480 + tid * 64 + c] =
        __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + sk::SB + sw128_offset(tid, c)));
  if (stages >= 1) {
    // phase 6: W to bf16 (the chunk kernel's code), phase 8: P = W S, OQ = Q S
    for (int c0 = 0; c0 < 128; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + lane_base + 128 + c0, v);
      if (lane < 16) st_row16_bf16(sm + sk::W + 8192 * (c0 >> 6), r64, c0 & 63, v);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      for (int k16 = 0; k16 < 8; ++k16) {
        const uint32_t kin = (uint32_t)(k16 & 3) * 32u;
        const uint64_t bdesc = sw128_desc(sbase + sk::SB + k16 * 2048, 8192, 1024);
        mma_bf16(tmem + 320, sw128_desc(sbase + sk::W + (k16 >> 2) * 8192 + kin, 16, 1024),
                 bdesc, idesc_bf16(64, 64, false, true), k16 > 0);
        mma_bf16(tmem + 384, sw128_desc(sbase + 8192 + (k16 >> 2) * 16384 + kin, 16, 1024), bdesc,
                 idesc_bf16(64, 64, false, true), k16 > 0);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph, status, 43); ph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    dump_tmem(tmem + 320, 64, 64, out + 28672);
    dump_tmem(tmem + 384, 64, 64, out + 32768);
  }
  if (stages >= 2) {
    // phase 9: U~ = U - P and its scaled copy (the chunk kernel's code)
    {
      const float f = lane < 16 ? __expf(Gs[63] - Gs[r64]) * rks[r64] : 0.f;
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float u[16], pp[16];
        tmem_ld16(tmem + lane_base + 256 + c0, u);
        tmem_ld16(tmem + lane_base + 320 + c0, pp);
        if (lane < 16) {
#pragma unroll
          for (int c = 0; c < 16; ++c) u[c] -= pp[c];
          st_row16_bf16(sm + sk::UT, r64, c0, u);
#pragma unroll
          for (int c = 0; c < 16; ++c) u[c] *= f;
          st_row16_bf16(sm + sk::US, r64, c0, u);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // phase 10: OA = Aqk U~, DS = K^T U~s
    if (tid == 0) {
      tc_fence_after();
      for (int k16 = 0; k16 < 4; ++k16) {
        mma_bf16(tmem + 448, sw128_desc(sbase + sk::AQK + k16 * 32, 16, 1024),
                 sw128_desc(sbase + sk::UT + k16 * 2048, 8192, 1024),
                 idesc_bf16(64, 64, false, true), k16 > 0);
        mma_bf16(tmem + 0, sw128_desc(sbase + k16 * 2048, 16384, 1024),
                 sw128_desc(sbase + sk::US + k16 * 2048, 8192, 1024),
                 idesc_bf16(128, 64, true, true), k16 > 0);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph, status, 44); ph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // dumps: Aqk, U~, U~s (dense bf16 values), OA, DS
    for (int x = tid; x < 64 * 64; x += 128) {
      const int rr = x / 64, c = x % 64;
      out[36864 + x] = __bfloat162float(
          *reinterpret_cast<const __nv_bfloat16*>(sm + sk::AQK + sw128_offset(rr, c)));
      out[40960 + x] = __bfloat162float(
          *reinterpret_cast<const __nv_bfloat16*>(sm + sk::UT + sw128_offset(rr, c)));
      out[45056 + x] = __bfloat162float(
          *reinterpret_cast<const __nv_bfloat16*>(sm + sk::US + sw128_offset(rr, c)));
    }
    dump_tmem(tmem + 448, 64, 64, out + 49152);
    dump_tmem(tmem + 0, 128, 64, out + 53248);
  }
  if (stages >= 3) {
    // phase 11: O = gamma sq (Q S) + Aqk U~, S <- gamma_C S + DS; then the state store
    {
      const bool has_row = lane < 16 && r64 < n;
      const float f = has_row ? __expf(Gs[r64]) * sqs[r64] : 0.f;
      TO* dst = o + (((size_t)bi * T + t0 + (has_row ? r64 : 0)) * Hv + hv) * 128 + c0v;
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float qq[16], pp[16];
        tmem_ld16(tmem + lane_base + 384 + c0, qq);
        tmem_ld16(tmem + lane_base + 448 + c0, pp);
        if (has_row) {
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c0 + c] = from_f32<TO>(f * qq[c] + pp[c]);
        }
      }
      const float gC = __expf(Gs[63]);
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float d[16];
        tmem_ld16(tmem + lane_base + 0 + c0, d);
#pragma unroll
        for (int c = 0; c < 16; ++c) S[c0 + c] = fmaf(gC, S[c0 + c], d[c]);
      }
    }
    tc_fence_before();
    __syncthreads();
    float* dst = out + 61440 + tid * 64;
#pragma unroll
    for (int c = 0; c < 64; c += 4)
      *reinterpret_cast<float4*>(dst + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
  }
  if (PRESSURE > 0) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < (PRESSURE > 0 ? PRESSURE : 1); ++i) acc += hold[i] * (float)(i + 1);
    if (acc == 12345.f) out[0] = acc;
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
}

}  // namespace

extern "C" {

int probe_tmem_roundtrip(float* out, int* status) {
  tmem_roundtrip_kernel<<<1, 128>>>(out, status);
  return (int)cudaGetLastError();
}

int probe_tma_load(const void* src, int T, int H, int c0, int h, int t0, int nbox, int prefetch,
                   float* out, int* status) {
  if (nbox < 1 || nbox > 8) return -1;
  auto enc = encode_fn();
  if (!enc) return -100;
  CUtensorMap m;
  cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, 1};
  cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(src), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return -200 - (int)r;
  const int smem = 8192 * nbox + 64 + 1024;
  cudaFuncSetAttribute(tma_load_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  tma_load_kernel<<<1, 128, smem>>>(m, c0, h, t0, nbox, prefetch, out, status);
  return (int)cudaGetLastError();
}

int probe_mma(const void* A, const void* B, float* D, int M, int N, int a_mn, int b_mn,
              int dcol, int base_off, int atom, int* status) {
  if (!((M == 64 || M == 128) && (N == 64 || N == 128))) return -1;
  if (dcol < 0 || dcol % 16 != 0 || dcol + N > 512) return -2;
  if (atom != 8192 && atom != 16384) return -3;
  if (base_off < 1024 || base_off % 1024 != 0) return -4;
  const int smem = base_off + 4 * atom + 1024;   // operands end at base_off + 4 * atom
  if (smem > 227 * 1024) return -5;
  cudaFuncSetAttribute(mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  mma_kernel<<<1, 128, smem>>>((const __nv_bfloat16*)A, (const __nv_bfloat16*)B, D, M, N, a_mn,
                               b_mn, dcol, base_off, atom, status);
  return (int)cudaGetLastError();
}

static bool map4(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int T) {
  cuuint64_t dims[4] = {128, 1, (cuuint64_t)T, 1};
  cuuint64_t strides[3] = {256, 256, (cuuint64_t)T * 256};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q, k, v: bf16 [1][T][1][128] (v's 64-column half blockIdx.y is loaded); NULL = no TMA.
int probe_skeleton(const void* tiles, float* out, int* status, const void* q, const void* k,
                   const void* v, int T, int mode, float* sink) {
  CUtensorMap mq, mk, mv;
  memset(&mq, 0, sizeof(mq)); memset(&mk, 0, sizeof(mk)); memset(&mv, 0, sizeof(mv));
  const int use_tma = q != nullptr;
  if (use_tma) {
    auto enc = encode_fn();
    if (!enc || !map4(enc, &mq, q, T) || !map4(enc, &mk, k, T) || !map4(enc, &mv, v, T))
      return -100;
  }
  cudaFuncSetAttribute(skeleton_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)sk::SMEM);
  skeleton_kernel<<<dim3(1, 2), 128, sk::SMEM>>>((const uint8_t*)tiles, out, status, mq, mk, mv,
                                                 use_tma, mode, sink);
  return (int)cudaGetLastError();
}

static bool map4h(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int B,
                  int T, int H) {
  cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B = 1, T tokens, Hk = Hv = 1, d = 128 bf16; one chunk; grid (1, 2) like the chunk kernel.
int probe_prologue(const void* q, const void* k, const void* v, const void* a, const void* b,
                   const float* A_log, const float* dt_bias, const float* h0, int T, float scale,
                   void* o, float* out, int* status, int stages) {
  auto enc = encode_fn();
  CUtensorMap mq, mk, mv;
  if (!enc || !map4h(enc, &mq, q, 1, T, 1) || !map4h(enc, &mk, k, 1, T, 1) ||
      !map4h(enc, &mv, v, 1, T, 1))
    return -100;
  auto kern = stages >= 100 ? prologue_kernel<__nv_bfloat16, 96> : prologue_kernel<__nv_bfloat16>;
  stages %= 100;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sk::SMEM);
  kern<<<dim3(1, 2), 128, sk::SMEM>>>(mq, mk, mv, a, b, A_log, dt_bias, h0, T, 1, 1, scale, 1,
                                      (__nv_bfloat16*)o, out, status, stages);
  return (int)cudaGetLastError();
}

}  // extern "C"
