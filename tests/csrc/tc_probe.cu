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


}  // extern "C"
