// kda.cu -- KDA (Kimi Delta Attention) on the Gated DeltaNet-2 path.  KDA keeps
// the channel-wise decay of Gated DeltaNet-2 but one scalar beta per (token,
// head) for both the erase and the write: S_t = (I - beta k k^T) D_t S + beta k
// v^T, which is Gated DeltaNet-2 with b_t = beta_t 1 and w_t = beta_t 1
// ("Gated DeltaNet-2", sections 标量绑定的数学表达 and 退化兼容性).  This file
// tiles beta into the per-channel erase and write gate tiles the Gated
// DeltaNet-2 kernels read; the gates are copied bit for bit, so the result is
// exactly that of gdn2_chunk_fwd on tiled gates.
#include <stdint.h>

#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

// b[row][c] = beta[row] for c < dk, w[row][c] = beta[row] for c < dv (E: the gate
// element, 2 or 4 bytes, copied as raw bits).
template <typename E>
__global__ void tie_gates_kernel(const E* __restrict__ beta, E* __restrict__ b, E* __restrict__ w,
                                 size_t rows, int dk, int dv) {
  const size_t nb = rows * (size_t)dk, n = nb + rows * (size_t)dv;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    if (i < nb) {
      b[i] = beta[i / dk];
    } else {
      const size_t j = i - nb;
      w[j] = beta[j / dv];
    }
  }
}

}  // namespace

cudaError_t launch_tie_gates(const void* beta, void* b, void* w, size_t rows, int dk, int dv,
                             int elem_bytes, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const size_t n = rows * (size_t)(dk + dv);
  const size_t want = (n + 255) / 256;
  const unsigned grid = (unsigned)(want < 148 * 16 ? want : 148 * 16);
  if (elem_bytes == 2)
    tie_gates_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(beta),
                                                    static_cast<uint16_t*>(b),
                                                    static_cast<uint16_t*>(w), rows, dk, dv);
  else
    tie_gates_kernel<uint32_t><<<grid, 256, 0, s>>>(static_cast<const uint32_t*>(beta),
                                                    static_cast<uint32_t*>(b),
                                                    static_cast<uint32_t*>(w), rows, dk, dv);
  return cudaGetLastError();
}

}  // namespace gdn
