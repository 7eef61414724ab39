// noalloc.cu -- gdn_chunk_fwd_noalloc: the chunkwise GDN forward with its
// scratch in a fixed, file-scope device array instead of a caller workspace.
// The array lives in this translation unit alone, so its device memory is
// reserved only when this entry point is first used on a device.
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of this device's copy of the array (looked up once per device).
void* static_scratch() {
  // host threads calling at once on a fresh device would race to fill the slot
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" int gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* a,
                                     const void* b, const float* A_log, const float* dt_bias,
                                     const float* h0, int B, int T, int Hk, int Hv, int dk,
                                     int dv, int dtype, float scale, int flags, void* o,
                                     float* ht, gdn_stream_t stream) {
  // Shapes that need no scratch, and invalid arguments, are handled exactly as
  // gdn_chunk_fwd handles them (it is called with no workspace).
  const size_t need = gdn_chunk_workspace_bytes(B, T, Hk, Hv, dk, dv, dtype);
  if (need == 0)
    return gdn_chunk_fwd(q, k, v, a, b, A_log, dt_bias, h0, B, T, Hk, Hv, dk, dv, dtype, scale,
                         flags, o, ht, nullptr, 0, stream);
  if (need > kStaticScratchBytes)  // argument errors first, else GDN_ERR_WORKSPACE; no launch
    return gdn_chunk_fwd(q, k, v, a, b, A_log, dt_bias, h0, B, T, Hk, Hv, dk, dv, dtype, scale,
                         flags, o, ht, nullptr, 0, stream);
  void* ws = static_scratch();
  if (ws == nullptr) return GDN_ERR_CUDA;
  return gdn_chunk_fwd(q, k, v, a, b, A_log, dt_bias, h0, B, T, Hk, Hv, dk, dv, dtype, scale,
                       flags, o, ht, ws, kStaticScratchBytes, stream);
}
