// host_pipeline.cu -- gdn_chunk_fwd_host: the chunkwise GDN forward for inputs
// and outputs in host memory.  The sequence is cut into pieces of whole chunks;
// the inputs of piece i are copied in on one stream while piece i - 1 is
// computed on the caller's stream and the output of piece i - 2 is copied out on
// a third, so the two directions of the host link and the kernels overlap.  The
// state is carried from piece to piece in device memory (each piece's call takes
// the state the previous one left, the chunk recurrence run in order).
#include <cstring>
#include <mutex>

#include <stdint.h>

#include "chunk_layout.cuh"
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kMaxDevices = 64;

// Copy streams of a device, created on first use; the mutex orders the enqueue
// of concurrent calls on one device (their work itself is asynchronous).
struct CopyStreams {
  std::mutex mu;
  cudaStream_t in = nullptr, out = nullptr;
};
CopyStreams g_copy[kMaxDevices];

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Sizes of one token row of each array, and the device layout of the buffers.
struct HostPlan {
  int Tc, pieces;
  size_t row_q, row_k, row_v, row_g, row_o;  // bytes per (batch, token)
  size_t in_off[2][5], o_off[2], state_off, alog_off, dtb_off, ws_off, ws_bytes, total;
};

bool make_plan(int B, int T, int Hk, int Hv, int dk, int dv, int dtype, int flags,
               int piece_tokens, HostPlan* p) {
  if (B <= 0 || T <= 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return false;
  if (dtype != GDN_F32 && dtype != GDN_BF16) return false;
  const size_t es = dtype == GDN_F32 ? 4 : 2;
  const size_t ges = (flags & GDN_GATES_PRECOMPUTED) ? 4 : es;
  const size_t oes = (flags & GDN_OUT_F32) ? 4 : es;
  // piece length in whole chunks, rounded in 64-bit arithmetic (a piece_tokens near
  // INT_MAX must not wrap) and never longer than the sequence rounded up to a chunk
  long long Tc = piece_tokens;
  if (Tc <= 0) Tc = ((long long)T + 7) / 8;  // about eight pieces by default
  const long long Tmax = (((long long)T + kC - 1) / kC) * kC;
  if (Tmax > 0x7fffffc0LL) return false;
  if (Tc > Tmax) Tc = Tmax;
  Tc = ((Tc + kC - 1) / kC) * kC;  // whole chunks
  if (Tc < kC) Tc = kC;
  p->Tc = (int)Tc;
  p->pieces = (int)(((long long)T + Tc - 1) / Tc);
  p->row_q = (size_t)Hk * dk * es;
  p->row_k = p->row_q;
  p->row_v = (size_t)Hv * dv * es;
  p->row_g = (size_t)Hv * ges;
  p->row_o = (size_t)Hv * dv * oes;
  const size_t rows[5] = {p->row_q, p->row_k, p->row_v, p->row_g, p->row_g};
  size_t off = 0;
  for (int s = 0; s < 2; ++s)
    for (int j = 0; j < 5; ++j) {
      p->in_off[s][j] = off;
      off += up256((size_t)B * p->Tc * rows[j]);
    }
  for (int s = 0; s < 2; ++s) {
    p->o_off[s] = off;
    off += up256((size_t)B * p->Tc * p->row_o);
  }
  p->state_off = off;
  off += up256((size_t)B * Hv * dk * dv * 4);
  p->alog_off = off;
  off += up256((size_t)Hv * 4);
  p->dtb_off = off;
  off += up256((size_t)Hv * 4);
  p->ws_off = off;
  p->ws_bytes = gdn_chunk_workspace_bytes(B, p->Tc, Hk, Hv, dk, dv, dtype);
  off += up256(p->ws_bytes);
  p->total = off;
  return true;
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" size_t gdn_chunk_fwd_host_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv,
                                                     int dtype, int flags, int piece_tokens) {
  HostPlan p;
  if (!make_plan(B, T, Hk, Hv, dk, dv, dtype, flags, piece_tokens, &p)) return 0;
  return p.total;
}

extern "C" int gdn_chunk_fwd_host(const void* q, const void* k, const void* v, const void* a,
                                  const void* b, const float* A_log, const float* dt_bias,
                                  const float* h0, int B, int T, int Hk, int Hv, int dk, int dv,
                                  int dtype, float scale, int flags, void* o, float* ht,
                                  int piece_tokens, void* dev_ws, size_t dev_ws_bytes,
                                  gdn_stream_t stream) {
  if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  if (B == 0) return GDN_OK;
  const bool pre = (flags & GDN_GATES_PRECOMPUTED) != 0;
  if (q == nullptr || k == nullptr || v == nullptr || a == nullptr || b == nullptr ||
      (T > 0 && o == nullptr) || (!pre && (A_log == nullptr || dt_bias == nullptr)))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t state_bytes = (size_t)B * Hv * dk * dv * 4;
  if (T == 0) {  // ht = h0 (or zeros), after the work already on the stream
    if (ht == nullptr) return GDN_OK;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (h0) memcpy(ht, h0, state_bytes);
    else memset(ht, 0, state_bytes);
    return GDN_OK;
  }
  HostPlan p;
  if (!make_plan(B, T, Hk, Hv, dk, dv, dtype, flags, piece_tokens, &p)) return GDN_ERR_INVALID_ARG;
  if (dev_ws == nullptr || dev_ws_bytes < p.total ||
      (reinterpret_cast<uintptr_t>(dev_ws) & 255u) != 0)
    return GDN_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  CopyStreams& cs = g_copy[dev];
  std::lock_guard<std::mutex> lock(cs.mu);
  if (cs.in == nullptr) {
    if (cudaStreamCreateWithFlags(&cs.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&cs.out, cudaStreamNonBlocking) != cudaSuccess)
      return GDN_ERR_CUDA;
  }
  uint8_t* W = static_cast<uint8_t*>(dev_ws);
  float* state = reinterpret_cast<float*>(W + p.state_off);
  cudaEvent_t ev_start, ev_in[2], ev_comp[2], ev_out[2];
  cudaEvent_t* all[7] = {&ev_start, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
  int made = 0;
  for (; made < 7; ++made)
    if (cudaEventCreateWithFlags(all[made], cudaEventDisableTiming) != cudaSuccess) break;
  int rc = GDN_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && rc == GDN_OK) rc = GDN_ERR_CUDA;
    return e == cudaSuccess;
  };
  if (made < 7) rc = GDN_ERR_CUDA;
  // the buffers may still be in use by earlier work on the caller's stream
  if (rc == GDN_OK) ck(cudaEventRecord(ev_start, s));
  if (rc == GDN_OK) ck(cudaStreamWaitEvent(cs.in, ev_start, 0));
  if (rc == GDN_OK && !pre) {
    ck(cudaMemcpyAsync(W + p.alog_off, A_log, (size_t)Hv * 4, cudaMemcpyHostToDevice, cs.in));
    ck(cudaMemcpyAsync(W + p.dtb_off, dt_bias, (size_t)Hv * 4, cudaMemcpyHostToDevice, cs.in));
  }
  if (rc == GDN_OK && h0 != nullptr)
    ck(cudaMemcpyAsync(state, h0, state_bytes, cudaMemcpyHostToDevice, cs.in));
  const void* src[5] = {q, k, v, a, b};
  const size_t rows[5] = {p.row_q, p.row_k, p.row_v, p.row_g, p.row_g};
  for (int i = 0; i < p.pieces && rc == GDN_OK; ++i) {
    const int buf = i & 1, t0 = i * p.Tc, Tl = T - t0 < p.Tc ? T - t0 : p.Tc;
    // inputs of piece i (batch row bb: tokens t0 .. t0 + Tl of its [T][...] block)
    if (i >= 2) ck(cudaStreamWaitEvent(cs.in, ev_comp[buf], 0));
    for (int j = 0; j < 5 && rc == GDN_OK; ++j)
      ck(cudaMemcpy2DAsync(W + p.in_off[buf][j], (size_t)Tl * rows[j],
                           static_cast<const uint8_t*>(src[j]) + (size_t)t0 * rows[j],
                           (size_t)T * rows[j], (size_t)Tl * rows[j], B,
                           cudaMemcpyHostToDevice, cs.in));
    if (rc != GDN_OK) break;
    ck(cudaEventRecord(ev_in[buf], cs.in));
    // piece i on the caller's stream, the state carried in `state`
    ck(cudaStreamWaitEvent(s, ev_in[buf], 0));
    if (i >= 2) ck(cudaStreamWaitEvent(s, ev_out[buf], 0));
    if (rc != GDN_OK) break;
    const float* hin = (i == 0 && h0 == nullptr) ? nullptr : state;
    const int r = gdn_chunk_fwd(
        W + p.in_off[buf][0], W + p.in_off[buf][1], W + p.in_off[buf][2], W + p.in_off[buf][3],
        W + p.in_off[buf][4], pre ? nullptr : reinterpret_cast<const float*>(W + p.alog_off),
        pre ? nullptr : reinterpret_cast<const float*>(W + p.dtb_off), hin, B, Tl, Hk, Hv, dk, dv,
        dtype, scale, flags, W + p.o_off[buf], state, p.ws_bytes ? W + p.ws_off : nullptr,
        p.ws_bytes, stream);
    if (r != GDN_OK) {
      rc = r;
      break;
    }
    ck(cudaEventRecord(ev_comp[buf], s));
    // output of piece i
    ck(cudaStreamWaitEvent(cs.out, ev_comp[buf], 0));
    ck(cudaMemcpy2DAsync(static_cast<uint8_t*>(o) + (size_t)t0 * p.row_o, (size_t)T * p.row_o,
                         W + p.o_off[buf], (size_t)Tl * p.row_o, (size_t)Tl * p.row_o, B,
                         cudaMemcpyDeviceToHost, cs.out));
    ck(cudaEventRecord(ev_out[buf], cs.out));
  }
  if (rc == GDN_OK && ht != nullptr)
    ck(cudaMemcpyAsync(ht, state, state_bytes, cudaMemcpyDeviceToHost, s));
  // the caller's stream completes only after every copy of the call
  if (made == 7) {
    cudaEventRecord(ev_start, cs.out);
    cudaStreamWaitEvent(s, ev_start, 0);
    cudaEventRecord(ev_out[0], cs.in);
    cudaStreamWaitEvent(s, ev_out[0], 0);
  }
  for (int j = 0; j < made; ++j) cudaEventDestroy(*all[j]);
  return rc;
}
