// chunk_layout.cuh -- constants and workspace layout shared by the kernels of
// the bf16 tensor-core chunk paths (the WY prep kernels and the state scans).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda_bf16.h>

namespace gdn {

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // dk = dv
constexpr int kScal = 260;     // floats per (head, chunk): fo[64], fs[64], gamma_C[128] (per state
                               // row), max|U|, pad
constexpr int kScGC = 2 * 64;  // offset of gamma_C in the scalar block
constexpr int kScMaxU = kScGC + 128;
constexpr float kF16Max = 65000.f;  // largest magnitude accepted for an fp16 operand

// Workspace of one call, per (batch, value head) unless noted; Tp = T rounded up to 64.
struct WsLayout {
  size_t w, u, a, qh, kh, scal, total;
};
inline WsLayout ws_layout(int B, int T, int Hk, int Hv) {
  const size_t Nc = ((size_t)T + kC - 1) / kC, Tp = Nc * kC;
  const size_t hv = (size_t)B * Hv, hk = (size_t)B * Hk;
  WsLayout L;
  L.w = 0;                                  // W      [B*Hv][Tp][128] f16
  L.u = L.w + hv * Tp * kD * 2;             // U      [B*Hv][Tp][128] f32
  L.a = L.u + hv * Tp * kD * 4;             // A_qk   [B*Hv][Tp][64]  f16
  L.qh = L.a + hv * Tp * kC * 2;            // Q rows [B*Hk][Tp][128] f16 (scan operand)
  L.kh = L.qh + hk * Tp * kD * 2;           // K rows [B*Hk][Tp][128] f16 (scan operand)
  L.scal = L.kh + hk * Tp * kD * 2;         // scalars [B*Hv][Nc][260] f32
  L.total = L.scal + hv * Nc * kScal * 4;
  return L;
}

// Packed batches of sequences of different lengths (gdn_chunk_fwd_varlen) run
// as one prep and one scan launch over a table with one entry per sequence:
// (first chunk in the packed chunk numbering, length, first token, 0).  The
// chunks of all sequences are numbered one after another (each sequence's first
// chunk starts at its first token), and the workspace is that of one batch row
// of Nv * 64 tokens (Nv chunks in all), followed by the table.  A launch pair
// takes at most kVarlenMaxSeqs sequences.
constexpr int kVarlenMaxSeqs = 1024;
struct VarlenTab {
  int n;
  int4 seq[kVarlenMaxSeqs];
};
inline size_t varlen_tab_offset(int Nv, int Hk, int Hv) {
  return (ws_layout(1, Nv * kC, Hk, Hv).total + 255) & ~size_t(255);
}
inline size_t varlen_ws_bytes(int Nv, int Hk, int Hv) {
  return varlen_tab_offset(Nv, Hk, Hv) + sizeof(int4) * kVarlenMaxSeqs;
}

// Two consecutive output values in the output type.
template <typename TO>
__device__ __forceinline__ void store2(TO* p, float x, float y);
template <>
__device__ __forceinline__ void store2<float>(float* p, float x, float y) {
  *reinterpret_cast<float2*>(p) = make_float2(x, y);
}
template <>
__device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float x, float y) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x, y);
}

}  // namespace gdn
