// launch.h -- internal launchers behind the C ABI (host side, C++).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdn {

struct ChunkArgs {
  const void* q; const void* k; const void* v; const void* a; const void* b;
  const void* w;  // GDN-2 write-gate logits, else NULL
  const float* A_log; const float* dt_bias; const float* h0;
  int B, T, Hk, Hv, dk, dv, dtype;
  float scale;
  int flags;
  void* o; float* ht;
  // gated RMSNorm of the output rows (o = RMSNormGated(core, z)); norm_z == NULL: none
  const void* norm_z = nullptr; const float* norm_w = nullptr; float norm_eps = 0.f;
  // packed batch (bf16 tensor-core path only): B sequences of the device table
  // vtab (chunk_layout.cuh) over T packed tokens, vNv chunks in all; NULL: dense
  const void* vtab = nullptr; int vNv = 0;
};

cudaError_t launch_gate_prep(const void* q, const void* k, int dtype, const void* a,
                             const void* b, const float* A_log, const float* dt_bias,
                             int B, int T, int Hk, int Hv, int d, float scale,
                             void* q_out, void* k_out, float* g_out, float* beta_out,
                             cudaStream_t s);

// Gated RMSNorm of the decode step's output rows; z == NULL: none.
struct DecodeNorm {
  const void* z = nullptr;  // [N, Hv, dv], the input dtype
  const float* w = nullptr; // [dv]
  float eps = 0.f;
};

cudaError_t launch_recurrent_step(const void* x, const float* conv_w, void* conv_state,
                                  const void* a, const void* b, const float* A_log,
                                  const float* dt_bias, float* state, void* o, int N,
                                  int Hk, int Hv, int dk, int dv, int dtype, float scale,
                                  bool out_f32, const DecodeNorm& nm, cudaStream_t s);

cudaError_t launch_conv_prefill(const void* x, const float* conv_w, void* conv_state, void* q,
                                void* k, void* v, int B, int T, int Hk, int Hv, int dk, int dv,
                                int dtype, cudaStream_t s);

// KDA on the Gated DeltaNet-2 path: beta [rows] tiled into b [rows][dk] and
// w [rows][dv] (elements of elem_bytes bytes, copied bit for bit).
cudaError_t launch_tie_gates(const void* beta, void* b, void* w, size_t rows, int dk, int dv,
                             int elem_bytes, cudaStream_t s);

cudaError_t launch_rmsnorm_gated(const void* o, const void* z, const float* weight, void* y,
                                 long rows, int dv, int dtype, float eps, cudaStream_t s);
// The same with float32 o / y and a bf16 gate z.
cudaError_t launch_rmsnorm_gated_f32_bf16z(const float* o, const void* z, const float* weight,
                                           float* y, long rows, int dv, float eps,
                                           cudaStream_t s);

// float32 CUDA-core chunk path (GDN and, with gdn2 = true, Gated DeltaNet-2).
cudaError_t launch_chunk_simt(const ChunkArgs& a, bool gdn2, cudaStream_t s);

// bf16 tensor-core chunk path (GDN and, with gdn2 = true, Gated DeltaNet-2;
// dk = dv = 128): WY prep + state scan, with its intermediates in a
// caller-provided workspace.
bool chunk_mma_supported(const ChunkArgs& a);
size_t chunk_mma_workspace_bytes(int B, int T, int Hk, int Hv);
cudaError_t launch_chunk_mma(const ChunkArgs& a, bool gdn2, void* workspace, cudaStream_t s);
// The GDN prep of that path on the tcgen05 tensor cores (one CTA per chunk and
// key head; writes the workspace the scan reads).
cudaError_t launch_prep_tc(const ChunkArgs& a, void* workspace, int* status, cudaStream_t s);
// The state scan of those paths on the tcgen05 tensor cores (reads the workspace
// the prep kernel wrote on the same stream).
cudaError_t launch_scan_tc(const ChunkArgs& a, const void* workspace, int* status, cudaStream_t s);

// Device address of this device's status word (set up once per device).
int* status_word();

// Test hook behind gdn_test_set_wait_fault: a site at which one kernel leaves a
// bounded wait to expire on purpose, and the poll limit of every bounded wait of
// the tensor-core chunk kernels (kWaitSpin unless a test lowered it).
constexpr unsigned kWaitSpin = 1u << 24;
enum WaitFaultSite { kFaultNone = 0, kFaultScanState = 1, kFaultPrepTiles = 2 };
struct WaitFault {
  int site;
  unsigned spin;
};
WaitFault wait_fault();

cudaError_t launch_copy_state(const float* h0, float* ht, size_t n, cudaStream_t s);
// Copy a packed batch's sequence table (passed by value) to device memory.
struct VarlenTab;
cudaError_t launch_varlen_table(const VarlenTab& tab, void* dst, cudaStream_t s);

// Arguments of the chunk backward (gdn_chunk_bwd); D = dk = dv.
struct BwdArgs {
  const void *q, *k, *v, *a, *b;
  const float *A_log, *dt_bias, *h0;
  const void* dout;
  const float* dht;
  int B, T, Hk, Hv, D, dtype;
  float scale;
  int flags;
  float *dq, *dk, *dv, *da, *db, *dA_log, *ddt_bias, *dh0;
};
// Workspace bytes of the backward for these sizes (fp32 intermediates).
size_t bwd_workspace_bytes(int B, int T, int Hk, int Hv, int D);
// The backward on the CUDA cores (T >= 1; the caller handles T = 0).
cudaError_t launch_chunk_bwd(const BwdArgs& a, void* workspace, cudaStream_t s);

}  // namespace gdn
