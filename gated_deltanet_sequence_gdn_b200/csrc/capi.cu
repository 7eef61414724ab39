// capi.cu -- the extern "C" entry points of libgdn.so declared in include/gdn.h:
// host-side argument validation, dispatch to the kernels, status reporting.
#include <stdint.h>

#include <atomic>
#include <memory>
#include <mutex>
#include <new>

#include "chunk_layout.cuh"
#include "common.cuh"
#include "launch.h"

namespace gdn {

// One status word per device; kernels with bounded waits get its address.
__device__ int g_gdn_status = 0;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
// element-aligned pointers (read with scalar loads): gates, decode inputs
bool ok_elem(const void* p, size_t elem) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) % elem) == 0;
}
size_t elem_size(int dtype) { return dtype == GDN_BF16 ? 2 : 4; }
bool ok_head_dim(int d) { return d == 64 || d == 128; }
bool ok_dtype(int t) { return t == GDN_F32 || t == GDN_BF16; }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

__global__ void copy_or_zero_kernel(const float* __restrict__ src, float* dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src ? src[i] : 0.f;
}

}  // namespace

int* status_word() {
  // one lookup per device; calls from several host threads may race to fill a slot,
  // which the lock serialises
  static std::mutex mu;
  static int* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gdn_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

namespace {
std::atomic<int> g_fault_site{kFaultNone};
std::atomic<unsigned> g_fault_spin{kWaitSpin};
}  // namespace

WaitFault wait_fault() { return WaitFault{g_fault_site.load(), g_fault_spin.load()}; }

cudaError_t launch_copy_state(const float* h0, float* ht, size_t n, cudaStream_t s) {
  if (n == 0 || ht == nullptr || h0 == ht) return cudaSuccess;
  const unsigned grid = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  copy_or_zero_kernel<<<grid, 256, 0, s>>>(h0, ht, n);
  return cudaGetLastError();
}

}  // namespace gdn

using namespace gdn;

extern "C" {

int gdn_version(void) { return 100; }  // 0.1.0

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_RANGE: return "GDN_ERR_RANGE";
    default: return "GDN_ERR_UNKNOWN";
  }
}

int gdn_gate_prep(const void* q, const void* k, int dtype, const void* a, const void* b,
                  const float* A_log, const float* dt_bias, int B, int T, int Hk, int Hv,
                  int d, float scale, void* q_out, void* k_out, float* g_out,
                  float* beta_out, gdn_stream_t stream) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(d) || Hv % Hk != 0) return GDN_ERR_UNSUPPORTED;
  if ((long)B * T == 0) return GDN_OK;
  const size_t es = elem_size(dtype);
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_elem(a, es) || !ok_elem(b, es) || !ok_elem(A_log, 4) ||
      !ok_elem(dt_bias, 4) || !ok_ptr(q_out) || !ok_ptr(k_out) || !ok_elem(g_out, 4) ||
      !ok_elem(beta_out, 4))
    return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_gate_prep(q, k, dtype, a, b, A_log, dt_bias, B, T, Hk, Hv, d, scale,
                                    q_out, k_out, g_out, beta_out, (cudaStream_t)stream));
}

size_t gdn_chunk_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int dtype) {
  if (B <= 0 || T <= 0 || Hk <= 0 || Hv <= 0 || Hv % Hk != 0) return 0;
  ChunkArgs c{};
  c.B = B; c.T = T; c.Hk = Hk; c.Hv = Hv; c.dk = dk; c.dv = dv; c.dtype = dtype;
  return chunk_mma_supported(c) ? chunk_mma_workspace_bytes(B, T, Hk, Hv) : 0;
}
size_t gdn2_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  return gdn_chunk_workspace_bytes(B, T, H, H, dk, dv, dtype);
}

static int validate_chunk(const ChunkArgs& c, bool gdn2) {
  if (c.B < 0 || c.T < 0 || c.Hk <= 0 || c.Hv <= 0 || !ok_dtype(c.dtype))
    return GDN_ERR_INVALID_ARG;
  if (c.flags & ~(GDN_QK_L2NORM | GDN_GATES_PRECOMPUTED | GDN_OUT_F32))
    return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(c.dk) || !ok_head_dim(c.dv) || c.Hv % c.Hk != 0) return GDN_ERR_UNSUPPORTED;
  if (!ok_opt(c.h0) || !ok_opt(c.ht)) return GDN_ERR_INVALID_ARG;
  if ((long)c.B * c.T == 0) return GDN_OK;
  const size_t ges = (c.flags & GDN_GATES_PRECOMPUTED) ? 4 : elem_size(c.dtype);
  if (!ok_ptr(c.q) || !ok_ptr(c.k) || !ok_ptr(c.v) || !ok_elem(c.a, ges) ||
      !ok_elem(c.b, ges) || !ok_ptr(c.o))
    return GDN_ERR_INVALID_ARG;
  if (gdn2 && !ok_elem(c.w, ges)) return GDN_ERR_INVALID_ARG;
  // the GDN-2 tensor-core prep copies its gate tiles in 16-byte pieces
  if (gdn2 && chunk_mma_supported(c) && (!aligned16(c.a) || !aligned16(c.b) || !aligned16(c.w)))
    return GDN_ERR_INVALID_ARG;
  if (!(c.flags & GDN_GATES_PRECOMPUTED) && (!ok_elem(c.A_log, 4) || !ok_elem(c.dt_bias, 4)))
    return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

static int run_chunk(const ChunkArgs& c, bool gdn2, void* ws, size_t ws_bytes,
                     cudaStream_t s) {
  const size_t state_elems = (size_t)c.B * c.Hv * c.dk * c.dv;
  if (c.T == 0 || c.B == 0) return from_cuda(launch_copy_state(c.h0, c.ht, state_elems, s));
  if (chunk_mma_supported(c)) {
    if (ws == nullptr || !aligned16(ws) ||
        ws_bytes < chunk_mma_workspace_bytes(c.B, c.T, c.Hk, c.Hv))
      return GDN_ERR_WORKSPACE;
    return from_cuda(launch_chunk_mma(c, gdn2, ws, s));
  }
  return from_cuda(launch_chunk_simt(c, gdn2, s));
}

int gdn_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                  const float* A_log, const float* dt_bias, const float* h0, int B, int T,
                  int Hk, int Hv, int dk, int dv, int dtype, float scale, int flags, void* o,
                  float* ht, void* workspace, size_t ws_bytes, gdn_stream_t stream) {
  ChunkArgs c{q, k, v, a, b, nullptr, A_log, dt_bias, h0, B, T, Hk, Hv, dk, dv, dtype,
              scale, flags, o, ht};
  int st = validate_chunk(c, false);
  if (st != GDN_OK) return st;
  return run_chunk(c, false, workspace, ws_bytes, (cudaStream_t)stream);
}

int gdn_chunk_fwd_gated_norm(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const float* A_log, const float* dt_bias,
                             const float* h0, const void* z, const float* norm_weight, float eps,
                             int B, int T, int Hk, int Hv, int dk, int dv, int dtype, float scale,
                             int flags, void* o, float* ht, void* workspace, size_t ws_bytes,
                             gdn_stream_t stream) {
  ChunkArgs c{q, k, v, a, b, nullptr, A_log, dt_bias, h0, B, T, Hk, Hv, dk, dv, dtype,
              scale, flags, o, ht};
  int st = validate_chunk(c, false);
  if (st != GDN_OK) return st;
  if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if ((long)B * T == 0) return run_chunk(c, false, workspace, ws_bytes, s);
  if (!ok_ptr(z) || !ok_elem(norm_weight, 4)) return GDN_ERR_INVALID_ARG;
  if (chunk_mma_supported(c)) {  // fused into the scan's output rows
    c.norm_z = z;
    c.norm_w = norm_weight;
    c.norm_eps = eps;
    return run_chunk(c, false, workspace, ws_bytes, s);
  }
  // the float32 / d = 64 path: the forward, then the gated RMSNorm over o in place
  st = run_chunk(c, false, workspace, ws_bytes, s);
  if (st != GDN_OK) return st;
  const long rows = (long)B * T * Hv;
  if (dtype == GDN_BF16 && (flags & GDN_OUT_F32))  // float32 cores, bf16 gate
    return from_cuda(launch_rmsnorm_gated_f32_bf16z(static_cast<float*>(o), z, norm_weight,
                                                    static_cast<float*>(o), rows, dv, eps, s));
  return from_cuda(launch_rmsnorm_gated(o, z, norm_weight, o, rows, dv, dtype, eps, s));
}

size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv) {
  if (B <= 0 || T <= 0 || Hk <= 0 || Hv <= 0 || dk != dv || !ok_head_dim(dk)) return 0;
  return bwd_workspace_bytes(B, T, Hk, Hv, dk);
}

int gdn_chunk_bwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                  const float* A_log, const float* dt_bias, const float* h0, const void* dout,
                  const float* dht, int B, int T, int Hk, int Hv, int dk, int dv, int dtype,
                  float scale, int flags, float* dq, float* dk_out, float* dv_out, float* da,
                  float* db, float* dA_log, float* ddt_bias, float* dh0, void* workspace,
                  size_t ws_bytes, gdn_stream_t stream) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (flags & ~(GDN_QK_L2NORM | GDN_GATES_PRECOMPUTED)) return GDN_ERR_INVALID_ARG;
  if (dk != dv || !ok_head_dim(dk) || Hv % Hk != 0) return GDN_ERR_UNSUPPORTED;
  if (!ok_opt(h0) || !ok_opt(dht) || !ok_opt(dh0)) return GDN_ERR_INVALID_ARG;
  const bool pre = (flags & GDN_GATES_PRECOMPUTED) != 0;
  if (!pre && (!ok_elem(A_log, 4) || !ok_elem(dt_bias, 4) || !ok_elem(dA_log, 4) ||
               !ok_elem(ddt_bias, 4)))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if ((long)B * T == 0) {  // no tokens: dh0 = dht, and nothing flows to the gates' parameters
    if (dh0) {
      const cudaError_t e = launch_copy_state(dht, dh0, (size_t)B * Hv * dk * dv, s);
      if (e != cudaSuccess) return from_cuda(e);
    }
    if (!pre) {
      cudaError_t e = cudaMemsetAsync(dA_log, 0, sizeof(float) * Hv, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(ddt_bias, 0, sizeof(float) * Hv, s);
      return from_cuda(e);
    }
    return GDN_OK;
  }
  const size_t ges = pre ? 4 : elem_size(dtype);
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_elem(a, ges) || !ok_elem(b, ges) ||
      !ok_ptr(dout) || !ok_ptr(dq) || !ok_ptr(dk_out) || !ok_ptr(dv_out) || !ok_elem(da, 4) ||
      !ok_elem(db, 4))
    return GDN_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace) ||
      ws_bytes < gdn_chunk_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv))
    return GDN_ERR_WORKSPACE;
  BwdArgs args{q,    k,     v,     a,  b,      A_log,  dt_bias, h0,     dout,
               dht,  B,     T,     Hk, Hv,     dk,     dtype,   scale,  flags,
               dq,   dk_out, dv_out, da, db,   dA_log, ddt_bias, dh0};
  return from_cuda(launch_chunk_bwd(args, workspace, s));
}

// Sequence i of a packed batch: the arguments of a one-sequence gdn_chunk_fwd call
// on its token range [t0, t0 + Ti) and its own initial / final state.
static ChunkArgs varlen_seq(const ChunkArgs& all, long long t0, int Ti, int i) {
  const size_t es = elem_size(all.dtype);
  const size_t ges = (all.flags & GDN_GATES_PRECOMPUTED) ? 4 : es;
  const size_t oes = (all.flags & GDN_OUT_F32) ? 4 : es;
  const size_t st = (size_t)all.Hv * all.dk * all.dv;
  auto at = [](const void* p, size_t off) -> const void* {
    return p ? static_cast<const uint8_t*>(p) + off : nullptr;
  };
  ChunkArgs c = all;
  c.q = at(all.q, (size_t)t0 * all.Hk * all.dk * es);
  c.k = at(all.k, (size_t)t0 * all.Hk * all.dk * es);
  c.v = at(all.v, (size_t)t0 * all.Hv * all.dv * es);
  c.a = at(all.a, (size_t)t0 * all.Hv * ges);
  c.b = at(all.b, (size_t)t0 * all.Hv * ges);
  c.o = all.o ? static_cast<uint8_t*>(all.o) + (size_t)t0 * all.Hv * all.dv * oes : nullptr;
  c.h0 = all.h0 ? all.h0 + (size_t)i * st : nullptr;
  c.ht = all.ht ? all.ht + (size_t)i * st : nullptr;
  c.B = 1;
  c.T = Ti;
  return c;
}

// Sequences per launch pair of a packed batch: at most kVarlenMaxSeqs, and few
// enough that the scan's grid (2, sequences x Hv) stays within 65535 rows.
static int varlen_group(int Hv) { return Hv > 0 && 65535 / Hv < kVarlenMaxSeqs ? 65535 / Hv : kVarlenMaxSeqs; }

// Chunks of the packed batch's sequences i0 .. i1 - 1 (each starts a new chunk).
static long long varlen_chunks(const long long* cu, int i0, int i1) {
  long long nv = 0;
  for (int i = i0; i < i1; ++i) nv += (cu[i + 1] - cu[i] + kC - 1) / kC;
  return nv;
}

// cu_seqlens starts at 0, does not decrease, and the packed token count fits an int.
static bool varlen_offsets_ok(const long long* cu, int N) {
  if (cu == nullptr || cu[0] != 0) return false;
  for (int i = 0; i < N; ++i)
    if (cu[i + 1] < cu[i]) return false;
  return cu[N] <= 0x7fffffffLL;
}

size_t gdn_chunk_varlen_workspace_bytes(const long long* cu_seqlens, int N, int Hk, int Hv,
                                        int dk, int dv, int dtype) {
  if (N <= 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype) || !varlen_offsets_ok(cu_seqlens, N))
    return 0;
  ChunkArgs probe{};
  probe.B = 1, probe.T = 1, probe.Hk = Hk, probe.Hv = Hv, probe.dk = dk, probe.dv = dv;
  probe.dtype = dtype;
  if (!chunk_mma_supported(probe)) return 0;  // the CUDA-core path needs none
  const int G = varlen_group(Hv);
  size_t need = 0;
  for (int i0 = 0; i0 < N; i0 += G) {
    const long long nv = varlen_chunks(cu_seqlens, i0, i0 + G < N ? i0 + G : N);
    if (nv > 0x7fffffffLL / kC) return 0;
    const size_t b = varlen_ws_bytes((int)nv, Hk, Hv);
    need = b > need ? b : need;
  }
  return need;
}

int gdn_chunk_fwd_varlen(const void* q, const void* k, const void* v, const void* a,
                         const void* b, const float* A_log, const float* dt_bias,
                         const float* h0, const long long* cu_seqlens, int N, int Hk, int Hv,
                         int dk, int dv, int dtype, float scale, int flags, void* o, float* ht,
                         void* workspace, size_t ws_bytes, gdn_stream_t stream) {
  if (N < 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (N == 0) return GDN_OK;
  if (!varlen_offsets_ok(cu_seqlens, N)) return GDN_ERR_INVALID_ARG;
  const ChunkArgs all{q, k, v, a, b, nullptr, A_log, dt_bias, h0, 1, 0, Hk, Hv, dk, dv,
                      dtype, scale, flags, o, ht};
  // every sequence is checked before anything is enqueued
  for (int i = 0; i < N; ++i) {
    const int Ti = (int)(cu_seqlens[i + 1] - cu_seqlens[i]);
    const int st = validate_chunk(varlen_seq(all, cu_seqlens[i], Ti, i), false);
    if (st != GDN_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  ChunkArgs probe = all;
  probe.T = 1;
  if (!chunk_mma_supported(probe)) {  // the CUDA-core path: one call per sequence
    for (int i = 0; i < N; ++i) {
      const int Ti = (int)(cu_seqlens[i + 1] - cu_seqlens[i]);
      const int st = run_chunk(varlen_seq(all, cu_seqlens[i], Ti, i), false, nullptr, 0, s);
      if (st != GDN_OK) return st;
    }
    return GDN_OK;
  }
  // the tensor-core path: one prep and one scan launch per group of sequences
  const size_t need = gdn_chunk_varlen_workspace_bytes(cu_seqlens, N, Hk, Hv, dk, dv, dtype);
  if (need == 0 || workspace == nullptr || !aligned16(workspace) || ws_bytes < need)
    return GDN_ERR_WORKSPACE;
  const size_t st_elems = (size_t)Hv * dk * dv;
  const int G = varlen_group(Hv);
  std::unique_ptr<VarlenTab> tp(new (std::nothrow) VarlenTab);  // 16 KB, host memory
  if (!tp) return GDN_ERR_CUDA;
  VarlenTab& tab = *tp;
  for (int i0 = 0; i0 < N; i0 += G) {
    const int i1 = i0 + G < N ? i0 + G : N;
    tab.n = i1 - i0;
    int nv = 0;
    for (int i = i0; i < i1; ++i) {
      const int Ti = (int)(cu_seqlens[i + 1] - cu_seqlens[i]);
      tab.seq[i - i0] = make_int4(nv, Ti, (int)cu_seqlens[i], 0);
      nv += (Ti + kC - 1) / kC;
    }
    ChunkArgs g = all;
    g.B = i1 - i0;
    g.T = (int)cu_seqlens[N];
    g.h0 = h0 ? h0 + (size_t)i0 * st_elems : nullptr;
    g.ht = ht ? ht + (size_t)i0 * st_elems : nullptr;
    cudaError_t e;
    if (nv == 0) {  // only empty sequences: their states are copied
      e = launch_copy_state(g.h0, g.ht, (size_t)g.B * st_elems, s);
    } else {
      uint8_t* tabp = static_cast<uint8_t*>(workspace) + varlen_tab_offset(nv, Hk, Hv);
      e = launch_varlen_table(tab, tabp, s);
      g.vtab = tabp;
      g.vNv = nv;
      if (e == cudaSuccess) e = launch_chunk_mma(g, false, workspace, s);
    }
    if (e != cudaSuccess) return from_cuda(e);
  }
  return GDN_OK;
}

int gdn2_chunk_fwd(const void* q, const void* k, const void* v, const void* a,
                   const void* b_logit, const void* w_logit, const float* A_log,
                   const float* dt_bias, const float* h0, int B, int T, int H, int dk, int dv,
                   int dtype, float scale, int flags, void* o, float* ht, void* workspace,
                   size_t ws_bytes, gdn_stream_t stream) {
  ChunkArgs c{q, k, v, a, b_logit, w_logit, A_log, dt_bias, h0, B, T, H, H, dk, dv, dtype,
              scale, flags, o, ht};
  int st = validate_chunk(c, true);
  if (st != GDN_OK) return st;
  return run_chunk(c, true, workspace, ws_bytes, (cudaStream_t)stream);
}

// KDA workspace: gdn2_chunk_fwd's, then the tiled erase gates [B*T*H][dk] and
// the tiled write gates [B*T*H][dv], each rounded up to 256 bytes.
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
static bool kda_layout(int B, int T, int H, int dk, int dv, int dtype, int flags, size_t* ws2,
                       size_t* tb, size_t* tw) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || !ok_dtype(dtype)) return false;
  const size_t ges = (flags & GDN_GATES_PRECOMPUTED) ? 4 : elem_size(dtype);
  const size_t rows = (size_t)B * T * H;
  *ws2 = up256(gdn2_chunk_workspace_bytes(B, T, H, dk, dv, dtype));
  *tb = up256(rows * dk * ges);
  *tw = up256(rows * dv * ges);
  return true;
}

size_t gdn_kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype, int flags) {
  size_t ws2, tb, tw;
  if (!kda_layout(B, T, H, dk, dv, dtype, flags, &ws2, &tb, &tw)) return 0;
  return ws2 + tb + tw;
}

int gdn_kda_chunk_fwd(const void* q, const void* k, const void* v, const void* a,
                      const void* beta, const float* A_log, const float* dt_bias,
                      const float* h0, int B, int T, int H, int dk, int dv, int dtype,
                      float scale, int flags, void* o, float* ht, void* workspace,
                      size_t ws_bytes, gdn_stream_t stream) {
  size_t ws2, tb, tw;
  if (!kda_layout(B, T, H, dk, dv, dtype, flags, &ws2, &tb, &tw)) return GDN_ERR_INVALID_ARG;
  uint8_t* W = static_cast<uint8_t*>(workspace);
  const bool any = (long)B * T > 0;
  // the gate tiles live in the workspace; the Gated DeltaNet-2 checks run on them
  ChunkArgs c{q, k, v, a, any ? W + ws2 : nullptr, any ? W + ws2 + tb : nullptr, A_log, dt_bias,
              h0, B, T, H, H, dk, dv, dtype, scale, flags, o, ht};
  if (any) {
    const size_t ges = (flags & GDN_GATES_PRECOMPUTED) ? 4 : elem_size(dtype);
    if (!ok_elem(beta, ges)) return GDN_ERR_INVALID_ARG;
    if (W == nullptr || !aligned16(W) || ws_bytes < ws2 + tb + tw) return GDN_ERR_WORKSPACE;
  }
  int st = validate_chunk(c, true);
  if (st != GDN_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (any) {
    const size_t ges = (flags & GDN_GATES_PRECOMPUTED) ? 4 : elem_size(dtype);
    st = from_cuda(launch_tie_gates(beta, W + ws2, W + ws2 + tb, (size_t)B * T * H, dk, dv,
                                    (int)ges, s));
    if (st != GDN_OK) return st;
  }
  return run_chunk(c, true, any ? W : nullptr, ws2, s);
}

int gdn_recurrent_step(const void* x_qkv, const float* conv_w, void* conv_state, const void* a,
                       const void* b, const float* A_log, const float* dt_bias, float* state,
                       void* o, int N, int Hk, int Hv, int dk, int dv, int dtype, float scale,
                       int flags, gdn_stream_t stream) {
  if (N < 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (flags & ~GDN_OUT_F32) return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(dk) || !ok_head_dim(dv) || Hv % Hk != 0) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  const size_t es = elem_size(dtype);
  if (!ok_elem(x_qkv, es) || !ok_elem(a, es) || !ok_elem(b, es) || !ok_elem(A_log, 4) ||
      !ok_elem(dt_bias, 4) || !ok_ptr(state) || !ok_elem(o, (flags & GDN_OUT_F32) ? 4 : es) ||
      !ok_opt(conv_w))
    return GDN_ERR_INVALID_ARG;
  if (conv_w != nullptr && !ok_elem(conv_state, es)) return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_recurrent_step(x_qkv, conv_w, conv_state, a, b, A_log, dt_bias,
                                         state, o, N, Hk, Hv, dk, dv, dtype, scale,
                                         (flags & GDN_OUT_F32) != 0, DecodeNorm{},
                                         (cudaStream_t)stream));
}

int gdn_recurrent_step_gated_norm(const void* x_qkv, const float* conv_w, void* conv_state,
                                  const void* a, const void* b, const float* A_log,
                                  const float* dt_bias, float* state, const void* z,
                                  const float* norm_weight, float eps, void* o, int N, int Hk,
                                  int Hv, int dk, int dv, int dtype, float scale, int flags,
                                  gdn_stream_t stream) {
  if (N < 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (flags & ~GDN_OUT_F32) return GDN_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(dk) || !ok_head_dim(dv) || Hv % Hk != 0) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  const size_t es = elem_size(dtype);
  if (!ok_elem(x_qkv, es) || !ok_elem(a, es) || !ok_elem(b, es) || !ok_elem(A_log, 4) ||
      !ok_elem(dt_bias, 4) || !ok_ptr(state) || !ok_elem(o, (flags & GDN_OUT_F32) ? 4 : es) ||
      !ok_opt(conv_w) || !ok_elem(z, es) || !ok_elem(norm_weight, 4))
    return GDN_ERR_INVALID_ARG;
  if (conv_w != nullptr && !ok_elem(conv_state, es)) return GDN_ERR_INVALID_ARG;
  DecodeNorm nm;
  nm.z = z;
  nm.w = norm_weight;
  nm.eps = eps;
  return from_cuda(launch_recurrent_step(x_qkv, conv_w, conv_state, a, b, A_log, dt_bias,
                                         state, o, N, Hk, Hv, dk, dv, dtype, scale,
                                         (flags & GDN_OUT_F32) != 0, nm, (cudaStream_t)stream));
}

int gdn_conv_prefill(const void* x_qkv, const float* conv_w, void* conv_state, void* q, void* k,
                     void* v, int B, int T, int Hk, int Hv, int dk, int dv, int dtype,
                     gdn_stream_t stream) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || !ok_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(dk) || !ok_head_dim(dv)) return GDN_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return GDN_OK;
  if ((T + 15) / 16 > 65535 || B > 65535) return GDN_ERR_UNSUPPORTED;
  if (!ok_ptr(x_qkv) || !ok_ptr(conv_w) || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) ||
      (conv_state != nullptr && !ok_elem(conv_state, elem_size(dtype))))
    return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_conv_prefill(x_qkv, conv_w, conv_state, q, k, v, B, T, Hk, Hv, dk, dv,
                                       dtype, (cudaStream_t)stream));
}

int gdn_rmsnorm_gated(const void* o, const void* z, const float* weight, void* y, long rows,
                      int dv, int dtype, float eps, gdn_stream_t stream) {
  if (rows < 0 || !ok_dtype(dtype) || !(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
  if (!ok_head_dim(dv)) return GDN_ERR_UNSUPPORTED;
  if (rows == 0) return GDN_OK;
  if (!ok_ptr(o) || !ok_ptr(z) || !ok_ptr(y) || !ok_elem(weight, 4)) return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_rmsnorm_gated(o, z, weight, y, rows, dv, dtype, eps,
                                        (cudaStream_t)stream));
}

int gdn_check_status(gdn_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDN_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_gdn_status, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_gdn_status, &zero, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    // an expired wait is reported first: the outputs after it are not computed at all
    return (h & ~kStatusRange) ? GDN_ERR_TIMEOUT : GDN_ERR_RANGE;
  }
  return GDN_OK;
}

int gdn_test_set_wait_fault(int site, unsigned spin_limit) {
  if (site < kFaultNone || site > kFaultPrepTiles) return GDN_ERR_INVALID_ARG;
  g_fault_site.store(site);
  g_fault_spin.store(spin_limit == 0 ? kWaitSpin : spin_limit);
  return GDN_OK;
}

}  // extern "C"
