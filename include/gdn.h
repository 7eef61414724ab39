/*
 * gdn.h -- C ABI of libgdn.so, the B200 (sm_100a) Gated DeltaNet hot path.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer into memory the caller owns
 *    (allocated by any means: cudaMalloc, a PyTorch tensor, a pool).  The
 *    library never allocates, frees or synchronises; each call only enqueues
 *    kernels on `stream` and returns.  NULL stream = the legacy default stream.
 *    Exceptions, each stated at its entry point: gdn_check_status synchronises
 *    the stream by design; gdn_chunk_fwd_host takes HOST pointers, creates two
 *    copy streams per device on its first call (kept until the process exits),
 *    synchronises the stream when T = 0, and its copies to or from pageable
 *    (not page-locked) host memory are synchronous.
 *  - Layouts are dense, row-major, token-major, with no padding:
 *      q, k        [B, T, Hk, dk]
 *      v, o        [B, T, Hv, dv]
 *      a, b        [B, T, Hv]              (GDN gate inputs, one per value head)
 *      A_log,
 *      dt_bias     [Hv] float32
 *      h0, ht      [B, Hv, dk, dv] float32 (state S, key index first; o = S^T q)
 *    Value head hv reads key/query head hv / (Hv / Hk) (contiguous groups).
 *  - `dtype` selects the element type of q, k, v, a, b, x, o and the conv
 *    state: GDN_F32 (float) or GDN_BF16 (__nv_bfloat16).  States, A_log,
 *    dt_bias and conv weights are always float32; arithmetic is float32 with
 *    float32 accumulation.
 *  - Tensors moved in 16-byte pieces must be 16-byte aligned: q, k, v, o and
 *    q_out/k_out of the chunk and gate-prep calls, h0, ht, the decode state,
 *    conv_w, and the per-channel gates a, b_logit, w_logit of gdn2_chunk_fwd on
 *    its bf16 d = 128 path.  The other pointers (the GDN gates a, b, A_log,
 *    dt_bias, g/beta outputs, the decode x, o and conv_state) need only their
 *    element alignment.  Head
 *    dims dk, dv must be 64 or 128 (heads are tiled in 64-column blocks); Hv
 *    must be a multiple of Hk.
 *  - Return value: GDN_OK or a negative gdn_status.  Argument errors are
 *    detected on the host before anything is enqueued.  GDN_ERR_CUDA reports a
 *    launch failure (the CUDA error is left for cudaGetLastError).  Kernels
 *    whose waits on the tensor-memory / TMA pipeline are bounded record an
 *    expired wait in a device status word instead of hanging; the host reads
 *    it with gdn_check_status().
 *
 * Method (pages: "Qwen3.5" rainlin-net, section GDN详解; "从 Full Attention 到
 * Gated DeltaNet" sections 9-10; "gated-deltanet-qwen3.5" architecture diagram;
 * "Gated DeltaNet-2" zhichai, sections 新更新公式 and 高效训练):
 *    g_t = -exp(A_log) * softplus(a_t + dt_bias),  alpha_t = e^{g_t},
 *    beta_t = sigmoid(b_t),
 *    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *    o_t = S_t^T q_t.
 */
#ifndef GDN_B200_GDN_H_
#define GDN_B200_GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = -1, /* null / misaligned pointer, negative size, bad dtype */
  GDN_ERR_UNSUPPORTED = -2, /* head dim not 64/128, Hv % Hk != 0, ...           */
  GDN_ERR_CUDA = -3,        /* a kernel launch or driver call failed            */
  GDN_ERR_TIMEOUT = -4,     /* a bounded device-side wait expired               */
  GDN_ERR_WORKSPACE = -5,   /* workspace smaller than gdn_*_workspace_bytes()   */
  GDN_ERR_RANGE = -6        /* an intermediate left the range of its fp16      */
                            /* operand format; that call's outputs are invalid  */
} gdn_status;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Flags of the chunk and decode entry points. */
enum {
  GDN_QK_L2NORM = 1,         /* normalise q and k per head: x / sqrt(|x|^2 + 1e-6)
                                (chunk entry points; decode always normalises)   */
  GDN_GATES_PRECOMPUTED = 2, /* a holds g (float32), b holds beta (float32);
                                A_log and dt_bias are ignored and may be NULL
                                (chunk entry points)                             */
  GDN_OUT_F32 = 4            /* o is written as float32 whatever `dtype` is      */
};

/*
 * gdn_gate_prep -- the gate and L2-norm prologue as one elementwise kernel.
 * ("Qwen3.5", module skeleton: beta = sigmoid(b), g = -exp(A_log) *
 *  softplus(a + dt_bias) in float32; L2 norm and the 1/sqrt(dk) query scale
 *  are this library's reading of the pages, applied after the norm.)
 *   q, k       [B,T,Hk,d]  dtype, read
 *   a, b       [B,T,Hv]    dtype, read
 *   A_log,
 *   dt_bias    [Hv]        float32, read
 *   q_out,
 *   k_out      [B,T,Hk,d]  dtype, written: scale*q/|q|, k/|k| (may alias q, k)
 *   g_out,
 *   beta_out   [B,T,Hv]    float32, written
 */
int gdn_gate_prep(const void* q, const void* k, int dtype, const void* a,
                  const void* b, const float* A_log, const float* dt_bias,
                  int B, int T, int Hk, int Hv, int d, float scale, void* q_out,
                  void* k_out, float* g_out, float* beta_out,
                  gdn_stream_t stream);

/*
 * gdn_chunk_fwd -- chunkwise-parallel GDN prefill (chunk_gated_delta_rule;
 * "gated-deltanet-qwen3.5" training/prefill branch).  Each 64-token chunk is
 * solved in WY form: A = (I + tril(diag(beta) K K^T (.) Gamma, -1))^-1 by
 * forward substitution, W = A diag(beta gamma) K, U = A diag(beta) V,
 * U~ = U - W S, O = diag(gamma) Q S + tril(Q K^T (.) Gamma) U~,
 * S <- gamma_C S + (diag(gamma_C/gamma) K)^T U~  ("Gated DeltaNet-2",
 * 高效训练, with scalar decay).  The float32 state stays on chip across the
 * chunks of one (batch, value head, 64 value columns).  bf16 with
 * dk = dv = 128 runs on the tensor cores in two kernels (a chunk-parallel WY
 * prep that writes W, U, A_qk and per-row factors to the workspace, then a
 * scan over the chunks that keeps the state in registers); other shapes and
 * float32 run a float32 CUDA-core path with no workspace.
 *   q, k [B,T,Hk,dk], v [B,T,Hv,dv], a, b [B,T,Hv]: dtype, read
 *     (with GDN_GATES_PRECOMPUTED: a = g, b = beta, float32)
 *   A_log, dt_bias [Hv] float32, read (unused with GDN_GATES_PRECOMPUTED)
 *   h0 [B,Hv,dk,dv] float32, read; NULL = zero initial state
 *   o  [B,T,Hv,dv] dtype (float32 with GDN_OUT_F32), written
 *   ht [B,Hv,dk,dv] float32, written; NULL = not stored; may alias h0
 *   flags: GDN_QK_L2NORM | GDN_GATES_PRECOMPUTED | GDN_OUT_F32; scale
 *     multiplies q after the norm (pass 1/sqrt(dk) for the usual scaling).
 *   workspace / ws_bytes: device scratch owned by the caller, 16-byte aligned,
 *     at least gdn_chunk_workspace_bytes() bytes (may be NULL / 0 when that
 *     returns 0); its contents are overwritten and need no initialisation.
 *     Too small or misaligned -> GDN_ERR_WORKSPACE, nothing launched.
 *   T may be any value >= 0 (a partial last chunk is masked); T = 0 copies h0
 *   to ht (or zeros).
 */
int gdn_chunk_fwd(const void* q, const void* k, const void* v, const void* a,
                  const void* b, const float* A_log, const float* dt_bias,
                  const float* h0, int B, int T, int Hk, int Hv, int dk, int dv,
                  int dtype, float scale, int flags, void* o, float* ht,
                  void* workspace, size_t ws_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_gated_norm -- gdn_chunk_fwd whose output rows leave through the
 * gated RMSNorm of the layer's output stage ("gated-deltanet-qwen3.5", section
 * 输出门控与 RMSNorm: RMSNormGated(core_attn_out, z); "Qwen3.5" module skeleton,
 * self.norm(core_attn_out, z)), per (token, value head) over the dv columns:
 *   o = core / sqrt(mean(core^2) + eps) * norm_weight * SiLU(z),
 * core being the output gdn_chunk_fwd writes.  On the bf16 dk = dv = 128 path the
 * norm is applied in the scan's output epilogue before the single store of o (the
 * two column-half CTAs of a head run as a cluster and exchange the rows' sums of
 * squares through distributed shared memory), so core never reaches memory; the
 * float32 / d = 64 path runs the forward and then gdn_rmsnorm_gated on o in place.
 *   z           [B,T,Hv,dv] dtype, read; 16-byte aligned
 *   norm_weight [dv] float32, read (shared by every head)
 *   eps         0 <= eps <= 1 (1e-6 in the binding)
 *   everything else as gdn_chunk_fwd (same workspace size).
 * Returns as gdn_chunk_fwd.
 */
int gdn_chunk_fwd_gated_norm(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const float* A_log, const float* dt_bias,
                             const float* h0, const void* z, const float* norm_weight,
                             float eps, int B, int T, int Hk, int Hv, int dk, int dv,
                             int dtype, float scale, int flags, void* o, float* ht,
                             void* workspace, size_t ws_bytes, gdn_stream_t stream);

/* Workspace bytes gdn_chunk_fwd needs for these sizes: for the tensor-core
 * path (bf16, dk = dv = 128) B*Hv*(Tp*896 + (Tp/64)*1040) + B*Hk*Tp*512 with
 * Tp = T rounded up to a multiple of 64 (per padded token and value head: a W
 * row of 128 fp16, a U row of 128 float32 and an A_qk row of 64 fp16; per
 * padded token and key head: fp16 copies of the scan's q and k rows; 1040 B of
 * per-row factors per chunk and value head); 0 for every other case and for
 * B*T = 0.  gdn2_chunk_workspace_bytes is the same with Hk = Hv = H. */
size_t gdn_chunk_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv,
                                 int dtype);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd without a caller workspace.  The pages
 * have no counterpart: this is a convenience of this library for callers that
 * cannot hand out device memory.  The scratch is a fixed 64 MiB device array
 * inside the library (one per device, reserved when this function is first
 * used on that device); the call allocates nothing.
 *   Arguments, layouts and results are those of gdn_chunk_fwd.
 *   Capacity: calls with gdn_chunk_workspace_bytes(...) > 64 MiB return
 *     GDN_ERR_WORKSPACE and launch nothing (argument errors are reported
 *     first); calls that need no workspace run as gdn_chunk_fwd does.
 *   The array is shared by every call on a device: calls on different
 *     streams must not run concurrently (calls on one stream are ordered).
 */
int gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                          const void* a, const void* b, const float* A_log,
                          const float* dt_bias, const float* h0, int B, int T,
                          int Hk, int Hv, int dk, int dv, int dtype, float scale,
                          int flags, void* o, float* ht, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_host -- gdn_chunk_fwd for inputs and outputs in host memory.
 * The pages have no counterpart: this is this library's pipeline for data that
 * starts and ends on the host.  The sequence is cut into pieces of
 * piece_tokens tokens (a multiple of the 64-token chunk; <= 0 picks about
 * T / 8); the inputs of one piece are copied to the device while the previous
 * piece is computed and the output of the one before is copied back, on two
 * copy streams of the library; the state is carried from piece to piece on the
 * device, so the result is that of one gdn_chunk_fwd call (the pieces' chunk
 * boundaries are the call's).
 *   q, k, v, a, b, A_log, dt_bias, h0: host pointers, layouts and meaning as
 *     for gdn_chunk_fwd (page-locked memory gives asynchronous copies; other
 *     host memory is copied synchronously by the runtime).
 *   o, ht: host pointers, written.
 *   dev_ws / dev_ws_bytes: device scratch owned by the caller, 256-byte aligned,
 *     at least gdn_chunk_fwd_host_workspace_bytes() bytes (two sets of piece
 *     buffers, the state, the piece's chunk workspace) -> else GDN_ERR_WORKSPACE.
 *   stream: the pieces are computed on it, and it completes only after every
 *     copy of the call; the host buffers must stay valid until then.
 *   Returns the first error of gdn_chunk_fwd for a piece (what was already
 *   enqueued still completes on the stream), GDN_ERR_CUDA if a stream or event
 *   of the pipeline could not be made.  T = 0 copies h0 to ht (or zeros) after
 *   synchronising the stream.
 *   Resources: the two copy streams of a device are created on its first call
 *   and live until the process exits (they are reused by every later call);
 *   the call itself allocates no memory.
 */
int gdn_chunk_fwd_host(const void* q, const void* k, const void* v, const void* a,
                       const void* b, const float* A_log, const float* dt_bias,
                       const float* h0, int B, int T, int Hk, int Hv, int dk, int dv,
                       int dtype, float scale, int flags, void* o, float* ht,
                       int piece_tokens, void* dev_ws, size_t dev_ws_bytes,
                       gdn_stream_t stream);

/* Device scratch bytes gdn_chunk_fwd_host needs (0 for invalid sizes). */
size_t gdn_chunk_fwd_host_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv,
                                          int dtype, int flags, int piece_tokens);

/*
 * gdn_recurrent_step -- one-token decode step for N independent sequences
 * (recurrent_gated_delta_rule; "gated-deltanet-qwen3.5" inference branch,
 * conv_states and recurrent_states updated in place), fused with the causal
 * depthwise conv1d (kernel 4) + SiLU over the mixed [q | k | v] stream
 * ("从 Full Attention 到 Gated DeltaNet" section 10).
 *   x_qkv      [N, Cc] dtype, Cc = 2*Hk*dk + Hv*dv, channel order q | k | v;
 *              pre-conv input when conv_w != NULL, else already post-conv
 *   conv_w     [Cc, 4] float32 or NULL; tap 3 multiplies the newest input
 *   conv_state [N, Cc, 3] dtype, read and updated in place (index 2 newest);
 *              ignored when conv_w == NULL
 *   a, b       [N, Hv] dtype; A_log, dt_bias [Hv] float32
 *   state      [N, Hv, dk, dv] float32, read and updated in place
 *   o          [N, Hv, dv] dtype (float32 with GDN_OUT_F32), written
 *   q and k are L2-normalised per head; q is multiplied by scale after that.
 *   flags: 0 or GDN_OUT_F32.
 */
int gdn_recurrent_step(const void* x_qkv, const float* conv_w, void* conv_state,
                       const void* a, const void* b, const float* A_log,
                       const float* dt_bias, float* state, void* o, int N,
                       int Hk, int Hv, int dk, int dv, int dtype, float scale,
                       int flags, gdn_stream_t stream);

/*
 * gdn_recurrent_step_gated_norm -- gdn_recurrent_step with the gated RMSNorm of
 * the output stage ("gated-deltanet-qwen3.5", 输出门控与 RMSNorm) fused into the
 * store of o: o = core / sqrt(mean(core^2) + eps) * norm_weight * SiLU(z) per
 * (sequence, value head) over dv (the CTA that forms a row holds all of it).
 *   z           [N, Hv, dv] dtype, read (element aligned)
 *   norm_weight [dv] float32; eps in [0, 1]
 *   everything else as gdn_recurrent_step.
 */
int gdn_recurrent_step_gated_norm(const void* x_qkv, const float* conv_w, void* conv_state,
                                  const void* a, const void* b, const float* A_log,
                                  const float* dt_bias, float* state, const void* z,
                                  const float* norm_weight, float eps, void* o, int N,
                                  int Hk, int Hv, int dk, int dv, int dtype, float scale,
                                  int flags, gdn_stream_t stream);

/*
 * gdn_conv_prefill -- the causal depthwise conv1d (kernel 4) + SiLU over a
 * whole prefill of the mixed [q | k | v] channel stream ("从 Full Attention 到
 * Gated DeltaNet" section 10: x -> CausalConv1D -> SiLU -> q, k, v;
 * "gated-deltanet-qwen3.5" section 因果卷积 and its architecture diagram, whose
 * conv_states carry the window into the inference branch).  The same conv as
 * gdn_recurrent_step, over T tokens at once: running it, then T decode steps'
 * worth of inputs one at a time, gives the same window and outputs.
 *   x_qkv      [B, T, Cc] dtype, Cc = 2*Hk*dk + Hv*dv, channel order q | k | v
 *   conv_w     [Cc, 4] float32; tap 3 multiplies the newest input
 *   conv_state [B, Cc, 3] dtype (index 2 newest) or NULL.  Non-NULL: read as the
 *              three inputs before token 0, then overwritten with the last three
 *              inputs (for T < 3 partly the old window, shifted).  NULL: a zero
 *              window, and nothing is written.
 *   q, k       [B, T, Hk, dk] dtype, written: SiLU(conv) of the q / k channels
 *              (not normalised: gdn_chunk_fwd with GDN_QK_L2NORM applies the L2
 *              norm in its prologue)
 *   v          [B, T, Hv, dv] dtype, written
 *   Ownership: every pointer is a device pointer owned by the caller; x_qkv,
 *   conv_w, q, k and v 16-byte aligned, conv_state element aligned; q, k, v must
 *   not overlap x_qkv or each other.  Arithmetic in float32, outputs rounded to
 *   dtype once.  B = 0 or T = 0 enqueues nothing (the window is unchanged).
 *   Returns GDN_ERR_INVALID_ARG (null or misaligned pointer, negative size, bad
 *   dtype), GDN_ERR_UNSUPPORTED (dk or dv not 64 / 128, more than 65535 * 16
 *   tokens or 65535 sequences), GDN_ERR_CUDA (launch failure).
 */
int gdn_conv_prefill(const void* x_qkv, const float* conv_w, void* conv_state,
                     void* q, void* k, void* v, int B, int T, int Hk, int Hv,
                     int dk, int dv, int dtype, gdn_stream_t stream);

/*
 * gdn_chunk_bwd -- the backward of gdn_chunk_fwd: the gradients of
 * sum(o * dout) + sum(ht * dht) for the forward's o and final state ht, by
 * reverse-mode differentiation of the WY chunk form ("Gated DeltaNet-2",
 * sections 高效训练：WY 算法依然成立 and Gate-aware 反向传播, with the scalar
 * decay of GDN; "Qwen3.5" (rainlin-net), GDN详解, for the gates and norms).  It
 * recomputes the forward's per-chunk factors and every chunk's start state,
 * carries the state gradient from the last chunk to the first, forms the
 * per-chunk gradients, then applies the chain rule through the L2 norms of q, k
 * and through the gates.  fp32 arithmetic on the CUDA cores for both input
 * types.
 *   q, k [B,T,Hk,dk], v [B,T,Hv,dv], a, b [B,T,Hv], A_log, dt_bias, h0, flags
 *     (GDN_QK_L2NORM, GDN_GATES_PRECOMPUTED) and scale: as given to
 *     gdn_chunk_fwd, read.  dk = dv = 64 or 128 (else GDN_ERR_UNSUPPORTED).
 *   dout [B,T,Hv,dv] dtype, read: the gradient at o.
 *   dht [B,Hv,dk,dv] float32, read; NULL = zero gradient at the final state.
 *   dq, dk_out [B,T,Hk,dk] float32, written (summed over the value heads of
 *     each key head); dv_out [B,T,Hv,dv] float32, written.
 *   da, db [B,T,Hv] float32, written: the gradients with respect to the gate
 *     logits a and b, or with GDN_GATES_PRECOMPUTED with respect to g and beta.
 *   dA_log, ddt_bias [Hv] float32, written (summed over batch and tokens);
 *     unused (may be NULL) with GDN_GATES_PRECOMPUTED.
 *   dh0 [B,Hv,dk,dv] float32, written; NULL = not stored.
 *   workspace / ws_bytes: device scratch owned by the caller, 16-byte aligned, at
 *     least gdn_chunk_bwd_workspace_bytes() bytes, overwritten; too small or
 *     misaligned -> GDN_ERR_WORKSPACE, nothing launched.
 *   T = 0 writes dh0 = dht (or zeros) and zero dA_log, ddt_bias.
 * Errors as for gdn_chunk_fwd; asynchronous on `stream`.
 */
int gdn_chunk_bwd(const void* q, const void* k, const void* v, const void* a,
                  const void* b, const float* A_log, const float* dt_bias,
                  const float* h0, const void* dout, const float* dht, int B, int T,
                  int Hk, int Hv, int dk, int dv, int dtype, float scale, int flags,
                  float* dq, float* dk_out, float* dv_out, float* da, float* db,
                  float* dA_log, float* ddt_bias, float* dh0, void* workspace,
                  size_t ws_bytes, gdn_stream_t stream);

/* Workspace bytes gdn_chunk_bwd needs: fp32 intermediates, about
 * B*T*(Hv*(12*dv*4 + (2*dk*dv*4 + 8*64*64*4)/64) + Hk*2*dk*4) bytes (5.5 GB at
 * B=1, T=8192, Hk=16, Hv=64, d=128); 0 for T = 0, B = 0 or unsupported sizes. */
size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv);

/*
 * gdn_chunk_fwd_varlen -- gdn_chunk_fwd over a packed batch of N sequences of
 * different lengths: sequence i is tokens cu_seqlens[i] .. cu_seqlens[i+1] - 1
 * of the packed arrays, with its own initial and final state, and its chunks
 * start at its first token (the result of N one-sequence calls).  The pages
 * batch sequences by padding ("gated-deltanet-qwen3.5" architecture diagram,
 * apply_mask_to_padding_states); packing is this library's way to batch without
 * the padded tokens.
 *   q, k [T_total, Hk, dk]; v, o [T_total, Hv, dv]; a, b [T_total, Hv]
 *     (T_total = cu_seqlens[N] < 2^31), dtypes, flags and scale as for
 *     gdn_chunk_fwd.
 *   h0 / ht [N, Hv, dk, dv] float32 or NULL (ht may alias h0).
 *   cu_seqlens: HOST array of N + 1 int64, cu_seqlens[0] = 0, non-decreasing;
 *     read during the call only.  Empty sequences copy their h0 to ht.
 *   workspace / ws_bytes: device scratch owned by the caller, 16-byte aligned, at
 *     least gdn_chunk_varlen_workspace_bytes(cu_seqlens, ...) bytes (0: none
 *     needed) -> else GDN_ERR_WORKSPACE, nothing launched.
 *   The bf16 dk = dv = 128 path runs the whole batch as one prep and one state
 *   scan launch (per group of up to 1024 sequences, and of at most 65535 / Hv):
 *   the chunks of all sequences are numbered one after another, the prep takes
 *   every chunk of every sequence in one grid, and the scan one CTA pair per
 *   (sequence, value head).  A small kernel first copies the group's sequence
 *   table (passed by value) into the workspace.  The float32 and d = 64 path
 *   runs one call per sequence.
 *   Every sequence is checked before anything is enqueued.  Returns as
 *   gdn_chunk_fwd, and GDN_ERR_INVALID_ARG for a bad cu_seqlens.
 */
int gdn_chunk_fwd_varlen(const void* q, const void* k, const void* v, const void* a,
                         const void* b, const float* A_log, const float* dt_bias,
                         const float* h0, const long long* cu_seqlens, int N, int Hk, int Hv,
                         int dk, int dv, int dtype, float scale, int flags, void* o,
                         float* ht, void* workspace, size_t ws_bytes, gdn_stream_t stream);

/* Device workspace bytes gdn_chunk_fwd_varlen needs for this packed batch (its
 * host cu_seqlens, N + 1 entries); 0 for the float32 / d = 64 path, which needs
 * none, and for invalid arguments. */
size_t gdn_chunk_varlen_workspace_bytes(const long long* cu_seqlens, int N, int Hk, int Hv,
                                        int dk, int dv, int dtype);

/*
 * gdn_kda_chunk_fwd -- KDA (Kimi Delta Attention): the channel-wise decay of
 * Gated DeltaNet-2 with one scalar beta per (token, head) for both the erase
 * and the write, S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T,
 * o_t = S_t^T q_t ("Gated DeltaNet-2", sections 标量绑定的数学表达 and
 * 退化兼容性: Gated DeltaNet-2 with b_t = beta_t 1 and w_t = beta_t 1).  It tiles
 * beta into per-channel gate tiles in the workspace and runs gdn2_chunk_fwd's
 * kernels on them, so the result is bit for bit that call's on tiled gates.
 *   q, k, a [B,T,H,dk]; v [B,T,H,dv]; A_log, dt_bias [H,dk]; h0 / ht / o /
 *   scale / flags as for gdn2_chunk_fwd.
 *   beta [B,T,H]: the beta logit in dtype, or beta itself in float32 with
 *     GDN_GATES_PRECOMPUTED (a then holds the per-channel log-decay in float32).
 *   workspace / ws_bytes: device scratch owned by the caller, 16-byte aligned, at
 *     least gdn_kda_chunk_workspace_bytes() bytes (the tiled gates and
 *     gdn2_chunk_fwd's workspace) -> else GDN_ERR_WORKSPACE.
 *   Returns as gdn2_chunk_fwd.  B = 0 or T = 0 copies h0 to ht (or zeros).
 */
int gdn_kda_chunk_fwd(const void* q, const void* k, const void* v, const void* a,
                      const void* beta, const float* A_log, const float* dt_bias,
                      const float* h0, int B, int T, int H, int dk, int dv, int dtype,
                      float scale, int flags, void* o, float* ht, void* workspace,
                      size_t ws_bytes, gdn_stream_t stream);

/* Device workspace bytes gdn_kda_chunk_fwd needs (0 for invalid sizes). */
size_t gdn_kda_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype,
                                     int flags);

/*
 * gdn_rmsnorm_gated -- the gated RMSNorm of the core output
 * ("gated-deltanet-qwen3.5" section 输出门控与 RMSNorm: RMSNormGated(core_attn_out,
 * z), an RMSNorm and then the SwiGLU-like z gate), per row of d_v channels:
 *   y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z)
 *   o, z   [rows, dv] dtype: rows = B*T*Hv for the chunk path's o (layout
 *          [B,T,Hv,dv]) or N*Hv for the decode step's o; z the matching slice of
 *          the z projection
 *   weight [dv] float32, shared by every row (and head)
 *   y      [rows, dv] dtype, written; may be o or z (in place)
 *   eps    added to mean(o^2) inside the root, 0 <= eps <= 1 (1e-6 by default in
 *          the binding)
 *   Ownership: device pointers owned by the caller; o, z, y 16-byte aligned,
 *   weight float aligned.  Arithmetic in float32, y rounded to dtype once.
 *   rows = 0 enqueues nothing.  Returns GDN_ERR_INVALID_ARG (null or misaligned
 *   pointer, negative rows, bad dtype or eps), GDN_ERR_UNSUPPORTED (dv not 64 /
 *   128), GDN_ERR_CUDA (launch failure).
 */
int gdn_rmsnorm_gated(const void* o, const void* z, const float* weight, void* y,
                      long rows, int dv, int dtype, float eps, gdn_stream_t stream);

/*
 * gdn2_chunk_fwd -- chunkwise Gated DeltaNet-2 forward ("Gated DeltaNet-2",
 * 新更新公式 and 高效训练): channel-wise decay
 * D_t = diag(exp(-exp(A_log) (.) softplus(a_t + dt_bias))), erase gate
 * b_t = sigmoid(b_logit_t), write gate w_t = sigmoid(w_logit_t),
 * S_t = (I - k_t (b_t (.) k_t)^T) D_t S_{t-1} + k_t (w_t (.) v_t)^T,
 * o_t = S_t^T q_t.  One key head per value head (H heads).
 *   q, k    [B,T,H,dk]  dtype      v  [B,T,H,dv] dtype
 *   a,
 *   b_logit [B,T,H,dk]  dtype      w_logit [B,T,H,dv] dtype
 *     (with GDN_GATES_PRECOMPUTED: a = per-channel log-decay g, b_logit = b,
 *      w_logit = w, all float32)
 *   A_log, dt_bias [H,dk] float32 (unused with GDN_GATES_PRECOMPUTED)
 *   h0, ht [B,H,dk,dv] float32 (NULL allowed; ht may alias h0)
 *   o [B,T,H,dv] dtype (float32 with GDN_OUT_F32), written
 *   workspace / ws_bytes: as for gdn_chunk_fwd, sized by
 *     gdn2_chunk_workspace_bytes (bf16 with dk = dv = 128 runs on the tensor
 *     cores and needs it; other cases run a float32 CUDA-core path without).
 */
int gdn2_chunk_fwd(const void* q, const void* k, const void* v, const void* a,
                   const void* b_logit, const void* w_logit, const float* A_log,
                   const float* dt_bias, const float* h0, int B, int T, int H,
                   int dk, int dv, int dtype, float scale, int flags, void* o,
                   float* ht, void* workspace, size_t ws_bytes,
                   gdn_stream_t stream);

size_t gdn2_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);

/*
 * gdn_check_status -- waits for `stream`, then reads and clears the device
 * status word of the current device.  Returns GDN_OK, GDN_ERR_TIMEOUT if a
 * bounded wait in a kernel expired since the last check (reported first when
 * both happened), GDN_ERR_RANGE if an intermediate of the tensor-core chunk
 * path left the fp16 operand range (inputs far outside the method's domain,
 * e.g. queries or keys of norm >> 1 with GDN_QK_L2NORM off; large values alone
 * do not trigger it, the scan's power-of-2 range scale absorbs them), or
 * GDN_ERR_CUDA.  The word is shared by every call on the device, so a code
 * belongs to some call since the previous check.
 */
int gdn_check_status(gdn_stream_t stream);

/*
 * gdn_test_set_wait_fault -- test hook for the bounded device waits; the pages
 * have no counterpart.  It makes the next tensor-core chunk calls leave one wait
 * to expire on purpose, without anything left in flight on the GPU, so that a
 * test can check that the kernel returns and gdn_check_status reports
 * GDN_ERR_TIMEOUT:
 *   site 0: no fault (the default);
 *   site 1: the state scan issues no first products, so its epilogue's wait for
 *           them expires;
 *   site 2: the WY prep withholds its K / Q tile loads.
 *   spin_limit: polls before a wait gives up, for every bounded wait of those
 *   kernels (0 = the default, 2^24).  The setting is process-wide and stays
 *   until changed; the outputs of a faulted call are not valid.
 * Returns GDN_OK, or GDN_ERR_INVALID_ARG for an unknown site.
 */
int gdn_test_set_wait_fault(int site, unsigned spin_limit);

/* Human-readable name of a gdn_status value (static string). */
const char* gdn_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_GDN_H_ */
