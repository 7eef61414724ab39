// scan_tc.cu -- the sequential state scan of the bf16 chunk paths on the tcgen05
// tensor cores (sm_100a): one CTA per (batch, value head, 64-column half of d_v),
// over the chunks of the sequence, with
//   [O_q; P] = [Q; W] S          (M = 128: Q rows in TMEM lanes 0-63, W rows in 64-127)
//   U~ = sigma U - P,  U~s = U~ diag(fs)
//   O_a = A_qk U~                (M = 128; lanes 64-127 of the result are unused)
//   DS = K^T U~s                 (M = 128 over the d_k rows of the state)
//   o = (fo O_q + O_a) / sigma,  S <- diag(gamma_C) S + DS
// The operands come from the workspace written by the prep kernels (fp16 W, A_qk,
// scan Q / K rows; fp32 U; per-chunk factors), see chunk_mma.cu for the algebra,
// the precision design and the range scale sigma.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: every tile of chunk n into stage n % 2 (10 bulk copies,
//               the [Q; W] tiles and the rest on separate barriers)
//               (the whole warp also allocates and releases the TMEM)
//   warp 1      tcgen05.mma issue (lane 0)
//   warps 2-9   epilogue, two warps per TMEM lane quarter (warps w and w + 4 take
//               columns 0-31 and 32-63): 32 columns of one state row (d_k row =
//               TMEM lane) per thread in fp32 registers; TMEM loads of the
//               accumulators, U~ / U~s / the state written back to shared memory
//               as fp16 operands, o stored.
// Per chunk the chain is [Q; W] S -> U~ (epilogue) -> DS -> state (epilogue) ->
// next chunk, with O_a issued behind DS and run while the state is updated.  The
// epilogue hands its operands to the MMA warp through a hardware named barrier
// that the MMA warp waits on (and that carries the vote on giving up), so the
// issue follows the last epilogue store without an mbarrier round trip, and no
// epilogue warp waits while the tensor pipe accepts the products.
// The tensor cores report completion through mbarriers (tcgen05.commit), the TMA
// producer through transaction counts; every wait is bounded and an expired wait
// ends the kernel through the status word (GDN_ERR_TIMEOUT) after its copies and
// tensor-core work in flight have drained.
//
// With NORM the output rows leave through the gated RMSNorm of the pages'
// output stage, y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) over the d_v columns
// of each (token, value head) ("gated-deltanet-qwen3.5", 输出门控与 RMSNorm).
// A row's columns are split over the two column-half CTAs of a head, which then
// run as a cluster of two: each sends the sums of squares of its 64 columns of
// the chunk's rows to the other through distributed shared memory (st.async into
// the peer's buffer, counted as transaction bytes on the peer's mbarrier, so no
// release fence waits on output stores).  The output-row threads (TMEM lanes
// 0-63) leave the chunk's rows in shared memory, with their gate z copied in
// behind them; during the next chunk step the P-row threads, which run on the
// other two SM sub-partitions and are idle after the state update, normalise and
// store them.  The peer's sums have a whole chunk step to arrive.
#include "chunk_layout.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace gdn {
namespace {

using namespace tc;
using bf16 = __nv_bfloat16;

constexpr int kScanTcThreads = 320;
constexpr int kEpi = 256;  // epilogue threads
// hand-off barrier between the epilogue and the MMA warp (hardware named barrier:
// the 256 epilogue threads and the 32 threads of the MMA warp)
constexpr int kHand = 5, kHandCount = kEpi + 32;
// shared memory map (offsets from a 1024-byte aligned base); 128-byte swizzled
// fp16 tiles are stored as 64-column halves of [64 rows][128 bytes]
constexpr uint32_t ST_QW = 0;        // [Q; W] K-major: half h at h * 16384 (Q rows, then W rows)
constexpr uint32_t ST_K = 32768;     // K rows: half h (d_k columns 64 h ..) at + h * 8192
constexpr uint32_t ST_A = 49152;     // A_qk [64][64]
constexpr uint32_t ST_U = 57344;     // U (fp32) columns c0 .. c0 + 63: two [64][32] boxes
constexpr uint32_t ST_SC = 73728;    // per-chunk factors (kScal floats)
constexpr uint32_t STAGE_BYTES = 75776;
// A stage fills in two parts with their own barriers: [Q; W], read by the first
// products only, and the rest (K, A_qk, U, factors)
constexpr uint32_t TXQ_BYTES = 32768;
constexpr uint32_t TX_BYTES = 16384 + 8192 + 16384 + kScal * 4;
constexpr uint32_t OFF_SB = 2 * STAGE_BYTES;  // state (scaled) fp16, MN-major B: [128][64]
constexpr uint32_t OFF_UT = OFF_SB + 16384;   // U~ fp16 [64][64]
constexpr uint32_t OFF_US = OFF_UT + 8192;    // U~s fp16 [64][64]
constexpr uint32_t OFF_RED = OFF_US + 8192;   // CTA max reduction (8 floats)
constexpr uint32_t OFF_NRM = OFF_RED + 64;    // NORM: row sums of squares [2 chunks][64][2],
                                              // and the peer's [4 chunks][64]
constexpr uint32_t OFF_BAR = OFF_NRM + 2048;  // mbarriers + TMEM address
constexpr uint32_t SCAN_TC_SMEM = OFF_BAR + 128 + 1024;
// NORM only: the previous chunk's output rows before the norm, [64 rows][64] fp32,
// and their gate z, [64 rows][64] bf16 (copied in one chunk ahead).  A warp's lanes
// own consecutive rows, so the rows are padded by 16 bytes: the 16-byte accesses of
// eight lanes then fall in distinct banks.
constexpr int kOS = 64 + 4;  // row stride of the row buffer (floats)
constexpr int kZS = 64 + 8;  // row stride of the gate buffer (bf16)
constexpr uint32_t OFF_OBUF = OFF_BAR + 128;
constexpr uint32_t OFF_ZBUF = OFF_OBUF + 64 * kOS * 4;
constexpr uint32_t OFF_WBUF = OFF_ZBUF + 64 * kZS * 2;  // the CTA's 64 norm weights
constexpr uint32_t SCAN_TC_SMEM_NORM = SCAN_TC_SMEM + 64 * kOS * 4 + 64 * kZS * 2 + 64 * 4;
static_assert(ST_SC + kScal * 4 <= STAGE_BYTES, "stage layout");
static_assert(SCAN_TC_SMEM_NORM <= 227 * 1024, "shared memory of the tcgen05 scan");

// TMEM columns of the accumulators (M = 128, N = 64 each); [O_q; P] alternates
// between two buffers by chunk parity, so that the output rows read O_q of chunk n
// while the products of chunk n + 1 run
constexpr uint32_t TM_QP0 = 0, TM_OA = 64, TM_DS = 128, TM_QP1 = 192, TM_COLS = 256;
__device__ __forceinline__ uint32_t tm_qp(int n) { return (n & 1) ? TM_QP1 : TM_QP0; }

// barrier indices
enum { B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_QP, B_DS, B_OA,
       B_PX0, B_PX1, B_PX2, B_PX3,  // NORM: the peer's row sums of a chunk have arrived
       B_FULLQ0, B_FULLQ1, B_EMPTYQ0, B_EMPTYQ1,  // the [Q; W] part of a stage
       B_COUNT };
static_assert(B_COUNT * 8 + 8 <= 128, "barrier area");

// Byte offset of 16-byte chunk c16 of row r in a 128-byte swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int c16) {
  return (uint32_t)(r * 128 + ((c16 ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack2h(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 32 fp32 values as 16-byte chunks c0 .. c0 + 3 of row r of a 128-byte swizzled fp16 tile.
__device__ __forceinline__ void store_half_row_f16(uint8_t* tile, int r, int c0, const float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 p;
    p.x = pack2h(v[8 * j + 0], v[8 * j + 1]);
    p.y = pack2h(v[8 * j + 2], v[8 * j + 3]);
    p.z = pack2h(v[8 * j + 4], v[8 * j + 5]);
    p.w = pack2h(v[8 * j + 6], v[8 * j + 7]);
    *reinterpret_cast<uint4*>(tile + swz(r, c0 + j)) = p;
  }
}

// Bounded wait that also gives up as soon as another role of the CTA has given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* status,
                                              int where, volatile int* abort_flag,
                                              uint32_t spin) {
  for (uint32_t i = 0; i < spin; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  report_timeout(status, where);
  *abort_flag = 1;
  return false;
}

// Parameters of the gated RMSNorm applied to the output rows (NORM).
struct NormArgs {
  const __nv_bfloat16* z;  // [B, T, Hv, dv]
  const float* w;          // [dv]
  float eps;
};

// 32 output values of one row with 16-byte stores.
template <typename TO>
__device__ __forceinline__ void store_row(TO* dst, const float* v);
template <>
__device__ __forceinline__ void store_row<float>(float* dst, const float* v) {
#pragma unroll
  for (int c = 0; c < 32; c += 4)
    *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
}
template <>
__device__ __forceinline__ void store_row<bf16>(bf16* dst, const float* v) {
#pragma unroll
  for (int c = 0; c < 32; c += 8) {
    uint4 p;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[c], v[c + 1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[c + 2], v[c + 3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[c + 4], v[c + 5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[c + 6], v[c + 7]);
    p.x = *reinterpret_cast<uint32_t*>(&h0);
    p.y = *reinterpret_cast<uint32_t*>(&h1);
    p.z = *reinterpret_cast<uint32_t*>(&h2);
    p.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(dst + c) = p;
  }
}

// 8 output values with one 16-byte store (bf16) or two (float32).
template <typename TO>
__device__ __forceinline__ void store8(TO* dst, const float* v);
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float* v) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store8<bf16>(bf16* dst, const float* v) {
  uint4 p;
  __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
  p.x = *reinterpret_cast<uint32_t*>(&h0);
  p.y = *reinterpret_cast<uint32_t*>(&h1);
  p.z = *reinterpret_cast<uint32_t*>(&h2);
  p.w = *reinterpret_cast<uint32_t*>(&h3);
  *reinterpret_cast<uint4*>(dst) = p;
}

struct ScanMaps {
  CUtensorMap q, w, k, a, u;
};

template <typename TO, bool NORM>
__global__ void __launch_bounds__(kScanTcThreads, 1)
state_scan_tc_kernel(const __grid_constant__ ScanMaps maps, const uint8_t* __restrict__ ws,
                     WsLayout L, const float* h0, int T, int Hk, int Hv, TO* __restrict__ o,
                     float* ht, int* status, int fault, uint32_t spin, NormArgs na,
                     const int4* __restrict__ vtab, int Nv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = 64 * blockIdx.x;
  const int head = blockIdx.y, b = head / Hv, hv = head % Hv, hk = hv / (Hv / Hk);
  // this CTA's sequence: Ts time steps from token tok0 of the o / z rows, Nc chunks
  // from chunk cb of its workspace head wsh (a dense batch row b: b T, all of T,
  // chunk 0 of head (b, hv); a packed batch: sequence b of the table, whose chunks
  // follow those of the sequences before it in one batch row of Nv chunks)
  int Ts = T, Nc = (T + kC - 1) / kC, cb = 0, wsh = head, khead = b * Hk + hk;
  size_t tok0 = (size_t)b * T;
  if (vtab != nullptr) {
    const int4 e = vtab[b];
    cb = e.x;
    Ts = e.y;
    Nc = (Ts + kC - 1) / kC;
    tok0 = (size_t)e.z;
    wsh = hv;
    khead = hk;
  }
  const int Tp = (vtab != nullptr ? Nv : Nc) * kC;  // workspace rows per head
  const float* Sg =
      reinterpret_cast<const float*>(ws + L.scal) + ((size_t)wsh * (Tp / kC) + cb) * kScal;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(&bar[i], (i == B_EMPTY0 || i == B_EMPTY1) ? 2 : 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (NORM)  // each chunk's 64 peer sums arrive as 256 transaction bytes
      for (int i = 0; i < 4; ++i) mbar_arrive_expect_tx(&bar[B_PX0 + i], 64 * 4);
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.w);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the peer's barriers are initialised before anything arrives on them
  if (NORM) cluster_sync();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // The [Q; W] part of chunk n's stage is loaded as soon as the first products
      // of chunk n - 2 have read it, the rest once all of chunk n - 2 is done, so
      // the tiles needed first have about two chunk steps to land.
      int issued_q = 0, issued = 0;  // parts armed so far
      for (int n = 0; n < Nc; ++n) {
        const int s = n & 1;
        if (n >= 2 && !wait_or_abort(&bar[B_EMPTYQ0 + s], ((n >> 1) - 1) & 1, status, 103,
                                     abort_flag, spin)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        uint8_t* st = sm + s * STAGE_BYTES;
        const int rq = khead * Tp + (cb + n) * kC, rw = wsh * Tp + (cb + n) * kC;
        uint64_t* fullq = &bar[B_FULLQ0 + s];
        mbar_arrive_expect_tx(fullq, TXQ_BYTES);
        tma_load_2d(st + ST_QW + 0, &maps.q, fullq, 0, rq);
        tma_load_2d(st + ST_QW + 16384, &maps.q, fullq, 64, rq);
        tma_load_2d(st + ST_QW + 8192, &maps.w, fullq, 0, rw);
        tma_load_2d(st + ST_QW + 24576, &maps.w, fullq, 64, rw);
        issued_q = n + 1;
        if (n >= 2 && !wait_or_abort(&bar[B_EMPTY0 + s], ((n >> 1) - 1) & 1, status, 101,
                                     abort_flag, spin)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        uint64_t* full = &bar[B_FULL0 + s];
        mbar_arrive_expect_tx(full, TX_BYTES);
        tma_load_2d(st + ST_K + 0, &maps.k, full, 0, rq);
        tma_load_2d(st + ST_K + 8192, &maps.k, full, 64, rq);
        tma_load_2d(st + ST_A, &maps.a, full, 0, rw);
        tma_load_2d(st + ST_U + 0, &maps.u, full, c0, rw);
        tma_load_2d(st + ST_U + 8192, &maps.u, full, c0 + 32, rw);
        bulk_load(st + ST_SC, Sg + (size_t)n * kScal, kScal * 4, full);
        issued = n + 1;
      }
      // drain: every part armed must have landed before the CTA may exit.  A part
      // of chunk n was armed only after the same part of chunk n - 2 had been
      // consumed, so only the last two armed of each kind can still be in flight.
      for (int n = (issued_q >= 2 ? issued_q - 2 : 0); n < issued_q; ++n)
        mbar_wait(&bar[B_FULLQ0 + (n & 1)], (n >> 1) & 1, nullptr, 0, 1u << 20);
      for (int n = (issued >= 2 ? issued - 2 : 0); n < issued; ++n)
        mbar_wait(&bar[B_FULL0 + (n & 1)], (n >> 1) & 1, nullptr, 0, 1u << 20);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // The whole warp takes part in the epilogue's hand-off barriers, which also
    // carry the vote on giving up; lane 0 issues the products right after each
    // (completion through tcgen05.commit on an mbarrier; a commit covers all
    // earlier products of the thread).
    const uint32_t id_qw = idesc_f16(128, 64, false, true);
    const uint32_t id_a = idesc_f16(128, 64, false, true);
    const uint32_t id_k = idesc_f16(128, 64, true, true);
    uint32_t qp_phases = 0;  // commits to B_QP so far (lane 0)
    bool quit = named_barrier_or(kHand, kHandCount, false);  // the initial state is stored
    for (int n = 0; n < Nc && !quit; ++n) {
      const int s = n & 1;
      const uint32_t st = sbase + s * STAGE_BYTES;
      bool ok = true;
      // [O_q; P] = [Q; W] S (K = d_k = 128: two 64-column halves of 4 steps), once
      // the stage's [Q; W] part has landed.  (A test of the bounded waits withholds
      // the first products: the epilogue's wait for them then expires and the CTA
      // leaves through the abort path.)
      if (lane == 0 && !(n == 0 && fault == kFaultScanState)) {
        ok = wait_or_abort(&bar[B_FULLQ0 + s], (n >> 1) & 1, status, 102, abort_flag, spin);
        if (ok) {
          tc_fence_after();
          for (int k16 = 0; k16 < 8; ++k16) {
            const uint32_t aoff = (uint32_t)(k16 >> 2) * 16384u + (uint32_t)(k16 & 3) * 32u;
            mma_bf16(tmem + tm_qp(n), sw128_desc(st + ST_QW + aoff, 16, 1024),
                     sw128_desc(sbase + OFF_SB + k16 * 2048, 8192, 1024), id_qw, k16 > 0);
          }
          mma_commit(&bar[B_QP]);
          mma_commit(&bar[B_EMPTYQ0 + s]);  // the stage's [Q; W] part has been read
          ++qp_phases;
        }
      }
      // the rest of the stage (K and A_qk for the next products), waited for while
      // the epilogue forms U~, which needs the same part
      if (lane == 0)
        ok = ok && wait_or_abort(&bar[B_FULL0 + s], (n >> 1) & 1, status, 104, abort_flag, spin);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (named_barrier_or(kHand, kHandCount, !ok)) break;  // U~ and U~s are stored
      // DS = K^T U~s (K = 64 tokens) first: the state update waits for it; then
      // O_a = A_qk U~, which runs while the state is updated
      if (lane == 0) {
        tc_fence_after();
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem + TM_DS, sw128_desc(st + ST_K + k16 * 2048, 8192, 1024),
                   sw128_desc(sbase + OFF_US + k16 * 2048, 8192, 1024), id_k, k16 > 0);
        mma_commit(&bar[B_DS]);
        for (int k16 = 0; k16 < 4; ++k16)
          mma_bf16(tmem + TM_OA, sw128_desc(st + ST_A + k16 * 32, 16, 1024),
                   sw128_desc(sbase + OFF_UT + k16 * 2048, 8192, 1024), id_a, k16 > 0);
        mma_commit(&bar[B_OA]);
        mma_commit(&bar[B_EMPTY0 + s]);  // the stage's operands have been read
      }
      __syncwarp();
      quit = named_barrier_or(kHand, kHandCount, false);  // the new state is stored
    }
    // drain: nothing of ours may still run on the tensor cores at teardown
    if (lane == 0) {
      mma_commit(&bar[B_QP]);
      mbar_wait(&bar[B_QP], qp_phases & 1, nullptr, 0, 1u << 20);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = tid - 64;                       // 0..255
    const int row = 32 * (warp & 3) + lane;       // TMEM lane = d_k row of the state
    const int half = (warp - 2) >> 2;             // columns 32 half .. 32 half + 31
    const int cb = 32 * half;
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)cb;
    const bool p_rows = row >= 64;                // lanes 64-127: rows of P (token row - 64)
    float S[32];
    float mx = 0.f;
    {
      const float* src = h0 ? h0 + ((size_t)head * kD + row) * kD + c0 + cb : nullptr;
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 t = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0, 0, 0, 0);
        S[c] = t.x; S[c + 1] = t.y; S[c + 2] = t.z; S[c + 3] = t.w;
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
      }
    }
    for (int n = e; n < Nc; n += kEpi) mx = fmaxf(mx, Sg[(size_t)n * kScal + kScMaxU]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp - 2] = mx;
    named_barrier(1, kEpi);
    mx = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
    const int ex = mx > 0.f ? min(max(ilogbf(mx) - 7, -100), 100) : 0;
    const float sigma = ldexpf(1.f, -ex), inv_sigma = ldexpf(1.f, ex);
    float range = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      S[c] *= sigma;
      range = fmaxf(range, fabsf(S[c]));
    }
    store_half_row_f16(sm + OFF_SB, row, 4 * half, S);
    fence_proxy_async_smem();
    named_barrier_or(kHand, kHandCount, false);  // to the MMA warp: the state is stored

    // NORM: the rows' sums of squares, this CTA's [2 chunks][64][2] and the peer's
    // [4 chunks][64]; the rows of the previous chunk and their gate z
    float* ssq = reinterpret_cast<float*>(sm + OFF_NRM);
    float* xin = ssq + 256;
    float* obuf = reinterpret_cast<float*>(sm + OFF_OBUF);
    bf16* zbuf = reinterpret_cast<bf16*>(sm + OFF_ZBUF);
    float* wbuf = reinterpret_cast<float*>(sm + OFF_WBUF);
    // the weights once, in shared memory: read from global memory inside the row
    // loop, each load would wait behind the row's own output stores (may alias)
    if (NORM && e < 64) wbuf[e] = na.w[c0 + e];  // first read after a barrier 1
    const uint32_t peer = NORM ? cluster_rank() ^ 1u : 0u;
    // Normalise and store row r of chunk m, columns cbase .. cbase + ncols - 1:
    // y = o / sqrt(mean(o^2) + eps) * w * SiLU(z), the mean over both CTAs' halves.
    // A row's 32 columns of a thread pair go 8 to the output-row thread (TMEM lanes
    // 0-63, barrier 2 among them), which also has the chunk's own rows to take, and
    // 24 to its P-row partner (barrier 3), so the norm's exponentials and divisions
    // spread over all four SM sub-partitions; each group calls this uniformly.  The
    // peer's sums arrive by st.async, whose transaction bytes complete the barrier
    // phase: a CTA-scope wait sees them.
    auto norm_rows = [&](int m, int r, int hf, int cbase, int ncols, int gbar) -> bool {
      const int slot = m & 3;
      const bool got =
          wait_or_abort(&bar[B_PX0 + slot], (m >> 2) & 1, status, 109, abort_flag, spin);
      if (named_barrier_or(gbar, 128, !got)) return false;
      const float* sq = ssq + 128 * (m & 1);
      const float rinv =
          rsqrtf((sq[2 * r] + sq[2 * r + 1] + xin[64 * slot + r]) * (1.f / kD) + na.eps);
      // the slot takes chunk m + 4 next: the peer sends that only after it has the
      // sums of chunk m + 2 from this CTA, which leave after both groups' reads
      if (gbar == 3 && r == 0 && hf == 0 && m + 4 < Nc)
        mbar_arrive_expect_tx(&bar[B_PX0 + slot], 64 * 4);
      const int tm = m * kC + r;
      if (tm < Ts) {
        const float* ob = obuf + r * kOS + cbase;
        const bf16* zr = zbuf + r * kZS + cbase;
        const float* wr = wbuf + cbase;
        TO* dst = o + ((tok0 + tm) * Hv + hv) * kD + c0 + cbase;
#pragma unroll
        for (int c8 = 0; c8 < ncols; c8 += 8) {
          float y[8];
          const uint4 zz = *reinterpret_cast<const uint4*>(zr + c8);
          const float4 wa = *reinterpret_cast<const float4*>(wr + c8);
          const float4 wb = *reinterpret_cast<const float4*>(wr + c8 + 4);
          const float4 oa = *reinterpret_cast<const float4*>(ob + c8);
          const float4 obb = *reinterpret_cast<const float4*>(ob + c8 + 4);
          const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
          const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
          const float ov[8] = {oa.x, oa.y, oa.z, oa.w, obb.x, obb.y, obb.z, obb.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[j]));
            y[2 * j] = ov[2 * j] * rinv * wv[2 * j] * __fdividef(zf.x, 1.f + __expf(-zf.x));
            y[2 * j + 1] =
                ov[2 * j + 1] * rinv * wv[2 * j + 1] * __fdividef(zf.y, 1.f + __expf(-zf.y));
          }
          store8<TO>(dst + c8, y);
        }
      }
      return true;
    };
    for (int n = 0; n < Nc; ++n) {
      const int s = n & 1;
      const uint8_t* st = sm + s * STAGE_BYTES;
      const float* sc = reinterpret_cast<const float*>(st + ST_SC);
      // an expired wait is decided on at the next barrier, by a vote of all epilogue
      // threads (no thread is left at a barrier; what is computed meanwhile is dropped)
      bool ok = wait_or_abort(&bar[B_FULL0 + s], (n >> 1) & 1, status, 105, abort_flag, spin);
      // what does not depend on the products is read before waiting for them: the
      // P-row threads' U row (sigma U) and factor, the output-row threads' factor
      float P[32], fs = 0.f, fo = 0.f;
      if (p_rows) {
        const int r = row - 64;
        fs = sc[kC + r];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {  // U box `half` holds columns cb .. cb + 31
          const float4 u = *reinterpret_cast<const float4*>(st + ST_U + half * 8192 + swz(r, ch));
          P[4 * ch + 0] = sigma * u.x;
          P[4 * ch + 1] = sigma * u.y;
          P[4 * ch + 2] = sigma * u.z;
          P[4 * ch + 3] = sigma * u.w;
        }
      } else {
        fo = sc[row];  // (O_q of the row is read with O_a, in the output step)
      }
      ok = ok && wait_or_abort(&bar[B_QP], n & 1, status, 106, abort_flag, spin);
      tc_fence_after();
      if (p_rows) {
        // U~ = sigma U - P and U~s = U~ fs for token r and this thread's 32 columns,
        // written as fp16 operand rows
        const int r = row - 64;
        {
          float Pm[32];
          tmem_ld32(tl + tm_qp(n), Pm);
#pragma unroll
          for (int c = 0; c < 32; ++c) P[c] -= Pm[c];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float* v = P + 8 * j;
          uint4 pu, ps;
          pu.x = pack2h(v[0], v[1]);
          pu.y = pack2h(v[2], v[3]);
          pu.z = pack2h(v[4], v[5]);
          pu.w = pack2h(v[6], v[7]);
          ps.x = pack2h(v[0] * fs, v[1] * fs);
          ps.y = pack2h(v[2] * fs, v[3] * fs);
          ps.z = pack2h(v[4] * fs, v[5] * fs);
          ps.w = pack2h(v[6] * fs, v[7] * fs);
          const uint32_t off = swz(r, 4 * half + j);
          *reinterpret_cast<uint4*>(sm + OFF_UT + off) = pu;
          *reinterpret_cast<uint4*>(sm + OFF_US + off) = ps;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (named_barrier_or(kHand, kHandCount, !ok || *abort_flag)) {  // to the MMA warp
        *abort_flag = 1;
        break;
      }
      // the fp16 range of U~, taken while the MMA warp issues the products
      if (p_rows) {
#pragma unroll
        for (int c = 0; c < 32; ++c) range = fmaxf(range, fabsf(P[c]));
      }
      // NORM: the gate of the previous chunk's rows has landed before the barrier
      // below, after which the P-row threads read it
      if (NORM && !p_rows) asm volatile("cp.async.wait_all;" ::: "memory");

      // the state update first: it is what the next chunk waits for
      const float gc = sc[kScGC + row];
      ok = wait_or_abort(&bar[B_DS], n & 1, status, 107, abort_flag, spin);
      tc_fence_after();
      {
        float D[32];
        tmem_ld32(tl + TM_DS, D);
#pragma unroll
        for (int c = 0; c < 32; ++c) S[c] = fmaf(gc, S[c], D[c]);
      }
      store_half_row_f16(sm + OFF_SB, row, 4 * half, S);
      fence_proxy_async_smem();
      tc_fence_before();
      if (named_barrier_or(kHand, kHandCount, !ok || *abort_flag)) {  // to the MMA warp
        *abort_flag = 1;
        break;
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) range = fmaxf(range, fabsf(S[c]));
      if (e == 0) mbar_arrive(&bar[B_EMPTY0 + s]);  // U and the factors of the stage are read
      // NORM: the P-row threads normalise and store their part of the previous
      // chunk's output rows, then release the row buffer to the output-row threads
      // (barrier 4: 128 arrive here, 128 wait before overwriting it)
      if (NORM && p_rows && n > 0) {
        if (!norm_rows(n - 1, row - 64, half, cb + 8, 24, 3)) *abort_flag = 1;
        named_barrier_arrive(4, 256);
      }

      // then the output rows (lanes 0-63), overlapping the next chunk's products
      if (!p_rows) {
        bool oa_ok = wait_or_abort(&bar[B_OA], n & 1, status, 108, abort_flag, spin);
        if (NORM) oa_ok = !named_barrier_or(2, 128, !oa_ok);  // the 128 row threads decide as one
        if (!oa_ok) continue;
        tc_fence_after();
        float OQ[32], OA[32];
        tmem_ld32(tl + tm_qp(n), OQ);  // O_q of token row, this thread's 32 columns
        tmem_ld32(tl + TM_OA, OA);
        tc_fence_before();
        const int t = n * kC + row;
#pragma unroll
        for (int c = 0; c < 32; ++c) OA[c] = (fo * OQ[c] + OA[c]) * inv_sigma;
        if (NORM) {
          // this chunk's rows: the sums of squares of the CTA's 64 columns to the
          // peer, the rows themselves to shared memory for the P-row threads
          float ss = 0.f;
#pragma unroll
          for (int c = 0; c < 32; ++c) ss = fmaf(OA[c], OA[c], ss);
          float* sq = ssq + 128 * (n & 1);
          sq[2 * row + half] = ss;
          named_barrier(2, 128);
          if (half == 0) {
            const int slot = n & 3;
            st_async_peer_f32(map_peer(xin + 64 * slot + row, peer), sq[2 * row] + sq[2 * row + 1],
                              map_peer(&bar[B_PX0 + slot], peer));
          }
          if (n > 0) {
            // the rest of the previous chunk's rows, then wait for the P rows
            if (!norm_rows(n - 1, row, half, cb, 8, 2)) *abort_flag = 1;
            named_barrier(4, 256);
          }
          float* ob = obuf + row * kOS + cb;
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(ob + c) = make_float4(OA[c], OA[c + 1], OA[c + 2], OA[c + 3]);
          // the gate of these rows, copied in while the next chunk runs
          if (t < Ts) {
            const bf16* zsrc = na.z + ((tok0 + t) * Hv + hv) * kD + c0 + cb;
            const uint32_t zdst = smem_u32(zbuf + row * kZS + cb);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(zdst + 16 * j),
                           "l"(zsrc + 8 * j)
                           : "memory");
            asm volatile("cp.async.commit_group;" ::: "memory");
          }
        } else if (t < Ts) {
          TO* dst = o + ((tok0 + t) * Hv + hv) * kD + c0 + cb;
          store_row<TO>(dst, OA);
        }
      }
    }
    // NORM: the last chunk's rows, by the P-row threads once the output-row threads'
    // buffers and gate copies are complete (every epilogue thread gets here: the
    // loop's exits are uniform)
    if (NORM && Nc > 0) {
      if (!p_rows) asm volatile("cp.async.wait_all;" ::: "memory");
      const bool aborted = named_barrier_or(1, kEpi, *abort_flag != 0);  // one answer for all
      if (!aborted) {
        if (p_rows)
          norm_rows(Nc - 1, row - 64, half, cb + 8, 24, 3);
        else
          norm_rows(Nc - 1, row, half, cb, 8, 2);
      }
    }
    if (!(range <= kF16Max)) report_range(status);
    if (ht != nullptr && !*abort_flag) {
      float* dst = ht + ((size_t)head * kD + row) * kD + c0 + cb;
#pragma unroll
      for (int c = 0; c < 32; c += 4)
        *reinterpret_cast<float4*>(dst + c) = make_float4(S[c] * inv_sigma, S[c + 1] * inv_sigma,
                                                          S[c + 2] * inv_sigma, S[c + 3] * inv_sigma);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
  // no CTA of the pair leaves while the other may still store into its shared memory
  if (NORM) cluster_sync();
}

// ---------------------------------------------------------------- host side
template <typename TO, bool NORM>
cudaError_t launch_t(const ChunkArgs& a, const WsLayout& L, const uint8_t* ws, int* status,
                     const NormArgs& na, cudaStream_t s) {
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  // a packed batch (a.vtab): a.B sequences in one batch row of a.vNv chunks
  const bool packed = a.vtab != nullptr;
  const uint64_t Tp = packed ? (uint64_t)a.vNv * kC : (uint64_t)((a.T + kC - 1) / kC) * kC;
  const uint64_t rows_b = packed ? 1 : (uint64_t)a.B;
  const uint64_t rv = rows_b * a.Hv * Tp, rk = rows_b * a.Hk * Tp;
  ScanMaps m;
  if (!make_map_rows(&m.q, ws + L.qh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.w, ws + L.w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rv) ||
      !make_map_rows(&m.k, ws + L.kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.a, ws + L.a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kC, rv) ||
      !make_map_rows(&m.u, ws + L.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kD, rv))
    return cudaErrorInvalidValue;
  auto kern = state_scan_tc_kernel<TO, NORM>;
  const uint32_t smem = NORM ? SCAN_TC_SMEM_NORM : SCAN_TC_SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const WaitFault f = wait_fault();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, a.B * a.Hv);
  cfg.blockDim = dim3(kScanTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (NORM) {  // the two column halves of a head form a cluster
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, kern, m, ws, L, a.h0, a.T, a.Hk, a.Hv, static_cast<TO*>(a.o),
                         a.ht, status, f.site, f.spin, na, static_cast<const int4*>(a.vtab),
                         a.vNv);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

__global__ void varlen_table_kernel(const __grid_constant__ VarlenTab tab, int4* dst) {
  for (int i = threadIdx.x; i < tab.n; i += blockDim.x) dst[i] = tab.seq[i];
}

}  // namespace

cudaError_t launch_varlen_table(const VarlenTab& tab, void* dst, cudaStream_t s) {
  varlen_table_kernel<<<1, 256, 0, s>>>(tab, static_cast<int4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_scan_tc(const ChunkArgs& a, const void* ws, int* status, cudaStream_t s) {
  const WsLayout L = a.vtab != nullptr ? ws_layout(1, a.vNv * kC, a.Hk, a.Hv)
                                       : ws_layout(a.B, a.T, a.Hk, a.Hv);
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  const NormArgs na{static_cast<const bf16*>(a.norm_z), a.norm_w, a.norm_eps};
  const bool norm = a.norm_z != nullptr;
  if (a.flags & GDN_OUT_F32)
    return norm ? launch_t<float, true>(a, L, w, status, na, s)
                : launch_t<float, false>(a, L, w, status, na, s);
  return norm ? launch_t<bf16, true>(a, L, w, status, na, s)
              : launch_t<bf16, false>(a, L, w, status, na, s);
}

}  // namespace gdn
