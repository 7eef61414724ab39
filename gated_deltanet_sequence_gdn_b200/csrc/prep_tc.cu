// prep_tc.cu -- chunk-parallel preparation of the bf16 chunkwise GDN forward
// (dk = dv = 128, chunk C = 64) on the tcgen05 tensor cores.
//
// One CTA per (chunk, batch row, key head), two CTAs per SM.  The Gram matrices
// K^ K^^T and Q^ K^^T depend on the key head only (the gates are per value head
// and enter as row / column factors and the decay mask), so the CTA forms the
// raw products [K; Q] K^T once (one M = 128 MMA, accumulator kept in tensor
// memory) and then serves the value heads of its GQA group one after another:
//   L    = strictly lower (beta_r rk_r rk_c e^(G_r - G_c) k_r.k_c)   -> shared fp32
//   A_qk = lower incl. diagonal (sq_r rk_c e^(G_r - G_c) q_r.k_c)   -> workspace fp16
//   X    = (I + L)^-1, blocked, in place
//   W^T  = K^T (X diag(beta e^G rk))^T     M = 128 (d), N = 64 (t), K = 64
//   U^T  = V^T (X diag(beta))^T            the same shape, X diag(beta) split
//                                          into bf16 hi + lo (two passes)
// The products are formed transposed so that an accumulator lane is a column d
// of W / U: the 32 lanes of a warp then store 32 consecutive columns of one row.
// The WY / UT chunk algebra is that of "Gated DeltaNet-2" (section on the
// chunkwise algorithm; GDN is its scalar-decay special case); the outputs are
// the workspace rows the state scan reads (W fp16, U fp32, A_qk fp16, fp16 raw
// q / k rows with their row exponents, and the per-row factors).
//
// Roles: thread 0 issues the TMA loads and stores and the MMAs (tcgen05.mma by
// one thread, completion through tcgen05.commit on an mbarrier); all 8 warps do
// the element work between MMAs; warp w reads TMEM lanes 32 (w % 4) .. + 31, the
// two warps of a lane quarter splitting the columns.  Every mbarrier wait is
// bounded; an expired wait is voted on by the whole CTA, which then drains its
// copies and MMAs in flight, frees its tensor memory and leaves.
#include "chunk_layout.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc_ptx.cuh"
#include "tmap.cuh"
#include "warp_mma.cuh"
#include "wy_common.cuh"

namespace gdn {
namespace {

using namespace wy;
using bf16 = __nv_bfloat16;

constexpr int kPT = 256;  // 8 warps

// shared memory (byte offsets from a 1024-byte aligned base); the tiles are
// 128-byte rows with the 128-byte swizzle (16-byte unit u of row r at u ^ r % 8)
constexpr int S_KQ = 0;             // [2 d-halves][K rows 0-63, Q rows 64-127][128 B]
constexpr int S_V = S_KQ + 32768;   // 2 slots of V: [2 d-halves][64 rows][128 B]
constexpr int S_R = S_V + 32768;    // region, used in turn as:
//   before the first head: fp16 q / k rows to store, [K, Q][2 d-halves][64][128 B]
constexpr int S_XW = S_R;           //   W operand [64 rows][64 columns] bf16 (during the
                                    //   inverse: its block products [4][16][LDB] f32)
constexpr int S_XH = S_R + 8192;    //   U operand, bf16 hi part
constexpr int S_XL = S_R + 16384;   //   U operand, bf16 lo part (before: A_qk to store,
                                    //   [64 rows][128 B] fp16)
constexpr int S_LX = S_R + 24576;   //   L, then X in place: [64][LDX] f32
constexpr int S_VEC = S_LX + kC * LDX * 4;
static_assert(S_VEC >= S_R + 32768, "q / k staging");
static_assert(4 * 16 * LDB * 4 <= 8192, "block products");
// rk, sq, 2^eq, 2^ek [64] (key head); G, beta [4 heads][64]; c1, lc, lk, lq [64]; misc [32]
constexpr int S_BAR = S_VEC + (4 * 64 + 8 * 64 + 4 * 64 + 32) * 4;
constexpr int PT_SMEM = S_BAR + 64 + 1024;  // 4 mbarriers + TMEM address; alignment slack
static_assert(2 * (PT_SMEM + 1024) <= 228 * 1024, "two prep CTAs per SM");

// tensor memory columns (fp32): raw Gram, W^T, U^T of the current head
constexpr uint32_t TM_G = 0, TM_W = 64, TM_U = 128, TM_COLS = 256;

// loads: the bf16 inputs [B][T][H][128]; stores: the workspace row arrays
struct PrepMaps {
  CUtensorMap q, k, v;
  CUtensorMap qh, kh, a;
};

// 16-byte unit j (0..15, columns 8j..8j+7) of row R (0..127) of the K/Q block
__device__ __forceinline__ int kq_off(int R, int j) {
  return ((j >> 3) << 14) + (R << 7) + (((j & 7) ^ (R & 7)) << 4);
}
// byte offset of the 16-byte unit u (0..7) of row t in a [64 rows][128 B] swizzled box
__device__ __forceinline__ int box_off(int t, int u) { return (t << 7) + ((u ^ (t & 7)) << 4); }

// 2^x (the hardware approximation, relative error about 2^-22)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool PRE>
__global__ void __launch_bounds__(kPT, 2)
wy_prep_tc_kernel(const __grid_constant__ PrepMaps maps, const void* __restrict__ ga,
                  const void* __restrict__ gb, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, int T, int Hk, int Hv, float scale, int l2,
                  uint8_t* __restrict__ ws, WsLayout L, int* status, int fault, uint32_t spin,
                  const int4* __restrict__ vtab, int nseq) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (tc::smem_u32(sm_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(sm);
  float* LX = reinterpret_cast<float*>(sm + S_LX);
  float* Tm = reinterpret_cast<float*>(sm + S_XW);
  float* rk = reinterpret_cast<float*>(sm + S_VEC);
  float* sq = rk + 64;
  float* pq = sq + 64;    // 2^e of the stored Q row
  float* pk = pq + 64;    // 2^e of the stored K row
  float* Gs = pk + 64;    // [4][64] in-chunk prefix sums of the log-decays (heads h % 4)
  float* bet = Gs + 256;  // [4][64]
  float* c1 = bet + 256;  // [64] column factor of W: beta e^G rk
  // log2 of the factors of the gated Gram entries: for c <= t,
  //   beta_t rk_t rk_c e^(G_t - G_c) = 2^(lk_t - lc_c),  sq_t rk_c e^(G_t - G_c) = 2^(lq_t - lc_c)
  float* lc = c1 + 64;    // G_c log2 e - log2 rk_c
  float* lk = lc + 64;    // G_t log2 e + log2 (beta_t rk_t)   (-inf for beta_t = 0)
  float* lq = lk + 64;    // G_t log2 e + log2 sq_t
  float* misc = lq + 64;  // [0..3] prefix carries, [8..15] per-warp max |U|
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_BAR);  // K/Q, V slot 0, V slot 1, MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S_BAR + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int G = Hv / Hk;
  const int n = blockIdx.x, Nc = gridDim.x, Tp = Nc * kC;
  const int b = blockIdx.y / Hk, hk = blockIdx.y % Hk;
  // first time step and valid rows of the chunk; the workspace rows of the chunk
  // start at row n * 64 of its head
  int t0 = n * kC, nv = min(kC, T - t0);
  if (vtab != nullptr) {  // packed batch: the sequence whose chunks include chunk n
    int lo = 0, hi = nseq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (vtab[mid].x <= n) lo = mid;
      else hi = mid - 1;
    }
    const int4 e = vtab[lo];
    const int j = n - e.x;
    t0 = e.z + j * kC;
    nv = min(kC, e.y - j * kC);
  }
  const int wrow = n * kC;
  const int q4 = warp & 3, hc = warp >> 2;  // TMEM lane quarter, column half
  const int r = 32 * q4 + lane;             // accumulator lane of this thread
  float range = 0.f;                        // largest magnitude converted to fp16

  // thread 0's record of the copies and MMAs in flight (for the exit after an
  // expired wait)
  uint32_t v_issued[2] = {0, 0}, v_done[2] = {0, 0}, mma_issued = 0, mma_done = 0;
  // (a test of the bounded waits withholds the K / Q tiles: every thread's first wait
  // then expires and the CTA leaves through the drain below)
  const bool kq_issued = fault != kFaultPrepTiles;
  bool kq_done = false;

  auto issue_v = [&](int h) {  // V tile of value head h into slot h % 2 (thread 0)
    const int slot = h & 1;
    tc::mbar_arrive_expect_tx(&bar[1 + slot], 16384);
#pragma unroll
    for (int dh = 0; dh < 2; ++dh)
      tc::tma_load_4d(sm + S_V + slot * 16384 + dh * 8192, &maps.v, &bar[1 + slot], 64 * dh,
                      hk * G + h, t0, b);
    ++v_issued[slot];
  };

  if (tid == 0) {
    tc::prefetch_tmap(&maps.k);
    tc::prefetch_tmap(&maps.q);
    tc::prefetch_tmap(&maps.v);
    for (int i = 0; i < 4; ++i) tc::mbar_init(&bar[i], 1);
    tc::fence_mbar_init();
    if (kq_issued) {
      tc::mbar_arrive_expect_tx(&bar[0], 32768);
#pragma unroll
      for (int dh = 0; dh < 2; ++dh) {
        tc::tma_load_4d(sm + S_KQ + dh * 16384, &maps.k, &bar[0], 64 * dh, hk, t0, b);
        tc::tma_load_4d(sm + S_KQ + dh * 16384 + 8192, &maps.q, &bar[0], 64 * dh, hk, t0, b);
      }
    }
    issue_v(0);
    if (G > 1) issue_v(1);
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, TM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);  // this warp's lane quarter

  // Leave after an expired wait (the decision is the same in every thread):
  // let the copies and MMAs in flight finish, free the tensor memory.
  auto drain_and_leave = [&]() {
    if (tid == 0) {
      if (kq_issued && !kq_done) tc::mbar_wait(&bar[0], 0, nullptr, 0, 1u << 20);
      for (int s = 0; s < 2; ++s)
        if (v_issued[s] > v_done[s]) tc::mbar_wait(&bar[1 + s], v_done[s] & 1, nullptr, 0, 1u << 20);
      if (mma_issued > mma_done) tc::mbar_wait(&bar[3], mma_done & 1, nullptr, 0, 1u << 20);
      tc::bulk_wait_all();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc::tc_fence_after();
      tc::tmem_dealloc(tmem, TM_COLS);
    }
  };

  // gates of value heads h0 .. h0 + 3 (thread: head h0 + tid / 64, row tid % 64),
  // zero past the end of the sequence and past the last head; in-chunk prefix
  // sums without the carry of the first 32 rows
  auto gates_partial = [&](int h0) {
    const int j = tid >> 6, t = tid & 63, h = h0 + j;
    float g = 0.f, be = 0.f;
    if (h < G && t < nv) {
      const int hv = hk * G + h;
      const size_t idx = ((size_t)b * T + t0 + t) * Hv + hv;
      if (PRE) {
        g = reinterpret_cast<const float*>(ga)[idx];
        be = reinterpret_cast<const float*>(gb)[idx];
      } else {
        g = gdn_log_decay(__bfloat162float(reinterpret_cast<const bf16*>(ga)[idx]), A_log[hv],
                          dt_bias[hv]);
        be = sigmoid_f(__bfloat162float(reinterpret_cast<const bf16*>(gb)[idx]));
      }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, g, off);
      if (lane >= off) g += y;
    }
    if (t == 31) misc[j] = g;
    Gs[tid] = g;
    bet[tid] = be;
  };
  auto gates_carry = [&]() {
    if ((tid & 63) >= 32) Gs[tid] += misc[tid >> 6];
  };
  // column factor of W and the log2 factors of value head h (after the carry and the norms)
  auto head_factors = [&](int h) {
    if (tid < kC) {
      const int j = 64 * (h & 3) + tid;
      const float g2 = Gs[j] * 1.4426950408889634f;
      c1[tid] = bet[j] * __expf(Gs[j]) * rk[tid];
      lc[tid] = g2 - __log2f(rk[tid]);
      lk[tid] = g2 + __log2f(bet[j] * rk[tid]);
      lq[tid] = g2 + __log2f(sq[tid]);
    }
  };

  // 1. gates of the first heads while the tiles land
  gates_partial(0);
  bool ok = tc::mbar_wait(&bar[0], 0, status, 121, spin);
  if (__syncthreads_or(!ok)) {
    drain_and_leave();
    return;
  }
  if (tid == 0) kq_done = true;

  // 2. raw Gram [K; Q] K^T (M = 128, N = 64, K = 128) while the norms run
  if (tid == 0) {
    tc::tc_fence_after();
#pragma unroll
    for (int k16 = 0; k16 < 8; ++k16) {
      const uint32_t off = sb + S_KQ + (k16 >> 2) * 16384 + (k16 & 3) * 32;
      tc::mma_bf16(tmem + TM_G, tc::sw128_desc(off, 16, 1024), tc::sw128_desc(off, 16, 1024),
                   tc::idesc_bf16(128, 64, false, false), k16 > 0);
    }
    tc::mma_commit(&bar[3]);
    ++mma_issued;
  }
  gates_carry();

  //    L2 norms: rk = 1 / |k|, sq = scale / |q|, the row exponents and the fp16
  //    copies of the raw rows (two threads per row, thread h on column half h;
  //    its m-th read is unit m ^ 4h of the half, so the 8 lanes of one 16-byte
  //    shared-memory phase touch 8 distinct bank groups)
  {
    const int which = tid >> 7, rr = (tid & 127) >> 1, h = tid & 1;
    const int R = 64 * which + rr;
    float ss = 0.f, mx = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const uint4 u = *reinterpret_cast<const uint4*>(sm + S_KQ + kq_off(R, 8 * h + (m ^ (4 * h))));
      const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
      ss += f0.x * f0.x + f0.y * f0.y + f1.x * f1.x + f1.y * f1.y + f2.x * f2.x + f2.y * f2.y +
            f3.x * f3.x + f3.y * f3.y;
      mx = fmaxf(mx, fmaxf(fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))),
                           fmaxf(fmaxf(fabsf(f2.x), fabsf(f2.y)), fmaxf(fabsf(f3.x), fabsf(f3.y)))));
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    const int e = row_exponent(mx);
    const float up = ldexpf(1.f, e), down = ldexpf(1.f, -e);  // exact powers of 2
    if (h == 0) {
      const float inv = l2 ? rsqrtf(ss + 1e-6f) : 1.f;
      if (which) {
        sq[rr] = inv * scale;
        pq[rr] = up;
      } else {
        rk[rr] = inv;
        pk[rr] = up;
      }
    }
    uint8_t* st = sm + S_R + which * 16384 + h * 8192;  // [K, Q][d-half][64][128 B]
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u8 = m ^ (4 * h);
      const uint4 u = *reinterpret_cast<const uint4*>(sm + S_KQ + kq_off(R, 8 * h + u8));
      const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
      uint4 o;
      o.x = pack2h(f0.x * down, f0.y * down);
      o.y = pack2h(f1.x * down, f1.y * down);
      o.z = pack2h(f2.x * down, f2.y * down);
      o.w = pack2h(f3.x * down, f3.y * down);
      *reinterpret_cast<uint4*>(st + box_off(rr, u8)) = o;
    }
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    const int row = blockIdx.y * Tp + wrow;
#pragma unroll
    for (int dh = 0; dh < 2; ++dh) {
      tc::tma_store_2d(&maps.kh, sm + S_R + dh * 8192, 64 * dh, row);
      tc::tma_store_2d(&maps.qh, sm + S_R + 16384 + dh * 8192, 64 * dh, row);
    }
    tc::bulk_commit();
  }
  ok = tc::mbar_wait(&bar[3], 0, status, 122, spin);
  if (__syncthreads_or(!ok)) {
    drain_and_leave();
    return;
  }
  if (tid == 0) ++mma_done;
  tc::tc_fence_after();

  for (int h = 0; h < G; ++h) {
    const size_t head = (size_t)b * Hv + hk * G + h;
    const int row0 = (int)(head * Tp) + wrow;  // first workspace row of this chunk and head
    if (h > 0 && (h & 3) == 0) {             // gates of the next four heads
      __syncthreads();
      gates_partial(h);
      __syncthreads();
      gates_carry();
      __syncthreads();
    }
    // the region's previous contents (the staged q / k rows or A_qk) must have
    // been read before it is written again
    if (tid == 0) tc::bulk_wait_read_all();
    head_factors(h);
    __syncthreads();

    // 3. L (shared) and A_qk (staged for a tensor store) from the raw Gram row
    //    of this thread (lane r: K rows 0-63, Q rows 64-127; columns 32 hc ..);
    //    the masked entries are selected away (their exponent may be large)
    {
      float gv[32];
      tc::tmem_ld32(tq + TM_G + 32 * hc, gv);
      const float* lch = lc + 32 * hc;
      if (r < kC) {
        const int t = r;
        const float lt = lk[t];
        float* dst = LX + t * LDX + 32 * hc;
#pragma unroll
        for (int c4 = 0; c4 < 32; c4 += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lch + c4);
          const float e[4] = {ex2_approx(lt - l4.x), ex2_approx(lt - l4.y), ex2_approx(lt - l4.z),
                              ex2_approx(lt - l4.w)};
          float v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = 32 * hc + c4 + i < t ? e[i] * gv[c4 + i] : 0.f;
          *reinterpret_cast<float4*>(dst + c4) = make_float4(v[0], v[1], v[2], v[3]);
        }
      } else {
        const int t = r - kC;
        const float lt = lq[t];
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) {
          const float4 la = *reinterpret_cast<const float4*>(lch + c8);
          const float4 lb = *reinterpret_cast<const float4*>(lch + c8 + 4);
          const float l8[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float e = ex2_approx(lt - l8[i]);
            v[i] = 32 * hc + c8 + i <= t ? e * gv[c8 + i] : 0.f;
            range = fmaxf(range, fabsf(v[i]));
          }
          uint4 o;
          o.x = pack2h(v[0], v[1]);
          o.y = pack2h(v[2], v[3]);
          o.z = pack2h(v[4], v[5]);
          o.w = pack2h(v[6], v[7]);
          *reinterpret_cast<uint4*>(sm + S_XL + box_off(t, 4 * hc + (c8 >> 3))) = o;
        }
      }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc::tma_store_2d(&maps.a, sm + S_XL, 0, row0);
      tc::bulk_commit();
    }

    // 4. X = (I + L)^-1 (block products in the W operand's space)
    invert_in_place(LX, Tm, tid, warp, g8, t4);
    bool vok = true;
    if (tid == 0) {
      vok = tc::mbar_wait(&bar[1 + (h & 1)], (h >> 1) & 1, status, 123, spin);
      if (vok) ++v_done[h & 1];
      tc::bulk_wait_read_all();  // the staged A_qk tile is read (the lo operand goes there)
    }
    __syncthreads();

    // 5. MMA operands (bf16, 128-byte swizzled rows of 64 columns): X diag(c1)
    //    and X diag(beta) = hi + lo
    for (int i = tid; i < kC * 8; i += kPT) {
      const int t = i >> 3, ch = i & 7;
      const float* xr = LX + t * LDX + 8 * ch;
      const float4 a0 = *reinterpret_cast<const float4*>(xr);
      const float4 a1 = *reinterpret_cast<const float4*>(xr + 4);
      const float x[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float* bh = bet + 64 * (h & 3);
      uint32_t pw[4], ph[4], pl[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 8 * ch + 2 * e;
        pw[e] = pack2(x[2 * e] * c1[c], x[2 * e + 1] * c1[c + 1]);
        split2(x[2 * e] * bh[c], x[2 * e + 1] * bh[c + 1], ph[e], pl[e]);
      }
      const int off = box_off(t, ch);
      *reinterpret_cast<uint4*>(sm + S_XW + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      *reinterpret_cast<uint4*>(sm + S_XH + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(sm + S_XL + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
    tc::fence_proxy_async_smem();  // generic-proxy writes -> the MMA's reads
    tc::tc_fence_before();
    if (__syncthreads_or(!vok)) {
      drain_and_leave();
      return;
    }

    // 6. W^T = K^T X'^T and U^T = V^T X"^T (M = 128 d, N = 64 t, K = 64 t'): the
    //    K and V tiles are read MN-major (d contiguous), the operands K-major
    if (tid == 0) {
      tc::tc_fence_after();
      const uint32_t vs = sb + S_V + (h & 1) * 16384;
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16)
        tc::mma_bf16(tmem + TM_W, tc::sw128_desc(sb + S_KQ + k16 * 2048, 16384, 1024),
                     tc::sw128_desc(sb + S_XW + k16 * 32, 16, 1024),
                     tc::idesc_bf16(128, 64, true, false), k16 > 0);
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16)
        tc::mma_bf16(tmem + TM_U, tc::sw128_desc(vs + (k16 & 3) * 2048, 8192, 1024),
                     tc::sw128_desc(sb + (k16 < 4 ? S_XH : S_XL) + (k16 & 3) * 32, 16, 1024),
                     tc::idesc_bf16(128, 64, true, false), k16 > 0);
      tc::mma_commit(&bar[3]);
      ++mma_issued;
    }
    ok = tc::mbar_wait(&bar[3], (uint32_t)(h + 1) & 1u, status, 124, spin);
    if (__syncthreads_or(!ok)) {
      drain_and_leave();
      return;
    }
    tc::tc_fence_after();
    if (tid == 0) {
      ++mma_done;
      if (h + 2 < G) issue_v(h + 2);  // the MMA reads of this slot are complete
    }

    // 7. W (fp16) and U (fp32) to the workspace: lane r is column d = r, this
    //    warp's columns of the accumulators are time steps 32 hc .. 32 hc + 31
    float umax = 0.f;
    {
      __half* dw = reinterpret_cast<__half*>(ws + L.w) + ((size_t)row0 + 32 * hc) * kD + r;
      float* du = reinterpret_cast<float*>(ws + L.u) + ((size_t)row0 + 32 * hc) * kD + r;
      float v[32];
      tc::tmem_ld32(tq + TM_W + 32 * hc, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        range = fmaxf(range, fabsf(v[j]));
        dw[j * kD] = __float2half_rn(v[j]);
      }
      tc::tmem_ld32(tq + TM_U + 32 * hc, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        umax = fmaxf(umax, fabsf(v[j]));
        du[j * kD] = v[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, o));
    if (lane == 0) misc[8 + warp] = umax;
    tc::tc_fence_before();
    __syncthreads();

    // 8. per-row factors of the scan: fo = gamma sq 2^eq, fs = rk 2^ek gamma_C / gamma,
    //    gamma_C for every state row, max |U|
    if (tid < 128) {
      const float* Gh = Gs + 64 * (h & 3);
      float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
      const float GC = Gh[kC - 1];
      if (tid < kC) {
        const float Gt = Gh[tid];
        sc[tid] = __expf(Gt) * sq[tid] * pq[tid];
        sc[kC + tid] = tid < nv ? rk[tid] * pk[tid] * __expf(GC - Gt) : 0.f;
      }
      sc[kScGC + tid] = __expf(GC);
      if (tid < 4) {
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) m = fmaxf(m, misc[8 + w]);
        sc[kScMaxU + tid] = tid == 0 ? m : 0.f;
      }
    }
  }
  if (!(range <= kF16Max)) report_range(status);

  if (tid == 0) tc::bulk_wait_all();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

cudaError_t launch_prep_tc(const ChunkArgs& a, void* ws, int* status, cudaStream_t s) {
  // a packed batch (a.vtab) is one batch row of a.T tokens cut into a.vNv chunks
  const bool packed = a.vtab != nullptr;
  const int B = packed ? 1 : a.B;
  const int Nc = packed ? a.vNv : (a.T + kC - 1) / kC;
  const WsLayout L = ws_layout(B, Nc * kC, a.Hk, a.Hv);
  const uint64_t Tp = (uint64_t)Nc * kC;
  const uint64_t rv = (uint64_t)B * a.Hv * Tp, rk = (uint64_t)B * a.Hk * Tp;
  uint8_t* w = static_cast<uint8_t*>(ws);
  PrepMaps m;
  if (!make_map_bthd(&m.q, a.q, B, a.T, a.Hk) || !make_map_bthd(&m.k, a.k, B, a.T, a.Hk) ||
      !make_map_bthd(&m.v, a.v, B, a.T, a.Hv) ||
      !make_map_rows(&m.qh, w + L.qh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.kh, w + L.kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.a, w + L.a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kC, rv))
    return cudaErrorInvalidValue;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  const int l2 = (a.flags & GDN_QK_L2NORM) ? 1 : 0;
  auto prep = pre ? wy_prep_tc_kernel<true> : wy_prep_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, PT_SMEM);
  if (e != cudaSuccess) return e;
  const WaitFault f = wait_fault();
  prep<<<dim3(Nc, B * a.Hk), kPT, PT_SMEM, s>>>(m, a.a, a.b, a.A_log, a.dt_bias, a.T, a.Hk,
                                                a.Hv, a.scale, l2, w, L, status, f.site, f.spin,
                                                static_cast<const int4*>(a.vtab), a.B);
  return cudaGetLastError();
}

}  // namespace gdn
