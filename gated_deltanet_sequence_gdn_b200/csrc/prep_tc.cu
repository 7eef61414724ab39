// prep_tc.cu -- chunk-parallel preparation of the bf16 chunkwise GDN forward
// (dk = dv = 128, chunk C = 64) on the tcgen05 tensor cores.
//
// One CTA per (chunk, batch row, key head).  The Gram matrices K^ K^^T and
// Q^ K^^T depend on the key head only (the gates are per value head and enter
// as row / column factors and the decay mask), so the CTA forms the raw products
// [K; Q] K^T once (one M = 128 MMA, accumulator in tensor memory) and then
// serves every value head of its GQA group, two at a time:
//   L   = strictly lower (beta_r rk_r rk_c e^(G_r - G_c) k_r.k_c)   -> shared fp32
//   A_qk = lower incl. diagonal (sq_r rk_c e^(G_r - G_c) q_r.k_c)   -> workspace fp16
//   X   = (I + L)^-1, in place, by both heads at once (four warps each)
//   W   = X diag(beta e^G rk) K      one M = 128 MMA for the pair (shared B = K)
//   U   = X diag(beta) V             one M = 128, N = 256 MMA for the pair, the
//         A operand split into bf16 hi + lo (two passes), B = [V_h0 | V_h1]; of the
//         128 x 256 result only the two diagonal 64 x 128 blocks are read.
// The WY / UT chunk algebra is that of "Gated DeltaNet-2" (section on the
// chunkwise algorithm; GDN is its scalar-decay special case); the outputs are
// the workspace rows the state scan reads (W fp16, U fp32, A_qk fp16, fp16 raw
// q / k rows with their row exponents, and the per-row factors).
//
// Every workspace tile leaves through shared memory and a TMA tensor store (the
// accumulator layout gives each thread one row, so direct stores would touch a
// separate line per lane).
//
// Roles: thread 0 issues the TMA loads and stores and the MMAs (tcgen05.mma by one thread,
// completion through tcgen05.commit on an mbarrier); all 8 warps do the element
// work between MMAs; warp w reads TMEM lanes 32 (w % 4) .. + 31, the two warps
// of a lane quarter splitting the columns.  Every mbarrier wait is bounded; an
// expired wait is voted on by the whole CTA, which then drains its copies and
// MMAs in flight, frees its tensor memory and leaves.
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
constexpr int S_V = S_KQ + 32768;   // V of the pair: [2 heads][2 d-halves][64 rows][128 B]
constexpr int S_R = S_V + 32768;    // 96 KB region, used in turn as:
//   before the first pair: fp16 q / k rows to store, [K, Q][2 d-halves][64][128 B]
constexpr int S_XW = S_R;           //   MMA operands: W operand [2 heads x 64 rows][64] bf16
constexpr int S_XH = S_R + 16384;   //     U operand, bf16 hi part
constexpr int S_XL = S_R + 32768;   //     U operand, bf16 lo part (before: A_qk to store,
                                    //     [2 heads][64 rows][128 B] fp16)
constexpr int S_LX = S_R + 49152;   //   L, then X in place: [2 heads][64][LDX] f32
constexpr int S_T = S_LX + 2 * kC * LDX * 4;  // block products [2 heads][3][16][LDB] f32
constexpr int S_SW = S_R;           //   after the MMAs: W to store [2 heads][2 d-halves][64][128 B]
constexpr int S_SU = S_R + 32768;   //     U to store [2 heads][4 d-quarters][64][128 B] fp32
constexpr int S_VEC = S_R + 98304;
static_assert(S_T + 2 * 3 * 16 * LDB * 4 <= S_VEC, "region");
// rk, sq, 2^eq, 2^ek [64] (key head); G, beta, c1, hc, hk, hq [2 heads][64]; misc [32]
constexpr int S_BAR = S_VEC + (4 * 64 + 12 * 64 + 32) * 4;
constexpr int PT_SMEM = S_BAR + 64 + 1024;  // 3 mbarriers + TMEM address; alignment slack
static_assert(PT_SMEM <= 227 * 1024, "prep shared memory");

// 2^x (the hardware approximation, relative error about 2^-22)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of the 16-byte unit u (0..7) of row t in a [64 rows][128 B] swizzled box
__device__ __forceinline__ int box_off(int t, int u) { return (t << 7) + ((u ^ (t & 7)) << 4); }

// tensor memory columns (fp32): raw Gram, W of the pair, U of the pair
constexpr uint32_t TM_G = 0, TM_W = 128, TM_U = 256, TM_COLS = 512;

// loads: the bf16 inputs [B][T][H][128]; stores: the workspace row arrays
struct PrepMaps {
  CUtensorMap q, k, v;
  CUtensorMap qh, kh, w, a, u;
};

// 16-byte unit j (0..15, columns 8j..8j+7) of row R (0..127) of the K/Q block
__device__ __forceinline__ int kq_off(int R, int j) {
  return ((j >> 3) << 14) + (R << 7) + (((j & 7) ^ (R & 7)) << 4);
}

// X = (I + L)^-1 in place for a strictly lower 64 x 64 fp32 L (row stride LDX,
// zero upper triangle), by the 128 threads of one named barrier: the four
// 16 x 16 diagonal blocks by forward substitution (thread = one column of one
// block), then block row by block row on the warp tensor cores with the fp32
// operands as bf16 hi + lo: warp j < i forms T = sum_{k=j}^{i-1} L_ik X_kj and
// X_ij = -X_ii T.  Each write waits at the barrier until every read of the L
// block it replaces is done.
__device__ void invert_in_place(float* M, float* Tm, int lt, int lw, int g8, int t4, int bar_id) {
  float x[16];
  const int base = 16 * (lt >> 4), cc = lt & 15;
  if (lt < kC) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float s = 0.f;
#pragma unroll
      for (int jj = 0; jj < r; ++jj) s = fmaf(M[(base + r) * LDX + base + jj], x[jj], s);
      x[r] = r == cc ? 1.f : -s;  // rows above cc come out as zero
    }
  }
  tc::named_barrier(bar_id, 128);
  if (lt < kC) {
#pragma unroll
    for (int r = 0; r < 16; ++r) M[(base + r) * LDX + base + cc] = x[r];
  }
  tc::named_barrier(bar_id, 128);
  for (int bi = 1; bi < 4; ++bi) {
    const int bj = lw;
    float* Tw = Tm + lw * 16 * LDB;
    if (lw < bi) {
      float t[2][4] = {};
      for (int kb = bj; kb < bi; ++kb) {
        uint32_t ah[4], al[4];
        frag_a_split(M, LDX, 16 * bi, 16 * kb, g8, t4, ah, al);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t bh[2], bl[2];
          frag_b_split(M, LDX, 16 * kb, 16 * bj + 8 * nt, g8, t4, bh, bl);
          mma_split3(t[nt], ah, al, bh, bl);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(Tw + g8 * LDB + 8 * nt + 2 * t4) = make_float2(t[nt][0], t[nt][1]);
        *reinterpret_cast<float2*>(Tw + (g8 + 8) * LDB + 8 * nt + 2 * t4) =
            make_float2(t[nt][2], t[nt][3]);
      }
    }
    tc::named_barrier(bar_id, 128);  // block row bi of L is read; T is visible
    if (lw < bi) {
      float xo[2][4] = {};
      uint32_t ah[4], al[4];
      frag_a_split(M, LDX, 16 * bi, 16 * bi, g8, t4, ah, al);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bh[2], bl[2];
        frag_b_split(Tw, LDB, 0, 8 * nt, g8, t4, bh, bl);
        mma_split3(xo[nt], ah, al, bh, bl);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int c = 16 * bj + 8 * nt + 2 * t4;
        *reinterpret_cast<float2*>(M + (16 * bi + g8) * LDX + c) = make_float2(-xo[nt][0], -xo[nt][1]);
        *reinterpret_cast<float2*>(M + (16 * bi + g8 + 8) * LDX + c) =
            make_float2(-xo[nt][2], -xo[nt][3]);
      }
    }
    tc::named_barrier(bar_id, 128);
  }
}

template <bool PRE>
__global__ void __launch_bounds__(kPT, 1)
wy_prep_tc_kernel(const __grid_constant__ PrepMaps maps, const void* __restrict__ ga,
                  const void* __restrict__ gb, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, int T, int Hk, int Hv, float scale, int l2,
                  uint8_t* __restrict__ ws, WsLayout L, int* status) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (tc::smem_u32(sm_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(sm);
  float* LX = reinterpret_cast<float*>(sm + S_LX);
  float* Tm = reinterpret_cast<float*>(sm + S_T);
  float* rk = reinterpret_cast<float*>(sm + S_VEC);
  float* sq = rk + 64;
  float* pq = sq + 64;    // 2^e of the stored Q row
  float* pk = pq + 64;    // 2^e of the stored K row
  float* Gs = pk + 64;    // [2][64] in-chunk prefix sums of the log-decays
  float* bet = Gs + 128;  // [2][64]
  float* c1 = bet + 128;  // [2][64] column factor of W: beta e^G rk
  // log2 of the factors of the gated Gram entries (per head): for c <= t,
  //   beta_t rk_t rk_c e^(G_t - G_c) = 2^(lk_t - lc_c),  sq_t rk_c e^(G_t - G_c) = 2^(lq_t - lc_c)
  float* lc = c1 + 128;   // [2][64] G_c log2 e - log2 rk_c
  float* lk = lc + 128;   // [2][64] G_t log2 e + log2 (beta_t rk_t)   (-inf for beta_t = 0)
  float* lq = lk + 128;   // [2][64] G_t log2 e + log2 sq_t
  float* misc = lq + 128; // [0..1] prefix carries, [8..15] per-warp max |U|
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S_BAR);  // K/Q, V, MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S_BAR + 24);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int G = Hv / Hk, npairs = (G + 1) >> 1;
  const int n = blockIdx.x, Nc = gridDim.x, Tp = Nc * kC;
  const int b = blockIdx.y / Hk, hk = blockIdx.y % Hk;
  const int t0 = n * kC, nv = min(kC, T - t0);
  const int q4 = warp & 3, hc = warp >> 2;  // TMEM lane quarter, column half
  const int r = 32 * q4 + lane;             // accumulator row of this thread
  float range = 0.f;                        // largest magnitude converted to fp16

  // thread 0's record of the copies and MMAs in flight (for the exit after an
  // expired wait)
  uint32_t v_issued = 0, v_done = 0, mma_issued = 0, mma_done = 0;
  bool kq_done = false;

  auto issue_v = [&](int p) {  // V tiles of pair p (thread 0)
    const int nh = min(2, G - 2 * p);
    tc::mbar_arrive_expect_tx(&bar[1], nh * 16384);
    for (int hs = 0; hs < nh; ++hs)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        tc::tma_load_4d(sm + S_V + hs * 16384 + h * 8192, &maps.v, &bar[1], 64 * h,
                        hk * G + 2 * p + hs, t0, b);
    ++v_issued;
  };

  if (tid == 0) {
    tc::prefetch_tmap(&maps.k);
    tc::prefetch_tmap(&maps.q);
    tc::prefetch_tmap(&maps.v);
    for (int i = 0; i < 3; ++i) tc::mbar_init(&bar[i], 1);
    tc::fence_mbar_init();
    tc::mbar_arrive_expect_tx(&bar[0], 32768);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tc::tma_load_4d(sm + S_KQ + h * 16384, &maps.k, &bar[0], 64 * h, hk, t0, b);
      tc::tma_load_4d(sm + S_KQ + h * 16384 + 8192, &maps.q, &bar[0], 64 * h, hk, t0, b);
    }
    issue_v(0);
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
      if (!kq_done) tc::mbar_wait(&bar[0], 0, nullptr, 0, 1u << 20);
      if (v_issued > v_done) tc::mbar_wait(&bar[1], v_done & 1, nullptr, 0, 1u << 20);
      if (mma_issued > mma_done) tc::mbar_wait(&bar[2], mma_done & 1, nullptr, 0, 1u << 20);
      tc::bulk_wait_all();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc::tc_fence_after();
      tc::tmem_dealloc(tmem, TM_COLS);
    }
  };

  // gates of pair p (threads 0-127: head slot tid / 64, row tid % 64), zero past
  // the end of the sequence and for a missing second head; in-chunk prefix sums
  // without the carry of the first 32 rows
  auto gates_partial = [&](int p) {
    if (tid < 128) {
      const int hs = tid >> 6, t = tid & 63, j = 2 * p + hs;
      float g = 0.f, be = 0.f;
      if (j < G && t < nv) {
        const int hv = hk * G + j;
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
      if (t == 31) misc[hs] = g;
      Gs[tid] = g;
      bet[tid] = be;
    }
  };
  auto gates_carry = [&]() {
    if (tid < 128 && (tid & 63) >= 32) Gs[tid] += misc[tid >> 6];
  };
  // column factor of W and the log2 factors of the pair (after the carry and the norms)
  auto factors_pair = [&]() {
    if (tid < 128) {
      const int t = tid & 63;
      const float g2 = Gs[tid] * 1.4426950408889634f;
      c1[tid] = bet[tid] * __expf(Gs[tid]) * rk[t];
      lc[tid] = g2 - __log2f(rk[t]);
      lk[tid] = g2 + __log2f(bet[tid] * rk[t]);
      lq[tid] = g2 + __log2f(sq[t]);
    }
  };

  // 1. gates of the first pair while the tiles land
  gates_partial(0);
  bool ok = tc::mbar_wait(&bar[0], 0, status, 121);
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
    tc::mma_commit(&bar[2]);
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
    const int row = blockIdx.y * Tp + t0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tc::tma_store_2d(&maps.kh, sm + S_R + h * 8192, 64 * h, row);
      tc::tma_store_2d(&maps.qh, sm + S_R + 16384 + h * 8192, 64 * h, row);
    }
    tc::bulk_commit();
  }

  factors_pair();

  // 3. the raw Gram row of this thread: 32 columns (32 hc ..) of row r (K rows
  //    0-63, Q rows 64-127), kept in registers for every value head
  ok = tc::mbar_wait(&bar[2], 0, status, 122);
  if (__syncthreads_or(!ok)) {
    drain_and_leave();
    return;
  }
  if (tid == 0) ++mma_done;
  tc::tc_fence_after();
  float gv[32];
  tc::tmem_ld32(tq + TM_G + 32 * hc, gv);

  for (int p = 0; p < npairs; ++p) {
    const int nh = min(2, G - 2 * p);
    const int hv0 = hk * G + 2 * p;
    // the region's previous contents (stores of the last pair, or the q / k
    // rows) must have been read before it is written again
    if (tid == 0) tc::bulk_wait_read_all();
    if (p > 0) {
      gates_partial(p);
      __syncthreads();
      gates_carry();
      __syncthreads();
      factors_pair();
    }
    __syncthreads();

    // 4. L (shared) and A_qk (staged for a tensor store) of both heads; the
    //    masked entries are selected away (their exponent may be large)
    for (int hs = 0; hs < nh; ++hs) {
      const float* lch = lc + 64 * hs + 32 * hc;
      if (r < kC) {
        const int t = r;
        const float lt = lk[64 * hs + t];
        float* dst = LX + hs * kC * LDX + t * LDX + 32 * hc;
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
        const float lt = lq[64 * hs + t];
        uint8_t* st = sm + S_XL + hs * 8192;
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
          *reinterpret_cast<uint4*>(st + box_off(t, 4 * hc + (c8 >> 3))) = o;
        }
      }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      for (int hs = 0; hs < nh; ++hs)
        tc::tma_store_2d(&maps.a, sm + S_XL + hs * 8192, 0, ((b * Hv + hv0 + hs) * Tp + t0));
      tc::bulk_commit();
    }

    // 5. X = (I + L)^-1 of both heads at once: warps 4 hs .. 4 hs + 3 on head hs
    {
      const int hs = warp >> 2;
      if (hs < nh)
        invert_in_place(LX + hs * kC * LDX, Tm + hs * 3 * 16 * LDB, tid & 127, warp & 3, g8, t4,
                        1 + hs);
    }
    bool vok = true;
    if (tid == 0) {
      vok = tc::mbar_wait(&bar[1], p & 1, status, 123);
      if (vok) ++v_done;
      tc::bulk_wait_read_all();  // the staged A_qk tiles are read (the lo operand goes there)
    }
    __syncthreads();

    // 6. MMA operands (bf16, 128-byte swizzled rows of 64 columns): X diag(c1)
    //    and X diag(beta) = hi + lo; rows of a missing second head are zero
    for (int i = tid; i < 2 * kC * 8; i += kPT) {
      const int hs = i >> 9, t = (i >> 3) & 63, ch = i & 7;
      const int R = 64 * hs + t;
      uint4 w = make_uint4(0, 0, 0, 0), hi = w, lo = w;
      if (hs < nh) {
        const float* xr = LX + hs * kC * LDX + t * LDX + 8 * ch;
        const float4 a0 = *reinterpret_cast<const float4*>(xr);
        const float4 a1 = *reinterpret_cast<const float4*>(xr + 4);
        const float x[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        uint32_t pw[4], ph[4], pl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 64 * hs + 8 * ch + 2 * e;
          pw[e] = pack2(x[2 * e] * c1[c], x[2 * e + 1] * c1[c + 1]);
          split2(x[2 * e] * bet[c], x[2 * e + 1] * bet[c + 1], ph[e], pl[e]);
        }
        w = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        hi = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        lo = make_uint4(pl[0], pl[1], pl[2], pl[3]);
      }
      const int off = R * 128 + ((ch ^ (R & 7)) << 4);
      *reinterpret_cast<uint4*>(sm + S_XW + off) = w;
      *reinterpret_cast<uint4*>(sm + S_XH + off) = hi;
      *reinterpret_cast<uint4*>(sm + S_XL + off) = lo;
    }
    tc::fence_proxy_async_smem();  // generic-proxy writes -> the MMA's reads
    tc::tc_fence_before();
    if (__syncthreads_or(!vok)) {
      drain_and_leave();
      return;
    }

    // 7. W = [X'_h0; X'_h1] K (M = 128, N = 128, K = 64; B = the K tile read
    //    MN-major) and U = [X"_h0; X"_h1] [V_h0 | V_h1] (M = 128, N = 256), hi then lo
    if (tid == 0) {
      tc::tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16)
        tc::mma_bf16(tmem + TM_W, tc::sw128_desc(sb + S_XW + k16 * 32, 16, 1024),
                     tc::sw128_desc(sb + S_KQ + k16 * 2048, 16384, 1024),
                     tc::idesc_bf16(128, 128, false, true), k16 > 0);
#pragma unroll
      for (int k16 = 0; k16 < 8; ++k16)
        tc::mma_bf16(tmem + TM_U,
                     tc::sw128_desc(sb + (k16 < 4 ? S_XH : S_XL) + (k16 & 3) * 32, 16, 1024),
                     tc::sw128_desc(sb + S_V + (k16 & 3) * 2048, 8192, 1024),
                     tc::idesc_bf16(128, 256, false, true), k16 > 0);
      tc::mma_commit(&bar[2]);
      ++mma_issued;
    }
    ok = tc::mbar_wait(&bar[2], (uint32_t)(p + 1) & 1u, status, 124);
    if (__syncthreads_or(!ok)) {
      drain_and_leave();
      return;
    }
    tc::tc_fence_after();
    if (tid == 0) {
      ++mma_done;
      if (p + 1 < npairs) issue_v(p + 1);  // the MMA reads of V are complete
    }

    // 8. W (fp16) and U (fp32) rows staged for tensor stores: row r = head r / 64,
    //    time step r % 64; this warp's 64 of the 128 columns
    float umax = 0.f;
    {
      const int hs = r >> 6, t = r & 63;  // hs is uniform in the warp
      if (hs < nh) {
        uint8_t* sw = sm + S_SW + hs * 16384 + hc * 8192;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          float v[32];
          tc::tmem_ld32(tq + TM_W + 64 * hc + 32 * k, v);
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) {
            uint4 o;
            o.x = pack2h(v[c8 + 0], v[c8 + 1]);
            o.y = pack2h(v[c8 + 2], v[c8 + 3]);
            o.z = pack2h(v[c8 + 4], v[c8 + 5]);
            o.w = pack2h(v[c8 + 6], v[c8 + 7]);
            *reinterpret_cast<uint4*>(sw + box_off(t, 4 * k + (c8 >> 3))) = o;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) range = fmaxf(range, fabsf(v[c]));
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          float v[32];
          tc::tmem_ld32(tq + TM_U + 128 * hs + 64 * hc + 32 * k, v);
          uint8_t* su = sm + S_SU + hs * 32768 + (2 * hc + k) * 8192;
#pragma unroll
          for (int c4 = 0; c4 < 32; c4 += 4) {
            *reinterpret_cast<float4*>(su + box_off(t, c4 >> 2)) =
                make_float4(v[c4], v[c4 + 1], v[c4 + 2], v[c4 + 3]);
            umax = fmaxf(umax, fmaxf(fmaxf(fabsf(v[c4]), fabsf(v[c4 + 1])),
                                     fmaxf(fabsf(v[c4 + 2]), fabsf(v[c4 + 3]))));
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, o));
    if (lane == 0) misc[8 + warp] = umax;
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      for (int hs = 0; hs < nh; ++hs) {
        const int row = (b * Hv + hv0 + hs) * Tp + t0;
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tc::tma_store_2d(&maps.w, sm + S_SW + hs * 16384 + h * 8192, 64 * h, row);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          tc::tma_store_2d(&maps.u, sm + S_SU + hs * 32768 + qq * 8192, 32 * qq, row);
      }
      tc::bulk_commit();
    }

    // 9. per-row factors of the scan for both heads: fo = gamma sq 2^eq,
    //    fs = rk 2^ek gamma_C / gamma, gamma_C for every state row, max |U|
    if (tid < 128) {
      const int hs = tid >> 6, t = tid & 63;
      if (hs < nh) {
        const size_t head = (size_t)b * Hv + hv0 + hs;
        float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
        const float GC = Gs[64 * hs + kC - 1], Gt = Gs[64 * hs + t];
        sc[t] = __expf(Gt) * sq[t] * pq[t];
        sc[kC + t] = t < nv ? rk[t] * pk[t] * __expf(GC - Gt) : 0.f;
        const float gc = __expf(GC);
        sc[kScGC + t] = gc;
        sc[kScGC + kC + t] = gc;
        if (t < 4) {
          // warps whose accumulator rows belong to head hs: lane quarters 2 hs, 2 hs + 1
          const float m = fmaxf(fmaxf(misc[8 + 2 * hs], misc[9 + 2 * hs]),
                                fmaxf(misc[12 + 2 * hs], misc[13 + 2 * hs]));
          sc[kScMaxU + t] = t == 0 ? m : 0.f;
        }
      }
    }
    if (p + 1 < npairs) __syncthreads();  // Gs, bet, misc are rewritten by the next pair
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
  const WsLayout L = ws_layout(a.B, a.T, a.Hk, a.Hv);
  const int Nc = (a.T + kC - 1) / kC;
  const uint64_t Tp = (uint64_t)Nc * kC;
  const uint64_t rv = (uint64_t)a.B * a.Hv * Tp, rk = (uint64_t)a.B * a.Hk * Tp;
  uint8_t* w = static_cast<uint8_t*>(ws);
  PrepMaps m;
  if (!make_map_bthd(&m.q, a.q, a.B, a.T, a.Hk) || !make_map_bthd(&m.k, a.k, a.B, a.T, a.Hk) ||
      !make_map_bthd(&m.v, a.v, a.B, a.T, a.Hv) ||
      !make_map_rows(&m.qh, w + L.qh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.kh, w + L.kh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rk) ||
      !make_map_rows(&m.w, w + L.w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kD, rv) ||
      !make_map_rows(&m.a, w + L.a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kC, rv) ||
      !make_map_rows(&m.u, w + L.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kD, rv))
    return cudaErrorInvalidValue;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  const int l2 = (a.flags & GDN_QK_L2NORM) ? 1 : 0;
  auto prep = pre ? wy_prep_tc_kernel<true> : wy_prep_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, PT_SMEM);
  if (e != cudaSuccess) return e;
  prep<<<dim3(Nc, a.B * a.Hk), kPT, PT_SMEM, s>>>(m, a.a, a.b, a.A_log, a.dt_bias, a.T, a.Hk,
                                                  a.Hv, a.scale, l2, w, L, status);
  return cudaGetLastError();
}

}  // namespace gdn
