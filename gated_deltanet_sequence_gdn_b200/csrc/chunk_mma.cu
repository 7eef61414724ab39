// chunk_mma.cu -- bf16 chunkwise GDN / Gated DeltaNet-2 forward (dk = dv = 128,
// chunk C = 64) on the tensor cores, in two kernels per call:
//
//  the prep, parallel over the whole sequence:
//    GDN   : wy_prep_tc_kernel (prep_tc.cu, tcgen05), one CTA per (chunk, key
//            head) serving the value heads of its GQA group;
//    GDN-2 : wy_prep2_kernel (this file), one CTA per (chunk, value head): TMA
//            tile loads, the element-wise diagonal blocks and the 16-row
//            off-diagonal blocks (warp-level mma.sync, below tcgen05's minimum
//            M of 64), and W, U as tcgen05 products with TMEM accumulators.
//    Both form the in-chunk prefix sums G_r of the log-decays, the strictly
//    lower L = diag(beta) (K^ K^^T o Gamma), X = (I + L)^-1 by blocked forward
//    substitution in fp32, W = X diag(beta gamma) K^, U = X diag(beta) V and
//    A_qk = tril(Q^ K^^T o Gamma) (diagonal included), written to the workspace
//    with the per-row factors of the scan and fp16 copies of the raw Q and K rows.
//  the state scan (scan_tc.cu, tcgen05): one CTA per (value head, 64-column
//      half of d_v), sequential over the chunks with the fp32 state held in
//      registers:  U~ = U - W S,  o = diag(gamma sq) Q S + A_qk U~,
//      S <- gamma_C S + K^T diag(rk gamma_C / gamma) U~.
//
// The algebra is the WY / UT chunk form of the delta rule ("Gated DeltaNet-2",
// section on the chunkwise algorithm; GDN is its scalar-decay special case):
// Gamma_rj = exp(G_r - G_j) only for j <= r, so every exponent is <= 0.
//
// Precision: fp32 accumulation and state.  The prep's products take bf16
// operands (the inputs are bf16; X (diag(beta)) is carried as bf16 hi + lo, one
// product per part, and U is stored in fp32).  The scan's products take fp16
// operands (11 significant bits): W, A_qk, the state, U~ and U~ diag(fs), and
// the raw Q / K rows.  fp16 has a narrow range, so every fp16 operand is kept in
// range by an exact power-of-2 scale folded into a factor applied in fp32:
//   - each raw Q / K row r is stored as q_r 2^-e_r with its largest entry in
//     [1, 2); 2^e_r is folded into fo_r / fs_r;
//   - the scan multiplies U, the state and the output of one CTA by one
//     sigma = 2^-e chosen from the largest |U| of its head and |h0| of its
//     slice, so that both are below 2^8 (the delta rule keeps |S| of the
//     order of |v|); the output and the final state are divided by sigma;
//   - W and A_qk are bounded by construction for unit-norm keys.
// A value that still leaves the fp16 range sets the range bit of the status
// word (read by gdn_check_status); nothing is clamped silently.
#include "common.cuh"
#include "launch.h"
#include "chunk_layout.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"
#include "warp_mma.cuh"
#include "wy_common.cuh"

namespace gdn {
namespace {

using namespace wm;
using namespace wy;
using bf16 = __nv_bfloat16;

constexpr int kThreads = 512;  // 16 warps
constexpr int LDT = kD + 8;    // 16-bit row stride of 128-wide tiles (272 B: ldmatrix conflict-free)

// ---------------------------------------------------------------- GDN-2 prep kernel
// Gate arithmetic of the tensor-core GDN-2 path with the hardware exp2/log2
// approximations (relative error ~1e-6, far below the bf16 path's budget):
// softplus(x) = max(x, 0) + log(1 + e^-|x|), sigmoid(x) = 1 / (1 + e^-x).
__device__ __forceinline__ float softplus_fast(float x) {
  return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// Gated DeltaNet-2: per-channel decay d_t = exp(g_t) (g_t in R^dk), erase
// direction e_t = b_t (.) k^_t, written value z_t = w_t (.) v_t.  With G the
// in-chunk prefix sum of g (per channel) the chunk form is
//   L_ji   = sum_c e_jc k^_ic exp(G_jc - G_ic)       (i < j)
//   A_tj   = sum_c q^_tc k^_jc exp(G_tc - G_jc)      (j <= t)
//   X = (I + L)^-1,  W = X (exp(G) (.) E),  U = X Z
//   o = (exp(G) (.) Q^) S + A (U - W S),   S <- diag(exp(G_C)) S + K_tail^T (U - W S)
// with K_tail rows exp(G_C - G_j) (.) k^_j ("Gated DeltaNet-2", 通道级衰减的吸收技巧
// and WY 形式).  The exponents differ per channel, so the 16 x 16 diagonal blocks
// of L and A are summed element by element (exp(G_j - G_i) there is the product of
// the per-token decays d = exp(g) of rows i+1..j), and each off-diagonal block row
// I is a product of operands scaled about its first row r = 16 I:
//   L_ji = sum_c [e_jc exp(G_jc - G_rc)] [k^_ic exp(G_rc - G_ic)]   (i < r <= j)
// where both exponents are <= 0, so every operand stays within its input's size.
constexpr int LDG = kD + 4;                    // f32 row stride of [64][128] channel tiles
constexpr int Q2_KT = 0;                       // raw K tile [64][LDT] bf16
constexpr int Q2_QT = Q2_KT + kC * LDT * 2;    // raw Q tile
constexpr int Q2_ZH = Q2_QT + kC * LDT * 2;    // raw V tile, then z = w (.) v (bf16 hi part)
constexpr int Q2_ZL = Q2_ZH + kC * LDT * 2;    // z lo part
constexpr int Q2_G = Q2_ZL + kC * LDT * 2;     // G [64][LDG] f32 (first: g, or the raw g tile)
constexpr int Q2_E = Q2_G + kC * LDG * 4;      // e [64][LDG] f32 (first: the raw b tile)
constexpr int Q2_L = Q2_E + kC * LDG * 4;      // L [64][LDX] f32, then X in place
constexpr int Q2_X = Q2_L + kC * LDX * 4;      // A staging (f32), then the inverse's block products
constexpr int Q2_OP = Q2_X + kC * LDX * 4;     // raw gate tiles, decays d, fp16 operands, E-bar
constexpr int Q2_OPB = 192 * LDT * 2;
constexpr int Q2_VEC = Q2_OP + Q2_OPB;         // rk, sq [64], carry [3][128], misc [64]
constexpr int Q2_BAR = Q2_VEC + 576 * 4;       // 2 mbarriers (tile loads, products) + TMEM address
constexpr int Q2_BYTES = Q2_BAR + 32 + 1024;   // + slack for the 1024-byte alignment of the base
// The products W^T = E-bar^T X^T and U^T = Z^T X^T on the tcgen05 tensor cores
// (M = 128 channels d, N = 64 tokens t, K = 64 tokens t'), accumulators in TMEM:
// E-bar and Z (bf16 hi, lo) as MN-major A operands, [2 d-halves][64 t'][128 B]
// with the 128-byte swizzle (in the operand scratch and the Z tiles' space), X as
// bf16 hi + lo K-major B operands, [64 t][128 B] swizzled (in the A staging's
// space, free once the inverse is done).
constexpr int Q2_XH = Q2_X;                    // X hi, then X lo at + 8192
constexpr uint32_t Q2_TM_W = 0, Q2_TM_U = 64, Q2_TM_COLS = 128;
static_assert(Q2_ZH % 1024 == 0 && Q2_ZL % 1024 == 0 && Q2_X % 1024 == 0 && Q2_OP % 1024 == 0,
              "swizzled operand tiles need 1024-byte alignment");
static_assert(2 * 8192 <= kC * LDX * 4, "X hi + lo fit the A staging's space");

// Byte offset of the 16-byte unit u (0..7) of row t in a [64 rows][128 B] swizzled box.
__device__ __forceinline__ int box16(int t, int u) { return (t << 7) + ((u ^ (t & 7)) << 4); }

// TMA maps of the tile loads: raw k, q, v rows and the three gate tiles, each a
// box of 64 time steps of one head, landing as padded rows (LDT bf16 or LDG f32).
struct Prep2Maps {
  CUtensorMap k, q, v, ga, gb, gw;
};
static_assert(Q2_BYTES <= 227 * 1024, "shared memory of the GDN-2 prep kernel");
static_assert(kC * LDG * 4 <= Q2_OPB, "a float32 [64][LDG] tile (raw w, the decays) fits the operand scratch");

template <bool PRE>
__global__ void __launch_bounds__(kThreads, 1)
wy_prep2_kernel(const __grid_constant__ Prep2Maps maps, const float* __restrict__ A_log,
                const float* __restrict__ dt_bias, int T, int H, float scale, int l2,
                uint8_t* __restrict__ ws, WsLayout L, int* status, uint32_t spin) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sm = sm_raw + ((1024u - (tc::smem_u32(sm_raw) & 1023u)) & 1023u);
  bf16* Kt = reinterpret_cast<bf16*>(sm + Q2_KT);
  bf16* Qt = reinterpret_cast<bf16*>(sm + Q2_QT);
  bf16* Zh = reinterpret_cast<bf16*>(sm + Q2_ZH);
  bf16* Zl = reinterpret_cast<bf16*>(sm + Q2_ZL);
  float* Gm = reinterpret_cast<float*>(sm + Q2_G);
  float* Em = reinterpret_cast<float*>(sm + Q2_E);
  float* Lm = reinterpret_cast<float*>(sm + Q2_L);
  float* Xm = reinterpret_cast<float*>(sm + Q2_X);
  uint8_t* op = sm + Q2_OP;
  float* rk = reinterpret_cast<float*>(sm + Q2_VEC);
  float* sq = rk + 64;
  float* carry = sq + 64;     // [3][128] prefix sums of the first three quarters
  float* misc = carry + 384;  // [8..23] per-warp max |U|
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Q2_BAR);  // tile loads, products
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Q2_BAR + 16);
  const uint32_t sb = tc::smem_u32(sm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int n = blockIdx.y, Nc = gridDim.y, Tp = Nc * kC;
  const int b = blockIdx.z / H, h = blockIdx.z % H;
  const size_t head = blockIdx.z;  // one key head per value head
  const int t0 = n * kC, nv = min(kC, T - t0);
  float range = 0.f;

  // 1. raw q, k, v tiles and the gate tiles by TMA, as padded rows (time steps past
  //    the end of the sequence and the pad columns read as zeros)
  if (tid == 0) {
    tc::mbar_init(&bar[0], 1);
    tc::mbar_init(&bar[1], 1);
    tc::fence_mbar_init();
    constexpr uint32_t kRow16 = kC * LDT * 2, kRow32 = kC * LDG * 4;
    tc::mbar_arrive_expect_tx(&bar[0], 3 * kRow16 + 3 * (PRE ? kRow32 : kRow16));
    tc::tma_load_4d(Kt, &maps.k, &bar[0], 0, h, t0, b);
    tc::tma_load_4d(Qt, &maps.q, &bar[0], 0, h, t0, b);
    tc::tma_load_4d(Zh, &maps.v, &bar[0], 0, h, t0, b);
    if (PRE) {  // g, b, w values in float32
      tc::tma_load_4d(Gm, &maps.ga, &bar[0], 0, h, t0, b);
      tc::tma_load_4d(Em, &maps.gb, &bar[0], 0, h, t0, b);
      tc::tma_load_4d(op, &maps.gw, &bar[0], 0, h, t0, b);
    } else {  // a, b, w logits in bf16
      tc::tma_load_4d(op, &maps.ga, &bar[0], 0, h, t0, b);
      tc::tma_load_4d(op + kRow16, &maps.gb, &bar[0], 0, h, t0, b);
      tc::tma_load_4d(op + 2 * kRow16, &maps.gw, &bar[0], 0, h, t0, b);
    }
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, Q2_TM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  {
    const bool ok = tc::mbar_wait(&bar[0], 0, status, 131, spin);
    if (__syncthreads_or(!ok)) {  // leave once the copies in flight have landed
      if (tid == 0) tc::mbar_wait(&bar[0], 0, nullptr, 0, 1u << 20);
      __syncthreads();
      if (warp == 0) tc::tmem_dealloc(tmem, Q2_TM_COLS);
      return;
    }
  }

  // 2. L2 norms: rk = 1 / |k|, sq = scale / |q| (four threads per row)
  {
    const int which = tid >> 8, r = (tid & 255) >> 2, hh = tid & 3;
    const bf16* row = (which ? Qt : Kt) + r * LDT + hh * 8;
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 128; c += 32) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c);
      const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
      ss += f0.x * f0.x + f0.y * f0.y + f1.x * f1.x + f1.y * f1.y + f2.x * f2.x + f2.y * f2.y +
            f3.x * f3.x + f3.y * f3.y;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    if (hh == 0) {
      const float inv = l2 ? rsqrtf(ss + 1e-6f) : 1.f;
      if (which) sq[r] = inv * scale;
      else rk[r] = inv;
    }
  }
  __syncthreads();

  // 3. per (token, channel), all independent: g, e = b (.) k^ and z = w (.) v (as
  //    bf16 hi + lo); a thread takes 8 channels of a row at a time (its channels
  //    c8 .. c8 + 7 are the same in every row); then the in-chunk prefix sums G down
  //    each channel (four threads per channel, 16 tokens each)
  {
    const int c8 = (tid & 15) * 8;
    float nal[8], dtb[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      nal[u] = PRE ? 0.f : -expf(A_log[(size_t)h * kD + c8 + u]);
      dtb[u] = PRE ? 0.f : dt_bias[(size_t)h * kD + c8 + u];
    }
    const bf16* at = reinterpret_cast<const bf16*>(op);
    const bf16* bt = at + kC * LDT;
    const bf16* wt = bt + kC * LDT;
    const float* wf = reinterpret_cast<const float*>(op);
#pragma unroll 1
    for (int it = tid; it < kC * 16; it += kThreads) {
      const int r = it >> 4;
      float g[8], bv[8], wv[8], kr[8], vr[8];
      if (PRE) {
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
          const float4 g4 = *reinterpret_cast<const float4*>(Gm + r * LDG + c8 + 4 * h4);
          const float4 b4 = *reinterpret_cast<const float4*>(Em + r * LDG + c8 + 4 * h4);
          const float4 w4 = *reinterpret_cast<const float4*>(wf + r * LDG + c8 + 4 * h4);
          g[4 * h4] = g4.x, g[4 * h4 + 1] = g4.y, g[4 * h4 + 2] = g4.z, g[4 * h4 + 3] = g4.w;
          bv[4 * h4] = b4.x, bv[4 * h4 + 1] = b4.y, bv[4 * h4 + 2] = b4.z, bv[4 * h4 + 3] = b4.w;
          wv[4 * h4] = w4.x, wv[4 * h4 + 1] = w4.y, wv[4 * h4 + 2] = w4.z, wv[4 * h4 + 3] = w4.w;
        }
      } else {
        const uint4 ua = *reinterpret_cast<const uint4*>(at + r * LDT + c8);
        const uint4 ub = *reinterpret_cast<const uint4*>(bt + r * LDT + c8);
        const uint4 uw = *reinterpret_cast<const uint4*>(wt + r * LDT + c8);
        const uint32_t* pa = reinterpret_cast<const uint32_t*>(&ua);
        const uint32_t* pb = reinterpret_cast<const uint32_t*>(&ub);
        const uint32_t* pw = reinterpret_cast<const uint32_t*>(&uw);
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
          const float2 a2 = unpack2(pa[u2]), b2 = unpack2(pb[u2]), w2 = unpack2(pw[u2]);
          g[2 * u2] = r < nv ? nal[2 * u2] * softplus_fast(a2.x + dtb[2 * u2]) : 0.f;
          g[2 * u2 + 1] = r < nv ? nal[2 * u2 + 1] * softplus_fast(a2.y + dtb[2 * u2 + 1]) : 0.f;
          bv[2 * u2] = sigmoid_fast(b2.x), bv[2 * u2 + 1] = sigmoid_fast(b2.y);
          wv[2 * u2] = sigmoid_fast(w2.x), wv[2 * u2 + 1] = sigmoid_fast(w2.y);
        }
      }
      {
        const uint4 uk = *reinterpret_cast<const uint4*>(Kt + r * LDT + c8);
        const uint4 uv = *reinterpret_cast<const uint4*>(Zh + r * LDT + c8);
        const uint32_t* pk = reinterpret_cast<const uint32_t*>(&uk);
        const uint32_t* pv = reinterpret_cast<const uint32_t*>(&uv);
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
          const float2 k2 = unpack2(pk[u2]), v2 = unpack2(pv[u2]);
          kr[2 * u2] = k2.x, kr[2 * u2 + 1] = k2.y, vr[2 * u2] = v2.x, vr[2 * u2 + 1] = v2.y;
        }
      }
      const float rkr = rk[r];
      uint4 zh4, zl4;
      uint32_t* ph = reinterpret_cast<uint32_t*>(&zh4);
      uint32_t* pl = reinterpret_cast<uint32_t*>(&zl4);
#pragma unroll
      for (int u2 = 0; u2 < 4; ++u2) {
        const float z0 = wv[2 * u2] * vr[2 * u2], z1 = wv[2 * u2 + 1] * vr[2 * u2 + 1];
        ph[u2] = pack2(z0, z1);
        const float2 zr = unpack2(ph[u2]);
        pl[u2] = pack2(z0 - zr.x, z1 - zr.y);
      }
      *reinterpret_cast<uint4*>(Zh + r * LDT + c8) = zh4;
      *reinterpret_cast<uint4*>(Zl + r * LDT + c8) = zl4;
#pragma unroll
      for (int h4 = 0; h4 < 2; ++h4) {
        const int u = 4 * h4;
        *reinterpret_cast<float4*>(Gm + r * LDG + c8 + u) =
            make_float4(g[u], g[u + 1], g[u + 2], g[u + 3]);
        *reinterpret_cast<float4*>(Em + r * LDG + c8 + u) =
            make_float4(bv[u] * kr[u] * rkr, bv[u + 1] * kr[u + 1] * rkr,
                        bv[u + 2] * kr[u + 2] * rkr, bv[u + 3] * kr[u + 3] * rkr);
      }
    }
  }
  const int ch = tid & 127, qtr = tid >> 7;
  __syncthreads();
  //    the raw gate tiles are consumed: the per-token decays d = exp(g) go to the
  //    operand scratch (for the diagonal blocks below), then g becomes G in place
  float* Dm = reinterpret_cast<float*>(op);
  {
    float run = 0.f;
#pragma unroll 8
    for (int tt = 0; tt < 16; ++tt) {
      const int r = 16 * qtr + tt;
      const float g = Gm[r * LDG + ch];
      Dm[r * LDG + ch] = __expf(g);
      run += g;
      Gm[r * LDG + ch] = run;
    }
    if (qtr < 3) carry[qtr * 128 + ch] = run;
  }
  __syncthreads();
  if (qtr > 0) {
    float cy = carry[ch];
    if (qtr > 1) cy += carry[128 + ch];
    if (qtr > 2) cy += carry[256 + ch];
#pragma unroll 8
    for (int tt = 0; tt < 16; ++tt) Gm[(16 * qtr + tt) * LDG + ch] += cy;
  }
  __syncthreads();

  // 4. diagonal 16 x 16 blocks of L and A, element by element.  Inside a block
  //    exp(G_j - G_i) = d_{i+1} ... d_j (each factor <= 1), so column i is one
  //    running product P = k_i d_{i+1} ... d_j per channel, walked down the rows
  //    j = i..15.  Lane: block bl = lane / 8 and the 16 channels 4 cg + 32 s + u
  //    (cg = lane % 8, s, u < 4); warp w takes column w (w < 8) or 23 - w of all
  //    four blocks, so that the four warps w = s, s + 4, s + 8, s + 12 of one
  //    scheduler walk 34 rows in all.  The eight lanes of a block then sum their
  //    partial L and A over the 128 channels.
  {
    const int bl = lane >> 3, cg = lane & 7;
    const bool odd = (cg & 1) != 0;
    {
      const int ic = warp < 8 ? warp : 23 - warp;  // column within the block (warp-uniform)
      const int ci = 16 * bl + ic;
      float2 P[8];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint2 kk = *reinterpret_cast<const uint2*>(Kt + ci * LDT + 4 * cg + 32 * s);
        P[2 * s] = unpack2(kk.x);
        P[2 * s + 1] = unpack2(kk.y);
      }
      const float rki = rk[ci];
#pragma unroll 1
      for (int jr = ic; jr < 16; ++jr) {
        const int rj = 16 * bl + jr;
        if (jr > ic) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const float4 d4 = *reinterpret_cast<const float4*>(Dm + rj * LDG + 4 * cg + 32 * s);
            P[2 * s] = fmul2(P[2 * s], make_float2(d4.x, d4.y));
            P[2 * s + 1] = fmul2(P[2 * s + 1], make_float2(d4.z, d4.w));
          }
        }
        float2 sl2 = make_float2(0.f, 0.f), sa2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const float4 e4 = *reinterpret_cast<const float4*>(Em + rj * LDG + 4 * cg + 32 * s);
          const uint2 qq = *reinterpret_cast<const uint2*>(Qt + rj * LDT + 4 * cg + 32 * s);
          sl2 = ffma2(make_float2(e4.x, e4.y), P[2 * s], sl2);
          sl2 = ffma2(make_float2(e4.z, e4.w), P[2 * s + 1], sl2);
          sa2 = ffma2(unpack2(qq.x), P[2 * s], sa2);
          sa2 = ffma2(unpack2(qq.y), P[2 * s + 1], sa2);
        }
        const float sl = sl2.x + sl2.y, sa = sa2.x + sa2.y;
        // even lanes go on with L, odd lanes with A, each summing over all eight
        float acc = (odd ? sa : sl) + __shfl_xor_sync(0xffffffffu, odd ? sl : sa, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (cg == 0) Lm[rj * LDX + ci] = jr > ic ? acc * rki : 0.f;
        if (cg == 1) Xm[rj * LDX + ci] = acc * sq[rj] * rki;
      }
    }
  }
  __syncthreads();  // the decays in the operand scratch are read

  // 5. off-diagonal blocks on the tensor cores: fp16 operands scaled about the
  //    reference row r = 16 I of block row I (I = 1..3).  Rows of the operand
  //    scratch: [0,48) e rows of blocks 1-3, [48,96) q^ rows, [96,192) k^ rows
  //    0..16 I - 1 for I = 1, 2, 3 (at 96, 112, 144).
  __half* Op = reinterpret_cast<__half*>(op);
  for (int row = warp; row < 192; row += kThreads / 32) {
    const int c = 4 * lane;
    int j, I;
    const float* src;  // row of e, or of raw q / k (bf16) below
    float f = 1.f;
    float4 sc;
    if (row < 96) {
      I = 1 + ((row < 48 ? row : row - 48) >> 4);
      j = 16 * I + (row & 15);
      const float4 gj = *reinterpret_cast<const float4*>(Gm + j * LDG + c);
      const float4 gr = *reinterpret_cast<const float4*>(Gm + 16 * I * LDG + c);
      sc = make_float4(__expf(gj.x - gr.x), __expf(gj.y - gr.y), __expf(gj.z - gr.z),
                       __expf(gj.w - gr.w));
    } else {
      const int kr = row - 96;
      I = kr < 16 ? 1 : (kr < 48 ? 2 : 3);
      j = kr - (I == 1 ? 0 : (I == 2 ? 16 : 48));
      const float4 gj = *reinterpret_cast<const float4*>(Gm + j * LDG + c);
      const float4 gr = *reinterpret_cast<const float4*>(Gm + 16 * I * LDG + c);
      sc = make_float4(__expf(gr.x - gj.x), __expf(gr.y - gj.y), __expf(gr.z - gj.z),
                       __expf(gr.w - gj.w));
    }
    float4 val;
    if (row < 48) {
      src = Em + j * LDG;
      val = *reinterpret_cast<const float4*>(src + c);
    } else {
      const uint2 raw = *reinterpret_cast<const uint2*>((row < 96 ? Qt : Kt) + j * LDT + c);
      const float2 v01 = unpack2(raw.x), v23 = unpack2(raw.y);
      f = row < 96 ? sq[j] : rk[j];
      val = make_float4(v01.x, v01.y, v23.x, v23.y);
    }
    uint2 o;
    o.x = pack2h(val.x * f * sc.x, val.y * f * sc.y);
    o.y = pack2h(val.z * f * sc.z, val.w * f * sc.w);
    *reinterpret_cast<uint2*>(Op + row * LDT + c) = o;
  }
  __syncthreads();
  //    tasks (matrix, I, column pair np < I): 6 for L, 6 for A
  if (warp < 12) {
    const int task = warp;
    const bool isa = task >= 6;
    const int tk = isa ? task - 6 : task;
    const int I = tk < 1 ? 1 : (tk < 3 ? 2 : 3);
    const int np = tk - (I == 1 ? 0 : (I == 2 ? 1 : 3));
    const __half* Arows = Op + ((isa ? 48 : 0) + 16 * (I - 1)) * LDT;
    const __half* Brows = Op + (96 + (I == 1 ? 0 : (I == 2 ? 16 : 48))) * LDT;
    float acc[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4], bb[4];
      ldsm_x4(a, Arows + lrow_a(lane) * LDT + 16 * ks + lcol_a(lane));
      ldsm_x4(bb, Brows + (16 * np + lrow_b(lane)) * LDT + 16 * ks + lcol_b(lane));
      mma_f16(acc[0], a, bb[0], bb[1]);
      mma_f16(acc[1], a, bb[2], bb[3]);
    }
    float* dst = isa ? Xm : Lm;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int r = 16 * I + g8, c = 16 * np + 8 * nt + 2 * t4;
      *reinterpret_cast<float2*>(dst + r * LDX + c) = make_float2(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<float2*>(dst + (r + 8) * LDX + c) = make_float2(acc[nt][2], acc[nt][3]);
    }
  }
  __syncthreads();
  //    A to the workspace (fp16, zeros above the diagonal)
  {
    __half* ag = reinterpret_cast<__half*>(ws + L.a) + (head * Tp + t0) * kC;
    for (int i = tid; i < kC * 8; i += kThreads) {
      const int r = i >> 3, c8 = (i & 7) * 8;
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c8 + 2 * u;
        ow[u] = pack2h(c <= r ? Xm[r * LDX + c] : 0.f, c + 1 <= r ? Xm[r * LDX + c + 1] : 0.f);
      }
      *reinterpret_cast<uint4*>(ag + (size_t)r * kC + c8) = o;
    }
  }
  __syncthreads();

  // 6. X = (I + L)^-1 in place of L (the A staging is free now and takes the
  //    block products); the blocks above the diagonal, never written, are zeroed
  for (int i = tid; i < 6 * 256; i += kThreads) {
    const int blk = i >> 8, e = i & 255;  // blocks (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
    const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
    const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
    Lm[(16 * bi + (e >> 4)) * LDX + 16 * bj + (e & 15)] = 0.f;
  }
  invert_in_place(Lm, Xm, tid, warp, g8, t4);
  float* Xi = Lm;  // X

  // 7. W^T = E-bar^T X^T and U^T = Z^T X^T on the tcgen05 tensor cores.  First
  //    E-bar = exp(G) (.) e in bf16 (MN-major A operand, in the operand scratch) and
  //    X as bf16 hi + lo (K-major B operands, in the A staging's space)
  {
    uint8_t* eb = op;
    for (int i = tid; i < kC * 16; i += kThreads) {
      const int r = i >> 4, c8 = (i & 15) * 8;
      uint4 o;
      uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int h4 = 0; h4 < 2; ++h4) {
        const float4 g4 = *reinterpret_cast<const float4*>(Gm + r * LDG + c8 + 4 * h4);
        const float4 e4 = *reinterpret_cast<const float4*>(Em + r * LDG + c8 + 4 * h4);
        po[2 * h4] = pack2(__expf(g4.x) * e4.x, __expf(g4.y) * e4.y);
        po[2 * h4 + 1] = pack2(__expf(g4.z) * e4.z, __expf(g4.w) * e4.w);
      }
      *reinterpret_cast<uint4*>(eb + (c8 >> 6) * 8192 + box16(r, (c8 & 63) >> 3)) = o;
    }
    uint8_t* xh = sm + Q2_XH;
    for (int i = tid; i < kC * 8; i += kThreads) {
      const int t = i >> 3, ch = i & 7;
      const float* xr = Xi + t * LDX + 8 * ch;
      const float4 a0 = *reinterpret_cast<const float4*>(xr);
      const float4 a1 = *reinterpret_cast<const float4*>(xr + 4);
      uint32_t ph[4], pl[4];
      split2(a0.x, a0.y, ph[0], pl[0]);
      split2(a0.z, a0.w, ph[1], pl[1]);
      split2(a1.x, a1.y, ph[2], pl[2]);
      split2(a1.z, a1.w, ph[3], pl[3]);
      const int off = box16(t, ch);
      *reinterpret_cast<uint4*>(xh + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(xh + 8192 + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
  }
  __syncthreads();  // e is read: its space takes the Z operand tiles
  //    Z = w (.) v, hi and lo (padded rows) -> MN-major operand tiles in e's space
  {
    const bf16* zl_rows = reinterpret_cast<const bf16*>(sm + Q2_ZL);
    uint8_t* zt = sm + Q2_E;
    for (int i = tid; i < 2 * kC * 16; i += kThreads) {
      const int part = i >> 10, r = (i >> 4) & 63, c8 = (i & 15) * 8;
      const uint4 u = *reinterpret_cast<const uint4*>((part ? zl_rows : Zh) + r * LDT + c8);
      *reinterpret_cast<uint4*>(zt + part * 16384 + (c8 >> 6) * 8192 + box16(r, (c8 & 63) >> 3)) =
          u;
    }
  }
  tc::fence_proxy_async_smem();  // generic-proxy writes -> the MMA's reads
  tc::tc_fence_before();
  __syncthreads();
  if (tid == 0) {  // W: X hi / lo against E-bar; U: the three hi / lo pairs but lo.lo
    tc::tc_fence_after();
    const uint32_t id = tc::idesc_bf16(128, 64, true, false);
    const uint32_t eb = sb + Q2_OP, zh = sb + Q2_E, zl = zh + 16384;
    const uint32_t xh = sb + Q2_XH, xl = xh + 8192;
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16) {
      const uint64_t dxh = tc::sw128_desc(xh + k16 * 32, 16, 1024);
      const uint64_t dxl = tc::sw128_desc(xl + k16 * 32, 16, 1024);
      const uint64_t de = tc::sw128_desc(eb + k16 * 2048, 8192, 1024);
      const uint64_t dzh = tc::sw128_desc(zh + k16 * 2048, 8192, 1024);
      const uint64_t dzl = tc::sw128_desc(zl + k16 * 2048, 8192, 1024);
      tc::mma_bf16(tmem + Q2_TM_W, de, dxh, id, k16 > 0);
      tc::mma_bf16(tmem + Q2_TM_W, de, dxl, id, 1u);
      tc::mma_bf16(tmem + Q2_TM_U, dzh, dxh, id, k16 > 0);
      tc::mma_bf16(tmem + Q2_TM_U, dzh, dxl, id, 1u);
      tc::mma_bf16(tmem + Q2_TM_U, dzl, dxh, id, 1u);
    }
    tc::mma_commit(&bar[1]);
  }
  {
    const bool ok = tc::mbar_wait(&bar[1], 0, status, 132, spin);
    if (__syncthreads_or(!ok)) {  // leave once the products in flight are done
      if (tid == 0) tc::mbar_wait(&bar[1], 0, nullptr, 0, 1u << 20);
      tc::tc_fence_before();
      __syncthreads();
      if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Q2_TM_COLS);
      }
      return;
    }
  }
  tc::tc_fence_after();
  //    W (fp16) and U (fp32) to the workspace: lane = channel d; warp w takes the 16
  //    tokens 16 (w / 4) .. + 15 of its lane quarter w % 4, so the 32 lanes of a
  //    warp store 32 consecutive channels of one row
  float umax = 0.f;
  {
    const int q4 = warp & 3, tb = 16 * (warp >> 2), d = 32 * q4 + lane;
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)tb;
    __half* dw = reinterpret_cast<__half*>(ws + L.w) + (head * Tp + t0 + tb) * kD + d;
    float* du = reinterpret_cast<float*>(ws + L.u) + (head * Tp + t0 + tb) * kD + d;
    float v[16];
    tc::tmem_ld16(tq + Q2_TM_W, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      range = fmaxf(range, fabsf(v[j]));
      dw[(size_t)j * kD] = __float2half_rn(v[j]);
    }
    tc::tmem_ld16(tq + Q2_TM_U, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      umax = fmaxf(umax, fabsf(v[j]));
      du[(size_t)j * kD] = v[j];
    }
  }
  if (!(range <= kF16Max)) report_range(status);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, o));
  if (lane == 0) misc[8 + warp] = umax;

  // 8. the scan's Q and K rows in fp16: exp(G) (.) q^ and exp(G_C - G) (.) k^ (both
  //    at most their unit-norm inputs), and the per-chunk factors
  {
    __half* qd = reinterpret_cast<__half*>(ws + L.qh) + (head * Tp + t0) * kD;
    __half* kd = reinterpret_cast<__half*>(ws + L.kh) + (head * Tp + t0) * kD;
    for (int i = tid; i < kC * 16; i += kThreads) {
      const int r = i >> 4, c8 = (i & 15) * 8;
      const uint4 uq = *reinterpret_cast<const uint4*>(Qt + r * LDT + c8);
      const uint4 uk = *reinterpret_cast<const uint4*>(Kt + r * LDT + c8);
      const uint32_t* pq = reinterpret_cast<const uint32_t*>(&uq);
      const uint32_t* pk = reinterpret_cast<const uint32_t*>(&uk);
      float gr[8], gc[8];
#pragma unroll
      for (int h4 = 0; h4 < 2; ++h4) {
        const float4 a4 = *reinterpret_cast<const float4*>(Gm + r * LDG + c8 + 4 * h4);
        const float4 b4 = *reinterpret_cast<const float4*>(Gm + (kC - 1) * LDG + c8 + 4 * h4);
        gr[4 * h4] = a4.x, gr[4 * h4 + 1] = a4.y, gr[4 * h4 + 2] = a4.z, gr[4 * h4 + 3] = a4.w;
        gc[4 * h4] = b4.x, gc[4 * h4 + 1] = b4.y, gc[4 * h4 + 2] = b4.z, gc[4 * h4 + 3] = b4.w;
      }
      const float sqr = sq[r], rkr = rk[r];
      uint4 oq, ok;
      uint32_t* wq = reinterpret_cast<uint32_t*>(&oq);
      uint32_t* wk = reinterpret_cast<uint32_t*>(&ok);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 qq = unpack2(pq[u]), kk = unpack2(pk[u]);
        wq[u] = pack2h(qq.x * sqr * __expf(gr[2 * u]), qq.y * sqr * __expf(gr[2 * u + 1]));
        wk[u] = pack2h(kk.x * rkr * __expf(gc[2 * u] - gr[2 * u]),
                       kk.y * rkr * __expf(gc[2 * u + 1] - gr[2 * u + 1]));
      }
      *reinterpret_cast<uint4*>(qd + (size_t)r * kD + c8) = oq;
      *reinterpret_cast<uint4*>(kd + (size_t)r * kD + c8) = ok;
    }
  }
  __syncthreads();
  if (tid < 128) {
    float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
    if (tid < kC) {
      sc[tid] = 1.f;
      sc[kC + tid] = tid < nv ? 1.f : 0.f;
    }
    sc[kScGC + tid] = __expf(Gm[(kC - 1) * LDG + tid]);
    if (tid < 4) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, misc[8 + w]);
      sc[kScMaxU + tid] = tid == 0 ? m : 0.f;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Q2_TM_COLS);
  }
}

template <typename TO>
cudaError_t launch_t(const ChunkArgs& a, bool gdn2, uint8_t* ws, const WsLayout& L,
                     cudaStream_t s) {
  const int Nc = (a.T + kC - 1) / kC;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  const int l2 = (a.flags & GDN_QK_L2NORM) ? 1 : 0;
  int* status = status_word();
  if (status == nullptr) return cudaErrorUnknown;
  cudaError_t e;
  if (gdn2) {
    if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
    Prep2Maps m;
    const CUtensorMapDataType g_dt =
        pre ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int g_es = pre ? 4 : 2, g_box = pre ? LDG : LDT;
    if (!make_map_bthd_rows(&m.k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, a.T, a.Hv, LDT) ||
        !make_map_bthd_rows(&m.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, a.T, a.Hv, LDT) ||
        !make_map_bthd_rows(&m.v, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, a.T, a.Hv, LDT) ||
        !make_map_bthd_rows(&m.ga, a.a, g_dt, g_es, a.B, a.T, a.Hv, g_box) ||
        !make_map_bthd_rows(&m.gb, a.b, g_dt, g_es, a.B, a.T, a.Hv, g_box) ||
        !make_map_bthd_rows(&m.gw, a.w, g_dt, g_es, a.B, a.T, a.Hv, g_box))
      return cudaErrorInvalidValue;
    auto prep = pre ? wy_prep2_kernel<true> : wy_prep2_kernel<false>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, Q2_BYTES);
    if (e != cudaSuccess) return e;
    prep<<<dim3(1, Nc, a.B * a.Hv), kThreads, Q2_BYTES, s>>>(
        m, a.A_log, a.dt_bias, a.T, a.Hv, a.scale, l2, ws, L, status, wait_fault().spin);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    e = launch_prep_tc(a, ws, status, s);
    if (e != cudaSuccess) return e;
  }
  return launch_scan_tc(a, ws, status, s);
}

}  // namespace

bool chunk_mma_supported(const ChunkArgs& a) {
  return a.dtype == GDN_BF16 && a.dk == kD && a.dv == kD && (long)a.B * a.Hv <= 65535 &&
         (long)a.B * a.Hk <= 65535 && ((long)a.T + kC - 1) / kC <= 65535;
}

size_t chunk_mma_workspace_bytes(int B, int T, int Hk, int Hv) {
  if (B <= 0 || T <= 0) return 0;
  return ws_layout(B, T, Hk, Hv).total;
}

cudaError_t launch_chunk_mma(const ChunkArgs& a, bool gdn2, void* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(a.B, a.T, a.Hk, a.Hv);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (a.flags & GDN_OUT_F32) return launch_t<float>(a, gdn2, w, L, s);
  return launch_t<bf16>(a, gdn2, w, L, s);
}

}  // namespace gdn
