// chunk_mma.cu -- bf16 chunkwise GDN forward (dk = dv = 128, chunk C = 64) on
// the tensor cores, in two kernels:
//
//  wy_prep_kernel  : one CTA per (chunk, value head), parallel over the whole
//      sequence; the CTAs of one GQA group are launched next to each other so
//      their shared K / Q tiles come from L2.  Forms the Gram matrices K K^T and
//      Q K^T (bf16 mma, fp32 accumulation) with the gates applied in registers:
//      the in-chunk prefix sums G_r of the log-decays, the strictly lower
//      L = diag(beta) (K^ K^^T o Gamma), X = (I + L)^-1 by blocked forward
//      substitution in fp32, W = X diag(beta gamma) K^, U = X diag(beta) V and
//      A_qk = tril(Q^ K^^T o Gamma) (diagonal included), written to the
//      workspace with the per-row factors of the second kernel.
//  state_scan_kernel : one CTA per (value head, 64-column half of d_v),
//      sequential over the chunks with the fp32 state slice held in mma
//      accumulator registers:  U~ = U - W S,  o = diag(gamma sq) Q S + A_qk U~,
//      S <- gamma_C S + K^T diag(rk gamma_C / gamma) U~.  The next chunk's tiles
//      are fetched with cp.async while the current one is computed.
//
// Precision: bf16 operands, fp32 accumulation and state.  Where one bf16
// rounding of an operand would cost more than the 2e-2 (max |err| / RMS)
// budget, the operand is carried as an unevaluated sum hi + lo of two bf16
// numbers (hi = rn(x), lo = rn(x - hi), about 16 significant bits) and the
// product takes one mma per term: X diag(beta) in U, U~ and A_qk in the
// output, U~ diag(fs) in the state update, and the state in Q S.  U is kept
// in fp32.  W S uses the state's hi part only.
//
// The algebra is the WY / UT chunk form of the delta rule ("Gated DeltaNet-2",
// section on the chunkwise algorithm; GDN is its scalar-decay special case):
// Gamma_rj = exp(G_r - G_j) only for j <= r, so every exponent is <= 0.
#include "common.cuh"
#include "launch.h"
#include "warp_mma.cuh"

namespace gdn {
namespace {

using namespace wm;
using bf16 = __nv_bfloat16;

constexpr int kC = 64;         // chunk length
constexpr int kD = 128;        // dk = dv
constexpr int kThreads = 256;  // 8 warps
constexpr int LDT = kD + 8;    // bf16 row stride of 128-wide tiles (272 B: ldmatrix conflict-free)
constexpr int LDH = 64 + 8;    // bf16 row stride of 64-wide tiles (144 B)
constexpr int LDF = 65;        // fp32 row stride of 64 x 64 matrices
constexpr int kScal = 132;     // floats per (head, chunk): fo[64], fs[64], gamma_C, pad

// ---------------------------------------------------------------- workspace
struct WsLayout {
  size_t w, u, ah, al, scal, total;
};
WsLayout ws_layout(int B, int T, int Hv) {
  const size_t Nc = ((size_t)T + kC - 1) / kC, Tp = Nc * kC, heads = (size_t)B * Hv;
  WsLayout L;
  L.w = 0;                                  // W        [B*Hv][Tp][128] bf16
  L.u = L.w + heads * Tp * kD * 2;          // U        [B*Hv][Tp][128] f32
  L.ah = L.u + heads * Tp * kD * 4;         // A_qk hi  [B*Hv][Tp][64]  bf16
  L.al = L.ah + heads * Tp * kC * 2;        // A_qk lo  [B*Hv][Tp][64]  bf16
  L.scal = L.al + heads * Tp * kC * 2;      // scalars  [B*Hv][Nc][132] f32
  L.total = L.scal + heads * Nc * kScal * 4;
  return L;
}

// x = hi + lo with hi = rn_bf16(x), lo = rn_bf16(x - hi), for a pair of values.
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack2(x, y);
  const float2 h = unpack2(hi);
  lo = pack2(x - h.x, y - h.y);
}

// ---------------------------------------------------------------- prep kernel
constexpr int LDX = 64 + 8;                  // f32 row stride of L and X (conflict-free float2)
constexpr int P_KT = 0;                      // K tile  [64][LDT] bf16 (key head)
constexpr int P_QT = P_KT + kC * LDT * 2;    // Q tile  (key head)
constexpr int P_VT = P_QT + kC * LDT * 2;    // V tile  (value head)
constexpr int P_L = P_VT + kC * LDT * 2;     // L [64][LDX] f32
constexpr int P_X = P_L + kC * LDX * 4;      // X = (I + L)^-1
constexpr int P_T = P_X + kC * LDX * 4;      // block products [3][16][17] f32
constexpr int P_VEC = P_T + 3 * 16 * 17 * 4; // rk, sq, G, beta, c1 [64] + misc
constexpr int P_BYTES = P_VEC + 6 * 64 * 4;
static_assert(2 * (P_BYTES + 1024) <= 228 * 1024, "two prep CTAs per SM");

template <bool PRE>
__global__ void __launch_bounds__(kThreads, 2)
wy_prep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
               const void* __restrict__ ga, const void* __restrict__ gb,
               const float* __restrict__ A_log, const float* __restrict__ dt_bias, int T, int Hk,
               int Hv, float scale, int l2, uint8_t* __restrict__ ws, WsLayout L) {
  extern __shared__ __align__(16) uint8_t sm[];
  bf16* Kt = reinterpret_cast<bf16*>(sm + P_KT);
  bf16* Qt = reinterpret_cast<bf16*>(sm + P_QT);
  bf16* Vt = reinterpret_cast<bf16*>(sm + P_VT);
  float* Lm = reinterpret_cast<float*>(sm + P_L);
  float* Xm = reinterpret_cast<float*>(sm + P_X);
  float* Tm = reinterpret_cast<float*>(sm + P_T);
  float* rk = reinterpret_cast<float*>(sm + P_VEC);
  float* sq = rk + 64;
  float* Gs = sq + 64;
  float* bet = Gs + 64;
  float* c1 = bet + 64;
  float* misc = c1 + 64;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int G = Hv / Hk;
  const int n = blockIdx.y, Nc = gridDim.y, Tp = Nc * kC;
  const int b = blockIdx.z / Hk, hk = blockIdx.z % Hk, hv = hk * G + blockIdx.x;
  const size_t head = (size_t)b * Hv + hv;
  const int t0 = n * kC, nv = min(kC, T - t0);

  // 1. raw K, Q tiles of the key head and the V tile of this value head (rows
  //    past the end of the sequence are zeros)
  for (int i = tid; i < 3 * kC * 16; i += kThreads) {
    const int which = i >> 10, r = (i >> 4) & 63, c16 = i & 15;
    const bool ok = r < nv;
    size_t off = 0;
    if (ok)
      off = which < 2 ? ((((size_t)b * T + t0 + r) * Hk + hk) * kD + c16 * 8)
                      : ((((size_t)b * T + t0 + r) * Hv + hv) * kD + c16 * 8);
    bf16* dst = (which == 0 ? Kt : (which == 1 ? Qt : Vt)) + r * LDT + c16 * 8;
    cp16(dst, (which == 0 ? k : (which == 1 ? q : v)) + off, ok ? 16 : 0);
  }
  cp_commit();

  // 2. gates (zero past the end of the sequence) and their in-chunk prefix sums,
  //    while the tiles land
  if (tid < kC) {
    float g = 0.f, be = 0.f;
    if (tid < nv) {
      const size_t idx = ((size_t)b * T + t0 + tid) * Hv + hv;
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
    if (tid == 31) misc[0] = g;
    Gs[tid] = g;
    bet[tid] = be;
  }
  cp_wait<0>();
  __syncthreads();
  if (tid >= 32 && tid < kC) Gs[tid] += misc[0];

  //    L2 norms: rk = 1 / |k|, sq = scale / |q| (two threads per row)
  {
    const int which = tid >> 7, r = (tid & 127) >> 1, h = tid & 1;
    const bf16* row = (which ? Qt : Kt) + r * LDT + h * 64;
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 64; c += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c);
      const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
      ss += f0.x * f0.x + f0.y * f0.y + f1.x * f1.x + f1.y * f1.y + f2.x * f2.x + f2.y * f2.y +
            f3.x * f3.x + f3.y * f3.y;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    if (h == 0) {
      const float inv = l2 ? rsqrtf(ss + 1e-6f) : 1.f;
      if (which) sq[r] = inv * scale;
      else rk[r] = inv;
    }
  }
  __syncthreads();
  if (tid < kC) c1[tid] = bet[tid] * __expf(Gs[tid]) * rk[tid];  // column factor of W

  // 3. Gram matrices on the tensor cores with the gates applied in registers:
  //    warps 0-3: L = strictly lower (beta_r rk_r rk_c e^(G_r - G_c) k_r.k_c) -> smem
  //    warps 4-7: A_qk = lower incl. diagonal (sq_r rk_c e^(G_r - G_c) q_r.k_c),
  //               stored to the workspace as bf16 hi + lo
  {
    const int mt = warp & 3;
    const bool isq = warp >= 4;
    const bf16* At = isq ? Qt : Kt;
    float acc[8][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4];
      ldsm_x4(a, At + (16 * mt + lrow_a(lane)) * LDT + 16 * ks + lcol_a(lane));
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        ldsm_x4(bb, Kt + (16 * np + lrow_b(lane)) * LDT + 16 * ks + lcol_b(lane));
        mma_bf16(acc[2 * np], a, bb[0], bb[1]);
        mma_bf16(acc[2 * np + 1], a, bb[2], bb[3]);
      }
    }
    const int ra = 16 * mt + g8, rb = ra + 8;
    const float Ga = Gs[ra], Gb = Gs[rb];
    const float fa = isq ? sq[ra] : bet[ra] * rk[ra];
    const float fb = isq ? sq[rb] : bet[rb] * rk[rb];
    bf16* ahg = reinterpret_cast<bf16*>(ws + L.ah) + (head * Tp + t0) * kC;
    bf16* alg = reinterpret_cast<bf16*>(ws + L.al) + (head * Tp + t0) * kC;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = 8 * nt + 2 * t4;
      const float k0 = rk[c] * __expf(fminf(Ga - Gs[c], 0.f));
      const float k1 = rk[c + 1] * __expf(fminf(Ga - Gs[c + 1], 0.f));
      const float k2 = rk[c] * __expf(fminf(Gb - Gs[c], 0.f));
      const float k3 = rk[c + 1] * __expf(fminf(Gb - Gs[c + 1], 0.f));
      if (!isq) {
        *reinterpret_cast<float2*>(Lm + ra * LDX + c) =
            make_float2(c < ra ? fa * k0 * acc[nt][0] : 0.f, c + 1 < ra ? fa * k1 * acc[nt][1] : 0.f);
        *reinterpret_cast<float2*>(Lm + rb * LDX + c) =
            make_float2(c < rb ? fb * k2 * acc[nt][2] : 0.f, c + 1 < rb ? fb * k3 * acc[nt][3] : 0.f);
      } else {
        uint32_t h, l;
        split2(c <= ra ? fa * k0 * acc[nt][0] : 0.f, c + 1 <= ra ? fa * k1 * acc[nt][1] : 0.f, h, l);
        *reinterpret_cast<uint32_t*>(ahg + ra * kC + c) = h;
        *reinterpret_cast<uint32_t*>(alg + ra * kC + c) = l;
        split2(c <= rb ? fb * k2 * acc[nt][2] : 0.f, c + 1 <= rb ? fb * k3 * acc[nt][3] : 0.f, h, l);
        *reinterpret_cast<uint32_t*>(ahg + rb * kC + c) = h;
        *reinterpret_cast<uint32_t*>(alg + rb * kC + c) = l;
      }
    }
  }
  __syncthreads();

  // 4. X = (I + L)^-1: the four 16 x 16 diagonal blocks by forward substitution
  //    (thread = one column of one block), zeros above the diagonal blocks
  if (tid < kC) {
    const int base = 16 * (tid >> 4), cc = tid & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float s = 0.f;
#pragma unroll
      for (int jj = 0; jj < r; ++jj) s = fmaf(Lm[(base + r) * LDX + base + jj], x[jj], s);
      x[r] = r == cc ? 1.f : -s;  // rows above cc come out as zero
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Xm[(base + r) * LDX + base + cc] = x[r];
  } else {
    for (int i = tid - kC; i < 6 * 256; i += kThreads - kC) {
      const int blk = i >> 8, e = i & 255;  // blocks (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
      const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
      const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      Xm[(16 * bi + (e >> 4)) * LDX + 16 * bj + (e & 15)] = 0.f;
    }
  }
  __syncthreads();
  //    then block row by block row: X_ij = -X_ii sum_{k=j}^{i-1} L_ik X_kj
  for (int bi = 1; bi < 4; ++bi) {
    for (int e = tid; e < bi * 256; e += kThreads) {
      const int bj = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
      for (int kb = bj; kb < bi; ++kb) {
#pragma unroll
        for (int qq = 0; qq < 16; ++qq)
          s = fmaf(Lm[(16 * bi + rr) * LDX + 16 * kb + qq], Xm[(16 * kb + qq) * LDX + 16 * bj + cc],
                   s);
      }
      Tm[(bj * 16 + rr) * 17 + cc] = s;
    }
    __syncthreads();
    for (int e = tid; e < bi * 256; e += kThreads) {
      const int bj = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float s = 0.f;
#pragma unroll
      for (int qq = 0; qq < 16; ++qq)
        s = fmaf(Xm[(16 * bi + rr) * LDX + 16 * bi + qq], Tm[(bj * 16 + qq) * 17 + cc], s);
      Xm[(16 * bi + rr) * LDX + 16 * bj + cc] = -s;
    }
    __syncthreads();
  }

  // 5. W = X diag(c1) K (bf16) and U = X diag(beta) V (fp32, X diag(beta) as bf16
  //    hi + lo); the A fragments are formed from X in registers.
  //    warp -> rows 16 (warp % 4), cols 64 (warp / 4)
  const int mt = warp & 3, nb = 64 * (warp >> 2);
  const int ra = 16 * mt + g8;
#pragma unroll 1
  for (int which = 0; which < 2; ++which) {
    float acc[8][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int ca = 16 * ks + 2 * t4;
      const float2 x00 = *reinterpret_cast<const float2*>(Xm + ra * LDX + ca);
      const float2 x10 = *reinterpret_cast<const float2*>(Xm + (ra + 8) * LDX + ca);
      const float2 x01 = *reinterpret_cast<const float2*>(Xm + ra * LDX + ca + 8);
      const float2 x11 = *reinterpret_cast<const float2*>(Xm + (ra + 8) * LDX + ca + 8);
      const float* f = which ? bet : c1;
      const float f0 = f[ca], f1 = f[ca + 1], f2 = f[ca + 8], f3 = f[ca + 9];
      uint32_t ah[4], al[4];
      split2(x00.x * f0, x00.y * f1, ah[0], al[0]);
      split2(x10.x * f0, x10.y * f1, ah[1], al[1]);
      split2(x01.x * f2, x01.y * f3, ah[2], al[2]);
      split2(x11.x * f2, x11.y * f3, ah[3], al[3]);
      const bf16* Bm = which ? Vt : Kt;
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        ldsm_x4_t(bb, Bm + (16 * ks + lrow_a(lane)) * LDT + nb + 16 * np + lcol_a(lane));
        mma_bf16(acc[2 * np], ah, bb[0], bb[1]);
        mma_bf16(acc[2 * np + 1], ah, bb[2], bb[3]);
        if (which) {
          mma_bf16(acc[2 * np], al, bb[0], bb[1]);
          mma_bf16(acc[2 * np + 1], al, bb[2], bb[3]);
        }
      }
    }
    if (which == 0) {
      bf16* dw = reinterpret_cast<bf16*>(ws + L.w) + (head * Tp + t0) * kD;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        *reinterpret_cast<uint32_t*>(dw + (size_t)ra * kD + c) = pack2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t*>(dw + (size_t)(ra + 8) * kD + c) = pack2(acc[nt][2], acc[nt][3]);
      }
    } else {
      float* du = reinterpret_cast<float*>(ws + L.u) + (head * Tp + t0) * kD;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        *reinterpret_cast<float2*>(du + (size_t)ra * kD + c) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(du + (size_t)(ra + 8) * kD + c) =
            make_float2(acc[nt][2], acc[nt][3]);
      }
    }
  }

  // 6. per-row factors of the scan: fo = gamma sq, fs = rk gamma_C / gamma, gamma_C
  if (tid < kC) {
    float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
    const float GC = Gs[kC - 1];
    sc[tid] = __expf(Gs[tid]) * sq[tid];
    sc[kC + tid] = tid < nv ? rk[tid] * __expf(GC - Gs[tid]) : 0.f;
    if (tid < 4) sc[2 * kC + tid] = tid == 0 ? __expf(GC) : 0.f;
  }
}

// ---------------------------------------------------------------- scan kernel
constexpr int LDU = 64 + 8;                 // f32 row stride of the U tile (conflict-free float2)
// double-buffered, fetched one chunk ahead
constexpr int S_W = 0;                      // W tile   [64][LDT] bf16
constexpr int S_Q = S_W + kC * LDT * 2;     // raw Q tile
constexpr int S_U = S_Q + kC * LDT * 2;     // U columns of this CTA [64][LDU] f32
constexpr int S_SC = S_U + kC * LDU * 4;    // scalars (132 f32)
constexpr int STAGE = S_SC + kScal * 4;
// single-buffered, fetched at the start of the chunk that uses them
constexpr int S_K = 2 * STAGE;              // raw K tile [64][LDT] bf16
constexpr int S_AH = S_K + kC * LDT * 2;    // A_qk hi [64][LDH] bf16
constexpr int S_AL = S_AH + kC * LDH * 2;   // A_qk lo
// on-chip operands
constexpr int S_SBH = S_AL + kC * LDH * 2;  // state slice, bf16 hi [128][LDH]
constexpr int S_SBL = S_SBH + kD * LDH * 2; // state slice, bf16 lo
constexpr int S_UTH = S_SBL + kD * LDH * 2; // U~ hi [64][LDH]
constexpr int S_UTL = S_UTH + kC * LDH * 2; // U~ lo
constexpr int S_USH = S_UTL + kC * LDH * 2; // U~ diag(fs) hi
constexpr int S_USL = S_USH + kC * LDH * 2; // U~ diag(fs) lo
constexpr int S_BYTES = S_USL + kC * LDH * 2;
static_assert(STAGE % 16 == 0, "stage buffers must stay 16-byte aligned");
static_assert(S_BYTES <= 227 * 1024, "shared memory of the scan kernel");

template <typename TO>
__device__ __forceinline__ void store2(TO* p, float x, float y);
template <>
__device__ __forceinline__ void store2<float>(float* p, float x, float y) {
  *reinterpret_cast<float2*>(p) = make_float2(x, y);
}
template <>
__device__ __forceinline__ void store2<bf16>(bf16* p, float x, float y) {
  *reinterpret_cast<uint32_t*>(p) = pack2(x, y);
}

template <typename TO>
__global__ void __launch_bounds__(kThreads, 1)
state_scan_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                  const uint8_t* __restrict__ ws, WsLayout L, const float* h0, int T, int Hk,
                  int Hv, TO* __restrict__ o, float* ht) {
  extern __shared__ __align__(16) uint8_t sm[];
  bf16* Kt = reinterpret_cast<bf16*>(sm + S_K);
  bf16* Ah = reinterpret_cast<bf16*>(sm + S_AH);
  bf16* Al = reinterpret_cast<bf16*>(sm + S_AL);
  bf16* Sbh = reinterpret_cast<bf16*>(sm + S_SBH);
  bf16* Sbl = reinterpret_cast<bf16*>(sm + S_SBL);
  bf16* Uth = reinterpret_cast<bf16*>(sm + S_UTH);
  bf16* Utl = reinterpret_cast<bf16*>(sm + S_UTL);
  bf16* Ush = reinterpret_cast<bf16*>(sm + S_USH);
  bf16* Usl = reinterpret_cast<bf16*>(sm + S_USL);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int c0 = 64 * blockIdx.x;
  const int head = blockIdx.y, b = head / Hv, hv = head % Hv, hk = hv / (Hv / Hk);
  const int Nc = (T + kC - 1) / kC, Tp = Nc * kC;
  const bf16* Wg = reinterpret_cast<const bf16*>(ws + L.w) + (size_t)head * Tp * kD;
  const float* Ug = reinterpret_cast<const float*>(ws + L.u) + (size_t)head * Tp * kD + c0;
  const bf16* Ahg = reinterpret_cast<const bf16*>(ws + L.ah) + (size_t)head * Tp * kC;
  const bf16* Alg = reinterpret_cast<const bf16*>(ws + L.al) + (size_t)head * Tp * kC;
  const float* Sg = reinterpret_cast<const float*>(ws + L.scal) + (size_t)head * Nc * kScal;

  // W, Q, U and the scalars of chunk n into stage n % 2
  auto issue_stage = [&](int n) {
    uint8_t* st = sm + (n & 1) * STAGE;
    const int t0 = n * kC, nv = min(kC, T - t0);
    for (int i = tid; i < kC * 16; i += kThreads) {
      const int r = i >> 4, c16 = i & 15;
      cp16(st + S_W + (r * LDT + c16 * 8) * 2, Wg + (size_t)(t0 + r) * kD + c16 * 8, 16);
      const bool ok = r < nv;
      const size_t off = ok ? ((((size_t)b * T + t0 + r) * Hk + hk) * kD + c16 * 8) : 0;
      cp16(st + S_Q + (r * LDT + c16 * 8) * 2, q + off, ok ? 16 : 0);
      cp16(st + S_U + (r * LDU + c16 * 4) * 4, Ug + (size_t)(t0 + r) * kD + c16 * 4, 16);
    }
    if (tid < kScal / 4) cp16(st + S_SC + tid * 16, Sg + (size_t)n * kScal + tid * 4, 16);
    cp_commit();
  };
  // K and A_qk of chunk n
  auto issue_ka = [&](int n) {
    const int t0 = n * kC, nv = min(kC, T - t0);
    for (int i = tid; i < kC * 16; i += kThreads) {
      const int r = i >> 4, c16 = i & 15;
      const bool ok = r < nv;
      const size_t off = ok ? ((((size_t)b * T + t0 + r) * Hk + hk) * kD + c16 * 8) : 0;
      cp16(Kt + r * LDT + c16 * 8, k + off, ok ? 16 : 0);
      if (c16 < 8) {
        cp16(Ah + r * LDH + c16 * 8, Ahg + (size_t)(t0 + r) * kC + c16 * 8, 16);
        cp16(Al + r * LDH + c16 * 8, Alg + (size_t)(t0 + r) * kC + c16 * 8, 16);
      }
    }
    cp_commit();
  };

  // state slice: warp w holds rows 16 w .. 16 w + 15, all 64 columns, as 8 C fragments
  float S[8][4];
  const int s0 = 16 * warp + g8;
  auto store_state_bf16 = [&]() {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = 8 * nt + 2 * t4;
      uint32_t h, l;
      split2(S[nt][0], S[nt][1], h, l);
      *reinterpret_cast<uint32_t*>(Sbh + s0 * LDH + c) = h;
      *reinterpret_cast<uint32_t*>(Sbl + s0 * LDH + c) = l;
      split2(S[nt][2], S[nt][3], h, l);
      *reinterpret_cast<uint32_t*>(Sbh + (s0 + 8) * LDH + c) = h;
      *reinterpret_cast<uint32_t*>(Sbl + (s0 + 8) * LDH + c) = l;
    }
  };
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    float2 x0 = make_float2(0.f, 0.f), x1 = x0;
    if (h0) {
      const float* src = h0 + ((size_t)head * kD + s0) * kD + c0 + 8 * nt + 2 * t4;
      x0 = *reinterpret_cast<const float2*>(src);
      x1 = *reinterpret_cast<const float2*>(src + 8 * kD);
    }
    S[nt][0] = x0.x; S[nt][1] = x0.y; S[nt][2] = x1.x; S[nt][3] = x1.y;
  }
  store_state_bf16();
  issue_stage(0);

  const int mt = warp & 3, nb = 32 * (warp >> 2);  // output tile of this warp: 16 rows x 32 cols
  const int r0 = 16 * mt + g8, r1 = r0 + 8;
  for (int n = 0; n < Nc; ++n) {
    cp_wait<0>();
    __syncthreads();  // stage n landed; the previous chunk's reads and state stores are done
    issue_ka(n);
    const bool more = n + 1 < Nc;
    if (more) issue_stage(n + 1);
    const uint8_t* st = sm + (n & 1) * STAGE;
    const bf16* Wt = reinterpret_cast<const bf16*>(st + S_W);
    const bf16* Qt = reinterpret_cast<const bf16*>(st + S_Q);
    const float* Uc = reinterpret_cast<const float*>(st + S_U);
    const float* sc = reinterpret_cast<const float*>(st + S_SC);
    const int t0 = n * kC;

    // P = W S_hi and OQ = Q (S_hi + S_lo) for this warp's tile
    float P[4][4] = {}, OQ[4][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t aw[4], aq[4];
      ldsm_x4(aw, Wt + (16 * mt + lrow_a(lane)) * LDT + 16 * ks + lcol_a(lane));
      ldsm_x4(aq, Qt + (16 * mt + lrow_a(lane)) * LDT + 16 * ks + lcol_a(lane));
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t bh[4], bl[4];
        const int so = (16 * ks + lrow_a(lane)) * LDH + nb + 16 * np + lcol_a(lane);
        ldsm_x4_t(bh, Sbh + so);
        ldsm_x4_t(bl, Sbl + so);
        mma_bf16(P[2 * np], aw, bh[0], bh[1]);
        mma_bf16(P[2 * np + 1], aw, bh[2], bh[3]);
        mma_bf16(OQ[2 * np], aq, bh[0], bh[1]);
        mma_bf16(OQ[2 * np + 1], aq, bh[2], bh[3]);
        mma_bf16(OQ[2 * np], aq, bl[0], bl[1]);
        mma_bf16(OQ[2 * np + 1], aq, bl[2], bl[3]);
      }
    }
    // U~ = U - P, and U~ diag(fs) for the state update, both as bf16 hi + lo
    {
      const float fs0 = sc[kC + r0], fs1 = sc[kC + r1];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        const float2 u0 = *reinterpret_cast<const float2*>(Uc + r0 * LDU + c);
        const float2 u1 = *reinterpret_cast<const float2*>(Uc + r1 * LDU + c);
        const float x0 = u0.x - P[nt][0], x1 = u0.y - P[nt][1];
        const float x2 = u1.x - P[nt][2], x3 = u1.y - P[nt][3];
        uint32_t h, l;
        split2(x0, x1, h, l);
        *reinterpret_cast<uint32_t*>(Uth + r0 * LDH + c) = h;
        *reinterpret_cast<uint32_t*>(Utl + r0 * LDH + c) = l;
        split2(x2, x3, h, l);
        *reinterpret_cast<uint32_t*>(Uth + r1 * LDH + c) = h;
        *reinterpret_cast<uint32_t*>(Utl + r1 * LDH + c) = l;
        split2(x0 * fs0, x1 * fs0, h, l);
        *reinterpret_cast<uint32_t*>(Ush + r0 * LDH + c) = h;
        *reinterpret_cast<uint32_t*>(Usl + r0 * LDH + c) = l;
        split2(x2 * fs1, x3 * fs1, h, l);
        *reinterpret_cast<uint32_t*>(Ush + r1 * LDH + c) = h;
        *reinterpret_cast<uint32_t*>(Usl + r1 * LDH + c) = l;
      }
    }
    if (more) cp_wait<1>();  // K and A_qk of chunk n (the next stage may still be in flight)
    else cp_wait<0>();
    __syncthreads();

    // o = fo (Q S) + (A_hi + A_lo)(U~_hi + U~_lo), the lo x lo term dropped
    {
      float OA[4][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t ah[4], al[4];
        ldsm_x4(ah, Ah + (16 * mt + lrow_a(lane)) * LDH + 16 * ks + lcol_a(lane));
        ldsm_x4(al, Al + (16 * mt + lrow_a(lane)) * LDH + 16 * ks + lcol_a(lane));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bh[4], bl[4];
          const int uo = (16 * ks + lrow_a(lane)) * LDH + nb + 16 * np + lcol_a(lane);
          ldsm_x4_t(bh, Uth + uo);
          ldsm_x4_t(bl, Utl + uo);
          mma_bf16(OA[2 * np], ah, bh[0], bh[1]);
          mma_bf16(OA[2 * np + 1], ah, bh[2], bh[3]);
          mma_bf16(OA[2 * np], ah, bl[0], bl[1]);
          mma_bf16(OA[2 * np + 1], ah, bl[2], bl[3]);
          mma_bf16(OA[2 * np], al, bh[0], bh[1]);
          mma_bf16(OA[2 * np + 1], al, bh[2], bh[3]);
        }
      }
      const float fo0 = sc[r0], fo1 = sc[r1];
      TO* o0 = o + (((size_t)b * T + t0 + r0) * Hv + hv) * kD + c0 + nb + 2 * t4;
      TO* o1 = o0 + (size_t)8 * Hv * kD;
      const bool w0 = t0 + r0 < T, w1 = t0 + r1 < T;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        if (w0) store2<TO>(o0 + 8 * nt, fo0 * OQ[nt][0] + OA[nt][0], fo0 * OQ[nt][1] + OA[nt][1]);
        if (w1) store2<TO>(o1 + 8 * nt, fo1 * OQ[nt][2] + OA[nt][2], fo1 * OQ[nt][3] + OA[nt][3]);
      }
    }

    // S <- gamma_C S + K^T (U~s_hi + U~s_lo)  (this warp's 16 state rows)
    {
      const float gC = sc[2 * kC];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) S[nt][e] *= gC;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4];
        ldsm_x4_t(a, Kt + (16 * ks + lrow_b(lane)) * LDT + 16 * warp + lcol_b(lane));
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bh[4], bl[4];
          const int uo = (16 * ks + lrow_a(lane)) * LDH + 16 * np + lcol_a(lane);
          ldsm_x4_t(bh, Ush + uo);
          ldsm_x4_t(bl, Usl + uo);
          mma_bf16(S[2 * np], a, bh[0], bh[1]);
          mma_bf16(S[2 * np + 1], a, bh[2], bh[3]);
          mma_bf16(S[2 * np], a, bl[0], bl[1]);
          mma_bf16(S[2 * np + 1], a, bl[2], bl[3]);
        }
      }
      store_state_bf16();
    }
  }

  if (ht != nullptr) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float* dst = ht + ((size_t)head * kD + s0) * kD + c0 + 8 * nt + 2 * t4;
      *reinterpret_cast<float2*>(dst) = make_float2(S[nt][0], S[nt][1]);
      *reinterpret_cast<float2*>(dst + 8 * kD) = make_float2(S[nt][2], S[nt][3]);
    }
  }
}

template <typename TO>
cudaError_t launch_t(const ChunkArgs& a, uint8_t* ws, const WsLayout& L, cudaStream_t s) {
  const int Nc = (a.T + kC - 1) / kC;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  auto prep = pre ? wy_prep_kernel<true> : wy_prep_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_scan_kernel<TO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           S_BYTES);
  if (e != cudaSuccess) return e;
  const bf16* q = static_cast<const bf16*>(a.q);
  const bf16* k = static_cast<const bf16*>(a.k);
  prep<<<dim3(a.Hv / a.Hk, Nc, a.B * a.Hk), kThreads, P_BYTES, s>>>(
      q, k, static_cast<const bf16*>(a.v), a.a, a.b, a.A_log, a.dt_bias, a.T, a.Hk, a.Hv,
      a.scale, (a.flags & GDN_QK_L2NORM) ? 1 : 0, ws, L);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  state_scan_kernel<TO><<<dim3(2, a.B * a.Hv), kThreads, S_BYTES, s>>>(
      q, k, ws, L, a.h0, a.T, a.Hk, a.Hv, static_cast<TO*>(a.o), a.ht);
  return cudaGetLastError();
}

}  // namespace

bool chunk_mma_supported(const ChunkArgs& a) {
  return a.dtype == GDN_BF16 && a.dk == kD && a.dv == kD && (long)a.B * a.Hv <= 65535 &&
         (long)a.B * a.Hk <= 65535 && ((long)a.T + kC - 1) / kC <= 65535;
}

size_t chunk_mma_workspace_bytes(int B, int T, int Hv) {
  if (B <= 0 || T <= 0) return 0;
  return ws_layout(B, T, Hv).total;
}

cudaError_t launch_chunk_mma(const ChunkArgs& a, void* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(a.B, a.T, a.Hv);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (a.flags & GDN_OUT_F32) return launch_t<float>(a, w, L, s);
  return launch_t<bf16>(a, w, L, s);
}

}  // namespace gdn
