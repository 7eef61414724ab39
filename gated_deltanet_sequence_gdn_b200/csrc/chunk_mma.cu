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
//      workspace with the per-row factors of the second kernel, together with
//      fp16 copies of the raw Q and K tiles.
//  state_scan_kernel : one CTA (8 warps) per (value head, 64-column half of
//      d_v), sequential over the chunks with the fp32 state slice held in mma
//      accumulator registers (16 x 64 per warp):  U~ = U - W S,  o = diag(gamma sq) Q S + A_qk U~,
//      S <- gamma_C S + K^T diag(rk gamma_C / gamma) U~.  All tiles of the next
//      chunk are fetched with cp.async while the current one is computed.
//
// The algebra is the WY / UT chunk form of the delta rule ("Gated DeltaNet-2",
// section on the chunkwise algorithm; GDN is its scalar-decay special case):
// Gamma_rj = exp(G_r - G_j) only for j <= r, so every exponent is <= 0.
//
// Precision: fp32 accumulation and state.  The prep's products take bf16
// operands (the inputs are bf16; X diag(beta) is carried as bf16 hi + lo, one
// mma per part, and U is stored in fp32).  The scan's products take fp16
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
#include "warp_mma.cuh"

namespace gdn {
namespace {

using namespace wm;
using bf16 = __nv_bfloat16;

constexpr int kC = 64;         // chunk length
constexpr int kD = 128;        // dk = dv
constexpr int kThreads = 256;  // 8 warps
constexpr int LDT = kD + 8;    // 16-bit row stride of 128-wide tiles (272 B: ldmatrix conflict-free)
constexpr int LDH = 64 + 8;    // 16-bit row stride of 64-wide tiles (144 B)
constexpr int kScal = 132;     // floats per (head, chunk): fo[64], fs[64], gamma_C, max|U|, pad
constexpr float kF16Max = 65000.f;  // largest magnitude accepted for an fp16 operand

// ---------------------------------------------------------------- workspace
struct WsLayout {
  size_t w, u, a, qh, kh, scal, total;
};
WsLayout ws_layout(int B, int T, int Hk, int Hv) {
  const size_t Nc = ((size_t)T + kC - 1) / kC, Tp = Nc * kC;
  const size_t hv = (size_t)B * Hv, hk = (size_t)B * Hk;
  WsLayout L;
  L.w = 0;                                  // W      [B*Hv][Tp][128] f16
  L.u = L.w + hv * Tp * kD * 2;             // U      [B*Hv][Tp][128] f32
  L.a = L.u + hv * Tp * kD * 4;             // A_qk   [B*Hv][Tp][64]  f16
  L.qh = L.a + hv * Tp * kC * 2;            // Q rows [B*Hk][Tp][128] f16 (row-scaled)
  L.kh = L.qh + hk * Tp * kD * 2;           // K rows [B*Hk][Tp][128] f16 (row-scaled)
  L.scal = L.kh + hk * Tp * kD * 2;         // scalars [B*Hv][Nc][132] f32
  L.total = L.scal + hv * Nc * kScal * 4;
  return L;
}

// x = hi + lo with hi = rn_bf16(x), lo = rn_bf16(x - hi), for a pair of values.
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack2(x, y);
  const float2 h = unpack2(hi);
  lo = pack2(x - h.x, y - h.y);
}

// A fragment (16 x 16, row-major) of an fp32 matrix M (row stride ld) at
// (r0, c0), as bf16 hi + lo parts.
__device__ __forceinline__ void frag_a_split(const float* M, int ld, int r0, int c0, int g8, int t4,
                                             uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  const float2 x00 = *reinterpret_cast<const float2*>(M + (r0 + g8) * ld + c0 + 2 * t4);
  const float2 x10 = *reinterpret_cast<const float2*>(M + (r0 + g8 + 8) * ld + c0 + 2 * t4);
  const float2 x01 = *reinterpret_cast<const float2*>(M + (r0 + g8) * ld + c0 + 2 * t4 + 8);
  const float2 x11 = *reinterpret_cast<const float2*>(M + (r0 + g8 + 8) * ld + c0 + 2 * t4 + 8);
  split2(x00.x, x00.y, hi[0], lo[0]);
  split2(x10.x, x10.y, hi[1], lo[1]);
  split2(x01.x, x01.y, hi[2], lo[2]);
  split2(x11.x, x11.y, hi[3], lo[3]);
}
// B fragment (16 x 8, k x n) of an fp32 matrix M (row = k) at (k0, n0), split.
__device__ __forceinline__ void frag_b_split(const float* M, int ld, int k0, int n0, int g8, int t4,
                                             uint32_t (&hi)[2], uint32_t (&lo)[2]) {
  const float* p = M + (k0 + 2 * t4) * ld + n0 + g8;
  split2(p[0], p[ld], hi[0], lo[0]);
  split2(p[8 * ld], p[9 * ld], hi[1], lo[1]);
}
// D += A B for split operands, the lo x lo term dropped (about 2^-16 relative).
__device__ __forceinline__ void mma_split3(float (&d)[4], const uint32_t (&ah)[4],
                                           const uint32_t (&al)[4], const uint32_t (&bh)[2],
                                           const uint32_t (&bl)[2]) {
  mma_bf16(d, ah, bh[0], bh[1]);
  mma_bf16(d, ah, bl[0], bl[1]);
  mma_bf16(d, al, bh[0], bh[1]);
}

// Exponent e with (max |row|) * 2^-e in [1, 2) (e = 0 for a zero row).
__device__ __forceinline__ int row_exponent(float m) { return m > 0.f ? ilogbf(m) : 0; }

// ---------------------------------------------------------------- prep kernel
constexpr int LDX = 64 + 8;                  // f32 row stride of L and X (conflict-free float2)
constexpr int P_KT = 0;                      // K tile  [64][LDT] bf16 (key head)
constexpr int P_QT = P_KT + kC * LDT * 2;    // Q tile  (key head)
constexpr int P_VT = P_QT + kC * LDT * 2;    // V tile  (value head)
constexpr int P_L = P_VT + kC * LDT * 2;     // L [64][LDX] f32
constexpr int P_X = P_L + kC * LDX * 4;      // X = (I + L)^-1
constexpr int LDB = 20;                      // f32 row stride of a 16 x 16 block product
constexpr int P_T = P_X + kC * LDX * 4;      // block products, one [16][LDB] f32 per warp 0-2
constexpr int P_VEC = P_T + 3 * 16 * LDB * 4; // rk, sq, G, beta, c1, 2^eq, 2^ek [64], misc
constexpr int P_BYTES = P_VEC + 8 * 64 * 4;
static_assert(2 * (P_BYTES + 1024) <= 228 * 1024, "two prep CTAs per SM");

template <bool PRE>
__global__ void __launch_bounds__(kThreads, 2)
wy_prep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
               const void* __restrict__ ga, const void* __restrict__ gb,
               const float* __restrict__ A_log, const float* __restrict__ dt_bias, int T, int Hk,
               int Hv, float scale, int l2, uint8_t* __restrict__ ws, WsLayout L, int* status) {
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
  float* pq = c1 + 64;   // 2^e of the stored Q row
  float* pk = pq + 64;   // 2^e of the stored K row
  float* misc = pk + 64; // [0] prefix carry, [8..15] per-warp max |U|

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int G = Hv / Hk;
  const int n = blockIdx.y, Nc = gridDim.y, Tp = Nc * kC;
  const int b = blockIdx.z / Hk, hk = blockIdx.z % Hk, hv = hk * G + blockIdx.x;
  const size_t head = (size_t)b * Hv + hv;
  const int t0 = n * kC, nv = min(kC, T - t0);
  float range = 0.f;  // largest magnitude this thread converted to fp16

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

  //    L2 norms: rk = 1 / |k|, sq = scale / |q|, and the row exponents of the
  //    fp16 copies (two threads per row)
  {
    const int which = tid >> 7, r = (tid & 127) >> 1, h = tid & 1;
    const bf16* row = (which ? Qt : Kt) + r * LDT + h * 8;  // 16-byte chunks h, h + 2, ...
    float ss = 0.f, mx = 0.f;
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c);
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
        sq[r] = inv * scale;
        pq[r] = up;
      } else {
        rk[r] = inv;
        pk[r] = up;
      }
    }
    // fp16 copies of the raw rows, row-scaled by 2^-e (written once per key head)
    if (blockIdx.x == 0) {
      __half* dst = reinterpret_cast<__half*>(ws + (which ? L.qh : L.kh)) +
                    ((size_t)blockIdx.z * Tp + t0 + r) * kD + h * 8;
#pragma unroll
      for (int c = 0; c < 128; c += 16) {
        const uint4 u = *reinterpret_cast<const uint4*>(row + c);
        const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
        uint4 o;
        o.x = pack2h(f0.x * down, f0.y * down);
        o.y = pack2h(f1.x * down, f1.y * down);
        o.z = pack2h(f2.x * down, f2.y * down);
        o.w = pack2h(f3.x * down, f3.y * down);
        *reinterpret_cast<uint4*>(dst + c) = o;
      }
    }
  }
  __syncthreads();
  if (tid < kC) c1[tid] = bet[tid] * __expf(Gs[tid]) * rk[tid];  // column factor of W

  // 3. Gram matrices on the tensor cores with the gates applied in registers:
  //    warps 0-3: L = strictly lower (beta_r rk_r rk_c e^(G_r - G_c) k_r.k_c) -> smem
  //    warps 4-7: A_qk = lower incl. diagonal (sq_r rk_c e^(G_r - G_c) q_r.k_c),
  //               stored to the workspace in fp16 (|A_qk| <= scale for unit rows)
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
    __half* ag = reinterpret_cast<__half*>(ws + L.a) + (head * Tp + t0) * kC;
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
        const float x0 = c <= ra ? fa * k0 * acc[nt][0] : 0.f;
        const float x1 = c + 1 <= ra ? fa * k1 * acc[nt][1] : 0.f;
        const float x2 = c <= rb ? fb * k2 * acc[nt][2] : 0.f;
        const float x3 = c + 1 <= rb ? fb * k3 * acc[nt][3] : 0.f;
        range = fmaxf(range, fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))));
        *reinterpret_cast<uint32_t*>(ag + ra * kC + c) = pack2h(x0, x1);
        *reinterpret_cast<uint32_t*>(ag + rb * kC + c) = pack2h(x2, x3);
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
  //    then block row by block row, on the tensor cores (fp32 operands as bf16
  //    hi + lo): warp j < i computes T = sum_{k=j}^{i-1} L_ik X_kj and
  //    X_ij = -X_ii T for its block (j = warp)
  for (int bi = 1; bi < 4; ++bi) {
    if (warp < bi) {
      const int bj = warp;
      float* Tw = Tm + warp * 16 * LDB;
      float t[2][4] = {};
      for (int kb = bj; kb < bi; ++kb) {
        uint32_t ah[4], al[4];
        frag_a_split(Lm, LDX, 16 * bi, 16 * kb, g8, t4, ah, al);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t bh[2], bl[2];
          frag_b_split(Xm, LDX, 16 * kb, 16 * bj + 8 * nt, g8, t4, bh, bl);
          mma_split3(t[nt], ah, al, bh, bl);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(Tw + g8 * LDB + 8 * nt + 2 * t4) = make_float2(t[nt][0], t[nt][1]);
        *reinterpret_cast<float2*>(Tw + (g8 + 8) * LDB + 8 * nt + 2 * t4) =
            make_float2(t[nt][2], t[nt][3]);
      }
      __syncwarp();
      float x[2][4] = {};
      uint32_t ah[4], al[4];
      frag_a_split(Xm, LDX, 16 * bi, 16 * bi, g8, t4, ah, al);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bh[2], bl[2];
        frag_b_split(Tw, LDB, 0, 8 * nt, g8, t4, bh, bl);
        mma_split3(x[nt], ah, al, bh, bl);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int c = 16 * bj + 8 * nt + 2 * t4;
        *reinterpret_cast<float2*>(Xm + (16 * bi + g8) * LDX + c) = make_float2(-x[nt][0], -x[nt][1]);
        *reinterpret_cast<float2*>(Xm + (16 * bi + g8 + 8) * LDX + c) =
            make_float2(-x[nt][2], -x[nt][3]);
      }
    }
    __syncthreads();
  }

  // 5. W = X diag(c1) K (stored in fp16) and U = X diag(beta) V (fp32, X diag(beta)
  //    as bf16 hi + lo); the A fragments are formed from X in registers.
  //    warp -> rows 16 (warp % 4), cols 64 (warp / 4)
  const int mt = warp & 3, nb = 64 * (warp >> 2);
  const int ra = 16 * mt + g8;
  float umax = 0.f;
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
      __half* dw = reinterpret_cast<__half*>(ws + L.w) + (head * Tp + t0) * kD;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        range = fmaxf(range, fmaxf(fmaxf(fabsf(acc[nt][0]), fabsf(acc[nt][1])),
                                   fmaxf(fabsf(acc[nt][2]), fabsf(acc[nt][3]))));
        *reinterpret_cast<uint32_t*>(dw + (size_t)ra * kD + c) = pack2h(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t*>(dw + (size_t)(ra + 8) * kD + c) =
            pack2h(acc[nt][2], acc[nt][3]);
      }
    } else {
      float* du = reinterpret_cast<float*>(ws + L.u) + (head * Tp + t0) * kD;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        umax = fmaxf(umax, fmaxf(fmaxf(fabsf(acc[nt][0]), fabsf(acc[nt][1])),
                                 fmaxf(fabsf(acc[nt][2]), fabsf(acc[nt][3]))));
        *reinterpret_cast<float2*>(du + (size_t)ra * kD + c) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(du + (size_t)(ra + 8) * kD + c) =
            make_float2(acc[nt][2], acc[nt][3]);
      }
    }
  }
  if (!(range <= kF16Max)) report_range(status);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, o));
  if (lane == 0) misc[8 + warp] = umax;
  __syncthreads();

  // 6. per-row factors of the scan: fo = gamma sq 2^eq, fs = rk 2^ek gamma_C / gamma,
  //    gamma_C, and the largest |U| of the chunk
  if (tid < kC) {
    float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
    const float GC = Gs[kC - 1];
    sc[tid] = __expf(Gs[tid]) * sq[tid] * pq[tid];
    sc[kC + tid] = tid < nv ? rk[tid] * pk[tid] * __expf(GC - Gs[tid]) : 0.f;
    if (tid < 4) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, misc[8 + w]);
      sc[2 * kC + tid] = tid == 0 ? __expf(GC) : (tid == 1 ? m : 0.f);
    }
  }
}

// ---------------------------------------------------------------- scan kernel
constexpr int kScanThreads = 256;           // 8 warps
constexpr int LDU = 64 + 8;                 // f32 row stride of the U tile (conflict-free float2)
// double-buffered, fetched one chunk ahead
constexpr int S_W = 0;                      // W tile     [64][LDT] f16
constexpr int S_Q = S_W + kC * LDT * 2;     // Q rows     [64][LDT] f16
constexpr int S_K = S_Q + kC * LDT * 2;     // K rows     [64][LDT] f16
constexpr int S_A = S_K + kC * LDT * 2;     // A_qk       [64][LDH] f16
constexpr int S_U = S_A + kC * LDH * 2;     // U columns of this CTA [64][LDU] f32
constexpr int S_SC = S_U + kC * LDU * 4;    // scalars (132 f32)
constexpr int STAGE = S_SC + kScal * 4;
// on-chip operands
constexpr int S_SB = 2 * STAGE;             // state slice (scaled) [128][LDH] f16
constexpr int S_UT = S_SB + kD * LDH * 2;   // U~ (scaled)          [64][LDH] f16
constexpr int S_US = S_UT + kC * LDH * 2;   // U~ diag(fs)          [64][LDH] f16
constexpr int S_RED = S_US + kC * LDH * 2;  // 8 floats for the CTA max
constexpr int S_BYTES = S_RED + 64;
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
__global__ void __launch_bounds__(kScanThreads, 1)
state_scan_kernel(const uint8_t* __restrict__ ws, WsLayout L, const float* h0, int T, int Hk,
                  int Hv, TO* __restrict__ o, float* ht, int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  __half* Sb = reinterpret_cast<__half*>(sm + S_SB);
  __half* Ut = reinterpret_cast<__half*>(sm + S_UT);
  __half* Us = reinterpret_cast<__half*>(sm + S_US);
  float* red = reinterpret_cast<float*>(sm + S_RED);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int c0 = 64 * blockIdx.x;
  const int head = blockIdx.y, b = head / Hv, hv = head % Hv, hk = hv / (Hv / Hk);
  const int Nc = (T + kC - 1) / kC, Tp = Nc * kC;
  const size_t khead = (size_t)b * Hk + hk;
  const __half* Wg = reinterpret_cast<const __half*>(ws + L.w) + (size_t)head * Tp * kD;
  const float* Ug = reinterpret_cast<const float*>(ws + L.u) + (size_t)head * Tp * kD + c0;
  const __half* Ag = reinterpret_cast<const __half*>(ws + L.a) + (size_t)head * Tp * kC;
  const __half* Qg = reinterpret_cast<const __half*>(ws + L.qh) + khead * Tp * kD;
  const __half* Kg = reinterpret_cast<const __half*>(ws + L.kh) + khead * Tp * kD;
  const float* Sg = reinterpret_cast<const float*>(ws + L.scal) + (size_t)head * Nc * kScal;

  // every tile of chunk n into stage n % 2
  auto issue_stage = [&](int n) {
    uint8_t* st = sm + (n & 1) * STAGE;
    const size_t r0 = (size_t)n * kC;
    for (int i = tid; i < kC * 16; i += kScanThreads) {
      const int r = i >> 4, c16 = i & 15;
      cp16(st + S_W + (r * LDT + c16 * 8) * 2, Wg + (r0 + r) * kD + c16 * 8, 16);
      cp16(st + S_Q + (r * LDT + c16 * 8) * 2, Qg + (r0 + r) * kD + c16 * 8, 16);
      cp16(st + S_K + (r * LDT + c16 * 8) * 2, Kg + (r0 + r) * kD + c16 * 8, 16);
      cp16(st + S_U + (r * LDU + c16 * 4) * 4, Ug + (r0 + r) * kD + c16 * 4, 16);
      if (c16 < 8) cp16(st + S_A + (r * LDH + c16 * 8) * 2, Ag + (r0 + r) * kC + c16 * 8, 16);
    }
    if (tid < kScal / 4) cp16(st + S_SC + tid * 16, Sg + (size_t)n * kScal + tid * 4, 16);
    cp_commit();
  };
  issue_stage(0);

  // state slice: warp w holds rows 16 w .. + 15 and all 64 columns of the CTA's
  // 128 x 64 slice, as 8 C fragments
  const int sr = 16 * warp + g8;
  float S[8][4];
  float mx = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    float2 x0 = make_float2(0.f, 0.f), x1 = x0;
    if (h0) {
      const float* src = h0 + ((size_t)head * kD + sr) * kD + c0 + 8 * nt + 2 * t4;
      x0 = *reinterpret_cast<const float2*>(src);
      x1 = *reinterpret_cast<const float2*>(src + 8 * kD);
    }
    S[nt][0] = x0.x; S[nt][1] = x0.y; S[nt][2] = x1.x; S[nt][3] = x1.y;
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x0.x), fabsf(x0.y)), fmaxf(fabsf(x1.x), fabsf(x1.y))));
  }
  // sigma = 2^-e: the largest |U| of the head and |h0| of this slice land below 2^8
  for (int n = tid; n < Nc; n += kScanThreads) mx = fmaxf(mx, Sg[(size_t)n * kScal + 2 * kC + 1]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  const int e = mx > 0.f ? min(max(ilogbf(mx) - 7, -100), 100) : 0;
  const float sigma = ldexpf(1.f, -e), inv_sigma = ldexpf(1.f, e);
  float range = 0.f;

  auto store_state = [&]() {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = 8 * nt + 2 * t4;
      range = fmaxf(range, fmaxf(fmaxf(fabsf(S[nt][0]), fabsf(S[nt][1])),
                                 fmaxf(fabsf(S[nt][2]), fabsf(S[nt][3]))));
      *reinterpret_cast<uint32_t*>(Sb + sr * LDH + c) = pack2h(S[nt][0], S[nt][1]);
      *reinterpret_cast<uint32_t*>(Sb + (sr + 8) * LDH + c) = pack2h(S[nt][2], S[nt][3]);
    }
  };
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) S[nt][i] *= sigma;
  store_state();

  // output tile of this warp: rows 16 (w % 4) .. + 15, columns 32 (w / 4) .. + 31
  const int mt = warp & 3, nb = 32 * (warp >> 2);
  const int r0 = 16 * mt + g8, r1 = r0 + 8;
  for (int n = 0; n < Nc; ++n) {
    cp_wait<0>();
    __syncthreads();  // chunk n landed; the previous chunk's reads and state stores are done
    if (n + 1 < Nc) issue_stage(n + 1);
    const uint8_t* st = sm + (n & 1) * STAGE;
    const __half* Wt = reinterpret_cast<const __half*>(st + S_W);
    const __half* Qt = reinterpret_cast<const __half*>(st + S_Q);
    const __half* Kt = reinterpret_cast<const __half*>(st + S_K);
    const __half* At = reinterpret_cast<const __half*>(st + S_A);
    const float* Uc = reinterpret_cast<const float*>(st + S_U);
    const float* sc = reinterpret_cast<const float*>(st + S_SC);
    const int t0 = n * kC;

    // P = W S and OQ = Q S for this warp's tile (S scaled by sigma)
    float P[4][4] = {}, OQ[4][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t aw[4], aq[4];
      ldsm_x4(aw, Wt + (16 * mt + lrow_a(lane)) * LDT + 16 * ks + lcol_a(lane));
      ldsm_x4(aq, Qt + (16 * mt + lrow_a(lane)) * LDT + 16 * ks + lcol_a(lane));
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t bb[4];
        ldsm_x4_t(bb, Sb + (16 * ks + lrow_a(lane)) * LDH + nb + 16 * np + lcol_a(lane));
        mma_f16(P[2 * np], aw, bb[0], bb[1]);
        mma_f16(P[2 * np + 1], aw, bb[2], bb[3]);
        mma_f16(OQ[2 * np], aq, bb[0], bb[1]);
        mma_f16(OQ[2 * np + 1], aq, bb[2], bb[3]);
      }
    }
    // U~ = sigma U - P, and U~ diag(fs) for the state update, in fp16
    {
      const float fs0 = sc[kC + r0], fs1 = sc[kC + r1];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int c = nb + 8 * nt + 2 * t4;
        const float2 u0 = *reinterpret_cast<const float2*>(Uc + r0 * LDU + c);
        const float2 u1 = *reinterpret_cast<const float2*>(Uc + r1 * LDU + c);
        const float x0 = fmaf(sigma, u0.x, -P[nt][0]), x1 = fmaf(sigma, u0.y, -P[nt][1]);
        const float x2 = fmaf(sigma, u1.x, -P[nt][2]), x3 = fmaf(sigma, u1.y, -P[nt][3]);
        range = fmaxf(range, fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))));
        *reinterpret_cast<uint32_t*>(Ut + r0 * LDH + c) = pack2h(x0, x1);
        *reinterpret_cast<uint32_t*>(Ut + r1 * LDH + c) = pack2h(x2, x3);
        *reinterpret_cast<uint32_t*>(Us + r0 * LDH + c) = pack2h(x0 * fs0, x1 * fs0);
        *reinterpret_cast<uint32_t*>(Us + r1 * LDH + c) = pack2h(x2 * fs1, x3 * fs1);
      }
    }
    __syncthreads();

    // o = (fo (Q S) + A_qk U~) / sigma
    {
      float OA[4][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, At + (16 * mt + lrow_a(lane)) * LDH + 16 * ks + lcol_a(lane));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bb[4];
          ldsm_x4_t(bb, Ut + (16 * ks + lrow_a(lane)) * LDH + nb + 16 * np + lcol_a(lane));
          mma_f16(OA[2 * np], a, bb[0], bb[1]);
          mma_f16(OA[2 * np + 1], a, bb[2], bb[3]);
        }
      }
      const float fo0 = sc[r0], fo1 = sc[r1];
      TO* o0 = o + (((size_t)b * T + t0 + r0) * Hv + hv) * kD + c0 + nb + 2 * t4;
      TO* o1 = o0 + (size_t)8 * Hv * kD;
      const bool w0 = t0 + r0 < T, w1 = t0 + r1 < T;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        if (w0)
          store2<TO>(o0 + 8 * nt, (fo0 * OQ[nt][0] + OA[nt][0]) * inv_sigma,
                     (fo0 * OQ[nt][1] + OA[nt][1]) * inv_sigma);
        if (w1)
          store2<TO>(o1 + 8 * nt, (fo1 * OQ[nt][2] + OA[nt][2]) * inv_sigma,
                     (fo1 * OQ[nt][3] + OA[nt][3]) * inv_sigma);
      }
    }

    // S <- gamma_C S + K^T U~s  (this warp's 16 state rows)
    {
      const float gC = sc[2 * kC];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) S[nt][i] *= gC;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4];
        ldsm_x4_t(a, Kt + (16 * ks + lrow_b(lane)) * LDT + 16 * warp + lcol_b(lane));
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bb[4];
          ldsm_x4_t(bb, Us + (16 * ks + lrow_a(lane)) * LDH + 16 * np + lcol_a(lane));
          mma_f16(S[2 * np], a, bb[0], bb[1]);
          mma_f16(S[2 * np + 1], a, bb[2], bb[3]);
        }
      }
      store_state();
    }
  }
  if (!(range <= kF16Max)) report_range(status);

  if (ht != nullptr) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float* dst = ht + ((size_t)head * kD + sr) * kD + c0 + 8 * nt + 2 * t4;
      *reinterpret_cast<float2*>(dst) = make_float2(S[nt][0] * inv_sigma, S[nt][1] * inv_sigma);
      *reinterpret_cast<float2*>(dst + 8 * kD) =
          make_float2(S[nt][2] * inv_sigma, S[nt][3] * inv_sigma);
    }
  }
}

template <typename TO>
cudaError_t launch_t(const ChunkArgs& a, uint8_t* ws, const WsLayout& L, cudaStream_t s) {
  const int Nc = (a.T + kC - 1) / kC;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  int* status = status_word();
  if (status == nullptr) return cudaErrorUnknown;
  auto prep = pre ? wy_prep_kernel<true> : wy_prep_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_scan_kernel<TO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           S_BYTES);
  if (e != cudaSuccess) return e;
  prep<<<dim3(a.Hv / a.Hk, Nc, a.B * a.Hk), kThreads, P_BYTES, s>>>(
      static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
      static_cast<const bf16*>(a.v), a.a, a.b, a.A_log, a.dt_bias, a.T, a.Hk, a.Hv, a.scale,
      (a.flags & GDN_QK_L2NORM) ? 1 : 0, ws, L, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  state_scan_kernel<TO><<<dim3(2, a.B * a.Hv), kScanThreads, S_BYTES, s>>>(
      ws, L, a.h0, a.T, a.Hk, a.Hv, static_cast<TO*>(a.o), a.ht, status);
  return cudaGetLastError();
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

cudaError_t launch_chunk_mma(const ChunkArgs& a, void* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(a.B, a.T, a.Hk, a.Hv);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (a.flags & GDN_OUT_F32) return launch_t<float>(a, w, L, s);
  return launch_t<bf16>(a, w, L, s);
}

}  // namespace gdn
