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
constexpr int kScal = 260;     // floats per (head, chunk): fo[64], fs[64], gamma_C[128] (per state
                               // row), max|U|, pad
constexpr int kScGC = 2 * 64;  // offset of gamma_C in the scalar block
constexpr int kScMaxU = kScGC + 128;
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
  L.scal = L.kh + hk * Tp * kD * 2;         // scalars [B*Hv][Nc][260] f32
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

// X = (I + L)^-1 for a strictly lower 64 x 64 fp32 L (row stride LDX) in shared
// memory, by the whole CTA: the four 16 x 16 diagonal blocks by forward
// substitution (thread = one column of one block), then block row by block row
// on the tensor cores with the fp32 operands as bf16 hi + lo: warp j < i
// computes T = sum_{k=j}^{i-1} L_ik X_kj and X_ij = -X_ii T.  Ends with a barrier.
__device__ void invert_unit_lower(const float* Lm, float* Xm, float* Tm, int tid, int warp, int g8,
                                  int t4) {
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
}

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

  // 4. X = (I + L)^-1
  invert_unit_lower(Lm, Xm, Tm, tid, warp, g8, t4);

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
  //    gamma_C for every state row, and the largest |U| of the chunk
  if (tid < 128) {
    float* sc = reinterpret_cast<float*>(ws + L.scal) + (head * Nc + n) * kScal;
    const float GC = Gs[kC - 1];
    if (tid < kC) {
      sc[tid] = __expf(Gs[tid]) * sq[tid] * pq[tid];
      sc[kC + tid] = tid < nv ? rk[tid] * pk[tid] * __expf(GC - Gs[tid]) : 0.f;
    }
    sc[kScGC + tid] = __expf(GC);  // one decay for every state row
    if (tid < 4) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, misc[8 + w]);
      sc[kScMaxU + tid] = tid == 0 ? m : 0.f;
    }
  }
}

// ---------------------------------------------------------------- GDN-2 prep kernel
// Gated DeltaNet-2: per-channel decay d_t = exp(g_t) (g_t in R^dk), erase
// direction e_t = b_t (.) k^_t, written value z_t = w_t (.) v_t.  With G the
// in-chunk prefix sum of g (per channel) the chunk form is
//   L_ji   = sum_c e_jc k^_ic exp(G_jc - G_ic)       (i < j)
//   A_tj   = sum_c q^_tc k^_jc exp(G_tc - G_jc)      (j <= t)
//   X = (I + L)^-1,  W = X (exp(G) (.) E),  U = X Z
//   o = (exp(G) (.) Q^) S + A (U - W S),   S <- diag(exp(G_C)) S + K_tail^T (U - W S)
// with K_tail rows exp(G_C - G_j) (.) k^_j ("Gated DeltaNet-2", 通道级衰减的吸收技巧
// and WY 形式).  The exponents differ per channel, so the 16 x 16 diagonal blocks
// of L and A are summed element by element, and each off-diagonal block row I is
// a product of operands scaled about its first row r = 16 I:
//   L_ji = sum_c [e_jc exp(G_jc - G_rc)] [k^_ic exp(G_rc - G_ic)]   (i < r <= j)
// where both exponents are <= 0, so every operand stays within its input's size.
constexpr int LDG = kD + 4;                    // f32 row stride of [64][128] channel tiles
constexpr int Q2_KT = 0;                       // raw K tile [64][LDT] bf16
constexpr int Q2_QT = Q2_KT + kC * LDT * 2;    // raw Q tile
constexpr int Q2_ZH = Q2_QT + kC * LDT * 2;    // raw V tile, then z = w (.) v (bf16 hi part)
constexpr int Q2_ZL = Q2_ZH + kC * LDT * 2;    // z lo part
constexpr int Q2_G = Q2_ZL + kC * LDT * 2;     // G [64][LDG] f32 (first: g, or the raw g tile)
constexpr int Q2_E = Q2_G + kC * LDG * 4;      // e [64][LDG] f32 (first: the raw b tile)
constexpr int Q2_L = Q2_E + kC * LDG * 4;      // L [64][LDX] f32
constexpr int Q2_X = Q2_L + kC * LDX * 4;      // A staging (f32), then X
constexpr int Q2_T = Q2_X + kC * LDX * 4;      // block products
constexpr int Q2_OP = Q2_T + 3 * 16 * LDB * 4; // raw gate tiles, then fp16 operands, then E-bar
constexpr int Q2_OPB = 192 * LDT * 2;
constexpr int Q2_VEC = Q2_OP + Q2_OPB;         // rk, sq [64], carry [128], misc [64]
constexpr int Q2_BYTES = Q2_VEC + 320 * 4;
static_assert(Q2_BYTES <= 227 * 1024, "shared memory of the GDN-2 prep kernel");
static_assert(kC * LDG * 4 <= Q2_OPB, "raw float32 w tile fits the operand scratch");

template <bool PRE>
__global__ void __launch_bounds__(kThreads, 1)
wy_prep2_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const void* __restrict__ ga, const void* __restrict__ gb,
                const void* __restrict__ gw, const float* __restrict__ A_log,
                const float* __restrict__ dt_bias, int T, int H, float scale, int l2,
                uint8_t* __restrict__ ws, WsLayout L, int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  bf16* Kt = reinterpret_cast<bf16*>(sm + Q2_KT);
  bf16* Qt = reinterpret_cast<bf16*>(sm + Q2_QT);
  bf16* Zh = reinterpret_cast<bf16*>(sm + Q2_ZH);
  bf16* Zl = reinterpret_cast<bf16*>(sm + Q2_ZL);
  float* Gm = reinterpret_cast<float*>(sm + Q2_G);
  float* Em = reinterpret_cast<float*>(sm + Q2_E);
  float* Lm = reinterpret_cast<float*>(sm + Q2_L);
  float* Xm = reinterpret_cast<float*>(sm + Q2_X);
  float* Tm = reinterpret_cast<float*>(sm + Q2_T);
  uint8_t* op = sm + Q2_OP;
  float* rk = reinterpret_cast<float*>(sm + Q2_VEC);
  float* sq = rk + 64;
  float* carry = sq + 64;
  float* misc = carry + 128;  // [8..15] per-warp max |U|

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int n = blockIdx.y, Nc = gridDim.y, Tp = Nc * kC;
  const int b = blockIdx.z / H, h = blockIdx.z % H;
  const size_t head = blockIdx.z;  // one key head per value head
  const int t0 = n * kC, nv = min(kC, T - t0);
  float range = 0.f;

  // 1. raw q, k, v tiles and the gate tiles (rows past the end of the sequence are zeros)
  for (int i = tid; i < 3 * kC * 16; i += kThreads) {
    const int which = i >> 10, r = (i >> 4) & 63, c16 = i & 15;
    const bool ok = r < nv;
    const size_t off = ok ? ((((size_t)b * T + t0 + r) * H + h) * kD + c16 * 8) : 0;
    bf16* dst = (which == 0 ? Kt : (which == 1 ? Qt : Zh)) + r * LDT + c16 * 8;
    cp16(dst, (which == 0 ? k : (which == 1 ? q : v)) + off, ok ? 16 : 0);
    if (!PRE) {  // a, b, w logits in bf16
      const bf16* src = reinterpret_cast<const bf16*>(which == 0 ? ga : (which == 1 ? gb : gw));
      cp16(reinterpret_cast<bf16*>(op + which * kC * LDT * 2) + r * LDT + c16 * 8, src + off,
           ok ? 16 : 0);
    }
  }
  if (PRE) {  // g, b, w values in float32
    for (int i = tid; i < 3 * kC * 32; i += kThreads) {
      const int which = i / (kC * 32), r = (i >> 5) & 63, c32 = i & 31;
      const bool ok = r < nv;
      const size_t off = ok ? ((((size_t)b * T + t0 + r) * H + h) * kD + c32 * 4) : 0;
      const float* src = reinterpret_cast<const float*>(which == 0 ? ga : (which == 1 ? gb : gw));
      float* dst = (which == 0 ? Gm : (which == 1 ? Em : reinterpret_cast<float*>(op))) + r * LDG;
      cp16(dst + c32 * 4, src + off, ok ? 16 : 0);
    }
  }
  cp_commit();
  for (int i = tid; i < kC * LDX; i += kThreads) Xm[i] = 0.f;  // A staging starts at zero
  cp_wait<0>();
  __syncthreads();

  // 2. L2 norms: rk = 1 / |k|, sq = scale / |q| (two threads per row)
  {
    const int which = tid >> 7, r = (tid & 127) >> 1, hh = tid & 1;
    const bf16* row = (which ? Qt : Kt) + r * LDT + hh * 8;
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c);
      const float2 f0 = unpack2(u.x), f1 = unpack2(u.y), f2 = unpack2(u.z), f3 = unpack2(u.w);
      ss += f0.x * f0.x + f0.y * f0.y + f1.x * f1.x + f1.y * f1.y + f2.x * f2.x + f2.y * f2.y +
            f3.x * f3.x + f3.y * f3.y;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    if (hh == 0) {
      const float inv = l2 ? rsqrtf(ss + 1e-6f) : 1.f;
      if (which) sq[r] = inv * scale;
      else rk[r] = inv;
    }
  }
  __syncthreads();

  // 3. per (token, channel): g, the in-chunk prefix sums G (two threads per channel,
  //    32 tokens each), e = b (.) k^ and z = w (.) v (as bf16 hi + lo)
  const int ch = tid & 127, half = tid >> 7;
  {
    float nal = 0.f, dtb = 0.f;
    if (!PRE) {
      nal = -expf(A_log[(size_t)h * kD + ch]);
      dtb = dt_bias[(size_t)h * kD + ch];
    }
    const bf16* at = reinterpret_cast<const bf16*>(op);
    const bf16* bt = at + kC * LDT;
    const bf16* wt = bt + kC * LDT;
    const float* wf = reinterpret_cast<const float*>(op);
    float run = 0.f;
    for (int tt = 0; tt < 32; ++tt) {
      const int r = 32 * half + tt;
      float g, bv, wv;
      if (PRE) {
        g = Gm[r * LDG + ch];
        bv = Em[r * LDG + ch];
        wv = wf[r * LDG + ch];
      } else {
        g = r < nv ? nal * softplus_f(__bfloat162float(at[r * LDT + ch]) + dtb) : 0.f;
        bv = sigmoid_f(__bfloat162float(bt[r * LDT + ch]));
        wv = sigmoid_f(__bfloat162float(wt[r * LDT + ch]));
      }
      run += g;
      Gm[r * LDG + ch] = run;
      Em[r * LDG + ch] = bv * __bfloat162float(Kt[r * LDT + ch]) * rk[r];
      const float z = wv * __bfloat162float(Zh[r * LDT + ch]);
      const bf16 zh = __float2bfloat16_rn(z);
      Zh[r * LDT + ch] = zh;
      Zl[r * LDT + ch] = __float2bfloat16_rn(z - __bfloat162float(zh));
    }
    if (half == 0) carry[ch] = run;
  }
  __syncthreads();
  if (half == 1)
    for (int r = 32; r < kC; ++r) Gm[r * LDG + ch] += carry[ch];
  __syncthreads();

  // 4. diagonal 16 x 16 blocks of L and A, element by element: warp per (j, i)
  //    pair, lanes over channels (4 each); exp(G_j - G_i) <= 1 for i <= j
  for (int p = warp; p < 4 * 136; p += 8) {
    const int blk = p / 136;
    int rem = p - blk * 136, jj = 0;
    while (rem > jj) {
      rem -= jj + 1;
      ++jj;
    }
    const int j = 16 * blk + jj, i = 16 * blk + rem;  // i <= j
    const float4 gj = *reinterpret_cast<const float4*>(Gm + j * LDG + 4 * lane);
    const float4 gi = *reinterpret_cast<const float4*>(Gm + i * LDG + 4 * lane);
    const float4 ej = *reinterpret_cast<const float4*>(Em + j * LDG + 4 * lane);
    const uint2 qj = *reinterpret_cast<const uint2*>(Qt + j * LDT + 4 * lane);
    const uint2 ki = *reinterpret_cast<const uint2*>(Kt + i * LDT + 4 * lane);
    const float2 q01 = unpack2(qj.x), q23 = unpack2(qj.y);
    const float2 k01 = unpack2(ki.x), k23 = unpack2(ki.y);
    const float x0 = __expf(gj.x - gi.x) * k01.x, x1 = __expf(gj.y - gi.y) * k01.y;
    const float x2 = __expf(gj.z - gi.z) * k23.x, x3 = __expf(gj.w - gi.w) * k23.y;
    float sl = ej.x * x0 + ej.y * x1 + ej.z * x2 + ej.w * x3;
    float sa = q01.x * x0 + q01.y * x1 + q23.x * x2 + q23.y * x3;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sl += __shfl_xor_sync(0xffffffffu, sl, o);
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
    }
    if (lane == 0) {
      Lm[j * LDX + i] = i < j ? sl * rk[i] : 0.f;
      Xm[j * LDX + i] = sa * sq[j] * rk[i];
    }
  }

  // 5. off-diagonal blocks on the tensor cores: fp16 operands scaled about the
  //    reference row r = 16 I of block row I (I = 1..3).  Rows of the operand
  //    scratch: [0,48) e rows of blocks 1-3, [48,96) q^ rows, [96,192) k^ rows
  //    0..16 I - 1 for I = 1, 2, 3 (at 96, 112, 144).
  __half* Op = reinterpret_cast<__half*>(op);
  for (int e = tid; e < 192 * kD; e += kThreads) {
    const int row = e >> 7, c = e & 127;
    float val;
    if (row < 96) {
      const int I = 1 + ((row % 48) >> 4), j = 16 * I + (row & 15);
      const float sc = __expf(Gm[j * LDG + c] - Gm[16 * I * LDG + c]);
      val = row < 48 ? Em[j * LDG + c] * sc : __bfloat162float(Qt[j * LDT + c]) * sq[j] * sc;
    } else {
      const int kr = row - 96;
      const int I = kr < 16 ? 1 : (kr < 48 ? 2 : 3);
      const int i = kr - (I == 1 ? 0 : (I == 2 ? 16 : 48));
      val = __bfloat162float(Kt[i * LDT + c]) * rk[i] *
            __expf(Gm[16 * I * LDG + c] - Gm[i * LDG + c]);
    }
    Op[row * LDT + c] = __float2half_rn(val);
  }
  __syncthreads();
  //    tasks (matrix, I, column pair np < I): 6 for L, 6 for A
  for (int task = warp; task < 12; task += 8) {
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

  // 6. X = (I + L)^-1
  invert_unit_lower(Lm, Xm, Tm, tid, warp, g8, t4);

  // 7. E-bar = exp(G) (.) e in bf16 (the B operand of W), in the operand scratch
  bf16* Eb = reinterpret_cast<bf16*>(op);
  for (int e = tid; e < kC * kD; e += kThreads) {
    const int r = e >> 7, c = e & 127;
    Eb[r * LDT + c] = __float2bfloat16_rn(__expf(Gm[r * LDG + c]) * Em[r * LDG + c]);
  }
  __syncthreads();

  //    W = X E-bar (fp16 out) and U = X Z (fp32 out, X and Z both as hi + lo);
  //    warp -> rows 16 (warp % 4), cols 64 (warp / 4)
  const int mt = warp & 3, nb = 64 * (warp >> 2);
  const int ra = 16 * mt + g8;
  float umax = 0.f;
#pragma unroll 1
  for (int which = 0; which < 2; ++which) {
    float acc[8][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t ah[4], al[4];
      frag_a_split(Xm, LDX, 16 * mt, 16 * ks, g8, t4, ah, al);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int bo = (16 * ks + lrow_a(lane)) * LDT + nb + 16 * np + lcol_a(lane);
        uint32_t bh[4];
        ldsm_x4_t(bh, (which ? Zh : Eb) + bo);
        mma_bf16(acc[2 * np], ah, bh[0], bh[1]);
        mma_bf16(acc[2 * np + 1], ah, bh[2], bh[3]);
        if (which) {
          uint32_t bl[4];
          ldsm_x4_t(bl, Zl + bo);
          mma_bf16(acc[2 * np], ah, bl[0], bl[1]);
          mma_bf16(acc[2 * np + 1], ah, bl[2], bl[3]);
          mma_bf16(acc[2 * np], al, bh[0], bh[1]);
          mma_bf16(acc[2 * np + 1], al, bh[2], bh[3]);
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

  // 8. the scan's Q and K rows in fp16: exp(G) (.) q^ and exp(G_C - G) (.) k^ (both
  //    at most their unit-norm inputs), and the per-chunk factors
  {
    __half* qd = reinterpret_cast<__half*>(ws + L.qh) + (head * Tp + t0) * kD;
    __half* kd = reinterpret_cast<__half*>(ws + L.kh) + (head * Tp + t0) * kD;
    for (int i = tid; i < kC * 16; i += kThreads) {
      const int r = i >> 4, c8 = (i & 15) * 8;
      uint4 oq, ok;
      uint32_t* wq = reinterpret_cast<uint32_t*>(&oq);
      uint32_t* wk = reinterpret_cast<uint32_t*>(&ok);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c8 + 2 * u;
        const float2 qq = unpack2(*reinterpret_cast<const uint32_t*>(Qt + r * LDT + c));
        const float2 kk = unpack2(*reinterpret_cast<const uint32_t*>(Kt + r * LDT + c));
        wq[u] = pack2h(qq.x * sq[r] * __expf(Gm[r * LDG + c]), qq.y * sq[r] * __expf(Gm[r * LDG + c + 1]));
        wk[u] = pack2h(kk.x * rk[r] * __expf(Gm[(kC - 1) * LDG + c] - Gm[r * LDG + c]),
                       kk.y * rk[r] * __expf(Gm[(kC - 1) * LDG + c + 1] - Gm[r * LDG + c + 1]));
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
      for (int w = 0; w < 8; ++w) m = fmaxf(m, misc[8 + w]);
      sc[kScMaxU + tid] = tid == 0 ? m : 0.f;
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
  for (int n = tid; n < Nc; n += kScanThreads) mx = fmaxf(mx, Sg[(size_t)n * kScal + kScMaxU]);
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

    // S <- diag(gamma_C) S + K^T U~s  (this warp's 16 state rows)
    {
      const float gA = sc[kScGC + sr], gB = sc[kScGC + sr + 8];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        S[nt][0] *= gA; S[nt][1] *= gA; S[nt][2] *= gB; S[nt][3] *= gB;
      }
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
cudaError_t launch_t(const ChunkArgs& a, bool gdn2, uint8_t* ws, const WsLayout& L,
                     cudaStream_t s) {
  const int Nc = (a.T + kC - 1) / kC;
  const bool pre = (a.flags & GDN_GATES_PRECOMPUTED) != 0;
  const int l2 = (a.flags & GDN_QK_L2NORM) ? 1 : 0;
  int* status = status_word();
  if (status == nullptr) return cudaErrorUnknown;
  cudaError_t e;
  if (gdn2) {
    auto prep = pre ? wy_prep2_kernel<true> : wy_prep2_kernel<false>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, Q2_BYTES);
    if (e != cudaSuccess) return e;
    prep<<<dim3(1, Nc, a.B * a.Hv), kThreads, Q2_BYTES, s>>>(
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
        static_cast<const bf16*>(a.v), a.a, a.b, a.w, a.A_log, a.dt_bias, a.T, a.Hv, a.scale, l2,
        ws, L, status);
  } else {
    auto prep = pre ? wy_prep_kernel<true> : wy_prep_kernel<false>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, P_BYTES);
    if (e != cudaSuccess) return e;
    prep<<<dim3(a.Hv / a.Hk, Nc, a.B * a.Hk), kThreads, P_BYTES, s>>>(
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
        static_cast<const bf16*>(a.v), a.a, a.b, a.A_log, a.dt_bias, a.T, a.Hk, a.Hv, a.scale, l2,
        ws, L, status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(state_scan_kernel<TO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           S_BYTES);
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

cudaError_t launch_chunk_mma(const ChunkArgs& a, bool gdn2, void* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(a.B, a.T, a.Hk, a.Hv);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (a.flags & GDN_OUT_F32) return launch_t<float>(a, gdn2, w, L, s);
  return launch_t<bf16>(a, gdn2, w, L, s);
}

}  // namespace gdn
