// Online activation quantization with the Kronecker transform computed
// EXACTLY on the integer tensor cores (FlatQuant notes, 高效 Kernel 设计: the
// transform and the quantization fused, intermediates kept on chip;
// Kronecker 分解: X̂ = P1^T Xbar P2 for each token's n1 x n2 reshape Xbar).
//
// Why integers.  A float32 evaluation of the two 64-to-128-term contractions
// rounds every partial sum relative to its largest term, and an outlier
// channel (tens of times the others) makes that error far larger than the
// transformed values near zero can tolerate.  Here every operand is written
// as a fixed-point integer in balanced base-256 digits ("limbs", each a
// signed byte in [-128, 127]) and every product of two limbs is summed
// exactly by `tcgen05.mma.kind::i8` into int32 tensor memory; the only
// roundings are the fixed-point representations themselves (2^-22 of a
// sub-row's largest fp16 value, 2^-31 with c; 2^-30 of the largest factor
// entry; 2^-29 of the intermediate bound), far below float32's.
//
// Structure (all shapes n2 in {64, 128}, n1 <= 128; one CTA of 128 threads,
// thread t = tensor-memory lane t, two CTAs per SM when shared memory allows).
// An item is G tokens (G = 2 when n1 <= 64, else 1), so that stage A has
// 128 rows (token s, tile row i):
//   1. thread (s, i) loads its tile row (n2 fp16 values, times c), picks a
//      power-of-two scale for it, and writes its XL limbs (XL = 3, 4 with c)
//      as the K-major A operand rows of stage A;
//   2. stage A: D[(s, i)][(level, l)] = sum_j Xbar_s[i][j] P2[j][l] by
//      levels: limb products of equal weight 256^L accumulate together.  P2
//      is held as 4 limbs stacked along N ([p3; p2; p1; p0] per 64-column
//      chunk of l), so one MMA per X limb fills several level blocks;
//   3. thread (s, i) combines its row's levels into an exact 64-bit value,
//      rescales it to a per-token 30-bit fixed point V (the bound comes from
//      the token's largest |x| times the largest column sum of |P2|), and
//      writes V's 4 limbs as the MN-major A operand of stage B (row i of the
//      operand holds the 128 M positions (s, l));
//   4. stage B: D[(s, l)][(level, k)] = sum_i V_s[i][l] P1[i][k], P1 as 4
//      stacked limbs per 64-column chunk of k;
//   5. thread = (s, l): levels -> exact 64-bit value -> float32 X̂ (one
//      rounding), per-token / per-group maxima by warp reductions, scales,
//      round-half-even codes (reciprocal fast path outside a tie band, IEEE
//      quotient inside it), a 3-step shuffle transpose into 32-bit stores.
#include <cuda_fp16.h>

#include <algorithm>

#include "fq_device.cuh"
#include "fq_host.h"

namespace fq {

struct QuantTcParams {
  const __half* X;
  int M, K, n1, n2, gran;
  float alpha;
  const float* P1;
  const float* P2;
  const float* c;
  const float* sstatic;
  uint8_t* Q;
  float* s_row;
  __half* s_grp;
  float* xhat;
  unsigned* err;
};

namespace {

constexpr int kIntThreads = 128;
constexpr float kMagic = 12582912.0f;       // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

template <int N2, int NP, bool HAS_C>
struct IC {
  static constexpr int G = NP == 64 ? 2 : 1;  // tokens per item: stage A has G * NP = 128 rows
  static constexpr int XL = 4;                // limbs of a tile row (a 30-bit fixed point per tile row)
  static constexpr int LCH = N2 / 64;         // 64-column chunks of l (stage A)
  static constexpr int KCB = NP / 32;         // 32-column chunks of k (stage B)
  static constexpr int BG = (G * N2) / 128;   // stage-B row groups (of 128 M rows) per item
  static constexpr int P2_CH = 256 * N2;      // one l-chunk stack: rows (b, l), K = j
  static constexpr int P1_CH = 160 * NP;      // one k-chunk stack: rows (b, k) and 32 zero rows, K = i
  static constexpr int X_PL = 128 * N2;       // one limb plane of the tile rows
  static constexpr int U_PL = NP * 128;       // one limb plane of V: NP K-rows x 128 M bytes
  static constexpr int OFF_P2 = 0;
  static constexpr int OFF_P1 = OFF_P2 + LCH * P2_CH;
  static constexpr int OFF_X = OFF_P1 + KCB * P1_CH;
  // V's limbs are written once stage A has finished reading the tile limbs,
  // so both can share the bytes
  static constexpr int XU = (XL * X_PL > BG * 4 * U_PL) ? XL * X_PL : BG * 4 * U_PL;
  static constexpr int OFF_U = OFF_X;
  static constexpr int OFF_RED = OFF_X + XU;
  // reduction scratch (32-bit words): [4] warp maxima, [2][128] group maxima
  // (uint bits), [2][128] group scales, [2][128] their inverses
  static constexpr int R_WARP = 0;
  static constexpr int R_GMAX = 4;
  static constexpr int R_SG = R_GMAX + 2 * 128;
  static constexpr int R_SINV = R_SG + 2 * 128;
  static constexpr int R_WORDS = R_SINV + 2 * 128;
  static constexpr int OFF_BAR = OFF_RED + R_WORDS * 4;
  static constexpr int OFF_CONST = OFF_BAR + 8;  // ints: [0] f2, [1] f1, [4] tensor memory, [8 + 2 s + c] t
  static constexpr int SMEM = OFF_CONST + 64 + 1024;
  static_assert(N2 == 64 || N2 == 128, "n2");
  static_assert(NP == 64 || NP == 128, "padded n1");
  static_assert(BG >= 1, "a stage-B group is 128 rows (token, column)");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(OFF_P1 % 1024 == 0 && OFF_X % 1024 == 0 && X_PL % 1024 == 0 && U_PL % 1024 == 0 &&
                P1_CH % 1024 == 0, "alignment");
};

// ---- layouts of the operands in shared memory

// K-major operand with 64-byte rows in the 64-byte swizzle (8-row atoms of
// 512 bytes, 16-byte chunk index XORed with (row / 2) mod 4).
__host__ __device__ constexpr uint32_t sw64_offset(uint32_t row, uint32_t byte) {
  return (row >> 3) * 512u + (row & 7u) * 64u + ((((byte >> 4) ^ (row >> 1)) & 3u) << 4) + (byte & 15u);
}

__device__ __forceinline__ uint64_t sdesc_k64_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);  // start address
  d |= uint64_t(16u >> 4) << 16;           // leading byte offset (unused for this layout)
  d |= uint64_t(512u >> 4) << 32;          // stride byte offset: next 8-row atom
  d |= uint64_t(1) << 46;                  // descriptor version for tcgen05
  d |= uint64_t(4) << 61;                  // 64-byte swizzle
  return d;
}

// MN-major operand of 128 M bytes per K row in the 128-byte swizzle (8 K-rows
// per 1024-byte atom; the M extent is one atom wide, so the leading byte
// offset is unused).
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(16u >> 4) << 16;
  d |= uint64_t(1024u >> 4) << 32;         // next 8 K-rows
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;                  // 128-byte swizzle
  return d;
}

template <int ROWB>
__device__ __forceinline__ uint32_t krow_offset(uint32_t row, uint32_t byte) {
  return ROWB == 64 ? sw64_offset(row, byte) : sw128_offset(row, byte);
}

template <int ROWB>
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) {
  return ROWB == 64 ? sdesc_k64_sw64(saddr) : sdesc_k128_sw128(saddr);
}

// tcgen05.mma .kind::i8: s8 x s8 -> s32, M = 128, A K-major (a_mn = 0) or
// MN-major (a_mn = 1), B K-major.
__host__ __device__ constexpr uint32_t idesc_i8_major(int n, int a_mn) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(n >> 3) << 17) |
         (uint32_t(128 >> 4) << 24);
}

// ---- small arithmetic helpers

// floor(log2 x) for a positive normal float.
__device__ __forceinline__ int ilog2f(float x) { return int((__float_as_uint(x) >> 23) & 0xFFu) - 127; }
// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// Four words holding biased digits (digit + 128 in each byte) of four values
// -> limb plane b (byte b of each, as signed digits) for b = 0..3.
__device__ __forceinline__ void planes4(uint32_t y0, uint32_t y1, uint32_t y2, uint32_t y3, uint32_t (&w)[4]) {
  const uint32_t a = __byte_perm(y0, y1, 0x5140);  // y0.0 y1.0 y0.1 y1.1
  const uint32_t b = __byte_perm(y0, y1, 0x7362);  // y0.2 y1.2 y0.3 y1.3
  const uint32_t c = __byte_perm(y2, y3, 0x5140);
  const uint32_t d = __byte_perm(y2, y3, 0x7362);
  w[0] = __byte_perm(a, c, 0x5410) ^ 0x80808080u;
  w[1] = __byte_perm(a, c, 0x7632) ^ 0x80808080u;
  w[2] = __byte_perm(b, d, 0x5410) ^ 0x80808080u;
  w[3] = __byte_perm(b, d, 0x7632) ^ 0x80808080u;
}

__device__ __forceinline__ uint32_t put_nibble(uint32_t w, int q, int pos) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(r) : "r"(q), "r"(w), "r"(pos));
  return r;
}

__device__ __noinline__ int code_ieee(float v, float s) {
  if (s == 0.0f) return 0;
  const float r = rintf(__fdiv_rn(v, s));
  return static_cast<int>(fminf(fmaxf(r, -8.0f), 7.0f));
}

__device__ __noinline__ __half group_scale_h(float amax, float alpha) {
  return __float2half_rn(__fdiv_rn(__fmul_rn(amax, alpha), 7.0f));
}

// Lanes 8g..8g+7 each hold 8 nibbles (nibble b = code of row k0 + b, column
// l0 + a for lane a of the group); afterwards lane a holds the 8 codes of
// row k0 + a, columns l0..l0+7.
__device__ __forceinline__ uint32_t transpose_nibbles8(uint32_t w, int lane) {
  const int a = lane & 7;
  uint32_t x = __shfl_xor_sync(0xffffffffu, w, 4);
  w = (a & 4) ? ((w & 0xFFFF0000u) | ((x & 0xFFFF0000u) >> 16)) : ((w & 0x0000FFFFu) | ((x & 0x0000FFFFu) << 16));
  x = __shfl_xor_sync(0xffffffffu, w, 2);
  w = (a & 2) ? ((w & 0xFF00FF00u) | ((x & 0xFF00FF00u) >> 8)) : ((w & 0x00FF00FFu) | ((x & 0x00FF00FFu) << 8));
  x = __shfl_xor_sync(0xffffffffu, w, 1);
  w = (a & 1) ? ((w & 0xF0F0F0F0u) | ((x & 0xF0F0F0F0u) >> 4)) : ((w & 0x0F0F0F0Fu) | ((x & 0x0F0F0F0Fu) << 4));
  return w;
}

// The four level blocks of one 16-column slice of D (columns col..col+15 of
// each 64-column block) combined into the exact 64-bit value
// W = (D0 * 256 + D1) * 2^16 + (D2 * 256 + D3), then shifted right by n.
__device__ __forceinline__ void load_levels16(uint32_t taddr, uint32_t (&d)[4][16]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) tmem_ld_32x16(taddr + uint32_t(64 * b), *reinterpret_cast<uint32_t(*)[32]>(d[b]));
}

__device__ __forceinline__ long long combine_levels(uint32_t d0, uint32_t d1, uint32_t d2, uint32_t d3) {
  const int hi = int(d0) * 256 + int(d1);
  const int lo = int(d2) * 256 + int(d3);
  return (static_cast<long long>(hi) << 16) + lo;
}

// The MMAs of one stage.  A limb a (AL limbs, a = AL - 1 is the top one)
// meets B limbs 3, 2, 1, 0 stacked in that order along N (BW rows each, then
// BW zero rows); the product of A limb a and B limb b has weight
// 256^(a + b), and the NLEV heaviest weights land in the level blocks
// 0 .. NLEV - 1 of D (BW columns each): block (AL - 1 - a) + (3 - b).  So
// limb a's MMA covers min(4, NLEV - gap) blocks of the B stack from block
// gap = AL - 1 - a on; the top limb covers all NLEV blocks (the zero rows
// fill the ones below its lowest limb), so its first MMA initializes every
// block of D.  A: K-major rows of AROWB bytes (planes A_PLANE bytes apart)
// or, with A_MN, MN-major with 128-byte K-rows (K step = 32 rows = 4096 bytes).
template <int AL, int NLEV, int BW, int KSTEPS, bool A_MN, int AROWB, int A_PLANE, int BROWB>
__device__ __forceinline__ void issue_stage(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
#pragma unroll
  for (int a = AL - 1; a >= 0; --a) {
    const int gap = AL - 1 - a;
    const int nblk = gap == 0 ? NLEV : min(4, NLEV - gap);
    if (nblk <= 0) continue;
    const uint32_t idesc = idesc_i8_major(BW * nblk, A_MN ? 1 : 0);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const uint32_t aa = a_base + uint32_t(a * A_PLANE) + uint32_t(kk * (A_MN ? 4096 : 32));
      const uint64_t adesc = A_MN ? sdesc_mn_sw128(aa) : kdesc<AROWB>(aa);
      const uint64_t bdesc = kdesc<BROWB>(b_base + uint32_t(kk * 32));
      mma_i8(d_tmem + uint32_t(BW * gap), adesc, bdesc, idesc, uint32_t(!(gap == 0 && kk == 0)));
    }
  }
}

// Token rows of an item, stage-B view: D row t is (token s, column l).
template <int N2, int G>
struct RowB {
  __device__ __forceinline__ static int token(int t, int g) { return N2 == 64 ? (t >> 6) : g; }
  __device__ __forceinline__ static int col(int t) { return N2 == 64 ? (t & 63) : t; }
};

template <int N2, int NP, int GRAN, bool HAS_C>
__global__ void __launch_bounds__(kIntThreads) quant_act_int_kernel(const QuantTcParams p) {
  using C = IC<N2, NP, HAS_C>;
  constexpr int G = C::G, XL = C::XL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int n1 = p.n1, K = p.K, M = p.M;
  const int nitems = (M + G - 1) / G;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  int* cst = reinterpret_cast<int*>(sm + C::OFF_CONST);  // [0] f2 [1] f1 [4] tmem [8 + 2 s + c] t of V
  uint32_t* red = reinterpret_cast<uint32_t*>(sm + C::OFF_RED);
  float* sg = reinterpret_cast<float*>(red + C::R_SG);
  float* sinv = reinterpret_cast<float*>(red + C::R_SINV);
  uint32_t* gmax = red + C::R_GMAX;
  const uint32_t sbase = smem_u32(sm);
  (void)sinv;

  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(cst + 4), 256);
    tmem_relinquish();
  }
  // The next kernel may be scheduled once every CTA of this one runs.  The
  // factors are parameters (no kernel of this library writes them) and are
  // prepared below while the kernels ahead on the stream may still run; the
  // activations, c and the outputs are touched only after pdl_wait().
  pdl_launch_dependents();

  // ---- factors: fixed-point exponents and stacked limbs
  {
    float m2 = 0.f, m1 = 0.f;
    for (int e = t; e < N2 * N2; e += kIntThreads) m2 = fmaxf(m2, fabsf(__ldg(p.P2 + e)));
    for (int e = t; e < n1 * n1; e += kIntThreads) m1 = fmaxf(m1, fabsf(__ldg(p.P1 + e)));
    m2 = __uint_as_float(warp_max_u32(__float_as_uint(m2)));
    m1 = __uint_as_float(warp_max_u32(__float_as_uint(m1)));
    if (lane == 0) {
      red[2 * warp + 0] = __float_as_uint(m2);
      red[2 * warp + 1] = __float_as_uint(m1);
    }
    __syncthreads();
    if (t == 0) {
      float a = 0.f, b = 0.f;
      for (int w = 0; w < 4; ++w) {
        a = fmaxf(a, __uint_as_float(red[2 * w]));
        b = fmaxf(b, __uint_as_float(red[2 * w + 1]));
      }
      cst[0] = a > 0.f ? ilog2f(a) - 29 : 0;  // |P2| * 2^-f2 < 2^30
      cst[1] = b > 0.f ? ilog2f(b) - 29 : 0;
    }
    __syncthreads();
    const int f2 = cst[0], f1 = cst[1];
    const float s2 = pow2f(-f2), s1 = pow2f(-f1);
    // P2 stacks: chunk c, row (3 - b) * 64 + l', byte j = limb b of P2[j][64 c + l']
    for (int e = t; e < N2 * (N2 / 4); e += kIntThreads) {
      const int l = e % N2, j0 = (e / N2) * 4;
      uint32_t y[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) y[q] = uint32_t(__float2int_rn(__ldg(p.P2 + (j0 + q) * N2 + l) * s2)) + 0x80808080u;
      uint32_t w[4];
      planes4(y[0], y[1], y[2], y[3], w);
      uint8_t* stk = sm + C::OFF_P2 + (l >> 6) * C::P2_CH;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        *reinterpret_cast<uint32_t*>(stk + krow_offset<N2>(uint32_t((3 - b) * 64 + (l & 63)), uint32_t(j0))) = w[b];
    }
    // P1 stacks: chunk kc (32 columns k), row (3 - b) * 32 + k', byte i = limb b
    // of P1[i][32 kc + k'] (0 past n1); rows 128..159 of a chunk are zero
    for (int e = t; e < NP * (NP / 4); e += kIntThreads) {
      const int k = e % NP, i0 = (e / NP) * 4;
      uint32_t y[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q;
        const int v = (i < n1 && k < n1) ? __float2int_rn(__ldg(p.P1 + i * n1 + k) * s1) : 0;
        y[q] = uint32_t(v) + 0x80808080u;
      }
      uint32_t w[4];
      planes4(y[0], y[1], y[2], y[3], w);
      uint8_t* stk = sm + C::OFF_P1 + (k >> 5) * C::P1_CH;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        *reinterpret_cast<uint32_t*>(stk + krow_offset<NP>(uint32_t((3 - b) * 32 + (k & 31)), uint32_t(i0))) = w[b];
    }
    for (int e = t; e < C::KCB * 32 * (NP / 16); e += kIntThreads) {
      const int kc = e / (32 * (NP / 16)), r = (e / (NP / 16)) % 32, c16 = e % (NP / 16);
      *reinterpret_cast<uint4*>(sm + C::OFF_P1 + kc * C::P1_CH + krow_offset<NP>(uint32_t(128 + r), uint32_t(16 * c16))) =
          make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = uint32_t(cst[4]);
  const int f2 = cst[0], f1 = cst[1];
  const uint32_t lane_off = uint32_t(warp * 32) << 16;
  const uint32_t xbase = sbase + C::OFF_X, ubase = sbase + C::OFF_U;
  const uint32_t p2base = sbase + C::OFF_P2, p1base = sbase + C::OFF_P1;
  pdl_wait();  // X, c and the outputs may be touched from here on

  uint32_t ph = 0;
  bool bad = false;
  for (int item = blockIdx.x; item < nitems && !bad; item += gridDim.x) {
    const int tok0 = item * G;
    // ---------------------------------------------------------------- 1. tile row -> limbs
    const int s = G == 2 ? (t >> 6) : 0, i = G == 2 ? (t & 63) : t;
    const int tok = tok0 + s;
    const bool rv = i < n1 && tok < M;
    uint4 raw[N2 / 8];
    const __half* xrow = p.X + size_t(tok) * K + size_t(i) * N2;
#pragma unroll
    for (int q = 0; q < N2 / 8; ++q) raw[q] = rv ? *reinterpret_cast<const uint4*>(xrow + 8 * q) : make_uint4(0, 0, 0, 0);
    const float* crow = HAS_C ? p.c + size_t(i) * N2 : nullptr;
    float mx = 0.f;
#pragma unroll
    for (int q = 0; q < N2 / 8; ++q) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw[q]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float2 v = __half22float2(h2[u]);
        if (HAS_C && rv) {
          v.x = __fmul_rn(v.x, __ldg(crow + 8 * q + 2 * u));
          v.y = __fmul_rn(v.y, __ldg(crow + 8 * q + 2 * u + 1));
        }
        mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
      }
    }
    const int ei = mx > 0.f ? ilog2f(mx) - 29 : 0;  // |x c| 2^-e < 2^30
    {
      const float sc = pow2f(-ei);
      uint8_t* xs = sm + C::OFF_X;
#pragma unroll
      for (int q0 = 0; q0 < N2 / 16; ++q0) {  // 16 values: raw[2 q0], raw[2 q0 + 1]
        uint32_t y[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const __half2* h2 = reinterpret_cast<const __half2*>(&raw[2 * q0 + h]);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 v = __half22float2(h2[u]);
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const float x = z ? v.y : v.x;
              const int jj = 16 * q0 + 8 * h + 2 * u + z;
              // x (times c) exactly as hi + lo, then round(x c 2^-e) as A * 256 + B
              // with both parts in the range where adding 1.5 * 2^23 rounds to an
              // integer (|A| <= 2^22, |B| <= 2^7 + 1)
              float hi = x, lo = 0.f;
              if (HAS_C) {
                const float cv = rv ? __ldg(crow + jj) : 0.f;
                hi = __fmul_rn(x, cv);
                lo = __fmaf_rn(x, cv, -hi);
              }
              const float af = __fmaf_rn(hi, sc * (1.0f / 256.0f), kMagic);
              const float Af = __fsub_rn(af, kMagic);
              const float r = __fmaf_rn(Af, -256.0f * pow2f(ei), hi);
              const float bf = __fmaf_rn(HAS_C ? __fadd_rn(r, lo) : r, sc, kMagic);
              const int Ai = int(__float_as_uint(af) - kMagicBits), Bi = int(__float_as_uint(bf) - kMagicBits);
              y[8 * h + 2 * u + z] = uint32_t(Ai * 256 + Bi) + 0x80808080u;
            }
          }
        }
        uint32_t w[4][4];  // [group of 4 values][plane]
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) planes4(y[4 * g4], y[4 * g4 + 1], y[4 * g4 + 2], y[4 * g4 + 3], w[g4]);
#pragma unroll
        for (int a = 0; a < XL; ++a)
          *reinterpret_cast<uint4*>(xs + a * C::X_PL + krow_offset<N2>(uint32_t(t), uint32_t(16 * q0))) =
              make_uint4(w[0][a], w[1][a], w[2][a], w[3][a]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------------------------------------------------------- 2-3. stage A, V
    // V = U 2^-t per (token, 64-column chunk of l): t from the chunk's
    // largest |U| (its scale only has to be common along the contraction
    // index i of stage B).  Row (s, i) holds U = W 2^(8 (XL - 1) + e_i + f2)
    // with W = hi 2^16 + lo; |lo| < 2^31 bounds the low part.
    int vv[C::LCH][64];
#pragma unroll
    for (int ch = 0; ch < C::LCH; ++ch) {
      if (t == 0) {
        tc_fence_after();
        issue_stage<XL, 4, 64, N2 / 32, false, N2, C::X_PL, N2>(tmem, xbase, p2base + uint32_t(ch * C::P2_CH));
        mma_commit(bar);
      }
      if (!warp_wait(bar, ph)) bad = true;
      ph ^= 1u;
      tc_fence_after();
      // pass 1: this row's largest |hi|, in units common to the token's rows
      uint32_t mh = 0;
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        uint32_t d0[16], d1[16];
        tmem_ld_32x16(tmem + lane_off + uint32_t(16 * sl), *reinterpret_cast<uint32_t(*)[32]>(d0));
        tmem_ld_32x16(tmem + lane_off + uint32_t(16 * sl + 64), *reinterpret_cast<uint32_t(*)[32]>(d1));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) mh = max(mh, uint32_t(abs(int(d0[q]) * 256 + int(d1[q]))));
      }
      const float rowmax = mx > 0.f ? (float(mh) + 32768.0f) * pow2f(16 + ei) : 0.f;
      const uint32_t wmx = warp_max_u32(__float_as_uint(rowmax));
      if (lane == 0) red[C::R_WARP + warp] = wmx;
      bad = __syncthreads_or(bad);
      if (t < G) {
        float tm = 0.f;
        for (int w = (G == 2 ? 2 * t : 0); w < (G == 2 ? 2 * t + 2 : 4); ++w) tm = fmaxf(tm, __uint_as_float(red[C::R_WARP + w]));
        // |V| = |U| 2^-t < 2^29
        cst[8 + 2 * t + ch] = tm > 0.f ? ilog2f(tm) + 1 + 8 * (XL - 1) + f2 - 29 : 0;
      }
      __syncthreads();
      const int n = min(63, max(0, cst[8 + 2 * s + ch] - ei - f2 - 8 * (XL - 1)));
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        uint32_t d[4][16];
        load_levels16(tmem + lane_off + uint32_t(16 * sl), d);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) vv[ch][16 * sl + q] = int(combine_levels(d[0][q], d[1][q], d[2][q], d[3][q]) >> n);
      }
      tc_fence_before();
      __syncthreads();  // D has been read: the next MMA may overwrite it
    }
    if (__syncthreads_or(bad)) break;
    // the tile limbs are no longer read: V's limbs take their bytes.
    // Operand row (K) = i, M byte = (s, l) for n2 = 64, else l (group s).
    {
      const int g = N2 == 64 ? 0 : s;
      uint8_t* ub = sm + C::OFF_U + g * 4 * C::U_PL;
#pragma unroll
      for (int ch = 0; ch < C::LCH; ++ch) {
#pragma unroll
        for (int q0 = 0; q0 < 4; ++q0) {
          uint32_t w[4][4];
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            const int l = 16 * q0 + 4 * g4;
            planes4(uint32_t(vv[ch][l]) + 0x80808080u, uint32_t(vv[ch][l + 1]) + 0x80808080u,
                    uint32_t(vv[ch][l + 2]) + 0x80808080u, uint32_t(vv[ch][l + 3]) + 0x80808080u, w[g4]);
          }
          const int m0 = (N2 == 64 ? s * 64 : ch * 64) + 16 * q0;
#pragma unroll
          for (int b = 0; b < 4; ++b)
            *reinterpret_cast<uint4*>(ub + b * C::U_PL + sw128_offset(uint32_t(i), uint32_t(m0))) =
                make_uint4(w[0][b], w[1][b], w[2][b], w[3][b]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---------------------------------------------------------------- 4-5. stage B, quantization
    // Per 32-column chunk of k: five level blocks of 32 columns (weights
    // 256^6 .. 256^2 of V's limbs times P1's), so that the rows of V far
    // below its largest one (an outlier row sets the token's scale) keep
    // their full precision.
    for (int g = 0; g < C::BG && !bad; ++g) {
      const int sb = RowB<N2, G>::token(t, g);
      const int l = RowB<N2, G>::col(t);
      const int tk = tok0 + sb;
      const bool tok_ok = tk < M;
      // X̂ = W' 2^(16 + t + f1), W' = D0 2^32 + D1 2^24 + D2 2^16 + D3 2^8 + D4,
      // t of this row's (token, l-chunk)
      const int Es = 16 + cst[8 + 2 * sb + (N2 == 128 ? (l >> 6) : 0)] + f1;
      const float up = pow2f(Es);
      float fv[NP];
      float tmax = 0.f;
#pragma unroll
      for (int kc = 0; kc < C::KCB; ++kc) {
        if (t == 0) {
          tc_fence_after();
          issue_stage<4, 5, 32, NP / 32, true, 0, C::U_PL, NP>(tmem, ubase + uint32_t(g * 4 * C::U_PL),
                                                                p1base + uint32_t(kc * C::P1_CH));
          mma_commit(bar);
        }
        if (!warp_wait(bar, ph)) bad = true;
        ph ^= 1u;
        tc_fence_after();
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          uint32_t d[5][16];
#pragma unroll
          for (int bk = 0; bk < 5; ++bk)
            tmem_ld_32x16(tmem + lane_off + uint32_t(32 * bk + 16 * sl), *reinterpret_cast<uint32_t(*)[32]>(d[bk]));
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            // float(W') = hi 2^24 + mid 2^8 + D4: the conversions of hi and mid
            // round only when they exceed 2^24, i.e. when W' itself is that
            // large, so the result is within a few float32 ulps of |W'| or of
            // 2^31 units (far below the transformed values' tolerance)
            const int hi = int(d[0][q]) * 256 + int(d[1][q]);
            const int mid = int(d[2][q]) * 256 + int(d[3][q]);
            const float f = __fmaf_rn(__int2float_rn(hi), 16777216.0f,
                                      __fmaf_rn(__int2float_rn(mid), 256.0f, __int2float_rn(int(d[4][q]))));
            fv[32 * kc + 16 * sl + q] = f;
            tmax = fmaxf(tmax, fabsf(f));
          }
        }
        tc_fence_before();
        bad = __syncthreads_or(bad);  // D read by every thread: free for the next MMA
        if (GRAN == FQ_DYNAMIC_GROUP) {
          // groups: n2 = 128 -> row k (all 128 rows of D); n2 = 64 -> rows k, k + 1 of token sb (64 rows)
          constexpr int KPG = 128 / N2;
#pragma unroll
          for (int k = 0; k < 32; k += KPG) {
            float a = fabsf(fv[32 * kc + k]);
            if (KPG == 2) a = fmaxf(a, fabsf(fv[32 * kc + k + 1]));
            const uint32_t r = warp_max_u32(__float_as_uint(a * up));  // exact: a power of two
            if (lane == 0) gmax[warp * 64 + k / KPG] = r;
          }
          __syncthreads();
          // group scales of this chunk: n2 = 128: 32 groups, over 4 warps;
          // n2 = 64: 16 groups per token, over the token's 2 warps
          if (t < 32) {
            const int tt = N2 == 128 ? 0 : (t >> 4), gi = N2 == 128 ? t : (t & 15);
            const int w0 = N2 == 128 ? 0 : 2 * tt, nw = N2 == 128 ? 4 : 2;
            float am = 0.f;
            for (int w = w0; w < w0 + nw; ++w) am = fmaxf(am, __uint_as_float(gmax[w * 64 + gi]));
            const __half sh = group_scale_h(am, p.alpha);
            sg[tt * 64 + gi] = __half2float(sh);
            const int tkk = tok0 + (N2 == 128 ? g : tt);
            const int kg = N2 == 128 ? kc * 32 + gi : kc * 16 + gi;  // group index within the token
            if (tkk < M && kg * 128 < n1 * N2) p.s_grp[size_t(kg) * M + tkk] = sh;
          }
          __syncthreads();
        }
        if (GRAN != FQ_DYNAMIC_ROW) {
          // codes of this chunk
          const int sidx = N2 == 128 ? 0 : sb;
#pragma unroll
          for (int k0 = 0; k0 < 32; k0 += 8) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              const int k = kc * 32 + k0 + b;
              const float v = fv[k] * up;
              int qv;
              if (GRAN == FQ_STATIC_CHANNEL) {
                qv = (k < n1 && tok_ok) ? code_ieee(v, __ldg(p.sstatic + k * N2 + l)) : 0;
              } else {
                qv = code_ieee(v, sg[sidx * 64 + (k0 + b) / (128 / N2)]);
              }
              word = put_nibble(word, qv, 4 * b);
            }
            if (p.xhat && tok_ok) {
#pragma unroll
              for (int b = 0; b < 8; ++b)
                if (kc * 32 + k0 + b < n1) p.xhat[size_t(tk) * K + size_t(kc * 32 + k0 + b) * N2 + l] = fv[kc * 32 + k0 + b] * up;
            }
            word = transpose_nibbles8(word, lane);
            const int kr = kc * 32 + k0 + (lane & 7);
            if (tok_ok && kr < n1)
              *reinterpret_cast<uint32_t*>(p.Q + size_t(tk) * (K / 2) + (size_t(kr) * N2 + (l & ~7)) / 2) = word;
          }
          if (GRAN == FQ_DYNAMIC_GROUP) __syncthreads();  // sg is rewritten by the next chunk
        }
      }
      if (GRAN == FQ_DYNAMIC_ROW) {
        // token maximum: n2 = 64 -> warps 2 sb, 2 sb + 1; n2 = 128 -> all four
        const uint32_t r = warp_max_u32(__float_as_uint(tmax * up));  // exact: a power of two
        if (lane == 0) red[C::R_WARP + warp] = r;
        __syncthreads();
        float amax = 0.f;
        for (int w = (N2 == 64 ? 2 * sb : 0); w < (N2 == 64 ? 2 * sb + 2 : 4); ++w)
          amax = fmaxf(amax, __uint_as_float(red[C::R_WARP + w]));
        const float s_tok = __fdiv_rn(__fmul_rn(amax, p.alpha), 7.0f);
        if (tok_ok && l == 0) p.s_row[tk] = s_tok;
        const float ftok = s_tok != 0.f ? (1.0f / s_tok) * up : 0.f;
        // x = fma(f, ftok, 1.5 * 2^23) holds rint(f * ftok) in its low bits;
        // next to a tie (or for s = 0) the IEEE quotient decides
        const float th = 0.5f - (8.0f / fminf(p.alpha, 1.0f) + 1.0f) * 9.5367431640625e-07f;
        const bool clampq = !(p.alpha >= 1.0f);
#pragma unroll
        for (int k0 = 0; k0 < NP; k0 += 8) {
          uint32_t word = 0;
          bool redo = s_tok == 0.f;
#pragma unroll
          for (int b = 0; b < 8; b += 2) {
            const float2 dd = make_float2(fv[k0 + b], fv[k0 + b + 1]);
            float2 x = ffma2(dd, make_float2(ftok, ftok), make_float2(kMagic, kMagic));
            const float2 rr =
                ffma2(dd, make_float2(ftok, ftok), ffma2(x, make_float2(-1.f, -1.f), make_float2(kMagic, kMagic)));
            if (clampq) {
              x.x = fminf(fmaxf(x.x, kMagic - 8.0f), kMagic + 7.0f);
              x.y = fminf(fmaxf(x.y, kMagic - 8.0f), kMagic + 7.0f);
            }
            redo |= fabsf(rr.x) >= th || fabsf(rr.y) >= th;
            word = put_nibble(word, int(__float_as_uint(x.x)), 4 * b);
            word = put_nibble(word, int(__float_as_uint(x.y)), 4 * b + 4);
          }
          if (redo) {
            word = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) word = put_nibble(word, code_ieee(fv[k0 + b] * up, s_tok), 4 * b);
          }
          if (p.xhat && tok_ok) {
#pragma unroll
            for (int b = 0; b < 8; ++b)
              if (k0 + b < n1) p.xhat[size_t(tk) * K + size_t(k0 + b) * N2 + l] = fv[k0 + b] * up;
          }
          word = transpose_nibbles8(word, lane);
          const int kr = k0 + (lane & 7);
          if (tok_ok && kr < n1)
            *reinterpret_cast<uint32_t*>(p.Q + size_t(tk) * (K / 2) + (size_t(kr) * N2 + (l & ~7)) / 2) = word;
        }
        __syncthreads();  // red is reused by the next group / item
      }
    }
    if (__syncthreads_or(bad)) break;
  }
  if (bad && t == 0) record_error(p.err, kErrTimeoutMma);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int N2, int NP, int GRAN, bool HAS_C>
fq_status launch_int4(const QuantTcParams& p, cudaStream_t stream) {
  using C = IC<N2, NP, HAS_C>;
  auto kern = quant_act_int_kernel<N2, NP, GRAN, HAS_C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the transform kernel", C::SMEM);
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kIntThreads, C::SMEM) != cudaSuccess) per_sm = 1;
  per_sm = std::max(1, std::min(per_sm, 2));  // 256 tensor-memory columns each
  const int nitems = (p.M + C::G - 1) / C::G;
  const int grid = std::max(1, std::min(nitems, sm_count() * per_sm));
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kIntThreads), C::SMEM, stream, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FQ_ERR_CUDA, "quant_act_int_kernel: %s", cudaGetErrorString(e));
  }
  return check_launch("quant_act_int_kernel");
}

template <int N2, int NP, bool HAS_C>
fq_status launch_int3(const QuantTcParams& p, cudaStream_t stream) {
  if (p.gran == FQ_DYNAMIC_ROW) return launch_int4<N2, NP, FQ_DYNAMIC_ROW, HAS_C>(p, stream);
  if (p.gran == FQ_DYNAMIC_GROUP) return launch_int4<N2, NP, FQ_DYNAMIC_GROUP, HAS_C>(p, stream);
  return launch_int4<N2, NP, FQ_STATIC_CHANNEL, HAS_C>(p, stream);
}

template <int N2, int NP>
fq_status launch_int(const QuantTcParams& p, cudaStream_t stream) {
  return p.c ? launch_int3<N2, NP, true>(p, stream) : launch_int3<N2, NP, false>(p, stream);
}

}  // namespace

// True when the integer tensor-core transform kernel covers this shape:
// n2 = 64 with n1 <= 64 (two tokens per 128-row item) or n2 = 128 with
// n1 <= 128 (one token per item, or two when n1 <= 64).
bool quant_act_tc_supported(int K, int n1, int n2) {
  if (n1 < 1 || n1 * n2 != K) return false;
  return (n2 == 64 && n1 <= 64) || (n2 == 128 && n1 <= 128);
}

fq_status launch_quant_act_tc(const QuantTcParams& p, cudaStream_t stream) {
  if (p.n2 == 64) return launch_int<64, 64>(p, stream);
  return p.n1 <= 64 ? launch_int<128, 64>(p, stream) : launch_int<128, 128>(p, stream);
}

}  // namespace fq
