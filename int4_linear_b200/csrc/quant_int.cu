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
// Structure (all shapes n2 in {64, 128}, n1 <= 128; one CTA of 256 threads,
// two per tile row (tensor-memory lane t and its second half), two CTAs per
// SM when shared memory allows).  An item is G tokens (G = 2 when n1 <= 64,
// else 1), so that stage A has 128 rows (token s, tile row i):
//   1. the threads of row (s, i) load its tile row (n2 fp16 values, times c),
//      pick a power-of-two scale for it, and write its XL = 4 limbs as the
//      K-major A operand rows of stage A;
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
//      stacked limbs per 32-column chunk of k (five levels, a zero block
//      padding the stack); P1 = NULL stages the identity;
//   5. thread = (s, l): levels -> exact 64-bit value -> float32 X̂ (one
//      rounding), per-token / per-group maxima by warp reductions, scales,
//      round-half-even codes (reciprocal fast path outside a tie band, IEEE
//      quotient inside it) into a shared-memory code tile that leaves by one
//      bulk store per item; group scales go out through caller strides.
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
  long long sg_g, sg_m;  // element strides of s_grp: group g of token m at g * sg_g + m * sg_m
  float* xhat;
  unsigned* err;
};

namespace {

constexpr int kIntThreads = 256;
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
  // the item's packed codes (G tokens of up to NP * N2 / 2 bytes), written to
  // global memory by one bulk copy
  static constexpr int CODE = G * NP * N2 / 2;
  static constexpr int OFF_CODE = OFF_X + XU;
  static constexpr int OFF_RED = OFF_CODE + CODE;
  // tensor memory: stage A's four level blocks (256 columns), stage B's five
  // blocks reuse them; with four stage-B chunks (NP = 128) the float values
  // of the row wait in columns 320..447 for the token's scale
  // With 512 columns (n2 = 128: one CTA per SM) stage A's two chunks get
  // their own blocks and stage B's chunks alternate between two 160-column
  // buffers, so the next chunk's MMAs run while this one is read.
  static constexpr int TMEM_COLS = N2 == 128 ? 512 : 256;
  static constexpr bool DB = TMEM_COLS == 512;
  static constexpr int STASH = 320;
  // reduction scratch (32-bit words): [8] warp maxima, [2][128] halves of
  // the tile rows' maxima, [8][64] group maxima (uint bits), [2][64] group scales
  static constexpr int R_WARP = 0;
  static constexpr int R_XM = 8;
  static constexpr int R_GMAX = R_XM + 2 * 128;
  static constexpr int R_SG = R_GMAX + 8 * 64;
  static constexpr int R_WORDS = R_SG + 2 * 64;
  // mbarriers: [0] factor loads, [1 + c] MMAs of stage-A chunk buffer c,
  // [3 + b] MMAs of stage-B buffer b (one barrier per buffer, so that none
  // runs more than one phase ahead of its waiters)
  static constexpr int OFF_BAR = OFF_RED + R_WORDS * 4;
  static constexpr int OFF_CONST = OFF_BAR + 40;  // ints: [0] f2, [1] f1, [4] tensor memory, [8 + 2 s + c] t
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
__global__ void __launch_bounds__(kIntThreads, (N2 == 64 ? 2 : 1)) quant_act_int_kernel(const QuantTcParams p) {
  using C = IC<N2, NP, HAS_C>;
  constexpr int G = C::G, XL = C::XL;
  constexpr int H2 = N2 / 2;  // tile columns (l, or j) per thread: a row's two halves
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int r = t & 127, h = t >> 7;  // the row (tensor-memory lane) and the half of it this thread owns
  const int n1 = p.n1, K = p.K, M = p.M;
  const int nitems = (M + G - 1) / G;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  int* cst = reinterpret_cast<int*>(sm + C::OFF_CONST);  // [0] f2 [1] f1 [4] tmem [8 + 2 s + c] t of V
  uint32_t* red = reinterpret_cast<uint32_t*>(sm + C::OFF_RED);
  float* sg = reinterpret_cast<float*>(red + C::R_SG);
  float* xm = reinterpret_cast<float*>(red + C::R_XM);
  uint32_t* gmax = red + C::R_GMAX;
  const uint32_t sbase = smem_u32(sm);

  uint64_t* lbar = bar;
  uint64_t* mA = bar + 1;  // [2]
  uint64_t* mB = bar + 3;  // [2]
  if (t == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(bar + b, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(cst + 4), C::TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  // The next kernel may be scheduled once every CTA of this one runs.  The
  // factors are parameters (no kernel of this library writes them) and are
  // prepared below while the kernels ahead on the stream may still run; the
  // activations, c and the outputs are touched only after pdl_wait().
  pdl_launch_dependents();

  // ---- factors: staged as float32 in the operand bytes (one bulk copy each
  // when aligned), then fixed-point exponents and stacked limbs
  {
    float* sf = reinterpret_cast<float*>(sm + C::OFF_X);
    auto stage = [&](const float* src, int count, uint32_t parity) {
      const uint32_t bytes = uint32_t(count) * 4u;
      const bool bulk = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (bytes & 15u) == 0;
      if (bulk) {
        if (t == 0) {
          mbar_arrive_expect_tx(lbar, bytes);
          bulk_load(sf, src, bytes, lbar);
        }
        if (!mbar_wait(lbar, parity)) record_error(p.err, kErrTimeoutProducer);
      } else {
        for (int e = t; e < count; e += kIntThreads) sf[e] = __ldg(src + e);
        __syncthreads();
      }
    };
    auto maxabs = [&](int count) {
      float m = 0.f;
      for (int e = t; e < count; e += kIntThreads) m = fmaxf(m, fabsf(sf[e]));
      m = __uint_as_float(warp_max_u32(__float_as_uint(m)));
      if (lane == 0) red[C::R_WARP + warp] = __float_as_uint(m);
      __syncthreads();
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kIntThreads / 32; ++w) a = fmaxf(a, __uint_as_float(red[C::R_WARP + w]));
      return a > 0.f ? ilog2f(a) - 29 : 0;  // |P| * 2^-f < 2^30
    };
    // P2 stacks: chunk c, row (3 - b) * 64 + l', byte j = limb b of P2[j][64 c + l']
    stage(p.P2, N2 * N2, 0);
    const int f2 = maxabs(N2 * N2);
    const float s2 = pow2f(-f2);
    for (int e = t; e < N2 * (N2 / 4); e += kIntThreads) {
      const int l = e % N2, j0 = (e / N2) * 4;
      uint32_t y[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) y[q] = uint32_t(__float2int_rn(sf[(j0 + q) * N2 + l] * s2)) + 0x80808080u;
      uint32_t w[4];
      planes4(y[0], y[1], y[2], y[3], w);
      uint8_t* stk = sm + C::OFF_P2 + (l >> 6) * C::P2_CH;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        *reinterpret_cast<uint32_t*>(stk + krow_offset<N2>(uint32_t((3 - b) * 64 + (l & 63)), uint32_t(j0))) = w[b];
    }
    fence_proxy_async_smem();
    __syncthreads();  // P2 read: the staging bytes take P1
    // P1 stacks: chunk kc (32 columns k), row (3 - b) * 32 + k', byte i = limb b
    // of P1[i][32 kc + k'] (0 past n1); rows 128..159 of a chunk are zero
    if (p.P1) {
      stage(p.P1, n1 * n1, 1);
    } else {  // P1 = I: the rows of the n1 x n2 reshape are transformed on their own
      for (int e = t; e < n1 * n1; e += kIntThreads) sf[e] = (e / n1 == e % n1) ? 1.f : 0.f;
      __syncthreads();
    }
    const int f1 = maxabs(n1 * n1);
    const float s1 = pow2f(-f1);
    for (int e = t; e < NP * (NP / 4); e += kIntThreads) {
      const int k = e % NP, i0 = (e / NP) * 4;
      uint32_t y[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q;
        const int v = (i < n1 && k < n1) ? __float2int_rn(sf[i * n1 + k] * s1) : 0;
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
      const int kc = e / (32 * (NP / 16)), rr = (e / (NP / 16)) % 32, c16 = e % (NP / 16);
      *reinterpret_cast<uint4*>(sm + C::OFF_P1 + kc * C::P1_CH + krow_offset<NP>(uint32_t(128 + rr), uint32_t(16 * c16))) =
          make_uint4(0, 0, 0, 0);
    }
    if (t == 0) {
      cst[0] = f2;
      cst[1] = f1;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = uint32_t(cst[4]);
  const int f2 = cst[0], f1 = cst[1];
  const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
  const uint32_t xbase = sbase + C::OFF_X, ubase = sbase + C::OFF_U;
  const uint32_t p2base = sbase + C::OFF_P2, p1base = sbase + C::OFF_P1;
  pdl_wait();  // X, c and the outputs may be touched from here on

  uint32_t phA[2] = {0, 0}, phB[2] = {0, 0};
  bool bad = false;
  // this thread's tile row of an item: (token s, tile row i), columns [h H2, h H2 + H2)
  const int s = G == 2 ? (r >> 6) : 0, i = G == 2 ? (r & 63) : r;
  auto load_row = [&](int item, uint4 (&raw)[H2 / 8]) {
    const int tok = item * G + s;
    const bool ok = item < nitems && i < n1 && tok < M;
    const __half* xrow = p.X + size_t(tok) * K + size_t(i) * N2 + h * H2;
#pragma unroll
    for (int q = 0; q < H2 / 8; ++q) raw[q] = ok ? *reinterpret_cast<const uint4*>(xrow + 8 * q) : make_uint4(0, 0, 0, 0);
  };
  uint4 raw[H2 / 8];
  load_row(blockIdx.x, raw);
  for (int item = blockIdx.x; item < nitems && !bad; item += gridDim.x) {
    const int tok0 = item * G;
    // the previous item's code tile has been read by its bulk copy before
    // any thread writes this item's codes (several barriers lie between)
    if (t == 0) bulk_wait_group_read<0>();
    // ---------------------------------------------------------------- 1. tile row -> limbs
    const int tok = tok0 + s;
    const bool rv = i < n1 && tok < M;
    const float4* crow = HAS_C ? reinterpret_cast<const float4*>(p.c + size_t(i) * N2 + h * H2) : nullptr;
    float mh = 0.f;
#pragma unroll
    for (int q = 0; q < H2 / 8; ++q) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw[q]);
      float4 c0 = make_float4(1.f, 1.f, 1.f, 1.f), c1 = c0;
      if (HAS_C && rv) {
        c0 = __ldg(crow + 2 * q);
        c1 = __ldg(crow + 2 * q + 1);
      }
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float2 v = __half22float2(h2[u]);
        if (HAS_C) {
          v.x = __fmul_rn(v.x, cv[2 * u]);
          v.y = __fmul_rn(v.y, cv[2 * u + 1]);
        }
        mh = fmaxf(mh, fmaxf(fabsf(v.x), fabsf(v.y)));
      }
    }
    // the row's largest |x c| from its two halves
    xm[h * 128 + r] = mh;
    __syncthreads();
    const float mx = fmaxf(xm[r], xm[128 + r]);
    const int ei = mx > 0.f ? ilog2f(mx) - 29 : 0;  // |x c| 2^-e < 2^30
    {
      const float sc = pow2f(-ei);
      uint8_t* xs = sm + C::OFF_X;
#pragma unroll
      for (int q0 = 0; q0 < H2 / 16; ++q0) {  // 16 values: raw[2 q0], raw[2 q0 + 1]
        uint32_t y[16];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const __half2* h2 = reinterpret_cast<const __half2*>(&raw[2 * q0 + hh]);
          float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0;
          if (HAS_C && rv) {
            c0 = __ldg(crow + 2 * (2 * q0 + hh));
            c1 = __ldg(crow + 2 * (2 * q0 + hh) + 1);
          }
          const float cv8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 v = __half22float2(h2[u]);
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const float x = z ? v.y : v.x;
              // x (times c) exactly as hi + lo, then round(x c 2^-e) as A * 256 + B
              // with both parts in the range where adding 1.5 * 2^23 rounds to an
              // integer (|A| <= 2^22, |B| <= 2^7 + 1)
              float hi = x, lo = 0.f;
              if (HAS_C) {
                const float cv = cv8[2 * u + z];
                hi = __fmul_rn(x, cv);
                lo = __fmaf_rn(x, cv, -hi);
              }
              const float af = __fmaf_rn(hi, sc * (1.0f / 256.0f), kMagic);
              const float Af = __fsub_rn(af, kMagic);
              const float rr = __fmaf_rn(Af, -256.0f * pow2f(ei), hi);
              const float bf = __fmaf_rn(HAS_C ? __fadd_rn(rr, lo) : rr, sc, kMagic);
              const int Ai = int(__float_as_uint(af) - kMagicBits), Bi = int(__float_as_uint(bf) - kMagicBits);
              y[8 * hh + 2 * u + z] = uint32_t(Ai * 256 + Bi) + 0x80808080u;
            }
          }
        }
        uint32_t w[4][4];  // [group of 4 values][plane]
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) planes4(y[4 * g4], y[4 * g4 + 1], y[4 * g4 + 2], y[4 * g4 + 3], w[g4]);
#pragma unroll
        for (int a = 0; a < XL; ++a)
          *reinterpret_cast<uint4*>(xs + a * C::X_PL + krow_offset<N2>(uint32_t(r), uint32_t(h * H2 + 16 * q0))) =
              make_uint4(w[0][a], w[1][a], w[2][a], w[3][a]);
      }
    }
    // the next item's rows load while this item runs
    load_row(item + gridDim.x, raw);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------------------------------------------------------- 2-3. stage A, V
    // V = U 2^-t per (token, 64-column chunk of l): t from the chunk's
    // largest |U| (its scale only has to be common along the contraction
    // index i of stage B).  Row (s, i) holds U = W 2^(8 (XL - 1) + e_i + f2)
    // with W = hi 2^16 + lo; |lo| < 2^31 bounds the low part.  This thread
    // takes columns l in [32 h, 32 h + 32) of each chunk.
    int vv[C::LCH][32];
    if (t == 0) {
      tc_fence_after();
      // both chunks up front when each has its own columns
#pragma unroll
      for (int ch = 0; ch < (C::DB ? C::LCH : 1); ++ch) {
        issue_stage<XL, 4, 64, N2 / 32, false, N2, C::X_PL, N2>(tmem + uint32_t(C::DB ? 256 * ch : 0), xbase,
                                                                 p2base + uint32_t(ch * C::P2_CH));
        mma_commit(&mA[ch]);
      }
    }
#pragma unroll
    for (int ch = 0; ch < C::LCH; ++ch) {
      const uint32_t dA = tmem + uint32_t(C::DB ? 256 * ch : 0);
      const int ba = C::DB ? ch : 0;
      if (!C::DB && ch > 0 && t == 0) {
        tc_fence_after();
        issue_stage<XL, 4, 64, N2 / 32, false, N2, C::X_PL, N2>(tmem, xbase, p2base + uint32_t(ch * C::P2_CH));
        mma_commit(&mA[0]);
      }
      if (!warp_wait(&mA[ba], phA[ba])) bad = true;
      phA[ba] ^= 1u;
      tc_fence_after();
      // pass 1: the largest |hi| of this row half, in units common to the token's rows
      uint32_t mhi = 0;
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        uint32_t d0[16], d1[16];
        const uint32_t col = uint32_t(32 * h + 16 * sl);
        tmem_ld_32x16(dA + lane_off + col, *reinterpret_cast<uint32_t(*)[32]>(d0));
        tmem_ld_32x16(dA + lane_off + col + 64u, *reinterpret_cast<uint32_t(*)[32]>(d1));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) mhi = max(mhi, uint32_t(abs(int(d0[q]) * 256 + int(d1[q]))));
      }
      const float rowmax = mx > 0.f ? (float(mhi) + 32768.0f) * pow2f(16 + ei) : 0.f;
      const uint32_t wmx = warp_max_u32(__float_as_uint(rowmax));
      if (lane == 0) red[C::R_WARP + warp] = wmx;
      bad = __syncthreads_or(bad);
      if (t < G) {
        // token t: rows [64 t, 64 t + 64) (G = 2: warps 2t, 2t + 1 and their second halves), else all
        float tm = 0.f;
        for (int w = 0; w < kIntThreads / 32; ++w)
          if (G == 1 || ((w & 3) >> 1) == t) tm = fmaxf(tm, __uint_as_float(red[C::R_WARP + w]));
        // |V| = |U| 2^-t < 2^29
        cst[8 + 2 * t + ch] = tm > 0.f ? ilog2f(tm) + 1 + 8 * (XL - 1) + f2 - 29 : 0;
      }
      __syncthreads();
      const int n = min(63, max(0, cst[8 + 2 * s + ch] - ei - f2 - 8 * (XL - 1)));
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        uint32_t d[4][16];
        load_levels16(dA + lane_off + uint32_t(32 * h + 16 * sl), d);
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
        for (int q0 = 0; q0 < 2; ++q0) {
          uint32_t w[4][4];
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            const int l = 16 * q0 + 4 * g4;
            planes4(uint32_t(vv[ch][l]) + 0x80808080u, uint32_t(vv[ch][l + 1]) + 0x80808080u,
                    uint32_t(vv[ch][l + 2]) + 0x80808080u, uint32_t(vv[ch][l + 3]) + 0x80808080u, w[g4]);
          }
          const int m0 = (N2 == 64 ? s * 64 : ch * 64) + 32 * h + 16 * q0;
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
    // their full precision.  This thread takes k in [16 h, 16 h + 16) of each
    // chunk.  The packed codes of the item go to a shared-memory tile and
    // leave in one bulk copy.
    uint8_t* ctile = sm + C::OFF_CODE;
    for (int g = 0; g < C::BG && !bad; ++g) {
      const int sb = RowB<N2, G>::token(r, g);
      const int l = RowB<N2, G>::col(r);
      const int tk = tok0 + sb;
      const bool tok_ok = tk < M;
      uint8_t* crow_t = ctile + sb * (K / 2);  // this row's token in the tile
      // X̂ = W' 2^(16 + t + f1), W' = D0 2^32 + D1 2^24 + D2 2^16 + D3 2^8 + D4,
      // t of this row's (token, l-chunk)
      const int Es = 16 + cst[8 + 2 * sb + (N2 == 128 ? (l >> 6) : 0)] + f1;
      const float up = pow2f(Es);
      constexpr bool kStash = NP == 128;  // four chunks: the values wait in tensor memory
      float fv[kStash ? 16 : NP / 2];
      float tmax = 0.f;
      // 8 codes (k = kbase .. kbase + 7 of this row's column l) into the tile
      auto put_codes = [&](int kbase, uint32_t word) {
        word = transpose_nibbles8(word, lane);
        const int kr = kbase + (lane & 7);
        if (tok_ok && kr < n1)
          *reinterpret_cast<uint32_t*>(crow_t + (size_t(kr) * N2 + (l & ~7)) / 2) = word;
      };
      // the 4 warps (n2 = 128) or 2 warps (n2 = 64, token sb) that hold half hh of the chunk
      auto half_warp = [&](int tt, int hh, int q) { return N2 == 128 ? 4 * hh + q : 4 * hh + 2 * tt + q; };
      auto issue_b = [&](int kc) {
        tc_fence_after();
        issue_stage<4, 5, 32, NP / 32, true, 0, C::U_PL, NP>(tmem + uint32_t(C::DB ? 160 * (kc & 1) : 0),
                                                              ubase + uint32_t(g * 4 * C::U_PL),
                                                              p1base + uint32_t(kc * C::P1_CH));
        mma_commit(&mB[C::DB ? (kc & 1) : 0]);
      };
      if (t == 0) issue_b(0);
#pragma unroll
      for (int kc = 0; kc < C::KCB; ++kc) {
        float* fc = fv + (kStash ? 0 : 16 * kc);
        // the next chunk's MMAs run while this one is read (its buffer was
        // last read before the barrier that closed the previous chunk)
        if (t == 0 && kc + 1 < C::KCB && C::DB) issue_b(kc + 1);
        {
          const int bb = C::DB ? (kc & 1) : 0;
          if (!warp_wait(&mB[bb], phB[bb])) bad = true;
          phB[bb] ^= 1u;
        }
        tc_fence_after();
        {
          const uint32_t dB = tmem + uint32_t(C::DB ? 160 * (kc & 1) : 0);
          uint32_t d[5][16];
#pragma unroll
          for (int bk = 0; bk < 5; ++bk)
            tmem_ld_32x16(dB + lane_off + uint32_t(32 * bk + 16 * h), *reinterpret_cast<uint32_t(*)[32]>(d[bk]));
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
            fc[q] = f;
            tmax = fmaxf(tmax, fabsf(f));
          }
        }
        if (kStash && GRAN == FQ_DYNAMIC_ROW) {
          uint32_t u[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) u[q] = __float_as_uint(fc[q]);
          tmem_st_32x16(tmem + lane_off + uint32_t(C::STASH + 32 * kc + 16 * h), u);
          tmem_wait_st();
        }
        tc_fence_before();
        bad = __syncthreads_or(bad);  // D read by every thread: free for the next MMA
        if (t == 0 && kc + 1 < C::KCB && !C::DB) issue_b(kc + 1);
        if (GRAN == FQ_DYNAMIC_GROUP) {
          // groups: n2 = 128 -> row k (all 128 rows of D); n2 = 64 -> rows k, k + 1 of token sb (64 rows)
          constexpr int KPG = 128 / N2;
#pragma unroll
          for (int k = 0; k < 16; k += KPG) {
            float a = fabsf(fc[k]);
            if (KPG == 2) a = fmaxf(a, fabsf(fc[k + 1]));
            const uint32_t rx = warp_max_u32(__float_as_uint(a * up));  // exact: a power of two
            if (lane == 0) gmax[warp * 64 + k / KPG] = rx;
          }
          __syncthreads();
          // group scales of this chunk: n2 = 128: 32 groups (k), over the 4 warps of
          // the k's half; n2 = 64: 16 groups (k pairs) per token, over 2 warps
          if (t < 32) {
            const int tt = N2 == 128 ? 0 : (t >> 4), gi = N2 == 128 ? t : (t & 15);
            const int per_half = N2 == 128 ? 16 : 8;  // groups per half of the chunk
            const int hh = gi / per_half, gl = gi % per_half;
            const int nw = N2 == 128 ? 4 : 2;
            float am = 0.f;
            for (int q = 0; q < nw; ++q) am = fmaxf(am, __uint_as_float(gmax[half_warp(tt, hh, q) * 64 + gl]));
            const __half sh = group_scale_h(am, p.alpha);
            sg[tt * 64 + gi] = __half2float(sh);
            const int tkk = tok0 + (N2 == 128 ? g : tt);
            const int kg = N2 == 128 ? kc * 32 + gi : kc * 16 + gi;  // group index within the token
            if (tkk < M && kg * 128 < n1 * N2) p.s_grp[kg * p.sg_g + tkk * p.sg_m] = sh;
          }
          __syncthreads();
        }
        if (GRAN != FQ_DYNAMIC_ROW) {
          // codes of this chunk half
          const int sidx = N2 == 128 ? 0 : sb;
#pragma unroll
          for (int k0 = 0; k0 < 16; k0 += 8) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              const int kl = 16 * h + k0 + b;  // within the chunk
              const int k = kc * 32 + kl;
              const float v = fc[k0 + b] * up;
              int qv;
              if (GRAN == FQ_STATIC_CHANNEL) {
                qv = (k < n1 && tok_ok) ? code_ieee(v, __ldg(p.sstatic + k * N2 + l)) : 0;
              } else {
                qv = code_ieee(v, sg[sidx * 64 + kl / (128 / N2)]);
              }
              word = put_nibble(word, qv, 4 * b);
            }
            if (p.xhat && tok_ok) {
#pragma unroll
              for (int b = 0; b < 8; ++b) {
                const int k = kc * 32 + 16 * h + k0 + b;
                if (k < n1) p.xhat[size_t(tk) * K + size_t(k) * N2 + l] = fc[k0 + b] * up;
              }
            }
            put_codes(kc * 32 + 16 * h + k0, word);
          }
          if (GRAN == FQ_DYNAMIC_GROUP) __syncthreads();  // sg is rewritten by the next chunk
        }
      }
      if (GRAN == FQ_DYNAMIC_ROW) {
        // token maximum: n2 = 64 -> the 4 warps of token sb; n2 = 128 -> all 8
        const uint32_t rx = warp_max_u32(__float_as_uint(tmax * up));  // exact: a power of two
        if (lane == 0) red[C::R_WARP + warp] = rx;
        __syncthreads();
        float amax = 0.f;
        for (int w = 0; w < kIntThreads / 32; ++w)
          if (N2 == 128 || ((w & 3) >> 1) == sb) amax = fmaxf(amax, __uint_as_float(red[C::R_WARP + w]));
        const float s_tok = __fdiv_rn(__fmul_rn(amax, p.alpha), 7.0f);
        if (tok_ok && l == 0 && h == 0) p.s_row[tk] = s_tok;
        const float ftok = s_tok != 0.f ? (1.0f / s_tok) * up : 0.f;
        // x = fma(f, ftok, 1.5 * 2^23) holds rint(f * ftok) in its low bits;
        // next to a tie (or for s = 0) the IEEE quotient decides
        const float th = 0.5f - (8.0f / fminf(p.alpha, 1.0f) + 1.0f) * 9.5367431640625e-07f;
        const bool clampq = !(p.alpha >= 1.0f);
#pragma unroll
        for (int kc = 0; kc < C::KCB; ++kc) {
          float* fc = fv + (kStash ? 0 : 16 * kc);
          if (kStash) {
            uint32_t u[16];
            tmem_ld_32x16(tmem + lane_off + uint32_t(C::STASH + 32 * kc + 16 * h), *reinterpret_cast<uint32_t(*)[32]>(u));
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) fc[q] = __uint_as_float(u[q]);
          }
#pragma unroll
          for (int k0 = 0; k0 < 16; k0 += 8) {
            uint32_t word = 0;
            bool redo = s_tok == 0.f;
#pragma unroll
            for (int b = 0; b < 8; b += 2) {
              const float2 dd = make_float2(fc[k0 + b], fc[k0 + b + 1]);
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
              for (int b = 0; b < 8; ++b) word = put_nibble(word, code_ieee(fc[k0 + b] * up, s_tok), 4 * b);
            }
            if (p.xhat && tok_ok) {
#pragma unroll
              for (int b = 0; b < 8; ++b) {
                const int k = kc * 32 + 16 * h + k0 + b;
                if (k < n1) p.xhat[size_t(tk) * K + size_t(k) * N2 + l] = fc[k0 + b] * up;
              }
            }
            put_codes(kc * 32 + 16 * h + k0, word);
          }
        }
        __syncthreads();  // red is reused by the next group / item
      }
    }
    // the item's codes: one bulk copy of the valid tokens' rows
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0 && !bad) {
      const int ntok = min(G, M - tok0);
      bulk_store(p.Q + size_t(tok0) * (K / 2), ctile, uint32_t(ntok * (K / 2)));
      bulk_commit_group();
    }
    if (__syncthreads_or(bad)) break;
  }
  if (bad && t == 0) record_error(p.err, kErrTimeoutMma);
  if (t == 0) bulk_wait_group<0>();  // the codes are written before the CTA leaves
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int N2, int NP, int GRAN, bool HAS_C>
fq_status launch_int4(const QuantTcParams& p, cudaStream_t stream) {
  using C = IC<N2, NP, HAS_C>;
  auto kern = quant_act_int_kernel<N2, NP, GRAN, HAS_C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the transform kernel", C::SMEM);
  // CTAs per SM: 256 tensor-memory columns each (at most 2), and what fits in
  // the SM's 228 KB of shared memory (1 KB of it reserved per CTA)
  const int per_sm = (2 * (C::SMEM + 1024) <= 228 * 1024) ? 2 : 1;
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
