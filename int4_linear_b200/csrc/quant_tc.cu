// Online activation quantization with the Kronecker transform on the tensor
// cores (FlatQuant notes, 高效 Kernel 设计: transform and quantization fused,
// intermediates kept on chip; Kronecker 分解: X̂ = P1^T Xbar P2 per token).
//
// Each token row is viewed as Xbar (n1 x n2).  Per tile of T tokens a CTA runs:
//   1. load the fp16 rows (128-bit, coalesced), scale them by c and by a
//      per-token power of two 2^-e (exact; every fp16 operand and the
//      intermediate stay below 2^14), split into fp16 hi (+ lo when c is
//      given; fp16 inputs times 2^-e are exact in fp16) and store them as the
//      K-major B operand "rows i, K = j" in the 128-byte swizzle;
//   2. stage A on the tensor cores: U^T = P2^T Xbar^T, i.e. D[l][i] =
//      sum_j P2[j][l] Xbar[i][j] (tcgen05.mma kind::f16, float32 in tensor
//      memory).  For n2 = 64 two tokens share one MMA through a
//      block-diagonal P2^T (token s in K half s, D rows (s, l));
//   3. U^T is read back row by row (thread = row (s, l), contiguous i), split
//      into fp16 hi + lo and stored with 16-byte stores as the A operand of
//   4. stage B: D[(s, l)][k] = sum_i U^T[(s, l)][i] P1[i][k] = X̂_s[k][l],
//      three passes (hi*hi + hi*lo + lo*hi);
//   5. thread = column l of X̂ of one token: per-token / per-group absmax via
//      warp reductions and shared atomics, scale, round-half-even (multiply by
//      1/s, IEEE division next to ties), clamp, and the codes of 8 x 8 blocks
//      are packed with a 3-step shuffle transpose into 32-bit stores.
// Products of fp16 hi/lo parts keep ~22 bits of every operand, so the
// transform is accurate to float32 level.
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

constexpr int kTcThreads = 512;
constexpr int kSplit = kTcThreads / 128;           // warps sharing one tensor-memory lane quadrant
constexpr int kMaxPieces = 2048 / kTcThreads;      // 16-byte pieces of the X tile per thread

template <int N2, int NP>
struct TcCfg {
  // tokens per tile: n2 = 64 pairs two tokens in K; n2 = 128 stacks 128/NP tokens in N
  static constexpr int T = N2 == 64 ? 2 : 128 / NP;
  static constexpr int XROWS = N2 == 64 ? NP : 128;  // rows of the X tile operand (= stage-A N)
  static constexpr int XKR = 2;                      // 64-wide K regions of the X tile
  static constexpr int USETS = N2 == 64 ? 1 : T;     // stage-B A operands (one per token when n2 = 128)
  static constexpr int UKR = NP / 64;                // K regions of the stage-B operands (K = n1 padded)
  static constexpr int REG = 128 * 128;              // one 128-row x 128-byte region
  // stage-A A operand P2^T: n2 = 64 keeps [0; P2^T; 0] (192 rows) so that the
  // two K halves see [P2^T; 0] and [0; P2^T]; n2 = 128 keeps two K regions
  static constexpr int SA_HALF = (N2 == 64 ? 192 : 256) * 128;
  static constexpr int SA = 0;
  static constexpr int SX = SA + 2 * SA_HALF;
  static constexpr int SX_XHALF = XKR * XROWS * 128;      // X tile hi (lo follows)
  static constexpr int SX_UHALF = USETS * UKR * REG;      // U^T hi (lo follows)
  static constexpr int SX_BYTES = (2 * SX_XHALF > 2 * SX_UHALF) ? 2 * SX_XHALF : 2 * SX_UHALF;
  static constexpr int SL = SX + SX_BYTES;                 // stage-B B operand P1: rows k, K = i
  static constexpr int SL_HALF = UKR * NP * 128;
  static constexpr int STG = SL + 2 * SL_HALF;             // fp16 staging of the next tile's rows
  static constexpr int STG_BYTES = T * NP * N2 * 2;        // (T tokens of at most NP x N2)
  static constexpr int OFF_MAX = STG + STG_BYTES;          // uint [2] token max, [2][128] group max
  static constexpr int OFF_BAR = OFF_MAX + 4 * (2 + 256) + 8;
  static constexpr int OFF_SLOT = OFF_BAR + 24;
  static constexpr int SMEM = OFF_SLOT + 16 + 1024;
  static constexpr int TMEM_COLS = 128;
  static_assert(N2 == 64 || N2 == 128, "n2");
  static_assert(NP == 64 || NP == 128, "n1 padding");
  static_assert((OFF_BAR & 7) == 0, "barrier alignment");
};

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Kept out of line: it is the rare path of code_fast and the static path,
// and inlining its division everywhere bloats the kernel's instruction stream.
__device__ __noinline__ int code_of(float v, float s) {
  if (s == 0.0f) return 0;
  const float r = rintf(__fdiv_rn(v, s));
  return static_cast<int>(fminf(fmaxf(r, -8.0f), 7.0f));
}

// fp16 group scale from a group absmax: fp16((amax * alpha) / 7).
__device__ __noinline__ __half group_scale(float amax, float alpha) {
  return __float2half_rn(__fdiv_rn(__fmul_rn(amax, alpha), 7.0f));
}

// The same code as code_of(v, s) = clamp(rint(v / s)) with IEEE division,
// computed with a multiply by inv_s = 1/s (rounded): that quotient is within
// 1.5 units in the last place of the correctly rounded one, so rounding it
// to an integer can only differ from rounding the IEEE quotient next to a
// tie (x.5); there the IEEE division decides.
__device__ __forceinline__ int code_fast(float v, float s, float inv_s) {
  if (s == 0.0f) return 0;
  const float qa = v * inv_s;
  const float f = qa - floorf(qa);
  if (fabsf(f - 0.5f) <= fabsf(qa) * 9.5367431640625e-07f + 1e-30f)  // 2^-20 relative margin
    return code_of(v, s);
  return static_cast<int>(fminf(fmaxf(rintf(qa), -8.0f), 7.0f));
}

// The code of v = u * up (up a power of two, exact) for scale s, given
// f = up * (1/s) (also exact scaling of the rounded reciprocal): the quotient
// u * f equals v * fl(1/s), so the tie test of code_fast applies unchanged.
// Returns the code in the low 4 bits position-free (caller masks).
__device__ __forceinline__ int code_scaled(float u, float f, float up, float s) {
  const float qa = u * f;
  const float r = rintf(qa);
  const float d = fabsf(qa - r);  // distance to the nearest integer
  if (0.5f - d <= fabsf(qa) * 9.5367431640625e-07f + 1e-30f) return code_of(u * up, s);
  return __float2int_rn(fminf(fmaxf(r, -8.0f), 7.0f));
}

// w with bits [pos, pos + 4) replaced by the low 4 bits of q.
__device__ __forceinline__ uint32_t put_nibble(uint32_t w, int q, int pos) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(r) : "r"(q), "r"(w), "r"(pos));
  return r;
}

// 2^e as a float for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// Lanes 8g..8g+7 each hold 8 nibbles (nibble b = code of row k0 + b, column
// l0 + a for lane a of the group); afterwards lane a holds the 8 codes of row
// k0 + a, columns l0..l0+7 (nibble order = column order).
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

// Two CTAs per SM where the shared memory allows it (n2 = n1 = 64).
template <int N2, int NP>
constexpr int tc_min_blocks() { return 1; }

template <int N2, int NP, int GRAN>
__global__ void __launch_bounds__(kTcThreads, tc_min_blocks<N2, NP>()) quant_act_tc_kernel(const QuantTcParams p) {
  using C = TcCfg<N2, NP>;
  constexpr int T = C::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned* tokmax = reinterpret_cast<unsigned*>(sm + C::OFF_MAX);  // [2] float bits
  unsigned* grpmax = tokmax + 2;                                     // [2][128] float bits
  uint64_t* barA = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* barB = barA + 1;
  uint64_t* barX = barA + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::OFF_SLOT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n1 = p.n1, K = p.K, M = p.M;
  const bool has_c = p.c != nullptr;
  const int ntiles = (M + T - 1) / T;

  // rows of tile `tile` -> staging buffer (bulk copy, async proxy)
  auto issue_tile = [&](int tile) {
    if (tile < ntiles) {
      const int tok0 = tile * T;
      const int ntok = min(T, M - tok0);
      const uint32_t bytes = uint32_t(ntok) * uint32_t(K) * 2u;
      mbar_arrive_expect_tx(barX, bytes);
      bulk_load(sm + C::STG, p.X + size_t(tok0) * K, bytes, barX);
    }
  };

  if (tid == 0) {
    mbar_init(barA, 1);
    mbar_init(barB, 1);
    mbar_init(barX, 1);
    fence_mbar_init();
    issue_tile(blockIdx.x);
  }
  if (warp == 0) {
    tmem_alloc(tslot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // ---- factors -> fp16 hi/lo operands, once per CTA (zero-filled first)
  for (int c = tid; c < (2 * C::SA_HALF) / 16; c += kTcThreads)
    *reinterpret_cast<uint4*>(sm + C::SA + c * 16) = make_uint4(0, 0, 0, 0);
  for (int c = tid; c < (2 * C::SL_HALF) / 16; c += kTcThreads)
    *reinterpret_cast<uint4*>(sm + C::SL + c * 16) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  float csum = 0.f;  // part of the |P2| column sum of column tid % N2
  for (int e = tid; e < N2 * N2; e += kTcThreads) {
    const int j = e / N2, l = e % N2;  // A operand of stage A: row l, K index j, value P2[j][l]
    const float v = __ldg(p.P2 + e);
    csum += fabsf(v);
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    const int row = N2 == 64 ? 64 + l : l;
    const uint32_t off = (N2 == 64 ? 0u : uint32_t(j >> 6) * C::REG) + sw128_offset(row, (j & 63) * 2);
    *reinterpret_cast<__half*>(sm + C::SA + off) = hi;
    *reinterpret_cast<__half*>(sm + C::SA + C::SA_HALF + off) = lo;
  }
  for (int e = tid; e < n1 * n1; e += kTcThreads) {
    const int i = e / n1, k = e % n1;  // B operand of stage B: row k, K index i, value P1[i][k]
    const float v = __ldg(p.P1 + e);
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    const uint32_t off = uint32_t(i >> 6) * (NP * 128) + sw128_offset(k, (i & 63) * 2);
    *reinterpret_cast<__half*>(sm + C::SL + off) = hi;
    *reinterpret_cast<__half*>(sm + C::SL + C::SL_HALF + off) = lo;
  }
  // largest absolute column sum of P2 (bounds |U| by max|x| * colsum)
  // column sums: thread tid holds part of column tid % N2; fold into 256 slots first
  float* colsum = reinterpret_cast<float*>(grpmax);
  if (tid < 256) colsum[tid] = 0.f;
  __syncthreads();
  atomicAdd(&colsum[tid & 255], csum);  // 256 is a multiple of N2: slot keeps the column
  __syncthreads();
  float cs = 0.f;
  if (tid < N2)
    for (int r = tid; r < 256; r += N2) cs += colsum[r];
  cs = warp_max_f(cs);
  __syncthreads();
  if (lane == 0) colsum[warp] = cs;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float guard = 1.f;
  for (int w = 0; w < kTcThreads / 32; ++w) guard = fmaxf(guard, colsum[w]);
  const uint32_t tmem = *tslot;
  __syncthreads();

  const int npieces = T * K / 8;
  const int q4 = warp & 3, part = warp >> 2;  // lane quadrant, column part (0..kSplit-1)
  const uint32_t tl = tmem + (uint32_t(q4 * 32) << 16);
  const int m = q4 * 32 + lane;  // tensor-memory lane of this thread
  constexpr uint32_t idescA = idesc_f16_m128(C::XROWS);
  constexpr uint32_t idescB = idesc_f16_m128(NP);

  uint32_t phase = 0;
  bool inflight = blockIdx.x < ntiles;  // a bulk copy into the staging buffer is outstanding
  uint32_t inflight_parity = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int tok0 = tile * T;
    if (tid < 2) tokmax[tid] = 0u;
    for (int i = tid; i < 256; i += kTcThreads) grpmax[i] = 0u;
    bool okx = warp_wait(barX, phase);  // this tile's rows are in the staging buffer
    inflight = false;

    // ---- 1a. per-token max of c * x
    uint4 buf[kMaxPieces];
    float mx0 = 0.f, mx1 = 0.f;
#pragma unroll
    for (int it = 0; it < kMaxPieces; ++it) {
      const int pc = tid + kTcThreads * it;
      buf[it] = make_uint4(0, 0, 0, 0);
      if (pc < npieces && tok0 + (pc * 8) / K < M) buf[it] = *reinterpret_cast<const uint4*>(sm + C::STG + pc * 16);
    }
#pragma unroll
    for (int it = 0; it < kMaxPieces; ++it) {
      const int pc = tid + kTcThreads * it;
      if (pc < npieces) {
        const int e = pc * 8, t = e / K, f = e - t * K;
        const __half2* h2 = reinterpret_cast<const __half2*>(&buf[it]);
        float mm = 0.f;
        if (has_c) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 v = __half22float2(h2[j]);
            const float a = __fmul_rn(v.x, __ldg(p.c + f + 2 * j));
            const float b = __fmul_rn(v.y, __ldg(p.c + f + 2 * j + 1));
            mm = fmaxf(mm, fmaxf(fabsf(a), fabsf(b)));
          }
        } else {
          // the max of |x| is exact in fp16
          const __half2 m2 = __hmax2(__hmax2(__habs2(h2[0]), __habs2(h2[1])), __hmax2(__habs2(h2[2]), __habs2(h2[3])));
          mm = fmaxf(__low2float(m2), __high2float(m2));
        }
        if (t == 0) mx0 = fmaxf(mx0, mm); else mx1 = fmaxf(mx1, mm);
      }
    }
    mx0 = warp_max_f(mx0);
    mx1 = warp_max_f(mx1);
    __syncthreads();  // maxima cleared, previous tile finished
    if (lane == 0) {
      atomicMax(&tokmax[0], __float_as_uint(mx0));
      atomicMax(&tokmax[1], __float_as_uint(mx1));
    }
    __syncthreads();
    int texp[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float mt = __uint_as_float(tokmax[t]);
      int E = 0;
      if (mt > 0.f) frexpf(mt * guard, &E);
      texp[t] = mt > 0.f ? min(max(E - 14, -100), 100) : 0;  // scaled max * guard <= 2^14
    }
    __syncthreads();  // everyone has read the token maxima
    if (tid < 2) tokmax[tid] = 0u;  // reused for the maxima of the transformed values
    // ---- 1b. scaled X tile: element (token t, row i, column j) -> operand row, K index
#pragma unroll
    for (int it = 0; it < kMaxPieces; ++it) {
      const int pc = tid + kTcThreads * it;
      if (pc < npieces) {
        const int e = pc * 8, t = e / K, f = e - t * K;
        const int i = f / N2, j = f % N2;
        const int row = N2 == 64 ? i : t * NP + i;
        const int kidx = N2 == 64 ? t * 64 + j : j;
        const uint32_t off = uint32_t(kidx >> 6) * (C::XROWS * 128) + sw128_offset(row, (kidx & 63) * 2);
        const float sc = exp2i(-texp[t]);
        const __half2* h2 = reinterpret_cast<const __half2*>(&buf[it]);
        uint4 hi, lo;
        __half2* hh = reinterpret_cast<__half2*>(&hi);
        __half2* ll = reinterpret_cast<__half2*>(&lo);
        if (!has_c && texp[t] >= -15 && texp[t] <= 14) {
          // fp16 x times an fp16 power of two: exact (the result stays below 2^14)
          const __half2 sc2 = __float2half2_rn(sc);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) hh[jj] = __hmul2(h2[jj], sc2);
          *reinterpret_cast<uint4*>(sm + C::SX + off) = hi;
          continue;
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float2 v = __half22float2(h2[jj]);
          if (has_c) {
            v.x = __fmul_rn(v.x, __ldg(p.c + f + 2 * jj));
            v.y = __fmul_rn(v.y, __ldg(p.c + f + 2 * jj + 1));
          }
          v.x *= sc;
          v.y *= sc;
          const __half2 a = __floats2half2_rn(v.x, v.y);
          const float2 af = __half22float2(a);
          hh[jj] = a;
          ll[jj] = __floats2half2_rn(v.x - af.x, v.y - af.y);
        }
        *reinterpret_cast<uint4*>(sm + C::SX + off) = hi;
        if (has_c) *reinterpret_cast<uint4*>(sm + C::SX + C::SX_XHALF + off) = lo;
      }
    }
    // zero the padding rows i >= n1 of every token slot (all rows of an empty slot)
    {
      constexpr int kRegPerRow = N2 == 64 ? 1 : 2;  // K regions a token row spans
      constexpr int chunks = 8 * kRegPerRow;       // 16-byte chunks per padded row
      for (int t = 0; t < T; ++t) {
        const int i0 = (tok0 + t < M) ? n1 : 0;
        const int total = (NP - i0) * chunks;
        for (int cidx = tid; cidx < total; cidx += kTcThreads) {
          const int r = cidx / chunks, rem = cidx % chunks;
          const int kidx = (N2 == 64 ? t * 64 : (rem / 8) * 64) + (rem % 8) * 8;
          const int row = N2 == 64 ? i0 + r : t * NP + i0 + r;
          const uint32_t off = uint32_t(kidx >> 6) * (C::XROWS * 128) + sw128_offset(row, (kidx & 63) * 2);
          *reinterpret_cast<uint4*>(sm + C::SX + off) = make_uint4(0, 0, 0, 0);
          if (has_c) *reinterpret_cast<uint4*>(sm + C::SX + C::SX_XHALF + off) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(!okx)) {
      if (tid == 0) record_error(p.err, kErrTimeoutUnpack);
      break;
    }
    if (tid == 0) issue_tile(tile + gridDim.x);  // the next tile's rows land during this one
    inflight = tile + int(gridDim.x) < ntiles;
    inflight_parity = phase ^ 1u;

    // ---- 2. stage A: D[l][i] = sum_j P2^T[l][j] Xbar[i][j]
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sa = smem_u32(sm + C::SA), sx = smem_u32(sm + C::SX);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int kr = kk >> 2;
        const uint32_t oa =
            (N2 == 64 ? uint32_t(kr == 0 ? 64 : 0) * 128u : uint32_t(kr) * C::REG) + uint32_t(kk & 3) * 32u;
        const uint32_t ob = uint32_t(kr) * (C::XROWS * 128) + uint32_t(kk & 3) * 32u;
        const uint64_t ahi = sdesc_k128_sw128(sa + oa), alo = sdesc_k128_sw128(sa + C::SA_HALF + oa);
        const uint64_t bhi = sdesc_k128_sw128(sx + ob);
        mma_f16(tmem, ahi, bhi, idescA, kk > 0);
        mma_f16(tmem, alo, bhi, idescA, 1);
        if (has_c) mma_f16(tmem, ahi, sdesc_k128_sw128(sx + C::SX_XHALF + ob), idescA, 1);
      }
      mma_commit(barA);
    }
    bool ok = warp_wait(barA, phase);
    tc_fence_after();

    // ---- 3. U^T rows -> fp16 hi/lo, 16-byte stores (stage-B operand A: row m, K index i)
    {
      constexpr int CW = C::XROWS / kSplit;  // columns per thread: 16 or 32
      uint32_t u[32];
      if (CW == 32)
        tmem_ld_32x32(tl + uint32_t(part * CW), u);
      else
        tmem_ld_32x16(tl + uint32_t(part * CW), u);
      tmem_wait_ld();
      {
        const int col = part * CW;  // D column = X tile row = (t, i)
        const int us = N2 == 64 ? 0 : col / NP;
        const int i0 = N2 == 64 ? col : col % NP;
        uint8_t* ub = sm + C::SX + us * (C::UKR * C::REG) + (i0 >> 6) * C::REG;
#pragma unroll
        for (int g = 0; g < CW / 8; ++g) {
          uint4 hi, lo;
          __half2* hh = reinterpret_cast<__half2*>(&hi);
          __half2* ll = reinterpret_cast<__half2*>(&lo);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const float a = __uint_as_float(u[g * 8 + 2 * jj]), b = __uint_as_float(u[g * 8 + 2 * jj + 1]);
            const __half2 h = __floats2half2_rn(a, b);
            const float2 hf = __half22float2(h);
            hh[jj] = h;
            ll[jj] = __floats2half2_rn(a - hf.x, b - hf.y);
          }
          const uint32_t off = sw128_offset(m, ((i0 & 63) + g * 8) * 2);
          *reinterpret_cast<uint4*>(ub + off) = hi;
          *reinterpret_cast<uint4*>(ub + C::SX_UHALF + off) = lo;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
      if (tid == 0) record_error(p.err, kErrTimeoutMma);
      break;
    }

    // ---- 4. stage B: D[(s, l)][k] = sum_i U^T[(s, l)][i] P1[i][k]
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sx = smem_u32(sm + C::SX), sl = smem_u32(sm + C::SL);
#pragma unroll
      for (int us = 0; us < C::USETS; ++us) {
#pragma unroll
        for (int kk = 0; kk < NP / 16; ++kk) {
          const uint32_t oa = uint32_t(us * C::UKR + (kk >> 2)) * C::REG + uint32_t(kk & 3) * 32u;
          const uint32_t ob = uint32_t(kk >> 2) * (NP * 128) + uint32_t(kk & 3) * 32u;
          const uint64_t ahi = sdesc_k128_sw128(sx + oa), alo = sdesc_k128_sw128(sx + C::SX_UHALF + oa);
          const uint64_t bhi = sdesc_k128_sw128(sl + ob), blo = sdesc_k128_sw128(sl + C::SL_HALF + ob);
          const uint32_t d = tmem + uint32_t(us * NP);
          mma_f16(d, ahi, bhi, idescB, kk > 0);
          mma_f16(d, ahi, blo, idescB, 1);
          mma_f16(d, alo, bhi, idescB, 1);
        }
      }
      mma_commit(barB);
    }
    ok = warp_wait(barB, phase);
    tc_fence_after();
    if (__syncthreads_or(!ok)) {
      if (tid == 0) record_error(p.err, kErrTimeoutMma);
      break;
    }

    // ---- 5. quantize: thread = column l of X̂ of one token, columns k in chunks of 8
    for (int us = 0; us < C::USETS; ++us) {
      const int t = N2 == 64 ? (m >> 6) : us;  // token slot of this thread
      const int l = N2 == 64 ? (m & 63) : m;
      const int tok = tok0 + t;
      const bool tok_ok = tok < M;
      const float up = exp2i(texp[t]);
      const uint32_t cbase = tl + uint32_t(us * NP);
      constexpr int NCH = NP / 8 / kSplit;  // 8-column chunks of this thread (part, part + kSplit, ...)
      uint32_t u[NCH][8];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld_32x8(cbase + uint32_t((kSplit * c + part) * 8), u[c]);
      tmem_wait_ld();
      // pass 1: token / group maxima (rows k >= n1 and empty token slots hold zeros)
      float tm = 0.f;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int ch = kSplit * c + part;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float a = fabsf(__uint_as_float(u[c][j]));
          tm = fmaxf(tm, a);
          if (GRAN == FQ_DYNAMIC_GROUP) {
            const int k = ch * 8 + j;
            const float w = warp_max_f(a) * up;
            if (lane == 0 && k < n1) atomicMax(&grpmax[t * 128 + (k * N2) / kGroup], __float_as_uint(w));
          }
        }
      }
      tm = warp_max_f(tm) * up;
      if (lane == 0) atomicMax(&tokmax[t], __float_as_uint(tm));
      __syncthreads();
      // pass 2: codes
      float s_tok = 0.f, f_tok = 0.f;
      if (GRAN == FQ_DYNAMIC_ROW) {
        s_tok = __fdiv_rn(__fmul_rn(__uint_as_float(tokmax[t]), p.alpha), 7.0f);
        f_tok = s_tok != 0.f ? (1.0f / s_tok) * up : 0.f;
        if (tok_ok && l == 0 && part == 0) p.s_row[tok] = s_tok;
      }
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int ch = kSplit * c + part;
        uint32_t word = 0;
        float sg = 0.f, inv_g = 0.f;
        int gcur = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int k = ch * 8 + j;
          const float uu = __uint_as_float(u[c][j]);
          const float v = uu * up;
          int q = 0;
          if (k < n1) {
            if (GRAN == FQ_DYNAMIC_ROW) {
              q = s_tok != 0.f ? code_scaled(uu, f_tok, up, s_tok) : 0;
            } else if (GRAN == FQ_DYNAMIC_GROUP) {
              const int g = (k * N2) / kGroup;
              if (g != gcur) {
                gcur = g;
                const __half sh = group_scale(__uint_as_float(grpmax[t * 128 + g]), p.alpha);
                sg = __half2float(sh);
                inv_g = sg != 0.f ? 1.0f / sg : 0.f;
                if (tok_ok && l == 0 && (k * N2) % kGroup == 0) p.s_grp[size_t(g) * M + tok] = sh;
              }
              q = code_fast(v, sg, inv_g);
            } else {
              q = code_of(v, __ldg(p.sstatic + k * N2 + l));
            }
            if (p.xhat && tok_ok) p.xhat[size_t(tok) * K + k * N2 + l] = v;
          }
          word = put_nibble(word, q, 4 * j);
        }
        word = transpose_nibbles8(word, lane);
        const int k = ch * 8 + (lane & 7);
        const int l0 = l & ~7;
        if (tok_ok && k < n1)
          *reinterpret_cast<uint32_t*>(p.Q + size_t(tok) * (K / 2) + (k * N2 + l0) / 2) = word;
      }
      __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    phase ^= 1u;
  }

  // a copy still in flight after an early exit lands before the CTA leaves
  if (tid == 0 && inflight && !mbar_wait(barX, inflight_parity)) record_error(p.err, kErrTimeoutDrain);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int N2, int NP, int GRAN>
fq_status launch_tc3(const QuantTcParams& p, cudaStream_t stream) {
  using C = TcCfg<N2, NP>;
  auto kern = quant_act_tc_kernel<N2, NP, GRAN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the transform kernel", C::SMEM);
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTcThreads, C::SMEM) != cudaSuccess) per_sm = 1;
  per_sm = std::max(1, std::min(per_sm, 512 / C::TMEM_COLS));
  const int ntiles = (p.M + C::T - 1) / C::T;
  const int grid = std::max(1, std::min(ntiles, sm_count() * per_sm));
  kern<<<grid, kTcThreads, C::SMEM, stream>>>(p);
  return check_launch("quant_act_tc_kernel");
}

template <int N2, int NP>
fq_status launch_tc(const QuantTcParams& p, cudaStream_t stream) {
  if (p.gran == FQ_DYNAMIC_ROW) return launch_tc3<N2, NP, FQ_DYNAMIC_ROW>(p, stream);
  if (p.gran == FQ_DYNAMIC_GROUP) return launch_tc3<N2, NP, FQ_DYNAMIC_GROUP>(p, stream);
  return launch_tc3<N2, NP, FQ_STATIC_CHANNEL>(p, stream);
}

}  // namespace

// True when the tensor-core transform kernel covers this shape.
bool quant_act_tc_supported(int K, int n1, int n2) {
  if (!(n2 == 64 || n2 == 128)) return false;
  return n1 >= 1 && n1 <= 128 && n1 * n2 == K;
}

fq_status launch_quant_act_tc(const QuantTcParams& p, cudaStream_t stream) {
  const bool np64 = p.n1 <= 64;
  if (p.n2 == 64) return np64 ? launch_tc<64, 64>(p, stream) : launch_tc<64, 128>(p, stream);
  return np64 ? launch_tc<128, 64>(p, stream) : launch_tc<128, 128>(p, stream);
}

}  // namespace fq
