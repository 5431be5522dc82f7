// Online activation quantization with the Kronecker transform on the tensor
// cores (FlatQuant notes, 高效 Kernel 设计: transform and quantization fused,
// intermediates kept on chip; Kronecker 分解: X̂ = P1^T Xbar P2 per token).
//
// Each token row is viewed as Xbar (n1 x n2, row-major).  A CTA runs P
// independent pipelines (4 when the padded n1 is 64, else 2; 1 when c is
// given with n1 > 64), each with its own tensor-memory region, shared-memory
// X tile, mbarriers and named barrier, so that one pipeline's tensor-core
// round trips overlap another's SIMT work.  A pipeline handles one "group"
// of G tokens at a time (G = 2 for n2 = 64: two tokens share the 128 MMA
// rows through a block-diagonal P2^T; G = 1 for n2 = 128):
//   1. the X tile: without c, the fp16 rows land by TMA directly in the
//      128-byte-swizzled K-major layout of the MMA's B operand (rows i of
//      Xbar, K = j); with c, the threads form x * c in float32, scale each
//      row i by a power of two 2^-e_i and store fp16 hi and lo parts;
//   2. stage A: D[row][i] = sum_j P2[j][l] Xbar[i][j] (row = (s, l) for token
//      s of the group), P2^T as fp16 hi + lo, float32 accumulation in tensor
//      memory (kind::f16);
//   3. thread = row: U^T row = D row (times 2^e_i with c), scaled by a power
//      of two 2^-e_row that brings its largest entry into [2^13, 2^14), split
//      into fp16 hi + lo and stored back into tensor memory as the A operand
//      of
//   4. stage B: D[row][k] = sum_i U^T[row][i] P1[i][k] (three products
//      hi*hi + hi*lo + lo*hi, A read from tensor memory);
//   5. thread = row = column l of token s: X̂[k][l] = D[row][k] * 2^e_row;
//      per-token (warp max reductions) or per-group maxima, scales,
//      round-half-even codes (multiply by 1/s, IEEE division next to ties),
//      and a 3-step shuffle transpose that packs 8 x 8 code blocks into
//      32-bit stores.
// Products of fp16 hi/lo parts keep about 22 bits of every operand, so the
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
constexpr int kTcWarps = kTcThreads / 32;

template <int N2, int NP, bool HAS_C>
struct TcCfg {
  static constexpr int G = N2 == 64 ? 2 : 1;                // tokens per group (128 MMA rows)
  static constexpr int P = NP == 64 ? 4 : (HAS_C ? 1 : 2);  // pipelines per CTA
  static constexpr int WPP = kTcWarps / P;                  // warps per pipeline
  static constexpr int TPP = WPP * 32;                      // threads per pipeline
  static constexpr int KSPLIT = WPP / 4;                    // warps sharing a lane quadrant
  static constexpr int COLS = NP / KSPLIT;                  // D columns per thread (64 or 32)
  static constexpr int TMEM_PIPE = 2 * NP;                  // D (stage A, then B) + U^T (hi, lo)
  static constexpr int REG = 128 * 128;                     // one 128-row x 128-byte region
  // stage-A A operand P2^T hi/lo: n2 = 64 keeps [0; P2^T; 0] (192 rows) so
  // that the two K halves see [P2^T; 0] and [0; P2^T]; n2 = 128 two K regions
  static constexpr int SA_HALF = (N2 == 64 ? 192 : 256) * 128;
  // X tile: two K regions of NP rows (n2 = 64: one per token; n2 = 128: j halves)
  static constexpr int X_REG = NP * 128;
  static constexpr int X_HALF = 2 * X_REG;
  static constexpr int X_BYTES = HAS_C ? 2 * X_HALF : X_HALF;  // hi (+ lo)
  // stage-B B operand P1 hi/lo: rows k, K = i in 64-wide regions
  static constexpr int SL_HALF = (NP / 64) * NP * 128;
  // per-pipeline scratch (floats): row-max parts [KSPLIT][128], token-max
  // parts [WPP], group maxima [G][128] (uint), group scales and inverses
  // [G][128] each, row exponents of the X tile [G][NP] (int, with c)
  static constexpr int R_RMAX = 0;
  static constexpr int R_TMAX = R_RMAX + KSPLIT * 128;
  static constexpr int R_GMAX = R_TMAX + 16;
  static constexpr int R_SG = R_GMAX + G * 128;
  static constexpr int R_SINV = R_SG + G * 128;
  static constexpr int R_XEXP = R_SINV + G * 128;
  static constexpr int RED_FLOATS = R_XEXP + G * NP;
  static constexpr int OFF_SA = 0;
  static constexpr int OFF_SL = OFF_SA + 2 * SA_HALF;
  static constexpr int OFF_X = OFF_SL + 2 * SL_HALF;
  static constexpr int OFF_RED = OFF_X + P * X_BYTES;
  static constexpr int OFF_BAR = OFF_RED + P * RED_FLOATS * 4;
  static constexpr int OFF_SLOT = OFF_BAR + 3 * P * 8;
  static constexpr int SMEM = OFF_SLOT + 16 + 1024;
  static_assert(N2 == 64 || N2 == 128, "n2");
  static_assert(NP == 64 || NP == 128, "padded n1");
  static_assert(COLS == 64 || COLS == 32, "columns per thread");
  static_assert(P * TMEM_PIPE <= 512, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert((OFF_X % 1024) == 0 && (X_REG % 1024) == 0 && (OFF_BAR % 8) == 0, "alignment");
};

// Kept out of line: it is the rare path of code_scaled / code_fast and the
// static path, and inlining its division everywhere bloats the kernel.
__device__ __noinline__ int code_of(float v, float s) {
  if (s == 0.0f) return 0;
  const float r = rintf(__fdiv_rn(v, s));
  return static_cast<int>(fminf(fmaxf(r, -8.0f), 7.0f));
}

// fp16 group scale from a group absmax: fp16((amax * alpha) / 7).
__device__ __noinline__ __half group_scale(float amax, float alpha) {
  return __float2half_rn(__fdiv_rn(__fmul_rn(amax, alpha), 7.0f));
}

// w with bits [pos, pos + 4) replaced by the low 4 bits of q.
__device__ __forceinline__ uint32_t put_nibble(uint32_t w, int q, int pos) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(r) : "r"(q), "r"(w), "r"(pos));
  return r;
}

// 2^e as a float for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// Exponent e with 2^-e * mx in [2^13, 2^14) (0 for mx == 0), clamped so that
// 2^-e and 2^e stay normal floats.
__device__ __forceinline__ int row_exponent(float mx) {
  if (!(mx > 0.f)) return 0;
  const int e = ((__float_as_int(mx) >> 23) & 0xFF) - 127 - 13;
  return min(max(e, -100), 100);
}

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

template <int N2, int NP, int GRAN, bool HAS_C>
__global__ void __launch_bounds__(kTcThreads, 1)
    quant_act_tc_kernel(const QuantTcParams p, const __grid_constant__ CUtensorMap tmX) {
  using C = TcCfg<N2, NP, HAS_C>;
  constexpr int G = C::G, COLS = C::COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pipe = warp / C::WPP, pw = warp % C::WPP;  // pipeline, warp within it
  const int ptid = tid - pipe * C::TPP;
  const int q4 = warp & 3;                             // tensor-memory lane quadrant
  const int part = pw >> 2;                            // column part of the row
  const int m = q4 * 32 + lane;                        // D row of this thread
  const int n1 = p.n1, K = p.K, M = p.M;
  const int ngroups = (M + G - 1) / G;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + 3 * pipe;
  uint64_t* mmaA = xfull + 1;
  uint64_t* mmaB = xfull + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::OFF_SLOT);
  float* red = reinterpret_cast<float*>(sm + C::OFF_RED) + pipe * C::RED_FLOATS;
  uint32_t* gmax = reinterpret_cast<uint32_t*>(red + C::R_GMAX);
  int* xexp = reinterpret_cast<int*>(red + C::R_XEXP);
  uint8_t* xt = sm + C::OFF_X + pipe * C::X_BYTES;

  if (tid == 0) {
    for (int b = 0; b < 3 * C::P; ++b) mbar_init(reinterpret_cast<uint64_t*>(sm + C::OFF_BAR) + b, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  // zero what no copy or factor store writes: the zero rows of the
  // block-diagonal P2^T, and the padding rows/columns beyond n1
  if (N2 == 64) {
    constexpr int kZeroChunks = 128 * 128 / 16;  // per half: rows 0..63 and 128..191
    for (int c = tid; c < 2 * kZeroChunks; c += kTcThreads) {
      const int half = c / kZeroChunks, r = c % kZeroChunks;
      const int off = half * C::SA_HALF + (r < kZeroChunks / 2 ? r * 16 : 64 * 128 + r * 16);
      *reinterpret_cast<uint4*>(sm + C::OFF_SA + off) = make_uint4(0, 0, 0, 0);
    }
  }
  if (n1 < NP) {
    for (int c = tid; c < (2 * C::SL_HALF) / 16; c += kTcThreads)
      *reinterpret_cast<uint4*>(sm + C::OFF_SL + c * 16) = make_uint4(0, 0, 0, 0);
    for (int c = tid; c < (C::P * C::X_BYTES) / 16; c += kTcThreads)
      *reinterpret_cast<uint4*>(sm + C::OFF_X + c * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  __syncthreads();
  // The next kernel may be scheduled once every CTA of this one is running.
  // The transform factors (parameters: no kernel of this library writes them)
  // are staged below while the kernels ahead on the stream may still run;
  // the activations, scales and outputs are touched only after pdl_wait().
  pdl_launch_dependents();

  const uint32_t lane_off = uint32_t(q4 * 32) << 16;
  const int bar_id = 1 + pipe;
  const bool leader = pw == 0 && lane == 0;
  const uint32_t idesc = idesc_f16_m128(NP);
  const bool c_vec = HAS_C && (reinterpret_cast<uintptr_t>(p.c) & 15u) == 0;  // c in 16-byte pieces
  const int s_of_row = N2 == 64 ? (m >> 6) : 0;  // token of this D row within the group
  const int l_of_row = N2 == 64 ? (m & 63) : m;  // column l of X̂ this row holds

  // TMA of the fp16 X tile of group grp (rows i of Xbar, K = j)
  auto issue_x = [&](int grp) {
    const int tok0 = grp * G;
    mbar_arrive_expect_tx(xfull, uint32_t(256 * n1));
    if (N2 == 64) {
      tma_load_2d(xt, &tmX, xfull, 0, tok0 * n1);
      tma_load_2d(xt + C::X_REG, &tmX, xfull, 0, (tok0 + 1) * n1);
    } else {
      tma_load_2d(xt, &tmX, xfull, 0, tok0 * n1);
      tma_load_2d(xt + C::X_REG, &tmX, xfull, 64, tok0 * n1);
    }
  };

  const int gstride = gridDim.x * C::P;
  int grp = blockIdx.x * C::P + pipe;
  bool x_pending = false;  // (leader) a TMA into the X tile has not been waited for
  if (!HAS_C && leader) prefetch_tensormap(&tmX);

  // ---- factors -> fp16 hi/lo operands, once per CTA, 8 consecutive K per 16-byte store.
  // Each thread first issues the loads of all its items, so their latencies
  // overlap, then converts and stores.
  {
    // stage-A A operand: row l, K = j, value P2[j][l]; consecutive threads
    // take consecutive l, so every load instruction reads whole rows of P2
    constexpr int kItems = N2 * (N2 / 8);
    constexpr int kPer = (kItems + kTcThreads - 1) / kTcThreads;
    float v[kPer][8];
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
      const int e = tid + it * kTcThreads;
      const int l = e % N2, j0 = (e / N2) * 8;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) v[it][jj] = e < kItems ? __ldg(p.P2 + (j0 + jj) * N2 + l) : 0.f;
    }
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
      const int e = tid + it * kTcThreads;
      if (e >= kItems) break;
      const int l = e % N2, j0 = (e / N2) * 8;
      uint4 hi, lo;
      __half* hh = reinterpret_cast<__half*>(&hi);
      __half* ll = reinterpret_cast<__half*>(&lo);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        hh[jj] = __float2half_rn(v[it][jj]);
        ll[jj] = __float2half_rn(v[it][jj] - __half2float(hh[jj]));
      }
      const int row = N2 == 64 ? 64 + l : l;
      const uint32_t off = (N2 == 64 ? 0u : uint32_t(j0 >> 6) * C::REG) + sw128_offset(row, (j0 & 63) * 2);
      *reinterpret_cast<uint4*>(sm + C::OFF_SA + off) = hi;
      *reinterpret_cast<uint4*>(sm + C::OFF_SA + C::SA_HALF + off) = lo;
    }
  }
  {
    // stage-B B operand: row k, K = i, value P1[i][k]
    const int n1c = (n1 + 7) / 8;
    constexpr int kPer = (NP * (NP / 8) + kTcThreads - 1) / kTcThreads;
    const int items = n1 * n1c;
    float v[kPer][8];
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
      const int e = tid + it * kTcThreads;
      const int k = e % n1, i0 = (e / n1) * 8;
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) v[it][ii] = (e < items && i0 + ii < n1) ? __ldg(p.P1 + (i0 + ii) * n1 + k) : 0.f;
    }
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
      const int e = tid + it * kTcThreads;
      if (e >= items) break;
      const int k = e % n1, i0 = (e / n1) * 8;
      uint4 hi, lo;
      __half* hh = reinterpret_cast<__half*>(&hi);
      __half* ll = reinterpret_cast<__half*>(&lo);
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) {
        hh[ii] = __float2half_rn(v[it][ii]);
        ll[ii] = __float2half_rn(v[it][ii] - __half2float(hh[ii]));
      }
      const uint32_t off = uint32_t(i0 >> 6) * (NP * 128) + sw128_offset(k, (i0 & 63) * 2);
      *reinterpret_cast<uint4*>(sm + C::OFF_SL + off) = hi;
      *reinterpret_cast<uint4*>(sm + C::OFF_SL + C::SL_HALF + off) = lo;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();  // the kernels ahead on the stream have completed: X may be read
  if (!HAS_C && leader && grp < ngroups) {
    issue_x(grp);
    x_pending = true;
  }
  const uint32_t tD = tmem + uint32_t(pipe * C::TMEM_PIPE);  // D: stage A, then stage B
  const uint32_t tU = tD + uint32_t(NP);                      // U^T: hi [0, NP/2), lo [NP/2, NP)

  uint32_t ph = 0;
  bool bad = false;
  for (; grp < ngroups; grp += gstride, ph ^= 1u) {
    const int tok0 = grp * G;

    // ---- 1. X tile
    if (HAS_C) {
      constexpr int PPR = N2 / 8;  // 16-byte pieces per row i of Xbar
      const int npieces = G * K / 8;
      for (int pc = ptid; pc < npieces; pc += C::TPP) {
        const int t = pc / (K / 8), f = (pc - t * (K / 8)) * 8;
        const int i = f / N2, j0 = f % N2;
        const int tok = tok0 + t;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (tok < M) raw = *reinterpret_cast<const uint4*>(p.X + size_t(tok) * K + f);
        float cv[8];
        if (c_vec) {
          const float4 c0 = __ldg(reinterpret_cast<const float4*>(p.c + f));
          const float4 c1 = __ldg(reinterpret_cast<const float4*>(p.c + f + 4));
          cv[0] = c0.x, cv[1] = c0.y, cv[2] = c0.z, cv[3] = c0.w;
          cv[4] = c1.x, cv[5] = c1.y, cv[6] = c1.z, cv[7] = c1.w;
        } else {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) cv[jj] = __ldg(p.c + f + jj);
        }
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
        float v[8];
        float mx = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float2 x2 = __half22float2(h2[jj]);
          v[2 * jj] = __fmul_rn(x2.x, cv[2 * jj]);
          v[2 * jj + 1] = __fmul_rn(x2.y, cv[2 * jj + 1]);
          mx = fmaxf(mx, fmaxf(fabsf(v[2 * jj]), fabsf(v[2 * jj + 1])));
        }
        // max over the row's PPR pieces (consecutive lanes)
#pragma unroll
        for (int o = 1; o < PPR; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const int e = row_exponent(mx);
        const float sc = exp2i(-e);
        if (j0 == 0) xexp[t * NP + i] = e;
        uint4 hi, lo;
        __half2* hh = reinterpret_cast<__half2*>(&hi);
        __half2* ll = reinterpret_cast<__half2*>(&lo);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float a = v[2 * jj] * sc, b = v[2 * jj + 1] * sc;
          const __half2 h = __floats2half2_rn(a, b);
          const float2 hf = __half22float2(h);
          hh[jj] = h;
          ll[jj] = __floats2half2_rn(a - hf.x, b - hf.y);
        }
        const int region = N2 == 64 ? t : (j0 >> 6);
        const uint32_t off = uint32_t(region) * C::X_REG + sw128_offset(i, (j0 & 63) * 2);
        *reinterpret_cast<uint4*>(xt + off) = hi;
        *reinterpret_cast<uint4*>(xt + C::X_HALF + off) = lo;
      }
      fence_proxy_async_smem();
      named_barrier(bar_id, C::TPP);
    } else if (leader) {
      if (mbar_wait(xfull, ph)) {
        x_pending = false;
      } else {
        record_error(p.err, kErrTimeoutProducer);
        bad = true;
      }
    }

    // ---- 2. stage A: D[row][i] = sum_j P2^T[l][j] Xbar_s[i][j]
    // The pipelines of a CTA start one stage A apart (pipeline p's first one
    // waits for pipeline p - 1's), so afterwards one pipeline's tensor-core
    // work overlaps the others' SIMT work instead of all of them alternating
    // in lockstep.
    if (leader && !bad && ph == 0 && grp == int(blockIdx.x) * C::P + pipe && pipe > 0 &&
        !mbar_wait(mmaA - 3, 0)) {
      record_error(p.err, kErrTimeoutMma);
      bad = true;
    }
    if (leader && !bad) {
      tc_fence_after();
      const uint32_t sa = smem_u32(sm + C::OFF_SA), sx = smem_u32(xt);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int kr = kk >> 2;
        const uint32_t oa =
            (N2 == 64 ? uint32_t(kr == 0 ? 64 : 0) * 128u : uint32_t(kr) * C::REG) + uint32_t(kk & 3) * 32u;
        const uint32_t ob = uint32_t(kr) * C::X_REG + uint32_t(kk & 3) * 32u;
        const uint64_t ahi = sdesc_k128_sw128(sa + oa), alo = sdesc_k128_sw128(sa + C::SA_HALF + oa);
        const uint64_t bhi = sdesc_k128_sw128(sx + ob);
        mma_f16(tD, ahi, bhi, idesc, kk > 0);
        mma_f16(tD, alo, bhi, idesc, 1);
        if (HAS_C) mma_f16(tD, ahi, sdesc_k128_sw128(sx + C::X_HALF + ob), idesc, 1);
      }
      mma_commit(mmaA);
    }
    if (!warp_wait(mmaA, ph)) bad = true;
    tc_fence_after();
    // the X tile is free again: the next group's rows land during steps 3-5
    if (!HAS_C && leader && !bad && grp + gstride < ngroups) {
      issue_x(grp + gstride);
      x_pending = true;
    }

    // ---- 3. U^T rows: D row (times 2^e_i with c), row scale 2^-e_row, fp16 hi/lo -> tensor memory
    int e_row;
    {
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32(tD + lane_off + uint32_t(part * COLS + 32 * c), u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float v = __uint_as_float(u[j]);
          if (HAS_C) v *= exp2i(xexp[s_of_row * NP + part * COLS + 32 * c + j]);
          mx = fmaxf(mx, fabsf(v));
        }
      }
      if (C::KSPLIT > 1) {
        red[C::R_RMAX + part * 128 + m] = mx;
        named_barrier(bar_id, C::TPP);
#pragma unroll
        for (int pp = 0; pp < C::KSPLIT; ++pp) mx = fmaxf(mx, red[C::R_RMAX + pp * 128 + m]);
      }
      e_row = row_exponent(mx);
      const float sc = exp2i(-e_row);
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32(tD + lane_off + uint32_t(part * COLS + 32 * c), u);
        tmem_wait_ld();
        uint32_t hi[16], lo[16];
        const float2 sc2 = make_float2(sc, sc), m1 = make_float2(-1.f, -1.f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float2 ab = make_float2(__uint_as_float(u[2 * j]), __uint_as_float(u[2 * j + 1]));
          if (HAS_C) {
            ab.x *= exp2i(xexp[s_of_row * NP + part * COLS + 32 * c + 2 * j]);
            ab.y *= exp2i(xexp[s_of_row * NP + part * COLS + 32 * c + 2 * j + 1]);
          }
          ab = fmul2(ab, sc2);  // exact: a power of two
          const __half2 h = __floats2half2_rn(ab.x, ab.y);
          const float2 r = ffma2(__half22float2(h), m1, ab);  // ab - hi, exact
          const __half2 l2 = __floats2half2_rn(r.x, r.y);
          hi[j] = *reinterpret_cast<const uint32_t*>(&h);
          lo[j] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const uint32_t col = uint32_t(part * COLS / 2 + 16 * c);
        tmem_st_32x16(tU + lane_off + col, hi);
        tmem_st_32x16(tU + lane_off + uint32_t(NP / 2) + col, lo);
      }
    }
    // the group maxima of step 5 start from zero
    if (GRAN == FQ_DYNAMIC_GROUP)
      for (int e = ptid; e < G * 128; e += C::TPP) gmax[e] = 0u;
    tmem_wait_st();
    tc_fence_before();
    bad = named_barrier_or(bar_id, C::TPP, bad);
    if (bad) break;

    // ---- 4. stage B: D[row][k] = sum_i U^T[row][i] P1[i][k]
    if (leader) {
      tc_fence_after();
      const uint32_t sl = smem_u32(sm + C::OFF_SL);
#pragma unroll
      for (int kk = 0; kk < NP / 16; ++kk) {
        const uint32_t ob = uint32_t(kk >> 2) * (NP * 128) + uint32_t(kk & 3) * 32u;
        const uint64_t bhi = sdesc_k128_sw128(sl + ob), blo = sdesc_k128_sw128(sl + C::SL_HALF + ob);
        const uint32_t ahi = tU + uint32_t(8 * kk), alo = tU + uint32_t(NP / 2 + 8 * kk);
        mma_f16_ts(tD, ahi, bhi, idesc, kk > 0);
        mma_f16_ts(tD, ahi, blo, idesc, 1);
        mma_f16_ts(tD, alo, bhi, idesc, 1);
      }
      mma_commit(mmaB);
    }
    if (!warp_wait(mmaB, ph)) bad = true;
    tc_fence_after();

    // ---- 5. quantize: thread = row (s, l), columns k of this part
    {
      const int s = s_of_row, l = l_of_row;
      const int tok = tok0 + s;
      const bool tok_ok = tok < M;
      const float up = exp2i(e_row);
      // pass 1: maxima (columns k >= n1 and empty token slots hold zeros)
      float tm = 0.f;
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32(tD + lane_off + uint32_t(part * COLS + 32 * c), u);
        tmem_wait_ld();
        if (GRAN == FQ_DYNAMIC_GROUP) {
          // group of element (k, l): (k * n2 + l) / 128, i.e. k (n2 = 128) or k / 2 (n2 = 64)
          constexpr int KPG = 128 / N2;  // columns k per group
#pragma unroll
          for (int j = 0; j < 32; j += KPG) {
            float a = fabsf(__uint_as_float(u[j]));
            if (KPG == 2) a = fmaxf(a, fabsf(__uint_as_float(u[j + 1])));
            const uint32_t r = warp_max_u32(__float_as_uint(a * up));
            const int g = (part * COLS + 32 * c + j) / KPG;
            if (lane == 0) atomicMax(&gmax[s * 128 + g], r);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) tm = fmaxf(tm, fabsf(__uint_as_float(u[j])));
        }
      }
      float s_tok = 0.f, f_tok = 0.f;
      if (GRAN == FQ_DYNAMIC_ROW) {
        const uint32_t r = warp_max_u32(__float_as_uint(tm * up));
        if (lane == 0) red[C::R_TMAX + pw] = __uint_as_float(r);
        named_barrier(bar_id, C::TPP);
        // warps holding the rows of token s: quadrants 2s, 2s + 1 (n2 = 64) or all four
        float amax = 0.f;
#pragma unroll
        for (int pp = 0; pp < C::KSPLIT; ++pp) {
          if (N2 == 64) {
            amax = fmaxf(amax, red[C::R_TMAX + pp * 4 + 2 * s]);
            amax = fmaxf(amax, red[C::R_TMAX + pp * 4 + 2 * s + 1]);
          } else {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) amax = fmaxf(amax, red[C::R_TMAX + pp * 4 + qq]);
          }
        }
        s_tok = __fdiv_rn(__fmul_rn(amax, p.alpha), 7.0f);
        f_tok = s_tok != 0.f ? (1.0f / s_tok) * up : 0.f;
        if (tok_ok && l == 0 && part == 0) p.s_row[tok] = s_tok;
      } else if (GRAN == FQ_DYNAMIC_GROUP) {
        named_barrier(bar_id, C::TPP);
        const int ngr = n1 * N2 / 128;  // groups per token
        for (int e = ptid; e < G * ngr; e += C::TPP) {
          const int ts = e / ngr, g = e - ts * ngr;
          const __half sh = group_scale(__uint_as_float(gmax[ts * 128 + g]), p.alpha);
          const float sg = __half2float(sh);
          red[C::R_SG + ts * 128 + g] = sg;
          red[C::R_SINV + ts * 128 + g] = sg != 0.f ? 1.0f / sg : 0.f;
          if (tok0 + ts < M) p.s_grp[size_t(g) * M + tok0 + ts] = sh;
        }
        named_barrier(bar_id, C::TPP);
      }
      // pass 2: codes, 8 columns k per 32-bit word, transposed to 8 columns l.
      // Two values at a time (f32x2): x = fma(d, f, 1.5 * 2^23) holds the
      // round-half-even integer of d * f (= v / s up to the rounding of 1/s)
      // in its low mantissa bits, so its low 4 bits are the two's-complement
      // nibble; t = d * f - that integer (exact residual) flags the values
      // next to a tie, where the IEEE quotient decides (code_of).  |v / s|
      // stays below 7.5 when alpha >= 1, so the clamp to [-8, 7] is needed
      // only for alpha < 1.
      constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
      const float2 cc = make_float2(kMagic, kMagic), m1 = make_float2(-1.f, -1.f);
      const float th = 0.5f - (8.0f / fminf(p.alpha, 1.0f) + 1.0f) * 9.5367431640625e-07f;  // tie band
      const bool clamp = !(p.alpha >= 1.0f);
#pragma unroll
      for (int c = 0; c < COLS / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32(tD + lane_off + uint32_t(part * COLS + 32 * c), u);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int k0 = part * COLS + 32 * c + 8 * ch;
          const uint32_t* uc = u + 8 * ch;
          uint32_t word = 0;
          if (GRAN == FQ_STATIC_CHANNEL) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int k = k0 + j;
              const int qv = k < n1 ? code_of(__uint_as_float(uc[j]) * up, __ldg(p.sstatic + k * N2 + l)) : 0;
              word = put_nibble(word, qv, 4 * j);
            }
          } else {
            bool redo = false;  // a value next to a tie, or a zero scale: the IEEE path decides
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
              const int k = k0 + j;
              const float2 dd = make_float2(__uint_as_float(uc[j]), __uint_as_float(uc[j + 1]));
              float2 ff;
              if (GRAN == FQ_DYNAMIC_ROW) {
                ff = make_float2(f_tok, f_tok);
              } else {
                const int g0 = k * N2 / 128, g1 = (k + 1) * N2 / 128;
                ff = fmul2(make_float2(red[C::R_SINV + s * 128 + g0], red[C::R_SINV + s * 128 + g1]),
                           make_float2(up, up));
                redo |= red[C::R_SG + s * 128 + g0] == 0.f || red[C::R_SG + s * 128 + g1] == 0.f;
              }
              float2 x = ffma2(dd, ff, cc);                      // 1.5 * 2^23 + rint(d f)
              const float2 t = ffma2(dd, ff, ffma2(x, m1, cc));  // d f - rint(d f)
              if (clamp) {
                x.x = fminf(fmaxf(x.x, kMagic - 8.0f), kMagic + 7.0f);
                x.y = fminf(fmaxf(x.y, kMagic - 8.0f), kMagic + 7.0f);
              }
              redo |= fabsf(t.x) >= th || fabsf(t.y) >= th;
              word = put_nibble(word, int(__float_as_uint(x.x)), 4 * j);
              word = put_nibble(word, int(__float_as_uint(x.y)), 4 * j + 4);
            }
            if (GRAN == FQ_DYNAMIC_ROW) redo |= s_tok == 0.f;
            if (redo) {
              word = 0;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int k = k0 + j;
                const float sk = GRAN == FQ_DYNAMIC_ROW ? s_tok : red[C::R_SG + s * 128 + k * N2 / 128];
                word = put_nibble(word, code_of(__uint_as_float(uc[j]) * up, sk), 4 * j);
              }
            }
          }
          if (p.xhat && tok_ok) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (k0 + j < n1) p.xhat[size_t(tok) * K + (k0 + j) * N2 + l] = __uint_as_float(uc[j]) * up;
          }
          word = transpose_nibbles8(word, lane);
          const int kr = k0 + (lane & 7);
          const int l0 = l & ~7;
          if (tok_ok && kr < n1)
            *reinterpret_cast<uint32_t*>(p.Q + size_t(tok) * (K / 2) + (kr * N2 + l0) / 2) = word;
        }
      }
    }
    tc_fence_before();
    bad = named_barrier_or(bar_id, C::TPP, bad);  // D, U^T and the scratch are free again
    if (bad) break;
  }
  if (bad && ptid == 0) record_error(p.err, kErrTimeoutMma);

  // a copy still in flight after an early exit lands before the CTA leaves
  if (!HAS_C && leader && x_pending && !mbar_wait(xfull, ph)) record_error(p.err, kErrTimeoutDrain);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int N2, int NP, int GRAN, bool HAS_C>
fq_status launch_tc4(const QuantTcParams& p, cudaStream_t stream) {
  using C = TcCfg<N2, NP, HAS_C>;
  CUtensorMap tm;
  // X viewed as [M * n1 rows][n2] fp16; one box = 64 columns (128 bytes) x n1 rows
  fq_status st = make_tmap_2d(&tm, p.X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, uint64_t(p.n2), uint64_t(p.M) * p.n1,
                              uint64_t(p.n2) * 2, 64u, uint32_t(p.n1), CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != FQ_OK) return st;
  auto kern = quant_act_tc_kernel<N2, NP, GRAN, HAS_C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the transform kernel", C::SMEM);
  const int ngroups = (p.M + C::G - 1) / C::G;
  const int grid = std::max(1, std::min((ngroups + C::P - 1) / C::P, sm_count()));
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kTcThreads), C::SMEM, stream, p, tm);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FQ_ERR_CUDA, "quant_act_tc_kernel: %s", cudaGetErrorString(e));
  }
  return check_launch("quant_act_tc_kernel");
}

template <int N2, int NP, bool HAS_C>
fq_status launch_tc3(const QuantTcParams& p, cudaStream_t stream) {
  if (p.gran == FQ_DYNAMIC_ROW) return launch_tc4<N2, NP, FQ_DYNAMIC_ROW, HAS_C>(p, stream);
  if (p.gran == FQ_DYNAMIC_GROUP) return launch_tc4<N2, NP, FQ_DYNAMIC_GROUP, HAS_C>(p, stream);
  return launch_tc4<N2, NP, FQ_STATIC_CHANNEL, HAS_C>(p, stream);
}

template <int N2, int NP>
fq_status launch_tc(const QuantTcParams& p, cudaStream_t stream) {
  return p.c ? launch_tc3<N2, NP, true>(p, stream) : launch_tc3<N2, NP, false>(p, stream);
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
