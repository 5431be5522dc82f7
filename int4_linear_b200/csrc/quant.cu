// Row quantization kernels: online activation quantization (fq_quant_act)
// and offline weight quantization (fq_quant_weight).
//
// One CTA owns one row at a time (grid-stride over rows), keeps the whole
// row in shared memory as float32, and in order:
//   1. loads the fp16 row with 128-bit loads and applies the channel scale
//      (activations: x * c; weights: w / c)  (FlatQuant notes, 逐通道缩放);
//   2. applies the Kronecker-factored transform on the n1 x n2 reshape,
//      activations P1^T Xbar P2, weights P1^-1 Wbar P2^-T (FlatQuant notes,
//      Kronecker 分解), as two in-place passes: first every tile row times the
//      right factor, then every tile column times the left factor;
//   3. weights only: folds the static activation scales s_k into the columns
//      (MergeQuant, quantization step migration);
//   4. reduces the absmax per row or per 128-group with warp shuffles, forms
//      s = (amax * alpha) / 7 (group scales rounded to fp16), or reads the
//      static scales (FRM-PTQ page, 初步介绍; FlatQuant notes, 可学习裁剪阈值);
//   5. rounds half-to-even after an IEEE division, clamps to [-8, 7], packs
//      two codes per byte and stores 32 bits per thread, coalesced.
// The transform factors live in shared memory (read once per CTA) when they
// fit, otherwise they are read through L1.
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
  long long sg_g, sg_m;
  float* xhat;
  unsigned* err;
};
bool quant_act_tc_supported(int K, int n1, int n2);
fq_status launch_quant_act_tc(const QuantTcParams& p, cudaStream_t stream);

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemBudget = 220 * 1024;

enum Side { kAct = 0, kWeight = 1 };

struct QuantParams {
  const __half* X;
  int R, K;
  int gran;
  float alpha;
  int n1, n2;            // transform tile (0 = none)
  const float* L;        // P1 (act) or P1^-1 (weight), [n1][n1]
  const float* Rt;       // P2 (act) or P2^-1 (weight), [n2][n2]
  const float* c;        // [K] or null
  const float* qsm;      // weights: [K] or null
  const float* sstatic;  // act static: [K]
  uint8_t* Q;            // [R][K/2]
  float* s_row;          // [R]
  __half* s_grp;         // [K/128][R]
  float* xhat;           // [R][K] or null
  // general quantizer (per-row min-max zero point, b = 3 or 4): per row the
  // offset o = 2^(b-1) - z and the sum of the stored signed codes
  int asym, bits;
  int32_t* zoff;         // [R]
  int32_t* zsum;         // [R]
};

// Left factor as used by the column pass: Lc(k, i) multiplies U[i][l] into
// Xhat[k][l].  Activations: P1^T, so Lc(k, i) = P1[i][k]; weights: P1^-1.
template <int SIDE>
__device__ __forceinline__ float left_at(const float* L, int n1, int k, int i) {
  if (!L) return k == i ? 1.f : 0.f;  // P1 = I
  return SIDE == kAct ? L[i * n1 + k] : L[k * n1 + i];
}
// Right factor as used by the row pass: Rr(j, l) multiplies Xbar[i][j] into
// U[i][l].  Activations: P2, so Rr(j, l) = P2[j][l]; weights: P2^-T.
template <int SIDE>
__device__ __forceinline__ float right_at(const float* Rt, int n2, int j, int l) {
  return SIDE == kAct ? Rt[j * n2 + l] : Rt[l * n2 + j];
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Index of flat element e in the row buffer: padded by one float per tile row
// when a transform is applied, so that the column pass is free of bank conflicts.
__device__ __forceinline__ int slot(int e, int n2, int pad) { return pad ? (e / n2) * (n2 + 1) + (e % n2) : e; }

// An unsigned 128-bit integer (hi, lo) rounded once to the nearest float64:
// the top 64 significant bits, with every bit below them folded into a
// sticky bit 0, are rounded by the 64-bit conversion (its rounding position
// lies 11 bits above bit 0), then scaled by the exact power of two.
__device__ __forceinline__ double u128_to_double_rn(unsigned long long hi, unsigned long long lo) {
  if (hi == 0) return __ull2double_rn(lo);
  const int lz = __clzll(static_cast<long long>(hi));
  const unsigned long long top = lz ? (hi << lz) | (lo >> (64 - lz)) : hi;
  const unsigned long long rest = lz ? (lo << lz) : lo;
  return ldexp(__ull2double_rn(top | (rest ? 1ull : 0ull)), 64 - lz);
}

template <int SIDE, bool PSMEM>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(QuantParams p) {
  extern __shared__ __align__(16) float smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, n1 = p.n1, n2 = p.n2;
  const bool xf = n1 > 0;
  const int pad = xf ? 1 : 0;
  const int row_floats = xf ? n1 * (n2 + 1) : K;
  float* xs = smem;                       // row buffer
  // activations with a transform: the fp16 input row, tile rows padded to
  // n2 + 2 halves (an odd word stride: lane-per-row reads are conflict-free)
  __half* xin = reinterpret_cast<__half*>(xs + row_floats);
  const int xstride = n2 + 2;
  const int xin_floats = (SIDE == kAct && xf) ? (n1 * xstride + 1) / 2 : 0;
  float* sL = xs + row_floats + xin_floats;  // [i][k] = Lc(k, i)   (PSMEM)
  float* sR = sL + (PSMEM ? n1 * n1 : 0); // [j][l] = Rr(j, l)   (PSMEM)
  float* red = sR + (PSMEM ? n2 * n2 : 0);  // [4][kWarps] (8-byte aligned when there is no transform)
  float* gsc = red + 4 * kWarps;            // [K/128] group scales

  if (PSMEM && xf) {
    for (int e = tid; e < n1 * n1; e += kThreads) {
      const int i = e / n1, k = e % n1;
      sL[e] = left_at<SIDE>(p.L, n1, k, i);
    }
    for (int e = tid; e < n2 * n2; e += kThreads) {
      const int j = e / n2, l = e % n2;
      sR[e] = right_at<SIDE>(p.Rt, n2, j, l);
    }
  }
  __syncthreads();

  const int ngroups = K / kGroup;
  for (int r = blockIdx.x; r < p.R; r += gridDim.x) {
    // 1. load + channel scale (activations with a transform: the fp16 row as
    // is; c is applied in float64 inside the transform)
    const __half* xrow = p.X + size_t(r) * K;
    if (SIDE == kAct && xf) {
      for (int e0 = tid * 8; e0 < K; e0 += kThreads * 8) {
        const uint4 raw = *reinterpret_cast<const uint4*>(xrow + e0);
        const __half* h = reinterpret_cast<const __half*>(&raw);
#pragma unroll
        for (int j = 0; j < 8; ++j) xin[((e0 + j) / n2) * xstride + (e0 + j) % n2] = h[j];
      }
    }
    for (int e0 = tid * 8; e0 < K && !(SIDE == kAct && xf); e0 += kThreads * 8) {
      const uint4 raw = *reinterpret_cast<const uint4*>(xrow + e0);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h2[j]);
        float v0 = f.x, v1 = f.y;
        if (p.c) {
          if (SIDE == kAct) {
            v0 = __fmul_rn(v0, p.c[e0 + 2 * j]);
            v1 = __fmul_rn(v1, p.c[e0 + 2 * j + 1]);
          } else {
            v0 = __fdiv_rn(v0, p.c[e0 + 2 * j]);
            v1 = __fdiv_rn(v1, p.c[e0 + 2 * j + 1]);
          }
        }
        xs[slot(e0 + 2 * j, n2, pad)] = v0;
        xs[slot(e0 + 2 * j + 1, n2, pad)] = v1;
      }
    }
    __syncthreads();

    // 1b. per-token residual scaling (FPTQuant S_n): the token's sum of
    // squares taken exactly -- every fp16 square is an integer multiple of
    // 2^-48 below 2^82, so a 128-bit integer sum of K <= 2^16 of them cannot
    // overflow -- rounded once to float64, then /K, sqrt and float32; then
    // v = fl32(x / S_n) in place (v = 0 unless S_n > 0).  Non-finite
    // entries give S_n = +inf (an infinity) or NaN (a NaN), as the float64
    // sum would.
    if (SIDE == kAct && p.gran == FQ_STATIC_RESIDUAL) {
      unsigned long long lo = 0, hi = 0;
      unsigned nonfin = 0;
      for (int e = tid; e < K; e += kThreads) {
        const unsigned h = __half_as_ushort(__float2half_rn(xs[e]));  // exact: xs holds fp16 values
        const unsigned E = (h >> 10) & 31u, F = h & 1023u;
        if (E == 31u) {
          nonfin |= F ? 2u : 1u;
          continue;
        }
        const unsigned long long m = E ? (F | 1024u) : F;
        const unsigned long long m2 = m * m;  // x^2 = m2 * 2^(2E-50), or m2 * 2^-48 when E = 0
        const int sh = E ? int(2 * E) - 2 : 0;  // in units of 2^-48, at most 58
        const unsigned long long alo = m2 << sh, ahi = sh ? m2 >> (64 - sh) : 0ull;
        lo += alo;
        hi += ahi + (lo < alo ? 1ull : 0ull);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long olo = __shfl_xor_sync(0xffffffffu, lo, o);
        const unsigned long long ohi = __shfl_xor_sync(0xffffffffu, hi, o);
        lo += olo;
        hi += ohi + (lo < olo ? 1ull : 0ull);
      }
      nonfin = __reduce_or_sync(0xffffffffu, nonfin);
      unsigned long long* red64 = reinterpret_cast<unsigned long long*>(red);  // [kWarps][2]
      if (lane == 0) {
        red64[2 * warp] = lo;
        red64[2 * warp + 1] = hi | (static_cast<unsigned long long>(nonfin) << 62);  // hi < 2^32
      }
      __syncthreads();
      unsigned long long tlo = 0, thi = 0;
      unsigned tnf = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const unsigned long long wlo = red64[2 * w], whi = red64[2 * w + 1];
        tlo += wlo;
        thi += (whi & ((1ull << 62) - 1)) + (tlo < wlo ? 1ull : 0ull);
        tnf |= unsigned(whi >> 62);
      }
      float s_n;
      if (tnf & 2u)
        s_n = __int_as_float(0x7fc00000);
      else if (tnf)
        s_n = __int_as_float(0x7f800000);
      else
        s_n = __double2float_rn(sqrt(u128_to_double_rn(thi, tlo) * 0x1p-48 / double(K)));
      __syncthreads();  // every thread has read red64
      if (tid == 0) p.s_row[r] = s_n;
      for (int e = tid; e < K; e += kThreads) xs[e] = s_n > 0.f ? __fdiv_rn(xs[e], s_n) : 0.f;
      __syncthreads();
    }

    // 2. transform
    if (SIDE == kAct && xf) {
      // Activations: every product and sum in float64 (the fp16 inputs, c
      // and the float32 factors are exact in it), one rounding to float32
      // per element.  A warp takes 4 columns l at a time: lane owns the
      // tile rows i = lane + 32 q for U[i][l] = sum_j Xbar[i][j] P2[j][l],
      // then the outputs k = lane + 32 q of Xhat[k][l] = sum_i P1[i][k] U[i][l],
      // each U[i][l] broadcast from its owner lane.
      constexpr int CB = 4, NQ = 8;  // n1 <= 256
      const int nq = (n1 + 31) / 32;
      for (int l0 = warp * CB; l0 < n2; l0 += kWarps * CB) {
        double acc[NQ][CB];
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int c = 0; c < CB; ++c) acc[q][c] = 0.0;
        for (int j = 0; j < n2; ++j) {
          double pv[CB];
#pragma unroll
          for (int c = 0; c < CB; ++c)
            pv[c] = l0 + c < n2 ? double(PSMEM ? sR[j * n2 + l0 + c] : right_at<SIDE>(p.Rt, n2, j, l0 + c)) : 0.0;
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const int i = lane + 32 * q;
            if (q < nq) {
              double x = i < n1 ? double(__half2float(xin[i * xstride + j])) : 0.0;
              if (p.c && i < n1) x *= double(__ldg(p.c + i * n2 + j));
#pragma unroll
              for (int c = 0; c < CB; ++c) acc[q][c] = fma(x, pv[c], acc[q][c]);
            }
          }
        }
        double out[NQ][CB];
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int c = 0; c < CB; ++c) out[q][c] = 0.0;
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
          if (qi >= nq) break;
          for (int ii = 0; ii < 32; ++ii) {
            const int i = 32 * qi + ii;
            if (i >= n1) break;
            double u[CB];
#pragma unroll
            for (int c = 0; c < CB; ++c) u[c] = __shfl_sync(0xffffffffu, acc[qi][c], ii);
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              const int k = lane + 32 * q;
              if (q < nq) {
                const double lv = k < n1 ? double(PSMEM ? sL[i * n1 + k] : left_at<SIDE>(p.L, n1, k, i)) : 0.0;
#pragma unroll
                for (int c = 0; c < CB; ++c) out[q][c] = fma(lv, u[c], out[q][c]);
              }
            }
          }
        }
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int k = lane + 32 * q;
          if (q < nq && k < n1) {
#pragma unroll
            for (int c = 0; c < CB; ++c)
              if (l0 + c < n2) xs[k * (n2 + 1) + l0 + c] = float(out[q][c]);
          }
        }
      }
      __syncthreads();
    } else if (xf) {
      // row pass: U[i][l] = sum_j Xbar[i][j] Rr(j, l), rows split over warps
      for (int i = warp; i < n1; i += kWarps) {
        float acc[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[t] = 0.f;
        const float* xr = xs + i * (n2 + 1);
        for (int j = 0; j < n2; ++j) {
          const float x = xr[j];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int l = lane + 32 * t;
            if (l < n2) {
              const float rv = PSMEM ? sR[j * n2 + l] : right_at<SIDE>(p.Rt, n2, j, l);
              acc[t] = fmaf(x, rv, acc[t]);
            }
          }
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int l = lane + 32 * t;
          if (l < n2) xs[i * (n2 + 1) + l] = acc[t];
        }
      }
      __syncthreads();
      // column pass: Xhat[k][l] = sum_i Lc(k, i) U[i][l], columns split over warps
      for (int l = warp; l < n2; l += kWarps) {
        float acc[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[t] = 0.f;
        for (int i = 0; i < n1; ++i) {
          const float u = xs[i * (n2 + 1) + l];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int k = lane + 32 * t;
            if (k < n1) {
              const float lv = PSMEM ? sL[i * n1 + k] : left_at<SIDE>(p.L, n1, k, i);
              acc[t] = fmaf(lv, u, acc[t]);
            }
          }
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int k = lane + 32 * t;
          if (k < n1) xs[k * (n2 + 1) + l] = acc[t];
        }
      }
      __syncthreads();
    }

    // 3. weights: quantization step migration
    if (SIDE == kWeight && p.qsm) {
      for (int e = tid; e < K; e += kThreads) xs[slot(e, n2, pad)] = __fmul_rn(xs[slot(e, n2, pad)], p.qsm[e]);
      __syncthreads();
    }

    if (p.xhat) {
      float* xo = p.xhat + size_t(r) * K;
      for (int e = tid; e < K; e += kThreads) xo[e] = xs[slot(e, n2, pad)];
    }

    // 4. scales
    float s_row = 0.f;
    int z_row = 0;
    if (p.asym) {
      // Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) with the row's range widened
      // to contain 0: lo = min(0, min v), hi = max(0, max v),
      // s = ((hi - lo) alpha) / (2^b - 1), z = clamp(round(-lo / s), 0, 2^b - 1)
      float mn = 0.f, mx = 0.f;
      for (int e = tid; e < K; e += kThreads) {
        const float v = xs[slot(e, n2, pad)];
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        red[warp] = mn;
        red[kWarps + warp] = mx;
      }
      __syncthreads();
      float lo = red[0], hi = red[kWarps];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) {
        lo = fminf(lo, red[w]);
        hi = fmaxf(hi, red[kWarps + w]);
      }
      const float qmax = float((1 << p.bits) - 1);
      s_row = __fdiv_rn(__fmul_rn(__fsub_rn(hi, lo), p.alpha), qmax);
      z_row = s_row == 0.f ? 0 : int(fminf(fmaxf(rintf(__fdiv_rn(-lo, s_row)), 0.f), qmax));
      if (tid == 0) {
        p.s_row[r] = s_row;
        p.zoff[r] = (1 << (p.bits - 1)) - z_row;
      }
    } else if (p.gran == FQ_DYNAMIC_ROW) {
      float m = 0.f;
      for (int e = tid; e < K; e += kThreads) m = fmaxf(m, fabsf(xs[slot(e, n2, pad)]));
      m = warp_max(m);
      if (lane == 0) red[warp] = m;
      __syncthreads();
      float amax = red[0];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) amax = fmaxf(amax, red[w]);
      s_row = __fdiv_rn(__fmul_rn(amax, p.alpha), 7.0f);
      if (tid == 0) p.s_row[r] = s_row;
    } else if (p.gran == FQ_DYNAMIC_GROUP) {
      for (int g = warp; g < ngroups; g += kWarps) {
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) m = fmaxf(m, fabsf(xs[slot(g * kGroup + lane + 32 * t, n2, pad)]));
        m = warp_max(m);
        const __half sh = __float2half_rn(__fdiv_rn(__fmul_rn(m, p.alpha), 7.0f));
        if (lane == 0) {
          gsc[g] = __half2float(sh);
          p.s_grp[size_t(g) * p.R + r] = sh;
        }
      }
      __syncthreads();
    }

    // 5. codes, packed 8 per thread-iteration (one 32-bit store)
    uint32_t* qrow = reinterpret_cast<uint32_t*>(p.Q + size_t(r) * (K / 2));
    if (p.asym) {
      // u = clamp(round(v / s) + z, 0, 2^b - 1) (u = z when s = 0), stored as
      // the signed nibble q = u - 2^(b-1); the row's sum of q goes with it
      const int qmax = (1 << p.bits) - 1, half = 1 << (p.bits - 1);
      int sum = 0;
      for (int e0 = tid * 8; e0 < K; e0 += kThreads * 8) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v = xs[slot(e0 + j, n2, pad)];
          int u = z_row;
          if (s_row != 0.f) u = min(max(int(rintf(__fdiv_rn(v, s_row))) + z_row, 0), qmax);
          const int q = u - half;
          sum += q;
          word |= (uint32_t(q) & 0xFu) << (4 * j);
        }
        qrow[e0 / 8] = word;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncthreads();  // red is free again
      if (lane == 0) reinterpret_cast<int*>(red)[warp] = sum;
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < kWarps; ++w) tot += reinterpret_cast<int*>(red)[w];
        p.zsum[r] = tot;
      }
      __syncthreads();
      continue;
    }
    for (int e0 = tid * 8; e0 < K; e0 += kThreads * 8) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = e0 + j;
        const float v = xs[slot(e, n2, pad)];
        float s;
        if (p.gran == FQ_DYNAMIC_ROW)
          s = s_row;
        else if (p.gran == FQ_DYNAMIC_GROUP)
          s = gsc[e / kGroup];
        else
          s = p.sstatic[e];  // static, and static after the residual scaling
        word |= (uint32_t(rtn_code(v, s)) & 0xFu) << (4 * j);
      }
      qrow[e0 / 8] = word;
    }
    __syncthreads();
  }
}

// Static per-channel activation scales with no Kronecker transform: every
// element is independent (q = clamp(rint(x c / s_k))), so the elements are
// spread over the whole grid, 8 per thread-iteration (one 16-byte load, one
// 32-bit packed store), instead of one CTA per token row.
__global__ void __launch_bounds__(kThreads) quant_static_kernel(QuantParams p) {
  const size_t pieces = size_t(p.R) * (p.K / 8);
  const int kp = p.K / 8;
  for (size_t pc = blockIdx.x * size_t(kThreads) + threadIdx.x; pc < pieces; pc += size_t(gridDim.x) * kThreads) {
    const int r = int(pc / kp), e0 = int(pc % kp) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(p.X + size_t(r) * p.K + e0);
    float v[8];
    const uint32_t word = static_codes8(raw, p.sstatic + e0, p.c ? p.c + e0 : nullptr, v);
    reinterpret_cast<uint32_t*>(p.Q + size_t(r) * (p.K / 2))[e0 / 8] = word;
    if (p.xhat) {
      float4* xo = reinterpret_cast<float4*>(p.xhat + size_t(r) * p.K + e0);
      xo[0] = make_float4(v[0], v[1], v[2], v[3]);
      xo[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

fq_status launch_quant_static(const QuantParams& qp, cudaStream_t stream) {
  const size_t pieces = size_t(qp.R) * (qp.K / 8);
  const size_t want = (pieces + kThreads - 1) / kThreads;
  const int grid = int(std::max<size_t>(1, std::min<size_t>(want, size_t(sm_count()) * 8)));
  quant_static_kernel<<<grid, kThreads, 0, stream>>>(qp);
  return check_launch("quant_static_kernel");
}

size_t smem_bytes(int K, int n1, int n2, bool psmem, bool act) {
  const size_t row = n1 > 0 ? size_t(n1) * (n2 + 1) + (act ? (size_t(n1) * (n2 + 2) + 1) / 2 : 0) : size_t(K);
  const size_t pm = (psmem && n1 > 0) ? size_t(n1) * n1 + size_t(n2) * n2 : 0;
  return (row + pm + 4 * kWarps + K / kGroup) * sizeof(float);
}

template <int SIDE, bool PSMEM>
fq_status launch_quant(const QuantParams& qp, cudaStream_t stream) {
  const size_t smem = smem_bytes(qp.K, qp.n1, qp.n2, PSMEM, SIDE == kAct);
  auto kern = quant_rows_kernel<SIDE, PSMEM>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return fail(FQ_ERR_CUDA, "cannot reserve %zu bytes of shared memory", smem);
  }
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess) per_sm = 1;
  per_sm = std::max(per_sm, 1);
  const int grid = std::max(1, std::min(qp.R, sm_count() * per_sm));
  kern<<<grid, kThreads, smem, stream>>>(qp);
  return check_launch("quant_rows_kernel");
}

fq_status check_qparams(const fq_qparams* qp, bool act) {
  FQ_CHECK_ARG(qp != nullptr, "qparams is NULL");
  if (qp->zero_point == FQ_ZERO_POINT_MINMAX) {
    // the general quantizer: b = 3 or 4, per-row scale and zero point
    if (qp->bits != 3 && qp->bits != 4)
      return fail(FQ_ERR_UNSUPPORTED, "bits = %d: the min-max quantizer provides b = 3 and 4", qp->bits);
    if (qp->gran != FQ_DYNAMIC_ROW)
      return fail(FQ_ERR_UNSUPPORTED, "the min-max quantizer is per row (FQ_DYNAMIC_ROW) only");
  } else {
    if (qp->bits != 4) return fail(FQ_ERR_UNSUPPORTED, "bits = %d: the symmetric quantizer provides b = 4", qp->bits);
    if (qp->zero_point != 8)
      return fail(FQ_ERR_UNSUPPORTED,
                  "zero_point = %d: provided are the symmetric z = 2^(b-1) = 8 and FQ_ZERO_POINT_MINMAX",
                  qp->zero_point);
  }
  if (qp->gran == FQ_DYNAMIC_GROUP && qp->group_size != kGroup)
    return fail(FQ_ERR_UNSUPPORTED, "group_size = %d: only 128 is provided", qp->group_size);
  if (qp->gran != FQ_DYNAMIC_ROW && qp->gran != FQ_DYNAMIC_GROUP &&
      !(act && (qp->gran == FQ_STATIC_CHANNEL || qp->gran == FQ_STATIC_RESIDUAL)))
    return fail(FQ_ERR_UNSUPPORTED, "granularity %d is not provided here", int(qp->gran));
  if (qp->gran != FQ_STATIC_CHANNEL && qp->gran != FQ_STATIC_RESIDUAL)
    FQ_CHECK_ARG(qp->alpha > 0.f && qp->alpha <= 1.f, "alpha = %g must lie in (0, 1]", double(qp->alpha));
  return FQ_OK;
}

// dry: validate every argument as for a launch, launch nothing.  sg_g, sg_m
// (0: the default group-major [K/128][R]) are element strides of the group
// scales; only the tensor-core transform kernel takes other strides.
fq_status quant_common(int side, const uint16_t* X, int R, int K, const fq_qparams* qp, const fq_transform* t,
                       const float* extra, uint8_t* Q, void* s_out, float* xhat, void* stream, bool dry = false,
                       long long sg_g = 0, long long sg_m = 0) {
  clear_error();
  fq_status st = check_qparams(qp, side == kAct);
  if (st != FQ_OK) return st;
  FQ_CHECK_ARG(X && Q, "X and the packed output must be non-NULL");
  FQ_CHECK_ARG(R >= 1, "rows = %d must be >= 1", R);
  FQ_CHECK_ARG(K >= kGroup && K <= kMaxQuantK && K % kGroup == 0, "K = %d must be a multiple of 128 in [128, %d]",
               K, kMaxQuantK);
  FQ_CHECK_ARG(aligned(X, 16) && aligned(Q, 16), "X and the packed output must be 16-byte aligned");
  if (qp->gran == FQ_STATIC_CHANNEL || qp->gran == FQ_STATIC_RESIDUAL)
    FQ_CHECK_ARG(extra && aligned(extra, 4), "static scales [K] are required for the static granularities");
  if (qp->gran != FQ_STATIC_CHANNEL)
    FQ_CHECK_ARG(s_out && aligned(s_out, 4), "the scale output must be non-NULL and aligned");
  if (qp->gran == FQ_STATIC_RESIDUAL && t && (t->P1 || t->P2 || t->c))
    return fail(FQ_ERR_UNSUPPORTED, "FQ_STATIC_RESIDUAL takes no transform and no c");
  QuantParams p{};
  p.X = reinterpret_cast<const __half*>(X);
  p.R = R;
  p.K = K;
  p.gran = int(qp->gran);
  p.alpha = qp->alpha;
  p.Q = Q;
  p.xhat = xhat;
  if (qp->gran == FQ_DYNAMIC_ROW || qp->gran == FQ_STATIC_RESIDUAL) p.s_row = static_cast<float*>(s_out);
  if (qp->zero_point == FQ_ZERO_POINT_MINMAX) {
    // scale block: float32 s[R], int32 o[R] = 2^(b-1) - z, int32 code sums[R]
    p.asym = 1;
    p.bits = qp->bits;
    p.zoff = reinterpret_cast<int32_t*>(static_cast<float*>(s_out) + R);
    p.zsum = reinterpret_cast<int32_t*>(static_cast<float*>(s_out) + 2 * size_t(R));
  }
  if (qp->gran == FQ_DYNAMIC_GROUP) p.s_grp = static_cast<__half*>(s_out);
  if (side == kAct && (qp->gran == FQ_STATIC_CHANNEL || qp->gran == FQ_STATIC_RESIDUAL)) p.sstatic = extra;
  if (side == kWeight) p.qsm = extra;
  if (t) {
    p.c = t->c;
    if (t->c) FQ_CHECK_ARG(aligned(t->c, 4), "c must be 4-byte aligned");
    if (t->P1 || t->P2) {
      FQ_CHECK_ARG(t->P2 != nullptr, "P2 is NULL while P1 is given");
      FQ_CHECK_ARG(t->n1 >= 1 && t->n2 >= 1 && t->n1 <= 256 && t->n2 <= 256 && t->n1 * t->n2 == K,
                   "transform tile %d x %d must satisfy n1 * n2 = K = %d with 1 <= n1, n2 <= 256", t->n1, t->n2,
                   K);
      p.n1 = t->n1;
      p.n2 = t->n2;
      p.L = t->P1;
      p.Rt = t->P2;
    }
  }
  if (dry) return FQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (side == kAct && p.n1 > 0 && !p.asym && quant_act_tc_supported(K, p.n1, p.n2)) {
    // activations with the transform: tensor-core kernel
    unsigned* err = device_error_word();
    if (!err) return fail(FQ_ERR_CUDA, "device error word unavailable");
    QuantTcParams tp{};
    tp.X = p.X;
    tp.M = R;
    tp.K = K;
    tp.n1 = p.n1;
    tp.n2 = p.n2;
    tp.gran = p.gran;
    tp.alpha = p.alpha;
    tp.P1 = p.L;
    tp.P2 = p.Rt;
    tp.c = p.c;
    tp.sstatic = p.sstatic;
    tp.Q = p.Q;
    tp.s_row = p.s_row;
    tp.s_grp = p.s_grp;
    tp.sg_g = sg_g ? sg_g : R;
    tp.sg_m = sg_g ? sg_m : 1;
    tp.xhat = p.xhat;
    tp.err = err;
    return launch_quant_act_tc(tp, s);
  }
  // static scales without a transform: element-parallel kernel (its vector
  // loads need 16-byte aligned scales and c; otherwise the row kernel runs)
  if (side == kAct && qp->gran == FQ_STATIC_CHANNEL && p.n1 == 0 && aligned(extra, 16) &&
      (!p.c || aligned(p.c, 16)))
    return launch_quant_static(p, s);
  const bool act = side == kAct;
  const bool psmem = smem_bytes(K, p.n1, p.n2, true, act) <= size_t(kSmemBudget);
  if (smem_bytes(K, p.n1, p.n2, false, act) > size_t(kSmemBudget))
    return fail(FQ_ERR_UNSUPPORTED, "row of K = %d does not fit in shared memory", K);
  if (side == kAct) return psmem ? launch_quant<kAct, true>(p, s) : launch_quant<kAct, false>(p, s);
  return psmem ? launch_quant<kWeight, true>(p, s) : launch_quant<kWeight, false>(p, s);
}

}  // namespace

// The checks of fq_quant_act, with nothing launched (the fused decode linear
// quantizes inside the GEMM launch).
fq_status check_act_args(const uint16_t* X, int M, int K, const fq_qparams* qp, const fq_transform* t,
                         const float* static_scale, uint8_t* Xq, void* s_x) {
  return quant_common(kAct, X, M, K, qp, t, static_scale, Xq, s_x, nullptr, nullptr, true);
}

}  // namespace fq

extern "C" {

fq_status fq_quant_weight(const uint16_t* W, int N, int K, const fq_qparams* qp, const fq_transform* inv,
                          const float* qsm_scale, uint8_t* Wq, void* s_w, void* stream) {
  return fq::quant_common(fq::kWeight, W, N, K, qp, inv, qsm_scale, Wq, s_w, nullptr, stream);
}

fq_status fq_quant_act(const uint16_t* X, int M, int K, const fq_qparams* qp, const fq_transform* t,
                       const float* static_scale, uint8_t* Xq, void* s_x, void* stream) {
  return fq::quant_common(fq::kAct, X, M, K, qp, t, static_scale, Xq, s_x, nullptr, stream);
}

fq_status fq_quant_kv(const uint16_t* KV, int T, int H, const float* P_h, float alpha, uint8_t* Q, uint16_t* scales,
                      void* stream) {
  fq::clear_error();
  FQ_CHECK_ARG(T >= 1 && H >= 1 && H <= 128, "T = %d must be >= 1 and H = %d in [1, 128]", T, H);
  FQ_CHECK_ARG(P_h != nullptr, "P_h must be non-NULL");
  FQ_CHECK_ARG(scales && fq::aligned(scales, 2), "scales must be non-NULL and aligned");
  fq_qparams qp{};
  qp.bits = 4;
  qp.zero_point = 8;
  qp.gran = FQ_DYNAMIC_GROUP;
  qp.group_size = fq::kGroup;
  qp.alpha = alpha;
  const long long rows = static_cast<long long>(T) * H;  // head-rows of 128
  if (rows % 64 == 0 && rows / 64 <= 0x7fffffffLL) {
    // 64 head-rows (of any tokens) per item: P1 = I_64, P2 = P_h; the scale
    // of head-row r = 64 v + g (item v, group g) goes to r
    const fq_transform tt{64, 128, nullptr, P_h, nullptr};
    return fq::quant_common(fq::kAct, KV, int(rows / 64), 64 * 128, &qp, &tt, nullptr, Q, scales, nullptr, stream,
                            false, 1, 64);
  }
  // otherwise one token per item: P1 = I_H, P2 = P_h; head h of token t to t H + h
  const fq_transform tt{H, 128, nullptr, P_h, nullptr};
  return fq::quant_common(fq::kAct, KV, T, H * 128, &qp, &tt, nullptr, Q, scales, nullptr, stream, false, 1, H);
}

fq_status fq_quant_act_debug(const uint16_t* X, int M, int K, const fq_qparams* qp, const fq_transform* t,
                             const float* static_scale, uint8_t* Xq, void* s_x, float* xhat, void* stream) {
  if (!xhat || !fq::aligned(xhat, 4)) return fq::fail(FQ_ERR_INVALID, "xhat must be non-NULL and aligned");
  return fq::quant_common(fq::kAct, X, M, K, qp, t, static_scale, Xq, s_x, xhat, stream);
}

}  // extern "C"
