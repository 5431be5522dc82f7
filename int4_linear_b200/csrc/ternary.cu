// Ternary-weight linear layer (PT2-LLM page, 非对称三值量化器 ATQ):
// Y = X W^T with W^ = alpha T + mu per row and block of 128 columns,
// T in {-1, 0, +1}, fp16 activations (weight-only ternarization).
//
// Per output (m, n): y = sum_g (alpha[n][g] s[m][n][g] + mu[n][g] S[m][g])
// with s = sum_{k in g} x[m][k] t[n][k] and S = sum_{k in g} x[m][k], all in
// float32.  A ternary weight needs no multiplication, but at fp16
// activations it still costs a CUDA-core instruction or two: the code is
// turned into +-1.0 / 0 and accumulated with an FMA per token.  The tensor
// core does not help at decode sizes (an MMA of N <= 16 tokens holds its
// issuer far longer than its arithmetic takes), so this kernel is bound by
// ALU issue, not by the 2 bits per weight it streams.
//
// Mapping: one warp per two weight rows at a time (grid-stride over rows);
// lane l reads the 32-bit code words l, l + 32, ... of both rows (16 weights
// each, consecutive lanes on consecutive words, four words per lane in
// flight) and the matching 16 fp16 values of each token once for both rows;
// the 8 words of a 128-block share its alpha.  The block sums S of the CTA's
// token group sit in shared memory, one warp per (token, block).
#include <cuda_fp16.h>

#include <algorithm>

#include "fq_device.cuh"
#include "fq_host.h"

namespace fq {
namespace {

constexpr int kTerThreads = 256;
constexpr int kTerWarps = kTerThreads / 32;
constexpr int kTerMT = 8;         // tokens per pass over the weights
constexpr int kTerR = 2;          // weight rows per warp (they share every token load)
constexpr int kTerU = 4;          // code words per lane loaded ahead of their use
constexpr int kTerBlock = 128;    // columns per (alpha, mu)

struct TernaryParams {
  const __half* X;      // [M][K]
  const uint32_t* T;    // [N][K/16] codes, 2 bits per weight, low bits first
  const float* alpha;   // [N][K/128]
  const float* mu;      // [N][K/128]
  __half* Y;            // [M][N]
  int M, N, K;
};

// +1.0, -1.0 or 0.0 from a 2-bit code (bit 0: nonzero, bit 1: negative).
__device__ __forceinline__ float ternary_value(uint32_t code) {
  return __int_as_float(int((code & 1u) * 0x3F800000u) | int((code & 2u) << 30));
}

// The values of two weights from their 4-bit code pair, looked up in a
// 16-entry float2 table: the 16 entries of 8 bytes fill the 32 banks once,
// so a warp's lookups never conflict.
__device__ __forceinline__ float2 ternary_pair(const float2* lut, uint32_t w, int i) {
  return lut[(w >> (4 * i)) & 15u];
}

__global__ void __launch_bounds__(kTerThreads) ternary_linear_kernel(const TernaryParams p) {
  extern __shared__ float sS[];  // [kTerMT][K/128] block sums of the token group
  __shared__ float2 lut[16];     // code pair -> the two weights' values
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, nb = K / kTerBlock, words = K / 16;
  if (tid < 16) lut[tid] = make_float2(ternary_value(uint32_t(tid)), ternary_value(uint32_t(tid) >> 2));
  pdl_wait();
  for (int m0 = 0; m0 < p.M; m0 += kTerMT) {
    const int mt = min(kTerMT, p.M - m0);
    __syncthreads();  // the previous group's sums are no longer read
    // block sums: one warp per (token, block), 4 values per lane, coalesced,
    // four sums per warp in flight; the slots of absent tokens are zero
    for (int e0 = warp; e0 < mt * nb; e0 += 4 * kTerWarps) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * kTerWarps;
        v[u] = 0.f;
        if (e < mt * nb) {
          const int m = e / nb, g = e - m * nb;
          const uint2 raw =
              __ldg(reinterpret_cast<const uint2*>(p.X + size_t(m0 + m) * K + g * kTerBlock) + lane);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          v[u] = (a.x + a.y) + (b.x + b.y);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v[u] += __shfl_xor_sync(0xffffffffu, v[u], o);
        const int e = e0 + u * kTerWarps;
        if (lane == 0 && e < mt * nb) sS[e] = v[u];
      }
    }
    for (int e = mt * nb + tid; e < kTerMT * nb; e += kTerThreads) sS[e] = 0.f;
    __syncthreads();
    // kTerR rows per warp share every token load; kTerU code words per lane
    // are loaded ahead of their use
    for (int n0 = (blockIdx.x * kTerWarps + warp) * kTerR; n0 < p.N; n0 += gridDim.x * kTerWarps * kTerR) {
      float acc[kTerR][kTerMT];
#pragma unroll
      for (int r = 0; r < kTerR; ++r)
#pragma unroll
        for (int m = 0; m < kTerMT; ++m) acc[r][m] = 0.f;
      // code words (and alphas) of the next kTerU words per lane are loaded
      // while the current ones are used
      uint32_t wv[kTerU][kTerR];
      float av[kTerU][kTerR];
      auto load_words = [&](int jb, uint32_t (&w)[kTerU][kTerR], float (&a)[kTerU][kTerR]) {
#pragma unroll
        for (int u = 0; u < kTerU; ++u) {
          const int j = jb + 32 * u;
#pragma unroll
          for (int r = 0; r < kTerR; ++r) {
            const int n = n0 + r;
            const bool live = j < words && n < p.N;
            w[u][r] = live ? __ldg(p.T + size_t(n) * words + j) : 0u;
            a[u][r] = live ? __ldg(p.alpha + size_t(n) * nb + (j >> 3)) : 0.f;
          }
        }
      };
      load_words(lane, wv, av);
      for (int j0 = lane; j0 < words; j0 += 32 * kTerU) {
        uint32_t wn[kTerU][kTerR];
        float an[kTerU][kTerR];
        load_words(j0 + 32 * kTerU, wn, an);
#pragma unroll
        for (int u = 0; u < kTerU; ++u) {
          const int j = j0 + 32 * u;
          if (j >= words) break;
          float2 tv[kTerR][8];
#pragma unroll
          for (int r = 0; r < kTerR; ++r)
#pragma unroll
            for (int i = 0; i < 8; ++i) tv[r][i] = ternary_pair(lut, wv[u][r], i);
#pragma unroll
          for (int m = 0; m < kTerMT; ++m) {
            if (m >= mt) break;
            const uint4* xp = reinterpret_cast<const uint4*>(p.X + size_t(m0 + m) * K + 16 * j);
            const uint4 r0 = __ldg(xp), r1 = __ldg(xp + 1);
            const uint32_t hw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            // even and odd weights in the two lanes of packed float32 FMAs
            float2 sr[kTerR];
#pragma unroll
            for (int r = 0; r < kTerR; ++r) sr[r] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
#pragma unroll
              for (int r = 0; r < kTerR; ++r) sr[r] = ffma2(xf, tv[r][i], sr[r]);
            }
#pragma unroll
            for (int r = 0; r < kTerR; ++r) acc[r][m] = fmaf(av[u][r], sr[r].x + sr[r].y, acc[r][m]);
          }
        }
#pragma unroll
        for (int u = 0; u < kTerU; ++u)
#pragma unroll
          for (int r = 0; r < kTerR; ++r) {
            wv[u][r] = wn[u][r];
            av[u][r] = an[u][r];
          }
      }
#pragma unroll
      for (int r = 0; r < kTerR; ++r) {
        const int n = n0 + r;
        if (n >= p.N) break;
        // the offset term: sum_g mu[n][g] S[m][g], blocks over the lanes
        const float* mrow = p.mu + size_t(n) * nb;
        for (int g = lane; g < nb; g += 32) {
          const float u = __ldg(mrow + g);
#pragma unroll
          for (int m = 0; m < kTerMT; ++m) acc[r][m] = fmaf(u, sS[m * nb + g], acc[r][m]);
        }
#pragma unroll
        for (int m = 0; m < kTerMT; ++m) {
          float v = acc[r][m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0 && m < mt) p.Y[size_t(m0 + m) * p.N + n] = __float2half_rn(v);
        }
      }
    }
  }
  pdl_launch_dependents();
}

// int8 T [N][K] -> 2-bit codes, 16 per word: 1 -> 01, -1 -> 11, anything
// else -> 00 (zero).
__global__ void __launch_bounds__(256) ternary_pack_kernel(const int8_t* __restrict__ T, uint32_t* __restrict__ Tq,
                                                           size_t words) {
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < words; i += size_t(gridDim.x) * blockDim.x) {
    const int4 v = *reinterpret_cast<const int4*>(T + 16 * i);
    const int8_t* t = reinterpret_cast<const int8_t*>(&v);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) w |= (t[j] == 1 ? 1u : (t[j] == -1 ? 3u : 0u)) << (2 * j);
    Tq[i] = w;
  }
}

}  // namespace
}  // namespace fq

extern "C" {

fq_status fq_ternary_linear(const uint16_t* X, int M, int K, const uint8_t* Tq, const float* alpha, const float* mu,
                            int N, uint16_t* Y, void* stream) {
  fq::clear_error();
  FQ_CHECK_ARG(M >= 1 && N >= 1, "M = %d, N = %d must be >= 1", M, N);
  FQ_CHECK_ARG(K >= fq::kTerBlock && K <= fq::kMaxK && K % fq::kTerBlock == 0,
               "K = %d must be a multiple of 128 in [128, %d]", K, fq::kMaxK);
  FQ_CHECK_ARG(X && Tq && alpha && mu && Y, "X, Tq, alpha, mu and Y must be non-NULL");
  FQ_CHECK_ARG(fq::aligned(X, 16) && fq::aligned(Tq, 16) && fq::aligned(Y, 2) && fq::aligned(alpha, 4) &&
                   fq::aligned(mu, 4),
               "X and Tq must be 16-byte aligned, alpha and mu 4-byte aligned");
  fq::TernaryParams p{};
  p.X = reinterpret_cast<const __half*>(X);
  p.T = reinterpret_cast<const uint32_t*>(Tq);
  p.alpha = alpha;
  p.mu = mu;
  p.Y = reinterpret_cast<__half*>(Y);
  p.M = M;
  p.N = N;
  p.K = K;
  const size_t smem = size_t(fq::kTerMT) * (K / fq::kTerBlock) * sizeof(float);
  auto kern = fq::ternary_linear_kernel;
  if (smem > 48 * 1024 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
                              cudaSuccess)
    return fq::fail(FQ_ERR_CUDA, "cannot reserve %zu bytes of shared memory", smem);
  const int rows_per_cta = fq::kTerWarps * fq::kTerR;
  const int grid = std::max(1, std::min((N + rows_per_cta - 1) / rows_per_cta, 4 * fq::sm_count()));
  const cudaError_t e = fq::launch_pdl(kern, dim3(grid), dim3(fq::kTerThreads), smem,
                                       static_cast<cudaStream_t>(stream), p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fq::fail(FQ_ERR_CUDA, "ternary_linear_kernel: %s", cudaGetErrorString(e));
  }
  return fq::check_launch("ternary_linear_kernel");
}

fq_status fq_ternary_pack(const int8_t* T, int N, int K, uint8_t* Tq, void* stream) {
  fq::clear_error();
  FQ_CHECK_ARG(N >= 1 && K >= 16 && K % 16 == 0, "N = %d, K = %d (a multiple of 16) out of range", N, K);
  FQ_CHECK_ARG(T && Tq && fq::aligned(T, 16) && fq::aligned(Tq, 4), "T (16-byte) and Tq (4-byte) aligned, non-NULL");
  const size_t words = size_t(N) * (K / 16);
  const int grid = int(std::max<size_t>(1, std::min<size_t>((words + 255) / 256, size_t(fq::sm_count()) * 8)));
  fq::ternary_pack_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(T, reinterpret_cast<uint32_t*>(Tq),
                                                                               words);
  return fq::check_launch("ternary_pack_kernel");
}

}  // extern "C"
