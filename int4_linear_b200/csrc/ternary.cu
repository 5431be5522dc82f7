// Ternary-weight linear layer (PT2-LLM page, 非对称三值量化器 ATQ):
// Y = X W^T with W^ = alpha T + mu per row and block of 128 columns,
// T in {-1, 0, +1}, fp16 activations (weight-only ternarization).
//
// Per output (m, n): y = sum_g (alpha[n][g] s[m][n][g] + mu[n][g] S[m][g])
// with s = sum_{k in g} x[m][k] t[n][k] and S = sum_{k in g} x[m][k], all in
// float32.  A ternary weight needs no multiplication, but at fp16
// activations it still costs CUDA-core work per weight and token; the tensor
// core does not help at decode sizes (an MMA of N <= 16 tokens holds its
// issuer far longer than its arithmetic takes).  Two kernels:
//
// ternary_lut_kernel (M <= 16, K <= 32768): per-token tables of the 16
// possible sums of two adjacent weights' products, one table read and half
// an addition per weight; K split over a cluster of CTAs (layout and
// reduction described above the kernel).
//
// ternary_linear_kernel (the rest): one warp per two weight rows at a time
// (grid-stride over rows); lane l reads the 32-bit code words l, l + 32, ...
// of both rows (16 weights each, consecutive lanes on consecutive words,
// four words per lane in flight) and the matching 16 fp16 values of each
// token once for both rows; the 8 words of a 128-block share its alpha.  The
// block sums S of the CTA's token group sit in shared memory, one warp per
// (token, block).
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

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

// ------------------------------------------------------------------ pair-sum tables (M <= 16, K <= 32768)
//
// The partial product of two adjacent weights with one token takes one of
// nine values, 0, +-a, +-b, +-a +-b (a, b the two fp16 values).  Per token,
// the CTA writes all 16 code-pair entries of every weight pair of its K
// slice into shared memory; the product of a weight row is then one table
// read and half an addition per weight, with no per-weight decoding.
//
// A cluster of c CTAs splits K into c slices of at most 4096 columns (256
// code words) and walks one range of weight rows; each CTA writes its
// slice's partial sum of every row and token to its shared memory, and after
// a cluster barrier CTA r sums rows r, r + c, ... over the c slices in rank
// order through distributed shared memory (a fixed order: the result does not
// depend on scheduling).
//
// Table layout (128 KB, per 4-byte entry): lane l of a warp reads the 16
// code words 4 l + 128 u + v (v < 4, u < 2) of its row; the pair in the low
// nibble of byte j of word v (pair 2 j) is looked up in region L at
// code * 256 + (q / 2) * 4096 + (q % 2) * 128 + 4 l, the pair in the high
// nibble (pair 2 j + 1) in region H at 65536 + code * 4096 + q * 128 + 4 l,
// q = (4 j + v) * 2 + u.  Once byte j is shifted to bits 8-15 of a
// register, (reg & 0xF00) | 4 l and (reg & 0xF000) | 4 l are the byte
// offsets of both entries up to a constant, and every address of a warp's
// lookup falls in bank l: no conflicts.
constexpr int kLutThreads = 512;
constexpr int kLutWarps = kLutThreads / 32;
constexpr int kLutSliceWords = 256;      // code words of a CTA's K slice
constexpr int kLutRegion = 65536;        // bytes per table region (L, H)
constexpr int kLutPartials = 8192;       // floats of per-chunk partial sums
constexpr int kLutMaxM = 16;             // tokens per launch on this path
constexpr int kLutMaxCluster = 8;
constexpr size_t kLutSmem = 2 * size_t(kLutRegion) + kLutPartials * sizeof(float) + 32 * sizeof(float);

// Entries of the 16 codes of one weight pair: bits 0-1 the first weight's
// code, bits 2-3 the second's (01 = +1, 11 = -1, 00 and 10 = 0); every entry
// is the float32 rounding of the exact pair sum.
__device__ __forceinline__ void pair_entries(float a, float b, float (&e)[16]) {
  const float s = a + b, d = a - b;
  const float t[4] = {0.f, a, 0.f, -a};
#pragma unroll
  for (int ca = 0; ca < 4; ++ca) {
    e[ca] = t[ca];
    e[ca + 8] = t[ca];
  }
  e[4] = b, e[5] = s, e[6] = b, e[7] = -d;
  e[12] = -b, e[13] = d, e[14] = -b, e[15] = -s;
}

// Sum over the 32 weight pairs of a lane's quad U (code words w4) of their
// table entries: 32 lookups.
template <int U>
__device__ __forceinline__ float quad_sum(const uint8_t* tab, uint4 w4, uint32_t lb) {
  const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
  float2 s = make_float2(0.f, 0.f);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t src[4] = {wv[v] << 8, wv[v], wv[v] >> 8, wv[v] >> 16};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = (4 * j + v) * 2 + U;
      const float lo =
          *reinterpret_cast<const float*>(tab + ((src[j] & 0xF00u) | lb) + (q >> 1) * 4096 + (q & 1) * 128);
      const float hi = *reinterpret_cast<const float*>(tab + kLutRegion + ((src[j] & 0xF000u) | lb) + q * 128);
      s = fadd2(s, make_float2(lo, hi));
    }
  }
  return s.x + s.y;
}

struct LutRow {
  uint4 w[2];    // the lane's two quads of code words
  float al[2];   // their blocks' alpha
  float mu;      // mu of the slice's block `lane`
};

__global__ void __launch_bounds__(kLutThreads, 1)
    ternary_lut_kernel(const TernaryParams p, const int slice_words, const int rows_per_cluster, const int chunk_rows) {
  extern __shared__ __align__(16) uint8_t lsm[];
  float* part = reinterpret_cast<float*>(lsm + 2 * kLutRegion);  // [M][chunk_rows] partial sums
  float* sS = part + kLutPartials;                                // [32] block sums of the token
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t c = cluster_size(), rank = cluster_rank();
  const int cl = blockIdx.x / c;
  const int words = p.K / 16, nb = p.K / kTerBlock;
  const int w0 = int(rank) * slice_words;
  const int ws = max(0, min(words, w0 + slice_words) - w0);  // this CTA's code words
  const int gb0 = w0 / 8, nbs = ws / 8;                       // its first block, block count (<= 32)
  const int r_begin = cl * rows_per_cluster, r_end = min(p.N, r_begin + rows_per_cluster);
  const uint32_t lb = uint32_t(lane) * 4;
  const bool has0 = 4 * lane < ws, has1 = 4 * lane + 128 < ws;
  const uint4* tq = reinterpret_cast<const uint4*>(p.T);
  const size_t row_quads = size_t(words) / 4;
  pdl_wait();
  for (int cr0 = r_begin; cr0 < r_end; cr0 += chunk_rows) {
    const int rc = min(chunk_rows, r_end - cr0);
    for (int m = 0; m < p.M; ++m) {
      __syncthreads();  // the previous token's table is no longer read
      const __half* xm = p.X + size_t(m) * p.K + size_t(w0) * 16;
      for (int e = tid; e < 2048; e += kLutThreads) {
        const int region = e >> 10, q = (e >> 5) & 31, ln = e & 31;
        const int j = q >> 3, v = (q >> 1) & 3, u = q & 1;
        const int word = 4 * ln + 128 * u + v;
        float a = 0.f, b = 0.f;
        if (word < ws) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(xm + 16 * word + 2 * (2 * j + region)));
          a = f.x, b = f.y;
        }
        float ent[16];
        pair_entries(a, b, ent);
        uint8_t* dst = region == 0 ? lsm + (q >> 1) * 4096 + (q & 1) * 128 + 4 * ln
                                   : lsm + kLutRegion + q * 128 + 4 * ln;
        const int stride = region == 0 ? 256 : 4096;
#pragma unroll
        for (int code = 0; code < 16; ++code) *reinterpret_cast<float*>(dst + code * stride) = ent[code];
      }
      // the token's block sums over the slice (for the mu term)
      for (int g = warp; g < nbs; g += kLutWarps) {
        const uint2 raw = *reinterpret_cast<const uint2*>(xm + g * kTerBlock + 4 * lane);
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        float v = (fa.x + fa.y) + (fb.x + fb.y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) sS[g] = v;
      }
      __syncthreads();
      const float s_lane = lane < nbs ? sS[lane] : 0.f;
      float* pm = part + m * chunk_rows;
      auto load_row = [&](int rr, LutRow& r) {
        r.w[0] = r.w[1] = make_uint4(0u, 0u, 0u, 0u);
        r.al[0] = r.al[1] = r.mu = 0.f;
        if (rr < rc) {
          const int n = cr0 + rr;
          const uint4* row = tq + size_t(n) * row_quads + w0 / 4;
          const float* arow = p.alpha + size_t(n) * nb + gb0;
          if (has0) r.w[0] = __ldg(row + lane), r.al[0] = __ldg(arow + lane / 2);
          if (has1) r.w[1] = __ldg(row + lane + 32), r.al[1] = __ldg(arow + lane / 2 + 16);
          if (lane < nbs) r.mu = __ldg(p.mu + size_t(n) * nb + gb0 + lane);
        }
      };
      auto row_value = [&](const LutRow& r) {
        float acc = 0.f;
        if (has0) acc = fmaf(r.al[0], quad_sum<0>(lsm, r.w[0], lb), acc);
        if (has1) acc = fmaf(r.al[1], quad_sum<1>(lsm, r.w[1], lb), acc);
        acc = fmaf(r.mu, s_lane, acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        return acc;
      };
      // two rows per warp in flight: a row's loads are issued one row
      // computation ahead of their use
      LutRow ra, rb;
      load_row(warp, ra);
      load_row(warp + kLutWarps, rb);
      for (int rr = warp; rr < rc; rr += 2 * kLutWarps) {
        const float ya = row_value(ra);
        load_row(rr + 2 * kLutWarps, ra);
        if (lane == 0) pm[rr] = ya;
        if (rr + kLutWarps < rc) {
          const float yb = row_value(rb);
          if (lane == 0) pm[rr + kLutWarps] = yb;
        }
        load_row(rr + 3 * kLutWarps, rb);
      }
    }
    cluster_sync();  // every CTA's partial sums of the chunk are written
    const int nr = rc > int(rank) ? (rc - int(rank) + int(c) - 1) / int(c) : 0;
    for (int e = tid; e < p.M * nr; e += kLutThreads) {
      const int m = e / nr, rr = int(rank) + int(c) * (e - m * nr);
      float y = 0.f;
      for (uint32_t r = 0; r < c; ++r) y += ld_cluster_f32(part + m * chunk_rows + rr, r);
      p.Y[size_t(m) * p.N + cr0 + rr] = __float2half_rn(y);
    }
    cluster_sync();  // the peers have read this CTA's partial sums
  }
  pdl_launch_dependents();
}

}  // namespace

// Clusters of c CTAs of ternary_lut_kernel that fit on the device at once
// (0 if none or the query fails); cached per c.
static int lut_clusters(int c) {
  static std::atomic<int> cache[kLutMaxCluster + 1];
  static std::atomic<bool> attr_set{false};
  const int hit = cache[c].load(std::memory_order_relaxed);
  if (hit != 0) return hit > 0 ? hit : 0;
  if (!attr_set.load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(ternary_lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kLutSmem)) !=
        cudaSuccess) {
      cudaGetLastError();
      cache[c].store(-1);
      return 0;
    }
    attr_set.store(true);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c * sm_count());
  cfg.blockDim = dim3(kLutThreads);
  cfg.dynamicSmemBytes = kLutSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(c);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ternary_lut_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[c].store(n > 0 ? n : -1);
  return n > 0 ? n : 0;
}

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
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // pair-sum tables: one cluster of c CTAs per row range, c K slices of at
  // most 4096 columns (the table of a slice fills 128 KB)
  const int words = K / 16;
  const int c = (words + fq::kLutSliceWords - 1) / fq::kLutSliceWords;
  if (M <= fq::kLutMaxM && c <= fq::kLutMaxCluster) {
    const int ncl_max = fq::lut_clusters(c);
    if (ncl_max > 0) {
      const int slice_words = ((words + c - 1) / c + 7) / 8 * 8;
      const int rows_per_cluster = (N + ncl_max - 1) / ncl_max;
      const int ncl = (N + rows_per_cluster - 1) / rows_per_cluster;
      // one token: the whole range at once; several: 256-row chunks, whose
      // code words stay in L2 between the tokens' passes
      const int chunk_rows = M == 1 ? fq::kLutPartials : std::min(256, fq::kLutPartials / M);
      const cudaError_t e = fq::launch_pdl_cluster(fq::ternary_lut_kernel, dim3(ncl * c), dim3(fq::kLutThreads),
                                                   fq::kLutSmem, st, unsigned(c), p, slice_words, rows_per_cluster,
                                                   chunk_rows);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fq::fail(FQ_ERR_CUDA, "ternary_lut_kernel: %s", cudaGetErrorString(e));
      }
      return fq::check_launch("ternary_lut_kernel");
    }
  }
  const size_t smem = size_t(fq::kTerMT) * (K / fq::kTerBlock) * sizeof(float);
  auto kern = fq::ternary_linear_kernel;
  if (smem > 48 * 1024 && cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
                              cudaSuccess)
    return fq::fail(FQ_ERR_CUDA, "cannot reserve %zu bytes of shared memory", smem);
  const int rows_per_cta = fq::kTerWarps * fq::kTerR;
  const int grid = std::max(1, std::min((N + rows_per_cta - 1) / rows_per_cta, 4 * fq::sm_count()));
  const cudaError_t e = fq::launch_pdl(kern, dim3(grid), dim3(fq::kTerThreads), smem, st, p);
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
