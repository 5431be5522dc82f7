// INT4 x INT4 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8).
//
// Blackwell has no 4-bit integer MMA, so each 128-deep K slice of both
// operands is unpacked from nibbles to bytes in shared memory and multiplied
// with s8 x s8 -> s32 MMAs accumulating in tensor memory (FlatQuant notes,
// 核心思想: Y ~ Q(XP) Q(P^-1 W^T) with integer accumulation).
//
// Prefill with per-token or static scales (M > 64, gemm_w4a4_persistent_kernel):
// a persistent grid of CTA pairs (clusters of two; tcgen05 .cta_group::2)
// walks 256 x 256 output tiles.  Each CTA loads and unpacks its own 128
// activation rows and half of the tile's 256 weight rows, and one thread of
// the even CTA issues 256 x 256 MMAs that read both CTAs' operands, so each
// SM moves half the weight slice through its shared memory; dedicated
// epilogue warps drain the accumulator and TMA-store fp16 blocks while the
// next tile's slices are unpacked.  The group-scale epilogue and the raw
// int32 output run gemm_w4a4_kernel, one CTA per 128 x BN tile.  In both, the
// packed 128-deep K slices of both operands arrive by TMA into a ring in
// shared memory; A-warps unpack the activation rows into a tensor-memory ring
// (tcgen05.st), B-warps the weight rows into a 128-byte-swizzled
// shared-memory ring, and one thread issues the MMAs (A from tensor memory).
// The warp roles are listed beside each kernel.  Stages are handed over
// with mbarriers; every wait is bounded and a wait that gives up records a
// timeout code in the device error word.
//
// The nibble is unpacked into the high half of its byte (16 q, see
// unpack8_hi), so the tensor core accumulates 256 * sum(qx qw); the epilogues
// remove the factor exactly (an arithmetic shift, or a multiply by 2^-8).
//
// Epilogues: per-token x per-output-channel scales, static (migrated) scales,
// per-group scales summed in float32 (FRM-PTQ group quantization, one group
// per K slice, double-buffered accumulators) or raw int32.  For few tokens
// (decode, gemm_decode_kernel) the operands swap roles: the weights fill the
// 128-row MMA side and the tokens the N side.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "fq_device.cuh"
#include "fq_host.h"

namespace fq {

namespace {

enum Epi { kEpiRow = 0, kEpiStatic = 1, kEpiGroup = 2, kEpiS32 = 3 };

constexpr int kBM = 128;        // rows of the A operand per tile (MMA M)
constexpr int kBK = 128;        // int8 K per stage; equals the quantization group
constexpr int kPK = kBK / 2;    // packed bytes per row per stage
constexpr int kEpiWarps = 4;
constexpr int kUnpackWarps = 8;

// Warp roles (480 threads):
//   warp 0      group mode: keeps the per-slice scale ring filled; else idle
//   warp 1      tensor-memory allocation and the MMA-issuing thread
//   warps 2-5   epilogue (outside group mode they first unpack A)
//   warps 6-13  unpack B (outside group mode); group mode: 6-9 A,
//               10-13 a second epilogue set (the upper half of the columns)
//   warp 14     one thread issues the TMA loads of both packed slices
//   warps 15-16 group mode only: unpack B
// The packed 128-deep K slices of both operands arrive by TMA into a ring of
// SP stages (A in the 64-byte swizzle, so that the one-row-per-thread reads
// are free of bank conflicts; B unswizzled, read in consecutive 16-byte
// pieces); the A-warps unpack their row into a tensor-memory ring and the
// B-warps into a 128-byte-swizzled shared-memory ring of SU stages.  A
// packed stage goes back to the producer only after the unpacked data has
// been stored (its registers consumed), so a refill never overtakes a read.
constexpr int kProducerWarp = 14;

// Group mode runs its per-slice epilogue alongside the main loop on eight
// warps (two per tensor-memory lane quadrant), so it has 17 warps: the weight
// slice of a 128-column tile is unpacked by warps 15-16.
template <int EPI>
__host__ __device__ constexpr int threads_of() { return 32 * (EPI == kEpiGroup ? 17 : 15); }
template <int EPI>
__host__ __device__ constexpr int epi_warps() { return EPI == kEpiGroup ? 2 * kEpiWarps : kEpiWarps; }
template <int EPI>
__host__ __device__ constexpr int b_warps() { return EPI == kEpiGroup ? 2 : kUnpackWarps; }
template <int EPI>
__host__ __device__ constexpr int feed_warps() { return 4 + b_warps<EPI>(); }

template <int BN, int EPI>
struct Cfg {
  static constexpr int SP = 4;                 // packed stages (TMA ring)
  static constexpr int SU = BN == 256 ? 3 : 4; // unpacked stages (A in tensor memory, B in shared memory)
  static constexpr int PA = kBM * kPK;         // packed A slice: 128 rows x 64 bytes
  static constexpr int PB = BN * kPK;          // packed B slice
  static constexpr int P_STAGE = PA + PB;
  static constexpr int B_UNP = BN * kBK;
  static constexpr int ACC_COLS = EPI == kEpiGroup ? 3 * BN : BN;
  static constexpr int A_COL0 = ((ACC_COLS + 31) / 32) * 32;   // tensor-memory columns of the A ring
  static constexpr int A_STAGE_COLS = kBK / 4;                 // 4 int8 per 32-bit column
  static constexpr int TMEM_NEED = A_COL0 + SU * A_STAGE_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 64 ? 64 : (TMEM_NEED <= 128 ? 128 : (TMEM_NEED <= 256 ? 256 : 512));
  static constexpr int UNP_STAGE = B_UNP;
  static constexpr int OFF_P = 0;
  static constexpr int OFF_UNP = OFF_P + SP * P_STAGE;
  static constexpr int OFF_SCALE = OFF_UNP + SU * UNP_STAGE;
  // group mode: a ring of SS per-slice scale stages written by warp 0: the
  // weight scales s_w / 256 of the BN columns, then the activation scales of
  // the 128 rows
  static constexpr int SS = 8;
  static constexpr int SC_STAGE = BN * 4 + kBM * 4;
  // row/static: the tile's BN weight scales, staged once by warp 0
  static constexpr int SCALE_BYTES = EPI == kEpiGroup ? SS * SC_STAGE : ((EPI == kEpiRow || EPI == kEpiStatic) ? BN * 4 : 0);
  static constexpr int OFF_BAR = OFF_SCALE + SCALE_BYTES;
  static constexpr int NBAR = 2 * SP + 2 * SU + 6 + (EPI == kEpiGroup ? 2 * SS : 0);
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + slack to align the base to 1024
  // the fp16 output tile is staged in the (then idle) unpacked ring, rows padded by 16 bytes
  static constexpr int OUT_PITCH = 2 * BN + 16;
  static constexpr int OFF_OUT = OFF_UNP;
  static_assert(UNP_STAGE % 1024 == 0 && P_STAGE % 1024 == 0 && PA % 1024 == 0, "1024-byte stage alignment");
  static_assert(kBM * OUT_PITCH <= SU * UNP_STAGE, "output tile fits in the ring");
  static_assert(TMEM_NEED <= 512, "tensor memory");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(EPI != kEpiGroup || 3 * BN <= 512, "group epilogue needs 3 x BN tensor-memory columns");
};

struct GemmParams {
  const uint8_t* A;   // packed operand on the 128-row side: [rowsA][K/2]
  const uint8_t* B;   // packed operand on the BN-row side:  [rowsB][K/2]
  int M, N, K;        // Y is [M][N]
  int rowsA, rowsB;   // rows of the A (128-row tiles) and B (BN-row tiles) operands
  int num_kb;         // K / 128
  const float* sx;    // [M]           per-token scales
  const float* sw;    // [N]           per-channel (or migrated static) scales
  const __half* gsx;  // [K/128][M]    group scales of the activations
  const __half* gsw;  // [K/128][N]    group scales of the weights
  __half* Y;          // [M][N]
  int32_t* acc;       // [M][N]        int32 output
  unsigned* err;
  // decode
  unsigned* sync;     // the workspace's synchronization block (all zero between calls)
  int32_t* slots;     // [2 G][M][128]  int32 partial sums of the tiles split between CTAs
  // fused decode linear: the tokens are quantized inside the GEMM launch
  const __half* X;    // [M][K]        fp16 tokens
  const float* sst;   // [K]           static scales
  const float* cst;   // [K] or null   channel factors
  uint8_t* Xq;        // [M][K/2]      their packed codes (the B operand)
};

// The first kSyncBytes of a decode workspace: word 0 counts the CTAs at the
// fused kernel's grid barrier, word 1 is that barrier's generation number,
// words kSyncTile0 + t count the CTAs that have stored their share of split
// tile t.  Every counter returns to 0 by the end of a call (the generation
// number only changes).
constexpr size_t kSyncBytes = FQ_WORKSPACE_SYNC_BYTES;
constexpr int kSyncTile0 = 16;
constexpr int kMaxSyncTiles = int(kSyncBytes / 4) - kSyncTile0;

__device__ __forceinline__ void store_half8(__half* dst, const float* v) {
  uint4 o;
  __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
  *reinterpret_cast<uint4*>(dst) = o;
}

template <int BN, int EPI>
__global__ void __launch_bounds__(threads_of<EPI>(), 1)
    gemm_w4a4_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB) {
  using C = Cfg<BN, EPI>;
  constexpr int SU = C::SU, SP = C::SP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pfull = bars;
  uint64_t* pempty = pfull + SP;
  uint64_t* full_u = pempty + SP;
  uint64_t* empty_u = full_u + SU;
  uint64_t* acc_full = empty_u + SU;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done_bar = acc_empty + 2;
  uint64_t* sw_ready = done_bar + 1;  // row/static: the tile's weight scales are in shared memory
  uint64_t* sfull = sw_ready + 1;     // group mode: scale stages
  uint64_t* sempty = sfull + C::SS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tileA = blockIdx.x, tileB = blockIdx.y;
  const int kb0 = 0;  // every CTA covers the whole K
  const int nkb = p.num_kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], feed_warps<EPI>());
    }
    for (int s = 0; s < SU; ++s) {
      mbar_init(&full_u[s], feed_warps<EPI>());
      mbar_init(&empty_u[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], epi_warps<EPI>());
    }
    mbar_init(done_bar, 1);
    mbar_init(sw_ready, 1);
    if (EPI == kEpiGroup) {
      for (int s = 0; s < C::SS; ++s) {
        mbar_init(&sfull[s], 1);
        mbar_init(&sempty[s], epi_warps<EPI>());
      }
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the next kernel may be scheduled once every CTA of this one is running;
  // this one reads its inputs only after the kernels before it completed
  pdl_launch_dependents();
  pdl_wait();

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int sp = i % SP;
        if (!mbar_wait(&pempty[sp], ((i / SP) & 1) ^ 1)) {
          record_error(p.err, kErrTimeoutProducer);
          break;
        }
        uint8_t* st = smem + C::OFF_P + sp * C::P_STAGE;
        mbar_arrive_expect_tx(&pfull[sp], C::P_STAGE);
        tma_load_2d(st, &tmA, &pfull[sp], (kb0 + i) * kPK, tileA * kBM);
        tma_load_2d(st + C::PA, &tmB, &pfull[sp], (kb0 + i) * kPK, tileB * BN);
        ++issued;
      }
      // every issued copy has landed before the CTA may leave (normally the
      // unpacking warps already waited for each of them)
      for (int i = max(0, issued - SP); i < issued; ++i)
        if (!mbar_wait(&pfull[i % SP], (i / SP) & 1)) {
          record_error(p.err, kErrTimeoutDrain);
          break;
        }
    }
  } else if (warp == 0) {
    if (EPI == kEpiRow || EPI == kEpiStatic) {
      float* sws = reinterpret_cast<float*>(smem + C::OFF_SCALE);
      for (int c = lane; c < BN; c += 32) {
        const int n = tileB * BN + c;
        sws[c] = n < p.N ? __ldg(p.sw + n) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sw_ready);
    }
    if (EPI == kEpiGroup) {
      // ------------------------------------------------------------ group scales -> shared-memory ring
      // Loads run D slices ahead in registers, so their latency is paid once.
      constexpr int D = 4;
      constexpr int NP2 = BN / 64;  // column pairs per lane
      const int bbase = tileB * BN, abase = tileA * kBM;
      __half2 wv[D][NP2];
      __half xv[D][4];
      auto load = [&](int d, int i) {
        const int g = kb0 + i;
#pragma unroll
        for (int t = 0; t < NP2; ++t) {
          const int n = bbase + 2 * (lane + 32 * t);  // N is a multiple of 8: both columns or neither
          wv[d][t] = (i < nkb && n < p.N) ? *reinterpret_cast<const __half2*>(p.gsw + size_t(g) * p.N + n)
                                          : __floats2half2_rn(0.f, 0.f);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int m = abase + lane + 32 * t;
          xv[d][t] = (i < nkb && m < p.M) ? p.gsx[size_t(g) * p.M + m] : __float2half_rn(0.f);
        }
      };
#pragma unroll
      for (int d = 0; d < D; ++d) load(d, d);
      bool ok = true;
      for (int i0 = 0; i0 < nkb && ok; i0 += D) {
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const int i = i0 + d;
          if (i >= nkb) break;
          const int st = i % C::SS;
          if (!warp_wait(&sempty[st], ((i / C::SS) & 1) ^ 1)) {
            if (lane == 0) record_error(p.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          uint8_t* sc = smem + C::OFF_SCALE + st * C::SC_STAGE;
#pragma unroll
          for (int t = 0; t < NP2; ++t) {
            const float2 w = __half22float2(wv[d][t]);  // / 256 below: exact
            reinterpret_cast<float2*>(sc)[lane + 32 * t] = make_float2(w.x * 0.00390625f, w.y * 0.00390625f);
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) reinterpret_cast<float*>(sc + BN * 4)[lane + 32 * t] = __half2float(xv[d][t]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfull[st]);
          load(d, i + D);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, BN);
      for (int i = 0; i < nkb; ++i) {
        const int su = i % SU;
        uint32_t d = tmem;
        if (EPI == kEpiGroup) {
          // phase 0 of acc_empty[b] is the epilogue priming buffer b
          const int b = i & 1;
          if (!mbar_wait(&acc_empty[b], (i >> 1) & 1)) {
            record_error(p.err, kErrTimeoutMma);
            break;
          }
          tc_fence_after();
          d = tmem + uint32_t(b * BN);
        }
        if (!mbar_wait(&full_u[su], (i / SU) & 1)) {
          record_error(p.err, kErrTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t a0 = tmem + uint32_t(C::A_COL0 + su * C::A_STAGE_COLS);
        const uint32_t b0 = smem_u32(smem + C::OFF_UNP + su * C::UNP_STAGE);
#pragma unroll
        for (int k = 0; k < kBK / 32; ++k) {
          // group mode accumulates onto the primed offset (see the group epilogue)
          const uint32_t accum = EPI == kEpiGroup ? 1u : uint32_t(i > 0 || k > 0);
          mma_i8_ts(d, a0 + uint32_t(8 * k), sdesc_k128_sw128(b0 + 32 * k), idesc, accum);
        }
        mma_commit(&empty_u[su]);
        if (EPI == kEpiGroup) mma_commit(&acc_full[i & 1]);
      }
      if (EPI != kEpiGroup) mma_commit(&acc_full[0]);
      mma_commit(done_bar);
      if (!mbar_wait(done_bar, 0)) record_error(p.err, kErrTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ feeders
    constexpr int NB = b_warps<EPI>();
    const bool epi_warp = warp < 2 + kEpiWarps;
    const bool a_warp = EPI == kEpiGroup ? (warp >= 6 && warp < 10) : epi_warp;
    const bool b_warp = EPI == kEpiGroup ? (warp >= 15) : (warp >= 6);
    if (a_warp) {
      // one A row per thread (its tensor-memory lane): 64 packed bytes per slice
      const int q = warp & 3;
      const int row = q * 32 + lane;
      const int sw = (row >> 1) & 3;  // 64-byte swizzle: chunk c of this row sits at chunk c ^ sw
      const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + uint32_t(C::A_COL0);
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int sp = i % SP, su = i % SU;
        if (!warp_wait(&pfull[sp], (i / SP) & 1)) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + C::OFF_P + sp * C::P_STAGE + row * kPK;
        uint4 w[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
        if (!warp_wait(&empty_u[su], ((i / SU) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          unpack8_hi(w[c].x, r[8 * c + 0], r[8 * c + 1]);
          unpack8_hi(w[c].y, r[8 * c + 2], r[8 * c + 3]);
          unpack8_hi(w[c].z, r[8 * c + 4], r[8 * c + 5]);
          unpack8_hi(w[c].w, r[8 * c + 6], r[8 * c + 7]);
        }
        tmem_st_32x32(ta + uint32_t(su * C::A_STAGE_COLS), r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[sp]);
          mbar_arrive(&full_u[su]);
        }
      }
      if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
    } else if (b_warp) {
      const int uw = EPI == kEpiGroup ? warp - 15 : warp - 6;
      constexpr int kJobs = BN * 4;  // 16-byte packed pieces of B per stage
      constexpr int JPT = (kJobs + NB * 32 - 1) / (NB * 32);
      // per-lane pieces, the same in every stage: packed source offset, two swizzled destinations
      uint32_t dst0[JPT], dst1[JPT], srcj[JPT];
      bool live[JPT];
#pragma unroll
      for (int it = 0; it < JPT; ++it) {
        const int j = (it * NB + uw) * 32 + lane;
        live[it] = j < kJobs;
        const int row = live[it] ? (j >> 2) : 0, c = j & 3, r7 = row & 7;
        const uint32_t rb = uint32_t((row >> 3) * 1024 + r7 * 128);
        dst0[it] = rb + uint32_t(((2 * c) ^ r7) << 4);
        dst1[it] = rb + uint32_t(((2 * c + 1) ^ r7) << 4);
        srcj[it] = uint32_t(live[it] ? j * 16 : 0);
      }
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int sp = i % SP, su = i % SU;
        if (!warp_wait(&pfull[sp], (i / SP) & 1)) {
          ok = false;
          break;
        }
        const uint8_t* pb = smem + C::OFF_P + sp * C::P_STAGE + C::PA;
        uint4 w[JPT];
#pragma unroll
        for (int it = 0; it < JPT; ++it) w[it] = *reinterpret_cast<const uint4*>(pb + srcj[it]);
        if (!warp_wait(&empty_u[su], ((i / SU) & 1) ^ 1)) {
          ok = false;
          break;
        }
        uint8_t* uk = smem + C::OFF_UNP + su * C::UNP_STAGE;
#pragma unroll
        for (int it = 0; it < JPT; ++it) {
          if (!live[it]) continue;
          uint4 o0, o1;
          unpack8_hi(w[it].x, o0.x, o0.y);
          unpack8_hi(w[it].y, o0.z, o0.w);
          unpack8_hi(w[it].z, o1.x, o1.y);
          unpack8_hi(w[it].w, o1.z, o1.w);
          *reinterpret_cast<uint4*>(uk + dst0[it]) = o0;
          *reinterpret_cast<uint4*>(uk + dst1[it]) = o1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[sp]);
          mbar_arrive(&full_u[su]);
        }
      }
      if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
    }
    // the upper half of the columns: outside group mode the first four
    // B-warps (6..9) after their last slice, in group mode warps 10..13
    const bool epi_hi = EPI == kEpiGroup ? (warp >= 10 && warp < 14) : (warp >= 6 && warp < 10);
    if (epi_warp || epi_hi) {
    // ------------------------------------------------------------ epilogue
      const int q = warp & 3;  // tensor-memory lane quadrant this warp may access
      const int rloc = q * 32 + lane;
      const uint32_t tl = tmem + (uint32_t(q * 32) << 16);
      const int arow = tileA * kBM + rloc;
      const int bbase = tileB * BN;
      if (EPI != kEpiGroup) {
        if (!warp_wait(&acc_full[0], 0) && lane == 0) record_error(p.err, kErrTimeoutEpilogue);
        if ((EPI == kEpiRow || EPI == kEpiStatic) && !warp_wait(sw_ready, 0) && lane == 0)
          record_error(p.err, kErrTimeoutEpilogue);
        tc_fence_after();
        constexpr int CW = BN >= 32 ? 32 : 16;
        const float* sws = reinterpret_cast<const float*>(smem + C::OFF_SCALE);
        const int cbeg = epi_hi ? BN / 2 : 0, cend = (EPI == kEpiGroup || epi_hi) ? BN : BN / 2;
        for (int c0 = cbeg; c0 < cend; c0 += CW) {
          uint32_t v[32];
          if (CW == 32)
            tmem_ld_32x32(tl + c0, v);
          else
            tmem_ld_32x16(tl + c0, v);
          tmem_wait_ld();
          {
            // thread owns token row m = arow, columns n = bbase + c0 + j
            const int m = arow;
            if (m < p.M) {
              const int n0 = bbase + c0;
              float y[32];
              if (EPI == kEpiRow || EPI == kEpiStatic) {
                const float sxm = EPI == kEpiRow ? p.sx[m] : 1.0f;
  #pragma unroll
                for (int j = 0; j < CW; ++j) {
                  const float a = float(int(v[j]) >> 8);
                  const float swn = sws[c0 + j];  // the same address in every lane: a broadcast
                  y[j] = EPI == kEpiRow ? __fmul_rn(__fmul_rn(a, sxm), swn) : __fmul_rn(a, swn);
                }
                // staged in shared memory; written out coalesced after the barrier below
                __half* dst = reinterpret_cast<__half*>(smem + C::OFF_OUT + rloc * C::OUT_PITCH) + c0;
  #pragma unroll
                for (int j = 0; j < CW; j += 8) store_half8(dst + j, y + j);
              } else {
                int32_t* dst = p.acc + size_t(m) * p.N + n0;
                for (int j = 0; j < CW; ++j) {
                  if (n0 + j >= p.N) break;
                  dst[j] = int32_t(v[j]) >> 8;
                }
              }
            }
          }
        }
      } else {
        // group-128: one accumulator per K slice, double-buffered in tensor
        // memory; the running float32 sum lives in columns [2 BN, 3 BN).
        // Each accumulator buffer is primed with the integer 0x4B400000 (the
        // bits of 1.5 * 2^23) before the MMAs add 256 * sum(qx qw) (|.| <
        // 2^22) to it, so its bits read as the float 1.5 * 2^23 + acc
        // exactly, with no int-to-float conversion: f - 1.5 * 2^23 is the
        // accumulator, exact; times s' = s_w / 256 (exact) it gives
        // fl(sum * s_w) with a single rounding, and a fused multiply-add
        // adds that times s_x into the running sum (zeroed at the start);
        // two columns per instruction (f32x2).  Warp 0 keeps the slice's s'
        // and row scales ready in a shared-memory ring; one 16-byte load
        // gives the scales of four columns.
        constexpr uint32_t kMagic = 0x4B400000u;
        const uint32_t tsum = tl + uint32_t(2 * BN);
        const int gbeg = epi_hi ? BN / 2 : 0, gend = epi_hi ? BN : BN / 2;  // this warp's columns
        uint32_t mg[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) mg[j] = kMagic;
#pragma unroll
        for (int b = 0; b < 2; ++b)
          for (int c0 = gbeg; c0 < gend; c0 += 32) tmem_st_32x32(tl + uint32_t(b * BN + c0), mg);
        {
          uint32_t z[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) z[j] = 0u;
          for (int c0 = gbeg; c0 < gend; c0 += 32) tmem_st_32x32(tsum + c0, z);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[0]);
          mbar_arrive(&acc_empty[1]);
        }
        for (int i = 0; i < nkb; ++i) {
          const int b = i & 1, st = i % C::SS;
          if (!warp_wait(&sfull[st], (i / C::SS) & 1)) {
            if (lane == 0) record_error(p.err, kErrTimeoutEpilogue);
            break;
          }
          const float4* sbuf = reinterpret_cast<const float4*>(smem + C::OFF_SCALE + st * C::SC_STAGE);
          const float sxg = reinterpret_cast<const float*>(smem + C::OFF_SCALE + st * C::SC_STAGE + BN * 4)[rloc];
          const float2 sx2 = make_float2(sxg, sxg);
          const float2 nmag = make_float2(-12582912.0f, -12582912.0f);  // -1.5 * 2^23
          if (!warp_wait(&acc_full[b], (i >> 1) & 1)) {
            if (lane == 0) record_error(p.err, kErrTimeoutEpilogue);
            break;
          }
          tc_fence_after();
          for (int c0 = gbeg; c0 < gend; c0 += 32) {
            uint32_t v[32], s[32];
            tmem_ld_32x32(tl + uint32_t(b * BN + c0), v);
            tmem_ld_32x32(tsum + c0, s);
            tmem_wait_ld();
  #pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 q = sbuf[(c0 + j) / 4];
#pragma unroll
              for (int h = 0; h < 4; h += 2) {
                const float2 a = fadd2(make_float2(__uint_as_float(v[j + h]), __uint_as_float(v[j + h + 1])), nmag);
                const float2 u = fmul2(a, h == 0 ? make_float2(q.x, q.y) : make_float2(q.z, q.w));
                const float2 r = ffma2(u, sx2, make_float2(__uint_as_float(s[j + h]), __uint_as_float(s[j + h + 1])));
                s[j + h] = __float_as_uint(r.x);
                s[j + h + 1] = __float_as_uint(r.y);
              }
            }
            tmem_st_32x32(tsum + c0, s);
            tmem_st_32x32(tl + uint32_t(b * BN + c0), mg);  // re-prime for slice i + 2
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[b]);
            mbar_arrive(&sempty[st]);
          }
        }
        for (int c0 = gbeg; c0 < gend; c0 += 32) {
          uint32_t s[32];
          tmem_ld_32x32(tsum + c0, s);
          tmem_wait_ld();
          {
            float y[32];
  #pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = nkb > 0 ? __uint_as_float(s[j]) : 0.f;
            __half* dst = reinterpret_cast<__half*>(smem + C::OFF_OUT + rloc * C::OUT_PITCH) + c0;
  #pragma unroll
            for (int j = 0; j < 32; j += 8) store_half8(dst + j, y + j);
          }
        }
      }
    }
  }

  // fp16 tiles staged in shared memory leave as whole 512-byte row segments
  constexpr bool kStaged = EPI == kEpiRow || EPI == kEpiStatic || EPI == kEpiGroup;
  if (kStaged) {
    __syncthreads();
    const int n0 = tileB * BN;
    const int chunks = max(0, min(BN, p.N - n0)) / 8;  // 16-byte chunks per row (N % 8 == 0)
    for (int r = warp; r < kBM; r += threads_of<EPI>() / 32) {
      const int m = tileA * kBM + r;
      if (m >= p.M) break;
      const uint8_t* src = smem + C::OFF_OUT + r * C::OUT_PITCH;
      __half* dst = p.Y + size_t(m) * p.N + n0;
      for (int c = lane; c < chunks; c += 32)
        *reinterpret_cast<uint4*>(dst + c * 8) = *reinterpret_cast<const uint4*>(src + c * 16);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- persistent CTA-pair prefill kernel
//
// Per-token / static scales with M > 64.  A persistent grid of CTA pairs
// (one CTA per SM) walks the 256 x 256 output tiles (pairs of 128-row A
// tiles x 256 weight rows), so the operand pipeline runs on across tile
// boundaries and the epilogue of one tile overlaps the main loop of the next:
//   warp 0        one thread issues the TMA loads of the packed slices
//   warp 1        tensor-memory allocation; in CTA 0 the thread that issues
//                 the 256 x 256 pair MMAs (.cta_group::2)
//   warps 2-13    unpack this CTA's 128 A rows into the tensor-memory ring
//                 (three warps per lane quadrant, K slices in turn)
//   warps 14..    unpack this CTA's half of the weight rows, NB warps taking
//                 whole K slices in turn
//   last 8 warps  epilogue: drain the accumulator (two warps per lane
//                 quadrant, 128 columns each, 32 at a time), scale to fp16
//                 into a per-warp shared-memory block and TMA-store it; the
//                 accumulator goes back to the MMA thread as soon as its last
//                 columns are read
// The accumulator is single-buffered (256 columns + the A ring); the MMA
// thread waits for both CTAs' epilogues to have read it, while the feed
// warps fill the rings ahead of the next tile.
template <int NB>
struct PCfg {
  static constexpr int BN = 256;               // pair tile columns
  static constexpr int BR = BN / 2;            // weight rows per CTA
  static constexpr int SP = 6;                 // packed stages (TMA ring)
  static constexpr int SU = 5;                 // unpacked stages
  static constexpr int PA = kBM * kPK;
  static constexpr int PB = BR * kPK;
  static constexpr int P_STAGE = PA + PB;
  static constexpr int UNP_STAGE = BR * kBK;
  static constexpr int A_COL0 = BN;            // A ring after the accumulator
  static constexpr int A_STAGE_COLS = kBK / 4;
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_P = 0;
  static constexpr int OFF_UNP = OFF_P + SP * P_STAGE;
  static constexpr int OFF_SCALE = OFF_UNP + SU * UNP_STAGE;  // [2][BN] weight scales
  static constexpr int STG = 32 * 32 * 2;                     // one 32 x 32 fp16 output block
  static constexpr int OFF_STG = OFF_SCALE + 2 * BN * 4;      // [8 warps][2 blocks]
  static constexpr int OFF_BAR = OFF_STG + 8 * 2 * STG;
  static constexpr int NBAR = 2 * SP + 2 * SU + 4;          // + acc_full, acc_empty, done, fin
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;
  static constexpr int NA = 3;                 // A-warps per lane quadrant (slices in turn)
  static constexpr int B_WARP0 = 2 + 4 * NA;   // A: warps 2 .. 2 + 4 NA - 1
  static constexpr int EPI_WARP0 = B_WARP0 + NB;
  static constexpr int THREADS = 32 * (EPI_WARP0 + 8);
  static constexpr int FEED = 4 + 1;           // CTA 0's arrivals per slice: 4 A-warps, 1 B-warp
  // CTA 1's feed warps of one slice (the 4 A-warps and the B-warp of turn
  // g mod NA) meet at named barrier 2 + turn, and one of them publishes the
  // slice to CTA 0 with a single cluster-scope release (the barrier orders the
  // group's operand writes before it; release is cumulative)
  static_assert(NA == NB, "A- and B-warps take the slices in the same turns");
  static_assert(A_COL0 + SU * A_STAGE_COLS <= TMEM_COLS, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(P_STAGE % 1024 == 0 && UNP_STAGE % 1024 == 0 && PA % 1024 == 0, "1024-byte stage alignment");
  // A warp that takes every n-th slice (A: n = 2, B: n = NB) must never wait
  // on a stage more than one phase ahead of its barrier (parity waits alias).
  // For the unpacked ring the MMA has consumed slice h - n - SU when the warp
  // reaches slice h, so n <= SU suffices; for the packed ring the TMA copies
  // may land out of order, so the warp must itself have waited for the
  // stage's previous fill (slice h - SP): SP a multiple of n.
  static_assert(NB <= SU && NA <= SU && SP % NB == 0 && SP % NA == 0, "slices per feed warp");
};

template <int EPI, int NB>
__global__ void __launch_bounds__(PCfg<NB>::THREADS, 1)
    gemm_w4a4_persistent_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmA,
                                const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmY) {
  using C = PCfg<NB>;
  constexpr int SP = C::SP, SU = C::SU, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pfull = bars;
  uint64_t* pempty = pfull + SP;
  uint64_t* full_u = pempty + SP;
  uint64_t* empty_u = full_u + SU;
  uint64_t* acc_full = empty_u + SU;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* done_bar = acc_empty + 1;
  uint64_t* fin_bar = done_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);

  const uint32_t crank = cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs_m = (p.rowsA + 2 * kBM - 1) / (2 * kBM);
  const int tiles_n = (p.rowsB + BN - 1) / BN;
  const int ntiles = pairs_m * tiles_n;
  const int cid = int(blockIdx.x >> 1), ncl = int(gridDim.x >> 1);
  const int my_tiles = ntiles > cid ? (ntiles - cid + ncl - 1) / ncl : 0;
  const int nkb = p.num_kb;
  const uint32_t total = uint32_t(my_tiles) * uint32_t(nkb);  // K slices this CTA streams

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], C::FEED);
    }
    for (int s = 0; s < SU; ++s) {
      mbar_init(&full_u[s], C::FEED + 1);
      mbar_init(&empty_u[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * 8);
    mbar_init(done_bar, 1);
    mbar_init(fin_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the other CTA's barriers are initialized and its tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      uint32_t g = 0;
      int arow = 0, brow = 0;
      for (int t = cid, i = 0; g < total;) {
        if (i == 0) {
          // a pair's second CTA past the last A (or B) rows still feeds its
          // other operand; it loads in-range rows whose products are never stored
          const int ta = 2 * (t % pairs_m) + int(crank), tb = t / pairs_m;
          arow = ta * kBM < p.rowsA ? ta * kBM : 0;
          const int br = tb * BN + int(crank) * C::BR;
          brow = br < p.rowsB ? br : 0;
        }
        const int sp = int(g % SP);
        if (!mbar_wait(&pempty[sp], ((g / SP) & 1) ^ 1)) {
          record_error(p.err, kErrTimeoutProducer);
          break;
        }
        uint8_t* st = smem + C::OFF_P + sp * C::P_STAGE;
        mbar_arrive_expect_tx(&pfull[sp], C::P_STAGE);
        tma_load_2d(st, &tmA, &pfull[sp], i * kPK, arow);
        tma_load_2d(st + C::PA, &tmB, &pfull[sp], i * kPK, brow);
        ++g;
        if (++i == nkb) {
          i = 0;
          t += ncl;
        }
      }
      for (uint32_t j = g > uint32_t(SP) ? g - SP : 0; j < g; ++j)
        if (!mbar_wait(&pfull[j % SP], (j / SP) & 1)) {
          record_error(p.err, kErrTimeoutDrain);
          break;
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && crank == 0) {
      constexpr uint32_t idesc = idesc_i8(2 * kBM, BN);
      uint32_t g = 0;
      bool ok = true;
      for (int tl = 0; tl < my_tiles && ok; ++tl) {
        // both CTAs' epilogues have read the previous tile's accumulator
        if (!mbar_wait_cluster(acc_empty, (tl & 1) ^ 1)) {
          record_error(p.err, kErrTimeoutMma);
          break;
        }
        tc_fence_after();
        for (int i = 0; i < nkb; ++i, ++g) {
          const int su = int(g % SU);
          if (!mbar_wait_cluster(&full_u[su], (g / SU) & 1)) {
            record_error(p.err, kErrTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = tmem + uint32_t(C::A_COL0 + su * C::A_STAGE_COLS);
          const uint32_t b0 = smem_u32(smem + C::OFF_UNP + su * C::UNP_STAGE);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8_ts_pair(tmem, a0 + uint32_t(8 * k), sdesc_k128_sw128(b0 + 32 * k), idesc,
                           uint32_t(i > 0 || k > 0));
          mma_commit_pair(&empty_u[su], 3);
        }
        if (ok) mma_commit_pair(acc_full, 3);
      }
      mma_commit_pair(done_bar, 3);
      if (!mbar_wait(done_bar, 0)) record_error(p.err, kErrTimeoutDrain);
    } else if (lane == 0) {
      // CTA 1 stays until CTA 0's MMAs, which read its shared and tensor
      // memory, have completed
      if (!mbar_wait(done_bar, 0)) record_error(p.err, kErrTimeoutDrain);
    }
  } else if (warp < C::B_WARP0) {
    // ------------------------------------------------------------ A rows -> tensor-memory ring
    // NA warps per lane quadrant take the slices in turn, so each has NA
    // slice periods for its load - unpack - store - fence - arrive chain (in
    // CTA 1 the arrival is a cluster-scope release, a memory fence)
    const int q = warp & 3, par = (warp - 2) >> 2;  // quadrant, turn (0 .. NA - 1)
    const int row = q * 32 + lane;
    const int sw = (row >> 1) & 3;  // 64-byte swizzle: chunk c of this row sits at chunk c ^ sw
    const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + uint32_t(C::A_COL0);
    bool ok = true;
    for (uint32_t g = uint32_t(par); g < total; g += C::NA) {
      const int sp = int(g % SP), su = int(g % SU);
      bool fail = !warp_wait(&pfull[sp], (g / SP) & 1);
      uint4 w[4];
      if (!fail) {
        const uint8_t* src = smem + C::OFF_P + sp * C::P_STAGE + row * kPK;
#pragma unroll
        for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
        fail = !warp_wait(&empty_u[su], ((g / SU) & 1) ^ 1);
      }
      if (!fail) {
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          unpack8_hi(w[c].x, r[8 * c + 0], r[8 * c + 1]);
          unpack8_hi(w[c].y, r[8 * c + 2], r[8 * c + 3]);
          unpack8_hi(w[c].z, r[8 * c + 4], r[8 * c + 5]);
          unpack8_hi(w[c].w, r[8 * c + 6], r[8 * c + 7]);
        }
        tmem_st_32x32(ta + uint32_t(su * C::A_STAGE_COLS), r);
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (crank == 0) {
        if (fail) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive(&pempty[sp]);
          mbar_arrive(&full_u[su]);
        }
      } else {
        // the slice's group meets; its B-warp publishes the slice to CTA 0
        if (named_barrier_or(2 + par, 160, fail)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive(&pempty[sp]);
      }
    }
    if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
  } else if (warp < C::EPI_WARP0) {
    // ------------------------------------------------------------ weight rows -> shared-memory ring
    // B-warp b unpacks whole half-slices g = b, b + NB, ...: lane l takes the
    // 16-byte pieces it * 32 + l (row it * 8 + l / 4, piece l % 4 of the row)
    const int bw = warp - C::B_WARP0;
    const int r7 = lane >> 2, c = lane & 3;
    const uint32_t dst0 = uint32_t(r7 * 128 + (((2 * c) ^ r7) << 4));
    const uint32_t dst1 = uint32_t(r7 * 128 + (((2 * c + 1) ^ r7) << 4));
    bool ok = true;
    for (uint32_t g = uint32_t(bw); g < total; g += NB) {
      const int sp = int(g % SP), su = int(g % SU);
      bool fail = !warp_wait(&pfull[sp], (g / SP) & 1);
      if (!fail) {
        const uint8_t* pb = smem + C::OFF_P + sp * C::P_STAGE + C::PA + lane * 16;
        uint8_t* uk = smem + C::OFF_UNP + su * C::UNP_STAGE;
        constexpr int kIt = C::BR / 8;  // 8 rows (32 pieces) per step
#pragma unroll
        for (int it0 = 0; it0 < kIt; it0 += 4) {
          uint4 w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const uint4*>(pb + (it0 + u) * 512);
          if (it0 == 0 && !warp_wait(&empty_u[su], ((g / SU) & 1) ^ 1)) {
            fail = true;
            break;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 o0, o1;
            unpack8_hi(w[u].x, o0.x, o0.y);
            unpack8_hi(w[u].y, o0.z, o0.w);
            unpack8_hi(w[u].z, o1.x, o1.y);
            unpack8_hi(w[u].w, o1.z, o1.w);
            *reinterpret_cast<uint4*>(uk + (it0 + u) * 1024 + dst0) = o0;
            *reinterpret_cast<uint4*>(uk + (it0 + u) * 1024 + dst1) = o1;
          }
        }
      }
      if (!fail) fence_proxy_async_smem();
      __syncwarp();
      if (crank == 0) {
        if (fail) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive(&pempty[sp]);
          mbar_arrive(&full_u[su]);
        }
      } else {
        // the slice's group (this warp and the 4 A-warps of turn bw) meets;
        // one cluster-scope release publishes all their operand writes
        if (named_barrier_or(2 + bw, 160, fail)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive(&pempty[sp]);
          mbar_arrive_cluster(&full_u[su], 0);
        }
      }
    }
    if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::EPI_WARP0;  // 0..7
    const int q = warp & 3;             // tensor-memory lane quadrant this warp may access
    const int h = e >> 2;               // column half
    const int et = e * 32 + lane;       // 0..255: loads one weight scale per tile
    const uint32_t tq = tmem + (uint32_t(q * 32) << 16);
    float* sws = reinterpret_cast<float*>(smem + C::OFF_SCALE);
    uint8_t* stg = smem + C::OFF_STG + e * 2 * C::STG;
    const int swz = (lane >> 1) & 3;  // 64-byte swizzle of the staged block (row = lane)
    if (lane == 0) prefetch_tensormap(&tmY);
    int tl = 0, blk = 0;
    for (int t = cid; t < ntiles; t += ncl, ++tl) {
      const int ta = 2 * (t % pairs_m) + int(crank), n0 = (t / pairs_m) * BN;
      float* sb = sws + (tl & 1) * BN;  // double-buffered: the other buffer may still be read
      sb[et] = n0 + et < p.N ? __ldg(p.sw + n0 + et) : 0.f;
      const int row0 = ta * kBM + q * 32;
      const int row = row0 + lane;
      const float sxm = (EPI == kEpiRow && row < p.M) ? p.sx[row] : 1.0f;
      const bool got = warp_wait(acc_full, tl & 1);
      // one decision for all eight warps (they share the barrier below)
      if (named_barrier_or(1, 256, !got)) {
        if (lane == 0) record_error(p.err, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      // y = fl(fl(sum * s_x) * s_w) with sum = acc / 256 (exact: acc = 256 sum has
      // at most 23 significant bits, so its conversion is exact too)
      const float2 k8 = make_float2(0.00390625f, 0.00390625f);
      const float2 sx2 = make_float2(sxm, sxm);
#pragma unroll 1
      for (int c = 0; c < 4; ++c, ++blk) {
        const int c0 = h * 128 + c * 32;
        uint8_t* buf = stg + (blk & 1) * C::STG;
        // the TMA store that last read this block has finished reading it
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint32_t v[32];
        tmem_ld_32x32(tq + uint32_t(c0), v);
        tmem_wait_ld();
        if (c == 3) {
          // the accumulator is free for the next tile once every warp of both CTAs has read it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (crank == 0)
              mbar_arrive(acc_empty);
            else
              mbar_arrive_cluster(acc_empty, 0);
          }
        }
        const float4* sb4 = reinterpret_cast<const float4*>(sb + c0);
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {  // 16-byte pieces: 8 columns each
          uint4 o;
          uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float4 w = sb4[2 * pc + hh];  // the same address in every lane: a broadcast
            float2 a0 = make_float2(__int2float_rn(int(v[8 * pc + 4 * hh])), __int2float_rn(int(v[8 * pc + 4 * hh + 1])));
            float2 a1 = make_float2(__int2float_rn(int(v[8 * pc + 4 * hh + 2])), __int2float_rn(int(v[8 * pc + 4 * hh + 3])));
            a0 = fmul2(a0, k8);
            a1 = fmul2(a1, k8);
            if (EPI == kEpiRow) {
              a0 = fmul2(a0, sx2);
              a1 = fmul2(a1, sx2);
            }
            a0 = fmul2(a0, make_float2(w.x, w.y));
            a1 = fmul2(a1, make_float2(w.z, w.w));
            const __half2 h0 = __floats2half2_rn(a0.x, a0.y), h1 = __floats2half2_rn(a1.x, a1.y);
            ow[2 * hh] = *reinterpret_cast<const uint32_t*>(&h0);
            ow[2 * hh + 1] = *reinterpret_cast<const uint32_t*>(&h1);
          }
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((pc ^ swz) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // rows past M and columns past N are clipped by the copy
          tma_store_2d(&tmY, buf, n0 + c0, row0);
          bulk_commit_group();
        }
      }
    }
    // the output is written before the CTA leaves
    if (lane == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA frees the pair's tensor memory before both are done with it
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(fin_bar, crank ^ 1u);
    if (!mbar_wait_cluster(fin_bar, 0)) record_error(p.err, kErrTimeoutDrain);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- decode
//
// Few tokens (M <= 64): the GEMM is a stream of the packed weights, so the
// kernel is built around keeping that stream flowing.  The weights take the
// 128-row MMA side (tiles of 128 output channels), the tokens the N side
// (BN = 16, 32 or 64).  The launch is one persistent wave (two CTAs per SM);
// the (tile, K slice) pairs, tile-major, are split into equal contiguous
// ranges, one per CTA (stream-K), so every CTA streams the same number of
// weight bytes whatever the tile count.  A range covers whole tiles and at
// most a partial tile at each end; whole tiles are written directly.  For a
// split tile each CTA stores its exact int32 sums into its own slot of the
// workspace and counts itself in on the tile's counter; the CTA that arrives
// last adds the slots of all the tile's CTAs (integer sums: the order does
// not matter), dequantizes and writes the tile, and its arrival has already
// wrapped the counter back to 0.
// Fused decode linear (FUSED): the tokens arrive as fp16 and each CTA first
// quantizes an equal share of them with the static per-channel scales (the
// same static_codes8 as fq_quant_act) into the workspace; a grid barrier
// (the launch is cooperative, so every CTA is resident) orders those codes
// before the first token tile is loaded.  The first weight stages are issued
// before the quantization, so the weight stream starts at once.
//   warp 0      one thread issues TMA loads of packed 128 x 64-byte weight
//               slices (64-byte swizzle) and the tokens' slices into a ring
//   warp 1      tensor-memory allocation and the MMA-issuing thread; the
//               accumulator is double-buffered across tile segments
//   UG groups of 4 warps read one weight row each from the ring and unpack it
//               into a tensor-memory A ring (group g takes the slices
//               i = g mod UG, so UG slices are unpacked at once)
//   UG groups of 2 warps unpack the tokens into the 128-byte-swizzled B ring
//   4 warps     epilogue of each tile segment, overlapping the next one
// Two CTAs per SM run one unpacking group each; the fused kernel's single
// CTA per SM runs two.

// ONE: one CTA per SM (the fused kernel's cooperative launch: the occupancy
// calculation counts one resident CTA per SM for kernels that allocate
// tensor memory), with a deeper ring to keep as many weight bytes in flight
// as two CTAs do.
template <int BN, bool ONE = false>
struct DecCfg {
  // packed stages (weights + tokens); deeper rings (9-11 stages) measured
  // slower at two CTAs per SM
  static constexpr int SP = ONE ? (BN == 64 ? 12 : 16) : (BN == 64 ? 6 : 8);
  static constexpr int UG = ONE ? 2 : 1;          // unpacking groups
  static constexpr int ACC = BN < 32 ? 32 : BN;   // columns of one accumulator
  // MMA-issuing threads (warp 1, then warps I_WARP0...): a tcgen05.mma of
  // N = BN <= 64 holds its issuing thread for about as long as the tensor
  // core needs for it, so one issuer caps a CTA at about one K slice per four
  // MMA issue times.  Issuer j issues k-steps j, j + NI, ... of every slice
  // into its own accumulator; the epilogue adds the NI accumulators.
  static constexpr int NI = ONE ? (BN == 64 ? 2 : 4) : 2;
  // accumulator buffers per issuer (2: the epilogue of one tile segment
  // overlaps the MMAs of the next)
  static constexpr int NACC = (!ONE && BN == 64) ? 1 : 2;
  static constexpr int W_WARP0 = 2;               // first weight-unpacking warp
  static constexpr int T_WARP0 = W_WARP0 + 4 * UG;  // first token-unpacking warp
  static constexpr int E_WARP0 = T_WARP0 + 2 * UG;  // first epilogue warp
  static constexpr int I_WARP0 = E_WARP0 + 4;     // issuers 1 .. NI - 1
  static constexpr int THREADS = 32 * (I_WARP0 + NI - 1);
  static constexpr int SU = ONE ? 8 : 4;          // unpacked stages (each a full MMA round trip deep)
  static constexpr int P_STAGE = kBM * kPK;       // weights: 128 rows x 64 bytes
  static constexpr int X_STAGE = BN * kPK;        // tokens: BN rows x 64 bytes
  static constexpr int B_STAGE = BN * kBK;        // BN rows x 128 int8, 128-byte swizzle
  static constexpr int OFF_P = 0;
  static constexpr int OFF_X = OFF_P + SP * P_STAGE;
  static constexpr int OFF_B = OFF_X + SP * X_STAGE;
  static constexpr int OFF_BAR = OFF_B + SU * B_STAGE;
  static constexpr int NBAR = 2 * SP + 2 * SU + 5;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;  // tmem address, count of tiles to finish, those tiles
  // two per SM: at least 80 KB, so that no more than two CTAs (2 x 256
  // tensor-memory columns) are resident on one SM
  static constexpr int SMEM_MIN = ONE ? 0 : 80 * 1024;
  static constexpr int SMEM = (OFF_TMEM + 16 + 1024) > SMEM_MIN ? (OFF_TMEM + 16 + 1024) : SMEM_MIN;
  static constexpr int A_COL0 = NACC * NI * ACC;  // accumulators: [buffer][issuer][ACC]
  static constexpr int A_STAGE_COLS = kBK / 4;
  static constexpr int TMEM_NEED = A_COL0 + SU * A_STAGE_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 128 ? 128 : (TMEM_NEED <= 256 ? 256 : 512);
  static_assert(B_STAGE % 1024 == 0 && P_STAGE % 1024 == 0 && X_STAGE % 1024 == 0, "stage alignment");
  static_assert(TMEM_NEED <= (ONE ? 512 : 256), "tensor memory of the CTAs resident on one SM");
  static_assert(ONE ? SMEM <= 227 * 1024 : 2 * (SMEM + 1024) <= 228 * 1024, "resident CTAs per SM");
  static_assert(SP * P_STAGE >= 512, "the finishing pass keeps its slot table in the weight ring");
  static_assert(SP % UG == 0 && SU % UG == 0, "each stage is used by one unpacking group");
  static_assert((kBK / 32) % NI == 0, "every issuer issues the same k-steps of each slice");
};

// The slice range [b0, b1) of CTA c among g CTAs over t slices, and the CTA
// that owns slice s (the inverse: b_c = floor(c t / g)).
__host__ __device__ __forceinline__ long long sk_begin(long long c, long long g, long long t) { return c * t / g; }
__host__ __device__ __forceinline__ int sk_owner(long long s, long long g, long long t) {
  return int(((s + 1) * g - 1) / t);
}

template <int BN, int EPI, bool FUSED>
__global__ void __launch_bounds__(DecCfg<BN, FUSED>::THREADS, FUSED ? 1 : 2)
    gemm_decode_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmX) {
  using C = DecCfg<BN, FUSED>;
  constexpr int SP = C::SP, SU = C::SU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pfull = bars;
  uint64_t* pempty = pfull + SP;
  uint64_t* ufull = pempty + SP;
  uint64_t* uempty = ufull + SU;
  uint64_t* acc_full = uempty + SU;  // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* done_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  int* fin = reinterpret_cast<int*>(smem + C::OFF_TMEM + 4);  // [0] count, [1..2] split tiles this CTA finishes

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = p.num_kb;
  const long long T = (long long)((p.rowsA + kBM - 1) / kBM) * nkb;
  const long long b0 = sk_begin(blockIdx.x, gridDim.x, T), b1 = sk_begin(blockIdx.x + 1, gridDim.x, T);
  const int nsl = int(b1 - b0);  // slices of this CTA
  // fused: stages whose weight tiles are issued before the token quantization
  const int pre = FUSED ? min(nsl, SP) : 0;

  if (threadIdx.x == 0) {
    fin[0] = 0;
    for (int s = 0; s < SP; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], 6);  // 4 weight-row warps + 2 token warps
    }
    for (int s = 0; s < SU; ++s) {
      mbar_init(&ufull[s], 6);
      mbar_init(&uempty[s], C::NI);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], C::NI);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(done_bar, C::NI);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();

  unsigned gen = 0;
  if (FUSED) {
    // the first weight stages (their barriers expect the token bytes too)
    if (threadIdx.x == 0) {
      prefetch_tensormap(&tmA);
      const uint64_t pol = policy_evict_first();
      int tile = int(b0 / nkb), kb = int(b0 - (long long)tile * nkb);
      for (int i = 0; i < pre; ++i, kb = kb + 1 == nkb ? 0 : kb + 1, tile += kb == 0) {
        mbar_arrive_expect_tx(&pfull[i], C::P_STAGE + C::X_STAGE);
        tma_load_2d_hint(smem + C::OFF_P + i * C::P_STAGE, &tmA, &pfull[i], kb * kPK, tile * kBM, pol);
      }
    }
    // this CTA's share of the token codes, 8 per thread-iteration
    const int kp = p.K / 8;
    const long long pieces = (long long)p.M * kp;
    const long long lo = pieces * blockIdx.x / gridDim.x, hi = pieces * (blockIdx.x + 1) / gridDim.x;
    for (long long pc = lo + threadIdx.x; pc < hi; pc += C::THREADS) {
      const int r = int(pc / kp), e0 = int(pc - (long long)r * kp) * 8;
      const uint4 raw = *reinterpret_cast<const uint4*>(p.X + size_t(r) * p.K + e0);
      const uint32_t word = static_codes8(raw, p.sst + e0, p.cst ? p.cst + e0 : nullptr);
      reinterpret_cast<uint32_t*>(p.Xq + size_t(r) * (p.K / 2))[e0 / 8] = word;
    }
    __syncthreads();
    if (threadIdx.x == 0) gen = grid_barrier_arrive(p.sync, gridDim.x);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmX);
      const uint64_t pol = policy_evict_first();   // the weights are read once
      const uint64_t pol_x = policy_evict_last();  // the tokens are read by every CTA
      int issued = 0;
      int tile = int(b0 / nkb), kb = int(b0 - (long long)tile * nkb);  // advanced per slice
      if (FUSED) {
        // the token codes of every CTA are in memory; on a timeout the error
        // is recorded and the pipeline still runs to its end (every copy
        // lands, the results are not to be used)
        if (!grid_barrier_wait(p.sync, gen)) record_error(p.err, kErrTimeoutProducer);
        for (int i = 0; i < pre; ++i, kb = kb + 1 == nkb ? 0 : kb + 1, tile += kb == 0)
          tma_load_2d_hint(smem + C::OFF_X + i * C::X_STAGE, &tmX, &pfull[i], kb * kPK, 0, pol_x);
        issued = pre;
      }
      for (int i = pre; i < nsl; ++i, kb = kb + 1 == nkb ? 0 : kb + 1, tile += kb == 0) {
        const int sp = i % SP;
        if (!mbar_wait(&pempty[sp], ((i / SP) & 1) ^ 1)) {
          record_error(p.err, kErrTimeoutProducer);
          break;
        }
        mbar_arrive_expect_tx(&pfull[sp], C::P_STAGE + C::X_STAGE);
        tma_load_2d_hint(smem + C::OFF_P + sp * C::P_STAGE, &tmA, &pfull[sp], kb * kPK, tile * kBM, pol);
        tma_load_2d_hint(smem + C::OFF_X + sp * C::X_STAGE, &tmX, &pfull[sp], kb * kPK, 0, pol_x);
        ++issued;
      }
      // every issued copy has landed before the CTA may leave (normally the
      // unpacking warps already waited for each of them)
      for (int i = max(0, issued - SP); i < issued; ++i)
        if (!mbar_wait(&pfull[i % SP], (i / SP) & 1)) {
          record_error(p.err, kErrTimeoutDrain);
          break;
        }
    }
  } else if (warp == 1 || warp >= C::I_WARP0) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int iss = warp == 1 ? 0 : warp - C::I_WARP0 + 1;
      constexpr uint32_t idesc = idesc_i8_m128(BN);
      int seg = -1;
      bool ok = true;
      int kb = int(b0 % nkb);  // advanced per slice
      for (int i = 0; i < nsl && ok; ++i, kb = kb + 1 == nkb ? 0 : kb + 1) {
        const int su = i % SU;
        const bool first = i == 0 || kb == 0, last = i == nsl - 1 || kb == nkb - 1;
        if (first) {
          ++seg;
          // the first use of each buffer passes at once (the wait is for the
          // phase before the first); later uses wait for the epilogue of the
          // segment two back
          if (!mbar_wait(&acc_empty[seg % C::NACC], ((seg / C::NACC) & 1) ^ 1)) {
            record_error(p.err, kErrTimeoutMma);
            break;
          }
          tc_fence_after();
        }
        if (!mbar_wait(&ufull[su], (i / SU) & 1)) {
          record_error(p.err, kErrTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(((seg % C::NACC) * C::NI + iss) * C::ACC);
        const uint32_t a0 = tmem + uint32_t(C::A_COL0 + su * C::A_STAGE_COLS);
        const uint32_t bsm = smem_u32(smem + C::OFF_B + su * C::B_STAGE);
#pragma unroll
        for (int k = iss; k < kBK / 32; k += C::NI)
          mma_i8_ts(d, a0 + uint32_t(8 * k), sdesc_k128_sw128(bsm + 32 * k), idesc, uint32_t(!first || k >= C::NI));
        mma_commit(&uempty[su]);
        if (last) mma_commit(&acc_full[seg % C::NACC]);
      }
      mma_commit(done_bar);
      if (!mbar_wait(done_bar, 0)) record_error(p.err, kErrTimeoutDrain);
    }
  } else if (warp < C::T_WARP0) {
    // ------------------------------------------------------------ weight rows -> tensor memory
    const int q = warp & 3;  // tensor-memory lane quadrant this warp may access
    const int grp = (warp - C::W_WARP0) >> 2;
    const int row = q * 32 + lane;
    const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + uint32_t(C::A_COL0);
    const int sw = (row >> 1) & 3;  // 64-byte swizzle: chunk c of this row sits at chunk c ^ sw
    bool ok = true;
    for (int i = grp; i < nsl; i += C::UG) {
      const int sp = i % SP, su = i % SU;
      if (!warp_wait(&pfull[sp], (i / SP) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* src = smem + C::OFF_P + sp * C::P_STAGE + row * kPK;
      uint4 w[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) w[c] = *reinterpret_cast<const uint4*>(src + ((c ^ sw) << 4));
      if (!warp_wait(&uempty[su], ((i / SU) & 1) ^ 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        unpack8_hi(w[c].x, r[8 * c + 0], r[8 * c + 1]);
        unpack8_hi(w[c].y, r[8 * c + 2], r[8 * c + 3]);
        unpack8_hi(w[c].z, r[8 * c + 4], r[8 * c + 5]);
        unpack8_hi(w[c].w, r[8 * c + 6], r[8 * c + 7]);
      }
      tmem_st_32x32(ta + uint32_t(su * C::A_STAGE_COLS), r);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      // The packed stage goes back to the TMA producer only now, after the
      // tensor-memory store has consumed the registers it was read into: a
      // release right after issuing the shared-memory loads let the refill
      // overwrite rows whose reads had not completed yet.
      if (lane == 0) {
        mbar_arrive(&pempty[sp]);
        mbar_arrive(&ufull[su]);
      }
    }
    if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
  } else if (warp < C::E_WARP0) {
    // ------------------------------------------------------------ token rows -> shared memory
    // The packed token slice arrives with the weights in the TMA ring; each
    // lane unpacks fixed 16-byte pieces (consecutive lanes read consecutive
    // pieces, so the reads are free of bank conflicts).
    constexpr int kJobs = BN * 4;                  // 16-byte packed pieces per stage
    constexpr int JPT = (kJobs + 63) / 64;         // per thread (two warps)
    const int grp = (warp - C::T_WARP0) >> 1;
    const int t = ((warp - C::T_WARP0) & 1) * 32 + lane;
    uint32_t dst0[JPT], dst1[JPT];
    bool live[JPT];
#pragma unroll
    for (int it = 0; it < JPT; ++it) {
      const int j = it * 64 + t;
      live[it] = j < kJobs;
      const int brow = live[it] ? (j >> 2) : 0, c = j & 3, r7 = brow & 7;
      const uint32_t rb = uint32_t((brow >> 3) * 1024 + r7 * 128);
      dst0[it] = rb + uint32_t(((2 * c) ^ r7) << 4);
      dst1[it] = rb + uint32_t(((2 * c + 1) ^ r7) << 4);
    }
    bool ok = true;
    for (int i = grp; i < nsl; i += C::UG) {
      const int sp = i % SP, su = i % SU;
      if (!warp_wait(&pfull[sp], (i / SP) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* xs = smem + C::OFF_X + sp * C::X_STAGE;
      uint4 w[JPT];
#pragma unroll
      for (int it = 0; it < JPT; ++it)
        w[it] = live[it] ? *reinterpret_cast<const uint4*>(xs + (it * 64 + t) * 16) : make_uint4(0, 0, 0, 0);
      if (!warp_wait(&uempty[su], ((i / SU) & 1) ^ 1)) {
        ok = false;
        break;
      }
      uint8_t* uk = smem + C::OFF_B + su * C::B_STAGE;
#pragma unroll
      for (int it = 0; it < JPT; ++it) {
        if (!live[it]) continue;
        uint4 o0, o1;
        unpack8_hi(w[it].x, o0.x, o0.y);
        unpack8_hi(w[it].y, o0.z, o0.w);
        unpack8_hi(w[it].z, o1.x, o1.y);
        unpack8_hi(w[it].w, o1.z, o1.w);
        *reinterpret_cast<uint4*>(uk + dst0[it]) = o0;
        *reinterpret_cast<uint4*>(uk + dst1[it]) = o1;
      }
      fence_proxy_async_smem();
      __syncwarp();
      // both stages are released after the stores consumed the loaded registers
      if (lane == 0) {
        mbar_arrive(&pempty[sp]);
        mbar_arrive(&ufull[su]);
      }
    }
    if (!ok && lane == 0) record_error(p.err, kErrTimeoutUnpack);
  } else {
    // ------------------------------------------------------------ epilogue: thread = output channel n
    const int q = warp & 3;
    const int nl = q * 32 + lane;  // channel within the tile
    const uint32_t tl = tmem + (uint32_t(q * 32) << 16);
    const int tile0 = int(b0 / nkb);
    long long s = b0;
    for (int seg = 0; s < b1; ++seg) {
      const int tile = int(s / nkb), kb_lo = int(s - (long long)tile * nkb);
      const int len = int(min((long long)(nkb - kb_lo), b1 - s));
      const bool whole = kb_lo == 0 && len == nkb;
      s += len;
      const int b = seg % C::NACC;
      // the four epilogue warps agree on the outcome (they meet at named barriers below)
      const bool ok = warp_wait(&acc_full[b], (seg / C::NACC) & 1);
      if (named_barrier_or(1, 128, !ok)) {
        if (lane == 0) record_error(p.err, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      const int n = tile * kBM + nl;
      const float swn = (EPI == kEpiRow || EPI == kEpiStatic) && n < p.N ? __ldg(p.sw + n) : 0.f;
      // this CTA's slot for a split tile: 2c for its first tile, 2c + 1 for its last
      int32_t* slot = whole ? nullptr : p.slots + (size_t(2 * blockIdx.x + (tile == tile0 ? 0 : 1)) * p.M) * kBM + nl;
      constexpr int CW = BN >= 32 ? 32 : 16;
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += CW) {
        uint32_t v[32];
        const uint32_t col = tl + uint32_t(b * C::NI * C::ACC + c0);
        if (CW == 32)
          tmem_ld_32x32(col, v);
        else
          tmem_ld_32x16(col, v);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 1; ch < C::NI; ++ch) {
          uint32_t w[32];
          if (CW == 32)
            tmem_ld_32x32(col + uint32_t(ch * C::ACC), w);
          else
            tmem_ld_32x16(col + uint32_t(ch * C::ACC), w);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] += w[j];  // exact int32 sums (two's complement)
        }
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int m = c0 + j;
          if (m >= p.M) break;
          const int32_t ai = int32_t(v[j]) >> 8;
          if (!whole)
            slot[size_t(m) * kBM] = ai;
          else if (n >= p.N)
            continue;
          else if (EPI == kEpiRow)
            p.Y[size_t(m) * p.N + n] = __float2half_rn(__fmul_rn(__fmul_rn(float(ai), __ldg(p.sx + m)), swn));
          else
            p.Y[size_t(m) * p.N + n] = __float2half_rn(__fmul_rn(float(ai), swn));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      if (whole) continue;
      // split tile: count in; the last of its CTAs finishes it at the end
      named_barrier(1, 128);  // every slot row of this CTA is stored
      if (warp == C::E_WARP0 && lane == 0) {
        __threadfence();
        const int cf = sk_owner((long long)tile * nkb, gridDim.x, T);
        const int cl = sk_owner((long long)(tile + 1) * nkb - 1, gridDim.x, T);
        const unsigned nc = unsigned(cl - cf + 1);
        if (atomicInc(p.sync + kSyncTile0 + tile, nc - 1) == nc - 1) {
          __threadfence();
          fin[1 + fin[0]] = tile;
          fin[0] += 1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }

  // The split tiles this CTA arrived last at (at most its first and its
  // last): every thread adds the CTAs' slots, 4 channels per 16-byte load,
  // and writes the fp16 outputs.  The weight ring is idle now; it holds the
  // slot index of each contributing CTA.
  const int nfin = fin[0];
  int* sidx = reinterpret_cast<int*>(smem + C::OFF_P);
  for (int f = 0; f < nfin; ++f) {
    const int tile = fin[1 + f];
    const int cf = sk_owner((long long)tile * nkb, gridDim.x, T);
    const int cl = sk_owner((long long)(tile + 1) * nkb - 1, gridDim.x, T);
    const int nc = cl - cf + 1;
    const long long t_lo = (long long)tile * nkb;
    __syncthreads();  // the previous tile's readers are done with sidx
    for (int j = threadIdx.x; j < nc; j += C::THREADS)
      sidx[j] = 2 * (cf + j) + (sk_begin(cf + j, gridDim.x, T) >= t_lo ? 0 : 1);
    __syncthreads();
    for (int it = threadIdx.x; it < p.M * (kBM / 4); it += C::THREADS) {
      const int m = it / (kBM / 4), nl = (it % (kBM / 4)) * 4;
      const int n = tile * kBM + nl;
      if (n >= p.N) continue;  // N % 8 == 0: four channels are all in range or all out
      int4 a = make_int4(0, 0, 0, 0);
#pragma unroll 8
      for (int j = 0; j < nc; ++j) {
        const int4 v = __ldcg(reinterpret_cast<const int4*>(p.slots + (size_t(sidx[j]) * p.M + m) * kBM + nl));
        a.x += v.x;
        a.y += v.y;
        a.z += v.z;
        a.w += v.w;
      }
      const float4 w = make_float4(__ldg(p.sw + n), __ldg(p.sw + n + 1), __ldg(p.sw + n + 2), __ldg(p.sw + n + 3));
      float y[4];
      if (EPI == kEpiRow) {
        const float sxm = __ldg(p.sx + m);
        y[0] = __fmul_rn(__fmul_rn(float(a.x), sxm), w.x);
        y[1] = __fmul_rn(__fmul_rn(float(a.y), sxm), w.y);
        y[2] = __fmul_rn(__fmul_rn(float(a.z), sxm), w.z);
        y[3] = __fmul_rn(__fmul_rn(float(a.w), sxm), w.w);
      } else {
        y[0] = __fmul_rn(float(a.x), w.x);
        y[1] = __fmul_rn(float(a.y), w.y);
        y[2] = __fmul_rn(float(a.z), w.z);
        y[3] = __fmul_rn(float(a.w), w.w);
      }
      uint2 o;
      __half2* h = reinterpret_cast<__half2*>(&o);
      h[0] = __floats2half2_rn(y[0], y[1]);
      h[1] = __floats2half2_rn(y[2], y[3]);
      *reinterpret_cast<uint2*>(p.Y + size_t(m) * p.N + n) = o;
    }
  }
}

// Zero-point epilogue of the general (min-max) quantizer: with the exact
// int32 products acc = sum_k q_x q_w of the stored signed codes
// (q = u - 2^(b-1)), the product of the dequantized-up-to-scale codes is
// a = acc + o_w S_x + o_x S_w + K o_x o_w (o = 2^(b-1) - z, S = sum_k q per
// row: sum_k (u_x - z_x)(u_w - z_w) expanded), and y = fp16((a * s_x) * s_w).
// |a| <= 15 * 15 * K < 2^24, so its float32 conversion is exact.
// One thread: 8 consecutive outputs of one row (a 16-byte store).
__global__ void __launch_bounds__(256) zp_epilogue_kernel(const int32_t* __restrict__ acc,
                                                          const float* __restrict__ bx,
                                                          const float* __restrict__ bw, __half* __restrict__ Y,
                                                          int M, int N, int K) {
  const int32_t* ox = reinterpret_cast<const int32_t*>(bx + M);
  const int32_t* Sx = reinterpret_cast<const int32_t*>(bx + 2 * size_t(M));
  const int32_t* ow = reinterpret_cast<const int32_t*>(bw + N);
  const int32_t* Sw = reinterpret_cast<const int32_t*>(bw + 2 * size_t(N));
  const size_t pieces = size_t(M) * (N / 8);
  for (size_t pc = blockIdx.x * size_t(blockDim.x) + threadIdx.x; pc < pieces; pc += size_t(gridDim.x) * blockDim.x) {
    const int m = int(pc / (N / 8)), n0 = int(pc % (N / 8)) * 8;
    const int4 a0 = *reinterpret_cast<const int4*>(acc + size_t(m) * N + n0);
    const int4 a1 = *reinterpret_cast<const int4*>(acc + size_t(m) * N + n0 + 4);
    const int av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float sxm = __ldg(bx + m);
    const int oxm = __ldg(ox + m), Sxm = __ldg(Sx + m);
    float y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + j;
      const int own = __ldg(ow + n);
      const int a = av[j] + own * Sxm + oxm * __ldg(Sw + n) + K * oxm * own;
      y[j] = __fmul_rn(__fmul_rn(__int2float_rn(a), sxm), __ldg(bw + n));
    }
    store_half8(Y + size_t(m) * N + n0, y);
  }
}

struct Plan {
  bool swap;          // decode kernel (weights on the 128-row side)
  bool pair;          // prefill: 256 x BN tiles over CTA pairs
  int bn;
  int epi;
  int ctas;           // decode: persistent CTAs sharing the slice sequence
  bool partial;       // decode: some tile is split between CTAs (workspace slots + counters)
};

int pick_bn_swap(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

// fused: the decode kernel that quantizes the tokens itself waits at a grid
// barrier, so all its CTAs must be resident: one wave at most.
Plan make_plan(int M, int N, int K, int epi_final, int sms, bool fused = false) {
  Plan pl{};
  const int nkb = K / kBK;
  if (epi_final == kEpiGroup) {
    pl.swap = false;
    pl.bn = 128;
    pl.epi = kEpiGroup;
    return pl;
  }
  if (epi_final == kEpiS32 || M > 64) {
    pl.swap = false;
    pl.bn = 256;
    pl.epi = epi_final;
    pl.pair = epi_final != kEpiS32;
    return pl;
  }
  // decode: weights on the 128-row side, tokens on the N side; one wave of
  // two CTAs per SM, each with at least 8 K slices
  pl.swap = true;
  pl.bn = pick_bn_swap(M);
  pl.epi = epi_final;
  const long long tiles = (N + kBM - 1) / kBM;
  const long long T = tiles * nkb;
  // One CTA per tile when the tiles alone fill the resident slots and the
  // token count makes the split-tile path (slot stores, the finishing CTA's
  // reads) cost more than the last wave's imbalance; otherwise stream-K over
  // one wave.
  const long long slots = (fused ? 1LL : 2LL) * sms;
  if (tiles >= slots && M > 16 && !fused)
    pl.ctas = int(tiles);
  else
    pl.ctas = int(std::max<long long>(1, std::min<long long>(slots, T / 8)));
  pl.partial = false;
  for (long long c = 1; c < pl.ctas && !pl.partial; ++c) pl.partial = sk_begin(c, pl.ctas, T) % nkb != 0;
  return pl;
}

template <int BN, int EPI>
fq_status launch_gemm(const GemmParams& gp, dim3 grid, cudaStream_t stream) {
  using C = Cfg<BN, EPI>;
  CUtensorMap ta, tb;
  // packed A: 128 rows x 64 bytes per slice, 64-byte swizzle; packed B: BN rows x 64 bytes
  fq_status st = make_tmap_2d(&ta, gp.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsA),
                              uint64_t(gp.K) / 2, uint32_t(kPK), uint32_t(kBM), CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != FQ_OK) return st;
  st = make_tmap_2d(&tb, gp.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsB), uint64_t(gp.K) / 2,
                    uint32_t(kPK), uint32_t(BN));
  if (st != FQ_OK) return st;
  auto kern = gemm_w4a4_kernel<BN, EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the GEMM", C::SMEM);
  const cudaError_t e = launch_pdl(kern, grid, dim3(threads_of<EPI>()), C::SMEM, stream, gp, ta, tb);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FQ_ERR_CUDA, "gemm_w4a4_kernel: %s", cudaGetErrorString(e));
  }
  return check_launch("gemm_w4a4_kernel");
}

constexpr int kPersistNB = 3;  // weight-unpack warps of the persistent kernel

template <int EPI>
fq_status launch_gemm_persistent(const GemmParams& gp, cudaStream_t stream) {
  using C = PCfg<kPersistNB>;
  CUtensorMap ta, tb;
  fq_status st = make_tmap_2d(&ta, gp.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsA),
                              uint64_t(gp.K) / 2, uint32_t(kPK), uint32_t(kBM), CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != FQ_OK) return st;
  st = make_tmap_2d(&tb, gp.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsB), uint64_t(gp.K) / 2,
                    uint32_t(kPK), uint32_t(C::BR));
  if (st != FQ_OK) return st;
  CUtensorMap ty;  // fp16 output in 32 x 32 blocks, 64-byte swizzle (the staging layout)
  st = make_tmap_2d(&ty, gp.Y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, uint64_t(gp.N), uint64_t(gp.M), uint64_t(gp.N) * 2, 32u,
                    32u, CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != FQ_OK) return st;
  auto kern = gemm_w4a4_persistent_kernel<EPI, kPersistNB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the GEMM", C::SMEM);
  const int pairs_m = (gp.rowsA + 2 * kBM - 1) / (2 * kBM);
  const int tiles_n = (gp.rowsB + C::BN - 1) / C::BN;
  const int clusters = std::max(1, std::min(pairs_m * tiles_n, sm_count() / 2));
  const cudaError_t e =
      launch_pdl_cluster(kern, dim3(2 * clusters), dim3(C::THREADS), C::SMEM, stream, 2, gp, ta, tb, ty);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FQ_ERR_CUDA, "gemm_w4a4_persistent_kernel: %s", cudaGetErrorString(e));
  }
  return check_launch("gemm_w4a4_persistent_kernel");
}

template <int BN, int EPI, bool FUSED>
fq_status launch_decode(const GemmParams& gp, dim3 grid, cudaStream_t stream) {
  using C = DecCfg<BN, FUSED>;
  CUtensorMap tm, tx;
  fq_status st = make_tmap_2d(&tm, gp.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsA),
                              uint64_t(gp.K) / 2, uint32_t(kPK), uint32_t(kBM), CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != FQ_OK) return st;
  st = make_tmap_2d(&tx, gp.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, uint64_t(gp.K) / 2, uint64_t(gp.rowsB), uint64_t(gp.K) / 2,
                    uint32_t(kPK), uint32_t(BN));
  if (st != FQ_OK) return st;
  auto kern = gemm_decode_kernel<BN, EPI, FUSED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return fail(FQ_ERR_CUDA, "cannot reserve %d bytes of shared memory for the decode GEMM", C::SMEM);
  if (FUSED) {
    // every CTA must be resident at once for the grid barrier
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::THREADS, C::SMEM) != cudaSuccess ||
        static_cast<long long>(per_sm) * sm_count() < static_cast<long long>(grid.x)) {
      cudaGetLastError();
      return FQ_ERR_UNSUPPORTED;  // the caller quantizes separately
    }
    const cudaError_t e = launch_coop_pdl(kern, grid, dim3(C::THREADS), C::SMEM, stream, gp, tm, tx);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return FQ_ERR_UNSUPPORTED;
    }
  } else {
    const cudaError_t e = launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM, stream, gp, tm, tx);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(FQ_ERR_CUDA, "gemm_decode_kernel: %s", cudaGetErrorString(e));
    }
  }
  return check_launch("gemm_decode_kernel");
}

fq_status dispatch(const Plan& pl, const GemmParams& gp, dim3 grid, cudaStream_t s) {
  if (!pl.swap) {
    switch (pl.epi) {
      case kEpiRow: return pl.pair ? launch_gemm_persistent<kEpiRow>(gp, s) : launch_gemm<256, kEpiRow>(gp, grid, s);
      case kEpiStatic:
        return pl.pair ? launch_gemm_persistent<kEpiStatic>(gp, s) : launch_gemm<256, kEpiStatic>(gp, grid, s);
      case kEpiS32: return launch_gemm<256, kEpiS32>(gp, grid, s);
      case kEpiGroup: return launch_gemm<128, kEpiGroup>(gp, grid, s);
      default: break;
    }
  } else {
#define FQ_SWAP_CASES(BNV)                                                     \
  if (pl.bn == BNV) {                                                          \
    switch (pl.epi) {                                                          \
      case kEpiRow: return launch_decode<BNV, kEpiRow, false>(gp, grid, s);    \
      case kEpiStatic:                                                         \
        return gp.X ? launch_decode<BNV, kEpiStatic, true>(gp, grid, s)        \
                    : launch_decode<BNV, kEpiStatic, false>(gp, grid, s);      \
      default: break;                                                          \
    }                                                                          \
  }
    FQ_SWAP_CASES(16)
    FQ_SWAP_CASES(32)
    FQ_SWAP_CASES(64)
#undef FQ_SWAP_CASES
  }
  return fail(FQ_ERR_UNSUPPORTED, "no GEMM variant for this plan");
}

// Tokens that the fused decode kernel quantizes itself (static scales).
struct FusedTokens {
  const __half* X;
  const float* sst;
  const float* cst;
};

// Decode workspace: the synchronization block, then the split tiles' slots
// (two per CTA).  The fused kernel always needs the block (its grid barrier).
size_t decode_ws_bytes(const Plan& pl, int M, int N, bool fused) {
  (void)N;
  if (!pl.swap) return 0;
  if (!pl.partial) return fused ? kSyncBytes : 0;
  return kSyncBytes + size_t(2) * pl.ctas * M * kBM * sizeof(int32_t);
}

fq_status check_sizes(int M, int N, int K) {
  FQ_CHECK_ARG(M >= 1, "M = %d must be >= 1", M);
  FQ_CHECK_ARG(N >= 8 && N % 8 == 0, "N = %d must be a positive multiple of 8", N);
  FQ_CHECK_ARG(K >= kBK && K <= kMaxK && K % kBK == 0, "K = %d must be a multiple of 128 in [128, %d]", K, kMaxK);
  return FQ_OK;
}

fq_status gemm_impl(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w, int M, int N, int K,
                    int epi_final, uint16_t* Y, int32_t* acc_out, void* ws, size_t ws_bytes, cudaStream_t stream,
                    const FusedTokens* fused = nullptr) {
  fq_status st = check_sizes(M, N, K);
  if (st != FQ_OK) return st;
  FQ_CHECK_ARG(Xq && Wq, "Xq and Wq must be non-NULL");
  FQ_CHECK_ARG(aligned(Xq, 16) && aligned(Wq, 16), "Xq and Wq must be 16-byte aligned");
  if (epi_final == kEpiS32) {
    FQ_CHECK_ARG(acc_out && aligned(acc_out, 4), "the int32 output must be non-NULL and aligned");
  } else {
    FQ_CHECK_ARG(Y && aligned(Y, 16), "Y must be non-NULL and 16-byte aligned");
    FQ_CHECK_ARG(s_w && aligned(s_w, 4), "s_w must be non-NULL and aligned");
    if (epi_final != kEpiStatic) FQ_CHECK_ARG(s_x && aligned(s_x, 2), "s_x must be non-NULL and aligned");
  }
  unsigned* err = device_error_word();
  if (!err) return fail(FQ_ERR_CUDA, "device error word unavailable");
  const int sms = sm_count();
  Plan pl = make_plan(M, N, K, epi_final, sms, fused != nullptr);
  const size_t need = decode_ws_bytes(pl, M, N, fused != nullptr);
  if (need > 0) FQ_CHECK_ARG(ws && ws_bytes >= need && aligned(ws, 256), "workspace of %zu bytes required", need);
  if (pl.swap && pl.partial)
    FQ_CHECK_ARG((N + kBM - 1) / kBM <= kMaxSyncTiles, "N = %d has more than %d tiles of 128", N, kMaxSyncTiles);

  GemmParams gp{};
  gp.M = M;
  gp.N = N;
  gp.K = K;
  gp.num_kb = K / kBK;
  gp.err = err;
  gp.Y = reinterpret_cast<__half*>(Y);
  if (epi_final == kEpiRow) gp.sx = static_cast<const float*>(s_x);
  if (epi_final == kEpiRow || epi_final == kEpiStatic) gp.sw = static_cast<const float*>(s_w);
  if (epi_final == kEpiGroup) {
    gp.gsx = static_cast<const __half*>(s_x);
    gp.gsw = static_cast<const __half*>(s_w);
  }
  gp.acc = epi_final == kEpiS32 ? acc_out : nullptr;
  if (need > 0) {
    gp.sync = static_cast<unsigned*>(ws);
    gp.slots = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kSyncBytes);
  }
  if (fused) {
    gp.X = fused->X;
    gp.sst = fused->sst;
    gp.cst = fused->cst;
    gp.Xq = const_cast<uint8_t*>(Xq);
  }

  gp.A = pl.swap ? Wq : Xq;
  gp.B = pl.swap ? Xq : Wq;
  gp.rowsA = pl.swap ? N : M;
  gp.rowsB = pl.swap ? M : N;

  const dim3 grid = pl.swap ? dim3(pl.ctas) : dim3((gp.rowsA + kBM - 1) / kBM, (gp.rowsB + pl.bn - 1) / pl.bn, 1);
  return dispatch(pl, gp, grid, stream);
}

// The general quantizer's GEMM: the exact int32 products of the stored codes
// into the workspace, then the zero-point epilogue.
fq_status gemm_zp(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w, int M, int N, int K,
                  uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t stream) {
  fq_status st = check_sizes(M, N, K);
  if (st != FQ_OK) return st;
  FQ_CHECK_ARG(Y && aligned(Y, 16), "Y must be non-NULL and 16-byte aligned");
  FQ_CHECK_ARG(s_x && s_w && aligned(s_x, 4) && aligned(s_w, 4), "the scale blocks must be non-NULL and aligned");
  // the products go after the synchronization block, which stays untouched
  const size_t need = kSyncBytes + size_t(M) * N * sizeof(int32_t);
  FQ_CHECK_ARG(ws && ws_bytes >= need && aligned(ws, 256), "workspace of %zu bytes required", need);
  int32_t* acc = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kSyncBytes);
  st = gemm_impl(Xq, nullptr, Wq, nullptr, M, N, K, kEpiS32, nullptr, acc, nullptr, 0, stream);
  if (st != FQ_OK) return st;
  const size_t pieces = size_t(M) * (N / 8);
  const int grid = int(std::max<size_t>(1, std::min<size_t>((pieces + 255) / 256, size_t(sm_count()) * 8)));
  zp_epilogue_kernel<<<grid, 256, 0, stream>>>(acc, static_cast<const float*>(s_x),
                                               static_cast<const float*>(s_w), reinterpret_cast<__half*>(Y), M, N,
                                               K);
  return check_launch("zp_epilogue_kernel");
}

}  // namespace

size_t gemm_workspace_bytes(int M, int N, int K, fq_gran gran) {
  if (M < 1 || N < 8 || K < kBK || K % kBK) return 0;
  if (gran == FQ_DYNAMIC_ROW_ZP) return kSyncBytes + size_t(M) * N * sizeof(int32_t);  // the exact int32 products
  const int epi = gran == FQ_DYNAMIC_GROUP ? kEpiGroup : (gran == FQ_STATIC_CHANNEL ? kEpiStatic : kEpiRow);
  const Plan pl = make_plan(M, N, K, epi, sm_count());
  size_t need = decode_ws_bytes(pl, M, N, false);
  if (gran == FQ_STATIC_CHANNEL)  // room for the fused decode linear's plan too
    need = std::max(need, decode_ws_bytes(make_plan(M, N, K, epi, sm_count(), true), M, N, true));
  return need;
}

size_t sync_block_bytes() { return kSyncBytes; }

// The fused decode linear: static per-channel quantization of the tokens
// inside the decode GEMM launch.  FQ_ERR_UNSUPPORTED (with no error text and
// nothing launched) when the shape is not a decode shape or the cooperative
// launch is not available; the caller then quantizes in a launch of its own.
fq_status decode_linear_fused(const uint16_t* X, const float* sst, const float* cst, uint8_t* Xq, const uint8_t* Wq,
                              const void* s_w, int M, int N, int K, uint16_t* Y, void* ws, size_t ws_bytes,
                              cudaStream_t stream) {
  const Plan pl = make_plan(M, N, K, kEpiStatic, sm_count(), true);
  if (!pl.swap) return FQ_ERR_UNSUPPORTED;
  const FusedTokens ft{reinterpret_cast<const __half*>(X), sst, cst};
  return gemm_impl(Xq, nullptr, Wq, s_w, M, N, K, kEpiStatic, Y, nullptr, ws, ws_bytes, stream, &ft);
}

}  // namespace fq

extern "C" {

fq_status fq_w4a4_gemm(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w, int M, int N, int K,
                       fq_gran gran, uint16_t* Y, void* workspace, size_t ws_bytes, void* stream) {
  fq::clear_error();
  int epi;
  switch (gran) {
    case FQ_DYNAMIC_ROW: epi = fq::kEpiRow; break;
    case FQ_STATIC_CHANNEL: epi = fq::kEpiStatic; break;
    case FQ_DYNAMIC_GROUP: epi = fq::kEpiGroup; break;
    case FQ_DYNAMIC_ROW_ZP: return fq::gemm_zp(Xq, s_x, Wq, s_w, M, N, K, Y, workspace, ws_bytes,
                                               static_cast<cudaStream_t>(stream));
    default: return fq::fail(FQ_ERR_UNSUPPORTED, "granularity %d is not provided", int(gran));
  }
  return fq::gemm_impl(Xq, s_x, Wq, s_w, M, N, K, epi, Y, nullptr, workspace, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

fq_status fq_w4a4_gemm_s32(const uint8_t* Xq, const uint8_t* Wq, int M, int N, int K, int32_t* acc, void* stream) {
  fq::clear_error();
  return fq::gemm_impl(Xq, nullptr, Wq, nullptr, M, N, K, fq::kEpiS32, nullptr, acc, nullptr, 0,
                       static_cast<cudaStream_t>(stream));
}

size_t fq_gemm_workspace_size(int M, int N, int K, fq_gran gran) { return fq::gemm_workspace_bytes(M, N, K, gran); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point that allocates nothing.
//
// Some callers cannot hand the GEMM a workspace: for example a plugin or
// callback running inside another runtime that owns all device memory and
// gives out none, or a serving loop that forbids device allocation after
// start-up so that its memory use stays fixed (and because cudaMalloc may
// synchronize the device and stall other streams).  For them the split-K
// partial sums live in this file-scope buffer instead.  Every GPU that loads
// the library keeps this buffer for the life of the process.
namespace fq {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB: counters + split tiles' partial sums
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the buffer on the current device, looked up once per
// device (the host-side name of the array is not a device address).
void* noalloc_scratch(fq_status* st) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kNoAllocMaxDevices) {
    *st = fail(FQ_ERR_CUDA, "no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[d]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      *st = fail(FQ_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return nullptr;
    }
    g_noalloc_ptr[d] = ptr;
  }
  *st = FQ_OK;
  return g_noalloc_ptr[d];
}
}  // namespace
}  // namespace fq

extern "C" fq_status fq_w4a4_gemm_noalloc(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w,
                                          int M, int N, int K, fq_gran gran, uint16_t* Y, void* stream) {
  fq::clear_error();
  int epi;
  switch (gran) {
    case FQ_DYNAMIC_ROW: epi = fq::kEpiRow; break;
    case FQ_STATIC_CHANNEL: epi = fq::kEpiStatic; break;
    case FQ_DYNAMIC_GROUP: epi = fq::kEpiGroup; break;
    default: return fq::fail(FQ_ERR_UNSUPPORTED, "granularity %d is not provided", int(gran));
  }
  const size_t need = fq_gemm_workspace_size(M, N, K, gran);
  if (need > fq::kNoAllocScratchBytes)
    return fq::fail(FQ_ERR_INVALID,
                    "M = %d, N = %d, K = %d needs %zu bytes of split-K scratch, more than the %zu-byte static buffer "
                    "of fq_w4a4_gemm_noalloc; use fq_w4a4_gemm with a workspace",
                    M, N, K, need, fq::kNoAllocScratchBytes);
  void* ws = nullptr;
  if (need > 0) {
    fq_status st;
    ws = fq::noalloc_scratch(&st);
    if (!ws) return st;
  }
  return fq::gemm_impl(Xq, s_x, Wq, s_w, M, N, K, epi, Y, nullptr, ws, ws ? fq::kNoAllocScratchBytes : 0,
                       static_cast<cudaStream_t>(stream));
}
