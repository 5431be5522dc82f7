/*
 * fq.h - C ABI of libfq.so, a B200 (sm_100a) W4A4 quantized linear layer.
 *
 * The layer computes Y ~ Q(X P) Q(P^-1 W^T): activations X are optionally
 * scaled per channel and passed through a Kronecker-factored affine transform
 * P = P1 (x) P2, quantized online to signed INT4 codes, multiplied with
 * offline-quantized INT4 weights with exact integer accumulation, and
 * dequantized to fp16 (FlatQuant notes, sections 核心思想 and Kronecker 分解;
 * the quantizer Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) of the FRM-PTQ page,
 * section 初步介绍; static per-channel activation scales and quantization-step
 * migration from the MergeQuant page, 核心思路; group-128 scales from FRM-PTQ's
 * multi-granularity group quantization).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Memory. Every tensor pointer is DEVICE memory owned by the caller; the
 *   library never allocates, frees or keeps a pointer after a call returns.
 *   fp16 tensors are passed as uint16_t* holding IEEE binary16 bits.
 *   Matrices are row-major and densely packed.  Pointers read by the tensor
 *   memory accelerator (Xq, Wq, and group scales) must be 16-byte aligned;
 *   all others 4-byte aligned (16-byte for X and Y is recommended).
 * - Streams. `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Every call is asynchronous: it validates its arguments on the host,
 *   enqueues its kernels on `stream` and returns.  No call synchronizes,
 *   except fq_check_device_error.
 * - Errors. On any non-FQ_OK status nothing has been enqueued, except
 *   FQ_ERR_CUDA from a failed launch.  fq_last_error() returns a message
 *   for the calling thread's last failure.  Kernels never trap: a bounded
 *   wait that gives up records FQ_ERR_TIMEOUT in a device word that
 *   fq_check_device_error reads and clears.
 * - INT4 codes. Symmetric, b = 4, zero point z = 2^(b-1) = 8, so the signed
 *   code is q = clamp(round(x/s), -8, 7), round half to even, IEEE float32
 *   division, s = 0 giving q = 0.  Codes are stored two per byte as
 *   two's-complement nibbles: element 2j in bits 0-3 and element 2j+1 in
 *   bits 4-7 of byte j.  A packed [R, K] matrix is uint8 [R, K/2].
 * - Scales. Per row (token or output channel): float32 [R],
 *   s = (max|v| * alpha) / 7 in float32.  Per group of 128 along K: fp16,
 *   the same rule on each group, rounded to fp16 before it is used, stored
 *   GROUP-MAJOR as [K/128][R] (row r of group g at g*R + r).  Static
 *   per-input-channel activation scales: float32 [K], given by the caller.
 * - Sizes. K % 128 == 0 and 128 <= K <= 65536 (quantization kernels: K <=
 *   32768); N % 8 == 0; M >= 1; a transform needs n1 * n2 == K with
 *   1 <= n1, n2 <= 256.
 */
#ifndef FQ_H_
#define FQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FQ_OK = 0,
  FQ_ERR_INVALID = 1,      /* a NULL/misaligned pointer or a size outside the ranges above */
  FQ_ERR_UNSUPPORTED = 2,  /* b, z, group size or a mode/argument combination not provided */
  FQ_ERR_CUDA = 3,         /* the CUDA runtime or driver reported an error (launch, tensor-map encode) */
  FQ_ERR_TIMEOUT = 4       /* a kernel's bounded wait gave up (reported by fq_check_device_error) */
} fq_status;

/* Extent of one scale (FRM-PTQ multi-granularity; MergeQuant static calibration). */
typedef enum {
  FQ_DYNAMIC_ROW = 0,    /* one scale per token (activations) / per output channel (weights) */
  FQ_DYNAMIC_GROUP = 1,  /* one scale per row and group of 128 along K */
  FQ_STATIC_CHANNEL = 2, /* activations only: caller-given float32 scale per input channel */
  FQ_DYNAMIC_ROW_ZP = 3, /* GEMM / linear only: both operands from the min-max quantizer
                            (FQ_ZERO_POINT_MINMAX): per-row scale and zero point */
  FQ_STATIC_RESIDUAL = 4 /* activations only (no transform, no c): each token divided by its
                            root-mean-square S_n = sqrt(sum x^2 / K), then the static
                            per-channel scales (FPTQuant explainer, 伪动态残差缩放); s_x
                            receives S_n float32 [M], and the GEMM runs FQ_DYNAMIC_ROW
                            with s_x = S_n and weights whose s_w carries the static scales */
} fq_gran;

/* fq_qparams.zero_point value that selects the general (asymmetric) form of
 * Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) (FRM-PTQ page, 初步介绍) with the
 * min-max choice of s and z, per row (gran FQ_DYNAMIC_ROW), b = 3 or 4:
 *   lo = min(0, min v), hi = max(0, max v)   (the range always contains 0)
 *   s  = ((hi - lo) * alpha) / (2^b - 1)      float32, each step rounded
 *   z  = clamp(round(-lo / s), 0, 2^b - 1)    IEEE division, half to even; z = 0 when s = 0
 *   u  = clamp(round(v / s) + z, 0, 2^b - 1)  u = z when s = 0
 * Codes are stored as the signed nibble q = u - 2^(b-1) (in [-4, 3] for
 * b = 3), two per byte as usual.  The scale output is then a block of
 * 3 R 32-bit words: float32 s[R], int32 o[R] = 2^(b-1) - z, int32 S[R] =
 * sum over k of q[r][k]; the GEMM needs o and S to form
 * sum_k (u_x - z_x)(u_w - z_w) = sum q_x q_w + o_w S_x + o_x S_w + K o_x o_w. */
#define FQ_ZERO_POINT_MINMAX (-1)

/* Parameters of Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) (FRM-PTQ page, 初步介绍)
 * and the clip ratio alpha of s = max|v| * alpha / 7 (FlatQuant notes,
 * 可学习裁剪阈值).  Host memory, read during the call only. */
typedef struct {
  int bits;         /* b: 4 (symmetric), or 3 and 4 with FQ_ZERO_POINT_MINMAX */
  int zero_point;   /* z: 2^(b-1) = 8 (the symmetric quantizer) or FQ_ZERO_POINT_MINMAX */
  fq_gran gran;     /* scale extent */
  int group_size;   /* 128 when gran == FQ_DYNAMIC_GROUP, ignored otherwise */
  float alpha;      /* clip ratio in (0, 1]; unused for FQ_STATIC_CHANNEL */
} fq_qparams;

/* Kronecker-factored transform P = P1 (x) P2 and channel scale c (FlatQuant
 * notes, Kronecker 分解 and 逐通道缩放).  Host struct; the matrix pointers are
 * device float32, row-major.  For activations P1 [n1,n1], P2 [n2,n2] are the
 * factors and each row is mapped to c * x followed by P1^T Xbar P2 on its
 * row-major n1 x n2 reshape Xbar.  For weights the caller passes the
 * INVERSES P1^-1, P2^-1 and each weight row w (a column of W^T) is mapped to
 * w / c followed by P1^-1 Wbar (P2^-1)^T.  P1 == NULL and P2 == NULL: no
 * transform (n1, n2 ignored); P1 == NULL with P2 given: P1 = I (the n1 rows
 * of the reshape are transformed on their own, as FlatQuant's per-head P_h
 * and P_v act on the heads of a token); c == NULL means c = 1. */
typedef struct {
  int n1, n2;
  const float* P1;
  const float* P2;
  const float* c;   /* [K] */
} fq_transform;

/* Offline weight quantization (FlatQuant notes, Kronecker 分解: Q(P1^-1 W P2^-T);
 * MergeQuant 核心思路: quantization step migration).
 * W      fp16 [N, K]: weights, one row per output channel.
 * qp     gran FQ_DYNAMIC_ROW (s_w float32 [N]; with FQ_ZERO_POINT_MINMAX the 3 N-word
 *        scale block) or FQ_DYNAMIC_GROUP (s_w fp16 [K/128][N]); alpha = alpha_w.
 * inv    NULL or the inverse transform (P1^-1, P2^-1, c): see fq_transform.
 * qsm_scale NULL or float32 [K]: static activation scales s_k folded into the
 *        weights, w'[n,k] = v[n,k] * s_k in float32 after the transform, so
 *        that the GEMM epilogue needs s_w' only.
 * Wq     uint8 [N, K/2] packed codes (out).  s_w: scales (out).
 * Order per row: /c, inverse transform, x s_k, scale, round, pack. */
fq_status fq_quant_weight(const uint16_t* W, int N, int K, const fq_qparams* qp,
                          const fq_transform* inv, const float* qsm_scale,
                          uint8_t* Wq, void* s_w, void* stream);

/* Online activation quantization (FlatQuant notes, 高效 Kernel 设计: the
 * transform and the quantization fused, intermediates kept on chip).
 * X      fp16 [M, K] token rows.
 * qp     FQ_DYNAMIC_ROW: s_x float32 [M] (FQ_ZERO_POINT_MINMAX: the 3 M-word scale
 *        block);  FQ_DYNAMIC_GROUP: s_x fp16 [K/128][M];
 *        FQ_STATIC_CHANNEL: static_scale float32 [K] is used and s_x is not written
 *        (may be NULL); FQ_STATIC_RESIDUAL: static_scale float32 [K] is used on
 *        x / S_n and s_x receives S_n float32 [M] (S_n = 0, codes 0 for a token of
 *        zeros); alpha = alpha_a.
 * t      NULL or the transform (P1, P2, c).  P1 and P2 are parameters: the
 *        kernel may read them while the kernels enqueued just before it on
 *        the stream are still finishing (programmatic dependent launch), so
 *        they must not be written by such work (no call of this library
 *        writes them).  X, c and the scales are read only after the earlier
 *        work on the stream has completed.
 * Xq     uint8 [M, K/2] packed codes (out). */
fq_status fq_quant_act(const uint16_t* X, int M, int K, const fq_qparams* qp,
                       const fq_transform* t, const float* static_scale,
                       uint8_t* Xq, void* s_x, void* stream);

/* INT4 key or value cache with FlatQuant's per-head transform (FlatQuant
 * notes, Transformer 集成: P_h for the key cache, P_v for the value cache,
 * one head_dim x head_dim matrix applied to every head, not decomposed).
 * KV fp16 [T, H * 128] (T tokens of H heads of 128, 16-byte aligned);
 * P_h float32 [128, 128] (device, row-major); alpha the clip ratio in (0, 1].
 * Each head vector v = x_h P_h is quantized with its own scale
 * s = fp16((max |v| alpha) / 7): Q uint8 [T, H * 64] packed codes (16-byte
 * aligned), scales fp16 [T, H] (out).  The same transform, exactness and
 * codes as fq_quant_act with P1 = I_H, P2 = P_h and FQ_DYNAMIC_GROUP; when
 * T * H is a multiple of 64, 64 head vectors (of any tokens) share one
 * kernel item, so small head counts keep the kernel's tiles full.
 * H in [1, 128].  Enqueues one kernel; allocates nothing. */
fq_status fq_quant_kv(const uint16_t* KV, int T, int H, const float* P_h, float alpha, uint8_t* Q,
                      uint16_t* scales, void* stream);

/* fq_quant_act that also writes xhat float32 [M, K], the transformed values
 * that were quantized (for checking the transform on its own). */
fq_status fq_quant_act_debug(const uint16_t* X, int M, int K, const fq_qparams* qp,
                             const fq_transform* t, const float* static_scale,
                             uint8_t* Xq, void* s_x, float* xhat, void* stream);

/* Leading bytes of every workspace that the library reserves for counters
 * (see fq_w4a4_gemm and fq_linear). */
#define FQ_WORKSPACE_SYNC_BYTES 16384

/* INT4 x INT4 GEMM with exact integer accumulation and fp16 dequantization
 * (FlatQuant notes, 核心思想: Y ~ Q(XP) Q(P^-1 W^T)).
 * Xq uint8 [M, K/2], Wq uint8 [N, K/2] packed codes; Y fp16 [M, N] (out):
 *   FQ_DYNAMIC_ROW:    y = fp16((float(acc) * s_x[m]) * s_w[n]), s_x float32 [M], s_w float32 [N]
 *   FQ_STATIC_CHANNEL: y = fp16(float(acc) * s_w[n]), s_x unused (may be NULL)
 *   FQ_DYNAMIC_GROUP:  y = fp16(sum_g float(acc_g) * s_x[g][m] * s_w[g][n]), the sum in
 *                      float32, acc_g the exact product over k in [128g, 128g+128);
 *                      s_x fp16 [K/128][M], s_w fp16 [K/128][N].
 *   FQ_DYNAMIC_ROW_ZP: y = fp16((float(a) * s_x[m]) * s_w[n]) with the exact
 *                      a = sum_k (u_x - z_x)(u_w - z_w); s_x, s_w the 3 M- and 3 N-word
 *                      scale blocks of FQ_ZERO_POINT_MINMAX.  Runs as the exact int32
 *                      product into the workspace, then a zero-point epilogue.
 * workspace / ws_bytes: device scratch of at least fq_gemm_workspace_size()
 *   bytes, 256-byte aligned (may be NULL when that size is 0).  Its first
 *   FQ_WORKSPACE_SYNC_BYTES (when the size is nonzero) hold the decode
 *   kernels' counters: they must be zero before the first call on a
 *   workspace, and every call that returns FQ_OK leaves them as the next
 *   call needs them (all zero but for the 32-bit word at byte 4, a barrier
 *   generation number that may hold any value); after a call whose kernels
 *   recorded FQ_ERR_TIMEOUT, zero them again.  The rest of the workspace may
 *   hold anything on entry. */
fq_status fq_w4a4_gemm(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w,
                       int M, int N, int K, fq_gran gran, uint16_t* Y,
                       void* workspace, size_t ws_bytes, void* stream);

/* fq_w4a4_gemm for callers that cannot allocate device memory or provide
 * scratch (a plugin inside a runtime that owns all device memory, a serving
 * loop that forbids allocation after start-up).  The pages have no
 * counterpart of this call; it exists for those callers only.
 * Same arguments and results as fq_w4a4_gemm without the workspace: the
 * split-K partial sums use a static 32 MiB device buffer inside libfq.so,
 * which every GPU that loads the library holds until the process exits.
 * - Sizes whose split-K scratch (fq_gemm_workspace_size) exceeds 32 MiB are
 *   rejected with FQ_ERR_INVALID; the call enqueues nothing then (on a
 *   148-SM B200 no size needs more than 20 MiB: the scratch grows with M and
 *   the number of CTAs, not with N).
 * - The first call on a device that needs the buffer looks up its device
 *   address (cudaGetSymbolAddress) with that device current; make that
 *   first call before any stream capture.
 * - All calls share the one buffer: calls that may overlap on the GPU (on
 *   different streams, or from several threads) race and give wrong
 *   results; serialize them on one stream.  The buffer's counters start
 *   at zero and every call leaves them zero; its partial sums are written
 *   before they are read, so the previous call's contents do no harm.
 * - Calls no allocating routine (no cudaMalloc/cudaFree). */
fq_status fq_w4a4_gemm_noalloc(const uint8_t* Xq, const void* s_x, const uint8_t* Wq, const void* s_w,
                               int M, int N, int K, fq_gran gran, uint16_t* Y, void* stream);

/* The exact integer accumulators acc[m][n] = sum_k qx[m,k] qw[n,k] as int32
 * [M, N] (out), for checking the GEMM's integer part on its own. */
fq_status fq_w4a4_gemm_s32(const uint8_t* Xq, const uint8_t* Wq, int M, int N, int K,
                           int32_t* acc, void* stream);

/* The linear layer: fq_quant_act into the workspace, then fq_w4a4_gemm, on
 * one stream.  Arguments as in those two calls; Wq/s_w come from
 * fq_quant_weight with the matching inverse transform (and, for
 * FQ_STATIC_CHANNEL and FQ_STATIC_RESIDUAL, the same static scales folded
 * in; for FQ_ZERO_POINT_MINMAX, the weights' min-max scale block).
 * workspace: fq_linear_workspace_size() bytes,
 * 256-byte aligned (the GEMM's scratch with its counter block first, then the
 * packed activations and their scales; pass FQ_DYNAMIC_ROW_ZP there for the
 * min-max quantizer); its first FQ_WORKSPACE_SYNC_BYTES follow the rule of
 * fq_w4a4_gemm's workspace. */
fq_status fq_linear(const uint16_t* X, int M, int K, const fq_qparams* act_qp,
                    const fq_transform* t, const float* static_scale,
                    const uint8_t* Wq, const void* s_w, int N, uint16_t* Y,
                    void* workspace, size_t ws_bytes, void* stream);

/* Ternary-weight linear layer (PT2-LLM page, 非对称三值量化器 ATQ):
 * Y = X W^T with W^ = alpha T + mu per row and block of 128 columns, T in
 * {-1, 0, +1}, fp16 activations (weight-only ternarization).
 * X fp16 [M, K] (16-byte aligned); Tq uint8 [N, K/4]: 2 bits per weight,
 * low bits first, 00 = 0, 01 = +1, 11 = -1 (as fq_ternary_pack writes it;
 * 16-byte aligned); alpha, mu float32 [N, K/128] row-major; Y fp16 [M, N] (out).
 * K a multiple of 128 in [128, 65536]; M, N >= 1.
 * Arithmetic: per token, row and block, s = sum x t and S = sum x in
 * float32, y = fp16(sum over blocks of alpha s + mu S) accumulated in float32
 * (the summation order is the kernel's; not bit-reproducible against another
 * order, but the same on every run).  For M <= 16 and K <= 32768 the partial
 * products of weight pairs come from per-token tables of the 16 possible pair
 * sums (each the float32 rounding of the exact sum), one launch of clusters
 * of ceil(K / 4096) CTAs reads the weights from HBM once; otherwise tokens
 * are processed 8 at a time and M > 8 streams the weights ceil(M / 8) times.
 * Enqueues one kernel; allocates nothing. */
fq_status fq_ternary_linear(const uint16_t* X, int M, int K, const uint8_t* Tq, const float* alpha,
                            const float* mu, int N, uint16_t* Y, void* stream);

/* Packs int8 T [N, K] (16-byte aligned, K a multiple of 16) into Tq uint8
 * [N, K/4] (4-byte aligned): 1 -> 01, -1 -> 11, every other value -> 00. */
fq_status fq_ternary_pack(const int8_t* T, int N, int K, uint8_t* Tq, void* stream);

/* fq_linear as ONE kernel launch, for decode (M <= 64) with FQ_STATIC_CHANNEL,
 * no Kronecker factors (c allowed) and 16-byte aligned static_scale and c
 * (MergeQuant's setting): the decode GEMM quantizes the tokens itself, with
 * the same codes as fq_quant_act, before a grid-wide barrier, so the launch
 * is cooperative and runs one CTA per SM.  Same arguments, workspace and
 * results as fq_linear (bit-identical outputs); FQ_ERR_UNSUPPORTED where
 * the shape or granularity does not qualify or a cooperative launch is not
 * available.  On B200 the two launches of fq_linear are faster for every
 * decode shape measured (the single launch keeps half the CTAs resident);
 * this call is for callers that need one launch per layer. */
fq_status fq_linear_fused(const uint16_t* X, int M, int K, const fq_qparams* act_qp,
                          const fq_transform* t, const float* static_scale,
                          const uint8_t* Wq, const void* s_w, int N, uint16_t* Y,
                          void* workspace, size_t ws_bytes, void* stream);

/* Scratch sizes in bytes (0 when none is needed).  gran as in the calls. */
size_t fq_gemm_workspace_size(int M, int N, int K, fq_gran gran);
size_t fq_linear_workspace_size(int M, int N, int K, fq_gran gran);

/* Static text for a status. */
const char* fq_status_string(fq_status s);

/* Message describing the calling thread's last non-FQ_OK status ("" if none). */
const char* fq_last_error(void);

/* Synchronizes `stream`, then reads and clears the current device's timeout
 * word: FQ_ERR_TIMEOUT if a kernel's bounded wait gave up since the last
 * check, FQ_ERR_CUDA if the synchronization failed, FQ_OK otherwise. */
fq_status fq_check_device_error(void* stream);

/* Test hook for the timeout path: one CTA waits on a barrier that nothing
 * arrives at, gives up after `limit_us` microseconds (1..100000) and records
 * FQ_ERR_TIMEOUT as every kernel of the library does; the context stays usable. */
fq_status fq_debug_wait_timeout(unsigned limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FQ_H_ */
