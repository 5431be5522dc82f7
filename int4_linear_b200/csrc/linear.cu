// The W4A4 linear layer: online activation quantization into the caller's
// workspace, then the INT4 x INT4 GEMM, on one stream (FlatQuant notes,
// 核心思想: Y ~ Q(XP) Q(P^-1 W^T)).  fq_linear_fused runs decode with static
// per-channel scales and no Kronecker transform (MergeQuant's setting) as one
// launch: the decode GEMM quantizes the tokens itself.
#include <algorithm>

#include "fq_host.h"

namespace fq {
size_t gemm_workspace_bytes(int M, int N, int K, fq_gran gran);
size_t sync_block_bytes();
fq_status check_act_args(const uint16_t* X, int M, int K, const fq_qparams* qp, const fq_transform* t,
                         const float* static_scale, uint8_t* Xq, void* s_x);
fq_status decode_linear_fused(const uint16_t* X, const float* sst, const float* cst, uint8_t* Xq, const uint8_t* Wq,
                              const void* s_w, int M, int N, int K, uint16_t* Y, void* ws, size_t ws_bytes,
                              cudaStream_t stream);

namespace {
constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t act_scale_bytes(int M, int K, fq_gran gran) {
  if (gran == FQ_DYNAMIC_ROW || gran == FQ_STATIC_RESIDUAL) return size_t(M) * sizeof(float);
  if (gran == FQ_DYNAMIC_ROW_ZP) return 3 * size_t(M) * sizeof(float);  // s, o = 2^(b-1) - z, code sums
  if (gran == FQ_DYNAMIC_GROUP) return size_t(K / kGroup) * M * 2;
  return 0;
}
}  // namespace

// Workspace layout: the GEMM's part first (its synchronization block at
// offset 0 for every shape, so that no call writes there but to leave it
// zero), then the packed activations, then their scales.
size_t linear_gemm_part(int M, int N, int K, fq_gran gran) {
  return up(std::max(sync_block_bytes(), gemm_workspace_bytes(M, N, K, gran)));
}

size_t linear_workspace_bytes(int M, int N, int K, fq_gran gran) {
  if (M < 1 || K < kGroup || K % kGroup) return 0;
  return linear_gemm_part(M, N, K, gran) + up(size_t(M) * (K / 2)) + up(act_scale_bytes(M, K, gran));
}

}  // namespace fq

extern "C" {

size_t fq_linear_workspace_size(int M, int N, int K, fq_gran gran) {
  return fq::linear_workspace_bytes(M, N, K, gran);
}

namespace {
// fused: the one-launch decode path (FQ_ERR_UNSUPPORTED where it does not apply)
fq_status linear_impl(const uint16_t* X, int M, int K, const fq_qparams* act_qp, const fq_transform* t,
                      const float* static_scale, const uint8_t* Wq, const void* s_w, int N, uint16_t* Y,
                      void* workspace, size_t ws_bytes, void* stream, bool fused) {
  fq::clear_error();
  if (!act_qp) return fq::fail(FQ_ERR_INVALID, "act_qp is NULL");
  if (M < 1 || K < fq::kGroup || K % fq::kGroup || N < 8 || N % 8)
    return fq::fail(FQ_ERR_INVALID, "sizes M = %d, N = %d, K = %d out of range", M, N, K);
  // the min-max quantizer's activations go with the zero-point GEMM
  const fq_gran gran = act_qp->zero_point == FQ_ZERO_POINT_MINMAX ? FQ_DYNAMIC_ROW_ZP : act_qp->gran;
  const size_t need = fq::linear_workspace_bytes(M, N, K, gran);
  if (!workspace || ws_bytes < need || !fq::aligned(workspace, 256))
    return fq::fail(FQ_ERR_INVALID, "workspace of %zu bytes (256-byte aligned) required, got %zu", need, ws_bytes);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  void* gws = base;
  const size_t gws_bytes = fq::linear_gemm_part(M, N, K, gran);
  size_t off = gws_bytes;
  uint8_t* xq = base + off;
  off += fq::up(size_t(M) * (K / 2));
  void* sx = act_qp->gran == FQ_STATIC_CHANNEL ? nullptr : static_cast<void*>(base + off);
  fq_status st;
  if (fused) {
    if (!(gran == FQ_STATIC_CHANNEL && act_qp->zero_point == 8 && (!t || !t->P1) && fq::aligned(static_scale, 16) &&
          (!t || !t->c || fq::aligned(t->c, 16))))
      return fq::fail(FQ_ERR_UNSUPPORTED,
                      "the one-launch path takes static per-channel scales (16-byte aligned) and no Kronecker factors");
    st = fq::check_act_args(X, M, K, act_qp, t, static_scale, xq, sx);
    if (st != FQ_OK) return st;
    st = fq::decode_linear_fused(X, static_scale, t ? t->c : nullptr, xq, Wq, s_w, M, N, K, Y, gws, gws_bytes,
                                 static_cast<cudaStream_t>(stream));
    if (st == FQ_ERR_UNSUPPORTED && !fq_last_error()[0])
      return fq::fail(FQ_ERR_UNSUPPORTED,
                      "M = %d is not a decode size (M <= 64), or a cooperative launch is not available", M);
    return st;
  }
  st = fq_quant_act(X, M, K, act_qp, t, static_scale, xq, sx, stream);
  if (st != FQ_OK) return st;
  // the residual scaling leaves through the per-token epilogue: s_x = S_n
  const fq_gran ggran = gran == FQ_STATIC_RESIDUAL ? FQ_DYNAMIC_ROW : gran;
  return fq_w4a4_gemm(xq, sx, Wq, s_w, M, N, K, ggran, Y, gws, gws_bytes, stream);
}
}  // namespace

fq_status fq_linear(const uint16_t* X, int M, int K, const fq_qparams* act_qp, const fq_transform* t,
                    const float* static_scale, const uint8_t* Wq, const void* s_w, int N, uint16_t* Y,
                    void* workspace, size_t ws_bytes, void* stream) {
  return linear_impl(X, M, K, act_qp, t, static_scale, Wq, s_w, N, Y, workspace, ws_bytes, stream, false);
}

fq_status fq_linear_fused(const uint16_t* X, int M, int K, const fq_qparams* act_qp, const fq_transform* t,
                          const float* static_scale, const uint8_t* Wq, const void* s_w, int N, uint16_t* Y,
                          void* workspace, size_t ws_bytes, void* stream) {
  return linear_impl(X, M, K, act_qp, t, static_scale, Wq, s_w, N, Y, workspace, ws_bytes, stream, true);
}

}  // extern "C"
