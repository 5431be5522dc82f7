"""The C ABI on the host: libfq.so loads, exports every entry point that
include/fq.h declares, and rejects bad arguments before launching anything
(these calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

from int4_linear_b200 import fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(fq.LIB_PATH):
        from int4_linear_b200 import build
        build.build()
    return fq.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["fq_quant_weight", "fq_quant_act", "fq_w4a4_gemm", "fq_linear"]:
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(5):
        assert L.fq_status_string(s)
    assert L.fq_status_string(99) == b"unknown status"


def _qp(**kw):
    return fq.qparams(**kw)


# Fake, 256-byte-aligned device addresses: every case below fails validation
# before any CUDA call, so nothing is dereferenced.
A = 1 << 20


@pytest.mark.parametrize("kw,status", [
    (dict(bits=3), fq.FQ_ERR_UNSUPPORTED),            # symmetric b = 3: not provided
    (dict(zero_point=0), fq.FQ_ERR_UNSUPPORTED),
    (dict(bits=5, zero_point=fq.ZERO_POINT_MINMAX), fq.FQ_ERR_UNSUPPORTED),
    (dict(bits=2, zero_point=fq.ZERO_POINT_MINMAX), fq.FQ_ERR_UNSUPPORTED),
    (dict(gran=fq.GROUP, zero_point=fq.ZERO_POINT_MINMAX), fq.FQ_ERR_UNSUPPORTED),
    (dict(gran=fq.STATIC, zero_point=fq.ZERO_POINT_MINMAX), fq.FQ_ERR_UNSUPPORTED),
    (dict(gran=fq.GROUP, group_size=64), fq.FQ_ERR_UNSUPPORTED),
    (dict(alpha=0.0), fq.FQ_ERR_INVALID),
    (dict(alpha=1.5), fq.FQ_ERR_INVALID),
])
def test_quant_act_rejects_qparams(L, kw, status):
    qp = _qp(**kw)
    st = L.fq_quant_act(A, 4, 256, ctypes.byref(qp), None, None, A, A, None)
    assert st == status
    assert L.fq_last_error()


@pytest.mark.parametrize("m,k,x,xq,msg", [
    (4, 100, A, A, b"K"),
    (4, 128 * 300, A, A, b"K"),
    (0, 256, A, A, b"rows"),
    (4, 256, None, A, b"NULL"),
    (4, 256, A + 8, A, b"aligned"),
])
def test_quant_act_rejects_sizes(L, m, k, x, xq, msg):
    qp = _qp()
    st = L.fq_quant_act(x, m, k, ctypes.byref(qp), None, None, xq, A, None)
    assert st == fq.FQ_ERR_INVALID
    assert msg in L.fq_last_error()


def test_transform_shape_must_match_k(L):
    qp = _qp()
    t = fq._Transform(8, 16, A, A, None)  # 8 * 16 != 256
    st = L.fq_quant_act(A, 4, 256, ctypes.byref(qp), ctypes.byref(t), None, A, A, None)
    assert st == fq.FQ_ERR_INVALID and b"n1 * n2" in L.fq_last_error()


def test_static_needs_scales(L):
    qp = _qp(gran=fq.STATIC)
    st = L.fq_quant_act(A, 4, 256, ctypes.byref(qp), None, None, A, None, None)
    assert st == fq.FQ_ERR_INVALID
    st = L.fq_quant_weight(A, 4, 256, ctypes.byref(qp), None, None, A, A, None)
    assert st == fq.FQ_ERR_UNSUPPORTED  # weights have no static granularity


def test_residual_scaling_arguments(L):
    """FQ_STATIC_RESIDUAL needs the static scales and the S_n output, takes no
    transform and no c, and is an activation granularity only (the GEMM runs
    per token with s_x = S_n)."""
    qp = _qp(gran=fq.STATIC_RESIDUAL)
    assert L.fq_quant_act(A, 4, 256, ctypes.byref(qp), None, None, A, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_quant_act(A, 4, 256, ctypes.byref(qp), None, A, A, None, None) == fq.FQ_ERR_INVALID
    t = fq._Transform(16, 16, A, A, None)
    st = L.fq_quant_act(A, 4, 256, ctypes.byref(qp), ctypes.byref(t), A, A, A, None)
    assert st == fq.FQ_ERR_UNSUPPORTED and b"RESIDUAL" in L.fq_last_error()
    t = fq._Transform(0, 0, None, None, A)
    assert L.fq_quant_act(A, 4, 256, ctypes.byref(qp), ctypes.byref(t), A, A, A, None) == fq.FQ_ERR_UNSUPPORTED
    assert L.fq_quant_weight(A, 4, 256, ctypes.byref(qp), None, None, A, A, None) == fq.FQ_ERR_UNSUPPORTED
    assert L.fq_w4a4_gemm(A, A, A, A, 4, 256, 256, fq.STATIC_RESIDUAL, A, None, 0, None) == fq.FQ_ERR_UNSUPPORTED
    assert L.fq_linear_workspace_size(16, 256, 256, fq.STATIC_RESIDUAL) == L.fq_linear_workspace_size(16, 256, 256, fq.ROW)


@pytest.mark.parametrize("m,n,k", [(0, 256, 256), (4, 12, 256), (4, 256, 200), (4, 256, 131072)])
def test_gemm_rejects_sizes(L, m, n, k):
    st = L.fq_w4a4_gemm(A, A, A, A, m, n, k, fq.ROW, A, None, 0, None)
    assert st == fq.FQ_ERR_INVALID


def test_gemm_rejects_misaligned(L):
    st = L.fq_w4a4_gemm(A + 4, A, A, A, 4, 256, 256, fq.ROW, A, None, 0, None)
    assert st == fq.FQ_ERR_INVALID and b"aligned" in L.fq_last_error()
    st = L.fq_w4a4_gemm(A, A, A, A, 4, 256, 256, 7, A, None, 0, None)
    assert st == fq.FQ_ERR_UNSUPPORTED


def test_linear_needs_workspace(L):
    qp = _qp()
    need = L.fq_linear_workspace_size(16, 256, 256, fq.ROW)
    assert need >= 16 * 128 + 16 * 4
    st = L.fq_linear(A, 16, 256, ctypes.byref(qp), None, None, A, A, 256, A, A, need - 1, None)
    assert st == fq.FQ_ERR_INVALID and b"workspace" in L.fq_last_error()


def test_workspace_sizes(L):
    """Prefill needs no GEMM scratch.  Decode with few output tiles splits K
    over one wave of 2 x 148 CTAs (the SM count assumed without a GPU): the
    counter block plus two slots of M x 128 int32 per CTA, whatever N is.
    The fused static decode needs the counter block even without split tiles,
    and the linear layer always reserves it first."""
    assert L.fq_gemm_workspace_size(2048, 4096, 4096, fq.ROW) == 0
    assert L.fq_gemm_workspace_size(4096, 8192, 8192, fq.GROUP) == 0
    slots = 2 * 296 * 8 * 128 * 4
    assert L.fq_gemm_workspace_size(8, 8192, 28672, fq.ROW) == fq.SYNC_BYTES + slots
    assert L.fq_gemm_workspace_size(8, 139264, 8192, fq.ROW) == fq.SYNC_BYTES + slots
    ws = L.fq_linear_workspace_size(8, 8192, 28672, fq.STATIC)
    assert ws >= fq.SYNC_BYTES + slots + 8 * 28672 // 2
    assert L.fq_linear_workspace_size(2048, 4096, 4096, fq.ROW) >= fq.SYNC_BYTES + 2048 * 2048 + 2048 * 4
    # 64 tokens: the largest decode scratch stays within the no-alloc entry's 32 MiB
    assert L.fq_gemm_workspace_size(64, 8192, 28672, fq.ROW) <= 32 << 20


def test_debug_timeout_rejects_limits(L):
    assert L.fq_debug_wait_timeout(0, None) == fq.FQ_ERR_INVALID
    assert L.fq_debug_wait_timeout(1000000, None) == fq.FQ_ERR_INVALID


def test_zero_point_gemm_needs_its_workspace(L):
    """The min-max quantizer's GEMM keeps the exact int32 products in the
    caller's workspace: M * N * 4 bytes, and refuses to run without them."""
    assert L.fq_gemm_workspace_size(8, 256, 256, fq.ROW_ZP) == fq.SYNC_BYTES + 8 * 256 * 4
    st = L.fq_w4a4_gemm(A, A, A, A, 8, 256, 256, fq.ROW_ZP, A, None, 0, None)
    assert st == fq.FQ_ERR_INVALID and b"workspace" in L.fq_last_error()
    ws = L.fq_linear_workspace_size(8, 256, 256, fq.ROW_ZP)
    assert ws >= 8 * 128 + 3 * 8 * 4 + 8 * 256 * 4


def test_ternary_rejects_arguments(L):
    """Sizes, NULLs and alignment are checked before any launch."""
    assert L.fq_ternary_linear(A, 1, 100, A, A, A, 8, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_ternary_linear(A, 0, 128, A, A, A, 8, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_ternary_linear(A, 1, 128, None, A, A, 8, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_ternary_linear(A + 8, 1, 128, A, A, A, 8, A, None) == fq.FQ_ERR_INVALID
    assert b"aligned" in L.fq_last_error()
    assert L.fq_ternary_pack(A, 4, 24, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_ternary_pack(A + 4, 4, 32, A, None) == fq.FQ_ERR_INVALID


def test_fused_linear_rejects_what_it_does_not_cover(L):
    """The one-launch decode linear takes static per-channel scales only."""
    qp = _qp()  # dynamic per-token
    need = L.fq_linear_workspace_size(8, 256, 256, fq.ROW)
    st = L.fq_linear_fused(A, 8, 256, ctypes.byref(qp), None, None, A, A, 256, A, A, need, None)
    assert st == fq.FQ_ERR_UNSUPPORTED and b"static" in L.fq_last_error()


def test_quant_kv_rejects_arguments(L):
    """fq_quant_kv: T >= 1, 1 <= H <= 128, P_h and the scale output non-NULL, the
    same alignment rules as fq_quant_act (checked before any launch)."""
    assert L.fq_quant_kv(A, 0, 8, A, 1.0, A, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_quant_kv(A, 4, 129, A, 1.0, A, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_quant_kv(A, 4, 8, None, 1.0, A, A, None) == fq.FQ_ERR_INVALID
    assert L.fq_quant_kv(A, 4, 8, A, 1.0, A, None, None) == fq.FQ_ERR_INVALID
    assert L.fq_quant_kv(A + 8, 8, 8, A, 1.0, A, A, None) == fq.FQ_ERR_INVALID  # X not 16-byte aligned
    assert L.fq_quant_kv(A, 8, 8, A, 0.0, A, A, None) == fq.FQ_ERR_INVALID      # alpha out of (0, 1]


@pytest.mark.parametrize("m,n,k", [(1, 8192, 28672), (8, 57344, 8192), (64, 4096, 4096), (2048, 28672, 4096),
                                   (4096, 10240, 8192)])
def test_linear_workspace_holds_its_parts(L, m, n, k):
    """fq_linear's workspace: the GEMM's part (at least the 16 KB counter block,
    first), then the packed activations and their scales, each 256-byte aligned."""
    up = lambda v: (v + 255) // 256 * 256
    for gran, scale_bytes in ((fq.ROW, 4 * m), (fq.STATIC, 0), (fq.GROUP, 2 * m * (k // 128)),
                              (fq.STATIC_RESIDUAL, 4 * m), (fq.ROW_ZP, 12 * m)):
        gemm = max(fq.SYNC_BYTES, L.fq_gemm_workspace_size(m, n, k, gran))
        need = up(gemm) + up(m * k // 2) + up(scale_bytes)
        assert L.fq_linear_workspace_size(m, n, k, gran) == need, (gran, m, n, k)
