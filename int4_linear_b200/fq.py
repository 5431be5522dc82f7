"""Python binding of libfq.so (C ABI in include/fq.h).

Argument marshalling only: every function checks tensor dtypes/devices,
allocates outputs through PyTorch when the caller gives none, and calls the
C entry point of the same name on the current (or given) CUDA stream.  All
arithmetic runs in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

ROW, GROUP, STATIC, ROW_ZP, STATIC_RESIDUAL = 0, 1, 2, 3, 4  # fq_gran
SYNC_BYTES = 16384  # FQ_WORKSPACE_SYNC_BYTES: leading workspace bytes kept zero between calls
GROUP_SIZE = 128
ZERO_POINT_MINMAX = -1                   # fq_qparams.zero_point: per-row min-max (asymmetric) quantizer

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfq.so")

FQ_OK, FQ_ERR_INVALID, FQ_ERR_UNSUPPORTED, FQ_ERR_CUDA, FQ_ERR_TIMEOUT = range(5)


class FqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class QParams(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("zero_point", ctypes.c_int), ("gran", ctypes.c_int),
                ("group_size", ctypes.c_int), ("alpha", ctypes.c_float)]


class _Transform(ctypes.Structure):
    _fields_ = [("n1", ctypes.c_int), ("n2", ctypes.c_int), ("P1", ctypes.c_void_p),
                ("P2", ctypes.c_void_p), ("c", ctypes.c_void_p)]


@dataclass
class Transform:
    """Kronecker factors (device float32) and channel scale.  For fq_quant_weight
    pass the inverses P1^-1, P2^-1 (and the same c)."""
    P1: torch.Tensor | None = None
    P2: torch.Tensor | None = None
    c: torch.Tensor | None = None

    n1: int = 0  # with P1 None and P2 given: the number of rows of the reshape (P1 = I)

    def as_c(self) -> _Transform:
        t = _Transform()
        if self.P1 is not None or self.P2 is not None:
            _check(self.P1, torch.float32, "P1")
            _check(self.P2, torch.float32, "P2")
            t.n1 = self.P1.shape[0] if self.P1 is not None else self.n1
            t.n2 = self.P2.shape[0]
            t.P1 = self.P1.data_ptr() if self.P1 is not None else None
            t.P2 = self.P2.data_ptr()
        if self.c is not None:
            _check(self.c, torch.float32, "c")
            t.c = self.c.data_ptr()
        return t


def qparams(gran: int = ROW, alpha: float = 1.0, bits: int = 4, zero_point: int = 8,
            group_size: int = GROUP_SIZE) -> QParams:
    return QParams(bits, zero_point, gran, group_size, alpha)


_lib = None


def lib():
    """Load libfq.so (raises if it was not built: there is no other code path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FqError(FQ_ERR_CUDA, f"{LIB_PATH} is missing: build it with python -m int4_linear_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    qp, tp = ctypes.POINTER(QParams), ctypes.POINTER(_Transform)
    sigs = {
        "fq_quant_weight": [vp, i, i, qp, tp, vp, vp, vp, vp],
        "fq_quant_act": [vp, i, i, qp, tp, vp, vp, vp, vp],
        "fq_quant_act_debug": [vp, i, i, qp, tp, vp, vp, vp, vp, vp],
        "fq_w4a4_gemm": [vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp],
        "fq_w4a4_gemm_s32": [vp, vp, i, i, i, vp, vp],
        "fq_w4a4_gemm_noalloc": [vp, vp, vp, vp, i, i, i, i, vp, vp],
        "fq_linear": [vp, i, i, qp, tp, vp, vp, vp, i, vp, vp, sz, vp],
        "fq_linear_fused": [vp, i, i, qp, tp, vp, vp, vp, i, vp, vp, sz, vp],
        "fq_ternary_linear": [vp, i, i, vp, vp, vp, i, vp, vp],
        "fq_quant_kv": [vp, i, i, vp, ctypes.c_float, vp, vp, vp],
        "fq_ternary_pack": [vp, i, i, vp, vp],
        "fq_check_device_error": [vp],
        "fq_debug_wait_timeout": [ctypes.c_uint, vp],
    }
    for name, args in sigs.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    for name in ("fq_gemm_workspace_size", "fq_linear_workspace_size"):
        f = getattr(L, name)
        f.argtypes = [i, i, i, i]
        f.restype = sz
    L.fq_status_string.argtypes = [ctypes.c_int]
    L.fq_status_string.restype = ctypes.c_char_p
    L.fq_last_error.argtypes = []
    L.fq_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _raise(status: int):
    if status != FQ_OK:
        L = lib()
        raise FqError(status, f"{L.fq_status_string(status).decode()}: {L.fq_last_error().decode()}")


def _check(t, dtype, name):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _p(t):
    return None if t is None else t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _scales_out(gran, rows, k, dev, zero_point=8):
    if gran == ROW and zero_point == ZERO_POINT_MINMAX:
        # float32 s[rows], int32 o[rows] = 2^(b-1) - z, int32 code sums[rows]
        return torch.empty(3, rows, dtype=torch.float32, device=dev)
    if gran in (ROW, STATIC_RESIDUAL):
        return torch.empty(rows, dtype=torch.float32, device=dev)
    if gran == GROUP:
        return torch.empty(k // GROUP_SIZE, rows, dtype=torch.float16, device=dev)
    return None


def fq_quant_weight(W, qp: QParams, inv: Transform | None = None, qsm_scale=None,
                    Wq=None, s_w=None, stream=None):
    """Offline weight quantization: returns (Wq uint8 [N, K/2], s_w)."""
    _check(W, torch.float16, "W")
    _check(qsm_scale, torch.float32, "qsm_scale")
    n, k = W.shape
    Wq = torch.empty(n, k // 2, dtype=torch.uint8, device=W.device) if Wq is None else Wq
    s_w = _scales_out(qp.gran, n, k, W.device, qp.zero_point) if s_w is None else s_w
    t = inv.as_c() if inv is not None else None
    st = lib().fq_quant_weight(W.data_ptr(), n, k, ctypes.byref(qp), ctypes.byref(t) if t else None,
                               _p(qsm_scale), Wq.data_ptr(), _p(s_w), _s(stream))
    _raise(st)
    return Wq, s_w


def fq_quant_act(X, qp: QParams, t: Transform | None = None, static_scale=None,
                 Xq=None, s_x=None, stream=None):
    """Online activation quantization: returns (Xq uint8 [M, K/2], s_x or None)."""
    _check(X, torch.float16, "X")
    _check(static_scale, torch.float32, "static_scale")
    m, k = X.shape
    Xq = torch.empty(m, k // 2, dtype=torch.uint8, device=X.device) if Xq is None else Xq
    s_x = _scales_out(qp.gran, m, k, X.device, qp.zero_point) if s_x is None else s_x
    tc = t.as_c() if t is not None else None
    st = lib().fq_quant_act(X.data_ptr(), m, k, ctypes.byref(qp), ctypes.byref(tc) if tc else None,
                            _p(static_scale), Xq.data_ptr(), _p(s_x), _s(stream))
    _raise(st)
    return Xq, s_x


def fq_quant_act_debug(X, qp: QParams, t: Transform | None = None, static_scale=None, stream=None):
    """fq_quant_act that also returns the float32 transformed values: (Xq, s_x, xhat)."""
    _check(X, torch.float16, "X")
    _check(static_scale, torch.float32, "static_scale")
    m, k = X.shape
    Xq = torch.empty(m, k // 2, dtype=torch.uint8, device=X.device)
    s_x = _scales_out(qp.gran, m, k, X.device, qp.zero_point)
    xhat = torch.empty(m, k, dtype=torch.float32, device=X.device)
    tc = t.as_c() if t is not None else None
    st = lib().fq_quant_act_debug(X.data_ptr(), m, k, ctypes.byref(qp), ctypes.byref(tc) if tc else None,
                                  _p(static_scale), Xq.data_ptr(), _p(s_x), xhat.data_ptr(), _s(stream))
    _raise(st)
    return Xq, s_x, xhat


def split_zero_point_block(block):
    """The min-max quantizer's scale block -> (s float32 [R], o int32 [R] =
    2^(b-1) - z, S int32 [R] = the rows' sums of the stored codes)."""
    b = block.reshape(3, -1)
    return b[0], b[1].view(torch.int32), b[2].view(torch.int32)


def fq_gemm_workspace_size(m, n, k, gran) -> int:
    return int(lib().fq_gemm_workspace_size(m, n, k, gran))


def fq_linear_workspace_size(m, n, k, gran) -> int:
    return int(lib().fq_linear_workspace_size(m, n, k, gran))


def _workspace(nbytes, dev, ws):
    if nbytes == 0:
        return None, 0
    if ws is None:
        # zeroed: the library's counters at the start of a workspace must be 0 on first use
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    if ws.numel() < nbytes:
        raise ValueError(f"workspace needs {nbytes} bytes")
    return ws, ws.numel()


def fq_w4a4_gemm(Xq, s_x, Wq, s_w, gran: int, Y=None, workspace=None, stream=None):
    """Y fp16 [M, N] = dequant(Xq Wq^T)."""
    _check(Xq, torch.uint8, "Xq")
    _check(Wq, torch.uint8, "Wq")
    m, k2 = Xq.shape
    n = Wq.shape[0]
    k = 2 * k2
    Y = torch.empty(m, n, dtype=torch.float16, device=Xq.device) if Y is None else Y
    _check(Y, torch.float16, "Y")
    ws, wsb = _workspace(fq_gemm_workspace_size(m, n, k, gran), Xq.device, workspace)
    st = lib().fq_w4a4_gemm(Xq.data_ptr(), _p(s_x), Wq.data_ptr(), _p(s_w), m, n, k, gran, Y.data_ptr(),
                            _p(ws), wsb, _s(stream))
    _raise(st)
    return Y


def fq_w4a4_gemm_noalloc(Xq, s_x, Wq, s_w, gran: int, Y=None, stream=None):
    """fq_w4a4_gemm without a workspace, for callers that cannot allocate device
    memory: the library's static 32 MiB scratch holds the split-K partial sums.
    Calls that overlap on the GPU share that scratch and race; keep them on one
    stream.  (Y is allocated here only when the caller passes none.)"""
    _check(Xq, torch.uint8, "Xq")
    _check(Wq, torch.uint8, "Wq")
    m, k2 = Xq.shape
    n = Wq.shape[0]
    Y = torch.empty(m, n, dtype=torch.float16, device=Xq.device) if Y is None else Y
    _check(Y, torch.float16, "Y")
    st = lib().fq_w4a4_gemm_noalloc(Xq.data_ptr(), _p(s_x), Wq.data_ptr(), _p(s_w), m, n, 2 * k2, gran,
                                    Y.data_ptr(), _s(stream))
    _raise(st)
    return Y


def fq_w4a4_gemm_s32(Xq, Wq, acc=None, stream=None):
    """The exact int32 accumulators [M, N]."""
    _check(Xq, torch.uint8, "Xq")
    _check(Wq, torch.uint8, "Wq")
    m, k2 = Xq.shape
    n = Wq.shape[0]
    acc = torch.empty(m, n, dtype=torch.int32, device=Xq.device) if acc is None else acc
    _check(acc, torch.int32, "acc")
    st = lib().fq_w4a4_gemm_s32(Xq.data_ptr(), Wq.data_ptr(), m, n, 2 * k2, acc.data_ptr(), _s(stream))
    _raise(st)
    return acc


def fq_linear(X, qp: QParams, Wq, s_w, t: Transform | None = None, static_scale=None,
              Y=None, workspace=None, stream=None, fused=False):
    """Y fp16 [M, N] = dequant(Q(X P) Q(P^-1 W^T)), quantization + GEMM on one
    stream (fused=True: fq_linear_fused, one launch at decode sizes)."""
    _check(X, torch.float16, "X")
    _check(Wq, torch.uint8, "Wq")
    _check(static_scale, torch.float32, "static_scale")
    m, k = X.shape
    n = Wq.shape[0]
    Y = torch.empty(m, n, dtype=torch.float16, device=X.device) if Y is None else Y
    _check(Y, torch.float16, "Y")
    gran = ROW_ZP if qp.zero_point == ZERO_POINT_MINMAX else qp.gran
    ws, wsb = _workspace(fq_linear_workspace_size(m, n, k, gran), X.device, workspace)
    tc = t.as_c() if t is not None else None
    fn = lib().fq_linear_fused if fused else lib().fq_linear
    st = fn(X.data_ptr(), m, k, ctypes.byref(qp), ctypes.byref(tc) if tc else None,
                         _p(static_scale), Wq.data_ptr(), _p(s_w), n, Y.data_ptr(), _p(ws), wsb,
                         _s(stream))
    _raise(st)
    return Y


def fq_quant_kv(KV, P_h, alpha: float = 1.0, Q=None, scales=None, stream=None):
    """INT4 key/value cache: KV fp16 [T, H, 128] (or [T, H * 128]) with the
    per-head transform P_h [128, 128] -> (Q uint8 [T, H * 64], scales fp16 [T, H])."""
    _check(KV, torch.float16, "KV")
    _check(P_h, torch.float32, "P_h")
    t = KV.shape[0]
    h = KV[0].numel() // 128
    Q = torch.empty(t, h * 64, dtype=torch.uint8, device=KV.device) if Q is None else Q
    scales = torch.empty(t, h, dtype=torch.float16, device=KV.device) if scales is None else scales
    _raise(lib().fq_quant_kv(KV.data_ptr(), t, h, P_h.data_ptr(), alpha, Q.data_ptr(), scales.data_ptr(),
                             _s(stream)))
    return Q, scales


def fq_ternary_pack(T, Tq=None, stream=None):
    """int8 T [N, K] in {-1, 0, 1} -> packed 2-bit codes uint8 [N, K/4]."""
    _check(T, torch.int8, "T")
    n, k = T.shape
    Tq = torch.empty(n, k // 4, dtype=torch.uint8, device=T.device) if Tq is None else Tq
    _raise(lib().fq_ternary_pack(T.data_ptr(), n, k, Tq.data_ptr(), _s(stream)))
    return Tq


def fq_ternary_linear(X, Tq, alpha, mu, Y=None, stream=None):
    """Y fp16 [M, N] = X (alpha T + mu)^T for packed ternary codes Tq [N, K/4]
    and per-(row, 128-block) alpha, mu float32 [N, K/128]."""
    _check(X, torch.float16, "X")
    _check(Tq, torch.uint8, "Tq")
    _check(alpha, torch.float32, "alpha")
    _check(mu, torch.float32, "mu")
    m, k = X.shape
    n = Tq.shape[0]
    Y = torch.empty(m, n, dtype=torch.float16, device=X.device) if Y is None else Y
    _check(Y, torch.float16, "Y")
    _raise(lib().fq_ternary_linear(X.data_ptr(), m, k, Tq.data_ptr(), alpha.data_ptr(), mu.data_ptr(), n,
                                   Y.data_ptr(), _s(stream)))
    return Y


def fq_check_device_error(stream=None):
    _raise(lib().fq_check_device_error(_s(stream)))


def fq_debug_wait_timeout(limit_us: int, stream=None):
    _raise(lib().fq_debug_wait_timeout(limit_us, _s(stream)))
