"""Per-token residual scaling ahead of static INT4 quantization (FPTQuant
explainer, 伪动态残差缩放) on the GPU, against the oracle's residual_rms and
quant_act_residual.

Every step is exact or one IEEE rounding: the sum of squares is exact and
rounded once to float64 on both sides, then /K, sqrt and float32; the token is
divided by S_n in float32; the static codes round v / s_k.  So S_n, the codes
and (through the oracle's integer GEMM and per-token dequantization) the
linear layer's fp16 outputs are all compared bit-exactly.
"""
import numpy as np
import pytest
import torch

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def _quant(x, s_k):
    qp = fq.qparams(fq.STATIC_RESIDUAL)
    xq, s_n = fq.fq_quant_act(C.dev(x), qp, static_scale=C.dev(s_k))
    fq.fq_check_device_error()
    return C.host(xq), C.host(s_n)


def _check(x, s_k):
    q_ref, sn_ref, _ = O.quant_act_residual(x, s_k)
    xq, s_n = _quant(x, s_k)
    assert np.array_equal(s_n.view(np.uint32), sn_ref.view(np.uint32)), \
        f"S_n differs in {(s_n != sn_ref).sum()} of {len(s_n)} tokens"
    assert np.array_equal(xq, O.pack_int4(q_ref)), \
        f"{(C.unpack(xq) != q_ref).sum()} codes differ"
    return q_ref, sn_ref


@pytest.mark.parametrize("m,k", [(1, 128), (37, 1024), (300, 4096), (16, 8192), (5, 28672)])
def test_residual_quant_exact(m, k):
    d = synth.residual_static(m, k, 8, seed=m + k)
    _check(d["x"], d["static_scale"])


def test_residual_degenerate_tokens():
    """A token of zeros (S_n = 0, codes 0), a token of one fp16 subnormal, a
    token of +-65504 (squares near 2^32 each), and tokens whose float64
    running sums round (one large entry among many small ones)."""
    k = 1024
    g = synth.generator(5)
    x = (g.standard_normal((8, k))).astype(np.float16)
    x[0] = 0
    x[1] = 0
    x[1, 17] = np.float16(2.0 ** -24)
    x[2] = np.where(g.uniform(size=k) < 0.5, 65504.0, -65504.0).astype(np.float16)
    x[3] = np.float16(2.0 ** -12)
    x[3, 0] = np.float16(32768.0)
    x[4] = np.float16(2.0 ** -14) * np.sign(g.standard_normal(k)).astype(np.float16)
    x[4, 999] = np.float16(-40000.0)
    s_k = g.uniform(0.05, 0.5, k).astype(np.float32)
    q_ref, sn_ref = _check(x, s_k)
    assert sn_ref[0] == 0 and not q_ref[0].any()


@pytest.mark.parametrize("m,k,n", [(16, 4096, 4096), (256, 4096, 6144), (1, 8192, 1024)])
def test_residual_linear_exact(m, k, n):
    """The linear layer: static codes of x / S_n times the weights quantized
    with the static scales migrated into them, dequantized per token by S_n.
    fq_linear, and quantization + GEMM as separate calls, both bit-exact."""
    d = synth.residual_static(m, k, n, seed=7)
    s_k = d["static_scale"]
    X = C.dev(d["x"])
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0), None, C.dev(s_k))
    qp = fq.qparams(fq.STATIC_RESIDUAL)
    y_lin = C.host(fq.fq_linear(X, qp, wq, sw, static_scale=C.dev(s_k)))
    xq, s_n = fq.fq_quant_act(X, qp, static_scale=C.dev(s_k))
    ws = torch.zeros(max(fq.fq_gemm_workspace_size(m, n, k, fq.ROW), 256), dtype=torch.uint8, device="cuda")
    y = C.host(fq.fq_w4a4_gemm(xq, s_n, wq, sw, fq.ROW, workspace=ws))
    fq.fq_check_device_error()
    assert np.array_equal(y.view(np.uint16), y_lin.view(np.uint16)), "fq_linear differs from quant + GEMM"
    q_ref, sn_ref, _ = O.quant_act_residual(d["x"], s_k)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    assert np.array_equal(C.host(s_n), sn_ref)
    cols = C.tile_samples(m + n, n)
    qw, sw_ref, _ = O.quant_weight(d["w"][cols], O.ROW, 1.0, qsm_scale=s_k)
    assert np.array_equal(C.host(wq)[cols], O.pack_int4(qw))
    C.check_gemm_decoupled(y[:, cols], q_ref, sn_ref, qw, sw_ref, O.ROW)
