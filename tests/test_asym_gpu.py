"""The general quantizer on the GPU: Q(W) = clamp(round(W/s) + z, 0, 2^b - 1)
with b = 3 or 4 and the per-row min-max scale and zero point (FRM-PTQ page,
初步介绍; W3A3 in its abstract), against the oracle's minmax_params,
quantize_u and gemm_asym.

Without a transform every step is float32 as written or exact integer
arithmetic, so scales, zero points, codes, code sums and fp16 outputs are
compared bit-exactly.  With the Kronecker transform the transformed values
follow the parity rule of the other transform tests (gpu_checks)."""
import numpy as np
import pytest
import torch

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def _x(seed, m, k):
    g = synth.generator(seed)
    cs = np.ones(k)
    cs[g.permutation(k)[: max(1, k // 100)]] = 30.0
    x = synth._draw(g, (m, k), "normal", 1.0, col_scale=cs)
    x[:, :: 7] = np.abs(x[:, :: 7])           # skewed rows: the zero point moves off the middle
    return x


def _gpu_block(block, bits):
    s, o, S = fq.split_zero_point_block(block)
    s, o, S = C.host(s), C.host(o), C.host(S)
    return s, (1 << (bits - 1)) - o, S


def _check_rows(xq, block, v32, bits, alpha):
    """codes u, scales, zero points and code sums of rows v32 (float32)."""
    s_ref, z_ref = O.minmax_params(v32, bits, alpha)
    u_ref = O.quantize_u(v32, s_ref, z_ref, bits)
    s, z, S = _gpu_block(block, bits)
    q = C.unpack(C.host(xq)).astype(np.int64)
    u = q + (1 << (bits - 1))
    assert np.array_equal(s, s_ref), "scales differ"
    assert np.array_equal(z, z_ref), "zero points differ"
    assert np.array_equal(u, u_ref.astype(np.int64)), f"{(u != u_ref).sum()} codes differ"
    assert np.array_equal(S, q.sum(axis=1)), "code sums differ"
    return q, s, z


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("m,k", [(1, 128), (37, 1024), (200, 4096)])
@pytest.mark.parametrize("with_c", [False, True])
def test_minmax_act_exact(bits, m, k, with_c):
    x = _x(bits * 100 + m + k, m, k)
    c = synth.generator(9).uniform(0.5, 2.0, k).astype(np.float32) if with_c else None
    qp = fq.qparams(fq.ROW, 0.9, bits=bits, zero_point=fq.ZERO_POINT_MINMAX)
    xq, blk = fq.fq_quant_act(C.dev(x), qp, fq.Transform(c=C.dev(c)) if with_c else None)
    v32 = O.act_transform(x, c=c).astype(np.float32)
    _check_rows(xq, blk, v32, bits, 0.9)


@pytest.mark.parametrize("bits", [3, 4])
def test_minmax_weight_exact(bits):
    w = synth.prefill_linear(2048, 264, m=1, transform=False)["w"]
    qp = fq.qparams(fq.ROW, 1.0, bits=bits, zero_point=fq.ZERO_POINT_MINMAX)
    wq, blk = fq.fq_quant_weight(C.dev(w), qp)
    _check_rows(wq, blk, w.astype(np.float32), bits, 1.0)


def test_minmax_zero_and_constant_rows():
    """A row of zeros has s = 0, z = 0, codes u = 0; an all-positive row has z = 0."""
    x = np.zeros((3, 256), np.float16)
    x[1] = 2.0
    x[2, 5] = -1.0
    qp = fq.qparams(fq.ROW, 1.0, bits=4, zero_point=fq.ZERO_POINT_MINMAX)
    xq, blk = fq.fq_quant_act(C.dev(x), qp)
    _check_rows(xq, blk, x.astype(np.float32), 4, 1.0)


@pytest.mark.parametrize("bits", [3, 4])
def test_minmax_act_transform(bits):
    """With the Kronecker transform (float64 transform path): transformed
    values within the parity tolerance, scales within 1e-4, and scale, zero
    point and codes exactly those of the kernel's own transformed values."""
    d = synth.prefill_linear(4096, 128, m=48)
    qp = fq.qparams(fq.ROW, 1.0, bits=bits, zero_point=fq.ZERO_POINT_MINMAX)
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]))
    xq, blk, xhat = fq.fq_quant_act_debug(C.dev(d["x"]), qp, t)
    _, _, v_ref = O.quant_act(d["x"], O.ROW, 1.0, d["p1"], d["p2"])
    vg = C.host(xhat)
    C.check_values(vg, v_ref)
    q, s, z = _check_rows(xq, blk, vg, bits, 1.0)   # exactly the rule on its own values
    s_ref, z_ref = O.minmax_params(v_ref, bits, 1.0)
    assert np.all(np.abs(s.astype(np.float64) - s_ref) <= 1e-4 * s_ref)


def _zp_operands(seed, rows, k, bits):
    """Random codes u in [0, 2^b - 1] per row, a zero point and a scale."""
    g = synth.generator(seed)
    u = g.integers(0, 1 << bits, (rows, k))
    z = g.integers(0, 1 << bits, rows).astype(np.int32)
    s = synth.random_scales(g, rows)
    q = u - (1 << (bits - 1))
    blk = np.concatenate([s.view(np.int32), ((1 << (bits - 1)) - z).astype(np.int32),
                          q.sum(axis=1).astype(np.int32)]).view(np.float32)
    return u, z, s, O.pack_int4(q), blk


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("m,n,k", [(8, 264, 1024), (200, 512, 4096), (64, 8192, 8192), (1, 256, 65536)])
def test_gemm_zero_point_exact(bits, m, n, k):
    ux, zx, sx, xq, bx = _zp_operands(m + k, m, k, bits)
    uw, zw, sw, wq, bw = _zp_operands(n + k + 1, n, k, bits)
    y = fq.fq_w4a4_gemm(C.dev(xq), C.dev(bx), C.dev(wq), C.dev(bw), fq.ROW_ZP)
    acc = O.gemm_asym(ux, zx, uw, zw)
    C.check_fp16_exact(C.host(y), O.dequant_row(acc, sx, sw))
    fq.fq_check_device_error()


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("m", [5, 300])
def test_linear_minmax_exact(bits, m):
    """W3A3 / W4A4 with the min-max quantizer on both sides, end to end."""
    d = synth.prefill_linear(1024, 264, m=m, transform=False)
    qp = fq.qparams(fq.ROW, 1.0, bits=bits, zero_point=fq.ZERO_POINT_MINMAX)
    wq, bw = fq.fq_quant_weight(C.dev(d["w"]), qp)
    y = C.host(fq.fq_linear(C.dev(d["x"]), qp, wq, bw))
    xv = d["x"].astype(np.float32)
    wv = d["w"].astype(np.float32)
    sx, zx = O.minmax_params(xv, bits)
    sw, zw = O.minmax_params(wv, bits)
    acc = O.gemm_asym(O.quantize_u(xv, sx, zx, bits), zx, O.quantize_u(wv, sw, zw, bits), zw)
    C.check_fp16_exact(y, O.dequant_row(acc, sx, sw))
    fq.fq_check_device_error()
