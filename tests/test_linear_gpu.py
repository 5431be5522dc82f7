"""fq_linear end to end at the workloads' full sizes, in the launch
configuration the benchmark times, against the CPU oracle on sampled outputs."""
import numpy as np
import pytest

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def test_linear_tiny_exact():
    """16 x 256 x 256, no transform, per-token x per-channel: every output bit-exact."""
    d = synth.tiny_linear()
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0))
    y = fq.fq_linear(C.dev(d["x"]), fq.qparams(fq.ROW, 1.0), wq, sw)
    qw, sw_ref, _ = O.quant_weight(d["w"], O.ROW, 1.0)
    ref = O.linear(d["x"], qw, sw_ref, O.ROW, 1.0)
    C.check_fp16_exact(C.host(y), ref)
    fq.fq_check_device_error()


def _samples(seed, m, n, nm=24, nn=384):
    g = synth.generator(seed)
    ms = np.unique(np.concatenate([[0, m - 1], g.integers(0, m, nm)]))
    ns = np.unique(np.concatenate([[0, n - 1], g.integers(0, n, nn)]))
    return ms, ns


def _check_sampled(y_gpu, d, ms, ns, gran_o, wgran_o):
    """Oracle on the sampled token rows and output channels (rows are independent)."""
    x = d["x"][ms]
    alpha = d.get("alpha_a", 1.0)
    qw, sw, _ = O.quant_weight(d["w"][ns], wgran_o, d.get("alpha_w", 1.0))
    qx, sx, vx = O.quant_act(x, gran_o, alpha, d.get("p1"), d.get("p2"), d.get("c"))
    yg = y_gpu[np.ix_(ms, ns)].astype(np.float64)
    if gran_o == O.ROW:
        ref = O.dequant_row(O.gemm_int(qx, qw), sx, sw).astype(np.float64)
        ex = C.exempt_mask(vx, sx, sx * (1 + C.TOL_REL), O.ROW) if "p1" in d else np.zeros(qx.shape, bool)
        wsum = (ex.astype(np.float64) @ np.abs(qw).T.astype(np.float64)) * sx[:, None] * sw[None, :]
        bound = C.ulp16(ref) + np.abs(ref) * 1.01 * C.TOL_REL + wsum
        err = np.abs(yg - ref)
        assert np.all(err <= bound), f"{(err > bound).sum()} outputs beyond the bound (max {err.max()})"
        exact = (err == 0).mean()
    else:
        ref = O.dequant_group(qx, qw, sx, sw).astype(np.float64)
        ex = C.exempt_mask(vx, sx, sx * (1 + 2 ** -10), O.GROUPED) if "p1" in d else np.zeros(qx.shape, bool)
        absum = np.zeros_like(ref)
        wsum = np.zeros_like(ref)
        for g in range(qx.shape[1] // O.GROUP):
            sl = slice(g * O.GROUP, (g + 1) * O.GROUP)
            s2 = sx[:, g:g + 1].astype(np.float64) * sw[None, :, g].astype(np.float64)
            absum += np.abs(O.gemm_int(qx[:, sl], qw[:, sl]).astype(np.float64) * s2)
            wsum += (ex[:, sl].astype(np.float64) @ np.abs(qw[:, sl]).T.astype(np.float64)) * s2
        ng = qx.shape[1] // O.GROUP
        slack = 2.0 ** -10 if "p1" in d else 0.0
        bound = C.ulp16(ref) + (ng * 2.0 ** -23 + slack) * absum + wsum
        err = np.abs(yg - ref)
        assert np.all(err <= bound), f"{(err > bound).sum()} outputs beyond the bound (max {err.max()})"
        exact = (err <= C.ulp16(ref)).mean()
    print(f"{d['name']}: {len(ms)}x{len(ns)} sampled outputs, exempt act codes {int(ex.sum())}, "
          f"fraction within 1 ulp/exact {exact:.4f}")


@pytest.mark.parametrize("k,n", synth.PREFILL_8B_SHAPES)
def test_linear_prefill_8b(k, n):
    """M = 2048 tokens, Kronecker-transformed per-token activations, per-channel weights."""
    d = synth.prefill_linear(k, n, m=2048)
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]))
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0))
    y = C.host(fq.fq_linear(C.dev(d["x"]), fq.qparams(fq.ROW, 1.0), wq, sw, t))
    fq.fq_check_device_error()
    ms, ns = _samples(k + n, 2048, n)
    _check_sampled(y, d, ms, ns, O.ROW, O.ROW)


@pytest.mark.parametrize("k,n", synth.GROUP_70B_SHAPES)
def test_linear_group_70b(k, n):
    """M = 4096, group-128 scales on both sides, Student-t weights."""
    d = synth.prefill_linear(k, n, m=4096, w_kind="t")
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]))
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.GROUP, 1.0))
    y = C.host(fq.fq_linear(C.dev(d["x"]), fq.qparams(fq.GROUP, 1.0), wq, sw, t))
    fq.fq_check_device_error()
    ms, ns = _samples(k + n + 1, 4096, n, nm=12, nn=256)
    _check_sampled(y, d, ms, ns, O.GROUPED, O.GROUPED)


@pytest.mark.parametrize("m", synth.DECODE_TOKENS)
@pytest.mark.parametrize("k,n", synth.DECODE_70B_SHAPES)
def test_linear_decode_static(m, k, n):
    """Static per-channel activation scales migrated into the weights: bit-exact."""
    d = synth.decode_static(m, k, n)
    s_k = d["static_scale"]
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0), None, C.dev(s_k))
    y = C.host(fq.fq_linear(C.dev(d["x"]), fq.qparams(fq.STATIC), wq, sw, static_scale=C.dev(s_k)))
    fq.fq_check_device_error()
    ns = _samples(m + k, m, n, nn=1024)[1]
    qw, sw_ref, _ = O.quant_weight(d["w"][ns], O.ROW, 1.0, qsm_scale=s_k)
    ref = O.linear(d["x"], qw, sw_ref, O.STATIC, static_scale=s_k)
    C.check_fp16_exact(y[:, ns], ref)
