"""The linear layer at the workloads' full sizes, in the launch configuration
the benchmark times, against the CPU oracle.

Each full-size case runs the layer three ways on the same device inputs:
fq_linear (the product call), and its two halves as the benchmark calls them
(fq_quant_act, then fq_w4a4_gemm with a preallocated workspace), plus the
debug quantization that also returns the transformed values.  The halves must
reproduce fq_linear bit for bit.  Then, on rows and columns sampled so that
every 256 x 256 output tile is hit:
* the quantization is checked against the oracle (transformed values, scales,
  codes; see gpu_checks), and
* the GEMM is checked DECOUPLED from it: the GPU's own codes and scales go
  through the oracle's integer GEMM and dequantization, and the fp16 outputs
  must match bit-exactly (per token, static) or within 1 fp16 ulp / the
  float32 cancellation bound (group).
"""
import numpy as np
import pytest
import torch

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


def _bits(y):
    return np.asarray(y).view(np.uint16)


def _run_three_ways(d, qp, gran, wq, sw, t=None, static_scale=None):
    """fq_linear, then quant + GEMM (bench's calls), then the debug quantization.
    Returns (Y, Xq, s_x, xhat) as host arrays (xhat None without a transform)."""
    X = C.dev(d["x"])
    m, k = d["x"].shape
    n = wq.shape[0]
    y_lin = C.host(fq.fq_linear(X, qp, wq, sw, t, static_scale=static_scale))
    xq, sx = fq.fq_quant_act(X, qp, t, static_scale)
    ws = torch.zeros(max(fq.fq_gemm_workspace_size(m, n, k, gran), 256), dtype=torch.uint8, device="cuda")
    y = C.host(fq.fq_w4a4_gemm(xq, sx, wq, sw, gran, workspace=ws))
    assert np.array_equal(_bits(y), _bits(y_lin)), "fq_linear differs from quantization + GEMM"
    xhat = None
    if t is not None:
        xq_d, sx_d, xhat_d = fq.fq_quant_act_debug(X, qp, t)
        assert torch.equal(xq_d, xq) and torch.equal(sx_d, sx), "the debug kernel quantized differently"
        xhat = C.host(xhat_d)
    fq.fq_check_device_error()
    return y, C.host(xq), (None if sx is None else C.host(sx)), xhat


def _quant_checks(d, rows, gran_o, alpha, xq, sx_rows, xhat):
    """Transformed values, scales and codes of the sampled rows against the oracle."""
    q_ref, s_ref, v_ref = O.quant_act(d["x"][rows], gran_o, alpha, d.get("p1"), d.get("p2"), d.get("c"))
    vg = xhat[rows]
    qg = C.unpack(xq[rows])
    worst = C.check_values(vg, v_ref)
    C.check_own_scales(sx_rows, vg, gran_o, alpha)
    C.check_own_codes(qg, vg, sx_rows, gran_o)
    if gran_o == O.ROW:
        C.check_scales_row(sx_rows, s_ref)
    else:
        C.check_scales_group(sx_rows, s_ref, v_ref, alpha)
    ex = C.exempt_mask(v_ref, s_ref, sx_rows, gran_o)
    n_ex, n_diff = C.check_codes(qg, q_ref, ex)
    print(f"{d['name']}: {len(rows)} rows, max |dv|/max(|v|, 2^-10 amax) {worst:.2e}, "
          f"boundary-exempt {n_ex}, differing codes {n_diff}")
    return qg


@pytest.mark.parametrize("k,n", synth.PREFILL_8B_SHAPES)
def test_linear_prefill_8b(k, n):
    """M = 2048 tokens, Kronecker-transformed per-token activations, per-channel weights."""
    d = synth.prefill_linear(k, n, m=2048)
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]))
    qp = fq.qparams(fq.ROW, 1.0)
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), qp)
    y, xq, sx, xhat = _run_three_ways(d, qp, fq.ROW, wq, sw, t)
    rows = C.tile_samples(k + n, d["m"])
    cols = C.tile_samples(k + n + 1, n)
    qx = _quant_checks(d, rows, O.ROW, 1.0, xq, sx[rows], xhat)
    qw, sw_ref, _ = O.quant_weight(d["w"][cols], O.ROW, 1.0)
    assert np.array_equal(C.host(wq)[cols], O.pack_int4(qw))
    assert np.array_equal(C.host(sw)[cols], sw_ref)
    C.check_gemm_decoupled(y[np.ix_(rows, cols)], qx, sx[rows], qw, sw_ref, O.ROW)


@pytest.mark.parametrize("k,n", synth.GROUP_70B_SHAPES)
def test_linear_group_70b(k, n):
    """M = 4096, group-128 scales on both sides, Student-t weights."""
    d = synth.prefill_linear(k, n, m=4096, w_kind="t")
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]))
    qp = fq.qparams(fq.GROUP, 1.0)
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), qp)
    y, xq, sx, xhat = _run_three_ways(d, qp, fq.GROUP, wq, sw, t)
    rows = C.tile_samples(k + n, d["m"])
    cols = C.tile_samples(k + n + 1, n)
    sx_rows = sx.T[rows].astype(np.float32)      # group-major [K/128][M] -> [rows, K/128]
    qx = _quant_checks(d, rows, O.GROUPED, 1.0, xq, sx_rows, xhat)
    qw, sw_ref, _ = O.quant_weight(d["w"][cols], O.GROUPED, 1.0)
    assert np.array_equal(C.host(wq)[cols], O.pack_int4(qw))
    assert np.array_equal(C.host(sw).T[cols].astype(np.float32), sw_ref)
    n_canc = C.check_gemm_decoupled(y[np.ix_(rows, cols)], qx, sx_rows, qw, sw_ref, O.GROUPED)
    print(f"{d['name']}: {len(rows)}x{len(cols)} outputs, {n_canc} within the cancellation bound only")


@pytest.mark.parametrize("m", synth.DECODE_TOKENS)
@pytest.mark.parametrize("k,n", synth.DECODE_70B_SHAPES)
def test_linear_decode_static(m, k, n):
    """Static per-channel activation scales migrated into the weights: bit-exact
    (no transform, so the oracle's codes are the GPU's)."""
    d = synth.decode_static(m, k, n)
    s_k = d["static_scale"]
    qp = fq.qparams(fq.STATIC)
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0), None, C.dev(s_k))
    y, xq, _, _ = _run_three_ways(d, qp, fq.STATIC, wq, sw, static_scale=C.dev(s_k))
    cols = C.tile_samples(m + k, n)
    q_ref, _, _ = O.quant_act(d["x"], O.STATIC, static_scale=s_k)
    assert np.array_equal(xq, O.pack_int4(q_ref))
    qw, sw_ref, _ = O.quant_weight(d["w"][cols], O.ROW, 1.0, qsm_scale=s_k)
    assert np.array_equal(C.host(wq)[cols], O.pack_int4(qw))
    C.check_gemm_decoupled(y[:, cols], q_ref, None, qw, sw_ref, O.STATIC)


def _kernel_names(fn):
    """Names of the kernels that fn launches (CUDA activity from the profiler)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events() if e.device_type.name == "CUDA"]


@pytest.mark.parametrize("m,k,n", [(1, 8192, 10240), (8, 28672, 8192), (64, 8192, 57344), (17, 1024, 3072)])
def test_linear_decode_fused_one_launch(m, k, n):
    """Decode with static scales (and a channel factor c) through fq_linear_fused:
    one kernel launch, no separate quantization, no memset; outputs bit-exact
    against the oracle; three calls in a row on one workspace whose bytes past
    the counter block are garbage, the counters (all words but the grid
    barrier's generation number, word 1) back at zero after each."""
    d = synth.decode_static(m, k, n, seed=3)
    s_k = d["static_scale"]
    c = synth.generator(m + 5).uniform(0.5, 2.0, k).astype(np.float32)
    qp = fq.qparams(fq.STATIC)
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(fq.ROW, 1.0), None, C.dev(s_k))
    X, SK, t = C.dev(d["x"]), C.dev(s_k), fq.Transform(c=C.dev(c))
    ws = torch.full((fq.fq_linear_workspace_size(m, n, k, fq.STATIC),), 0x5A, dtype=torch.uint8, device="cuda")
    ws[: fq.SYNC_BYTES].zero_()
    Y = torch.empty(m, n, dtype=torch.float16, device="cuda")
    names = _kernel_names(lambda: fq.fq_linear(X, qp, wq, sw, t, static_scale=SK, Y=Y, workspace=ws, fused=True))
    assert len(names) == 1 and "gemm_decode_kernel" in names[0], names
    q_ref, _, _ = O.quant_act(d["x"], O.STATIC, c=c, static_scale=s_k)
    cols = C.tile_samples(m + k + n, n)
    qw, sw_ref, _ = O.quant_weight(d["w"][cols], O.ROW, 1.0, qsm_scale=s_k)
    first = C.host(Y)
    C.check_gemm_decoupled(first[:, cols], q_ref, None, qw, sw_ref, O.STATIC)
    for _ in range(2):
        y = C.host(fq.fq_linear(X, qp, wq, sw, t, static_scale=SK, Y=Y, workspace=ws, fused=True))
        assert np.array_equal(y.view(np.uint16), first.view(np.uint16))
        words = ws[: fq.SYNC_BYTES].view(torch.int32)
        assert not words[0] and not words[2:].any(), "the counters are not back at zero"
    xq, _ = fq.fq_quant_act(X, qp, t, SK)
    y2 = C.host(fq.fq_w4a4_gemm(xq, None, wq, sw, fq.STATIC))
    assert np.array_equal(y2.view(np.uint16), first.view(np.uint16)), "fused and two-launch paths differ"
    y3 = C.host(fq.fq_linear(X, qp, wq, sw, t, static_scale=SK))
    assert np.array_equal(y3.view(np.uint16), first.view(np.uint16)), "fq_linear differs from fq_linear_fused"
    fq.fq_check_device_error()
