"""fq_quant_act / fq_quant_weight on the GPU against the CPU oracle."""
import numpy as np
import pytest
import torch

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu

GRAN = {"row": (fq.ROW, O.ROW), "group": (fq.GROUP, O.GROUPED), "static": (fq.STATIC, O.STATIC)}


def _x(seed, m, k, scale=1.0):
    g = synth.generator(seed)
    cs = np.ones(k)
    cs[g.permutation(k)[: max(1, k // 100)]] = 30.0
    return synth._draw(g, (m, k), "normal", scale, col_scale=cs)


def _static_scales(seed, k):
    return synth.random_scales(synth.generator(seed), k, 0.05, 2.0)


def _gpu_scales(s, gran):
    if s is None:
        return None
    s = C.host(s)
    return s.T.astype(np.float32) if gran == fq.GROUP else s


@pytest.mark.parametrize("gname", ["row", "group", "static"])
@pytest.mark.parametrize("m,k", [(1, 128), (3, 256), (16, 256), (129, 4096), (64, 14336), (5, 32768)])
@pytest.mark.parametrize("with_c", [False, True])
def test_quant_act_exact(gname, m, k, with_c):
    """Without the transform every step is float32 as written: bit-exact."""
    gf, go = GRAN[gname]
    x = _x(m * 7 + k, m, k)
    c = synth.generator(5).uniform(0.5, 2.0, k).astype(np.float32) if with_c else None
    ss = _static_scales(k, k) if gname == "static" else None
    alpha = 0.9 if gname != "static" else 1.0
    t = fq.Transform(c=C.dev(c)) if with_c else None
    xq, sx = fq.fq_quant_act(C.dev(x), fq.qparams(gf, alpha), t, C.dev(ss) if ss is not None else None)
    q_ref, s_ref, _ = O.quant_act(x, go, alpha, c=c, static_scale=ss)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    if gname != "static":
        assert np.array_equal(_gpu_scales(sx, gf), s_ref)


@pytest.mark.parametrize("with_c", [False, True])
def test_quant_act_static_4byte_aligned_scales(with_c):
    """Static scales (and c) that are only 4-byte aligned take the row kernel
    instead of the element-parallel one; the codes are the same."""
    m, k = 37, 1024
    x = _x(11, m, k)
    ss = _static_scales(12, k)
    c = synth.generator(13).uniform(0.5, 2.0, k).astype(np.float32) if with_c else None
    ss_buf = torch.zeros(k + 1, dtype=torch.float32, device="cuda")
    ss_buf[1:] = torch.from_numpy(ss).cuda()
    t = None
    if with_c:
        c_buf = torch.zeros(k + 1, dtype=torch.float32, device="cuda")
        c_buf[1:] = torch.from_numpy(c).cuda()
        t = fq.Transform(c=c_buf[1:])
    xq, _ = fq.fq_quant_act(C.dev(x), fq.qparams(fq.STATIC), t, ss_buf[1:])
    q_ref, _, _ = O.quant_act(x, O.STATIC, 1.0, c=c, static_scale=ss)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))


def test_quant_act_tiny_workload():
    d = synth.tiny_linear()
    xq, sx = fq.fq_quant_act(C.dev(d["x"]), fq.qparams(fq.ROW, 1.0))
    q_ref, s_ref, _ = O.quant_act(d["x"], O.ROW, 1.0)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    assert np.array_equal(C.host(sx), s_ref)


def _transform_case(d, gname, m=None):
    """Transformed values, scales and codes against the oracle (see gpu_checks)."""
    gf, go = GRAN[gname]
    x = d["x"] if m is None else d["x"][:m]
    alpha = d.get("alpha_a", 1.0)
    t = fq.Transform(C.dev(d["p1"]), C.dev(d["p2"]), C.dev(d["c"]) if d.get("c") is not None else None)
    xq, sx, xhat = fq.fq_quant_act_debug(C.dev(x), fq.qparams(gf, alpha), t)
    xq2, sx2 = fq.fq_quant_act(C.dev(x), fq.qparams(gf, alpha), t)
    assert torch.equal(xq, xq2) and torch.equal(sx, sx2), "the debug kernel quantized differently"
    q_ref, s_ref, v_ref = O.quant_act(x, go, alpha, d["p1"], d["p2"], d.get("c"))
    vg = C.host(xhat)
    qg = C.unpack(C.host(xq))
    worst = C.check_values(vg, v_ref)
    s_gpu = _gpu_scales(sx, gf)
    C.check_own_scales(s_gpu, vg, go, alpha)
    C.check_own_codes(qg, vg, s_gpu, go)
    if gname == "row":
        C.check_scales_row(s_gpu, s_ref)
    else:
        C.check_scales_group(s_gpu, s_ref, v_ref, alpha)
    ex = C.exempt_mask(v_ref, s_ref, s_gpu, go)
    n_ex, n_diff = C.check_codes(qg, q_ref, ex)
    print(f"{d['name']} {gname}: max |dv|/max(|v|, 2^-10 amax) {worst:.2e}, boundary-exempt {n_ex}, "
          f"differing codes {n_diff}")
    return n_ex, n_diff


@pytest.mark.parametrize("m", [256, 2048])
def test_quant_act_transform_hidden(m):
    """LLaMA-3-8B-like hidden size: Kronecker (64, 64), c, alpha 0.9, pivot token."""
    _transform_case(synth.transform_quant(m=m), "row")


def test_quant_act_transform_group():
    d = synth.prefill_linear(8192, 128, m=96, transform=True)
    d["alpha_a"] = 0.95
    _transform_case(d, "group")


@pytest.mark.parametrize("tokens,heads", [(64, 8), (1000, 8), (256, 32)])
def test_quant_kv_cache_per_head(tokens, heads):
    """INT4 key / value cache: FlatQuant's per-head P_h as the Kronecker
    transform P1 = I_H, P2 = P_h, one scale per token and head (the 128-group
    of a 128-wide head); the identity passed as a matrix and as P1 = NULL."""
    d = synth.kv_cache(tokens, heads)
    _transform_case(d, "group")
    x, t = C.dev(d["x"]), fq.Transform(None, C.dev(d["p2"]), n1=heads)
    q1, s1, v1 = fq.fq_quant_act_debug(x, fq.qparams(fq.GROUP, 1.0), t)
    q2, s2, v2 = fq.fq_quant_act_debug(x, fq.qparams(fq.GROUP, 1.0), fq.Transform(C.dev(d["p1"]), C.dev(d["p2"])))
    assert torch.equal(q1, q2) and torch.equal(s1, s2) and torch.equal(v1, v2), "P1 = NULL differs from P1 = I"


@pytest.mark.parametrize("tokens,heads", [(64, 8), (1000, 8), (40, 5), (256, 32), (3, 1)])
def test_fq_quant_kv(tokens, heads):
    """fq_quant_kv: 64 head vectors per kernel item when tokens * heads is a
    multiple of 64 (else one token per item); codes and token-major scales
    against the oracle (the transformed-value tolerance of gpu_checks:
    scales equal or one fp16 step apart at a midpoint, codes equal outside
    the tie band)."""
    d = synth.kv_cache(tokens, heads, seed=tokens + heads)
    q, s = fq.fq_quant_kv(C.dev(d["x"]), C.dev(d["p2"]), 0.95)
    q_ref, s_ref, v_ref = O.quant_act(d["x"], O.GROUPED, 0.95, d["p1"], d["p2"])
    sg = C.host(s).astype(np.float32)
    C.check_scales_group(sg, s_ref, v_ref, 0.95)
    ex = C.exempt_mask(v_ref, s_ref, sg, O.GROUPED)
    n_ex, n_diff = C.check_codes(C.unpack(C.host(q)), q_ref, ex)
    print(f"{d['name']}: boundary-exempt {n_ex}, differing codes {n_diff}")
    fq.fq_check_device_error()


def test_fq_quant_kv_bench_size():
    """The benchmark's KV workload (16384 tokens x 8 heads) in its launch
    configuration, on sampled tokens covering every 128-token stretch."""
    d = synth.kv_cache(16384, 8)
    q, s = fq.fq_quant_kv(C.dev(d["x"]), C.dev(d["p2"]))
    rows = C.tile_samples(17, 16384)
    q_ref, s_ref, v_ref = O.quant_act(d["x"][rows], O.GROUPED, 1.0, d["p1"], d["p2"])
    sg = C.host(s)[rows].astype(np.float32)
    C.check_scales_group(sg, s_ref, v_ref, 1.0)
    ex = C.exempt_mask(v_ref, s_ref, sg, O.GROUPED)
    n_ex, n_diff = C.check_codes(C.unpack(C.host(q)[rows]), q_ref, ex)
    print(f"{d['name']}: {len(rows)} tokens, boundary-exempt {n_ex}, differing codes {n_diff}")
    fq.fq_check_device_error()


@pytest.mark.parametrize("k", [14336, 28672])
def test_quant_act_transform_wide(k):
    """(112, 128) keeps the factors in shared memory; (224, 128) reads them through L1."""
    d = synth.prefill_linear(k, 128, m=24, transform=True)
    _transform_case(d, "row")
    _transform_case(d, "group")


def test_quant_act_identity_transform_is_exact():
    d = synth.transform_quant(m=64, k=4096)
    eye = np.eye(64, dtype=np.float32)
    t = fq.Transform(C.dev(eye), C.dev(eye), None)
    xq, sx = fq.fq_quant_act(C.dev(d["x"]), fq.qparams(fq.ROW, 0.9), t)
    q_ref, s_ref, _ = O.quant_act(d["x"], O.ROW, 0.9)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    assert np.array_equal(C.host(sx), s_ref)


@pytest.mark.parametrize("gname", ["row", "group"])
@pytest.mark.parametrize("qsm", [False, True])
def test_quant_weight_exact(gname, qsm):
    gf, go = GRAN[gname]
    d = synth.prefill_linear(4096, 264, m=1, transform=False)
    s_k = _static_scales(3, 4096) if qsm else None
    wq, sw = fq.fq_quant_weight(C.dev(d["w"]), fq.qparams(gf, 0.95), None, C.dev(s_k) if qsm else None)
    q_ref, s_ref, _ = O.quant_weight(d["w"], go, 0.95, qsm_scale=s_k)
    assert np.array_equal(C.host(wq), O.pack_int4(q_ref))
    assert np.array_equal(_gpu_scales(sw, gf), s_ref)


@pytest.mark.parametrize("gname", ["row", "group"])
def test_quant_weight_inverse_transform(gname):
    gf, go = GRAN[gname]
    d = synth.transform_quant(m=8, k=8192)
    w = synth.prefill_linear(8192, 136, m=1, transform=False)["w"]
    inv = fq.Transform(C.dev(d["p1_inv"]), C.dev(d["p2_inv"]), C.dev(d["c"]))
    wq, sw = fq.fq_quant_weight(C.dev(w), fq.qparams(gf, 1.0), inv)
    q_ref, s_ref, v_ref = O.quant_weight(w, go, 1.0, d["p1_inv"], d["p2_inv"], d["c"])
    s_gpu = _gpu_scales(sw, gf)
    if gname == "row":
        C.check_scales_row(s_gpu, s_ref)
    else:
        C.check_scales_group(s_gpu, s_ref, v_ref, 1.0)
    C.check_codes(C.unpack(C.host(wq)), q_ref, C.exempt_mask(v_ref, s_ref, s_gpu, go))


def test_quant_act_zero_rows():
    x = np.zeros((4, 256), np.float16)
    x[2, 5] = 1.0
    xq, sx = fq.fq_quant_act(C.dev(x), fq.qparams(fq.ROW, 1.0))
    q_ref, s_ref, _ = O.quant_act(x, O.ROW, 1.0)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    assert np.array_equal(C.host(sx), s_ref)
    xq, sx = fq.fq_quant_act(C.dev(x), fq.qparams(fq.GROUP, 1.0))
    q_ref, s_ref, _ = O.quant_act(x, O.GROUPED, 1.0)
    assert np.array_equal(C.host(xq), O.pack_int4(q_ref))
    assert np.array_equal(C.host(sx).T.astype(np.float32), s_ref)
    torch.cuda.synchronize()
    fq.fq_check_device_error()
