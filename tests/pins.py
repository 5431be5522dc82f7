"""Checks that pin the CPU oracle to what the pages and the mathematics fix.

Each check takes the oracle module (or a copy with one planted mistake) and
raises AssertionError when it disagrees.  ``test_oracle_pins`` runs every check
on the oracle as it stands and, through ``test_oracle_mutants``, shows that a
plausible mistake in any step (a transposed factor, a dropped term, a wrong
sign, rounding or nibble order) fails at least one of them.
"""
from __future__ import annotations

import os
import types

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


# ------------------------------------------------------------------ quantizer

def check_rtn_golden(o):
    """Hand-worked rows in tests/golden/rtn_worked.txt (Q(W), FRM-PTQ page 初步介绍)."""
    for ln in _lines("rtn_worked.txt"):
        head, xs, ss, qs = [p.strip() for p in ln.split("|")]
        mode, alpha = head.split()
        x = np.array([float(v) for v in xs.split()], dtype=np.float16)
        s_exp = np.float32(float(ss))
        q_exp = np.array([int(v) for v in qs.split()], dtype=np.int8)
        if mode == "row":
            q, s, _ = o.quant_act(x[None, :], o.ROW, float(alpha))
            assert np.float32(s[0]) == s_exp, (ln, s[0])
            assert np.array_equal(q[0], q_exp), (ln, q[0])
        elif mode == "group1":
            xx = np.zeros((1, o.GROUP), dtype=np.float16)
            xx[0, :x.size] = x
            q, s, _ = o.quant_act(xx, o.GROUPED, float(alpha))
            assert np.float32(s[0, 0]) == s_exp, (ln, s[0, 0])
            assert np.array_equal(q[0, :x.size], q_exp), (ln, q[0, :x.size])
        else:
            raise ValueError(mode)


def check_rtn_bounds(o):
    """Every unclipped element satisfies |v - s q| <= s/2; codes lie in [-8, 7];
    alpha = 1 never produces -8 and maps each row's absmax to +-7."""
    g = np.random.Generator(np.random.PCG64(11))
    x = (g.standard_normal((64, 256)) * g.uniform(0.01, 30, (64, 1))).astype(np.float16)
    for alpha in (1.0, 0.8):
        q, s, v = o.quant_act(x, o.ROW, alpha)
        assert q.min() >= -8 and q.max() <= 7
        deq = q.astype(np.float64) * s[:, None].astype(np.float64)
        unclipped = (q > -8) & (q < 7)
        err = np.abs(v.astype(np.float64) - deq)
        bound = s[:, None].astype(np.float64) / 2 * (1 + 1e-6)
        assert np.all(err[unclipped] <= np.broadcast_to(bound, err.shape)[unclipped])
        if alpha == 1.0:
            assert q.min() > -8
            idx = np.abs(v).argmax(axis=1)
            assert np.all(np.abs(q[np.arange(64), idx]) == 7)
    qg, sg, vg = o.quant_act(x, o.GROUPED, 1.0)
    deq = qg.astype(np.float64) * np.repeat(sg, o.GROUP, axis=1)
    unclipped = (qg > -8) & (qg < 7)
    err = np.abs(vg.astype(np.float64) - deq)
    bound = np.repeat(sg, o.GROUP, axis=1) / 2 * (1 + 1e-6)
    assert np.all(err[unclipped] <= bound[unclipped])


def check_pack(o):
    """tests/golden/pack_int4.txt and the round trip over all 16 x 16 code pairs."""
    for ln in _lines("pack_int4.txt"):
        codes, byte = [p.strip() for p in ln.split("|")]
        q = np.array([[int(v) for v in codes.split()]], dtype=np.int8)
        assert o.pack_int4(q)[0, 0] == int(byte, 16), ln
    a, b = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8))
    q = np.stack([a.ravel(), b.ravel()], axis=1).reshape(1, -1).astype(np.int8)
    assert np.array_equal(o.unpack_int4(o.pack_int4(q)), q)


# ------------------------------------------------------------------ transform

def check_kron_golden(o):
    """tests/golden/kron_worked.txt (FlatQuant notes, Kronecker 分解)."""
    d = {}
    for ln in _lines("kron_worked.txt"):
        key, *vals = ln.split()
        d[key] = np.array([float(v) for v in vals])
    n1, n2 = int(d["n1"][0]), int(d["n2"][0])
    p1 = d["P1"].reshape(n1, n1)
    p2 = d["P2"].reshape(n2, n2)
    p1i = d["P1inv"].reshape(n1, n1)
    p2i = d["P2inv"].reshape(n2, n2)
    xh = o.act_transform(d["x"][None, :], p1, p2)
    assert np.array_equal(xh[0], d["xhat"]), xh
    wh = o.weight_transform(d["w"][None, :], p1i, p2i)
    assert np.array_equal(wh[0], d["what"]), wh


def check_kron_explicit(o):
    """x (P1 (x) P2) against the explicit n x n Kronecker matrix, and the weight
    side against (P1^-1 (x) P2^-1) w, on tiny n, float64, <= 1e-12 relative."""
    g = np.random.Generator(np.random.PCG64(5))
    for n1, n2 in [(2, 4), (3, 5), (8, 8), (4, 2)]:
        n = n1 * n2
        x = g.standard_normal((3, n))
        p1 = g.standard_normal((n1, n1))
        p2 = g.standard_normal((n2, n2))
        c = g.uniform(0.5, 2, n)
        ref = (x * c) @ np.kron(p1, p2)
        got = o.act_transform(x, p1, p2, c)
        assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max(), (n1, n2)
        p1i, p2i = np.linalg.inv(p1), np.linalg.inv(p2)
        w = g.standard_normal((2, n))
        refw = (w / c) @ np.kron(p1i, p2i).T
        gotw = o.weight_transform(w, p1i, p2i, c)
        assert np.abs(gotw - refw).max() <= 1e-12 * np.abs(refw).max(), (n1, n2)


def check_function_preservation(o):
    """X P (P^-1 W^T) = X W^T in float64 (FlatQuant notes, 核心思想), with the
    channel scale c on both sides; and a permutation P (PT2-LLM page, SSR:
    X' W'^T = X W^T) is exact."""
    g = np.random.Generator(np.random.PCG64(6))
    n1, n2 = 8, 16
    n = n1 * n2
    x = g.standard_normal((5, n))
    w = g.standard_normal((7, n))
    p1 = g.standard_normal((n1, n1)) + 4 * np.eye(n1)
    p2 = g.standard_normal((n2, n2)) + 4 * np.eye(n2)
    c = g.uniform(0.5, 2, n)
    y = o.act_transform(x, p1, p2, c) @ o.weight_transform(w, np.linalg.inv(p1), np.linalg.inv(p2), c).T
    ref = x @ w.T
    assert np.abs(y - ref).max() <= 1e-10 * np.abs(ref).max()
    # permutation factors (PT2-LLM page, SSR: W' = W P, X' = X P): the transform
    # only moves values, and on integer data the product is exactly unchanged
    e1 = np.eye(n1)[g.permutation(n1)]
    e2 = np.eye(n2)[g.permutation(n2)]
    xi = g.integers(-50, 50, (5, n)).astype(np.float64)
    wi = g.integers(-50, 50, (7, n)).astype(np.float64)
    xp = o.act_transform(xi, e1, e2)
    wp = o.weight_transform(wi, e1.T, e2.T)
    assert np.array_equal(np.sort(xp, axis=1), np.sort(xi, axis=1))
    assert np.array_equal(xp @ wp.T, xi @ wi.T)


def check_identity_transform(o):
    """P1 = P2 = I and c = 1 reduce the transformed path to the plain one, bit for bit."""
    g = np.random.Generator(np.random.PCG64(7))
    x = g.standard_normal((4, 256)).astype(np.float16)
    a = o.quant_act(x, o.ROW, 0.9, np.eye(16, dtype=np.float32), np.eye(16, dtype=np.float32),
                    np.ones(256, np.float32))
    b = o.quant_act(x, o.ROW, 0.9)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


def check_flop_count(o):
    """Per row, a dense n x n transform costs 2 n^2 flops and the Kronecker form
    2 n (n1 + n2); with n1 = n2 = sqrt(n) the saving is sqrt(n)/2, and the
    parameters shrink from n^2 to n1^2 + n2^2, a saving of n/2 (FlatQuant notes,
    Kronecker 分解)."""
    for r in (8, 16, 64, 128):
        n = r * r
        assert o.kron_flops(r, r) == 2 * n * 2 * r
        assert o.dense_transform_flops(n) / o.kron_flops(r, r) == np.sqrt(n) / 2
        assert (n * n) / (r * r + r * r) == n / 2
    assert o.kron_flops(64, 128) == 2 * 8192 * 192


# ------------------------------------------------------------------ GEMM + dequant

def _brute(qx, qw):
    m, k = qx.shape
    n = qw.shape[0]
    out = [[0] * n for _ in range(m)]
    for i in range(m):
        for j in range(n):
            t = 0
            for kk in range(k):
                t += int(qx[i, kk]) * int(qw[j, kk])
            out[i][j] = t
    return np.array(out, dtype=np.int64)


def check_gemm_bruteforce(o):
    """Integer accumulation against a pure-Python triple loop on tiny shapes, and
    the extreme -8 * -8 over K = 28672 (the largest K in use)."""
    g = np.random.Generator(np.random.PCG64(8))
    for m, n, k in [(1, 1, 1), (3, 5, 7), (4, 6, 128), (2, 3, 256)]:
        qx = g.integers(-8, 8, (m, k), dtype=np.int8)
        qw = g.integers(-8, 8, (n, k), dtype=np.int8)
        assert np.array_equal(o.gemm_int(qx, qw), _brute(qx, qw)), (m, n, k)
    k = 28672
    qx = np.full((1, k), -8, np.int8)
    assert o.gemm_int(qx, qx)[0, 0] == 64 * k
    qw = np.full((1, k), 7, np.int8)
    assert o.gemm_int(qx, qw)[0, 0] == -56 * k


def check_linear_golden(o):
    """tests/golden/linear_worked.txt: the whole layer on a hand-worked 1 x 4 x 2 case."""
    d = {}
    for ln in _lines("linear_worked.txt"):
        key, *vals = ln.split()
        d[key] = np.array([float(v) for v in vals])
    x = d["x"].astype(np.float16)[None, :]
    w = np.stack([d["w0"], d["w1"]]).astype(np.float16)
    qw, sw, _ = o.quant_weight(w, o.ROW, 1.0)
    assert np.array_equal(qw[0], d["qw0"]) and np.array_equal(qw[1], d["qw1"]), qw
    qx, sx, _ = o.quant_act(x, o.ROW, 1.0)
    assert np.array_equal(qx[0], d["qx"]), qx
    acc = o.gemm_int(qx, qw)
    assert np.array_equal(acc[0], d["acc"]), acc
    y = o.linear(x, qw, sw, o.ROW, 1.0)
    assert np.array_equal(y[0].astype(np.float64), d["y"]), y


def check_dequant_bound(o):
    """The per-row epilogue equals the float64 product of the dequantized
    operands up to the float32 and float16 roundings: |y - ref| <= 1 fp16 ulp
    of ref + 2^-22 |ref|; the group epilogue likewise with per-group scales."""
    g = np.random.Generator(np.random.PCG64(9))
    m, n, k = 8, 16, 512
    x = (g.standard_normal((m, k)) * 3).astype(np.float16)
    w = (g.standard_normal((n, k)) * 0.02).astype(np.float16)
    for gran in (o.ROW, o.GROUPED):
        qx, sx, _ = o.quant_act(x, gran, 1.0)
        qw, sw, _ = o.quant_weight(w, gran, 1.0)
        y = o.linear(x, qw, sw, gran, 1.0).astype(np.float64)
        if gran == o.ROW:
            xd = qx * sx[:, None].astype(np.float64)
            wd = qw * sw[:, None].astype(np.float64)
        else:
            xd = qx * np.repeat(sx, o.GROUP, axis=1)
            wd = qw * np.repeat(sw, o.GROUP, axis=1)
        ref = xd @ wd.T
        ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
        assert np.all(np.abs(y - ref) <= ulp + 2.0 ** -22 * np.abs(ref)), gran


def check_group_equals_row(o):
    """With K = 128 (one group) and float16-exact scales the group path equals the
    per-row path (FRM-PTQ: the granularities differ only in the scale's extent)."""
    g = np.random.Generator(np.random.PCG64(10))
    m, n, k = 4, 8, 128
    x = g.standard_normal((m, k))
    x = x / np.abs(x).max(axis=1, keepdims=True) * (7 * 2.0 ** g.integers(-3, 3, (m, 1)))
    w = g.standard_normal((n, k))
    w = w / np.abs(w).max(axis=1, keepdims=True) * (7 * 2.0 ** g.integers(-9, -5, (n, 1)))
    x, w = x.astype(np.float16), w.astype(np.float16)
    qxr, sxr, _ = o.quant_act(x, o.ROW, 1.0)
    qxg, sxg, _ = o.quant_act(x, o.GROUPED, 1.0)
    assert np.array_equal(qxr, qxg) and np.array_equal(sxr, sxg[:, 0])
    qwr, swr, _ = o.quant_weight(w, o.ROW, 1.0)
    qwg, swg, _ = o.quant_weight(w, o.GROUPED, 1.0)
    assert np.array_equal(qwr, qwg)
    yr = o.linear(x, qwr, swr, o.ROW, 1.0)
    yg = o.linear(x, qwg, swg, o.GROUPED, 1.0)
    assert np.array_equal(yr, yg)


def check_static_equals_row(o):
    """Static per-channel scales all equal to a row's dynamic scale give that row's
    dynamic codes (MergeQuant static vs per-token dynamic calibration)."""
    g = np.random.Generator(np.random.PCG64(12))
    x = g.standard_normal((3, 256)).astype(np.float16)
    q, s, _ = o.quant_act(x, o.ROW, 1.0)
    for r in range(3):
        qs, _, _ = o.quant_act(x[r:r + 1], o.STATIC, static_scale=np.full(256, s[r], np.float32))
        assert np.array_equal(qs[0], q[r])


def check_qsm_fold(o):
    """Quantization step migration: folding s_k into the weights and dequantizing
    with s_w' alone approximates sum_k q_x s_k w (MergeQuant 核心思路), and the fold
    multiplies the weight columns, not the rows."""
    g = np.random.Generator(np.random.PCG64(13))
    m, n, k = 4, 6, 256
    x = g.standard_normal((m, k)).astype(np.float16)
    w = (g.standard_normal((n, k)) * 0.02).astype(np.float16)
    s_k = g.uniform(0.2, 0.6, k).astype(np.float32)
    qx, _, _ = o.quant_act(x, o.STATIC, static_scale=s_k)
    qw, sw, v = o.quant_weight(w, o.ROW, 1.0, qsm_scale=s_k)
    assert np.array_equal(v, w.astype(np.float32) * s_k[None, :])
    y = o.linear(x, qw, sw, o.STATIC, static_scale=s_k).astype(np.float64)
    ref = (qx * s_k.astype(np.float64)) @ w.astype(np.float64).T
    # error of W4 weights: |sum_k qx_k dq_k| <= sum |qx| s_w / 2 per output
    bound = np.abs(qx).sum(axis=1, keepdims=True) * sw[None, :] / 2 + 1e-2 * np.abs(ref)
    assert np.all(np.abs(y - ref) <= bound)


def check_asym_golden(o):
    """Hand-worked rows of the general quantizer in tests/golden/rtn_asym_worked.txt
    (Q(W) with a zero point and any bit width; FRM-PTQ page, 初步介绍)."""
    for ln in _lines("rtn_asym_worked.txt"):
        head, xs, ss, zs, us = [p.strip() for p in ln.split("|")]
        bits, alpha = head.split()
        x = np.array([[float(v) for v in xs.split()]], dtype=np.float16).astype(np.float32)
        s, z = o.minmax_params(x, int(bits), float(alpha))
        assert np.float32(s[0]) == np.float32(float(ss)), (ln, s[0])
        assert int(z[0]) == int(zs), (ln, z[0])
        u = o.quantize_u(x, s, z, int(bits))
        assert np.array_equal(u[0], np.array([int(v) for v in us.split()])), (ln, u[0])


def check_asym_bounds(o):
    """Codes lie in [0, 2^b - 1]; 0 quantizes to z exactly; every unclipped value
    satisfies |v - s (u - z)| <= s/2; with alpha = 1 nothing clips, and each
    row's extremes land within one code of the ends of the range."""
    g = np.random.Generator(np.random.PCG64(17))
    x = (g.standard_normal((48, 200)) * g.uniform(0.01, 20, (48, 1)) + g.uniform(-3, 3, (48, 1)))
    x = x.astype(np.float16).astype(np.float32)
    x[5] = np.abs(x[5])       # all non-negative: lo = 0, z = 0
    x[6] = -np.abs(x[6])      # all non-positive: hi = 0
    for bits in (2, 3, 4, 8):
        qmax = (1 << bits) - 1
        for alpha in (1.0, 0.9):
            s, z = o.minmax_params(x, bits, alpha)
            u = o.quantize_u(x, s, z, bits).astype(np.int64)
            assert u.min() >= 0 and u.max() <= qmax
            assert np.all((z >= 0) & (z <= qmax))
            zero_code = o.quantize_u(np.zeros_like(x[:, :1]), s, z, bits)[:, 0]
            assert np.array_equal(zero_code.astype(np.int64), z.astype(np.int64))
            deq = (u - z[:, None]).astype(np.float64) * s[:, None].astype(np.float64)
            r32 = (x / s[:, None]).astype(np.float32)   # the float32 quotient the codes come from
            unclipped = (np.rint(r32) + z[:, None] >= 0) & (np.rint(r32) + z[:, None] <= qmax)
            # s/2, plus the float32 rounding of the quotient (at most 2^b ulps of 1)
            bound = s[:, None].astype(np.float64) * (0.5 + (1 << bits) * 2.0 ** -23) * np.ones_like(x, dtype=np.float64)
            assert np.all(np.abs(deq - x)[unclipped] <= bound[unclipped])
            if alpha == 1.0:
                assert unclipped.all()
                assert np.all(u.max(axis=1) >= qmax - 1) or np.all(u.min(axis=1) <= 1)
    assert x[5].min() >= 0 and o.minmax_params(x[5:6], 4)[1][0] == 0


def check_asym_symmetric_case(o):
    """b = 4 with z = 8 and the symmetric absmax scale is the symmetric quantizer."""
    g = np.random.Generator(np.random.PCG64(19))
    x = (g.standard_normal((32, 256)) * 3).astype(np.float16).astype(np.float32)
    s = o.scale_row(x, 1.0)
    u = o.quantize_u(x, s, np.full(32, 8), 4).astype(np.int64)
    assert np.array_equal(u - 8, o.quantize(x, s[:, None]).astype(np.int64))


def check_asym_gemm(o):
    """gemm_asym equals the brute-force centred sum on tiny shapes and the
    expansion sum ux uw - zw sum ux - zx sum uw + K zx zw (no cross term dropped)."""
    g = np.random.Generator(np.random.PCG64(23))
    for (m, n, k) in ((1, 1, 1), (3, 5, 7), (4, 6, 256)):
        ux = g.integers(0, 16, (m, k))
        uw = g.integers(0, 16, (n, k))
        zx = g.integers(0, 16, m)
        zw = g.integers(0, 16, n)
        acc = o.gemm_asym(ux, zx, uw, zw)
        for i in range(m):
            for j in range(n):
                assert acc[i, j] == sum((int(ux[i, t]) - int(zx[i])) * (int(uw[j, t]) - int(zw[j])) for t in range(k))
        expand = (ux @ uw.T) - zw[None, :] * ux.sum(1)[:, None] - zx[:, None] * uw.sum(1)[None, :] + k * np.outer(zx, zw)
        assert np.array_equal(acc, expand)


ALL_CHECKS = [
    check_asym_golden,
    check_asym_bounds,
    check_asym_symmetric_case,
    check_asym_gemm,
    check_rtn_golden, check_rtn_bounds, check_pack, check_kron_golden,
    check_kron_explicit, check_function_preservation, check_identity_transform,
    check_flop_count, check_gemm_bruteforce, check_linear_golden,
    check_dequant_bound, check_group_equals_row, check_static_equals_row,
    check_qsm_fold,
]


def mutant(o, **overrides):
    """A copy of the oracle module with some functions replaced."""
    m = types.ModuleType(o.__name__ + "_mutant")
    m.__dict__.update(o.__dict__)
    m.__dict__.update(overrides)
    # functions resolve globals in their own module: rebind them to the copy
    for name, f in list(m.__dict__.items()):
        if isinstance(f, types.FunctionType) and f.__module__ == o.__name__ and name not in overrides:
            m.__dict__[name] = types.FunctionType(f.__code__, m.__dict__, f.__name__, f.__defaults__, f.__closure__)
    for name in overrides:
        f = m.__dict__[name]
        if isinstance(f, types.FunctionType):
            m.__dict__[name] = types.FunctionType(f.__code__, m.__dict__, f.__name__, f.__defaults__, f.__closure__)
    return m


# ------------------------------------------------------------------ residual scaling (S_n)

RES_SCALES = (0.4, 0.4, 1.0, 0.25)


def check_residual_golden(o):
    """Hand-worked tokens in tests/golden/residual_worked.txt (FPTQuant, 伪动态残差缩放)."""
    s = np.array(RES_SCALES, dtype=np.float32)
    for ln in _lines("residual_worked.txt"):
        xs, ss, qs = [p.strip() for p in ln.split("|")]
        x = np.array([float(v) for v in xs.split()], dtype=np.float16)[None, :]
        q, s_n, _ = o.quant_act_residual(x, s)
        assert np.float32(s_n[0]) == np.float32(float(ss)), (ln, s_n[0])
        assert np.array_equal(q[0], np.array([int(v) for v in qs.split()], dtype=np.int8)), (ln, q[0])


def check_residual_invariants(o):
    """S_n is the root-mean-square (mean of x^2 over K, then a square root):
    a token times 2^p has S_n times 2^p and the same codes; the codes
    reconstruct x / S_n within s/2 where unclipped; and the residual-scaled
    codes of a token whose RMS is 1 equal the plain static codes."""
    g = np.random.Generator(np.random.PCG64(21))
    k = 256
    x = (g.standard_normal((32, k)) * g.uniform(0.05, 20, (32, 1))).astype(np.float16)
    s = (g.uniform(0.05, 0.6, k)).astype(np.float32)
    q, s_n, v = o.quant_act_residual(x, s)
    ref = np.sqrt((x.astype(np.float64) ** 2).mean(axis=1))
    assert np.allclose(s_n, ref, rtol=1e-6), "S_n is not the root-mean-square"
    for p in (-3, 2, 5):
        q2, s2, _ = o.quant_act_residual((x.astype(np.float32) * np.float32(2.0 ** p)).astype(np.float16), s)
        assert np.array_equal(q2, q) and np.array_equal(s2, (s_n * np.float32(2.0 ** p)).astype(np.float32))
    un = (q > -8) & (q < 7)
    err = np.abs(v.astype(np.float64) - q.astype(np.float64) * s[None, :].astype(np.float64))
    assert np.all(err[un] <= s[None, :].repeat(32, 0)[un] / 2 * (1 + 1e-6))
    # a token with RMS exactly 1 (entries +-1): the codes are the static codes of x itself
    ones = np.where(g.standard_normal((4, k)) > 0, 1.0, -1.0).astype(np.float16)
    q1, s1, _ = o.quant_act_residual(ones, s)
    assert np.all(s1 == 1.0)
    assert np.array_equal(q1, o.quant_act(ones, o.STATIC, static_scale=s)[0])


def check_residual_exact_sum(o):
    """The sum of squares inside S_n is the exact sum rounded once: checked by
    rational arithmetic on tokens mixing one large entry with many small ones
    (2^30 + 255 * 2^-24 needs 55 bits), where a float64 running or pairwise
    sum drops the small squares."""
    from fractions import Fraction
    g = np.random.Generator(np.random.PCG64(23))
    rows = [np.array([32768.0] + [2.0 ** -12] * 255, np.float16),
            np.array([2.0 ** -12] * 200 + [-32768.0] + [2.0 ** -12] * 55, np.float16),
            (g.standard_normal(256) * np.where(g.uniform(size=256) < 0.02, 4000.0, 0.01)).astype(np.float16)]
    x = np.stack(rows)
    got = o.residual_sumsq(x)
    for i, row in enumerate(x):
        exact = sum(Fraction(float(v)) ** 2 for v in row)
        assert got[i] == float(exact), (i, got[i], float(exact))
    assert np.array_equal(o.residual_rms(x), np.sqrt(got / 256).astype(np.float32))


ALL_CHECKS += [check_residual_golden, check_residual_invariants, check_residual_exact_sum]


# ------------------------------------------------------------------ ternary weights (PT2-LLM ATQ)

def check_ternary_golden(o):
    """Hand-worked ITF rows in tests/golden/ternary_worked.txt (PT2-LLM, ATQ)."""
    from fractions import Fraction
    for ln in _lines("ternary_worked.txt"):
        ws, a_s, m_s, ts, byte = [p.strip() for p in ln.split("|")]
        w = np.array([float(v) for v in ws.split()], dtype=np.float16)[None, :]
        t, a, m = o.ternary_fit(w, iters=10, block=w.shape[1])
        assert np.array_equal(t[0], np.array([int(v) for v in ts.split()], np.int8)), (ln, t)
        assert a[0, 0] == np.float32(float(Fraction(a_s))), (ln, a)
        assert m[0, 0] == np.float32(float(Fraction(m_s))), (ln, m)
        assert int(o.pack_ternary(t)[0, 0]) == int(byte), (ln, o.pack_ternary(t))


def check_ternary_closed_form(o):
    """The closed-form (alpha, mu) for fixed T is the least-squares fit of each
    row by alpha T + mu (numpy lstsq on [T, 1]), including rows with sum(T) != 0."""
    g = np.random.Generator(np.random.PCG64(31))
    w = g.standard_normal((16, 128)) * 0.02 + g.uniform(-0.01, 0.01, (16, 1))
    t = g.integers(-1, 2, (16, 128))
    t[0] = 1  # a constant row: alpha = 0, mu = the mean
    a, m = o.ternary_alpha_mu(w, t)
    for r in range(1, 16):
        sol = np.linalg.lstsq(np.stack([t[r].astype(np.float64), np.ones(128)], 1), w[r], rcond=None)[0]
        assert np.allclose([a[r], m[r]], sol, rtol=1e-10, atol=1e-14), (r, a[r], m[r], sol)
    assert a[0] == 0 and np.isclose(m[0], w[0].mean())


def check_ternary_itf_monotone(o):
    """Each ITF step solves its sub-problem exactly, so the weight error
    ||W - W^||_F never increases with the number of iterations; the fit beats
    the symmetric grid alpha T (mu = 0) on rows with a mean offset."""
    g = np.random.Generator(np.random.PCG64(32))
    w = (g.standard_normal((32, 256)) * 0.02 + g.uniform(-0.02, 0.02, (32, 1))).astype(np.float16)
    w64 = w.astype(np.float64)
    errs = []
    for it in range(0, 11):
        t, a, m = o.ternary_fit(w, iters=it)
        errs.append(((w64 - o.ternary_dequant(t, a.astype(np.float64), m.astype(np.float64))) ** 2).sum())
    assert all(errs[i + 1] <= errs[i] * (1 + 1e-9) for i in range(10)), errs
    t, a, m = o.ternary_fit(w)
    assert set(np.unique(t)) <= {-1, 0, 1}
    sym = ((w64 - np.repeat(a.astype(np.float64), 128, 1) * t) ** 2).sum()
    assert errs[-1] < sym


def check_ternary_linear_loops(o):
    """Y = X (alpha T + mu)^T by plain Python loops on a tiny case (block 4)."""
    g = np.random.Generator(np.random.PCG64(33))
    x = g.standard_normal((2, 8)).astype(np.float16)
    t = g.integers(-1, 2, (3, 8)).astype(np.int8)
    a = g.uniform(0.01, 0.05, (3, 2)).astype(np.float32)
    mu = g.uniform(-0.01, 0.01, (3, 2)).astype(np.float32)
    y = o.ternary_linear(x, t, a, mu, block=4)
    for i in range(2):
        for n in range(3):
            ref = 0.0
            for k in range(8):
                ref += float(x[i, k]) * (float(a[n, k // 4]) * int(t[n, k]) + float(mu[n, k // 4]))
            assert abs(y[i, n] - ref) <= 1e-12 * max(1.0, abs(ref)), (i, n, y[i, n], ref)


ALL_CHECKS += [check_ternary_golden, check_ternary_closed_form, check_ternary_itf_monotone,
               check_ternary_linear_loops]
