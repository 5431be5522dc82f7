"""The ternary-weight linear layer on the GPU (PT2-LLM page, 非对称三值量化器
ATQ: W^ = alpha T + mu per row and 128-column block, fp16 activations)
against the oracle's pack_ternary and ternary_linear.

Packing is integer work and is compared bit-exactly.  The product is float32
arithmetic in the kernel's own order against the float64 definition, so
each output must lie within 1 fp16 ulp of the exact value plus a float32
accumulation bound derived from the summation, each rounding at most 2^-24
of B = sum_k |x_k| (|alpha t_k| + |mu|).  Per-token tables of pair sums
(M <= 16, K <= 32768): a partial sum passes through 1 (the table entry) + 16
(a lane's 32 lookups in two float32 lanes) + 3 (alpha) + 8 (the offset term's
block sum) + 5 (the warp) + 8 (the cluster's slices) roundings.  Direct
kernel: 16 (a 16-weight word) + K/512 (a lane's words) + 5 (the warp
reduction) + 8 + K/4096 (the block sums of the offset term).  The test
allows (K/16 + 160) 2^-24 B.
"""
import numpy as np
import pytest
import torch

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def _check_close(y, x, t, alpha, mu, rows=None, cols=None):
    x = x if rows is None else x[rows]
    tt, aa, mm = (t, alpha, mu) if cols is None else (t[cols], alpha[cols], mu[cols])
    ref = O.ternary_linear(x, tt, aa, mm)
    k = x.shape[1]
    bound = np.abs(x.astype(np.float64)) @ (np.abs(O.ternary_dequant(tt, aa, mm) - np.repeat(mm, 128, 1)) +
                                             np.abs(np.repeat(mm.astype(np.float64), 128, 1))).T
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    tol = ulp + (k / 16 + 160) * 2.0 ** -24 * bound
    err = np.abs(y.astype(np.float64) - ref)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} outputs beyond the bound; worst err/tol {(err / tol).max():.3f}"
    return float((err / tol).max())


@pytest.mark.parametrize("n,k", [(8, 16), (3, 1024), (200, 4096), (1000, 28672)])
def test_ternary_pack_exact(n, k):
    g = synth.generator(n + k)
    t = g.integers(-1, 2, (n, k)).astype(np.int8)
    tq = C.host(fq.fq_ternary_pack(C.dev(t)))
    assert np.array_equal(tq, O.pack_ternary(t))
    fq.fq_check_device_error()


@pytest.mark.parametrize("m", [1, 3, 8, 13, 64])
@pytest.mark.parametrize("k,n", [(128, 8), (1024, 203), (4096, 1024)])
def test_ternary_linear_small(m, k, n):
    """Ragged token groups (m = 3, 13: a partial group of 8), N not a
    multiple of the 8 rows of a CTA, one 128-block; every output checked."""
    d = synth.ternary_linear(m, k, n, seed=m * 7 + k + n)
    tq = fq.fq_ternary_pack(C.dev(d["t"]))
    y = C.host(fq.fq_ternary_linear(C.dev(d["x"]), tq, C.dev(d["alpha"]), C.dev(d["mu"])))
    _check_close(y, d["x"], d["t"], d["alpha"], d["mu"])
    fq.fq_check_device_error()


@pytest.mark.parametrize("m", [1, 8])
@pytest.mark.parametrize("k,n", synth.TERNARY_SHAPES)
def test_ternary_linear_decode_full(m, k, n):
    """The benchmark's decode shapes in the benchmark's launch; outputs on
    columns sampled so that every 128-row stretch of the weights is hit."""
    d = synth.ternary_linear(m, k, n)
    tq = fq.fq_ternary_pack(C.dev(d["t"]))
    assert np.array_equal(C.host(tq)[:64], O.pack_ternary(d["t"][:64]))
    y = C.host(fq.fq_ternary_linear(C.dev(d["x"]), tq, C.dev(d["alpha"]), C.dev(d["mu"])))
    cols = C.tile_samples(m + k + n, n)
    worst = _check_close(y[:, cols], d["x"], d["t"], d["alpha"], d["mu"], cols=cols)
    print(f"{d['name']}: {len(cols)} columns, worst err / bound {worst:.3f}")
    fq.fq_check_device_error()


@pytest.mark.parametrize("m,k,n", [
    (2, 8192, 20000),   # tables, two K slices, several 256-row chunks per cluster
    (1, 32768, 300),    # tables, the largest cluster (8 slices)
    (16, 4224, 130),    # tables, the most tokens; a 33-block K in two ragged slices
    (1, 12288, 5),      # tables, three slices, fewer rows than clusters
    (17, 1024, 77),     # direct kernel: more tokens than the tables take
    (1, 32896, 50),     # direct kernel: K beyond 8 slices of 4096
])
def test_ternary_linear_paths(m, k, n):
    """Both kernels and the edges between them; every output checked below
    10000 rows, above that columns hitting every 128-row stretch."""
    d = synth.ternary_linear(m, k, n, seed=m + k + n)
    tq = fq.fq_ternary_pack(C.dev(d["t"]))
    y = C.host(fq.fq_ternary_linear(C.dev(d["x"]), tq, C.dev(d["alpha"]), C.dev(d["mu"])))
    if n < 10000:
        _check_close(y, d["x"], d["t"], d["alpha"], d["mu"])
    else:
        cols = C.tile_samples(m + k + n, n)
        _check_close(y[:, cols], d["x"], d["t"], d["alpha"], d["mu"], cols=cols)
    fq.fq_check_device_error()


def test_ternary_linear_repeatable():
    """The summation order is fixed: two launches give the same bits."""
    d = synth.ternary_linear(8, 8192, 4096, seed=11)
    tq = fq.fq_ternary_pack(C.dev(d["t"]))
    args = (C.dev(d["x"]), tq, C.dev(d["alpha"]), C.dev(d["mu"]))
    y1 = C.host(fq.fq_ternary_linear(*args))
    y2 = C.host(fq.fq_ternary_linear(*args))
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    fq.fq_check_device_error()


def test_ternary_zero_weights_and_tokens():
    """T = 0 leaves y = sum_g mu S_g; zero tokens give y = 0."""
    m, k, n = 4, 512, 64
    d = synth.ternary_linear(m, k, n, seed=5)
    d["t"][:] = 0
    d["x"][1] = 0
    tq = fq.fq_ternary_pack(C.dev(d["t"]))
    y = C.host(fq.fq_ternary_linear(C.dev(d["x"]), tq, C.dev(d["alpha"]), C.dev(d["mu"])))
    _check_close(y, d["x"], d["t"], d["alpha"], d["mu"])
    assert not y[1].any()
    fq.fq_check_device_error()
