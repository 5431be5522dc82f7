"""Comparison rules shared by the GPU parity tests.

Bars (written out here, used by every GPU test):
* integer and byte results (codes, packed bytes, int32 accumulators) and
  everything computed without the transform: bit-exact;
* transformed values v (the float32 X-hat the kernel quantized):
  |gpu - oracle| <= 1e-4 * max(|v|, 2^-10 * amax_row), amax_row the largest
  |v| of the token row (the oracle's value);
* scales of transformed rows: within 1e-4 relative of the oracle's (per row),
  or equal / one fp16 step apart at an fp16 rounding midpoint (per group);
  and bit-exactly the scale of the GPU's own transformed values;
* codes of transformed values: bit-exactly the round-half-even codes of the
  GPU's own transformed values and scales; against the oracle's codes equal,
  except where the oracle's v/s lies within 1e-4 * |v/s| (plus the measured
  relative scale difference times |v/s|) of a rounding tie, where they may
  differ by one ("boundary-exempt"; the count is reported);
* GEMM outputs, decoupled from the quantization: the GPU's own codes and
  scales fed to the oracle's integer GEMM and dequantization give the GPU's
  fp16 outputs bit-exactly (per token / static), or within 1 fp16 ulp of the
  oracle's float64 sum (group), except where the float32 sum of the group
  terms cancels, where (K/128) * 2^-23 * sum_g |term_g| also passes and the
  count of such outputs is reported.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import fq_oracle as O

TOL_REL = 1e-4


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    return t.detach().cpu().numpy()


def unpack(p):
    return O.unpack_int4(p)


def ulp16(y):
    return np.spacing(np.abs(np.asarray(y, np.float64)).astype(np.float16)).astype(np.float64)


def row_amax(v32):
    """Largest |value| of each element's token row, broadcast to v's shape."""
    a = np.abs(np.asarray(v32, np.float64))
    return np.broadcast_to(a.max(axis=1, keepdims=True), a.shape)


def check_values(v_gpu, v_ref, gran=None):
    """Transformed values within 1e-4 * max(|v|, 2^-10 * amax_row); returns
    the largest |dv| / max(|v|, 2^-10 amax_row) seen."""
    vr = np.asarray(v_ref, np.float64)
    scale = np.maximum(np.abs(vr), 2.0 ** -10 * row_amax(vr))
    err = np.abs(np.asarray(v_gpu, np.float64) - vr)
    bad = err > TOL_REL * scale
    assert not bad.any(), (f"{bad.sum()} transformed values off by more than 1e-4 * max(|v|, 2^-10 amax_row) "
                           f"(worst ratio {float((err / np.maximum(scale, 1e-300)).max()):.3g})")
    return float((err / np.maximum(scale, 1e-300)).max())


def scale_full(s, gran, k):
    s = np.asarray(s, np.float64)
    if gran == O.ROW:
        return np.repeat(s[:, None], k, axis=1)
    if gran == O.GROUPED:  # [rows, K/128]
        return np.repeat(s, O.GROUP, axis=1)
    return np.broadcast_to(s[None, :], (1, k))


def exempt_mask(v_ref, s_ref, s_gpu, gran):
    """Elements whose oracle code may differ by one: the oracle's r = v/s lies
    within 1e-4 * |r| + |r| * |s_gpu - s_ref| / s_ref of a rounding tie."""
    r_, k = v_ref.shape
    sr = scale_full(s_ref, gran, k)
    sg = scale_full(s_gpu, gran, k)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(sr > 0, v_ref.astype(np.float64) / sr, 0.0)
        ds = np.where(sr > 0, np.abs(sg - sr) / sr, 0.0)
    margin = np.abs(ratio) * (TOL_REL + ds)
    dist = np.abs(ratio - (np.floor(ratio) + 0.5))
    return dist <= margin


def check_own_codes(q_gpu, v_gpu, s_gpu, gran):
    """The kernel's codes are exactly the round-half-even codes of its own
    transformed values and scales (float32 IEEE division, as the oracle's
    quantize)."""
    k = v_gpu.shape[1]
    if gran == O.ROW:
        s = np.asarray(s_gpu, np.float32)[:, None]
    else:
        s = np.repeat(np.asarray(s_gpu, np.float32), O.GROUP, axis=1)
    q_own = O.quantize(np.asarray(v_gpu, np.float32), s)
    bad = q_own != q_gpu
    assert not bad.any(), f"{bad.sum()} codes differ from the codes of the kernel's own transformed values"


def check_own_scales(s_gpu, v_gpu, gran, alpha):
    """The kernel's scales are exactly the scale rule applied to its own transformed values."""
    v = np.asarray(v_gpu, np.float32)
    own = O.scale_row(v, alpha) if gran == O.ROW else O.scale_group(v, alpha)
    assert np.array_equal(np.asarray(s_gpu, np.float32), own.astype(np.float32)), \
        "scales differ from the scale rule applied to the kernel's own transformed values"


def check_codes(q_gpu, q_ref, exempt):
    """Codes equal outside the exempt set, and within one inside it."""
    diff = q_gpu.astype(np.int16) - q_ref.astype(np.int16)
    bad = (diff != 0) & ~exempt
    assert not bad.any(), f"{bad.sum()} codes differ away from a rounding boundary"
    assert np.abs(diff).max(initial=0) <= 1
    return int(exempt.sum()), int((diff != 0).sum())


def check_scales_row(s_gpu, s_ref):
    s_gpu = np.asarray(s_gpu, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    assert np.all(np.abs(s_gpu - s_ref) <= TOL_REL * s_ref), "per-row scales differ by more than 1e-4"


def check_scales_group(s_gpu, s_ref, v_ref, alpha):
    """fp16 group scales: equal, or one fp16 step apart where the oracle's
    unrounded scale sits within 1e-4 of the rounding midpoint."""
    s_gpu = np.asarray(s_gpu, np.float32)
    s_ref = np.asarray(s_ref, np.float32)
    r, k = v_ref.shape
    amax = np.abs(v_ref.reshape(r, k // O.GROUP, O.GROUP)).max(axis=2).astype(np.float32)
    raw = ((amax * np.float32(alpha)) / np.float32(7)).astype(np.float64)
    diff = s_gpu != s_ref
    if diff.any():
        mid = (s_gpu.astype(np.float64) + s_ref.astype(np.float64)) / 2
        near = np.abs(raw - mid) <= 2 * TOL_REL * raw
        step = np.abs(s_gpu.astype(np.float64) - s_ref.astype(np.float64)) <= ulp16(s_ref) * 1.0001
        assert np.all((near & step)[diff]), "group scales differ away from an fp16 rounding midpoint"
    return int(diff.sum())


def check_fp16_exact(y_gpu, y_ref):
    a = np.asarray(y_gpu).view(np.uint16)
    b = np.asarray(y_ref).view(np.uint16)
    bad = a != b
    # +0 and -0 are the same value
    bad &= ~((np.asarray(y_gpu) == 0) & (np.asarray(y_ref) == 0))
    assert not bad.any(), f"{bad.sum()} fp16 outputs differ (first at {np.argwhere(bad)[:3].tolist()})"


def check_fp16_group(y_gpu, qx, qw, sx_g, sw_g):
    """Group epilogue: 1 fp16 ulp, or the float32 cancellation bound.
    sx_g [M, K/128], sw_g [N, K/128] hold fp16 values."""
    ref = O.dequant_group(qx, qw, sx_g, sw_g).astype(np.float64)
    m, k = qx.shape
    absum = np.zeros((m, qw.shape[0]))
    for g in range(k // O.GROUP):
        sl = slice(g * O.GROUP, (g + 1) * O.GROUP)
        acc = O.gemm_int(qx[:, sl], qw[:, sl]).astype(np.float64)
        absum += np.abs(acc * sx_g[:, g:g + 1].astype(np.float64) * sw_g[None, :, g].astype(np.float64))
    err = np.abs(np.asarray(y_gpu, np.float64) - ref)
    ok = (err <= ulp16(ref)) | (err <= (k // O.GROUP) * 2.0 ** -23 * absum + ulp16(ref))
    assert ok.all(), f"{(~ok).sum()} group outputs beyond 1 ulp (max err {err.max()})"
    return int((err > ulp16(ref)).sum())


def tile_samples(seed, extent, block=128, per_block=2):
    """Sorted indices with `per_block` seeded draws inside every `block`-wide
    block of [0, extent), plus 0 and extent - 1: every output tile position
    of the GEMM (128 x 256 or 256 x 256 tiles) is hit at least once."""
    g = np.random.Generator(np.random.PCG64(seed))
    idx = [0, extent - 1]
    for b0 in range(0, extent, block):
        b1 = min(extent, b0 + block)
        idx.extend(g.integers(b0, b1, per_block).tolist())
    return np.unique(np.asarray(idx))


def check_gemm_decoupled(y_gpu, qx, sx, qw, sw, gran):
    """The GPU's fp16 outputs against the oracle's integer GEMM and
    dequantization of the GPU's OWN activation codes and scales (so the
    quantization tolerance never enters the GEMM check).
    qx [m, K] int8, qw [n, K] int8; sx float32 [m] (ROW), ignored (STATIC) or
    float32-held fp16 [m, K/128] (GROUPED); sw float32 [n] or [n, K/128].
    Returns the number of group outputs that needed the cancellation bound."""
    if gran == O.ROW:
        check_fp16_exact(y_gpu, O.dequant_row(O.gemm_int(qx, qw), sx, sw))
        return 0
    if gran == O.STATIC:
        check_fp16_exact(y_gpu, O.dequant_static(O.gemm_int(qx, qw), sw))
        return 0
    return check_fp16_group(y_gpu, qx, qw, sx, sw)
