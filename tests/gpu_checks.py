"""Comparison rules shared by the GPU parity tests.

Bars (written out here, used by every GPU test):
* integer and byte results (codes, packed bytes, int32 accumulators) and
  everything computed without the transform: bit-exact;
* transformed values: |gpu - oracle| <= 1e-4 * (largest |value| of the
  quantization unit, i.e. the row, or the 128-group in group mode);
* codes of transformed values: equal, except where the oracle's v/s lies so
  close to a rounding tie that the value tolerance and the observed scale
  difference can move it across (the "boundary-exempt" elements); there the
  codes may differ by one;
* fp16 outputs: within 1 fp16 ulp; for the group epilogue's float32 sum also
  within (K/128) * 2^-23 * sum_g |term_g| where the terms cancel; for outputs
  whose activation codes had boundary-exempt elements, plus one code unit per
  exempt element and the scale tolerance.
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


def unit_amax(v32, gran):
    """Largest |value| of each element's quantization unit, broadcast to v's shape."""
    a = np.abs(v32.astype(np.float64))
    if gran == O.GROUPED:
        r, k = a.shape
        g = a.reshape(r, k // O.GROUP, O.GROUP).max(axis=2)
        return np.repeat(g, O.GROUP, axis=1)
    return np.broadcast_to(a.max(axis=1, keepdims=True), a.shape)


def check_values(v_gpu, v_ref, gran):
    """Transformed values within 1e-4 of the unit's absmax; returns the max ratio."""
    tol = TOL_REL * unit_amax(v_ref, gran)
    err = np.abs(v_gpu.astype(np.float64) - v_ref.astype(np.float64))
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} transformed values off by more than 1e-4 of their unit's absmax"
    return float((err / np.maximum(tol, 1e-30)).max() * TOL_REL)


def scale_full(s, gran, k):
    s = np.asarray(s, np.float64)
    if gran == O.ROW:
        return np.repeat(s[:, None], k, axis=1)
    if gran == O.GROUPED:  # [rows, K/128]
        return np.repeat(s, O.GROUP, axis=1)
    return np.broadcast_to(s[None, :], (1, k))


def exempt_mask(v_ref, s_ref, s_gpu, gran):
    """Elements whose oracle code may legitimately differ (see module docstring)."""
    r, k = v_ref.shape
    sr = scale_full(s_ref, gran, k)
    sg = scale_full(s_gpu, gran, k)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(sr > 0, v_ref.astype(np.float64) / sr, 0.0)
        tol_v = TOL_REL * unit_amax(v_ref, gran)
        ds = np.where(sr > 0, np.abs(sg - sr) / sr, 0.0)
        margin = np.where(sr > 0, tol_v / sr, 0.0) + np.abs(ratio) * ds + 1e-6
    frac = ratio - np.floor(ratio)
    dist = np.abs(frac - 0.5)
    return dist <= margin


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
