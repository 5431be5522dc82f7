"""The CPU oracle against hand-worked examples, closed forms, invariants and
brute force (see tests/pins.py), plus planted mistakes that must be caught."""
import numpy as np
import pytest

import pins
from oracle import fq_oracle as O


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(O)


# ---- planted mistakes: each plausible slip in one step must fail some pin

def _act_transform_untransposed(x, p1=None, p2=None, c=None):
    v = np.asarray(x, dtype=np.float64)
    if c is not None:
        v = v * np.asarray(c, dtype=np.float64)[None, :]
    if p1 is not None:
        v = kron_apply(v, np.asarray(p1), np.asarray(p2))  # noqa: F821 (mutant globals)
    return v


def _weight_transform_untransposed(w, p1_inv=None, p2_inv=None, c=None):
    v = np.asarray(w, dtype=np.float64)
    if c is not None:
        v = v / np.asarray(c, dtype=np.float64)[None, :]
    if p1_inv is not None:
        v = kron_apply(v, np.asarray(p1_inv), np.asarray(p2_inv))  # noqa: F821
    return v


def _weight_transform_c_times(w, p1_inv=None, p2_inv=None, c=None):
    v = np.asarray(w, dtype=np.float64)
    if c is not None:
        v = v * np.asarray(c, dtype=np.float64)[None, :]
    if p1_inv is not None:
        v = kron_apply(v, np.asarray(p1_inv), np.asarray(p2_inv).T)  # noqa: F821
    return v


def _kron_apply_swapped(v64, left, right):
    n1, n2 = left.shape[0], right.shape[0]
    xbar = v64.reshape(v64.shape[0], n1, n2)
    out = np.matmul(np.matmul(left[None], xbar), right.T[None])
    return out.reshape(v64.shape[0], n1 * n2)


def _quantize_half_away(v32, s32):
    v32 = np.asarray(v32, np.float32)
    s32 = np.asarray(s32, np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = v32 / s32
    q = np.clip(np.sign(r) * np.floor(np.abs(r) + 0.5), -8, 7)
    return np.where(s32 == 0, 0, q).astype(np.int8)


def _quantize_no_minus8(v32, s32):
    v32 = np.asarray(v32, np.float32)
    s32 = np.asarray(s32, np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = v32 / s32
    q = np.clip(np.rint(r), -7, 7)
    return np.where(s32 == 0, 0, q).astype(np.int8)


def _scale_row_over8(v32, alpha):
    amax = np.abs(v32).max(axis=-1).astype(np.float32)
    return (amax * np.float32(alpha)) / np.float32(8)


def _scale_group_fp32(v32, alpha, group=128):
    r, k = v32.shape
    amax = np.abs(v32.reshape(r, k // group, group)).max(axis=-1).astype(np.float32)
    return (amax * np.float32(alpha)) / np.float32(7)


def _pack_swapped(q):
    q = np.asarray(q, dtype=np.int16)
    return ((q[..., 1::2] & 0xF) | ((q[..., 0::2] & 0xF) << 4)).astype(np.uint8)


def _gemm_drop_last(qx, qw):
    return (np.asarray(qx[:, :-1], np.float64) @ np.asarray(qw[:, :-1], np.float64).T).astype(np.int64)


def _dequant_row_sx_twice(acc, s_x, s_w):
    a = acc.astype(np.float32)
    sx = np.asarray(s_x, np.float32)
    return ((a * sx[:, None]) * sx[:1][None, :] * np.ones_like(np.asarray(s_w, np.float32))[None, :]).astype(np.float16)


def _dequant_group_shifted(qx, qw, s_x, s_w):
    m, k = qx.shape
    y = np.zeros((m, qw.shape[0]))
    ng = k // 128
    for g in range(ng):
        sl = slice(g * 128, (g + 1) * 128)
        acc_g = gemm_int(qx[:, sl], qw[:, sl]).astype(np.float64)  # noqa: F821
        h = (g + 1) % ng
        y += acc_g * np.asarray(s_x, np.float64)[:, g:g + 1] * np.asarray(s_w, np.float64)[None, :, h]
    return y.astype(np.float16)


def _quant_weight_qsm_rows(w, gran=0, alpha=1.0, p1_inv=None, p2_inv=None, c=None, qsm_scale=None):
    v32 = weight_transform(w, p1_inv, p2_inv, c).astype(np.float32)  # noqa: F821
    if qsm_scale is not None:
        q = np.asarray(qsm_scale, np.float32)
        v32 = v32 * q[:v32.shape[0], None]
    s = scale_row(v32, alpha)  # noqa: F821
    return quantize(v32, s[:, None]), s, v32  # noqa: F821


def _minmax_no_zero(v32, bits, alpha=1.0):
    # range not widened to contain 0
    v32 = np.asarray(v32, dtype=np.float32)
    qmax = np.float32((1 << bits) - 1)
    lo, hi = v32.min(axis=-1), v32.max(axis=-1)
    s = ((hi - lo) * np.float32(alpha)) / qmax
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s == 0, 0, np.clip(np.rint(-lo / s), 0, qmax)).astype(np.int32)
    return s.astype(np.float32), z


def _minmax_zero_sign(v32, bits, alpha=1.0):
    # zero point from +lo instead of -lo
    v32 = np.asarray(v32, dtype=np.float32)
    qmax = np.float32((1 << bits) - 1)
    lo = np.minimum(v32.min(axis=-1), np.float32(0))
    hi = np.maximum(v32.max(axis=-1), np.float32(0))
    s = ((hi - lo) * np.float32(alpha)) / qmax
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s == 0, 0, np.clip(np.rint(lo / s), 0, qmax)).astype(np.int32)
    return s.astype(np.float32), z


def _gemm_asym_no_cross(ux, zx, uw, zw):
    # the K zx zw term dropped
    ux, uw = np.asarray(ux, np.int64), np.asarray(uw, np.int64)
    zx, zw = np.asarray(zx, np.int64), np.asarray(zw, np.int64)
    return ux @ uw.T - zw[None, :] * ux.sum(1)[:, None] - zx[:, None] * uw.sum(1)[None, :]


def _residual_rms_no_mean(x):
    # sum of squares without the division by K
    x64 = np.asarray(x, np.float64)
    return np.sqrt((x64 * x64).sum(axis=1)).astype(np.float32)


def _residual_rms_no_sqrt(x):
    # mean square instead of its root
    x64 = np.asarray(x, np.float64)
    return ((x64 * x64).sum(axis=1) / x64.shape[1]).astype(np.float32)


def _residual_sumsq_pairwise(x):
    # float64 numpy sum (order-dependent rounding) instead of the exact sum
    x64 = np.asarray(x, np.float64)
    return (x64 * x64).sum(axis=1)


def _quant_act_residual_times(x, static_scale):
    # the token multiplied by S_n instead of divided
    s_n = residual_rms(x)  # noqa: F821
    v = (np.asarray(x, np.float32) * s_n[:, None]).astype(np.float32)
    return quantize(v, np.asarray(static_scale, np.float32)[None, :]), s_n, v  # noqa: F821


def _ternary_alpha_mu_no_m(w, t):
    # the factor m dropped from the numerator of alpha*
    w = np.asarray(w, np.float64)
    t = np.asarray(t, np.float64)
    m = w.shape[1]
    num = (w * t).sum(1) - t.sum(1) * w.sum(1)
    den = m * (t * t).sum(1) - t.sum(1) ** 2
    alpha = np.where(den != 0, num / np.where(den != 0, den, 1.0), 0.0)
    return alpha, (w.sum(1) - alpha * t.sum(1)) / m


def _ternary_alpha_mu_mu_sign(w, t):
    # mu with the alpha T term added instead of subtracted
    w = np.asarray(w, np.float64)
    t = np.asarray(t, np.float64)
    m = w.shape[1]
    num = m * (w * t).sum(1) - t.sum(1) * w.sum(1)
    den = m * (t * t).sum(1) - t.sum(1) ** 2
    alpha = np.where(den != 0, num / np.where(den != 0, den, 1.0), 0.0)
    return alpha, (w.sum(1) + alpha * t.sum(1)) / m


def _ternary_round_floor(w, alpha, mu):
    # floor instead of nearest
    a = np.asarray(alpha, np.float64)[:, None]
    z = np.where(a != 0, (np.asarray(w, np.float64) - np.asarray(mu, np.float64)[:, None]) / np.where(a != 0, a, 1.0), 0.0)
    return np.clip(np.floor(z), -1, 1).astype(np.int8)


def _ternary_linear_no_mu(x, t, alpha, mu, block=128):
    # the offset term dropped
    a = np.repeat(np.asarray(alpha, np.float64), block, axis=1)
    return np.asarray(x, np.float64) @ (a * np.asarray(t, np.float64)).T


def _pack_ternary_swapped(t):
    # the two code bits swapped (bit 0 negative, bit 1 nonzero)
    t = np.asarray(t, np.int64)
    code = np.where(t == 0, 0, np.where(t > 0, 2, 3))
    n, k = t.shape
    c = code.reshape(n, k // 4, 4)
    return (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)


MUTANTS = {
    "ternary_alpha_without_m": dict(ternary_alpha_mu=_ternary_alpha_mu_no_m),
    "ternary_mu_sign": dict(ternary_alpha_mu=_ternary_alpha_mu_mu_sign),
    "ternary_round_floor": dict(ternary_round=_ternary_round_floor),
    "ternary_linear_without_mu": dict(ternary_linear=_ternary_linear_no_mu),
    "ternary_pack_bits_swapped": dict(pack_ternary=_pack_ternary_swapped),
    "residual_rms_without_mean": dict(residual_rms=_residual_rms_no_mean),
    "residual_rms_without_sqrt": dict(residual_rms=_residual_rms_no_sqrt),
    "residual_multiplied": dict(quant_act_residual=_quant_act_residual_times),
    "residual_sum_rounded_per_add": dict(residual_sumsq=_residual_sumsq_pairwise),
    "asym_range_without_zero": dict(minmax_params=_minmax_no_zero),
    "asym_zero_point_sign": dict(minmax_params=_minmax_zero_sign),
    "asym_gemm_drops_cross_term": dict(gemm_asym=_gemm_asym_no_cross),
    "act_P1_not_transposed": dict(act_transform=_act_transform_untransposed),
    "weight_P2inv_not_transposed": dict(weight_transform=_weight_transform_untransposed),
    "weight_c_multiplied": dict(weight_transform=_weight_transform_c_times),
    "kron_right_transposed": dict(kron_apply=_kron_apply_swapped),
    "round_half_away": dict(quantize=_quantize_half_away),
    "clamp_without_minus8": dict(quantize=_quantize_no_minus8),
    "scale_over_8": dict(scale_row=_scale_row_over8),
    "group_scale_not_fp16": dict(scale_group=_scale_group_fp32),
    "nibbles_swapped": dict(pack_int4=_pack_swapped),
    "gemm_drops_a_term": dict(gemm_int=_gemm_drop_last),
    "dequant_wrong_scale_index": dict(dequant_row=_dequant_row_sx_twice),
    "dequant_group_wrong_group": dict(dequant_group=_dequant_group_shifted),
    "qsm_fold_on_rows": dict(quant_weight=_quant_weight_qsm_rows),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_oracle_mutant_is_caught(name):
    m = pins.mutant(O, **MUTANTS[name])
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(m)
        except Exception:
            failed.append(check.__name__)
    assert failed, f"planted mistake {name} passed every pin"
