"""CPU oracle for the W4A4 quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module: the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
are its only callers.  It shares no code with the CUDA path.

It restates, step by step and in plain numpy, what the pages define:

* the uniform quantizer Q(W) = clamp(round(W/s) + z, 0, 2^b - 1)
  (FRM-PTQ page, section 初步介绍), used symmetric with b = 4 and z = 2^(b-1);
* the per-channel scaling diag(c) placed before the affine transform and the
  clip ratios alpha_w, alpha_a (FlatQuant notes, "额外可学习组件");
* the Kronecker-factored affine transform P = P1 (x) P2 applied to the
  n1 x n2 reshape of a row: activations go through P1^T x1 X x2 P2, weights
  through P1^-1 x1 W x2 (P2^-1)^T (FlatQuant notes, "Kronecker 分解");
* static per-channel activation scales and quantization-step migration into
  the weights (MergeQuant page, 核心思路 / 关键设计);
* group-wise quantization in groups of 128 along K (FRM-PTQ abstract,
  multi-granularity group quantization);
* the INT4 x INT4 product with integer accumulation and the dequantization
  y = acc * s_x * s_w (FlatQuant notes, 核心思想: Y ~ Q(XP) Q(P^-1 W^T));
* the general quantizer (any b, min-max zero point; FRM-PTQ page) and the
  per-token residual scaling S_n ahead of static quantization (FPTQuant
  explainer, 伪动态残差缩放);
* the asymmetric ternary quantizer W^ = alpha T + mu with its iterative
  closed-form fit, and the product of fp16 activations with such weights
  (PT2-LLM page, 非对称三值量化器 ATQ).

Precision: the transform is evaluated in float64 and rounded once to float32
(the "transformed value"); scales, the division and round-half-to-even are
float32 exactly as written; integer products are exact.

Every function carries "parity pinned by" notes naming the CPU tests that
check it against something other than itself.
"""
from __future__ import annotations

import math

import numpy as np

BITS = 4                      # b in Q(W)
ZERO_POINT = 1 << (BITS - 1)  # z = 2^(b-1) = 8: the symmetric case
QMAX_U = (1 << BITS) - 1      # 2^b - 1 = 15
QMAX = QMAX_U - ZERO_POINT    # 7: largest signed code, the scale denominator
QMIN = -ZERO_POINT            # -8
GROUP = 128

ROW, GROUPED, STATIC = 0, 1, 2   # per-token/per-channel, group-128, static per-channel


# ------------------------------------------------------------------ quantizer

def quantize(v32: np.ndarray, s32: np.ndarray) -> np.ndarray:
    """Signed INT4 codes of Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) - z.

    FRM-PTQ page, 初步介绍 (the garbled brackets read as round-to-nearest,
    ties to even; the garbled "2^b?1" read as 2^b - 1).  The division is an
    IEEE float32 division; s = 0 gives code 0.
    Parity pinned by: tests/golden/rtn_worked.txt, the |v - s*q| <= s/2 bound.
    """
    v32 = np.asarray(v32, dtype=np.float32)
    s32 = np.asarray(s32, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = v32 / s32                       # float32 / float32 -> float32
    u = np.clip(np.rint(ratio) + ZERO_POINT, 0, QMAX_U)   # unsigned form of Q(W)
    q = u - ZERO_POINT
    q = np.where(s32 == 0, 0, q)
    return q.astype(np.int8)


def scale_row(v32: np.ndarray, alpha: float) -> np.ndarray:
    """One float32 scale per row: s = (max|v| * alpha) / 7.

    Symmetric absmax scale with the clip ratio alpha (FlatQuant notes,
    "可学习裁剪阈值"); 7 = 2^(b-1) - 1 maps the clipped absmax to the largest code.
    Parity pinned by: tests/golden/rtn_worked.txt.
    """
    amax = np.abs(v32).max(axis=-1).astype(np.float32)
    return (amax * np.float32(alpha)) / np.float32(QMAX)


def scale_group(v32: np.ndarray, alpha: float, group: int = GROUP) -> np.ndarray:
    """One scale per row and group of ``group`` columns, stored in float16.

    Same rule as scale_row on each group (FRM-PTQ multi-granularity group
    quantization); the scale is rounded to float16 before it is used, so
    quantization and dequantization use the same value.
    Returns float32 [rows, K/group] holding float16 values.
    Parity pinned by: the group == row special case, tests/golden/rtn_worked.txt.
    """
    r, k = v32.shape
    amax = np.abs(v32.reshape(r, k // group, group)).max(axis=-1).astype(np.float32)
    s = (amax * np.float32(alpha)) / np.float32(QMAX)
    return s.astype(np.float16).astype(np.float32)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, element 2j in bits 0-3 and 2j+1 in bits 4-7 of byte j.

    Parity pinned by: tests/golden/pack_int4.txt and the round trip over all codes.
    """
    q = np.asarray(q, dtype=np.int16)
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# ------------------------------------------------------------------ general quantizer
#
# Q(W) = clamp(round(W/s) + z, 0, 2^b - 1) for any bit width b and zero point
# z (FRM-PTQ page, 初步介绍), with the asymmetric (min-max) choice of s and z.

def minmax_params(v32: np.ndarray, bits: int, alpha: float = 1.0):
    """Per-row asymmetric scale and zero point.

    The row's range is widened to contain 0 (so that 0 is exactly a code):
    lo = min(0, min v), hi = max(0, max v); s = ((hi - lo) * alpha) / (2^b - 1)
    in float32; z = clamp(round(-lo / s), 0, 2^b - 1) with an IEEE float32
    division and round half to even; a row of zeros has s = 0 and z = 0.
    Returns (s float32 [rows], z int32 [rows]).
    Parity pinned by: tests/golden/rtn_asym_worked.txt, the bound
    |v - s (u - z)| <= s/2 on unclipped values, 0 mapping to z.
    """
    v32 = np.asarray(v32, dtype=np.float32)
    qmax = np.float32((1 << bits) - 1)
    lo = np.minimum(v32.min(axis=-1), np.float32(0))
    hi = np.maximum(v32.max(axis=-1), np.float32(0))
    s = ((hi - lo) * np.float32(alpha)) / qmax        # float32 throughout
    with np.errstate(divide="ignore", invalid="ignore"):
        zf = np.rint(-lo / s)
    z = np.where(s == 0, 0, np.clip(zf, 0, qmax)).astype(np.int32)
    return s.astype(np.float32), z


def quantize_u(v32: np.ndarray, s32: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """Unsigned codes u = clamp(round(v/s) + z, 0, 2^b - 1), one (s, z) per row.

    FRM-PTQ page, 初步介绍; IEEE float32 division, round half to even; s = 0
    gives u = z (the code of 0).
    Parity pinned by: tests/golden/rtn_asym_worked.txt; with b = 4, z = 8 and
    the symmetric scale it equals quantize() + 8.
    """
    v32 = np.asarray(v32, dtype=np.float32)
    s32 = np.asarray(s32, dtype=np.float32).reshape(-1, 1)
    z = np.asarray(z, dtype=np.int64).reshape(-1, 1)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = v32 / s32
    u = np.clip(np.rint(ratio) + z, 0, (1 << bits) - 1)
    u = np.where(s32 == 0, z, u)
    return u.astype(np.uint8)


def gemm_asym(ux: np.ndarray, zx: np.ndarray, uw: np.ndarray, zw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k (ux[m, k] - zx[m]) (uw[n, k] - zw[n]), exact, int64:
    the integer product of the dequantized-up-to-scale codes, so that
    y = fl(fl(acc * s_x[m]) * s_w[n]) as in dequant_row.
    Parity pinned by: brute force on tiny shapes, and its expansion
    sum ux uw - zw sum ux - zx sum uw + K zx zw (the form a kernel computes).
    """
    cx = np.asarray(ux, np.float64) - np.asarray(zx, np.float64).reshape(-1, 1)
    cw = np.asarray(uw, np.float64) - np.asarray(zw, np.float64).reshape(-1, 1)
    return (cx @ cw.T).astype(np.int64)


# ------------------------------------------------------------------ transform

def kron_apply(v64: np.ndarray, left: np.ndarray, right: np.ndarray) -> np.ndarray:
    """Row-wise left @ Xbar @ right, where Xbar is the row-major n1 x n2 reshape.

    Evaluated in float64: first T = left @ Xbar, then T @ right.
    """
    n1, n2 = left.shape[0], right.shape[0]
    r = v64.shape[0]
    xbar = v64.reshape(r, n1, n2)
    t = np.matmul(left.astype(np.float64)[None], xbar)
    out = np.matmul(t, right.astype(np.float64)[None])
    return out.reshape(r, n1 * n2)


def act_transform(x: np.ndarray, p1=None, p2=None, c=None) -> np.ndarray:
    """float64 value of (x * c) (P1 (x) P2) for each token row x.

    The channel scale c multiplies before the transform (FlatQuant notes,
    "逐通道缩放 diag(c)...在仿射变换之前引入"); the transform is
    P1^T x1 Xbar x2 P2 on the n1 x n2 reshape (FlatQuant notes, "Kronecker 分解").
    Parity pinned by: explicit np.kron(P1, P2) product, the worked example in
    tests/golden/kron_worked.txt, function preservation with weight_transform.
    """
    v = np.asarray(x, dtype=np.float64)
    if c is not None:
        v = v * np.asarray(c, dtype=np.float64)[None, :]
    if p1 is not None:
        v = kron_apply(v, np.asarray(p1).T, np.asarray(p2))
    return v


def weight_transform(w: np.ndarray, p1_inv=None, p2_inv=None, c=None) -> np.ndarray:
    """float64 value of P^-1 applied to each weight row (as a column of W^T).

    The weight side divides by c and applies P1^-1 x1 Wbar x2 (P2^-1)^T
    (FlatQuant notes, "Kronecker 分解"); the inverses are the caller's.
    Parity pinned by: explicit np.kron(P1^-1, P2^-1) product and function
    preservation X P P^-1 W^T = X W^T.
    """
    v = np.asarray(w, dtype=np.float64)
    if c is not None:
        v = v / np.asarray(c, dtype=np.float64)[None, :]
    if p1_inv is not None:
        v = kron_apply(v, np.asarray(p1_inv), np.asarray(p2_inv).T)
    return v


# ------------------------------------------------------------------ quant steps

def quant_act(x, gran=ROW, alpha=1.0, p1=None, p2=None, c=None, static_scale=None):
    """Online activation quantization of fp16 rows.

    Returns (codes int8 [M, K], scales, transformed float32 [M, K]) where the
    scales are float32 [M] (ROW), float32-held float16 [M, K/128] (GROUPED) or
    the given static scale float32 [K] (STATIC, MergeQuant page).
    """
    v32 = act_transform(x, p1, p2, c).astype(np.float32)
    if gran == ROW:
        s = scale_row(v32, alpha)
        q = quantize(v32, s[:, None])
    elif gran == GROUPED:
        s = scale_group(v32, alpha)
        q = quantize(v32, np.repeat(s, GROUP, axis=1))
    elif gran == STATIC:
        s = np.asarray(static_scale, dtype=np.float32)
        q = quantize(v32, s[None, :])
    else:
        raise ValueError(gran)
    return q, s, v32


def quant_weight(w, gran=ROW, alpha=1.0, p1_inv=None, p2_inv=None, c=None,
                 qsm_scale=None):
    """Offline weight quantization of fp16 rows W [N, K].

    Steps: divide by c, apply the inverse Kronecker transform (float64), round
    once to float32, fold the static activation scales s_k into the weights
    with one float32 multiply (quantization step migration, MergeQuant page,
    关键设计), then per-output-channel (ROW) or group-128 (GROUPED) scales and
    codes.  Returns (codes int8 [N, K], scales, float32 values quantized).
    """
    v32 = weight_transform(w, p1_inv, p2_inv, c).astype(np.float32)
    if qsm_scale is not None:
        v32 = v32 * np.asarray(qsm_scale, dtype=np.float32)[None, :]
    if gran == ROW:
        s = scale_row(v32, alpha)
        q = quantize(v32, s[:, None])
    elif gran == GROUPED:
        s = scale_group(v32, alpha)
        q = quantize(v32, np.repeat(s, GROUP, axis=1))
    else:
        raise ValueError(gran)
    return q, s, v32


# ------------------------------------------------------------------ residual scaling

def residual_rms(x) -> np.ndarray:
    """S_n = sqrt(sum_k x_k^2 / K) per token, rounded once to float32.

    FPTQuant explainer, 伪动态残差缩放 (S_n): a per-token factor from the
    root-mean-square of the residual stream (RMSNorm applied to the
    residual; the page gives no epsilon, so none is added).  The page fixes
    no summation order, so the sum of squares is taken exactly and rounded
    once to float64 (math.fsum; every square of a float32 value is exact in
    float64), then divided by K and square-rooted in float64 and rounded to
    float32: a result that does not depend on any order of additions.
    Parity pinned by: tests/golden/residual_worked.txt, scaling a token by a
    power of two scaling S_n by the same power, and an exact rational
    evaluation of tokens whose float64 partial sums round.
    """
    return np.sqrt(residual_sumsq(x) / np.asarray(x).shape[1]).astype(np.float32)


def residual_sumsq(x) -> np.ndarray:
    """sum_k x_k^2 per token, exact, rounded once to float64 (the sum inside S_n).

    Parity pinned by: an exact rational evaluation (fractions) of tokens
    whose float64 partial sums round in any order of additions.
    """
    x64 = np.asarray(x, np.float64)
    return np.array([math.fsum(row * row) for row in x64], np.float64)


def quant_act_residual(x, static_scale):
    """Static per-channel INT4 codes of the token divided by its S_n.

    v = fl32(x / S_n) (IEEE float32 division; a token of zeros gives v = 0),
    then the static quantizer of quant_act with the caller's s_k.  The
    per-token factor leaves through the GEMM: a bias-free linear layer
    commutes with per-token scaling, so y = (acc * S_n) * s_w' with the
    static scales migrated into s_w' (MergeQuant quantization step
    migration) restores the unscaled output.
    Returns (codes int8 [M, K], S_n float32 [M], v float32 [M, K]).
    Parity pinned by: tests/golden/residual_worked.txt, invariance of the
    codes under power-of-two token scaling, |x / S_n - s q| <= s/2.
    """
    s_n = residual_rms(x)
    x32 = np.asarray(x, np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s_n[:, None] > 0, x32 / s_n[:, None], np.float32(0)).astype(np.float32)
    q = quantize(v, np.asarray(static_scale, np.float32)[None, :])
    return q, s_n, v


# ------------------------------------------------------------------ GEMM + dequant

def gemm_int(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qx[m, k] * qw[n, k], exact, as int64.

    The matmul runs on float64 holding integers: every product is at most 64
    in magnitude and every partial sum at most 64*K < 2^53, so each float64
    operation is exact whatever the summation order.
    Parity pinned by: the pure-Python triple loop on tiny shapes.
    """
    k = qx.shape[1]
    assert 64 * k < (1 << 53)
    acc = np.asarray(qx, np.float64) @ np.asarray(qw, np.float64).T
    return acc.astype(np.int64)


def dequant_row(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """y = fp16_rne((float32(acc) * s_x[m]) * s_w[n]), two float32 multiplies."""
    assert np.abs(acc).max(initial=0) < (1 << 24)
    a = acc.astype(np.float32)
    y = (a * np.asarray(s_x, np.float32)[:, None]) * np.asarray(s_w, np.float32)[None, :]
    return y.astype(np.float16)


def dequant_static(acc: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """y = fp16_rne(float32(acc) * s_w'[n]) where s_w' already carries the migrated
    activation scales (MergeQuant quantization step migration)."""
    assert np.abs(acc).max(initial=0) < (1 << 24)
    y = acc.astype(np.float32) * np.asarray(s_w, np.float32)[None, :]
    return y.astype(np.float16)


def dequant_group(qx, qw, s_x, s_w) -> np.ndarray:
    """y = fp16_rne(sum_g acc_g * s_x[m, g] * s_w[n, g]) in float64, g ascending,
    where acc_g is the exact integer product over k in [128 g, 128 g + 128).

    s_x [M, K/128] and s_w [N, K/128] hold float16 values.
    Parity pinned by: the single-group case against dequant_row and the
    float64 dequantize-then-multiply bound.
    """
    m, k = qx.shape
    n = qw.shape[0]
    y = np.zeros((m, n), dtype=np.float64)
    for g in range(k // GROUP):
        sl = slice(g * GROUP, (g + 1) * GROUP)
        acc_g = gemm_int(qx[:, sl], qw[:, sl]).astype(np.float64)
        y += acc_g * np.asarray(s_x, np.float64)[:, g:g + 1] * np.asarray(s_w, np.float64)[None, :, g]
    return y.astype(np.float16)


def linear(x, wq, s_w, gran=ROW, alpha=1.0, p1=None, p2=None, c=None,
           static_scale=None):
    """Y = dequant(Q(X P) Q(P^-1 W^T)) for fp16 X [M, K] and weight codes wq [N, K]."""
    qx, s_x, _ = quant_act(x, gran, alpha, p1, p2, c, static_scale)
    if gran == ROW:
        return dequant_row(gemm_int(qx, wq), s_x, s_w)
    if gran == STATIC:
        return dequant_static(gemm_int(qx, wq), s_w)
    return dequant_group(qx, wq, s_x, s_w)


# ------------------------------------------------------------------ ternary weights

TERNARY_BLOCK = 128


def ternary_alpha_mu(w, t):
    """Closed-form (alpha, mu) of one block for a fixed ternary matrix T.

    PT2-LLM page, 非对称三值量化器 ATQ (ITF): with T fixed, the per-row scale
    alpha* = (m (W o T) 1 - (T 1) o (W 1)) / (m (T o T) 1 - (T 1)^2) (m the
    block's column count); it is the least-squares alpha when the offset is
    solved jointly, so the offset is mu* = (W 1 - alpha* T 1) / m.  A row
    whose denominator is 0 (T constant on the row) gets alpha = 0 and mu = the
    row mean (then W^ = mu is that row's least-squares fit).
    w float64 [R, m], t int [R, m] -> (alpha, mu) float64 [R].
    Parity pinned by: least squares on [T, 1] (numpy lstsq) for random blocks.
    """
    w = np.asarray(w, np.float64)
    t = np.asarray(t, np.float64)
    m = w.shape[1]
    num = m * (w * t).sum(1) - t.sum(1) * w.sum(1)
    den = m * (t * t).sum(1) - t.sum(1) ** 2
    ok = den != 0
    alpha = np.where(ok, num / np.where(ok, den, 1.0), 0.0)
    mu = (w.sum(1) - alpha * t.sum(1)) / m
    return alpha, mu


def ternary_round(w, alpha, mu):
    """T_ij = argmin over t in {-1, 0, 1} of |Z_ij - t|, Z = (W - mu) / alpha
    (PT2-LLM page, ITF); ties |Z| = 1/2 go to 0 (round half to even), and a
    row with alpha = 0 gets T = 0."""
    w = np.asarray(w, np.float64)
    a = np.asarray(alpha, np.float64)[:, None]
    z = np.where(a != 0, (w - np.asarray(mu, np.float64)[:, None]) / np.where(a != 0, a, 1.0), 0.0)
    return np.clip(np.rint(z), -1, 1).astype(np.int8)


def ternary_fit(w, iters: int = 10, block: int = TERNARY_BLOCK):
    """Asymmetric ternary quantization of weight rows, per block of 128 columns.

    PT2-LLM page, 非对称三值量化器 ATQ, iterative ternary fitting (ITF): mu
    starts at each row's mean, then `iters` rounds of (T from the current
    grid, then alpha and mu in closed form for that T).  The page gives no
    starting alpha; this takes alpha_0 = 2 mean|W - mu_0| (a ternary threshold
    at mean|W - mu_0|).  Returns (T int8 [N, K], alpha float32 [N, K/block],
    mu float32 [N, K/block]); alpha and mu are the float64 values rounded to
    float32, T is the last rounding's.
    Parity pinned by: the weight error ||W - W^||_F never increasing over the
    iterations, the closed form against least squares, tests/golden/ternary_worked.txt.
    """
    w = np.asarray(w, np.float64)
    n, k = w.shape
    nb = k // block
    t_out = np.zeros((n, k), np.int8)
    a_out = np.zeros((n, nb), np.float32)
    m_out = np.zeros((n, nb), np.float32)
    for g in range(nb):
        wb = w[:, g * block:(g + 1) * block]
        mu = wb.mean(1)
        alpha = 2.0 * np.abs(wb - mu[:, None]).mean(1)
        t = ternary_round(wb, alpha, mu)
        for _ in range(iters):
            alpha, mu = ternary_alpha_mu(wb, t)
            t = ternary_round(wb, alpha, mu)
        alpha, mu = ternary_alpha_mu(wb, t)
        t_out[:, g * block:(g + 1) * block] = t
        a_out[:, g] = alpha.astype(np.float32)
        m_out[:, g] = mu.astype(np.float32)
    return t_out, a_out, m_out


def ternary_dequant(t, alpha, mu, block: int = TERNARY_BLOCK) -> np.ndarray:
    """W^ = alpha T + mu per row and block (PT2-LLM page, ATQ), float64 [N, K]."""
    t = np.asarray(t, np.float64)
    a = np.repeat(np.asarray(alpha, np.float64), block, axis=1)
    m = np.repeat(np.asarray(mu, np.float64), block, axis=1)
    return a * t + m


def ternary_linear(x, t, alpha, mu, block: int = TERNARY_BLOCK) -> np.ndarray:
    """Y = X W^T with W^ = alpha T + mu and fp16 activations X [M, K], in
    float64 (the product as defined; weight-only ternarization keeps the
    activations in fp16).  Returns float64 [M, N].
    Parity pinned by: pure-Python loops over a tiny case.
    """
    return np.asarray(x, np.float64) @ ternary_dequant(t, alpha, mu, block).T


def pack_ternary(t) -> np.ndarray:
    """Ternary codes packed 4 per byte, low bits first: 2 bits per weight,
    00 = 0, 01 = +1, 11 = -1 (bit 0: nonzero, bit 1: negative).
    int8 [N, K] -> uint8 [N, K/4].  (T carries log2(3) = 1.58 bits of
    information per weight; the stored width is 2 bits.)
    Parity pinned by: hand-packed bytes in tests/golden/ternary_worked.txt."""
    t = np.asarray(t, np.int64)
    code = np.where(t == 0, 0, np.where(t > 0, 1, 3))
    n, k = t.shape
    c = code.reshape(n, k // 4, 4)
    return (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)


# ------------------------------------------------------------------ sampled rows

def linear_rows(rows, x, wq, s_w, **kw):
    """The rows ``rows`` of linear(...): every step above is row-independent."""
    rows = np.asarray(rows)
    return linear(np.asarray(x)[rows], wq, s_w, **kw)


# ------------------------------------------------------------------ counts

def kron_flops(n1: int, n2: int) -> int:
    """Multiply-adds x2 per row for P1^T Xbar P2: 2 n (n1 + n2), n = n1 n2
    (FlatQuant notes: computation saving sqrt(n)/2 against a dense n x n P)."""
    n = n1 * n2
    return 2 * n * (n1 + n2)


def dense_transform_flops(n: int) -> int:
    return 2 * n * n
