"""Seeded synthetic workloads for the W4A4 linear layer.

This module only draws numbers: it holds none of the layer's arithmetic
(no transform, no scale, no rounding to codes, no GEMM).  Both the CPU oracle
and the CUDA path receive the arrays built here.

Shapes follow the LLaMA-family layers the pages quantize (FlatQuant notes,
"Transformer 集成"; MergeQuant, "实验亮点": Llama-2-7B/70B; FRM-PTQ, "实验设置"):
the pages measure on WikiText-2 / C4 activations of trained models, which are
not available here, so these seeded Gaussian / Student-t tensors with planted
outlier channels and a pivot token stand in for them.

Every tensor is drawn in float64 from ``numpy.random.Generator(PCG64(seed))``
in the order stated in each builder's docstring, then cast to float16
(round-to-nearest-even) or float32.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
_CHUNK = 1 << 22  # elements drawn per call; the stream is consumed in order


def generator(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _draw(g: np.random.Generator, shape, kind: str, scale: float, df: float = 5.0,
          col_scale: np.ndarray | None = None, row_scale: np.ndarray | None = None,
          dtype=np.float16) -> np.ndarray:
    """Draw ``shape`` values row-chunk by row-chunk (same stream order as one call)."""
    rows, cols = shape
    out = np.empty((rows, cols), dtype=dtype)
    step = max(1, _CHUNK // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        if kind == "normal":
            v = g.standard_normal((r1 - r0, cols))
        elif kind == "t":
            v = g.standard_t(df, (r1 - r0, cols))
        else:
            raise ValueError(kind)
        v *= scale
        if col_scale is not None:
            v *= col_scale[None, :]
        if row_scale is not None:
            v *= row_scale[r0:r1, None]
        out[r0:r1] = v.astype(dtype)
    return out


def kron_factors(k: int) -> tuple[int, int]:
    """(n1, n2) with n1*n2 = k and the smallest n1 + n2 (FlatQuant notes,
    "Kronecker 分解": the pair with the least n1 + n2, e.g. 8192 -> (64, 128)).

    Reading: n2 is kept at most 128 so that one row of the n1 x n2 tile never
    straddles a 128-wide quantization group; ties go to the larger n2.
    """
    best = None
    for n2 in range(1, 129):
        if k % n2:
            continue
        n1 = k // n2
        key = (n1 + n2, -n2)
        if best is None or key < best[0]:
            best = (key, (n1, n2))
    if best is None:
        raise ValueError(f"no factorization for {k}")
    return best[1]


def orthogonal_scaled(g: np.random.Generator, n: int):
    """P = Q @ diag(u): Q from the QR factorization of a Gaussian matrix with
    the signs fixed so that R has a positive diagonal, u ~ U[0.8, 1.2].

    Returns (P, P_inv) as float32, both computed in float64 first
    (P_inv = diag(1/u) @ Q^T).  Draw order: n*n normals, then n uniforms.
    """
    a = g.standard_normal((n, n))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))[None, :]
    u = g.uniform(0.8, 1.2, n)
    p = q * u[None, :]
    p_inv = (q / u[None, :]).T
    return p.astype(np.float32), p_inv.astype(np.float32)


def outlier_channels(g: np.random.Generator, k: int, frac: float = 0.01) -> np.ndarray:
    """A seeded choice of round(frac * k) channel indices (a permutation prefix)."""
    n = int(round(frac * k))
    return np.sort(g.permutation(k)[:n])


# ---------------------------------------------------------------- workloads


def tiny_linear(seed: int = 0) -> dict:
    """Tiny W4A4 linear, no transform.

    X fp16 [16, 256] ~ N(0, 1) with channels 3 and 77 scaled x50;
    W fp16 [256, 256] ~ N(0, 0.02).  Draw order: X, W.
    """
    g = generator(seed)
    m, k, n = 16, 256, 256
    cs = np.ones(k)
    cs[[3, 77]] = 50.0
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs)
    w = _draw(g, (n, k), "normal", 0.02)
    return dict(name="tiny_linear_16x256x256", x=x, w=w, m=m, k=k, n=n,
                alpha_a=1.0, alpha_w=1.0)


def transform_quant(seed: int = 0, m: int = 2048, k: int = 4096) -> dict:
    """Transform + quantize, LLaMA-3-8B-like hidden size.

    X fp16 [m, k] ~ N(0, 1); 1% of the channels (seeded permutation) x30; token 0
    x100 (the pivot token); P1, P2 = random orthogonal x diag(U[0.8, 1.2]) with
    (n1, n2) = kron_factors(k); c ~ U[0.5, 2]; alpha_a = 0.9.
    Draw order: X, P1, P2, c; the outlier channels come from a second stream
    (seed + 1_000_003) because they must be known before X is cast.
    """
    g = generator(seed)
    h = generator(seed + 1_000_003)
    cols = outlier_channels(h, k)
    cs = np.ones(k)
    cs[cols] = 30.0
    rs = np.ones(m)
    rs[0] = 100.0
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs, row_scale=rs)
    n1, n2 = kron_factors(k)
    p1, p1i = orthogonal_scaled(g, n1)
    p2, p2i = orthogonal_scaled(g, n2)
    c = g.uniform(0.5, 2.0, k).astype(np.float32)
    return dict(name=f"transform_quant_{m}x{k}", x=x, m=m, k=k, n1=n1, n2=n2,
                p1=p1, p2=p2, p1_inv=p1i, p2_inv=p2i, c=c, alpha_a=0.9,
                outlier_cols=cols)


def prefill_linear(k: int, n: int, m: int = 2048, seed: int = 0,
                   w_kind: str = "normal", transform: bool = True) -> dict:
    """Prefill W4A4 linear at LLaMA-like shapes.

    X fp16 [m, k] ~ N(0, 1) with channels 3 and 77 x50 (the tiny recipe);
    W fp16 [n, k] ~ N(0, 0.02) (w_kind="normal") or Student-t(5) * 0.02
    (w_kind="t"); Kronecker factors P1, P2 (random orthogonal x diag(U[0.8,1.2]),
    (n1, n2) = kron_factors(k)); c = 1; alpha_a = alpha_w = 1.
    Draw order: X, W, P1, P2.
    """
    g = generator(seed)
    cs = np.ones(k)
    cs[[3, 77]] = 50.0
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs)
    w = _draw(g, (n, k), w_kind, 0.02)
    d = dict(name=f"prefill_{m}x{k}x{n}_{w_kind}", x=x, w=w, m=m, k=k, n=n,
             alpha_a=1.0, alpha_w=1.0)
    if transform:
        n1, n2 = kron_factors(k)
        p1, p1i = orthogonal_scaled(g, n1)
        p2, p2i = orthogonal_scaled(g, n2)
        d.update(n1=n1, n2=n2, p1=p1, p2=p2, p1_inv=p1i, p2_inv=p2i)
    return d


def decode_static(m: int, k: int, n: int, seed: int = 0, calib_seed: int = 1,
                  calib_tokens: int = 512) -> dict:
    """Decode, static per-channel activation scales (MergeQuant-style).

    X fp16 [m, k] ~ N(0, 1) with 1% outlier channels x30; W fp16 [n, k] ~ N(0, 0.02).
    The calibration draw is X_cal fp16 [calib_tokens, k] from the same recipe
    with ``calib_seed``; the outlier channels are shared (drawn from a stream
    of ``seed`` + 1_000_003).  The stand-in static scale is
    s_k = float32(max_t |X_cal[t, k]|) / 7 (the pages leave MergeQuant's
    calibration unspecified).  Draw order: X, W; calibration stream: X_cal.
    """
    h = generator(seed + 1_000_003)
    cols = outlier_channels(h, k)
    cs = np.ones(k)
    cs[cols] = 30.0
    g = generator(seed)
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs)
    w = _draw(g, (n, k), "normal", 0.02)
    gc = generator(calib_seed)
    xc = _draw(gc, (calib_tokens, k), "normal", 1.0, col_scale=cs)
    amax = np.abs(xc.astype(np.float32)).max(axis=0)
    s_k = (amax / np.float32(7.0)).astype(np.float32)
    return dict(name=f"decode_static_{m}x{k}x{n}", x=x, w=w, m=m, k=k, n=n,
                static_scale=s_k, alpha_a=1.0, alpha_w=1.0, outlier_cols=cols)


def residual_static(m: int, k: int, n: int, seed: int = 0, calib_seed: int = 1,
                    calib_tokens: int = 512) -> dict:
    """Residual-stream tokens for the static quantizer with per-token S_n
    (FPTQuant explainer, 伪动态残差缩放): token magnitudes that vary by orders.

    X fp16 [m, k] = r_t * z_t with z ~ N(0, 1) and 1% outlier channels x30 and
    r_t = 2^u, u ~ U(-4, 6) per token (the residual stream's norm grows and
    spikes across tokens); W fp16 [n, k] ~ N(0, 0.02).  The stand-in static
    scale comes from a calibration draw Z_cal [calib_tokens, k] of z alone
    (the unit-magnitude tokens the scaling is meant to produce):
    s_k = float32(max_t |Z_cal[t, k]|) / (7 * rms_cs), rms_cs = the root of
    the mean square of the column scales (the expected RMS of z) -- a property
    of this generator, not S_n itself.  Draw order: r, z, W; calibration
    stream: Z_cal.
    """
    h = generator(seed + 1_000_003)
    cols = outlier_channels(h, k)
    cs = np.ones(k)
    cs[cols] = 30.0
    g = generator(seed)
    r = 2.0 ** g.uniform(-4.0, 6.0, m)
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs, row_scale=r)
    w = _draw(g, (n, k), "normal", 0.02)
    gc = generator(calib_seed)
    zc = _draw(gc, (calib_tokens, k), "normal", 1.0, col_scale=cs)
    amax = np.abs(zc.astype(np.float32)).max(axis=0)
    rms_cs = np.float32(np.sqrt(np.mean(cs * cs)))
    s_k = (amax / (np.float32(7.0) * rms_cs)).astype(np.float32)
    return dict(name=f"residual_static_{m}x{k}x{n}", x=x, w=w, m=m, k=k, n=n,
                static_scale=s_k, token_scale=r, outlier_cols=cols)


def kv_cache(tokens: int, heads: int = 8, head_dim: int = 128, seed: int = 0) -> dict:
    """Key or value cache entries for INT4 KV quantization with FlatQuant's
    per-head transform (FlatQuant notes, Transformer 集成: P_h for the keys, P_v
    for the values, one head_dim x head_dim matrix applied to every head,
    not decomposed).  As a Kronecker transform of the token's H x D reshape:
    P1 = I_H, P2 = P_h.

    X fp16 [tokens, heads * head_dim] ~ N(0, 1) with 2 of every head's dims
    x20 (the same dims in every head: keys carry fixed outlier dims); P_h =
    random orthogonal x diag(U[0.8, 1.2]).  LLaMA-3-8B-like: 8 KV heads of 128.
    Draw order: outlier dims (head_dim permutation), X, P_h.
    """
    g = generator(seed)
    dims = g.permutation(head_dim)[:2]
    cs = np.ones(heads * head_dim)
    for h_ in range(heads):
        cs[h_ * head_dim + dims] = 20.0
    x = _draw(g, (tokens, heads * head_dim), "normal", 1.0, col_scale=cs)
    p_h, p_h_inv = orthogonal_scaled(g, head_dim)
    return dict(name=f"kv_cache_{tokens}x{heads}x{head_dim}", x=x, m=tokens, k=heads * head_dim,
                n1=heads, n2=head_dim, p1=np.eye(heads, dtype=np.float32), p2=p_h, p2_inv=p_h_inv,
                alpha_a=1.0, outlier_dims=dims)


def ternary_linear(m: int, k: int, n: int, seed: int = 0) -> dict:
    """Decode tokens against ternary weights W^ = alpha T + mu (PT2-LLM page,
    非对称三值量化器 ATQ), drawn directly (the offline fit needs trained weights).

    X fp16 [m, k] ~ N(0, 1) with 1% outlier channels x30; T int8 [n, k] in
    {-1, 0, 1} with probabilities (0.275, 0.45, 0.275) (about the share of
    zeros a ternary fit of Gaussian rows leaves); alpha float32 [n, k/128] ~
    U[0.01, 0.03]; mu float32 [n, k/128] ~ U[-0.005, 0.005] (the per-row
    offsets the asymmetric grid exists for).  Draw order: X, T, alpha, mu;
    the outlier channels come from the stream seed + 1_000_003.
    """
    h = generator(seed + 1_000_003)
    cols = outlier_channels(h, k)
    cs = np.ones(k)
    cs[cols] = 30.0
    g = generator(seed)
    x = _draw(g, (m, k), "normal", 1.0, col_scale=cs)
    u = g.uniform(0.0, 1.0, (n, k))
    t = np.where(u < 0.275, -1, np.where(u < 0.725, 0, 1)).astype(np.int8)
    alpha = g.uniform(0.01, 0.03, (n, k // GROUP)).astype(np.float32)
    mu = g.uniform(-0.005, 0.005, (n, k // GROUP)).astype(np.float32)
    return dict(name=f"ternary_{m}x{k}x{n}", x=x, t=t, alpha=alpha, mu=mu, m=m, k=k, n=n)


# Decode shapes of the ternary workload: the LLaMA-3-70B-like gate+up and down.
TERNARY_SHAPES = [(8192, 57344), (28672, 8192)]


# The LLaMA-3-8B-like decoder-layer linears at prefill, M = 2048 tokens:
# (K, N) for qkv, o, gate+up, down.
PREFILL_8B_SHAPES = [(4096, 6144), (4096, 4096), (4096, 28672), (14336, 4096)]
# The LLaMA-3-70B-like group-128 shapes at M = 4096.
GROUP_70B_SHAPES = [(8192, 10240), (8192, 57344), (28672, 8192)]
# Decode shapes.
DECODE_70B_SHAPES = [(8192, 57344), (28672, 8192)]
DECODE_TOKENS = [1, 8, 32, 64]


# ---------------------------------------------------------------- GEMM operands
# Packed INT4 operands for testing the GEMM on its own: every byte is a valid
# pair of nibbles, so uniform random bytes give uniform random codes in [-8, 7].


def random_packed(g: np.random.Generator, rows: int, k: int) -> np.ndarray:
    """uint8 [rows, k/2], uniform random bytes (two uniform INT4 codes each)."""
    return g.integers(0, 256, (rows, k // 2), dtype=np.uint8)


def constant_packed(rows: int, k: int, byte: int) -> np.ndarray:
    return np.full((rows, k // 2), byte, dtype=np.uint8)


def random_scales(g: np.random.Generator, n: int, lo: float = 1e-3, hi: float = 1e-1) -> np.ndarray:
    """float32 [n], log-uniform in [lo, hi]."""
    return np.exp(g.uniform(np.log(lo), np.log(hi), n)).astype(np.float32)


def random_group_scales(g: np.random.Generator, groups: int, rows: int, lo: float = 1e-3,
                        hi: float = 1e-1) -> np.ndarray:
    """float16 [groups, rows] (group-major), log-uniform in [lo, hi]."""
    return np.exp(g.uniform(np.log(lo), np.log(hi), (groups, rows))).astype(np.float16)
