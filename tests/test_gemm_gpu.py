"""fq_w4a4_gemm on the GPU against the CPU oracle, on seeded packed operands."""
import numpy as np
import pytest
import torch

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def _operands(seed, m, n, k):
    g = synth.generator(seed)
    return synth.random_packed(g, m, k), synth.random_packed(g, n, k)


SHAPES = [
    (128, 256, 128),      # one tile, one K slice
    (1, 8, 128),          # smallest
    (200, 264, 384),      # ragged M and N tiles
    (257, 520, 1024),     # ragged, several K slices
    (64, 1024, 4096),     # decode-style swap path
    (8, 8192, 28672),     # decode with split-K
    (33, 136, 640),       # swap path with 48-wide token tile
    (2048, 512, 4096),    # prefill, many M tiles
]


@pytest.mark.parametrize("m,n,k", SHAPES)
def test_gemm_int32_exact(m, n, k):
    a, b = _operands(m + n + k, m, n, k)
    acc = fq.fq_w4a4_gemm_s32(C.dev(a), C.dev(b))
    ref = O.gemm_int(C.unpack(a), C.unpack(b))
    assert np.array_equal(C.host(acc).astype(np.int64), ref)


def test_gemm_int32_extremes():
    """-8 x -8 over the largest K: 64 * 65536 per output, exact in int32 and float32."""
    m, n, k = 4, 16, 65536
    a = synth.constant_packed(m, k, 0x88)
    b = synth.constant_packed(n, k, 0x88)
    acc = C.host(fq.fq_w4a4_gemm_s32(C.dev(a), C.dev(b)))
    assert np.all(acc == 64 * k)
    b7 = synth.constant_packed(n, k, 0x77)
    acc = C.host(fq.fq_w4a4_gemm_s32(C.dev(a), C.dev(b7)))
    assert np.all(acc == -56 * k)


@pytest.mark.parametrize("m,n,k", SHAPES + [(1, 8192, 28672), (32, 8192, 28672), (64, 57344, 8192)])
def test_gemm_row_exact(m, n, k):
    a, b = _operands(3 * m + n + k, m, n, k)
    g = synth.generator(m + 1)
    sx = synth.random_scales(g, m)
    sw = synth.random_scales(g, n)
    y = fq.fq_w4a4_gemm(C.dev(a), C.dev(sx), C.dev(b), C.dev(sw), fq.ROW)
    ref = O.dequant_row(O.gemm_int(C.unpack(a), C.unpack(b)), sx, sw)
    C.check_fp16_exact(C.host(y), ref)


@pytest.mark.parametrize("m,n,k", [(1, 8192, 28672), (8, 256, 512), (64, 57344, 8192), (300, 264, 1024)])
def test_gemm_static_exact(m, n, k):
    a, b = _operands(5 * m + n + k, m, n, k)
    sw = synth.random_scales(synth.generator(m + 2), n, 1e-4, 1e-2)
    y = fq.fq_w4a4_gemm(C.dev(a), None, C.dev(b), C.dev(sw), fq.STATIC)
    ref = O.dequant_static(O.gemm_int(C.unpack(a), C.unpack(b)), sw)
    C.check_fp16_exact(C.host(y), ref)


@pytest.mark.parametrize("m,n,k", [(128, 128, 128), (200, 264, 1024), (1, 136, 2048), (512, 1024, 8192)])
def test_gemm_group(m, n, k):
    a, b = _operands(7 * m + n + k, m, n, k)
    g = synth.generator(m + 3)
    sx = synth.random_group_scales(g, k // 128, m)
    sw = synth.random_group_scales(g, k // 128, n)
    y = fq.fq_w4a4_gemm(C.dev(a), C.dev(sx), C.dev(b), C.dev(sw), fq.GROUP)
    n_beyond = C.check_fp16_group(C.host(y), C.unpack(a), C.unpack(b), sx.T, sw.T)
    print(f"group {m}x{n}x{k}: {n_beyond} outputs beyond 1 ulp (cancellation bound)")


@pytest.mark.parametrize("m", [17, 32, 64])
def test_gemm_decode_split_k_repeatable(m):
    """Decode shapes with split-K over a long K, run several times: every run
    bit-exact (a stage handed back too early corrupts random rows in some runs)."""
    n, k = 8192, 28672
    a, b = _operands(11 * m, m, n, k)
    sw = synth.random_scales(synth.generator(m + 5), n, 1e-4, 1e-2)
    ref = O.dequant_static(O.gemm_int(C.unpack(a), C.unpack(b)), sw)
    A, B, S = C.dev(a), C.dev(b), C.dev(sw)
    for _ in range(4):
        C.check_fp16_exact(C.host(fq.fq_w4a4_gemm(A, None, B, S, fq.STATIC)), ref)
    fq.fq_check_device_error()


def test_gemm_workspace_is_reused_correctly():
    """Two split-K calls in a row on one workspace give the same exact result:
    garbage beyond the counter block does not leak into the sums, and the
    counters are back at zero after each call."""
    m, n, k = 8, 8192, 28672
    a, b = _operands(99, m, n, k)
    g = synth.generator(4)
    sx, sw = synth.random_scales(g, m), synth.random_scales(g, n)
    ws = torch.full((fq.fq_gemm_workspace_size(m, n, k, fq.ROW),), 0x5A, dtype=torch.uint8, device="cuda")
    ws[: fq.SYNC_BYTES].zero_()
    y1 = C.host(fq.fq_w4a4_gemm(C.dev(a), C.dev(sx), C.dev(b), C.dev(sw), fq.ROW, workspace=ws))
    y2 = C.host(fq.fq_w4a4_gemm(C.dev(a), C.dev(sx), C.dev(b), C.dev(sw), fq.ROW, workspace=ws))
    ref = O.dequant_row(O.gemm_int(C.unpack(a), C.unpack(b)), sx, sw)
    C.check_fp16_exact(y1, ref)
    C.check_fp16_exact(y2, ref)
    fq.fq_check_device_error()
    assert not ws[: fq.SYNC_BYTES].any(), "the counter block is not back at zero"


# Prefill shapes for the persistent CTA-pair kernel: tile counts below, at and
# above the 74 pairs, ragged A pairs and weight tiles, repeated launches on a
# garbage workspace, and the entry point without a workspace.
PERSISTENT_SHAPES = [
    (1024, 4096, 2048),   # 64 tiles: fewer tiles than pairs
    (2048, 10240, 1024),  # 320 tiles: four rounds, the last one partial
    (384, 1024, 8192),    # 8 tiles, the second A pair half out of range
    (640, 776, 8192),     # ragged M and N tiles
]


@pytest.mark.parametrize("m,n,k", PERSISTENT_SHAPES)
def test_gemm_persistent_exact(m, n, k):
    a, b = _operands(13 * m + n + k, m, n, k)
    g = synth.generator(m + 6)
    sx, sw = synth.random_scales(g, m), synth.random_scales(g, n)
    acc = O.gemm_int(C.unpack(a), C.unpack(b))
    A, B = C.dev(a), C.dev(b)
    ws = torch.full((max(fq.fq_gemm_workspace_size(m, n, k, fq.ROW), 256),), 0xA5, dtype=torch.uint8, device="cuda")
    ref = O.dequant_row(acc, sx, sw)
    for _ in range(3):
        C.check_fp16_exact(C.host(fq.fq_w4a4_gemm(A, C.dev(sx), B, C.dev(sw), fq.ROW, workspace=ws)), ref)
    refs = O.dequant_static(acc, sw)
    C.check_fp16_exact(C.host(fq.fq_w4a4_gemm(A, None, B, C.dev(sw), fq.STATIC, workspace=ws)), refs)
    C.check_fp16_exact(C.host(fq.fq_w4a4_gemm_noalloc(A, C.dev(sx), B, C.dev(sw), fq.ROW)), ref)
    fq.fq_check_device_error()


def test_gemm_persistent_stress_repeated():
    """The CTA-pair GEMM 50 times, interleaving tile counts from 1 to 512 (so the
    pairs' share of tiles and the cross-CTA barrier phases differ from launch
    to launch): every launch bit-exact, no bounded wait giving up."""
    shapes = [(256, 256, 512), (1024, 2048, 512), (2048, 10240, 256), (640, 776, 1024), (4096, 8192, 256)]
    cases = []
    for i, (m, n, k) in enumerate(shapes):
        a, b = _operands(17 * i + 1, m, n, k)
        g = synth.generator(i + 40)
        sx, sw = synth.random_scales(g, m), synth.random_scales(g, n)
        ref = O.dequant_row(O.gemm_int(C.unpack(a), C.unpack(b)), sx, sw)
        ws = torch.zeros(max(fq.fq_gemm_workspace_size(m, n, k, fq.ROW), 256), dtype=torch.uint8, device="cuda")
        cases.append((C.dev(a), C.dev(sx), C.dev(b), C.dev(sw), ws, C.dev(ref.view(np.uint16).astype(np.int16))))
    for it in range(50):
        A, SX, B, SW, ws, ref = cases[(it * 3) % len(cases)]
        y = fq.fq_w4a4_gemm(A, SX, B, SW, fq.ROW, workspace=ws)
        assert torch.equal(y.view(torch.int16), ref), f"launch {it} differs"
    fq.fq_check_device_error()
