"""fq_w4a4_gemm_noalloc: the GEMM entry point for callers that cannot allocate.

Some users of this library cannot give the GEMM device scratch memory: a
plugin running inside another runtime that owns all device memory, or a
serving loop that forbids allocation once it has started.  This entry point
keeps the split-K partial sums in a static buffer inside libfq.so instead.
These tests call it through the C ABI and compare its output with the
workspace-taking fq_w4a4_gemm, with the same bar as every other per-token /
static GEMM test here: bit-exact fp16 outputs.  Two calls in a row check that
the shared buffer's leftover contents do not leak into the next result.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest

import gpu_checks as C
from int4_linear_b200 import fq, synth

pytestmark = pytest.mark.gpu

# decode shapes that split K (and so use the static scratch), and one that does not
CASES = [(8, 8192, 28672, fq.ROW), (64, 8192, 28672, fq.STATIC), (1, 8192, 8192, fq.ROW),
         (256, 512, 1024, fq.ROW)]


@pytest.mark.parametrize("m,n,k,gran", CASES)
def test_noalloc_matches_workspace_gemm_twice(m, n, k, gran):
    g = synth.generator(m + n + k)
    a = C.dev(synth.random_packed(g, m, k))
    b = C.dev(synth.random_packed(g, n, k))
    sx = C.dev(synth.random_scales(g, m)) if gran == fq.ROW else None
    sw = C.dev(synth.random_scales(g, n))
    ref = C.host(fq.fq_w4a4_gemm(a, sx, b, sw, gran))
    for _ in range(2):
        y = C.host(fq.fq_w4a4_gemm_noalloc(a, sx, b, sw, gran))
        C.check_fp16_exact(y, ref)
    fq.fq_check_device_error()


def test_noalloc_scratch_covers_every_decode_shape():
    """The split-K scratch grows with the token count and the number of CTAs,
    not with N: at the largest decode token count (64) and a very wide layer it
    still fits the 32 MiB static buffer, and such a call runs bit-exact."""
    for m in (1, 16, 17, 32, 64):
        for n in (1024, 8192, 139264):
            assert fq.fq_gemm_workspace_size(m, n, 8192, fq.ROW) <= 32 << 20
    m, n, k = 16, 139264, 1024
    g = synth.generator(77)
    a = C.dev(synth.random_packed(g, m, k))
    b = C.dev(synth.random_packed(g, n, k))
    sx, sw = C.dev(synth.random_scales(g, m)), C.dev(synth.random_scales(g, n))
    ref = C.host(fq.fq_w4a4_gemm(a, sx, b, sw, fq.ROW))
    C.check_fp16_exact(C.host(fq.fq_w4a4_gemm_noalloc(a, sx, b, sw, fq.ROW)), ref)
    fq.fq_check_device_error()
