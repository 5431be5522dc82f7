"""Failure detection on the GPU without a fault: a bounded wait that runs out
records FQ_ERR_TIMEOUT, the host reads it, and the context stays usable."""
import numpy as np
import pytest

import gpu_checks as C
from int4_linear_b200 import fq, synth
from oracle import fq_oracle as O

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_cleared():
    fq.fq_check_device_error()  # start clean
    fq.fq_debug_wait_timeout(2000)
    with pytest.raises(fq.FqError) as e:
        fq.fq_check_device_error()
    assert e.value.status == fq.FQ_ERR_TIMEOUT
    fq.fq_check_device_error()  # cleared
    # the context still runs the real kernels correctly
    g = synth.generator(1)
    a, b = synth.random_packed(g, 16, 256), synth.random_packed(g, 64, 256)
    acc = fq.fq_w4a4_gemm_s32(C.dev(a), C.dev(b))
    assert np.array_equal(C.host(acc).astype(np.int64), O.gemm_int(O.unpack_int4(a), O.unpack_int4(b)))
    fq.fq_check_device_error()
