"""Device-side failure detection without a GPU fault.

Every wait in the library's kernels is bounded: on expiry the kernel records a code in a
device error word, unwinds and returns, so the CUDA context stays usable.  The self-test
kernel waits on a barrier that nothing arrives on, with a 10 ms limit; the host reads the
code back and then runs a GEMM on the same context.
"""
import numpy as np
import pytest

import workloads
from tests._helpers import host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


def test_bounded_wait_reports_timeout_and_context_survives(fq):
    import time
    import torch
    L = fq.lib()
    assert fq.device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert L.fp8q_selftest_wait_timeout(10_000_000, stream) == 0
    code = fq.device_error()                 # synchronizes the stream
    elapsed = time.perf_counter() - t0
    assert code == (7 << 8) | 6, hex(code)
    assert elapsed < 5.0
    assert fq.device_error() == 0            # reading clears the word
    assert L.fp8q_selftest_wait_timeout(0, stream) == 2
    # the context is still usable: an exact unit-scale GEMM right after
    rng = workloads.rng_for(1, 9)
    qa, ia = workloads.small_int_e4m3_codes(rng, (128, 256))
    qb, ib = workloads.small_int_e4m3_codes(rng, (128, 256))
    C = fq.gemm_blockscaled(to_dev(qa), to_dev(np.ones((2, 128), np.float32)), to_dev(qb),
                            to_dev(np.ones((1, 2), np.float32)), out_dtype=torch.float32)
    assert np.array_equal(host(C), (ia @ ib.T).astype(np.float32))
    assert fq.device_error() == 0
