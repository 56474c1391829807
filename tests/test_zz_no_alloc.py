"""The allocation-free GEMM entry point, fp8_gemm_blockscaled_noalloc.

Some callers cannot allocate device memory at the moment they run a GEMM: code with a
memory budget fixed in advance, allocator callbacks that must not re-enter the
allocator, or hot paths where cudaMalloc is forbidden.  For them the library runs the
split-K GEMM with its workspace in a fixed device array of its own.

Every case here is one whose last wave is split along K (the test asserts that the
workspace size is nonzero), so the fixed scratch is used, and the second of two calls in
a row finds the first call's partial tiles in it.  Both results are checked against the
oracle's float64 product within the fp32 acceptance band the other GEMM tests use, and
bit for bit against the workspace entry point on the same stream (the two run the same
plan, and the split-K sum has a fixed order).  It is kept in a file of its own that pytest
collects last, and it needs nothing from the other tests.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from tests._helpers import assert_gemm_close, host, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


def _gemm_args(qa, sa, qb, sb, C):
    M, K = qa.shape
    N = qb.shape[0]
    return (qa.data_ptr(), sa.data_ptr(), sa.stride(0), qb.data_ptr(), sb.data_ptr(), 0,
            0, C.data_ptr(), 1, M, N, K, qa.stride(0), qb.stride(0), C.stride(0))


# Each shape leaves a partial last wave that is split along K: a full-size dense problem
# with a short K, one single tile, and a ragged M over a few tiles.
@pytest.mark.parametrize("M,N,K", [(4096, 7168, 1024), (128, 256, 512), (300, 1024, 2048)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(fq, M, N, K):
    import torch
    L = fq.lib()
    rng = np.random.default_rng(M + N + K)
    a_bits = workloads.normal_bf16(rng, (M, K), 1.0, 0.001)
    b_bits = workloads.normal_bf16(rng, (N, K), 0.02)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a_bits), False)
    qb, sb = fq.quant_weight_128x128(to_dev_bf16(b_bits), False)
    stream = torch.cuda.current_stream().cuda_stream

    need = ctypes.c_size_t(0)
    assert L.fp8_gemm_workspace_size(M, N, K, ctypes.byref(need)) == 0
    assert need.value > 0, "this shape was chosen to split its last wave along K"

    # the existing entry point with a caller workspace
    ws = torch.empty(int(need.value), dtype=torch.uint8, device="cuda")
    C_ws = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    assert L.fp8_gemm_blockscaled_ws(*_gemm_args(qa, sa, qb, sb, C_ws), ws.data_ptr(),
                                     ws.numel(), stream) == 0

    # the allocation-free entry point, twice in a row on the same stream
    outs = []
    for _ in range(2):
        C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert L.fp8_gemm_blockscaled_noalloc(*_gemm_args(qa, sa, qb, sb, C), stream) == 0
        outs.append(C)
    torch.cuda.synchronize()
    assert fq.device_error() == 0

    rows = np.unique(np.concatenate([np.arange(0, M, max(1, M // 64)), [M - 1]]))
    qa_r, sa_r = oracle.quant_act_1x128(a_bits[rows], False)
    qb_r, sb_r = oracle.quant_weight_128x128(b_bits, False)
    C_ref, T = oracle.gemm_blockscaled_ref(qa_r, sa_r, qb_r, sb_r)
    assert_gemm_close("workspace entry point", host(C_ws)[rows], C_ref, T, bf16=False)
    for i, C in enumerate(outs):
        assert_gemm_close(f"noalloc call {i + 1}", host(C)[rows], C_ref, T, bf16=False)
        assert torch.equal(C, C_ws), f"noalloc call {i + 1} differs from the workspace entry point"
