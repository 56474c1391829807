"""GPU parity of the FP8 linear layer (Fprop / Dgrad / Wgrad through the C ABI) and of the
128x128 block transpose, against the oracle.

the-good.kr wr_id=2169793 para 3: all three GEMMs of a linear layer in FP8.  Each GEMM's
operands are quantized by the oracle from the same bf16 tensors (the transposed copies
by quantizing the transposes), and each output is compared with the oracle's GEMM of
those codes under the bf16 criterion of the other GEMM tests.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests._helpers import assert_bytes_equal, assert_gemm_close, host, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (1024, 512)])
def test_transpose_blocks_is_the_quantization_of_the_transpose(fq, N, K):
    rng = np.random.default_rng(N + K)
    w = workloads.normal_bf16(rng, (N, K), 0.02)
    q, s = fq.quant_weight_128x128(to_dev_bf16(w), False)
    qt, st = fq.transpose_blocks(q, s)
    qt_ref, st_ref = oracle.quant_weight_128x128(np.ascontiguousarray(w.T), False)
    assert_bytes_equal("qt", host(qt), qt_ref)
    assert_bytes_equal("st", host(st), st_ref)
    assert fq.device_error() == 0


@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("T,K,N", [(256, 384, 512), (384, 256, 256)])
def test_fp8_linear_forward_backward(fq, T, K, N, pow2):
    import torch
    from fp8_fine_grained_weight_b200.linear import fp8_linear
    rng = np.random.default_rng(T * 7 + K * 3 + N)
    x_bits = workloads.normal_bf16(rng, (T, K), 1.0, 0.001)
    w_bits = workloads.normal_bf16(rng, (N, K), 0.02)
    dy_bits = workloads.normal_bf16(rng, (T, N), 1e-3)
    x = to_dev_bf16(x_bits).requires_grad_(True)
    w = to_dev_bf16(w_bits).requires_grad_(True)
    y = fp8_linear(x, w, pow2)
    y.backward(to_dev_bf16(dy_bits))
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    assert y.dtype == x.grad.dtype == w.grad.dtype == torch.bfloat16

    def q_rows(bits):          # 1x128 along the last dimension
        return oracle.quant_act_1x128(np.ascontiguousarray(bits), pow2)

    # Fprop: X (1x128 along K) x W (128x128)
    qa, sa = q_rows(x_bits)
    qb, sb = oracle.quant_weight_128x128(w_bits, pow2)
    C, Tm = oracle.gemm_blockscaled_ref(qa, sa, qb, sb)
    assert_gemm_close("fprop", host(y), C, Tm, bf16=True)
    # Dgrad: dY (1x128 along N) x W^T (128x128)
    qa, sa = q_rows(dy_bits)
    qb, sb = oracle.quant_weight_128x128(np.ascontiguousarray(w_bits.T), pow2)
    C, Tm = oracle.gemm_blockscaled_ref(qa, sa, qb, sb)
    assert_gemm_close("dgrad", host(x.grad), C, Tm, bf16=True)
    # Wgrad: dY^T (1x128 along T) x X^T (1x128 along T)
    qa, sa = q_rows(dy_bits.T)
    qb, sb = q_rows(x_bits.T)
    C, Tm = oracle.gemm_blockscaled_ref(qa, sa, qb, sb, b_rowwise=True)
    assert_gemm_close("wgrad", host(w.grad), C, Tm, bf16=True)


def test_fp8_linear_tracks_the_bf16_layer(fq):
    """Against torch's fp32 product of the same bf16 tensors: the FP8 layer's outputs and
    gradients stay within a few percent (the E4M3 quantization error, not a parity test)."""
    import torch
    from fp8_fine_grained_weight_b200.linear import FP8Linear
    torch.manual_seed(0)
    layer = FP8Linear(512, 384, pow2=True, device="cuda")
    x = torch.randn(256, 512, device="cuda").to(torch.bfloat16).requires_grad_(True)
    y = layer(x)
    dy = torch.randn_like(y)
    y.backward(dy)
    xf, wf = x.detach().float().requires_grad_(True), layer.weight.detach().float().requires_grad_(True)
    yf = xf @ wf.T
    yf.backward(dy.float())

    def rel(a, b):
        return float((a.detach().float() - b.detach()).norm() / b.detach().norm())

    assert rel(y, yf) < 0.06
    assert rel(x.grad, xf.grad) < 0.06
    assert rel(layer.weight.grad, wf.grad) < 0.06


def test_entry_points_on_a_fresh_thread(fq):
    """A thread that has made no CUDA call yet (as a framework's backward worker thread may
    be) can call the entry points that encode TMA descriptors: the library binds the
    device's context itself."""
    import threading
    import torch
    rng = np.random.default_rng(41)
    x_bits = workloads.normal_bf16(rng, (256, 256), 1.0)
    w_bits = workloads.normal_bf16(rng, (256, 256), 0.02)
    x, w = to_dev_bf16(x_bits), to_dev_bf16(w_bits)
    q, s = fq.quant_act_1x128(x, True)
    qw, sw = fq.quant_weight_128x128(w, True)
    torch.cuda.synchronize()
    out, err = {}, []

    def work():
        try:   # the GEMMs (which encode TMA descriptors) are this thread's first CUDA calls
            out["c"] = fq.gemm_blockscaled_ue8m0(q, s, qw, sw)
            out["c2"] = fq.gemm_blockscaled(q, s, qw, sw)
            out["qt"] = fq.quant_act_dual(x, True)[2]
            torch.cuda.synchronize()
        except Exception as e:                    # reported below, on the test's thread
            err.append(e)

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert not err, err
    qt_ref, _ = oracle.quant_act_1x128(np.ascontiguousarray(x_bits.T), True)
    assert_bytes_equal("fresh-thread qt", host(out["qt"]), qt_ref)
    qa, sa = oracle.quant_act_1x128(x_bits, True)
    qb, sb = oracle.quant_weight_128x128(w_bits, True)
    C, Tm = oracle.gemm_blockscaled_ref(qa, sa, qb, sb)
    assert_gemm_close("fresh-thread ue8m0", host(out["c"]), C, Tm, bf16=True)
    assert_gemm_close("fresh-thread promoted", host(out["c2"]), C, Tm, bf16=True)
