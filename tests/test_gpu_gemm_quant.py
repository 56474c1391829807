"""GPU parity of the GEMM whose epilogue also quantizes its output (fp8_gemm_blockscaled_quant).

Contract: the bf16 C equals fp8_gemm_blockscaled's bf16 C bit for bit (same kernel, same
promotion order, no split), C is within the parity band of the FP64 oracle product, and
the codes and scales equal the oracle's 1x128 quantization of that bf16 C bit for bit
(and the library's own quantizer on it, which the quantizer tests tie to the oracle).
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


def _case(fq, M, N, K, pow2_in, pow2_out, b_rowwise=False, seed=0, rows=None, std_a=1.0,
          outlier_frac=0.0):
    import torch
    rng = np.random.default_rng(seed)
    a_bits = workloads.normal_bf16(rng, (M, K), std_a, outlier_frac)
    b_bits = workloads.normal_bf16(rng, (N, K), 0.02)
    a, b = to_dev_bf16(a_bits), to_dev_bf16(b_bits)
    qa, sa = fq.quant_act_1x128(a, pow2_in)
    qb, sb = (fq.quant_act_1x128(b, pow2_in) if b_rowwise else fq.quant_weight_128x128(b, pow2_in))
    C, qc, sc = fq.gemm_blockscaled_quant(qa, sa, qb, sb, pow2=pow2_out, b_rowwise=b_rowwise)
    C_plain = fq.gemm_blockscaled(qa, sa, qb, sb, b_rowwise=b_rowwise, split_k=False)
    _, qc2, sc2 = fq.gemm_blockscaled_quant(qa, sa, qb, sb, pow2=pow2_out, b_rowwise=b_rowwise,
                                            with_c=False)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    name = f"quant-out {M}x{N}x{K} pow2 {pow2_in}/{pow2_out}"
    Cb = host(C.view(torch.int16)).view(np.uint16)                  # bf16 bit patterns
    assert_bytes_equal(name + " C vs gemm_blockscaled", Cb, host(C_plain.view(torch.int16)).view(np.uint16))
    assert_bytes_equal(name + " qc without C", host(qc2), host(qc))
    assert_bytes_equal(name + " sc without C", host(sc2), host(sc))

    rows = np.arange(M) if rows is None else np.asarray(rows)
    # C against the oracle's FP64 product of the oracle's own codes (checked equal to the GPU's)
    qa_ref, sa_ref = oracle.quant_act_1x128(a_bits[rows], pow2_in)
    qb_ref, sb_ref = (oracle.quant_act_1x128(b_bits, pow2_in) if b_rowwise
                      else oracle.quant_weight_128x128(b_bits, pow2_in))
    assert_bytes_equal(name + " qa", host(qa)[rows], qa_ref)
    C_ref, T = oracle.gemm_blockscaled_ref(qa_ref, sa_ref, qb_ref, sb_ref, b_rowwise)
    assert_gemm_close(name, host(C.float())[rows], C_ref, T, bf16=True)
    # the output's codes and scales against the oracle's quantizer on the GPU's bf16 C
    q_ref, s_ref = oracle.quant_act_1x128(np.ascontiguousarray(Cb[rows]), pow2_out)
    assert_bytes_equal(name + " qc", host(qc)[rows], q_ref)
    assert_bytes_equal(name + " sc", host(sc)[:, rows], s_ref)
    # and the library's own quantizer on the same C
    q_lib, s_lib = fq.quant_act_1x128(C, pow2_out)
    assert_bytes_equal(name + " qc vs quantizer", host(qc), host(q_lib))
    assert_bytes_equal(name + " sc vs quantizer", host(sc), host(s_lib))
    return qc, sc


@pytest.mark.parametrize("pow2_out", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (128, 256, 256), (300, 384, 640), (257, 1280, 1152)])
def test_quant_out_ragged(fq, M, N, K, pow2_out):
    """Ragged M, N = 128 mod 256 (the last tile's second column half lies outside C), group
    counts of 1 to 10."""
    _case(fq, M, N, K, False, pow2_out, seed=M + N + K)


def test_quant_out_rowwise_b_pow2_inputs(fq):
    _case(fq, 200, 512, 1024, True, True, b_rowwise=True, seed=5)


def test_quant_out_outliers(fq):
    """Activations with 0.1% x100 outliers: the output tiles' amax spread widely."""
    _case(fq, 384, 768, 896, False, False, seed=6, outlier_frac=1e-3)


def test_quant_out_zero_rows(fq):
    """All-zero A rows give all-zero output tiles: scale 1, codes +0."""
    import torch
    M, N, K = 130, 256, 256
    qa = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.ones((K // 128, M), dtype=torch.float32, device="cuda")
    b = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(3), (N, K), 0.02))
    qb, sb = fq.quant_weight_128x128(b, False)
    C, qc, sc = fq.gemm_blockscaled_quant(qa, sa, qb, sb)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    assert int(host(qc).max()) == 0
    assert np.all(host(sc) == 1.0)
    assert float(host(C.float()).max()) == 0.0


def test_quant_out_dense_full_size_sampled_rows(fq):
    """The dense workload's shape (4096 x 7168 x 7168, power-of-two scales in and out):
    every row's codes against the library's quantizer, 64 sampled rows against the oracle."""
    w = workloads.dense()
    rng = np.random.default_rng(12)
    rows = np.unique(np.concatenate([rng.choice(w.M, 62, replace=False), [0, w.M - 1]]))
    _case(fq, w.M, w.N, w.K, True, True, seed=13, rows=rows)
