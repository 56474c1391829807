"""GPU parity of the quantization kernels: E4M3 bytes and fp32 scales bit-exact with the
oracle, through the C ABI, on the workloads' inputs and on edge cases."""
import numpy as np
import pytest

import oracle
import workloads
from tests._helpers import assert_bytes_equal, host, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


def _act_parity(fq, bits, pow2, ld_scale=None, name="act"):
    x = to_dev_bf16(bits)
    q, s = fq.quant_act_1x128(x, pow2, ld_scale=ld_scale)
    q_ref, s_ref = oracle.quant_act_1x128(bits, pow2)
    M = bits.shape[0]
    assert_bytes_equal(name + ".q", host(q), q_ref)
    assert_bytes_equal(name + ".s", host(s)[:, :M], s_ref)
    assert fq.device_error() == 0


def _weight_parity(fq, bits, pow2, name="weight"):
    w = to_dev_bf16(bits)
    q, s = fq.quant_weight_128x128(w, pow2)
    q_ref, s_ref = oracle.quant_weight_128x128(bits.reshape(-1, bits.shape[-1]), pow2)
    assert_bytes_equal(name + ".q", host(q).reshape(q_ref.shape), q_ref)
    assert_bytes_equal(name + ".s", host(s).reshape(s_ref.shape), s_ref)


@pytest.mark.parametrize("pow2", [False, True])
def test_act_tiny(fq, pow2):
    _act_parity(fq, workloads.tiny().gen_a(), pow2)


@pytest.mark.parametrize("M,K", [(1, 128), (7, 256), (65, 640), (300, 1024), (1000, 384)])
@pytest.mark.parametrize("pow2", [False, True])
def test_act_ragged(fq, M, K, pow2):
    bits = workloads.normal_bf16(np.random.default_rng(M * 7 + K), (M, K), 1.0, 0.01)
    _act_parity(fq, bits, pow2, ld_scale=M + (4 - M % 4) % 4 + 4)


def test_act_edge_values(fq):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 512)).astype(np.float32)
    x[0] = 0.0                                         # all-zero row: s = 1, q = 0
    x[1, :128] = -0.0                                  # signed zeros
    x[2, 128:256] = 0.0
    x[2, 200] = 1e-3                                   # single nonzero
    x[3, :128] *= 2.0 ** -125                          # subnormal-range scales
    x[3, 128:256] *= 2.0 ** -132
    x[4, :128] *= 1e30                                 # huge magnitudes
    x[5, :] = np.where(np.arange(512) % 2, 3.0, -3.0)  # constant magnitude: codes +-448
    x[6, :128] = -1e-40                                # bf16 subnormals, negative
    x[6, 5] = 1.0                                      # ... quotient underflows to -0
    x[7, :128] = np.linspace(-1, 1, 128) * 448 * 2.0 ** -9   # E4M3 grid points and midpoints
    bits = workloads.fp32_to_bf16_bits(x)
    for pow2 in (False, True):
        _act_parity(fq, bits, pow2, name=f"edge pow2={pow2}")


@pytest.mark.parametrize("pow2", [False, True])
def test_act_dense_full(fq, pow2):
    _act_parity(fq, workloads.dense().gen_a(), pow2, name="dense A")


def test_act_decode_full(fq):
    _act_parity(fq, workloads.decode().gen_a(), True, name="decode A")


def test_act_wgrad_full_sampled_rows(fq):
    """dY [7168, 16384] and X [2048, 16384], quantized on the GPU in one launch each;
    every 7th row compared with the oracle (rows are independent tiles)."""
    w = workloads.wgrad()
    for name, bits in (("dY", w.gen_a()), ("X", w.gen_b())):
        x = to_dev_bf16(bits)
        q, s = fq.quant_act_1x128(x, False)
        rows = np.arange(0, bits.shape[0], 7)
        q_ref, s_ref = oracle.quant_act_1x128(bits[rows], False)
        assert_bytes_equal(name + ".q", host(q)[rows], q_ref)
        assert_bytes_equal(name + ".s", host(s)[:, rows], s_ref)


@pytest.mark.parametrize("pow2", [False, True])
def test_weight_tiny_and_ragged(fq, pow2):
    _weight_parity(fq, workloads.tiny().gen_b(), pow2)
    bits = workloads.normal_bf16(np.random.default_rng(3), (384, 640), 0.02)
    bits[200, 300] = workloads.fp32_to_bf16_bits(np.array([7.0], np.float32))[0]
    _weight_parity(fq, bits, pow2, name="ragged")


def test_weight_edge_blocks(fq):
    x = np.random.default_rng(9).standard_normal((256, 256)).astype(np.float32) * 0.01
    x[:128, :128] = 0.0
    x[128:, :128] *= 2.0 ** -120
    x[:128, 128:] = -0.0
    for pow2 in (False, True):
        _weight_parity(fq, workloads.fp32_to_bf16_bits(x), pow2, name=f"edge pow2={pow2}")


@pytest.mark.parametrize("pow2", [False, True])
def test_weight_dense_full(fq, pow2):
    _weight_parity(fq, workloads.dense().gen_b(), pow2, name="dense W")


def test_weight_prefill_full_sampled_blocks(fq):
    """All 32 experts [32, 4096, 7168] in one launch; 3 experts compared in full."""
    w = workloads.prefill()
    bits = w.gen_b()
    q, s = fq.quant_weight_128x128(to_dev_bf16(bits), False)
    qh, sh = host(q), host(s)
    for e in (0, 13, 31):
        q_ref, s_ref = oracle.quant_weight_128x128(bits[e], False)
        assert_bytes_equal(f"expert {e}.q", qh[e], q_ref)
        assert_bytes_equal(f"expert {e}.s", sh[e], s_ref)


def test_weight_decode_full(fq):
    _weight_parity(fq, workloads.decode().gen_b(), False, name="decode W")


def test_rowwise(fq):
    bits = workloads.normal_bf16(np.random.default_rng(4), (37, 4096), 1.0, 0.001)
    for pow2 in (False, True):
        q, s = fq.quant_rowwise(to_dev_bf16(bits), pow2)
        q_ref, s_ref = oracle.quant_rowwise(bits, pow2)
        assert_bytes_equal("rowwise.q", host(q), q_ref)
        assert_bytes_equal("rowwise.s", host(s), s_ref)


# ---------------------------------------------------------- rows and columns in one pass

def _dual_parity(fq, bits, pow2, name="dual"):
    """Both outputs bit-exact: (q, s) with the 1x128 quantization of X, (qt, st) with the
    1x128 quantization of X^T (the definition of the transposed copy)."""
    q, s, qt, st = fq.quant_act_dual(to_dev_bf16(bits), pow2)
    q_ref, s_ref = oracle.quant_act_1x128(bits, pow2)
    qt_ref, st_ref = oracle.quant_act_1x128(np.ascontiguousarray(bits.T), pow2)
    assert_bytes_equal(name + ".q", host(q), q_ref)
    assert_bytes_equal(name + ".s", host(s), s_ref)
    assert_bytes_equal(name + ".qt", host(qt), qt_ref)
    assert_bytes_equal(name + ".st", host(st), st_ref)
    assert fq.device_error() == 0


@pytest.mark.parametrize("M,K", [(128, 128), (256, 384), (384, 1024), (1024, 256)])
@pytest.mark.parametrize("pow2", [False, True])
def test_dual_shapes(fq, M, K, pow2):
    rng = np.random.default_rng(M * 3 + K)
    _dual_parity(fq, workloads.normal_bf16(rng, (M, K), 1.0, 0.001), pow2, f"dual {M}x{K}")


def test_dual_edge_tiles(fq):
    """Zero, signed-zero and single-value columns, tiny magnitudes (subnormal scales),
    one huge outlier per column tile."""
    rng = np.random.default_rng(17)
    x = workloads.bf16_bits_to_fp32(workloads.normal_bf16(rng, (256, 256), 1.0)).copy()
    x[:128, :128] = 0.0
    x[:128, 5] = -0.0
    x[:128, 7] = 0.0
    x[3, 7] = 3.0
    x[128:, :128] *= np.float32(1e-38)
    x[128:, 200] = 1e30
    for pow2 in (False, True):
        _dual_parity(fq, workloads.fp32_to_bf16_bits(x), pow2, "dual edges")


def test_dual_dense_activation_full(fq):
    """The dense workload's A [4096, 7168] (power-of-two scales): both copies in full."""
    w = workloads.dense()
    _dual_parity(fq, w.gen_a(), True, "dual dense A")
