"""GPU parity of the block-scaled FP8 GEMMs against the FP64 oracle, through the C ABI.

Acceptance: fp32 output |C - C_ref| <= 2e-5 sum_k|a~ b~| + 1e-30; bf16 output within
1 bf16 ulp of C_ref (cancellation fallback: the bf16 rounding of a value inside the
fp32 band); the unit-scale integer case bit-exact.  Inputs are quantized by each side
on its own (the GPU's codes are first checked bit-exact against the oracle's).
"""
import numpy as np
import pytest

import oracle
import workloads
from tests._helpers import (assert_bytes_equal, assert_gemm_close, host, rel_err_stats, to_dev,
                            to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


def _dense_case(fq, a_bits, b_bits, pow2_a, pow2_b, out_fp32, b_rowwise=False, rows=None,
                name="dense", ue8m0=False):
    """Quantize on both sides, check the codes, run the GEMM, compare (sampled) rows.
    ue8m0: the power-of-two-scale GEMM that scales inside the tensor core."""
    import torch
    a, b = to_dev_bf16(a_bits), to_dev_bf16(b_bits)
    qa, sa = fq.quant_act_1x128(a, pow2_a)
    if b_rowwise:
        qb, sb = fq.quant_act_1x128(b, pow2_b)
    else:
        qb, sb = fq.quant_weight_128x128(b, pow2_b)
    out_dtype = torch.float32 if out_fp32 else torch.bfloat16
    gemm = fq.gemm_blockscaled_ue8m0 if ue8m0 else fq.gemm_blockscaled
    C = gemm(qa, sa, qb, sb, out_dtype=out_dtype, b_rowwise=b_rowwise)
    torch.cuda.synchronize()
    assert fq.device_error() == 0

    rows = np.arange(a_bits.shape[0]) if rows is None else np.asarray(rows)
    qa_ref, sa_ref = oracle.quant_act_1x128(a_bits[rows], pow2_a)
    if b_rowwise:
        qb_ref, sb_ref = oracle.quant_act_1x128(b_bits, pow2_b)
    else:
        qb_ref, sb_ref = oracle.quant_weight_128x128(b_bits, pow2_b)
    assert_bytes_equal(name + ".qa", host(qa)[rows], qa_ref)
    assert_bytes_equal(name + ".qb", host(qb), qb_ref)
    C_ref, T = oracle.gemm_blockscaled_ref(qa_ref, sa_ref, qb_ref, sb_ref, b_rowwise)
    Ch = host(C)[rows]
    fb = assert_gemm_close(name, Ch, C_ref, T, bf16=not out_fp32)
    return Ch, C_ref, T, fb


def test_tiny_fp32(fq):
    w = workloads.tiny()
    C, C_ref, T, _ = _dense_case(fq, w.gen_a(), w.gen_b(), False, False, True, name="tiny")
    mx, med = rel_err_stats(C, C_ref, T)
    assert mx <= 2e-5


def test_tiny_unit_scale_integers_exact(fq):
    """qA, qB small E4M3 integers, unit scales: every partial sum is an integer below 2^14,
    so the result must equal the integer product exactly."""
    import torch
    rng = workloads.rng_for(1, 9)
    qa, ia = workloads.small_int_e4m3_codes(rng, (128, 512))
    qb, ib = workloads.small_int_e4m3_codes(rng, (256, 512))
    sa = np.ones((4, 128), np.float32)
    sb = np.ones((2, 4), np.float32)
    C = fq.gemm_blockscaled(to_dev(qa), to_dev(sa), to_dev(qb), to_dev(sb), out_dtype=torch.float32)
    want = (ia @ ib.T).astype(np.float32)
    assert_bytes_equal("unit-scale C", host(C), want)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (129, 256, 128), (200, 384, 640),
                                   (257, 512, 256), (64, 128, 1024), (300, 1280, 384)])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_ragged_shapes(fq, M, N, K, out_fp32):
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    a = workloads.normal_bf16(rng, (M, K), 1.0, 0.01)
    b = workloads.normal_bf16(rng, (N, K), 0.02)
    _dense_case(fq, a, b, False, False, out_fp32, name=f"ragged {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K,rowwise", [(128, 256, 512, False), (300, 1280, 1024, False),
                                           (4096, 7168, 1024, False), (2048, 512, 2048, True)])
def test_split_last_wave_matches_unsplit(fq, M, N, K, rowwise):
    """With a workspace the last partial wave is split along K; the result is deterministic
    and inside the band of the unsplit result (and both inside the oracle's band)."""
    import torch
    rng = np.random.default_rng(M + N + K)
    a = workloads.normal_bf16(rng, (M, K), 1.0, 0.001)
    b = workloads.normal_bf16(rng, (N, K), 0.02 if not rowwise else 1.0)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a), False)
    qb, sb = (fq.quant_act_1x128(to_dev_bf16(b), False) if rowwise
              else fq.quant_weight_128x128(to_dev_bf16(b), False))
    assert fq.workspace_bytes(M, N, K) > 0
    C1 = fq.gemm_blockscaled(qa, sa, qb, sb, out_dtype=torch.float32, b_rowwise=rowwise, split_k=True)
    C1b = fq.gemm_blockscaled(qa, sa, qb, sb, out_dtype=torch.float32, b_rowwise=rowwise, split_k=True)
    C0 = fq.gemm_blockscaled(qa, sa, qb, sb, out_dtype=torch.float32, b_rowwise=rowwise, split_k=False)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    assert torch.equal(C1, C1b), "split result is deterministic"
    rows = np.unique(np.concatenate([np.arange(0, M, max(1, M // 48)), [M - 1]]))
    qa_r, sa_r = oracle.quant_act_1x128(a[rows], False)
    qb_r, sb_r = oracle.quant_act_1x128(b, False) if rowwise else oracle.quant_weight_128x128(b, False)
    C_ref, T = oracle.gemm_blockscaled_ref(qa_r, sa_r, qb_r, sb_r, rowwise)
    assert_gemm_close("split", host(C1)[rows], C_ref, T, bf16=False)
    assert_gemm_close("unsplit", host(C0)[rows], C_ref, T, bf16=False)


@pytest.mark.parametrize("M,N,K", [(77, 256, 512), (128, 384, 256)])
def test_rowwise_b_scales(fq, M, N, K):
    rng = np.random.default_rng(M * N)
    a = workloads.normal_bf16(rng, (M, K), 1e-3)
    b = workloads.normal_bf16(rng, (N, K), 1.0)
    _dense_case(fq, a, b, False, False, True, b_rowwise=True, name="row-b")


def test_linearity_per_group_on_gpu(fq):
    """Doubling the A scales of group g adds the group-g term (within the fp32 band)."""
    import torch
    rng = np.random.default_rng(21)
    a = workloads.normal_bf16(rng, (128, 512), 1.0)
    b = workloads.normal_bf16(rng, (256, 512), 0.02)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a), False)
    qb, sb = fq.quant_weight_128x128(to_dev_bf16(b), False)
    C0 = host(fq.gemm_blockscaled(qa, sa, qb, sb, out_dtype=torch.float32)).astype(np.float64)
    qa_ref, sa_ref = oracle.quant_act_1x128(a, False)
    qb_ref, sb_ref = oracle.quant_weight_128x128(b, False)
    for g in range(4):
        sa2 = sa.clone()
        sa2[g] *= 2
        C2 = host(fq.gemm_blockscaled(qa, sa2, qb, sb, out_dtype=torch.float32)).astype(np.float64)
        qg = qa_ref.copy()
        mask = np.ones(512, bool)
        mask[g * 128:(g + 1) * 128] = False
        qg[:, mask] = 0
        Cg, Tg = oracle.gemm_blockscaled_ref(qg, sa_ref, qb_ref, sb_ref)
        _, T = oracle.gemm_blockscaled_ref(qa_ref, sa_ref, qb_ref, sb_ref)
        assert np.all(np.abs((C2 - C0) - Cg) <= 2e-5 * (2 * T + Tg) + 1e-30)


def test_dense_full_size_sampled_rows(fq):
    """The dense workload at full size, in the bench's launch configuration; 96 sampled
    rows (spanning every M tile and the last row) compared with the oracle."""
    w = workloads.dense()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(w.M, 94, replace=False), [0, w.M - 1]]))
    _, _, _, fb = _dense_case(fq, w.gen_a(), w.gen_b(), True, True, False, rows=rows,
                              name="dense full")


def test_wgrad_full_size_sampled_rows(fq):
    w = workloads.wgrad()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([rng.choice(w.M, 30, replace=False), [w.M - 1]]))
    C, C_ref, T, _ = _dense_case(fq, w.gen_a(), w.gen_b(), False, False, True, b_rowwise=True,
                                 rows=rows, name="wgrad full")


# ------------------------------------------------------------------------------------ grouped

def _grouped_case(fq, counts, N, K, pow2_a, out_fp32, a_std=1.0, b_std=0.006, rows=None,
                  seed=0, bits=None, name="grouped", alloc_rows=1, pow2_w=False, ue8m0=False):
    import torch
    counts = np.asarray(counts, dtype=np.int64)
    E = counts.size
    off = workloads.offsets_from_counts(counts)
    M = int(off[-1])
    if bits is None:
        rng = np.random.default_rng(seed)
        a_bits = workloads.normal_bf16(rng, (max(M, alloc_rows), K), a_std, 0.001)
        w_bits = workloads.normal_bf16(rng, (E, N, K), b_std)
    else:
        a_bits, w_bits = bits
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a_bits), pow2_a)
    qw, sw = fq.quant_weight_128x128(to_dev_bf16(w_bits), pow2_w)
    out_dtype = torch.float32 if out_fp32 else torch.bfloat16
    C = torch.full((max(M, alloc_rows), N), float("nan"), dtype=out_dtype, device="cuda")
    gemm = fq.gemm_grouped_ue8m0 if ue8m0 else fq.gemm_grouped
    gemm(qa, sa, qw, sw, to_dev(off), out_dtype=out_dtype, out=C)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    assert torch.isnan(C[M:]).all(), "rows past the last offset are not written"
    if M == 0:
        return
    rows = np.arange(M) if rows is None else np.asarray(rows)
    qa_ref, sa_ref = oracle.quant_act_1x128(a_bits[rows], pow2_a)
    assert_bytes_equal(name + ".qa", host(qa)[rows], qa_ref)
    # experts touched by the sampled rows
    expert = np.searchsorted(off, rows, side="right") - 1
    qw_h, sw_h = host(qw), host(sw)
    for e in np.unique(expert):
        q_ref, s_ref = oracle.quant_weight_128x128(w_bits[e], pow2_w)
        assert_bytes_equal(f"{name}.qw[{e}]", qw_h[e], q_ref)
        assert_bytes_equal(f"{name}.sw[{e}]", sw_h[e], s_ref)
    # oracle over the sampled rows: sA columns re-indexed to the sampled rows
    qa_full = np.zeros((M, K), np.uint8)
    qa_full[rows] = qa_ref
    sa_full = np.zeros((K // 128, M), np.float32)
    sa_full[:, rows] = sa_ref
    qw_ref = np.stack([oracle.quant_weight_128x128(w_bits[e], pow2_w)[0] if e in expert else
                       np.zeros((N, K), np.uint8) for e in range(E)])
    sw_ref = np.stack([oracle.quant_weight_128x128(w_bits[e], pow2_w)[1] if e in expert else
                       np.ones((N // 128, K // 128), np.float32) for e in range(E)])
    C_ref, T = oracle.gemm_grouped_ref(qa_full, sa_full, qw_ref, sw_ref, off, rows=rows)
    assert_gemm_close(name, host(C)[rows], C_ref, T, bf16=not out_fp32)


@pytest.mark.parametrize("out_fp32", [True, False])
def test_grouped_small_with_empty_groups(fq, out_fp32):
    _grouped_case(fq, [0, 5, 130, 1, 0, 77, 256, 0], 256, 384, False, out_fp32, seed=1)


@pytest.mark.parametrize("out_fp32", [True, False])
def test_grouped_ragged_with_slack_rows(fq, out_fp32):
    """Ragged experts (1..600 rows, some empty), N = 384, and an A allocation of 4096 rows
    of which only the first 983 belong to experts: the slack rows stay unwritten."""
    _grouped_case(fq, [0, 5, 300, 1, 0, 77, 600, 0], 384, 384, False, out_fp32, seed=5,
                  alloc_rows=4096)


@pytest.mark.parametrize("out_fp32", [True, False])
def test_grouped_decode_expert_sizes(fq, out_fp32):
    """Experts of 1, 16, 128, 129 and 256 tokens: one and two row tiles, nearly empty and
    full ones."""
    _grouped_case(fq, [1, 16, 128, 129, 256], 384, 512, True, out_fp32, seed=41, name="expert sizes")


def test_grouped_unwritten_rows_untouched(fq):
    """Rows past the last offset (allocation slack) are not written."""
    import torch
    rng = np.random.default_rng(2)
    counts = np.array([3, 0, 40])
    off = workloads.offsets_from_counts(counts)
    a = workloads.normal_bf16(rng, (64, 256), 1.0)
    w = workloads.normal_bf16(rng, (3, 128, 256), 0.02)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a), False)
    qw, sw = fq.quant_weight_128x128(to_dev_bf16(w), False)
    C = torch.full((64, 128), 7.0, dtype=torch.float32, device="cuda")
    fq.gemm_grouped(qa, sa, qw, sw, to_dev(off), out_dtype=torch.float32, out=C)
    assert np.all(host(C)[43:] == 7.0)


def test_grouped_all_empty(fq):
    _grouped_case(fq, [0, 0, 0], 128, 256, False, True, seed=3)


def test_grouped_decode_full_size(fq):
    """64 experts, M_e ~ U{1..256}, W [7168, 2048]; every 9th row compared."""
    w = workloads.decode()
    rows = np.arange(0, w.M, 9)
    _grouped_case(fq, w.counts, w.N, w.K, True, False, rows=rows, bits=(w.gen_a(), w.gen_b()),
                  name="decode full")


def test_grouped_prefill_full_size(fq):
    """32 experts, Zipf routing (sum M ~ 87K), W [4096, 7168]; sampled rows of 4 experts."""
    w = workloads.prefill()
    off = w.offsets
    rng = np.random.default_rng(4)
    rows = []
    for e in (0, 1, 17, 31):
        lo, hi = int(off[e]), int(off[e + 1])
        rows += list(rng.choice(np.arange(lo, hi), 12, replace=False)) + [hi - 1]
    _grouped_case(fq, w.counts, w.N, w.K, False, False, rows=np.array(sorted(set(rows))),
                  bits=(w.gen_a(), w.gen_b()), name="prefill full")


# ------------------------------------------------------------------------------ no promotion

def test_nopromo_matches_oracle_on_rowwise_codes(fq):
    """One accumulator over all of K: compared with FP64 on the same 1xK codes."""
    import torch
    rng = np.random.default_rng(6)
    a = workloads.normal_bf16(rng, (200, 2048), 1e-3)
    b = workloads.normal_bf16(rng, (256, 2048), 1.0)
    qa, sa = fq.quant_rowwise(to_dev_bf16(a))
    qb, sb = fq.quant_rowwise(to_dev_bf16(b))
    C = fq.gemm_nopromo(qa, sa, qb, sb)
    qa_r, sa_r = oracle.quant_rowwise(a)
    qb_r, sb_r = oracle.quant_rowwise(b)
    assert_bytes_equal("nopromo.qa", host(qa), qa_r)
    C_ref, T = oracle.gemm_ref(oracle.dequant_rowwise(qa_r, sa_r), oracle.dequant_rowwise(qb_r, sb_r))
    # no acceptance band is claimed for this variant; it must still be a close FP32 result
    mx, _ = rel_err_stats(host(C), C_ref, T)
    assert mx < 1e-3


# ------------------------------------------------------- power-of-two scales in the MMA

def _spread_scales(rng, bits, rows_per_block, span=24):
    """Multiply each (row block, 128-column group) of a bf16 matrix by 2^u, u uniform in
    [-span, span], so that neighbouring rows / columns / groups get very different
    power-of-two scales (a wrong row, column or group in the scale layout shows up as an
    error of a power of two)."""
    R, K = bits.shape
    x = workloads.bf16_bits_to_fp32(bits).astype(np.float64)
    nb, G = -(-R // rows_per_block), K // 128
    u = rng.integers(-span, span + 1, size=(nb, G))
    f = np.repeat(np.repeat(np.exp2(u), rows_per_block, axis=0)[:R], 128, axis=1)
    return workloads.fp32_to_bf16_bits((x * f).astype(np.float32))


def test_ue8m0_tiny_fp32(fq):
    w = workloads.tiny()
    C, C_ref, T, _ = _dense_case(fq, w.gen_a(), w.gen_b(), True, True, True, name="ue8m0 tiny",
                                 ue8m0=True)
    mx, _ = rel_err_stats(C, C_ref, T)
    assert mx <= 2e-5


def test_ue8m0_unit_scale_integers_exact(fq):
    """Small E4M3 integers with unit scales (UE8M0 byte 127): the exact integer product."""
    import torch
    rng = workloads.rng_for(1, 9)
    qa, ia = workloads.small_int_e4m3_codes(rng, (128, 512))
    qb, ib = workloads.small_int_e4m3_codes(rng, (384, 512))   # 224 + a ragged 160
    sa = np.ones((4, 128), np.float32)
    sb = np.ones((3, 4), np.float32)
    C = fq.gemm_blockscaled_ue8m0(to_dev(qa), to_dev(sa), to_dev(qb), to_dev(sb),
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    assert_bytes_equal("ue8m0 unit-scale C", host(C), (ia @ ib.T).astype(np.float32))


@pytest.mark.parametrize("out_fp32", [True, False])
@pytest.mark.parametrize("M,N,K", [(300, 512, 640), (129, 1280, 384)])
def test_ue8m0_spread_scales(fq, M, N, K, out_fp32):
    """Per-row-tile / per-block scales spread over 2^-24 .. 2^24, group counts that are not
    multiples of 4 (K = 640, 384: a scale slot holds four groups), ragged M and N."""
    rng = np.random.default_rng(M * 7 + N + K)
    a = _spread_scales(rng, workloads.normal_bf16(rng, (M, K), 1.0, 0.001), 1)
    b = _spread_scales(rng, workloads.normal_bf16(rng, (N, K), 0.02), 128)
    _dense_case(fq, a, b, True, True, out_fp32, name=f"ue8m0 spread {M}x{N}x{K}", ue8m0=True)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (129, 256, 128), (200, 384, 640),
                                   (257, 512, 256), (64, 128, 1024), (300, 1280, 384),
                                   (513, 2048, 1152)])
def test_ue8m0_ragged_shapes(fq, M, N, K):
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    a = workloads.normal_bf16(rng, (M, K), 1.0, 0.01)
    b = workloads.normal_bf16(rng, (N, K), 0.02)
    _dense_case(fq, a, b, True, True, False, name=f"ue8m0 ragged {M}x{N}x{K}", ue8m0=True)


@pytest.mark.parametrize("M,N,K", [(77, 256, 512), (128, 384, 384)])
def test_ue8m0_rowwise_b_scales(fq, M, N, K):
    rng = np.random.default_rng(M * N + 1)
    a = _spread_scales(rng, workloads.normal_bf16(rng, (M, K), 1e-3), 1, span=8)
    b = _spread_scales(rng, workloads.normal_bf16(rng, (N, K), 1.0), 1, span=8)
    _dense_case(fq, a, b, True, True, True, b_rowwise=True, name="ue8m0 row-b", ue8m0=True)


def test_ue8m0_long_k_rowwise(fq):
    """K = 16384 (128 groups, 32 scale slots per tile) with 1x128 scales on both operands,
    the wgrad shape at 512 x 640; all rows against the oracle."""
    rng = np.random.default_rng(77)
    a = _spread_scales(rng, workloads.normal_bf16(rng, (512, 16384), 1e-3), 1, span=6)
    b = workloads.normal_bf16(rng, (640, 16384), 1.0)
    _dense_case(fq, a, b, True, True, True, b_rowwise=True, name="ue8m0 long K", ue8m0=True)


def test_ue8m0_dense_full_size_sampled_rows(fq):
    """The dense workload (power-of-two scales) at full size through the tensor-core-scaled
    GEMM; 96 sampled rows spanning every M tile and the last row."""
    w = workloads.dense()
    rng = np.random.default_rng(10)
    rows = np.unique(np.concatenate([rng.choice(w.M, 94, replace=False), [0, w.M - 1]]))
    _dense_case(fq, w.gen_a(), w.gen_b(), True, True, False, rows=rows, name="ue8m0 dense full",
                ue8m0=True)


def test_ue8m0_rejects_scales_that_are_not_powers_of_two(fq):
    """FP32 (non power-of-two) scales cannot be UE8M0 bytes: the kernel finishes, records
    (8 << 8) | FP8Q_ERR_SCALE in the device error word, and the next call is clean."""
    import torch
    w = workloads.tiny()
    qa, sa = fq.quant_act_1x128(to_dev_bf16(w.gen_a()), False)
    qb, sb = fq.quant_weight_128x128(to_dev_bf16(w.gen_b()), False)
    assert not bool(torch.all(torch.frexp(sa)[0] == 0.5))     # some scale is not 2^e
    fq.gemm_blockscaled_ue8m0(qa, sa, qb, sb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fq.device_error() == (8 << 8) | 7
    assert fq.device_error() == 0                                # read and cleared
    qa2, sa2 = fq.quant_act_1x128(to_dev_bf16(w.gen_a()), True)
    qb2, sb2 = fq.quant_weight_128x128(to_dev_bf16(w.gen_b()), True)
    fq.gemm_blockscaled_ue8m0(qa2, sa2, qb2, sb2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fq.device_error() == 0


# ------------------------------------------- grouped, power-of-two scales in the MMA

@pytest.mark.parametrize("out_fp32", [True, False])
def test_grouped_ue8m0_ragged_with_empty_groups(fq, out_fp32):
    """Ragged experts (some empty), N = 384 (a full and a ragged 224-column tile), K = 640
    (a partial scale slot), slack rows in A; power-of-two scales on both operands."""
    _grouped_case(fq, [0, 5, 300, 1, 0, 77, 600, 0], 384, 640, True, out_fp32, seed=6,
                  alloc_rows=1100, pow2_w=True, ue8m0=True, name="grouped ue8m0")


def test_grouped_ue8m0_all_empty(fq):
    """Every expert empty: no tiles, the call is a clean no-op (C untouched)."""
    _grouped_case(fq, [0, 0, 0], 256, 256, True, True, seed=10, pow2_w=True, ue8m0=True,
                  name="grouped ue8m0 empty")


@pytest.mark.parametrize("ue8m0", [False, True])
def test_grouped_maximum_expert_count(fq, ue8m0):
    """1024 experts (the largest table the kernels hold), all but the first, a middle and
    the last one empty: the tile table's ends and its binary search."""
    counts = np.zeros(1024, np.int64)
    counts[0], counts[511], counts[1023] = 5, 130, 7
    _grouped_case(fq, counts, 128, 256, True, True, seed=11, pow2_w=ue8m0, ue8m0=ue8m0,
                  name=f"1024 experts ue8m0={ue8m0}")


def test_grouped_ue8m0_decode_full_size(fq):
    """The decode workload with power-of-two weight scales: 64 experts, M_e ~ U{1..256},
    W [7168, 2048]; every 9th row compared."""
    w = workloads.decode()
    rows = np.arange(0, w.M, 9)
    _grouped_case(fq, w.counts, w.N, w.K, True, False, rows=rows, bits=(w.gen_a(), w.gen_b()),
                  pow2_w=True, ue8m0=True, name="decode ue8m0")


def test_grouped_ue8m0_prefill_sampled(fq):
    """32 experts, Zipf routing (sum M ~ 87K), W [4096, 7168], power-of-two scales; sampled
    rows of 4 experts."""
    w = workloads.prefill()
    off = w.offsets
    rng = np.random.default_rng(8)
    rows = []
    for e in (0, 3, 17, 31):
        lo, hi = int(off[e]), int(off[e + 1])
        rows += list(rng.choice(np.arange(lo, hi), 10, replace=False)) + [lo, hi - 1]
    _grouped_case(fq, w.counts, w.N, w.K, True, False, rows=np.array(sorted(set(rows))),
                  bits=(w.gen_a(), w.gen_b()), pow2_w=True, ue8m0=True, name="prefill ue8m0")


def test_grouped_ue8m0_rejects_fp32_weight_scales(fq):
    import torch
    rng = np.random.default_rng(9)
    a = workloads.normal_bf16(rng, (200, 256), 1.0)
    w = workloads.normal_bf16(rng, (2, 256, 256), 0.02)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(a), True)
    qw, sw = fq.quant_weight_128x128(to_dev_bf16(w), False)       # FP32 scales
    off = to_dev(workloads.offsets_from_counts(np.array([120, 80])))
    fq.gemm_grouped_ue8m0(qa, sa, qw, sw, off)
    torch.cuda.synchronize()
    assert fq.device_error() == (8 << 8) | 7
