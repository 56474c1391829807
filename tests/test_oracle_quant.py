"""Pins of the oracle quantizers against properties the pages and arithmetic fix.

the-good.kr wr_id=2169793 para 4: the maximum absolute value of every 1x128
activation tile / 128x128 weight block is computed online and mapped to the
largest FP8 value; why-be.co.kr wr_id=72410 para 1: optional power-of-two
scales.  None of these tests retype the oracle's formula; each checks a
property that any correct implementation must have.
"""
import numpy as np
import pytest

import workloads

F32_ULP_REL = 2.0 ** -23


def _f32(bits):
    return workloads.bf16_bits_to_fp32(bits).astype(np.float64)


def _e4m3_spacing(v):
    """Spacing of E4M3 values at |v| (0 <= |v| <= 448): 2^(e-3), subnormal spacing 2^-9."""
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex - 1, -6)
    return np.exp2(e - 3.0)


def _rand_act(seed, M, K, outliers=0.001):
    return workloads.normal_bf16(np.random.default_rng(seed), (M, K), 1.0, outliers)


@pytest.mark.parametrize("pow2", [False, True])
def test_act_dequant_within_half_e4m3_spacing(orc, pow2):
    x = _rand_act(1, 64, 1024)
    q, s = orc.quant_act_1x128(x, pow2)
    xf = _f32(x)
    sc = s.astype(np.float64).T.repeat(128, axis=1)            # [M, K]
    d = orc.decode_table()[q] * sc
    quot = xf / sc
    # one fp32 rounding of the quotient happens before the cast: allow one fp32 ulp
    bound = (0.5 * _e4m3_spacing(quot) + np.abs(quot) * F32_ULP_REL) * sc
    assert np.all(np.abs(xf - d) <= bound)


def test_act_plain_scale_maps_amax_to_448(orc):
    x = _rand_act(2, 96, 768)
    q, s = orc.quant_act_1x128(x, False)
    mag = np.abs(orc.decode_table()[q]).reshape(96, 6, 128).max(axis=2)   # [M, G]
    assert np.all(mag == 448.0)
    amax = np.abs(_f32(x)).reshape(96, 6, 128).max(axis=2)
    # s * 448 recovers amax within the one rounding of the division
    assert np.all(np.abs(s.T.astype(np.float64) * 448.0 - amax) <= amax * F32_ULP_REL)


def test_act_pow2_scales(orc):
    x = _rand_act(3, 64, 512)
    q, s = orc.quant_act_1x128(x, True)
    _, s_plain = orc.quant_act_1x128(x, False)
    sb = s.view(np.uint32)
    assert np.all((sb & 0x7FFFFF) == 0), "power of two: mantissa bits clear"
    assert np.all(s >= s_plain) and np.all(s < 2 * s_plain)   # smallest power of two >= s
    mag = np.abs(orc.decode_table()[q]).reshape(64, 4, 128).max(axis=2)
    assert np.all((mag >= 224.0) & (mag <= 448.0))


def test_act_zero_tiles_and_signed_zero(orc):
    x = np.zeros((3, 256), dtype=np.uint16)
    x[1, :128] = 0x8000                        # -0.0
    x[2, 128 + 5] = workloads.fp32_to_bf16_bits(np.array([-3.0], np.float32))[0]
    q, s = orc.quant_act_1x128(x, False)
    assert np.all(s[:, 0] == 1.0) and np.all(s[:, 1] == 1.0) and s[0, 2] == 1.0
    assert np.all(q[0] == 0) and np.all(q[1, :128] == 0x80) and np.all(q[1, 128:] == 0)
    assert q[2, 128 + 5] == 0xFE and np.count_nonzero(q[2]) == 1
    assert s[1, 2] == np.float32(3.0) / np.float32(448.0)


def test_act_single_nonzero_tile(orc):
    x = np.zeros((1, 128), dtype=np.uint16)
    x[0, 77] = workloads.fp32_to_bf16_bits(np.array([1e-3], np.float32))[0]
    q, _ = orc.quant_act_1x128(x, False)
    assert q[0, 77] == 0x7E and np.count_nonzero(q) == 1


def test_act_power_of_two_rescale_leaves_codes(orc):
    """Multiplying a tile by 2^j (exact in bf16) multiplies s by 2^j and leaves q unchanged."""
    x = _rand_act(4, 16, 512, outliers=0)
    q, s = orc.quant_act_1x128(x, False)
    for j in (-20, -3, 5, 30):
        y = workloads.fp32_to_bf16_bits(workloads.bf16_bits_to_fp32(x) * np.float32(2.0 ** j))
        q2, s2 = orc.quant_act_1x128(y, False)
        assert np.array_equal(q, q2)
        assert np.array_equal(s2, s * np.float32(2.0 ** j))


def test_act_sign_symmetry_and_permutation(orc):
    x = _rand_act(5, 8, 256)
    q, s = orc.quant_act_1x128(x, False)
    q_neg, s_neg = orc.quant_act_1x128(x ^ np.uint16(0x8000), False)
    assert np.array_equal(q_neg, q ^ np.uint8(0x80)) and np.array_equal(s_neg, s)
    perm = np.random.default_rng(0).permutation(128)
    xp = x.reshape(8, 2, 128)[:, :, perm].reshape(8, 256)
    qp, sp = orc.quant_act_1x128(xp, False)
    assert np.array_equal(qp, q.reshape(8, 2, 128)[:, :, perm].reshape(8, 256))
    assert np.array_equal(sp, s)


def test_act_scale_layout_is_group_major(orc):
    """Row m, group g holds magnitude 2^(m + 3g): its scale sits at s[g, m]."""
    M, G = 5, 3
    x = np.zeros((M, G * 128), dtype=np.float32)
    for m in range(M):
        for g in range(G):
            x[m, g * 128 + 1] = 2.0 ** (m + 3 * g)
    q, s = orc.quant_act_1x128(workloads.fp32_to_bf16_bits(x), True, ld_s=8)
    assert s.shape == (G, 8)
    for m in range(M):
        for g in range(G):
            # 2^(m+3g) / 448 rounded up to a power of two is 2^(m+3g-8)
            assert s[g, m] == 2.0 ** (m + 3 * g - 8)
    assert np.all(s[:, M:] == 0)   # padding columns untouched


def test_act_tiny_magnitudes_subnormal_scales(orc):
    """amax near the bottom of bf16 gives an fp32-subnormal scale; the invariants still hold."""
    x = np.zeros((2, 128), dtype=np.float32)
    x[0] = np.linspace(-1, 1, 128) * 2.0 ** -130
    x[1] = np.linspace(-1, 1, 128) * 2.0 ** -133 * 3
    xb = workloads.fp32_to_bf16_bits(x)
    for pow2 in (False, True):
        q, s = orc.quant_act_1x128(xb, pow2)
        assert np.all(s > 0) and np.all(s < 2.0 ** -126)
        mag = np.abs(orc.decode_table()[q]).max(axis=1)
        assert np.all(mag <= 448) and np.all(mag >= (224 if pow2 else 448))


def test_weight_block_invariants(orc):
    w = workloads.normal_bf16(np.random.default_rng(6), (256, 384), 0.006)
    w[130, 200] = workloads.fp32_to_bf16_bits(np.array([5.0], np.float32))[0]   # block (1, 1)
    for pow2 in (False, True):
        q, s = orc.quant_weight_128x128(w, pow2)
        assert s.shape == (2, 3)
        wf = _f32(w)
        sc = s.astype(np.float64).repeat(128, axis=0).repeat(128, axis=1)
        d = orc.decode_table()[q] * sc
        quot = wf / sc
        bound = (0.5 * _e4m3_spacing(quot) + np.abs(quot) * F32_ULP_REL) * sc
        assert np.all(np.abs(wf - d) <= bound)
        blk_max = np.abs(orc.decode_table()[q]).reshape(2, 128, 3, 128).max(axis=(1, 3))
        if pow2:
            assert np.all((s.view(np.uint32) & 0x7FFFFF) == 0)
            assert np.all((blk_max >= 224) & (blk_max <= 448))
        else:
            assert np.all(blk_max == 448)
    # the outlier raises the scale of its own block only
    _, s = orc.quant_weight_128x128(w, False)
    assert s[1, 1] == np.float32(5.0) / np.float32(448.0)
    assert np.all(np.delete(s.ravel(), 4) < 0.1 / 448)


def test_weight_block_equals_act_tiles_when_rows_share_amax(orc):
    """If every row of a 128x128 block carries the block maximum, the block's one scale
    equals every row tile's scale, so the two quantizers must agree byte for byte."""
    rng = np.random.default_rng(8)
    w = rng.uniform(-1, 1, (128, 256)).astype(np.float32)
    w[:, 3] = 2.0
    w[:, 131] = -2.0
    wb = workloads.fp32_to_bf16_bits(w)
    qw, sw = orc.quant_weight_128x128(wb, False)
    qa, sa = orc.quant_act_1x128(wb, False)
    assert np.array_equal(qw, qa)
    assert np.all(sa == sw[0][:, None])


def test_rowwise_invariants(orc):
    x = _rand_act(9, 8, 2048)
    q, s = orc.quant_rowwise(x)
    assert np.all(np.abs(orc.decode_table()[q]).max(axis=1) == 448)
    # with one 128-wide group the row quantizer is the tile quantizer
    q1, s1 = orc.quant_rowwise(x[:, :128])
    qa, sa = orc.quant_act_1x128(x[:, :128], False)
    assert np.array_equal(q1, qa) and np.array_equal(s1, sa[0])


def test_weight_blocks_are_symmetric_under_transposition(orc):
    """A 128x128 block's amax is that of its transpose: quantizing W^T gives the transposed
    codes and scales of W (the Dgrad operand needs no requantization)."""
    w = workloads.normal_bf16(np.random.default_rng(31), (256, 384), 0.02, 0.001)
    q, s = orc.quant_weight_128x128(w, False)
    qt, st = orc.quant_weight_128x128(np.ascontiguousarray(w.T), False)
    assert np.array_equal(qt, q.T) and np.array_equal(st, s.T)
