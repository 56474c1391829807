"""Pins of the oracle's one-scale-per-tensor quantizer (the coarse baseline of the
outlier study) and the study's central claim on the tiny workload.

the-good.kr wr_id=2169793 para 4: mapping the maximum absolute value of the whole input
tensor to the largest FP8 value leaves low-precision training very sensitive to activation
outliers; pkd.ac.th webboard 78017 para 1: scaling at a finer grain is the remedy.
"""
import numpy as np
import pytest

import workloads
from oracle import outlier_study

F32_ULP_REL = 2.0 ** -23


def _f32(bits):
    return workloads.bf16_bits_to_fp32(bits).astype(np.float64)


def _e4m3_spacing(v):
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    return np.exp2(np.maximum(ex - 1, -6) - 3.0)


def _act(seed, shape, outliers=0.001):
    return workloads.normal_bf16(np.random.default_rng(seed), shape, 1.0, outliers)


def test_tensorwise_scale_maps_the_tensor_amax_to_448(orc):
    x = _act(1, (96, 640))
    q, s = orc.quant_tensorwise(x)
    amax = np.abs(_f32(x)).max()
    assert abs(s * 448.0 - amax) <= amax * F32_ULP_REL
    assert np.abs(orc.decode_table()[q]).max() == 448.0


@pytest.mark.parametrize("pow2", [False, True])
def test_tensorwise_dequant_within_half_e4m3_spacing(orc, pow2):
    x = _act(2, (64, 384))
    q, s = orc.quant_tensorwise(x, pow2)
    xf = _f32(x)
    quot = xf / s
    bound = (0.5 * _e4m3_spacing(quot) + np.abs(quot) * F32_ULP_REL) * s
    assert np.all(np.abs(xf - orc.decode_table()[q] * s) <= bound)


def test_tensorwise_pow2_scale(orc):
    x = _act(3, (32, 256))
    _, s2 = orc.quant_tensorwise(x, True)
    _, s = orc.quant_tensorwise(x, False)
    m, _ = np.frexp(s2)
    assert m == 0.5 and s2 >= s and s2 < 2 * s


def test_tensorwise_of_one_tile_is_the_tile_quantizer(orc):
    x = _act(4, (1, 128))
    q, s = orc.quant_tensorwise(x)
    qa, sa = orc.quant_act_1x128(x, False)
    assert np.array_equal(q, qa) and s == float(sa[0, 0])


def test_tensorwise_outlier_shrinks_every_other_code(orc):
    """One element x1000 sets the scale: the remaining codes are those of the tensor
    divided by a 1000x larger scale (planted on the host, decided by the definition)."""
    x = workloads.normal_bf16(np.random.default_rng(5), (16, 128), 1.0)
    xf = workloads.bf16_bits_to_fp32(x)
    y = xf.copy()
    y[3, 7] = np.abs(xf).max() * 1000.0
    yb = workloads.fp32_to_bf16_bits(y)
    q, s = orc.quant_tensorwise(yb)
    _, s0 = orc.quant_tensorwise(x)
    assert s > 900 * s0
    mask = np.ones_like(q, bool)
    mask[3, 7] = False
    assert np.abs(orc.decode_table()[q][mask]).max() < 448.0 / 500


def test_outlier_sensitivity_of_one_scale_per_tensor():
    """Tiny shapes, 0.1% outliers x f: as f grows, one scale per tensor pushes the bulk of
    the tensor towards E4M3's subnormal range and then to zero codes, while 1x128 tiles keep
    it; without outliers the two are alike.  (E4M3 spans ~18 binades, so the loss is small
    up to f ~ 10^3 and total by f = 10^5, where ordinary values fall below 2^-9 s.)"""
    r = outlier_study.study_tiny()
    keys = ("x1", "x100", "x1000", "x10000", "x100000")
    fine = [r[k]["fine"]["bulk_rel_error"] for k in keys]
    zero = [r[k]["tensor"]["bulk_zero_share"] for k in keys]
    assert r["x1"]["tensor"]["bulk_rel_error"] < 1.5 * fine[0]   # no outliers: comparable
    assert all(z1 <= z2 for z1, z2 in zip(zero, zero[1:]))        # zero codes only grow
    assert zero[-1] > 0.3                                          # x10^5: much of the bulk is lost
    assert r["x100000"]["tensor"]["bulk_rel_error"] > 4 * fine[-1]
    # 1x128 tiles: only the ~13% of tiles that hold an outlier lose their other values
    assert max(fine[:4]) < 1.1 * fine[0] and fine[-1] < 0.1
    assert max(r[k]["fine"]["bulk_zero_share"] for k in keys) < 0.05
