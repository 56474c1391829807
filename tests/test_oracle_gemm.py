"""Pins of the oracle GEMM: closed forms, brute force, linearity, and planted mistakes.

The GEMM dequantizes with per-group scales along K (the-good.kr wr_id=2169793
para 1) and sums the products; its exact value is C = sum_k a~_k b~_k.
"""
import numpy as np
import pytest

import workloads


def _rand_quantized(orc, seed, M, N, K, b_rowwise=False):
    rng = np.random.default_rng(seed)
    a = workloads.normal_bf16(rng, (M, K), 1.0, 0.01)
    b = workloads.normal_bf16(rng, (N, K), 0.02)
    qa, sa = orc.quant_act_1x128(a, False)
    if b_rowwise:
        qb, sb = orc.quant_act_1x128(b, False)
    else:
        qb, sb = orc.quant_weight_128x128(b, False)
    return qa, sa, qb, sb


def test_unit_scale_integers_exact(orc):
    """Small E4M3 integers with unit scales: C must equal the integer product exactly."""
    rng = workloads.rng_for(1, 9)
    qa, ia = workloads.small_int_e4m3_codes(rng, (128, 512))
    qb, ib = workloads.small_int_e4m3_codes(rng, (256, 512))
    sa = np.ones((4, 128), np.float32)
    sb = np.ones((2, 4), np.float32)
    C, T = orc.gemm_blockscaled_ref(qa, sa, qb, sb)
    assert np.array_equal(C, (ia @ ib.T).astype(np.float64))
    assert np.array_equal(T, (np.abs(ia) @ np.abs(ib).T).astype(np.float64))


@pytest.mark.parametrize("b_rowwise", [False, True])
def test_triple_loop_matches_blas(orc, b_rowwise):
    qa, sa, qb, sb = _rand_quantized(orc, 11, 37, 256, 384, b_rowwise)
    C1, T1 = orc.gemm_blockscaled_ref(qa, sa, qb, sb, b_rowwise)
    C2, T2 = orc.gemm_triple(qa, sa, qb, sb, b_rowwise)
    assert np.all(np.abs(C1 - C2) <= 1e-12 * T2)
    assert np.allclose(T1, T2, rtol=1e-12, atol=0)


def test_linearity_per_group(orc):
    """Doubling the scales of group g adds exactly the group-g term."""
    qa, sa, qb, sb = _rand_quantized(orc, 12, 64, 128, 512)
    C, _ = orc.gemm_blockscaled_ref(qa, sa, qb, sb)
    for g in range(4):
        sa2 = sa.copy()
        sa2[g] *= 2
        C2, _ = orc.gemm_blockscaled_ref(qa, sa2, qb, sb)
        qa_g = np.zeros_like(qa)
        qa_g[:, g * 128:(g + 1) * 128] = qa[:, g * 128:(g + 1) * 128]
        Cg, Tg = orc.gemm_blockscaled_ref(qa_g, sa, qb, sb)
        assert np.all(np.abs((C2 - C) - Cg) <= 1e-13 * (np.abs(C) + Tg + 1e-300))


def test_rank_one_closed_form(orc):
    """A row of identical codes c with scale s: C[m, n] = decode(c) s sum_k b~[n, k]."""
    qa, sa, qb, sb = _rand_quantized(orc, 13, 4, 256, 256)
    qa[:] = 0x44                                  # 3.0
    sa[:] = np.float32(0.25)
    C, _ = orc.gemm_blockscaled_ref(qa, sa, qb, sb)
    Bd = orc.decode_table()[qb] * sb.astype(np.float64).repeat(128, 0).repeat(128, 1)
    want = 3.0 * 0.25 * Bd.sum(axis=1)
    assert np.allclose(C, np.broadcast_to(want, C.shape), rtol=1e-13, atol=0)


def test_grouped_equals_dense_per_expert(orc):
    rng = np.random.default_rng(14)
    counts = np.array([0, 5, 130, 1, 0, 77])
    off = workloads.offsets_from_counts(counts)
    M, N, K, E = int(off[-1]), 256, 256, len(counts)
    a = workloads.normal_bf16(rng, (M, K), 1.0)
    w = workloads.normal_bf16(rng, (E * N, K), 0.02)
    qa, sa = orc.quant_act_1x128(a, False)
    qw, sw = orc.quant_weight_128x128(w, False)
    qw, sw = qw.reshape(E, N, K), sw.reshape(E, N // 128, K // 128)
    C, T = orc.gemm_grouped_ref(qa, sa, qw, sw, off)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        Ce, Te = orc.gemm_triple(qa[lo:hi], sa[:, lo:hi], qw[e], sw[e])
        assert np.all(np.abs(C[lo:hi] - Ce) <= 1e-12 * Te)
    rows = np.array([5, 100, 212])
    Cs, Ts = orc.gemm_grouped_ref(qa, sa, qw, sw, off, rows=rows)
    assert np.all(np.abs(Cs - C[rows]) <= 1e-12 * Ts)   # BLAS blocking may differ with the row count


def test_tolerance_helpers(orc):
    ref = np.array([1.0, 1.0, 3.0, -0.0])
    T = np.array([1.0, 1.0, 3.0, 100.0])
    ok = orc.check_fp32(np.array([1.0 + 1.9e-5, 1.0 + 2.1e-5, 3.0, 1e-3]), ref, T)
    assert list(ok) == [True, False, True, True]
    assert orc.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert orc.bf16_ulp(np.array([1.99]))[0] == 2.0 ** -7
    assert orc.bf16_ulp(np.array([2.0]))[0] == 2.0 ** -6
    okb, fb = orc.check_bf16(np.array([1.0078125, 1.015625]), np.array([1.0, 1.0]),
                             np.array([1.0, 1.0]))
    assert list(okb) == [True, False] and not fb.any()


# --------------------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# --------------------------------------------------------------------------------------

def test_planted_transposed_block_scales_is_caught(orc, monkeypatch):
    qa, sa, qb, sb = _rand_quantized(orc, 15, 16, 256, 512)
    good, T = orc.gemm_triple(qa, sa, qb, sb)
    real = orc.dequant_blocks

    def wrong(q, s):                       # reads the [N/128, K/128] scales transposed
        N, K = q.shape
        st = np.resize(np.asarray(s).T.ravel(), s.shape)
        return real(q, st)

    monkeypatch.setattr(orc, "dequant_blocks", wrong)
    bad, _ = orc.gemm_blockscaled_ref(qa, sa, qb, sb)
    assert not np.all(np.abs(bad - good) <= 1e-12 * T)


def test_planted_wrong_decode_entry_is_caught(orc, monkeypatch):
    rng = workloads.rng_for(1, 9)
    qa, ia = workloads.small_int_e4m3_codes(rng, (32, 128))
    qb, ib = workloads.small_int_e4m3_codes(rng, (128, 128))
    table = orc.decode_table().copy()
    table[0x44] = 3.125                    # 3.0 decoded wrongly
    monkeypatch.setattr(orc, "decode_table", lambda: table)
    C, _ = orc.gemm_blockscaled_ref(qa, np.ones((1, 32), np.float32), qb, np.ones((1, 1), np.float32))
    assert not np.array_equal(C, (ia @ ib.T).astype(np.float64))


def test_planted_scale_without_448_is_caught(orc):
    """An amax-to-1 scale (forgetting the FP8 maximum) breaks the 448 invariant."""
    x = workloads.normal_bf16(np.random.default_rng(16), (4, 128), 1.0)
    q, s = orc.quant_act_1x128(x, False)
    xf = workloads.bf16_bits_to_fp32(x)
    s_bad = np.abs(xf).max(axis=1)         # planted: maps amax to 1, not 448
    q_bad = np.array([[orc.e4m3_encode(float(v) / float(sb)) for v in row]
                      for row, sb in zip(xf, s_bad)], dtype=np.uint8)
    assert np.all(np.abs(orc.decode_table()[q]).max(axis=1) == 448)
    assert not np.all(np.abs(orc.decode_table()[q_bad]).max(axis=1) == 448)
