"""Pins of the oracle's E4M3 codec against the format's own definition.

E4M3 (OCP 8-bit floating point, variant E4M3FN): 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest
finite value 1.75 * 2^8 = 448.  The pages (the-good.kr wr_id=2169793 para 4)
only fix "E4M3 on all tensors"; the bit layout and the round-to-nearest-even
/ saturating cast are the readings this project takes.
"""
import math

import numpy as np
import pytest

import workloads


def _value_of_fields(s, e, m):
    """Textbook value of the bit fields, written independently of the oracle."""
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_decode_all_256_codes_match_field_formula(orc):
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        v = orc.e4m3_decode(c)
        if e == 15 and m == 7:
            assert math.isnan(v), hex(c)
            continue
        assert v == _value_of_fields(s, e, m), hex(c)
        assert math.copysign(1.0, v) == (-1.0 if s else 1.0)


def test_roundtrip_every_finite_code(orc):
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert orc.e4m3_encode(orc.e4m3_decode(c)) == c, hex(c)


# (value, code, why) -- each code follows from the bit layout above.
KNOWN = [
    (1.0, 0x38, "2^0: exponent field 7, mantissa 0"),
    (448.0, 0x7E, "1.75 * 2^8: exponent 15, mantissa 6 (largest finite)"),
    (-448.0, 0xFE, "sign bit set on 0x7E"),
    (2.0 ** -6, 0x08, "smallest normal: exponent field 1"),
    (2.0 ** -9, 0x01, "smallest subnormal: 1/8 * 2^-6"),
    (0.5 * 2.0 ** -9, 0x00, "tie between 0 and 2^-9 goes to the even code 0"),
    (0.75 * 2.0 ** -9, 0x01, "above the tie rounds up"),
    (1.5 * 2.0 ** -9, 0x02, "tie between 1 and 2 (x 2^-9) goes to even 2"),
    (2.5 * 2.0 ** -9, 0x02, "tie between 2 and 3 goes to even 2"),
    (464.0, 0x7E, "tie between 448 and the non-existent 480: even mantissa 6 wins"),
    (465.0, 0x7E, "beyond the tie: saturates to the largest finite"),
    (1e6, 0x7E, "saturates"),
    (-1e30, 0xFE, "saturates with sign"),
    (-0.0, 0x80, "negative zero keeps its sign"),
    (-1e-30, 0x80, "negative underflow keeps its sign"),
    (1.0625, 0x38, "tie between 1 and 1.125 goes to even 1"),
    (1.1875, 0x3A, "tie between 1.125 and 1.25 goes to even 1.25"),
    (240.0, 0x77, "1.875 * 2^7"),
    (17.0, 0x58, "2^4 is exponent field 11; tie between 16 and 18 goes to even 16"),
    (19.0, 0x5A, "tie between 18 (mantissa 1) and 20 (mantissa 2) goes to even 20"),
]


@pytest.mark.parametrize("v,code,why", KNOWN)
def test_known_encodings(orc, v, code, why):
    assert orc.e4m3_encode(v) == code, why


def _positive_grid(orc):
    return np.array([orc.e4m3_decode(c) for c in range(0x00, 0x7F)])


def test_ties_go_to_even_and_neighbours_round_to_nearest(orc):
    grid = _positive_grid(orc)
    for i in range(len(grid) - 1):
        lo, hi = grid[i], grid[i + 1]
        mid = (lo + hi) / 2                      # exact in fp32: needs 4 significant bits
        assert np.float32(mid) == mid
        want = i if (i & 1) == 0 else i + 1     # code == index; even mantissa LSB wins
        assert orc.e4m3_encode(mid) == want, (lo, hi)
        below = float(np.nextafter(np.float32(mid), np.float32(0)))
        above = float(np.nextafter(np.float32(mid), np.float32(1e9)))
        assert orc.e4m3_encode(below) == i
        assert orc.e4m3_encode(above) == i + 1


def test_half_spacing_invariant_random(orc):
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.uniform(-448, 448, 4000),
        rng.standard_normal(4000) * 2.0 ** rng.integers(-14, 8, 4000),
    ]).astype(np.float32)
    grid = _positive_grid(orc)
    for v in vals:
        c = orc.e4m3_encode(float(v))
        d = orc.e4m3_decode(c)
        a = abs(float(v))
        j = np.searchsorted(grid, a)
        lo = grid[max(j - 1, 0)]
        hi = grid[min(j, len(grid) - 1)]
        spacing = max(hi - lo, 2.0 ** -9)
        assert abs(a - abs(d)) <= spacing / 2, v
        assert (c >> 7) == (1 if math.copysign(1, v) < 0 else 0)


def test_monotone(orc):
    rng = np.random.default_rng(3)
    vals = np.sort(rng.uniform(-500, 500, 20000).astype(np.float32))
    dec = np.array([orc.e4m3_decode(orc.e4m3_encode(float(v))) for v in vals])
    assert np.all(np.diff(dec) >= 0)


def test_cross_check_torch_cast_on_all_bf16_within_range(orc):
    """Independent library second opinion: torch.float8_e4m3fn's CPU cast (RNE)."""
    torch = pytest.importorskip("torch")
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = workloads.bf16_bits_to_fp32(bits)
    keep = np.isfinite(f) & (np.abs(f) <= 448.0)
    f = f[keep]
    ours = np.array([orc.e4m3_encode(float(v)) for v in f], dtype=np.uint8)
    theirs = torch.from_numpy(f.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != theirs)[0]
    assert bad.size == 0, [(float(f[i]), hex(ours[i]), hex(theirs[i])) for i in bad[:10]]


def test_nan_encodes_to_nan_code(orc):
    assert orc.e4m3_encode(float("nan")) == 0x7F
