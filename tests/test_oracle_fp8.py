"""Pins of the oracle's E4M3 rounding (oracle/fp8.py): values fixed by the format
(1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormal step 2^-9,
largest finite 448), and agreement with a brute-force search for the nearest of
all decoded codes (ties to the even mantissa) on random and adversarial inputs."""
import numpy as np
import pytest

from oracle import fp8


def test_decoded_codes():
    vals = [fp8.decode_e4m3(c) for c in range(256)]
    finite = [v for v in vals if not np.isnan(v)]
    assert len(finite) == 254                       # S.1111.111 is NaN for both signs
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert fp8.decode_e4m3(0x01) == 2.0 ** -9       # smallest subnormal
    assert fp8.decode_e4m3(0x08) == 2.0 ** -6       # smallest normal
    assert fp8.decode_e4m3(0x38) == 1.0             # exponent field 7 = bias
    assert fp8.decode_e4m3(0x39) == 1.125


@pytest.mark.parametrize("x,want", [
    (0.0, 0.0), (1.0, 1.0), (1.0625, 1.0),          # a tie between 1 (mantissa 000) and 1.125: to even
    (1.1875, 1.25),                                 # a tie between 1.125 (001) and 1.25 (010)
    (1.1, 1.125), (-1.0625, -1.0), (17.5, 18.0),    # binade [16, 32): step 2
    (448.0, 448.0), (460.0, 448.0), (1e4, 448.0), (-1e4, -448.0),   # saturation
    (2.0 ** -9, 2.0 ** -9), (2.0 ** -10, 0.0),      # half the smallest subnormal: a tie, to even (0)
    (3 * 2.0 ** -10, 2.0 ** -8),                    # a tie between 2^-9 (001) and 2^-8 (010)
    (0.0151, 0.015625),                             # 2^-6 = 0.015625: nearest
])
def test_hand_values(x, want):
    assert fp8.e4m3(x) == want


def _nearest_code_value(x, table, even):
    d = np.abs(table[None, :] - x[:, None])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equidistant codes take the even mantissa
    pick = np.where(cand & even[None, :], 1, 0)
    idx = np.where(pick.any(axis=1), pick.argmax(axis=1), cand.argmax(axis=1))
    return table[idx]


def test_matches_brute_force_nearest_code():
    codes = [c for c in range(256) if not np.isnan(fp8.decode_e4m3(c))]
    table = np.array([fp8.decode_e4m3(c) for c in codes])
    even = np.array([(c & 1) == 0 for c in codes])
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000) * s for s in (0.01, 0.3, 1.0, 3.0, 60.0)])
    # exact midpoints between neighbouring codes (the tie cases) inside the range
    pos = np.unique(table[table >= 0])
    x = np.concatenate([x, (pos[1:] + pos[:-1]) / 2, -(pos[1:] + pos[:-1]) / 2])
    x = x[np.abs(x) <= 448.0]
    np.testing.assert_array_equal(fp8.e4m3(x), _nearest_code_value(x, table, even))
