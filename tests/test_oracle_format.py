"""Pins of the oracle's format tables and roundings against what the formats fix.

Nothing here calls the CUDA path.  Independent references used:
  * the literal 16-entry E2M1 value set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6};
  * the E4M3 closed form (-1)^s 2^(e-7) (1 + m/8), subnormals m 2^-9, NaN at
    S.1111.111 (written here with exact fractions), and torch.float8_e4m3fn;
  * brute-force nearest-even rounding over exact fractions.
"""
from fractions import Fraction as F
import math

import numpy as np
import pytest
import torch

import oracle

E2M1_SET = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_closed_form(b):
    s, e, m = b >> 7, (b >> 3) & 0xF, b & 7
    if e == 15 and m == 7:
        return None
    v = F(m, 512) if e == 0 else F(8 + m, 8) * (F(2) ** (e - 7))
    return -v if s else v


def nearest_even(v: F, table):
    """Index of the entry of the sorted non-negative `table` (Fractions) nearest
    to v >= 0, ties to the even index, values above the top saturating."""
    best = None
    for i, t in enumerate(table):
        d = abs(v - t)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_e2m1_value_set():
    got = [oracle.e2m1_value(c) for c in range(16)]
    assert got[:8] == E2M1_SET
    assert got[8:] == [-x for x in E2M1_SET]
    assert math.copysign(1.0, got[8]) == -1.0      # code 0x8 is -0


def test_e4m3_all_256_closed_form():
    for b in range(256):
        ref = e4m3_closed_form(b)
        got = oracle.e4m3_value(b)
        if ref is None:
            assert math.isnan(got), hex(b)
        else:
            assert F(got) == ref, hex(b)
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_all_256_match_torch():
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        got = oracle.e4m3_value(b)
        if math.isnan(t[b]):
            assert math.isnan(got)
        else:
            assert got == t[b], hex(b)


POS_E4M3 = [e4m3_closed_form(b) for b in range(0x7F)]


def test_e4m3_rne_midpoints_and_exact_values():
    for c in range(0x7E):
        lo, hi = POS_E4M3[c], POS_E4M3[c + 1]
        mid = (lo + hi) / 2
        assert oracle.e4m3_rne(float(lo)) == c
        # a midpoint goes to the even code; floats just either side go to the neighbours
        if float(mid) == mid:
            assert oracle.e4m3_rne(float(mid)) == (c if c % 2 == 0 else c + 1), hex(c)
            below = np.nextafter(np.float32(mid), np.float32(0))
            above = np.nextafter(np.float32(mid), np.float32(1e9))
            assert oracle.e4m3_rne(float(below)) == c
            assert oracle.e4m3_rne(float(above)) == c + 1


def test_e4m3_rne_saturates():
    assert oracle.e4m3_rne(448.0) == 0x7E
    assert oracle.e4m3_rne(460.0) == 0x7E
    assert oracle.e4m3_rne(1e30) == 0x7E
    assert oracle.e4m3_rne(0.0) == 0x00


def test_e4m3_rne_bruteforce_random():
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-12, 6.1, 3000))]).astype(np.float32)
    for v in vals:
        expect = nearest_even(F(float(v)), POS_E4M3) if v < 448 else 0x7E
        assert oracle.e4m3_rne(float(v)) == expect, float(v)


def test_e4m3_rne_matches_torch_in_range():
    rng = np.random.default_rng(8)
    vals = np.exp(rng.uniform(-11, 6.1, 20000)).astype(np.float32)
    vals = vals[vals <= 448]
    t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne(float(v)) for v in vals])
    assert (got == t).all()


E2M1_POS = [F(x) for x in E2M1_SET]


@pytest.mark.parametrize(
    "v,code",
    [(0.0, 0x0), (0.25, 0x0), (0.2500001, 0x1), (0.5, 0x1), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4),
     (2.5, 0x4), (3.5, 0x6), (5.0, 0x6), (5.0001, 0x7), (6.0, 0x7), (7.0, 0x7), (1e9, 0x7),
     (-0.0, 0x8), (-0.1, 0x8), (-0.75, 0xA), (-5.5, 0xF), (-100.0, 0xF)],
)
def test_e2m1_rne_vectors(v, code):
    # Ties go to the even code: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4;
    # the sign is kept, so a negative value that rounds to zero is -0 (0x8).
    assert oracle.e2m1_rne(v) == code


def test_e2m1_rne_bruteforce_random():
    rng = np.random.default_rng(9)
    vals = rng.uniform(-8, 8, 5000).astype(np.float32)
    for v in vals:
        a = abs(F(float(v)))
        mag = nearest_even(a, E2M1_POS) if a < 6 else 7
        expect = mag | (8 if v < 0 else 0)
        assert oracle.e2m1_rne(float(v)) == expect, float(v)
