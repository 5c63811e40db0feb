"""Pins of the oracle's near-boundary flags, which decide the only
differences the GPU parity tests may tolerate (a value within 1e-6, relative,
of a rounding boundary, exact ties included).

Each flag is checked against a brute-force search written independently of
the oracle's code: exact rational arithmetic over EVERY boundary of the
rounding in question -- all code boundaries m8 + (k + 1/2) s8 of a group,
all midpoints between neighbouring E4M3 values, the midpoint between the two
BF16 values that bracket the number (found by search in the sorted list of
all BF16 values) -- on random inputs and on inputs placed exactly at, just
inside and just outside the window.  A flag that fired too often would excuse
real mismatches; one that fired too rarely would fail correct ties.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as orc

REL = Fraction(1, 10 ** 6)


def _fp8_table():
    return [Fraction(orc.fp8_value(c)) for c in range(0x7F)]          # 0 .. 448, ascending


def _bf16_positive_values() -> np.ndarray:
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint32)                  # positive finite BF16
    return (bits << 16).view(np.float32).astype(np.float64)


BF16_VALUES = _bf16_positive_values()


def brute_code_flags(x, bits):
    """Per element: within 1e-6 x max(|x|, |beta|, s8) of any code boundary
    beta = m8 + (k + 1/2) s8, k = 0 .. 2^bits - 2 (none when s8 = 0)."""
    _, s8c, m8c, _, _ = orc.quantize_group(np.asarray(x, np.float64), bits)
    s8, m8 = Fraction(orc.fp8_value(s8c)), Fraction(orc.fp8_value(m8c))
    out = []
    for v in x:
        v = Fraction(float(v))
        near = False
        if s8 != 0:
            for k in range((1 << bits) - 1):
                beta = m8 + (k + Fraction(1, 2)) * s8
                if abs(v - beta) <= REL * max(abs(v), abs(beta), s8):
                    near = True
        out.append(near)
    return np.array(out)


def brute_fp8_near(v: float) -> bool:
    a = abs(Fraction(v))
    t = _fp8_table()
    for lo, hi in zip(t[:-1], t[1:]):
        mid = (lo + hi) / 2
        if abs(a - mid) <= REL * max(a, mid):
            return True
    return False


def brute_bf16_near(v: float) -> bool:
    a = abs(v)
    if a == 0.0:
        return False
    i = int(np.searchsorted(BF16_VALUES, a, side="right"))
    if i == 0 or i >= len(BF16_VALUES):
        return False
    lo, hi = Fraction(float(BF16_VALUES[i - 1])), Fraction(float(BF16_VALUES[i]))
    if Fraction(a) == lo:                                              # on a value: nearest midpoints either side
        cands = [(lo + hi) / 2]
        if i >= 2:
            cands.append((Fraction(float(BF16_VALUES[i - 2])) + lo) / 2)
    else:
        cands = [(lo + hi) / 2]
    fa = Fraction(a)
    return any(abs(fa - m) <= REL * max(fa, m) for m in cands)


# ------------------------------------------------------------------ code flags
def _groups(bits, rng):
    qmax = (1 << bits) - 1
    out = [rng.standard_normal(16) * s for s in (0.01, 1.0, 30.0)]
    # elements placed at a code boundary, just inside and just outside the window
    base = rng.standard_normal(16)
    _, s8c, m8c, _, _ = orc.quantize_group(base, bits)
    s8, m8 = orc.fp8_value(s8c), orc.fp8_value(m8c)
    g = base.copy()
    for i, (k, f) in enumerate([(0, 0.0), (1, 3e-7), (2, -3e-7), (qmax - 1, 5e-6), (0, -5e-6), (1, 1.2e-6)]):
        beta = m8 + (min(k, qmax - 1) + 0.5) * s8
        ref = max(abs(beta), s8)
        g[2 + i] = beta + f * ref
    g[0], g[1] = base.min(), base.max()            # keep the range and hence s8, m8
    out.append(g)
    return out


@pytest.mark.parametrize("bits", [2, 4])
def test_code_flags_match_brute_force(bits):
    rng = np.random.default_rng(100 + bits)
    hits = 0
    for g in _groups(bits, rng):
        _, _, _, ef, _ = orc.quantize_group(g, bits)
        bf = brute_code_flags(g, bits)
        assert np.array_equal(ef.astype(bool), bf), (g, ef, bf)
        hits += int(bf.sum())
    assert hits >= 3          # the placed elements are flagged, the others not


# ------------------------------------------------------------------ FP8 flags
def test_fp8_flags_match_brute_force():
    rng = np.random.default_rng(7)
    t = [float(v) for v in _fp8_table()]
    mids = [(a + b) / 2 for a, b in zip(t[:-1], t[1:])]
    vals = list(rng.standard_normal(300) * 20) + list(rng.uniform(0, 0.02, 100))
    for m in mids[::5]:
        vals += [m, -m, m * (1 + 4e-7), m * (1 - 4e-7), m * (1 + 3e-6), m * (1 - 3e-6)]
    vals += [448.0, 500.0, 464.0, 2.0 ** -10, 2.0 ** -9 * 1.5, 0.0]
    flagged = 0
    for v in vals:
        _, near = orc.fp8_round(v)
        b = brute_fp8_near(v)
        assert near == b, (v, near, b)
        flagged += b
    assert flagged >= 2 * len(mids[::5])


# ------------------------------------------------------------------ BF16 flags
def test_bf16_flags_match_brute_force():
    rng = np.random.default_rng(8)
    vals = list(rng.standard_normal(300) * 3) + list(rng.standard_normal(50) * 1e-30)
    for lo in rng.choice(BF16_VALUES[5000:25000], 60):
        i = int(np.searchsorted(BF16_VALUES, lo))
        mid = (BF16_VALUES[i] + BF16_VALUES[i + 1]) / 2
        vals += [mid, -mid, mid * (1 + 4e-7), mid * (1 - 4e-7), mid * (1 + 3e-6), mid * (1 - 3e-6)]
    flagged = 0
    for v in vals:
        _, near = orc.bf16_round(v)
        b = brute_bf16_near(v)
        assert near == b, (v, near, b)
        flagged += b
    assert flagged >= 4 * 60
