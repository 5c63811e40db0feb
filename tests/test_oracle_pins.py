"""Pins for the fp64 CPU oracle: each check compares the oracle with
something other than itself -- a format specification, a library routine,
exact rational arithmetic, a closed form, a brute-force search, or an
invariant of the mathematics -- so that a dropped term, a wrong sign, a
wrong index or a transposed operand in the oracle fails here.

Method facts followed ("ResidualQuant: KV Cache Quantization for Looped
Transformers with 2-Bit Residuals", arXiv 2610.10381, and its ai4snews and
agihunt summaries): final-loop anchor at INT4, INT2 residuals for the other
loops, least-squares scaling with a BF16 coefficient, rotation of the
residuals only, group size 16 with FP8 scale and offset, reconstruction
from two reads (anchor + one residual), 80.7% storage reduction.
"""
import decimal
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ FP8 E4M3
def test_fp8_spec_points():
    """Spot values of the OCP E4M3 definition."""
    g = _golden("fp8_e4m3_points.json")
    for hexcode, val in g["points"]:
        assert orc.fp8_value(int(hexcode, 16)) == val, hexcode
    for hexcode in g["nan_codes"]:
        assert math.isnan(orc.fp8_value(int(hexcode, 16)))


def test_fp8_decode_matches_torch_all_codes():
    """All 256 codes decode exactly like torch.float8_e4m3fn."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = orc.fp8_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(v)
        else:
            assert v == ref[c], c
            assert math.copysign(1.0, v) == math.copysign(1.0, ref[c]), c


def test_fp8_round_trip_all_finite_codes():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        code, _ = orc.fp8_round(orc.fp8_value(c))
        assert code == c, hex(c)


def test_fp8_round_ties_and_saturation():
    # ties go to the even mantissa
    assert orc.fp8_round(1.0625)[0] == 0x38          # 1.0 vs 1.125 -> 1.0
    assert orc.fp8_round(1.1875)[0] == 0x3A          # 1.125 vs 1.25 -> 1.25
    assert orc.fp8_round(2.0 ** -10)[0] == 0x00      # 0 vs 2^-9 -> 0
    assert orc.fp8_round(3 * 2.0 ** -10)[0] == 0x02  # 2^-9 vs 2^-8 -> 2^-8
    assert orc.fp8_round(-1.0625)[0] == 0xB8
    # satfinite: everything at or beyond 448 clamps to +-448
    for v in (448.0, 449.0, 463.9, 464.0, 1e6, 1e300):
        assert orc.fp8_round(v)[0] == 0x7E
        assert orc.fp8_round(-v)[0] == 0xFE
    # exact midpoints are flagged as near a boundary
    assert orc.fp8_round(1.0625)[1] and not orc.fp8_round(1.03)[1]


def test_fp8_round_matches_torch_cast():
    """RNE against torch's float32 -> float8_e4m3fn cast (|v| < 448)."""
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(4000) * 3.0,
        rng.uniform(-440, 440, 2000),
        rng.uniform(-0.02, 0.02, 2000),          # subnormal range
        (np.arange(-447, 447, 0.5)),
    ]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(xs, ref):
        assert orc.fp8_round(float(x))[0] == r, float(x)


# ------------------------------------------------------------------ BF16
def _bf16_exact_rational(v: float) -> int:
    """Nearest BF16 by exact rational arithmetic, ties to even (independent
    of the oracle's floating-point steps)."""
    if v == 0:
        return 0x8000 if math.copysign(1, v) < 0 else 0
    a = Fraction(abs(v))
    m, e = math.frexp(abs(v))          # |v| = m 2^e, m in [0.5, 1)
    q = Fraction(2) ** (e - 8) if e - 1 >= -126 else Fraction(2) ** -133
    u = a / q
    fl = u.numerator // u.denominator
    rem = u - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    res = float(fl * q)
    bits = int(np.array([res], np.float32).view(np.uint32)[0]) >> 16
    return bits | (0x8000 if v < 0 else 0)


def test_bf16_round_matches_torch_for_float32_inputs():
    rng = np.random.default_rng(11)
    xs = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # float32 subnormals
    ])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    for x, r in zip(xs, ref):
        assert orc.bf16_round(float(x))[0] == r, float(x)


def test_bf16_round_double_inputs_single_rounding():
    rng = np.random.default_rng(12)
    xs = list(rng.standard_normal(3000) * 10.0)
    # values just off a BF16 midpoint, where a detour through binary32 would double-round
    for k in range(200):
        base = 1.0 + (2 * k + 1) / 256.0   # midpoints between BF16 neighbours in [1, 2)
        xs += [base + 2.0 ** -40, base - 2.0 ** -40, base]
    for x in xs:
        assert orc.bf16_round(float(x))[0] == _bf16_exact_rational(float(x)), x


def test_bf16_value_matches_torch():
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for b, r in zip(bits, ref):
        v = orc.bf16_value(int(b))
        assert (math.isnan(v) and math.isnan(r)) or v == r


# ------------------------------------------------------------------ rotation
def test_splitmix64_published_vectors():
    g = _golden("splitmix64_vectors.json")
    assert orc.splitmix64(0) == int(g["state0_first_output_hex"], 16)
    gamma = 0x9E3779B97F4A7C15
    s = 1234567
    outs = [orc.splitmix64((s + i * gamma) % 2 ** 64) for i in range(3)]
    assert outs == g["seed_1234567_first_three"]


def _fwht(x: np.ndarray) -> np.ndarray:
    """Independent recursive butterfly: returns H_n x (Sylvester order)."""
    n = x.shape[0]
    if n == 1:
        return x.copy()
    a = _fwht(x[: n // 2])
    b = _fwht(x[n // 2:])
    return np.concatenate([a + b, a - b])


@pytest.mark.parametrize("seed", [0xA11CE, 1, 12345])
def test_rotation_is_orthogonal_and_hadamard(seed):
    d = 128
    R = orc.rotation_matrix(seed, d)
    np.testing.assert_allclose(R @ R.T, np.eye(d), atol=1e-14)
    sigma = orc.rotation_signs(seed, d)
    assert set(np.unique(sigma)) <= {-1.0, 1.0}
    assert 30 < (sigma > 0).sum() < 98   # a seeded mix of signs, not all one sign
    H = np.rint(R * math.sqrt(d) * sigma[None, :])
    np.testing.assert_array_equal(H @ H, d * np.eye(d))
    np.testing.assert_array_equal(H, H.T)
    # R e_j = sigma_j * (column j of H) / sqrt(d)
    for j in (0, 1, 5, 77, 127):
        e = np.zeros(d)
        e[j] = 1
        np.testing.assert_allclose(R @ e, sigma[j] * H[:, j] / math.sqrt(d), atol=1e-16)
    # the O(d^2) product agrees with an independent butterfly on random vectors
    rng = np.random.default_rng(seed)
    for _ in range(5):
        r = rng.standard_normal(d)
        np.testing.assert_allclose(R @ r, _fwht(sigma * r) / math.sqrt(d), atol=1e-13)
    # H_ij = (-1)^popcount(i & j): first row all +1, row 1 alternates
    assert (H[0] == 1).all()
    assert (H[1] == np.array([1, -1] * (d // 2))).all()


def test_rotation_off_is_identity():
    np.testing.assert_array_equal(orc.rotation_matrix(5, 128, rotate=False), np.eye(128))


def test_signs_match_splitmix_top_bit():
    s = orc.rotation_signs(0xA11CE, 128)
    for j in range(128):
        top = orc.splitmix64((0xA11CE + j) % 2 ** 64) >> 63
        assert s[j] == (-1.0 if top else 1.0)


# ------------------------------------------------------------------ quantizer
def _fp8_table():
    return [(c, orc.fp8_value(c)) for c in range(256) if c not in (0x7F, 0xFF)]


@pytest.mark.parametrize("bits", [2, 4])
def test_quantizer_grid_round_trip(bits):
    """Grid-valued groups come back exactly: codes, scale and min."""
    rng = np.random.default_rng(bits)
    qmax = (1 << bits) - 1
    for trial in range(300):
        s8 = 2.0 ** int(rng.integers(-6, 2))
        m8 = float(rng.choice([-2.0, -1.5, -1.0, -0.75, -0.5, 0.0, 0.25, 1.0])) * (1 if trial % 2 else s8 * 4)
        m8c, _ = orc.fp8_round(m8)
        m8 = orc.fp8_value(m8c)
        c = rng.integers(0, qmax + 1, 16)
        c[rng.integers(0, 16)] = 0
        c[rng.integers(0, 16)] = qmax
        c[0], c[1] = 0, qmax
        x = m8 + c * s8
        # the grid values are exact in BF16 (few significant bits)
        assert all(orc.bf16_value(orc.bf16_round(v)[0]) == v for v in x)
        codes, sc, mc, ef, mf = orc.quantize_group(x, bits)
        assert orc.fp8_value(sc) == s8 and orc.fp8_value(mc) == m8
        np.testing.assert_array_equal(codes, c)
        np.testing.assert_array_equal(m8 + codes * s8, x)


@pytest.mark.parametrize("bits", [2, 4])
def test_quantizer_brute_force(bits):
    """Scale and min are the nearest FP8 values (table search); each code is
    the integer in [0, 2^b-1] nearest (x - m8)/s8 (exhaustive search)."""
    rng = np.random.default_rng(100 + bits)
    qmax = (1 << bits) - 1
    table = _fp8_table()
    for trial in range(400):
        x = rng.standard_normal(16) * float(rng.choice([0.01, 0.3, 1.0, 10.0]))
        codes, sc, mc, ef, mf = orc.quantize_group(x, bits)
        sig = (x.max() - x.min()) / qmax
        for target, code, bit in ((sig, sc, 1), (x.min(), mc, 2)):
            if mf & bit:
                continue
            best = min(table, key=lambda cv: (abs(cv[1] - target), cv[0] & 1))
            assert orc.fp8_value(code) == best[1], (target, code)
        s8, m8 = orc.fp8_value(sc), orc.fp8_value(mc)
        for i in range(16):
            if ef[i]:
                continue
            errs = [abs(x[i] - (m8 + c * s8)) for c in range(qmax + 1)]
            assert codes[i] == int(np.argmin(errs)), (i, x[i], m8, s8)


def test_quantizer_zero_range_group():
    x = np.full(16, 0.3)
    codes, sc, mc, ef, mf = orc.quantize_group(x, 4)
    assert sc == 0 and (codes == 0).all()
    assert orc.fp8_value(mc) == orc.fp8_value(orc.fp8_round(0.3)[0])
    # a -0 minimum is stored as +0
    codes, sc, mc, ef, mf = orc.quantize_group(np.array([-0.0] * 16), 2)
    assert mc == 0x00 and sc == 0x00


def test_pack_layout():
    # 2-bit: element i at byte i/4, bit 2*(i%4), LSB first
    c = np.zeros(128, np.uint8)
    c[:4] = [1, 2, 3, 0]
    c[127] = 3
    p = orc.pack(c, 2)
    assert p.size == 32 and p[0] == 0x39 and p[31] == 0xC0
    # 4-bit: element i at byte i/2, low nibble first
    c = np.zeros(128, np.uint8)
    c[0], c[1], c[126], c[127] = 0xA, 0x5, 0x1, 0xF
    p = orc.pack(c, 4)
    assert p.size == 64 and p[0] == 0x5A and p[63] == 0xF1
    # the little-endian 32-bit word view puts element i at bits 4*(i%8) of word i/8
    w = p.view(np.uint32)
    assert w[0] & 0xF == 0xA and (w[0] >> 4) & 0xF == 0x5
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        c = rng.integers(0, 1 << bits, 128).astype(np.uint8)
        np.testing.assert_array_equal(orc.unpack(orc.pack(c, bits), 128, bits), c)


def test_dequant_exact_in_fp32():
    """m8 + c*s8 is exactly representable in binary32 for every FP8 pair and
    4-bit code (FP8 values are multiples of 2^-9 below 2^9)."""
    vals = [v for _, v in _fp8_table()]
    rng = np.random.default_rng(5)
    for _ in range(20000):
        s = abs(vals[rng.integers(len(vals))])
        m = vals[rng.integers(len(vals))]
        c = int(rng.integers(0, 16))
        x = m + c * s
        assert float(np.float32(x)) == x


# ------------------------------------------------------------------ encoding
def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_least_squares_coefficient_is_the_minimiser():
    """s_hat = bf16(argmin_s ||x - s a_hat||^2): no BF16 neighbour of s_hat
    does better, and a brute-force scan finds the minimum within half a BF16
    step of s_hat."""
    rng = np.random.default_rng(21)
    n, d = 40, 128
    anchor = rng.standard_normal((n, d))
    loop = rng.uniform(0.8, 1.2, (n, 1)) * anchor + 0.3 * rng.standard_normal((n, d))
    x = np.stack([_bf16(loop), _bf16(anchor)])
    e = orc.encode(x, 16, 4, 2, True, 0xA11CE)
    recon = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, 2, d, 16, 4, 2, True, 0xA11CE)
    ahat = recon[1]
    xl = orc.bf16_bits_to_f64(x[0])
    for t in range(n):
        if e.r_cflag[0, t]:
            continue
        sh = orc.bf16_value(int(e.r_coef[0, t]))
        f = lambda s: float(((xl[t] - s * ahat[t]) ** 2).sum())
        up = orc.bf16_value(int(e.r_coef[0, t]) + 1)
        dn = orc.bf16_value(int(e.r_coef[0, t]) - 1)
        assert f(sh) <= f(up) and f(sh) <= f(dn)
        grid = sh + np.linspace(-0.05, 0.05, 10001)
        vals = ((xl[t][None, :] - grid[:, None] * ahat[t][None, :]) ** 2).sum(1)
        smin = grid[int(np.argmin(vals))]
        assert abs(smin - sh) <= (up - sh) / 2 + 1e-5
        # residual with the unrounded minimiser is orthogonal to a_hat
        s_star = float(xl[t] @ ahat[t]) / float(ahat[t] @ ahat[t])
        assert abs(float((xl[t] - s_star * ahat[t]) @ ahat[t])) < 1e-12 * float(ahat[t] @ ahat[t])
        assert orc.bf16_round(s_star)[0] == e.r_coef[0, t]


def test_identical_loops_zero_residual_exact_anchor():
    """Grid-valued anchor and identical loops: coefficient 1, zero residual
    codes, zero scale/min, and every loop reconstructs the input exactly."""
    rng = np.random.default_rng(31)
    n, d, L = 12, 128, 4
    s8 = 2.0 ** -3
    c = rng.integers(0, 16, (n, d))
    c[:, ::16] = 0
    c[:, 1::16] = 15
    xa = -1.0 + c * s8
    bits = _bf16(xa)
    assert (orc.bf16_bits_to_f64(bits) == xa).all()
    x = np.stack([bits] * L)
    e = orc.encode(x, 16, 4, 2, True, 0xA11CE)
    assert (e.r_coef == 0x3F80).all()          # BF16 1.0
    assert (e.r_codes == 0).all() and (e.r_meta == 0).all()
    rec = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, L, d, 16, 4, 2, True, 0xA11CE)
    for l in range(L):
        np.testing.assert_array_equal(rec[l], xa)


def test_residual_rotation_only_and_two_reads():
    """The anchor record does not depend on the rotation seed (the rotation
    touches residuals only); loop l's reconstruction reads the anchor and its
    own residual only, so corrupting another loop's residual changes nothing."""
    rng = np.random.default_rng(41)
    n, d, L = 16, 128, 4
    anchor = rng.standard_normal((n, d))
    loops = [rng.uniform(0.8, 1.2, (n, 1)) * anchor + s * rng.standard_normal((n, d)) for s in (0.3, 0.2, 0.1)]
    x = np.stack([_bf16(a) for a in loops + [anchor]])
    e1 = orc.encode(x, 16, 4, 2, True, 1)
    e2 = orc.encode(x, 16, 4, 2, True, 2)
    np.testing.assert_array_equal(e1.a_codes, e2.a_codes)
    np.testing.assert_array_equal(e1.a_meta, e2.a_meta)
    np.testing.assert_array_equal(e1.r_coef, e2.r_coef)
    assert not np.array_equal(e1.r_codes, e2.r_codes)
    args = (L, d, 16, 4, 2, True, 1)
    base = orc.reconstruct(e1.a_codes, e1.a_meta, e1.r_codes, e1.r_meta, e1.r_coef, *args)
    rc = e1.r_codes.copy()
    rc[0] ^= 0xFF
    alt = orc.reconstruct(e1.a_codes, e1.a_meta, rc, e1.r_meta, e1.r_coef, *args)
    np.testing.assert_array_equal(alt[1:], base[1:])
    assert not np.array_equal(alt[0], base[0])


def test_reconstruction_formula_by_hand():
    """x_hat_l = s_hat * a_hat + R^T y_hat, rebuilt here from the records with
    numpy (unpack by bit arithmetic, FP8 via torch)."""
    rng = np.random.default_rng(51)
    n, d, L = 6, 128, 3
    anchor = rng.standard_normal((n, d))
    loops = [0.9 * anchor + 0.2 * rng.standard_normal((n, d)) for _ in range(L - 1)]
    x = np.stack([_bf16(a) for a in loops + [anchor]])
    seed = 99
    e = orc.encode(x, 16, 4, 2, True, seed)
    rec = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, L, d, 16, 4, 2, True, seed)

    def fp8(b):
        return torch.from_numpy(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()

    def deq(packed, meta, bits):
        per = 8 // bits
        codes = np.stack([(packed >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], -1).reshape(-1)
        s = np.repeat(fp8(meta[0::2]), 16)
        m = np.repeat(fp8(meta[1::2]), 16)
        return m + codes * s

    sigma = orc.rotation_signs(seed, d)
    for t in range(n):
        ahat = deq(e.a_codes[t], e.a_meta[t], 4)
        np.testing.assert_array_equal(rec[L - 1, t], ahat)
        for l in range(L - 1):
            yhat = deq(e.r_codes[l, t], e.r_meta[l, t], 2)
            sh = orc.bf16_value(int(e.r_coef[l, t]))
            # R^T y = diag(sigma) H y / sqrt(d)
            back = sigma * _fwht(yhat) / math.sqrt(d)
            np.testing.assert_allclose(rec[l, t], sh * ahat + back, rtol=0, atol=1e-12)


def test_storage_fraction_reproduces_the_papers_figure():
    """Record sizes (codes + FP8 scale/min + BF16 coefficient) reproduce the
    80.7% storage reduction for 4 loops, INT4 anchor, INT2 residuals."""
    g = _golden("storage_fraction.json")
    d = g["head_dim"]
    for group, expect in ((32, 0.193359375), (16, 0.224609375)):
        e = orc.encode(np.zeros((4, 1, d), np.uint16), group, 4, 2, True, 0)
        a_bytes = e.a_codes.shape[1] + e.a_meta.shape[1]
        r_bytes = e.r_codes.shape[2] + e.r_meta.shape[2] + 2
        frac = (a_bytes + 3 * r_bytes) / (4 * 2 * d)
        assert frac == expect
    frac32 = 0.193359375
    assert round(100 * (1 - frac32), g["printed_decimals"]) == g["reduction_percent"]


# ------------------------------------------------------------------ attention
def test_attention_two_tokens_closed_form():
    rng = np.random.default_rng(61)
    d = 128
    q = rng.standard_normal((1, 1, d))
    k = rng.standard_normal((1, 2, 1, d))
    v = rng.standard_normal((1, 2, 1, d))
    scale = 1 / math.sqrt(d)
    out = orc.attention(q, k, v, scale)
    z0 = scale * float(q[0, 0] @ k[0, 0, 0])
    z1 = scale * float(q[0, 0] @ k[0, 1, 0])
    w1 = 1.0 / (1.0 + math.exp(z0 - z1))
    np.testing.assert_allclose(out[0, 0], w1 * v[0, 1, 0] + (1 - w1) * v[0, 0, 0], atol=1e-14)


def test_attention_equal_logits_dominant_and_permutation():
    rng = np.random.default_rng(62)
    d, T = 128, 9
    v = rng.standard_normal((1, T, 1, d))
    k = np.zeros((1, T, 1, d))
    q = rng.standard_normal((1, 1, d))
    np.testing.assert_allclose(orc.attention(q, k, v, 0.1)[0, 0], v[0, :, 0].mean(0), atol=1e-14)
    k2 = np.zeros((1, T, 1, d))
    k2[0, 4, 0, 0] = 50.0
    q2 = np.zeros((1, 1, d))
    q2[0, 0, 0] = 1.0
    np.testing.assert_allclose(orc.attention(q2, k2, v, 1.0)[0, 0], v[0, 4, 0], atol=1e-15)
    k3 = rng.standard_normal((1, T, 1, d))
    perm = rng.permutation(T)
    a = orc.attention(q, k3, v, 0.2)
    b = orc.attention(q, k3[:, perm], v[:, perm], 0.2)
    np.testing.assert_allclose(a, b, atol=1e-14)


def test_attention_gqa_head_mapping():
    """Query head h reads kv head h // (Hq/Hkv)."""
    rng = np.random.default_rng(63)
    B, T, Hkv, Hq, d = 2, 5, 2, 4, 128
    k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    q = rng.standard_normal((B, Hq, d))
    out = orc.attention(q, k, v, 0.3)
    for h in range(Hq):
        single = orc.attention(q[:, h:h + 1], k[:, :, h // 2:h // 2 + 1], v[:, :, h // 2:h // 2 + 1], 0.3)
        np.testing.assert_array_equal(out[:, h], single[:, 0])


def test_attention_brute_force_decimal():
    """T <= 8: softmax in 40-digit decimal arithmetic."""
    rng = np.random.default_rng(64)
    decimal.getcontext().prec = 40
    for T in range(1, 9):
        d = 128
        q = rng.standard_normal((1, 1, d))
        k = rng.standard_normal((1, T, 1, d)) * 2
        v = rng.standard_normal((1, T, 1, d))
        scale = 1 / math.sqrt(d)
        out = orc.attention(q, k, v, scale)[0, 0]
        D = decimal.Decimal
        z = [sum(D(float(a)) * D(float(b)) for a, b in zip(q[0, 0], k[0, t, 0])) * D(scale) for t in range(T)]
        w = [zz.exp() for zz in z]
        den = sum(w)
        ref = [float(sum(w[t] * D(float(v[0, t, 0, i])) for t in range(T)) / den) for i in range(d)]
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-14)


def test_attention_empty_is_zero():
    out = orc.attention(np.ones((1, 2, 128)), np.zeros((1, 0, 1, 128)), np.zeros((1, 0, 1, 128)), 1.0)
    assert (out == 0).all()


def test_encoded_records_quantize_the_rotated_residual():
    """Record-level check with an independent path: y = R (x_l - s_hat a_hat)
    computed here by a butterfly, then every residual group's scale/min must
    be the FP8 values nearest (max-min)/3 and min (table search), and every
    code the nearest grid point (exhaustive search).  The anchor record is
    checked the same way against x_L itself."""
    rng = np.random.default_rng(71)
    n, d, L, seed = 24, 128, 4, 0xA11CE
    anchor = rng.standard_normal((n, d))
    anchor[:, [3, 40, 77, 100]] *= 10.0
    loops = [rng.uniform(0.8, 1.2, (n, 1)) * anchor + s * rng.standard_normal((n, d)) for s in (0.3, 0.2, 0.02)]
    x = np.stack([_bf16(a) for a in loops + [anchor]])
    e = orc.encode(x, 16, 4, 2, True, seed)
    rec = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, L, d, 16, 4, 2, True, seed)
    table = _fp8_table()
    sigma = orc.rotation_signs(seed, d)

    def nearest_fp8(v):
        return min(table, key=lambda cv: (abs(cv[1] - v), cv[0] & 1))[1]

    def check(vec, packed, meta, bits, eflag, mflag):
        qmax = (1 << bits) - 1
        codes = orc.unpack(packed, d, bits)
        for grp in range(d // 16):
            seg = vec[grp * 16:(grp + 1) * 16]
            s8, m8 = orc.fp8_value(int(meta[2 * grp])), orc.fp8_value(int(meta[2 * grp + 1]))
            if not mflag[grp] & 1:
                assert s8 == nearest_fp8((seg.max() - seg.min()) / qmax)
            if not mflag[grp] & 2:
                assert m8 == nearest_fp8(seg.min())
            if mflag[grp]:
                continue
            for i in range(16):
                if eflag[grp * 16 + i] or s8 == 0:
                    continue
                errs = [abs(seg[i] - (m8 + c * s8)) for c in range(qmax + 1)]
                assert codes[grp * 16 + i] == int(np.argmin(errs))

    xf = orc.bf16_bits_to_f64(x)
    for t in range(n):
        check(xf[L - 1, t], e.a_codes[t], e.a_meta[t], 4, e.a_eflag[t], e.a_mflag[t])
        ahat = rec[L - 1, t]
        for l in range(L - 1):
            sh = orc.bf16_value(int(e.r_coef[l, t]))
            y = _fwht(sigma * (xf[l, t] - sh * ahat)) / math.sqrt(d)
            check(y, e.r_codes[l, t], e.r_meta[l, t], 2, e.r_eflag[l, t], e.r_mflag[l, t])


def test_rotation_scale_is_correctly_rounded():
    """1/sqrt(d) for d = 2^k is the double nearest the exact value (decimal
    arithmetic at 60 digits), so the oracle's rotation carries one rounding,
    as the definition R = H diag(sigma)/sqrt(d) does when applied in exact
    arithmetic and rounded once."""
    import decimal
    decimal.getcontext().prec = 60
    for k in range(0, 12):
        d = 2 ** k
        exact = decimal.Decimal(1) / decimal.Decimal(d).sqrt()
        assert orc.rotation_scale(d) == float(exact), k
    assert orc.rotation_scale(128, False) == 1.0
