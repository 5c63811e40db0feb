"""Pins of the oracle's ablation encoders (orc_encode_ablation): the reference
choices and scaling methods the ResidualQuant abstract compares (last-loop vs
previous-loop anchor; least-squares vs norm-ratio vs no scaling).

Each pin ties them to something other than their own formula: the method's
own encoder, a mirror identity, inputs on the quantization grid whose
residual is exactly zero, the least-squares minimum, and the read counts of
shared vs chained reconstruction.
"""
import numpy as np
import pytest

from oracle import oracle as orc

D = 128
SEED = 0xA11CE


def _bf16(x: np.ndarray) -> np.ndarray:
    """float -> BF16 bits, round to nearest even (inputs here are exact or
    random; exactness of the grid inputs is asserted separately)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _correlated(rng, L, n):
    """Loops sharing a common component (like the loops of one group), BF16."""
    base = rng.standard_normal((n, D))
    base[:, rng.choice(D, 4, replace=False)] *= 10.0
    xs = [base * (1.0 + 0.1 * j) + 0.2 * (L - j) * rng.standard_normal((n, D)) for j in range(L)]
    return _bf16(np.stack(xs))


@pytest.mark.parametrize("rotate,ba,br,g", [(True, 4, 2, 16), (False, 4, 2, 32), (True, 2, 2, 16)])
def test_method_mode_is_the_method_encoder(rotate, ba, br, g):
    x = _correlated(np.random.default_rng(1), 4, 37)
    xh, coef, reads = orc.encode_ablation(x, g, ba, br, rotate, SEED, orc.ANCHOR_LAST, orc.SCALE_LEAST_SQUARES)
    e = orc.encode(x, g, ba, br, rotate, SEED)
    ref = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, 4, D, g, ba, br, rotate, SEED)
    assert np.array_equal(xh, ref)
    assert np.array_equal(coef[:3], orc.bf16_bits_to_f64(e.r_coef)) and (coef[3] == 0).all()
    assert list(reads) == [2, 2, 2, 1]


@pytest.mark.parametrize("scale_mode", [orc.SCALE_LEAST_SQUARES, orc.SCALE_NORM_RATIO, orc.SCALE_NONE])
def test_two_loops_mirror(scale_mode):
    """With two loops, the previous-loop anchor of (x0, x1) is the last-loop
    anchor of (x1, x0)."""
    x = _correlated(np.random.default_rng(2), 2, 25)
    a, ca, ra = orc.encode_ablation(x, 16, 4, 2, True, SEED, orc.ANCHOR_PREVIOUS, scale_mode)
    b, cb, rb = orc.encode_ablation(x[::-1].copy(), 16, 4, 2, True, SEED, orc.ANCHOR_LAST, scale_mode)
    assert np.array_equal(a, b[::-1]) and np.array_equal(ca, cb[::-1])
    assert list(ra) == [1, 2] and list(rb) == [2, 1]


def _grid_anchor(rng, n):
    """Inputs on the INT4 grid of every group: min 0.5, scale 1/8, codes 0..15
    with both ends present, so the anchor quantizes exactly."""
    c = rng.integers(0, 16, size=(n, D))
    c[:, 0::16] = 0
    c[:, 1::16] = 15
    return 0.5 + c / 8.0


def test_scaled_copy_of_the_anchor():
    """x_l = -2 a exactly: least squares finds s = -2 and an exactly zero
    residual (exact reconstruction); norm ratio finds |s| = 2 with the wrong
    sign; no scaling uses s = 1."""
    rng = np.random.default_rng(3)
    a = _grid_anchor(rng, 9)
    x = np.stack([-2.0 * a, a])
    xb = _bf16(x)
    assert np.array_equal(orc.bf16_bits_to_f64(xb), x)   # the inputs are BF16-exact
    ls, c_ls, _ = orc.encode_ablation(xb, 16, 4, 2, True, SEED, orc.ANCHOR_LAST, orc.SCALE_LEAST_SQUARES)
    nr, c_nr, _ = orc.encode_ablation(xb, 16, 4, 2, True, SEED, orc.ANCHOR_LAST, orc.SCALE_NORM_RATIO)
    no, c_no, _ = orc.encode_ablation(xb, 16, 4, 2, True, SEED, orc.ANCHOR_LAST, orc.SCALE_NONE)
    assert np.array_equal(ls[1], a) and np.array_equal(ls[0], x[0])
    assert (c_ls[0] == -2.0).all() and (c_nr[0] == 2.0).all() and (c_no[0] == 1.0).all()
    assert orc.mse(nr[0], x[0]) > 0 and orc.mse(no[0], x[0]) > 0


def test_least_squares_minimises_the_residual():
    """Before the residual is quantized, the least-squares coefficient leaves
    less energy than the norm-ratio one or none (up to its BF16 rounding)."""
    x = _correlated(np.random.default_rng(4), 4, 64)
    xf = orc.bf16_bits_to_f64(x)
    out = {m: orc.encode_ablation(x, 16, 4, 2, True, SEED, orc.ANCHOR_LAST, m)
           for m in (orc.SCALE_LEAST_SQUARES, orc.SCALE_NORM_RATIO, orc.SCALE_NONE)}
    ahat = out[orc.SCALE_LEAST_SQUARES][0][3]
    for m, (xh, coef, _) in out.items():
        assert np.array_equal(xh[3], ahat)   # the anchor does not depend on the scaling
    for l in range(3):
        e = {m: ((xf[l] - out[m][1][l][:, None] * ahat) ** 2).sum(1) for m in out}
        ls = e[orc.SCALE_LEAST_SQUARES]
        for m in (orc.SCALE_NORM_RATIO, orc.SCALE_NONE):
            assert (ls <= e[m] * (1 + 1e-4) + 1e-12).all()


def test_chained_reference_is_the_reconstruction():
    """Previous-loop anchor, x2 = 2 x1: the chain references the lossy
    reconstruction of loop 1, not its input."""
    rng = np.random.default_rng(5)
    x0 = rng.standard_normal((6, D))
    x1 = _grid_anchor(rng, 6) * 0.25 + 0.1 * rng.standard_normal((6, D))
    xb = _bf16(np.stack([x0, x1, 2.0 * orc.bf16_bits_to_f64(_bf16(x1))]))
    xf = orc.bf16_bits_to_f64(xb)
    assert np.array_equal(xf[2], 2.0 * xf[1])
    xh, coef, reads = orc.encode_ablation(xb, 16, 4, 2, True, SEED, orc.ANCHOR_PREVIOUS, orc.SCALE_LEAST_SQUARES)
    assert list(reads) == [1, 2, 3]
    e1, e2 = orc.mse(xh[1], xf[1]), orc.mse(xh[2], xf[2])
    # loop 2 is x1_hat scaled plus a quantized residual against it: its error
    # is a fraction of loop 1's.  Encoding against the input x1 (s = 2, a zero
    # residual) but rebuilding from x1_hat would leave exactly 4 e1; encoding
    # and rebuilding from the input would leave 0.
    assert 0 < e2 < 2 * e1, (e1, e2)


def test_shared_reads_stay_two():
    x = _correlated(np.random.default_rng(6), 8, 3)
    _, _, r_last = orc.encode_ablation(x, 16, 4, 2, True, SEED, orc.ANCHOR_LAST, orc.SCALE_LEAST_SQUARES)
    _, _, r_prev = orc.encode_ablation(x, 16, 4, 2, True, SEED, orc.ANCHOR_PREVIOUS, orc.SCALE_LEAST_SQUARES)
    assert list(r_last) == [2] * 7 + [1]
    assert list(r_prev) == list(range(1, 9))


def test_study_on_synthetic_loops():
    """Relative reconstruction MSE of every (reference, scaling) pair on the
    seeded synthetic loop group (4 loops, H = 4, T = 256; loops at distance k
    from the last one carry noise 0.1 k on top of a scaled copy of it).
    Printed with -s; asserted: scaling beats none for both references."""
    import synth
    rows = {}
    for kv in (0, 1):
        K, V = synth.group_kv(0x5EED0001, 0, 0, 4, (0.1, 0.2, 0.3), 1, 256, 4, device="cpu")
        X = K if kv == 0 else V
        x = np.stack([synth.bf16_to_u16(X[j]).transpose(0, 2, 1, 3).reshape(-1, D) for j in range(4)])
        xf = orc.bf16_bits_to_f64(x)
        for am in (orc.ANCHOR_LAST, orc.ANCHOR_PREVIOUS):
            for sm in (orc.SCALE_LEAST_SQUARES, orc.SCALE_NORM_RATIO, orc.SCALE_NONE):
                xh, _, reads = orc.encode_ablation(x, 16, 4, 2, True, SEED, am, sm)
                rel = np.mean([orc.mse(xh[l], xf[l]) / np.mean(xf[l] ** 2) for l in range(4)])
                rows.setdefault((am, sm), []).append(rel)
                rows[(am, sm, "reads")] = [int(r) for r in reads]
    for am in (orc.ANCHOR_LAST, orc.ANCHOR_PREVIOUS):
        for sm in (orc.SCALE_LEAST_SQUARES, orc.SCALE_NORM_RATIO, orc.SCALE_NONE):
            k, v = rows[(am, sm)]
            print("anchor %-8s scaling %-13s K %.5f V %.5f reads %s" % (
                ("last", "previous")[am], ("least-squares", "norm-ratio", "none")[sm], k, v, rows[(am, sm, "reads")]))
        for kv in (0, 1):
            assert rows[(am, orc.SCALE_LEAST_SQUARES)][kv] < rows[(am, orc.SCALE_NONE)][kv]


@pytest.mark.parametrize("anchor_mode", [orc.ANCHOR_LAST, orc.ANCHOR_PREVIOUS])
@pytest.mark.parametrize("scale_mode", [orc.SCALE_LEAST_SQUARES, orc.SCALE_NORM_RATIO, orc.SCALE_NONE])
@pytest.mark.parametrize("rotate", [True, False])
def test_mode_records_rebuild_the_ablation(anchor_mode, scale_mode, rotate):
    """The records the oracle lays out for each mode (orc_encode_modes: the
    anchor record holds the last loop or, chained, the first; residual
    record j holds loop j or loop j + 1), rebuilt by orc_reconstruct_modes,
    give the ablation encoder's reconstruction bit for bit, and the stored
    coefficients are its coefficients; the method's mode gives the method's
    records."""
    L = 4
    x = _correlated(np.random.default_rng(40 + anchor_mode * 3 + scale_mode), L, 29)
    e = orc.encode_modes(x, 16, 4, 2, rotate, SEED, anchor_mode, scale_mode)
    xr = orc.reconstruct_modes(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, L, D, 16, 4, 2, rotate, SEED,
                               anchor_mode)
    xh, coef, _ = orc.encode_ablation(x, 16, 4, 2, rotate, SEED, anchor_mode, scale_mode)
    assert np.array_equal(xr, xh)
    loops = range(L - 1) if anchor_mode == orc.ANCHOR_LAST else range(1, L)
    for j, loop in enumerate(loops):
        assert np.array_equal(orc.bf16_bits_to_f64(e.r_coef[j]), coef[loop])
    if anchor_mode == orc.ANCHOR_LAST and scale_mode == orc.SCALE_LEAST_SQUARES:
        m = orc.encode(x, 16, 4, 2, rotate, SEED)
        for f in ("a_codes", "a_meta", "r_codes", "r_meta", "r_coef", "a_eflag", "r_eflag", "r_mflag", "r_cflag"):
            assert np.array_equal(getattr(e, f), getattr(m, f)), f
