"""GPU parity on the method's degenerate and boundary inputs.

Each case builds a one-layer cache of one loop group (4 loops: loop 4 the
INT4 anchor, loops 1-3 INT2 residuals) from constructed K/V through the C
ABI, then checks, against the fp64 oracle:
  * every packed code, FP8 scale/min and BF16 coefficient bit for bit; where
    the GPU and the oracle round the very same fp64 value (anchor records,
    coefficients, residuals without rotation) not even a flagged boundary
    value may differ, so these cases also require zero tolerated differences;
  * attention (every loop) within relative L2 1e-3 / max abs 2e-3 against
    the oracle fed the GPU's own records.

Cases (ai4snews summary, paragraphs 1-2: FP8 scales and offsets per group of
16, BF16 least-squares coefficients; the readings for zero ranges, zero
coefficients and the sign of a zero minimum are the library's):
  * an all-zero anchor (<a_hat, a_hat> = 0, so s_hat = 0 and the residual is
    the loop itself) on every third token;
  * constant groups (zero range: scale 0, all codes 0, x_hat = the minimum),
    in the anchor and, without rotation, in the residual;
  * magnitudes beyond the largest FP8 value (448): scales and minima saturate;
  * group ranges and minima exactly at FP8 rounding midpoints (ties to even)
    and one BF16 step either side of them;
  * least-squares coefficients exactly at BF16 midpoints, inside the 1e-6
    window, and just outside it;
  * -0 minima (stored as +0), in the anchor and in the residual;
  * identical loops (on an FP8 grid: s_hat = 1, zero residual, exact
    reconstruction; and on general data);
  * V divided by 64 (FP8-subnormal scales) through decode;
  * peaked softmax (q x 8 aligned with one key), uniform softmax (q = 0) and
    a very large query through decode.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as orc

import rqharness as H

pytestmark = pytest.mark.gpu

D = 128
LG = 4
B, HKV, HQ = 2, 2, 4
T, NTAIL = 150, 1


# ------------------------------------------------------------------ helpers
def bf16_exact(x: np.ndarray) -> np.ndarray:
    """x must hold BF16 values exactly; returns it as float64."""
    x = np.asarray(x, np.float64)
    r = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(r, x) and np.array_equal(np.signbit(r), np.signbit(x)), "not BF16-exact"
    return x


def to_dev(x: np.ndarray) -> torch.Tensor:
    """float64 [B][T][H][d] -> BF16 CUDA tensor (round to nearest)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda()


def lists(K: np.ndarray, V: np.ndarray):
    """[Lg][B][T][H][d] arrays -> the harness's lists of device tensors."""
    return [to_dev(K[j]) for j in range(LG)], [to_dev(V[j]) for j in range(LG)]


_FP8 = None


def fp8_values() -> np.ndarray:
    """The non-negative finite E4M3 values, ascending (from the oracle's table)."""
    global _FP8
    if _FP8 is None:
        _FP8 = np.array([orc.fp8_value(c) for c in range(0x7F)])
    return _FP8


def grid_group(rng, bits: int, lo_exp=-5, hi_exp=1) -> np.ndarray:
    """16 values m + c s with s a power of two, m an FP8 value, codes c
    covering 0 and 2^bits - 1: the quantizer returns exactly (c, s, m) and
    the dequantized group equals the input."""
    qmax = (1 << bits) - 1
    while True:
        s = 2.0 ** rng.integers(lo_exp, hi_exp + 1)
        m = float(rng.choice(fp8_values()[40:100])) * rng.choice([-1.0, 1.0])
        c = rng.integers(0, qmax + 1, 16)
        c[rng.integers(0, 16)] = 0
        c[rng.integers(0, 16)] = qmax
        if c.min() != 0 or c.max() != qmax:
            continue
        x = m + c * s
        if np.array_equal(torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy(), x) and \
                abs(m) <= 448 and s <= 448:
            return x


def grid_record(rng, bits: int) -> np.ndarray:
    return np.concatenate([grid_group(rng, bits) for _ in range(D // 16)])


def check_records(bt, strict: bool):
    for kv in (0, 1):
        r = H.compare_records(bt, 0, 0, kv)
        assert r["mismatch"] == 0, (kv, r)
        assert r["compared"] > 0
        if strict:
            assert r["tolerated"] == 0, (kv, r)


def check_decode(bt, q_of=None):
    cfg = bt.cfg
    for loop in range(LG):
        q = synth.queries(bt.seed, 0, loop, 0, cfg.batch, cfg.num_q_heads) if q_of is None else q_of(loop)
        out = bt.cache.decode(0, loop, q, out=H.guarded_out((cfg.batch, cfg.num_q_heads, D))).cpu().numpy()
        assert np.isfinite(out).all()
        ref = H.oracle_decode(bt, 0, loop, q)
        rel, mx = H.attn_errors(out, ref, cfg.num_q_heads // cfg.num_kv_heads)
        assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
    bt.cache.check()


def synthetic(seed, v_scale=1.0):
    """The synthetic recipe (outlier channels, c * anchor + sigma * noise) as float64."""
    K, V = synth.group_kv(seed, 0, 0, LG, (0.1, 0.2, 0.3), B, T + NTAIL, HKV, device="cpu")
    K = np.stack([k.double().numpy() for k in K])
    V = np.stack([v.double().numpy() for v in V]) * v_scale
    return K, V


def build(K, V, **kw):
    Kd, Vd = lists(K, V)
    return H.build_from(Kd, Vd, Hq=HQ, T=T, n_tail=NTAIL, chunk=64, seed=kw.pop("seed", 7), **kw)


# ------------------------------------------------------------------ cases
def test_zero_anchor_tokens():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((LG, B, T + NTAIL, HKV, D))
    V = rng.standard_normal((LG, B, T + NTAIL, HKV, D))
    K[LG - 1, :, ::3] = 0.0
    V[LG - 1, :, ::3] = 0.0
    bt = build(K, V)
    check_records(bt, strict=True)
    _, _, coef = bt.cache.export(0, 0)
    assert (coef[:, :, :, ::3] == 0).all()       # s_hat = 0 where the anchor is zero
    check_decode(bt)


def test_constant_groups_anchor():
    rng = np.random.default_rng(2)
    K, V = synthetic(0x5EED0101)
    for X in (K, V):
        for grp in range(D // 16):
            sel = (np.arange(T + NTAIL) + grp) % 4 == 0
            # (the boolean index moves the token axis first: [tokens][B][H][16])
            vals = rng.standard_normal((int(sel.sum()), B, HKV, 1))
            X[LG - 1, :, sel, :, grp * 16:(grp + 1) * 16] = np.round(vals * 8) / 8   # BF16-exact constants
    bt = build(K, V)
    check_records(bt, strict=True)
    codes, meta, _ = bt.cache.export(0, LG - 1)
    assert (meta[..., 0::2] == 0).any()            # zero scales occurred
    check_decode(bt)


def test_constant_groups_residual_without_rotation():
    """Anchor on an FP8 grid (exact reconstruction) with zero groups; each
    loop equals the anchor except constants in those groups, so s_hat = 1 and
    the residual is exactly 0 or a constant per group."""
    rng = np.random.default_rng(3)
    K = np.zeros((LG, B, T + NTAIL, HKV, D))
    V = np.zeros_like(K)
    for X in (K, V):
        for b in range(B):
            for t in range(T + NTAIL):
                for h in range(HKV):
                    a = grid_record(rng, 4)
                    zg = rng.choice(D // 16, 3, replace=False)
                    for gz in zg:
                        a[gz * 16:(gz + 1) * 16] = 0.0
                    X[LG - 1, b, t, h] = a
                    for j in range(LG - 1):
                        x = a.copy()
                        for gz in zg:
                            x[gz * 16:(gz + 1) * 16] = float(rng.integers(-12, 13)) / 4
                        X[j, b, t, h] = x
    bt = build(K, V, rotate=False)
    check_records(bt, strict=True)
    for loop in range(LG - 1):
        _, meta, coef = bt.cache.export(0, loop)
        assert (coef == 0x3F80).all()              # s_hat = 1.0 exactly
        assert (meta[..., 0::2] == 0).all()        # every residual group has zero range
    check_decode(bt)


@pytest.mark.parametrize("scaled", ["K", "KV"])
def test_beyond_fp8_range(scaled):
    """Two channels x 10^4 and x -7000 (|x| up to ~10^5): minima below
    -448 and ranges above 15 x 448 saturate.  Attention is checked when only
    K is scaled (V of thousands would put the output beyond what an absolute
    2e-3 bound can measure in fp32)."""
    K, V = synthetic(0x5EED0102)
    for X in ((K, V) if scaled == "KV" else (K,)):
        X[..., 5] *= 1.0e4
        X[..., 77] *= -7.0e3
    bt = build(K, V)
    check_records(bt, strict=True)
    _, meta, _ = bt.cache.export(0, LG - 1)
    assert (meta[0][..., 0::2] == 0x7E).any() and (meta[0][..., 1::2] == 0xFE).any()   # +448 scale, -448 min
    if scaled == "K":
        check_decode(bt)


def _midpoint_groups(bits: int):
    """Groups (16 BF16 values each) whose range / (2^bits - 1) or whose
    minimum is an FP8 rounding midpoint, or one BF16 step away from one."""
    vals = fp8_values()
    mids = (vals[:-1] + vals[1:]) / 2
    qmax = (1 << bits) - 1
    groups = []
    for mid in mids[20:110:3]:
        # range at the midpoint (minimum 0), then one BF16 step up and down
        top = mid * qmax
        for step in (0, 1, -1):
            t = torch.tensor([top], dtype=torch.float64).to(torch.bfloat16)
            if step:
                bits16 = t.view(torch.int16) + step
                t = bits16.view(torch.bfloat16)
            tv = float(t.to(torch.float64))
            if step == 0 and tv != top:
                continue                              # the midpoint range is not BF16-exact
            g = np.linspace(0.0, tv, 16)
            g = torch.from_numpy(g).to(torch.bfloat16).to(torch.float64).numpy()
            g[0], g[-1] = 0.0, tv
            groups.append(g)
        # minimum at the midpoint (either sign), range an exact power of two
        for sgn in (1.0, -1.0):
            m = sgn * mid
            g = m + np.arange(16) % (qmax + 1) * 2.0 ** (np.floor(np.log2(mid)) - 1)
            if np.array_equal(torch.from_numpy(g).to(torch.bfloat16).to(torch.float64).numpy(), g):
                groups.append(g)
    return groups


def test_fp8_rounding_midpoints():
    """Anchor groups (INT4) and, without rotation, residual groups (INT2)
    placed at FP8 midpoints: GPU and oracle round the same fp64 scale and
    minimum, so they must agree bit for bit (ties to even), flagged or not.
    The anchor is zero in groups 4-7, so the residual there is the loop's own
    midpoint group."""
    ga, gr = _midpoint_groups(4), _midpoint_groups(2)
    rng = np.random.default_rng(4)
    K = np.zeros((LG, B, T + NTAIL, HKV, D))
    V = np.zeros_like(K)
    i = 0
    for X in (K, V):
        for b in range(B):
            for t in range(T + NTAIL):
                for h in range(HKV):
                    # groups 0-3: anchor at midpoints; groups 4-7: anchor zero,
                    # loops hold midpoint groups there and equal the anchor elsewhere
                    a = np.zeros(D)
                    for grp in range(4):
                        a[grp * 16:(grp + 1) * 16] = ga[(i + grp) % len(ga)][rng.permutation(16)]
                    X[LG - 1, b, t, h] = a
                    for j in range(LG - 1):
                        x = a.copy()
                        for grp in range(4, 8):
                            x[grp * 16:(grp + 1) * 16] = gr[(i + 3 * j + grp) % len(gr)][rng.permutation(16)]
                        X[j, b, t, h] = x
                    i += 1
    bf16_exact(K)
    bf16_exact(V)
    bt = build(K, V, rotate=False)
    e = H.oracle_encode(bt, 0, 0, 0)
    assert e.a_mflag.any() and e.r_mflag.any()      # the ties are there (and flagged)
    check_records(bt, strict=True)
    check_decode(bt)


def test_bf16_midpoint_coefficients():
    """Anchor of all ones (every group constant: scale 0, minimum 1.0, so
    a_hat = 1 exactly): s = sum(x) / 128, set exactly at BF16 midpoints,
    2^-20 off (inside the 1e-6 window) and 2^-9 off (outside it).  Both sides
    round the same fp64 s."""
    base = [128.5, 129.5, 128.0 + 2 ** -1 + 2 ** -2, 127.75 - 2 ** -3]
    deltas = [0.0, 2.0 ** -20, -2.0 ** -20, 2.0 ** -9, -2.0 ** -9]
    rows = []
    for s0 in base:
        for d in deltas:
            x = np.ones(D)
            x[0] = 1.0 + (s0 - 128.0)                # the bulk of the offset
            x[1], x[2] = d, 2.0                      # +d, sum otherwise unchanged
            rows.append(x)
    rng = np.random.default_rng(5)
    K = np.zeros((LG, B, T + NTAIL, HKV, D))
    V = np.zeros_like(K)
    i = 0
    for X in (K, V):
        X[LG - 1] = 1.0
        for b in range(B):
            for t in range(T + NTAIL):
                for h in range(HKV):
                    for j in range(LG - 1):
                        X[j, b, t, h] = rows[(i + 5 * j) % len(rows)][rng.permutation(D)]
                    i += 1
    bf16_exact(K)
    bf16_exact(V)
    for rotate in (False, True):
        bt = build(K, V, rotate=rotate)
        e = H.oracle_encode(bt, 0, 0, 0)
        assert e.r_cflag.any() and not e.r_cflag.all()
        # coefficients are compared bit for bit even where flagged
        for kv in (0, 1):
            e = H.oracle_encode(bt, 0, 0, kv)
            for j in range(LG - 1):
                _, _, f = H.gpu_records(bt, 0, j, kv)
                assert np.array_equal(f, e.r_coef[j]), (rotate, kv, j)
        check_records(bt, strict=not rotate)
        check_decode(bt)
        bt.cache.close()


def test_negative_zero_minima():
    """Groups whose minimum is -0 (with positives, or all -0) in the anchor,
    and all -0 residual groups (a -0 loop over a +0 anchor group, no
    rotation): the minimum is stored as +0 (0x00), never 0x80."""
    rng = np.random.default_rng(6)
    K = np.zeros((LG, B, T + NTAIL, HKV, D))
    V = np.zeros_like(K)
    for X in (K, V):
        for b in range(B):
            for t in range(T + NTAIL):
                for h in range(HKV):
                    a = grid_record(rng, 4)
                    a[0:16] = np.abs(np.round(rng.standard_normal(16) * 4) / 4)
                    a[rng.integers(0, 16)] = -0.0
                    a[16:32] = -0.0
                    a[32:48] = 0.0
                    X[LG - 1, b, t, h] = a
                    for j in range(LG - 1):
                        x = a.copy()
                        x[32:48] = -0.0
                        X[j, b, t, h] = x
    bt = build(K, V, rotate=False)
    check_records(bt, strict=True)
    for loop in range(LG):
        _, meta, _ = bt.cache.export(0, loop)
        assert not (meta[..., 1::2] == 0x80).any()
    check_decode(bt)


def test_identical_loops_on_fp8_grid():
    """Every loop equals a grid-valued anchor: s_hat = 1, the residual is 0
    (codes 0, scale 0, minimum 0) and every loop reconstructs exactly."""
    rng = np.random.default_rng(7)
    K = np.zeros((LG, B, T + NTAIL, HKV, D))
    V = np.zeros_like(K)
    for X in (K, V):
        for b in range(B):
            for t in range(T + NTAIL):
                for h in range(HKV):
                    X[:, b, t, h] = grid_record(rng, 4)
    for rotate in (True, False):
        bt = build(K, V, rotate=rotate)
        check_records(bt, strict=True)
        for kv, X in ((0, K), (1, V)):
            rec = H.reconstruct_gpu(bt, 0, 0, kv)                       # [Lg][B*H*T][d]
            x = X[:, :, :T].transpose(0, 1, 3, 2, 4).reshape(LG, -1, D)
            assert np.array_equal(rec, x)
        for loop in range(LG - 1):
            codes, meta, coef = bt.cache.export(0, loop)
            assert (codes == 0).all() and (meta == 0).all() and (coef == 0x3F80).all()
        check_decode(bt)
        bt.cache.close()


def test_identical_loops_general():
    K, V = synthetic(0x5EED0103)
    K[:LG - 1] = K[LG - 1]
    V[:LG - 1] = V[LG - 1]
    bt = build(K, V)
    check_records(bt, strict=True)
    for kv in (0, 1):
        g, o = H.mse_check(bt, 0, 0, kv)
        assert abs(g / o - 1.0) <= H.MSE_REL_TOL, (kv, g, o)
    check_decode(bt)


def test_small_v_subnormal_scales():
    K, V = synthetic(0x5EED0104, v_scale=1.0 / 64)
    bt = build(K, V)
    check_records(bt, strict=True)
    _, meta, _ = bt.cache.export(0, LG - 1)
    s8 = meta[1][..., 0::2]
    assert ((s8 > 0) & (s8 < 8)).any()               # subnormal E4M3 scales among the V anchors
    check_decode(bt)


def test_peaked_uniform_and_huge_queries():
    K, V = synthetic(0x5EED0105)
    bt = build(K, V)
    Kd, _ = bt.inputs[(0, 0)]
    rng = np.random.default_rng(8)

    def peaked(loop):
        # q = 8 x the unit direction of one committed key per (sequence, head)
        k = Kd[loop].float().cpu().numpy()
        q = rng.standard_normal((B, HQ, D))
        for b in range(B):
            for hq in range(HQ):
                t = int(rng.integers(0, T))
                kk = k[b, t, hq // (HQ // HKV)]
                q[b, hq] = 8.0 * np.sqrt(D) * kk / np.linalg.norm(kk)
        return torch.from_numpy(q).to(torch.bfloat16).cuda()

    check_decode(bt, peaked)
    check_decode(bt, lambda loop: torch.zeros((B, HQ, D), dtype=torch.bfloat16, device="cuda"))
    check_decode(bt, lambda loop: synth.queries(9, 0, loop, 0, B, HQ) * 64)
