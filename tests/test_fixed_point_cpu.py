"""The decode kernel's fixed-point arithmetic, emulated on the CPU.

The kernel computes the two products of decode attention on integer
dot-product units, which rounds two quantities (everything else is fp32):
  * q and R q become integers, q_int = rint(q * 2^F), with 2^F the power of
    two putting max(|q|, |R q|) into [2^21, 2^22) -- 24-bit two's complement
    split into three byte planes;
  * the V weights of a split chunk, p_t * s_hat_t * scale_{t,g} (anchor basis)
    and p_t * scale'_{t,g} (rotated basis), become integers with a power of
    two putting the chunk's bound (max |s_hat| of the chunk x the largest
    anchor V scale of the (sequence, head) stream, resp. the largest residual
    V scale of the stream) into [2^21, 2^22); the group minima are summed in
    floating point.
This test restates that arithmetic with numpy on the oracle's records of the
Ouro-shaped synthetic workload and bounds its error against exact fp64
attention over the same records: the rounding alone must stay well inside the
parity bound (max abs 2e-3) that the GPU tests apply, with room left for the
fp32 arithmetic around it.  It exercises no GPU code; it documents why 24 and
22 bits were chosen (with 12-bit weights the same arithmetic breaks the
bound), and why the weight bound follows the stream's actual V scales rather
than the largest FP8 value: with V 64 times smaller the fixed bound loses
the output's relative precision, the stream bound keeps it.
"""
import math

import numpy as np
import pytest

import synth
from oracle import oracle as orc

D = 128
SEED = 0xA11CE


def _pow2_scale(bound: float, top: int) -> float:
    m, e = math.frexp(bound)   # bound = m 2^e, m in [0.5, 1)
    return 2.0 ** (top - e)


def _fp8(codes: np.ndarray) -> np.ndarray:
    table = np.array([orc.fp8_value(c) for c in range(256)])
    return table[codes]


def _unpack(packed: np.ndarray, bits: int) -> np.ndarray:
    per = 8 // bits
    return np.stack([(packed >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], -1).reshape(
        packed.shape[0], -1).astype(np.float64)


@pytest.fixture(scope="module")
def workload():
    T, H = 2048, 2
    K, V = synth.group_kv(0x5EED0001, 0, 0, 4, (0.1, 0.2, 0.3), 1, T, H, device="cpu")
    out = {}
    for name, X in (("K", K), ("V", V)):
        x = np.stack([synth.bf16_to_u16(X[j]).transpose(0, 2, 1, 3).reshape(-1, D) for j in range(4)])
        e = orc.encode(x, 16, 4, 2, True, SEED)
        xhat = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, 4, D, 16, 4, 2, True, SEED)
        out[name] = (e, xhat)
    return T, H, out


def _emulate(T, H, rec, q_unit, loop, chunk, q_bits=22, w_top=22, bound="stream"):
    """(emulated, exact) attention outputs [H][d] of one loop."""
    (eK, kh), (eV, vh) = rec["K"], rec["V"]
    R = orc.rotation_matrix(SEED, D)
    resid = loop < 3
    a_k = kh[3].reshape(H, T, D)
    a_v_codes = _unpack(eV.a_codes, 4).reshape(H, T, D)
    a_v_meta = eV.a_meta.reshape(H, T, 8, 2)
    if resid:
        shk = orc.bf16_bits_to_f64(eK.r_coef[loop]).reshape(H, T)
        shv = orc.bf16_bits_to_f64(eV.r_coef[loop]).reshape(H, T)
        y_k = (kh[loop].reshape(H, T, D) - shk[..., None] * a_k) @ R.T     # rotated residual, R (k - s a)
        r_v_codes = _unpack(eV.r_codes[loop], 2).reshape(H, T, D)
        r_v_meta = eV.r_meta[loop].reshape(H, T, 8, 2)
    emu, exact = [], []
    for h in range(H):
        q = q_unit[h] / math.sqrt(D) * math.log2(math.e)
        k_full = kh[loop].reshape(H, T, D)[h]
        v_full = vh[loop].reshape(H, T, D)[h]
        # exact
        z = k_full @ q
        p = 2.0 ** (z - z.max())
        exact.append((p[:, None] * v_full).sum(0) / p.sum())
        # logits with integer q
        rq = R @ q
        S = _pow2_scale(max(np.abs(q).max(), np.abs(rq).max() if resid else 0.0), q_bits)
        qi, rqi = np.rint(q * S), np.rint(rq * S)
        if resid:
            ze = (shk[h] * (a_k[h] @ qi) + y_k[h] @ rqi) / S
        else:
            ze = (a_k[h] @ qi) / S
        # V accumulation per split chunk with integer weights
        M = ze.max()
        num, den = np.zeros(D), 0.0
        for c0 in range(0, T, chunk):
            sl = slice(c0, min(T, c0 + chunk))
            m = ze[sl].max()
            pc = 2.0 ** (ze[sl] - m)
            sv = shv[h, sl] if resid else np.ones(sl.stop - sl.start)
            sc, mn = _fp8(a_v_meta[h, sl, :, 0]), _fp8(a_v_meta[h, sl, :, 1])
            vA = _fp8(a_v_meta[h, :, :, 0]).max() if bound == "stream" else 448.0
            cA = _pow2_scale(np.abs(sv).max() * vA, w_top)
            w = np.rint((pc * sv)[:, None] * sc * cA) / cA                          # [t][group]
            acc = (np.repeat(w, 16, 1) * a_v_codes[h, sl]).sum(0) + ((pc * sv)[:, None] * np.repeat(mn, 16, 1)).sum(0)
            if resid:
                scr, mnr = _fp8(r_v_meta[h, sl, :, 0]), _fp8(r_v_meta[h, sl, :, 1])
                vR = _fp8(r_v_meta[h, :, :, 0]).max() if bound == "stream" else 448.0
                cR = _pow2_scale(vR, w_top)
                wr = np.rint(pc[:, None] * scr * cR) / cR
                accr = (np.repeat(wr, 16, 1) * r_v_codes[h, sl]).sum(0) + (pc[:, None] * np.repeat(mnr, 16, 1)).sum(0)
                acc = acc + R.T @ accr
            f = 2.0 ** (m - M)
            num += f * acc
            den += f * pc.sum()
        emu.append(num / den)
    return np.array(emu), np.array(exact)


@pytest.mark.parametrize("loop", [0, 3])
def test_kernel_rounding_within_the_parity_bound(workload, loop):
    T, H, rec = workload
    rng = np.random.default_rng(11)
    q = rng.standard_normal((H, D))
    emu, exact = _emulate(T, H, rec, q, loop, chunk=256)
    assert np.abs(emu - exact).max() < 2e-4


def test_kernel_rounding_with_a_dominant_key(workload):
    """A query aligned with one key (logit gap of tens): the weights of the
    other keys are tiny, the dominant one near the bound."""
    T, H, rec = workload
    kh = rec["K"][1][1].reshape(H, T, D)
    rng = np.random.default_rng(12)
    q = rng.standard_normal((H, D)) + 8.0 * kh[:, T // 3] / np.linalg.norm(kh[:, T // 3], axis=1, keepdims=True)
    emu, exact = _emulate(T, H, rec, q, 1, chunk=256)
    assert np.abs(emu - exact).max() < 6e-4


def test_twelve_bit_weights_would_not_do(workload):
    """The same emulation with 12-bit V weights (bound in [2^11, 2^12)) breaks
    the parity bound: the 22-bit choice leaves a wide margin."""
    T, H, rec = workload
    rng = np.random.default_rng(11)
    q = rng.standard_normal((H, D))
    emu, exact = _emulate(T, H, rec, q, 0, chunk=256, w_top=12)
    assert np.abs(emu - exact).max() > 2e-3


@pytest.fixture(scope="module")
def small_v_workload():
    """The same loop group with V divided by 64 (exact in BF16): its FP8
    scales fall to the subnormal range."""
    T, H = 2048, 2
    K, V = synth.group_kv(0x5EED0001, 0, 0, 4, (0.1, 0.2, 0.3), 1, T, H, device="cpu")
    V = [v / 64 for v in V]
    out = {}
    for name, X in (("K", K), ("V", V)):
        x = np.stack([synth.bf16_to_u16(X[j]).transpose(0, 2, 1, 3).reshape(-1, D) for j in range(4)])
        e = orc.encode(x, 16, 4, 2, True, SEED)
        xhat = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes, e.r_meta, e.r_coef, 4, D, 16, 4, 2, True, SEED)
        out[name] = (e, xhat)
    return T, H, out


@pytest.mark.parametrize("loop", [0, 3])
def test_small_v_needs_the_stream_bound(small_v_workload, loop):
    """Relative L2 error of the output against exact attention with V / 64:
    within 2e-4 with the stream bound, beyond the 1e-3 parity bound with a
    bound fixed at the largest FP8 value (448)."""
    T, H, rec = small_v_workload
    q = np.random.default_rng(13).standard_normal((H, D))
    emu, exact = _emulate(T, H, rec, q, loop, chunk=256)
    assert np.linalg.norm(emu - exact) / np.linalg.norm(exact) < 2e-4
    emu, exact = _emulate(T, H, rec, q, loop, chunk=256, w_top=28, bound="fixed448")
    assert np.linalg.norm(emu - exact) / np.linalg.norm(exact) > 1e-3


def test_emulation_is_exact_attention_without_rounding(workload):
    """With 40-bit q and 50-bit weights the emulation is exact attention over
    the records (so the bounds above measure the rounding, not the emulation)."""
    T, H, rec = workload
    q = np.random.default_rng(11).standard_normal((H, D))
    for loop in (0, 3):
        emu, exact = _emulate(T, H, rec, q, loop, chunk=256, q_bits=40, w_top=50)
        assert np.abs(emu - exact).max() < 1e-9
