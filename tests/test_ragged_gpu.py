"""Ragged batches: sequences of one cache holding different numbers of
committed tokens (rq_cache_truncate_seq), against the fp64 oracle.

For each sequence b the decode attends to its own first len_b committed
tokens (plus the loop's tail tokens); later appends write each sequence's
tokens after its own last one.  References are the oracle's attention over
the oracle reconstruction of the GPU's exported records, row range [0, len_b)
of each sequence, so the encoding itself stays checked by the uniform tests.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth
from oracle import oracle as orc

import rqharness as H

pytestmark = pytest.mark.gpu


def _recon(cache, cfg, layer, grp):
    """[kv][Lg][B][H][len][d] fp64 from the GPU's records (len = longest sequence)."""
    Lg = cfg.loops_per_group
    n = cache.length(layer, grp)
    out = []
    for kv in range(2):
        ex = [cache.export(layer, grp * Lg + j) for j in range(Lg)]
        ac, am = ex[-1][0][kv].reshape(-1, ex[-1][0].shape[-1]), ex[-1][1][kv].reshape(-1, ex[-1][1].shape[-1])
        if Lg > 1:
            rc = np.stack([e[0][kv].reshape(-1, e[0].shape[-1]) for e in ex[:-1]])
            rm = np.stack([e[1][kv].reshape(-1, e[1].shape[-1]) for e in ex[:-1]])
            rf = np.stack([e[2][kv].reshape(-1) for e in ex[:-1]])
        else:
            rc = rm = rf = None
        r = orc.reconstruct(ac, am, rc, rm, rf, Lg, 128, cfg.group_size, cfg.anchor_bits, cfg.resid_bits,
                            bool(cfg.rotate), cfg.seed)
        out.append(r.reshape(Lg, cfg.batch, cfg.num_kv_heads, n, 128))
    return out


def _reference(keys, vals, q_bf16, lens, Gq, tail=None):
    """keys/vals [B][H][len][d]; tail = (k, v) [B][n][H][d] fp64 or None."""
    qf = orc.bf16_bits_to_f64(synth.bf16_to_u16(q_bf16))
    B, Hkv = keys.shape[0], keys.shape[1]
    out = np.zeros((B, Hkv * Gq, 128))
    for b in range(B):
        for h in range(Hkv):
            k, v = keys[b, h, :lens[b]], vals[b, h, :lens[b]]
            if tail is not None:
                k = np.concatenate([k, tail[0][b, :, h]])
                v = np.concatenate([v, tail[1][b, :, h]])
            q = qf[b:b + 1, h * Gq:(h + 1) * Gq]
            out[b, h * Gq:(h + 1) * Gq] = orc.attention(q, k[None, :, None, :], v[None, :, None, :], H.scale32())[0]
    return out


def _check(out, ref):
    rel = float(np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(out - ref).max())
    assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (rel, mx)


@pytest.mark.parametrize("lens", [[300, 0, 137, 64], [1, 299, 65, 300]])
def test_ragged_decode_and_append(lens):
    B, Hkv, Hq, T = 4, 2, 4, 300
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hq, n_tail=0, chunk=64, seed=0x5EED8000,
                 max_tokens=T + 2)
    cache, cfg = bt.cache, bt.cfg
    for b, n in enumerate(lens):
        cache.truncate_seq(0, 0, b, n)
    assert [cache.length_seq(0, 0, b) for b in range(B)] == lens
    assert cache.length(0, 0) == max(lens)
    K, V = _recon(cache, cfg, 0, 0)
    for loop in range(4):
        q = synth.queries(0x5EED8000, 0, loop, 1, B, Hq)
        out = cache.decode(0, loop, q).cpu().numpy().astype(np.float64)
        _check(out, _reference(K[loop], V[loop], q, lens, Hq // Hkv))
        for b in range(B):
            if lens[b] == 0:
                assert (out[b] == 0).all()
    # one decode step: every loop appends one token (tails first, the anchor commits)
    g = torch.Generator(device="cuda").manual_seed(99)
    nk = torch.randn((4, B, 1, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    nv = torch.randn((4, B, 1, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    for loop in range(3):
        q = synth.queries(0x5EED8000, 0, loop, 2, B, Hq)
        out = cache.append_decode(0, loop, nk[loop], nv[loop], q).cpu().numpy().astype(np.float64)
        tail = (orc.bf16_bits_to_f64(synth.bf16_to_u16(nk[loop])), orc.bf16_bits_to_f64(synth.bf16_to_u16(nv[loop])))
        _check(out, _reference(K[loop], V[loop], q, lens, Hq // Hkv, tail))
    cache.append(0, 3, nk[3], nv[3])
    new = [n + 1 for n in lens]
    assert [cache.length_seq(0, 0, b) for b in range(B)] == new
    K, V = _recon(cache, cfg, 0, 0)
    for loop in range(4):
        q = synth.queries(0x5EED8000, 0, loop, 3, B, Hq)
        out = cache.decode(0, loop, q).cpu().numpy().astype(np.float64)
        _check(out, _reference(K[loop], V[loop], q, new, Hq // Hkv))
    cache.check()


def test_ragged_bf16_cache():
    B, Hkv, Hq, T = 3, 2, 2, 200
    bt = H.build(layers=1, loops=2, Lg=1, B=B, T=T, H=Hkv, Hq=Hq, fmt=rq.RQ_FMT_BF16, seed=0x5EED8100)
    lens = [200, 3, 0]
    for b, n in enumerate(lens):
        bt.cache.truncate_seq(0, 1, b, n)
    for loop in (0, 1):
        K, V = bt.inputs[(0, loop)]
        keys = orc.bf16_bits_to_f64(synth.bf16_to_u16(K[0])).transpose(0, 2, 1, 3)
        vals = orc.bf16_bits_to_f64(synth.bf16_to_u16(V[0])).transpose(0, 2, 1, 3)
        q = synth.queries(0x5EED8100, 0, loop, 1, B, Hq)
        out = bt.cache.decode(0, loop, q, bf16=True).cpu().numpy().astype(np.float64)
        _check(out, _reference(keys, vals, q, lens if loop == 1 else [T] * B, Hq // Hkv))
    bt.cache.check()


def test_ragged_full_size_ouro_8k():
    """Ouro-1.4B-shaped call (H = 16, T = 8192, batch 4) with sequence lengths
    8192, 5000, 100 and 0; sampled heads."""
    B, Hkv, T = 4, 16, 8192
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hkv, n_tail=0, chunk=1024, seed=0x5EED8200)
    cache, cfg = bt.cache, bt.cfg
    lens = [8192, 5000, 100, 0]
    for b, n in enumerate(lens):
        cache.truncate_seq(0, 0, b, n)
    K, V = _recon(cache, cfg, 0, 0)
    for loop in (0, 3):
        q = synth.queries(0x5EED8200, 0, loop, 1, B, Hkv)
        out = cache.decode(0, loop, q).cpu().numpy().astype(np.float64)
        heads = [0, 7, 15]
        ref = _reference(K[loop][:, heads], V[loop][:, heads], q[:, heads], lens, 1)
        _check(out[:, heads], ref)
    cache.check()


def test_truncate_seq_errors():
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=20, H=1, Hq=1, n_tail=1, seed=0x5EED8300)
    c = bt.cache
    assert rq.rq_cache_truncate_seq(c.h, 0, 0, 0, 5) == rq.RQ_ERR_STATE   # tails hold a token
    assert rq.rq_cache_truncate_seq(c.h, 0, 0, 2, 5) == rq.RQ_ERR_INVALID  # no sequence 2
    assert rq.rq_cache_truncate_seq(c.h, 0, 1, 0, 5) == rq.RQ_ERR_INVALID  # no group 1
    assert c.length_seq(0, 0, 1) == 20
