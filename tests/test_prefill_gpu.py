"""Multi-token causal attention (rq_prefill_attn) against the fp64 oracle.

Query token i of n of sequence b sees the first len_b + n_tail - n + 1 + i
tokens of [committed tokens, tail tokens].  References are the oracle's
attention, one query row at a time, over the oracle reconstruction of the
GPU's exported records (the encoding itself is checked by the decode tests)
followed by the BF16 tail tokens.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth
from oracle import oracle as orc

import rqharness as H

pytestmark = pytest.mark.gpu


def _recon(cache, cfg, layer, grp, sel=None):
    """(K, V), each [Lg][nsel][len][d] fp64, from the GPU's records (len = the
    longest sequence)."""
    Lg = cfg.loops_per_group
    n = cache.length(layer, grp)
    sel = sel or [(b, h) for b in range(cfg.batch) for h in range(cfg.num_kv_heads)]
    out = []
    for kv in range(2):
        ex = [cache.export(layer, grp * Lg + j) for j in range(Lg)]

        def pick(a):
            a = a[kv]
            return np.stack([a[b, h] for (b, h) in sel]).reshape(-1, a.shape[-1])

        ac, am = pick(ex[-1][0]), pick(ex[-1][1])
        if Lg > 1:
            rc = np.stack([pick(e[0]) for e in ex[:-1]])
            rm = np.stack([pick(e[1]) for e in ex[:-1]])
            rf = np.stack([np.stack([e[2][kv][b, h] for (b, h) in sel]).reshape(-1) for e in ex[:-1]])
        else:
            rc = rm = rf = None
        r = orc.reconstruct(ac, am, rc, rm, rf, Lg, 128, cfg.group_size, cfg.anchor_bits, cfg.resid_bits,
                            bool(cfg.rotate), cfg.seed)
        out.append(r.reshape(Lg, len(sel), n, 128))
    return out


def _reference(keys, vals, q_bf16, lens, n_tail, G, sel, tail=None):
    """keys/vals [nsel][len][d] (committed); tail (k, v) [B][n_tail][H][d] fp64;
    q [B][n][Hq][d].  Returns {(b, h): [n][G][d]}."""
    qf = orc.bf16_bits_to_f64(synth.bf16_to_u16(q_bf16))
    n = qf.shape[1]
    out = {}
    for s, (b, h) in enumerate(sel):
        rows = []
        for i in range(n):
            tot = lens[b] + n_tail - n + 1 + i
            lc, lt = min(lens[b], tot), max(0, tot - lens[b])
            k, v = keys[s, :lc], vals[s, :lc]
            if lt:
                k = np.concatenate([k, tail[0][b, :lt, h]])
                v = np.concatenate([v, tail[1][b, :lt, h]])
            q = qf[b:b + 1, i, h * G:(h + 1) * G]
            rows.append(orc.attention(q, k[None, :, None, :], v[None, :, None, :], H.scale32())[0])
        out[(b, h)] = np.stack(rows)
    return out


def _check(out, ref, G):
    g = np.concatenate([out[b, :, h * G:(h + 1) * G] for (b, h) in ref]).astype(np.float64)
    r = np.concatenate(list(ref.values()))
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    mx = float(np.abs(g - r).max())
    assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (rel, mx)


def _new_tokens(seed, loops, B, n, Hkv):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randn((loops, B, n, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((loops, B, n, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    return k, v


def _queries(seed, B, n, Hq):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((B, n, Hq, 128), generator=g, device="cuda").to(torch.bfloat16)


def _f64(t):
    return orc.bf16_bits_to_f64(synth.bf16_to_u16(t))


@pytest.mark.parametrize("n,Hq", [(1, 4), (5, 4), (7, 8), (33, 4)])
def test_prefill_chunk_through_a_group(n, Hq):
    """A chunk of n tokens through loops 0..3: tails at loops 0-2, committed
    at the anchor loop; then loop 0 again with the chunk committed.  n * G
    query rows per kv head: 2, 10, 28 and 66 (1, 2, 4 and 8 rows per warp,
    the last over two row blocks)."""
    B, Hkv, T = 2, 2, 300
    G = Hq // Hkv
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hq, n_tail=0, chunk=64, seed=0x5EED9000,
                 max_tokens=T + n)
    cache, cfg = bt.cache, bt.cfg
    sel = [(b, h) for b in range(B) for h in range(Hkv)]
    K, V = _recon(cache, cfg, 0, 0)
    nk, nv = _new_tokens(7 + n, 4, B, n, Hkv)
    for loop in range(3):
        cache.append(0, loop, nk[loop], nv[loop])
        q = _queries(100 + loop, B, n, Hq)
        out = cache.prefill(0, loop, q).cpu().numpy()
        ref = _reference(K[loop], V[loop], q, [T] * B, n, G, sel, (_f64(nk[loop]), _f64(nv[loop])))
        _check(out, ref, G)
    cache.append(0, 3, nk[3], nv[3])
    assert cache.length(0, 0) == T + n
    K, V = _recon(cache, cfg, 0, 0)
    for loop in (3, 0):
        q = _queries(200 + loop, B, n, Hq)
        out = cache.prefill(0, loop, q).cpu().numpy()
        _check(out, _reference(K[loop], V[loop], q, [T + n] * B, 0, G, sel), G)
    cache.check()


def test_prefill_ragged_int2_no_rotation():
    """Per-sequence lengths (one sequence with no committed token: its
    queries see only the chunk), uniform INT2, rotation off, one q head per
    kv head."""
    B, Hkv, T, n = 3, 2, 260, 3
    bt = H.build(layers=1, loops=2, Lg=2, B=B, T=T, H=Hkv, Hq=Hkv, ba=2, br=2, rotate=False, n_tail=0, chunk=64,
                 seed=0x5EED9100, max_tokens=T + n)
    cache, cfg = bt.cache, bt.cfg
    lens = [260, 0, 77]
    for b, L in enumerate(lens):
        cache.truncate_seq(0, 0, b, L)
    sel = [(b, h) for b in range(B) for h in range(Hkv)]
    K, V = _recon(cache, cfg, 0, 0)
    nk, nv = _new_tokens(31, 2, B, n, Hkv)
    cache.append(0, 0, nk[0], nv[0])
    q = _queries(300, B, n, Hkv)
    out = cache.prefill(0, 0, q).cpu().numpy()
    _check(out, _reference(K[0], V[0], q, lens, n, 1, sel, (_f64(nk[0]), _f64(nv[0]))), 1)
    cache.append(0, 1, nk[1], nv[1])
    new = [L + n for L in lens]
    K, V = _recon(cache, cfg, 0, 0)
    q = _queries(301, B, n, Hkv)
    out = cache.prefill(0, 1, q).cpu().numpy()
    _check(out, _reference(K[1], V[1], q, new, 0, 1, sel), 1)
    cache.check()


def test_prefill_many_query_rows():
    """n * G = 160 query rows per kv head (three row blocks, the last partial),
    committed tokens over many splits, INT4 residuals, group 32."""
    B, Hkv, Hq, T, n = 1, 2, 8, 1000, 40
    G = Hq // Hkv
    bt = H.build(layers=1, loops=2, Lg=2, B=B, T=T, H=Hkv, Hq=Hq, g=32, br=4, n_tail=0, chunk=128,
                 seed=0x5EED9200, max_tokens=T + n)
    cache, cfg = bt.cache, bt.cfg
    sel = [(0, 0), (0, 1)]
    K, V = _recon(cache, cfg, 0, 0)
    nk, nv = _new_tokens(41, 2, B, n, Hkv)
    cache.append(0, 0, nk[0], nv[0])
    q = _queries(400, B, n, Hq)
    out = cache.prefill(0, 0, q).cpu().numpy()
    _check(out, _reference(K[0], V[0], q, [T], n, G, sel, (_f64(nk[0]), _f64(nv[0]))), G)
    cache.check()


def test_prefill_long_chunk_in_the_tail():
    """A 150-token chunk in the tail of loop 1: 150 query rows per kv head
    (three 64-row blocks), and tails longer than one 128-token batch of the
    combine kernel; then committed at the anchor loop."""
    B, Hkv, T, n = 2, 2, 700, 150
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hkv, n_tail=0, chunk=256, seed=0x5EED9250,
                 max_tokens=T + n)
    cache, cfg = bt.cache, bt.cfg
    sel = [(b, h) for b in range(B) for h in range(Hkv)]
    K, V = _recon(cache, cfg, 0, 0)
    nk, nv = _new_tokens(61, 4, B, n, Hkv)
    cache.append(0, 0, nk[0], nv[0])
    cache.append(0, 1, nk[1], nv[1])
    q = _queries(450, B, n, Hkv)
    out = cache.prefill(0, 1, q).cpu().numpy()
    _check(out, _reference(K[1], V[1], q, [T] * B, n, 1, sel, (_f64(nk[1]), _f64(nv[1]))), 1)
    cache.append(0, 2, nk[2], nv[2])
    cache.append(0, 3, nk[3], nv[3])
    K, V = _recon(cache, cfg, 0, 0)
    q = _queries(451, B, n, Hkv)
    out = cache.prefill(0, 3, q).cpu().numpy()
    _check(out, _reference(K[3], V[3], q, [T + n] * B, 0, 1, sel), 1)
    cache.check()


def test_prefill_repeated_calls_and_growing_row_blocks():
    """The last split of a row block merges the partials, found with arrival
    counters that every call leaves at zero: on one cache with many splits per
    row block, repeated calls give bit-identical outputs, also after a call
    with more row blocks (the counter buffer grows) and back, and both sizes
    match the oracle."""
    B, Hkv, Hq, T, nb = 2, 2, 4, 3000, 40   # nb * G = 80 query rows per kv head: two row blocks
    G = Hq // Hkv
    bt = H.build(layers=1, loops=2, Lg=2, B=B, T=T, H=Hkv, Hq=Hq, n_tail=0, chunk=128, seed=0x5EED9400,
                 max_tokens=T + nb)
    cache, cfg = bt.cache, bt.cfg
    sel = [(b, h) for b in range(B) for h in range(Hkv)]
    K, V = _recon(cache, cfg, 0, 0)
    nk, nv = _new_tokens(71, 2, B, nb, Hkv)
    cache.append(0, 0, nk[0], nv[0])   # in loop 0's tail
    tail = (_f64(nk[0]), _f64(nv[0]))
    q_small, q_big = _queries(500, B, 4, Hq), _queries(501, B, nb, Hq)
    o1 = cache.prefill(0, 0, q_small)
    o2 = cache.prefill(0, 0, q_small)
    o3 = cache.prefill(0, 0, q_big)
    o4 = cache.prefill(0, 0, q_small)
    o5 = cache.prefill(0, 0, q_big)
    assert torch.equal(o1, o2) and torch.equal(o1, o4) and torch.equal(o3, o5)
    _check(o1.cpu().numpy(), _reference(K[0], V[0], q_small, [T] * B, nb, G, sel, tail), G)
    _check(o3.cpu().numpy(), _reference(K[0], V[0], q_big, [T] * B, nb, G, sel, tail), G)
    cache.check()


def test_prefill_one_token_is_decode():
    B, Hkv, Hq, T = 2, 2, 4, 200
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hq, n_tail=1, chunk=64, seed=0x5EED9300)
    cache = bt.cache
    for loop in range(4):
        q = synth.queries(0x5EED9300, 0, loop, 1, B, Hq)
        d = cache.decode(0, loop, q).cpu().numpy()
        p = cache.prefill(0, loop, q[:, None].contiguous()).cpu().numpy()[:, 0]
        rel = np.linalg.norm(p - d) / np.linalg.norm(d)
        assert rel < 1e-3 and np.abs(p - d).max() < 1e-3, (loop, rel)


def test_prefill_full_size_ouro_8k_sampled():
    """Ouro-1.4B-shaped cache (H = 16, T = 8192, batch 4), a 16-token chunk in
    the tail of loop 1; sampled (sequence, head) units."""
    B, Hkv, T, n = 4, 16, 8192, 16
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hkv, n_tail=0, chunk=1024, seed=0x5EED9400,
                 max_tokens=T + n)
    cache, cfg = bt.cache, bt.cfg
    sel = [(0, 0), (1, 7), (3, 15)]
    K, V = _recon(cache, cfg, 0, 0, sel)
    nk, nv = _new_tokens(51, 4, B, n, Hkv)
    cache.append(0, 0, nk[0], nv[0])
    cache.append(0, 1, nk[1], nv[1])
    q = _queries(500, B, n, Hkv)
    out = cache.prefill(0, 1, q).cpu().numpy()
    _check(out, _reference(K[1], V[1], q, [T] * B, n, 1, sel, (_f64(nk[1]), _f64(nv[1]))), 1)
    cache.check()


def test_prefill_errors():
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=3, H=1, Hq=1, n_tail=1, seed=0x5EED9500)
    c = bt.cache
    q = torch.zeros((2, 5, 1, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((2, 5, 1, 128), dtype=torch.float32, device="cuda")
    assert rq.rq_prefill_attn(c.h, 0, 0, q, 5, out) == rq.RQ_ERR_STATE      # 3 + 1 tokens < 5
    assert rq.rq_prefill_attn(c.h, 0, 0, q, 0, out) == rq.RQ_ERR_INVALID
    assert rq.rq_prefill_attn(c.h, 0, 4, q, 1, out) == rq.RQ_ERR_INVALID    # no loop 4
    assert rq.rq_prefill_attn(c.h, 0, 0, q, 4, out) == rq.RQ_OK
    bf = H.build(layers=1, loops=1, Lg=1, B=2, T=3, H=1, Hq=1, fmt=rq.RQ_FMT_BF16, seed=0x5EED9600)
    assert rq.rq_prefill_attn(bf.cache.h, 0, 0, q, 1, out) == rq.RQ_ERR_STATE
    c.check()
