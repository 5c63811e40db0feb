"""rq_append_decode_attn against rq_append followed by rq_decode_attn.

The fused call must leave the cache in the same state and return the same
output bit for bit: for a non-anchor loop with committed tokens it is one
launch whose split-0 CTAs write the new tail rows before the combining CTA
reads them; otherwise it enqueues the two calls.  A decode step appends one
token to every loop of a group (the anchor last, which commits the token and
empties the tails), as the ai4snews summary's decode describes.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _step_inputs(seed, layer, grp, Lg, B, Hkv, Hq, step):
    g = torch.Generator(device="cuda").manual_seed(seed * 7919 + layer * 131 + grp * 17 + step)
    k = torch.randn((Lg, B, 1, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((Lg, B, 1, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    q = [synth.queries(seed, layer, grp * Lg + j, 1000 + step, B, Hq) for j in range(Lg)]
    return k, v, q


def _same_state(a, b, layers, loops, Lg):
    for layer in range(layers):
        for loop in range(loops):
            assert a.tail_length(layer, loop) == b.tail_length(layer, loop)
            if loop % Lg == Lg - 1:
                assert a.length(layer, loop // Lg) == b.length(layer, loop // Lg)
            ea, eb = a.export(layer, loop), b.export(layer, loop)
            for xa, xb in zip(ea, eb):
                if xa is None:
                    assert xb is None
                else:
                    assert np.array_equal(xa, xb), (layer, loop)


@pytest.mark.parametrize("T,B,Hkv,Hq,steps", [(200, 2, 2, 4, 2), (1000, 1, 2, 8, 1), (0, 1, 2, 2, 2), (64, 2, 3, 3, 3)])
def test_fused_step_matches_separate_calls(T, B, Hkv, Hq, steps):
    kw = dict(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hq, n_tail=0, seed=0x5EED6000 + T,
              max_tokens=T + steps)
    a, b = H.build(**kw), H.build(**kw)
    for step in range(steps):
        k, v, q = _step_inputs(0x5EED6000 + T, 0, 0, 4, B, Hkv, Hq, step)
        for j in range(4):
            a.cache.append(0, j, k[j], v[j])
            oa = a.cache.decode(0, j, q[j])
            ob = b.cache.append_decode(0, j, k[j], v[j], q[j])
            torch.cuda.synchronize()
            assert torch.equal(oa, ob), (step, j, (oa - ob).abs().max().item())
            assert a.cache.tail_length(0, j) == b.cache.tail_length(0, j)
    a.cache.check()
    b.cache.check()
    _same_state(a.cache, b.cache, 1, 4, 4)


def test_fused_repeated_tail_appends():
    """Several tokens kept in a non-anchor loop's tail before any commit."""
    kw = dict(layers=1, loops=4, Lg=4, B=2, T=300, H=2, Hq=2, n_tail=0, seed=0x5EED6100)
    a, b = H.build(**kw), H.build(**kw)
    for step in range(5):
        k, v, q = _step_inputs(0x5EED6100, 0, 0, 4, 2, 2, 2, step)
        a.cache.append(0, 1, k[1], v[1])
        oa = a.cache.decode(0, 1, q[1])
        ob = b.cache.append_decode(0, 1, k[1], v[1], q[1])
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), step
        assert b.cache.tail_length(0, 1) == step + 1
    _same_state(a.cache, b.cache, 1, 4, 4)


def test_fused_capacity_and_errors():
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=100, H=2, Hq=2, n_tail=0, chunk=4, seed=0x5EED6200)
    k, v, q = _step_inputs(0x5EED6200, 0, 0, 4, 1, 2, 2, 0)
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    for i in range(4):   # tail capacity is 4 tokens
        assert rq.rq_append_decode_attn(bt.cache.h, 0, 0, k[0], v[0], 1, q[0], out, 0.0) == rq.RQ_OK
    assert rq.rq_append_decode_attn(bt.cache.h, 0, 0, k[0], v[0], 1, q[0], out, 0.0) == rq.RQ_ERR_CAPACITY
    assert bt.cache.tail_length(0, 0) == 4
    assert rq.rq_append_decode_attn(bt.cache.h, 0, 9, k[0], v[0], 1, q[0], out, 0.0) == rq.RQ_ERR_INVALID
    assert rq.rq_append_decode_attn(bt.cache.h, 0, 0, k[0], v[0], 0, q[0], out, 0.0) == rq.RQ_ERR_INVALID
    assert rq.rq_append_decode_attn(bt.cache.h, 0, 0, k[0], v[0], 1, None, out, 0.0) == rq.RQ_ERR_INVALID
    assert bt.cache.tail_length(0, 0) == 4
    bt.cache.check()


def test_fused_full_size_ouro_8k():
    """Ouro-1.4B-shaped call (H = 16, T = 8192, batch 4): the launch the bench times."""
    kw = dict(layers=1, loops=4, Lg=4, B=4, T=8192, H=16, Hq=16, n_tail=0, chunk=1024, seed=0x5EED6300,
              max_tokens=8193)
    a, b = H.build(**kw), H.build(**kw)
    k, v, q = _step_inputs(0x5EED6300, 0, 0, 4, 4, 16, 16, 0)
    for j in range(4):
        a.cache.append(0, j, k[j], v[j])
        oa = a.cache.decode(0, j, q[j])
        ob = b.cache.append_decode(0, j, k[j], v[j], q[j])
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), j
    assert a.cache.length(0, 0) == b.cache.length(0, 0) == 8193
    a.cache.check()
    b.cache.check()
