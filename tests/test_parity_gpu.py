"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Encoding (rq_append): codes / FP8 meta / BF16 coefficients bit-exact except
oracle-flagged near-boundary values.  Decode (rq_decode_attn): relative L2
<= 1e-3 and max abs <= 2e-3 against the oracle fed the GPU's own records.
Reconstruction MSE within 1% of the oracle's own encoding.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _decode_and_check(bt, layer, loop, bh_sel=None, step=0):
    cfg = bt.cfg
    q = synth.queries(bt.seed, layer, loop, step, cfg.batch, cfg.num_q_heads)
    out = bt.cache.decode(layer, loop, q, out=H.guarded_out((cfg.batch, cfg.num_q_heads, 128))).cpu().numpy()
    ref = H.oracle_decode(bt, layer, loop, q, bh_sel)
    rel, mx = H.attn_errors(out, ref, cfg.num_q_heads // cfg.num_kv_heads)
    assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (layer, loop, rel, mx)
    return rel, mx


def _records_and_mse(bt, layer, grp, bh_sel=None):
    for kv in (0, 1):
        r = H.compare_records(bt, layer, grp, kv, bh_sel)
        assert r["mismatch"] == 0, r
        assert r["compared"] > 0
        # differences are only tolerated at flagged boundary values; they and
        # the records they exclude must stay rare
        assert r["tolerated"] == 0, r   # none on the synthetic workloads (reported when nonzero)
        assert r["excluded"] <= 1e-2 * r["compared"] + 64, r
        g, o = H.mse_check(bt, layer, grp, kv, bh_sel)
        assert abs(g / o - 1.0) <= H.MSE_REL_TOL, (kv, g, o)


# ------------------------------------------------------------ tiny config
def test_tiny_config_full():
    """1 layer, 4 loops (loop 4 INT4 anchor, loops 1-3 INT2 residuals),
    batch 1, T=256, H_kv=4, H_q=8, d=128, g=16."""
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=256, H=4, Hq=8, sigma=(0.1, 0.2, 0.3), seed=0x5EED0000)
    _records_and_mse(bt, 0, 0)
    for loop in range(4):
        _decode_and_check(bt, 0, loop)
    assert bt.cache.length(0, 0) == 256


@pytest.mark.parametrize("T,n_tail", [(1, 0), (1, 1), (15, 3), (63, 1), (64, 0), (65, 2), (200, 3), (1000, 1)])
def test_ragged_lengths_and_tails(T, n_tail):
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=T, H=2, Hq=4, n_tail=n_tail, seed=0x5EED1000 + T, chunk=64)
    _records_and_mse(bt, 0, 0)
    for loop in range(4):
        _decode_and_check(bt, 0, loop)
        assert bt.cache.tail_length(0, loop) == (n_tail if loop < 3 else 0)


def test_empty_cache_tail_only_and_nothing():
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=0, H=2, Hq=2, n_tail=2, seed=0x5EED2000)
    for loop in range(3):
        _decode_and_check(bt, 0, loop)     # tail tokens only
    q = synth.queries(1, 0, 3, 0, 1, 2)
    out = bt.cache.decode(0, 3, q)       # anchor loop, nothing committed: zeros
    assert (out == 0).all()


@pytest.mark.parametrize("g,ba,br,rotate", [(32, 4, 2, True), (16, 2, 2, True), (16, 4, 4, True),
                                            (16, 4, 2, False), (32, 2, 4, False)])
def test_format_variants(g, ba, br, rotate):
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=130, H=3, Hq=3, g=g, ba=ba, br=br, rotate=rotate,
                 n_tail=1, seed=0x5EED3000 + g + ba + br)
    _records_and_mse(bt, 0, 0)
    for loop in range(4):
        _decode_and_check(bt, 0, loop)


@pytest.mark.parametrize("Hq", [2, 4, 8])
def test_gqa_groupings(Hq):
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=96, H=1, Hq=Hq, n_tail=1, seed=0x5EED4000 + Hq)
    for loop in range(4):
        _decode_and_check(bt, 0, loop)


def test_every_loop_its_own_anchor():
    bt = H.build(layers=2, loops=3, Lg=1, B=1, T=70, H=2, Hq=2, seed=0x5EED5000)
    for layer in range(2):
        for grp in range(3):
            _records_and_mse(bt, layer, grp)
            _decode_and_check(bt, layer, grp)


def test_deep_recurrence_groups_small():
    """32 loops in 8 groups of 4 (each group anchored on its own last loop),
    sigma growing with distance from the group anchor 0.1 -> 0.4."""
    bt = H.build(layers=1, loops=32, Lg=4, B=1, T=80, H=2, Hq=2, sigma=(0.1, 0.25, 0.4), seed=0x5EED6000)
    for grp in (0, 5, 7):
        _records_and_mse(bt, 0, grp)
    for loop in (0, 3, 13, 31):
        _decode_and_check(bt, 0, loop)


@pytest.mark.parametrize("Lg", [8, 16])
def test_larger_loop_groups(Lg):
    """Loop groups of 8 and 16 (one anchor per group, Lg - 1 residual loops
    per anchor), sigma growing linearly with distance from the anchor."""
    sigma = tuple(0.1 + 0.3 * d / (Lg - 2) for d in range(Lg - 1))
    bt = H.build(layers=1, loops=2 * Lg, Lg=Lg, B=1, T=90, H=2, Hq=2, n_tail=1, sigma=sigma, seed=0x5EED6100 + Lg)
    for grp in (0, 1):
        _records_and_mse(bt, 0, grp)
    for loop in (0, Lg // 2, Lg - 1, Lg, 2 * Lg - 2, 2 * Lg - 1):
        _decode_and_check(bt, 0, loop)


def test_bf16_comparison_kernel():
    bt = H.build(layers=1, loops=2, Lg=1, B=2, T=300, H=2, Hq=4, fmt=rq.RQ_FMT_BF16, seed=0x5EED7000)
    for loop in range(2):
        q = synth.queries(bt.seed, 0, loop, 0, 2, 4)
        out = bt.cache.decode(0, loop, q, bf16=True).cpu().numpy()
        ref = H.oracle_decode(bt, 0, loop, q, bf16_cache=True)
        rel, mx = H.attn_errors(out, ref, 2)
        assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (rel, mx)


def test_repeat_calls_are_deterministic():
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=300, H=2, Hq=2, n_tail=1, seed=0x5EED8000)
    q = synth.queries(3, 0, 1, 0, 1, 2)
    a = bt.cache.decode(0, 1, q).clone()
    b = bt.cache.decode(0, 1, q)
    assert torch.equal(a, b)


# ------------------------------------------------------------ host-side errors
def test_state_and_capacity_errors():
    cfg = rq.make_config(num_layers=1, num_loops=4, loops_per_group=4, batch=1, max_tokens=8, max_tail_tokens=4,
                         num_kv_heads=1, num_q_heads=1)
    c = rq.Cache(cfg)
    k = torch.zeros((1, 2, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.RQError) as e:
        c.append(0, 3, k, k)                  # anchor before its loops
    assert e.value.status == rq.RQ_ERR_STATE
    c.append(0, 0, k, k)
    c.append(0, 1, k, k)
    with pytest.raises(rq.RQError) as e:
        c.append(0, 3, k, k)                  # loop 2 still missing
    assert e.value.status == rq.RQ_ERR_STATE
    c.append(0, 2, k, k)
    c.append(0, 3, k, k)
    assert c.length(0, 0) == 2 and c.tail_length(0, 0) == 0
    big = torch.zeros((1, 5, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.RQError) as e:
        c.append(0, 0, big, big)              # tail capacity 4
    assert e.value.status == rq.RQ_ERR_CAPACITY
    for _ in range(3):
        for loop in range(4):
            c.append(0, loop, k, k)
    with pytest.raises(rq.RQError) as e:
        for loop in range(4):
            c.append(0, loop, k, k)           # 10 > max_tokens 8
    assert e.value.status == rq.RQ_ERR_CAPACITY
    with pytest.raises(rq.RQError) as e:
        c.truncate(0, 0, 1)                   # tails not empty
    assert e.value.status == rq.RQ_ERR_STATE
    q = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rq.RQError) as e:
        c.decode(0, 0, q, bf16=True)          # wrong format
    assert e.value.status == rq.RQ_ERR_STATE
    assert rq.rq_decode_attn(c.h, 1, 0, q, q) == rq.RQ_ERR_INVALID
    c.check()


def test_truncate_rolls_back():
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=128, H=1, Hq=1, seed=0x5EED9000)
    q = synth.queries(9, 0, 0, 0, 1, 1)
    full = bt.cache.decode(0, 3, q).clone()
    bt.cache.truncate(0, 0, 100)
    assert bt.cache.length(0, 0) == 100
    part = bt.cache.decode(0, 3, q)
    assert not torch.equal(full, part)
    bt.T = 100
    ref = H.oracle_decode(bt, 0, 3, q)
    rel, mx = H.attn_errors(part.cpu().numpy(), ref, 1)
    assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL


def test_library_allocated_arena():
    cfg = rq.make_config(num_layers=1, num_loops=4, loops_per_group=4, batch=1, max_tokens=64, max_tail_tokens=4,
                         num_kv_heads=2, num_q_heads=2)
    c = rq.Cache(cfg, library_alloc=True)
    assert c.arena is None
    c.close()
