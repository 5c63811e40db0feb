"""GPU parity of the encoder's ablation modes and of per-layer rotations.

The arXiv abstract compares reference choices (the last loop as a shared
anchor vs the previous loop, chained) and scaling methods (least squares vs
norm ratio vs none); the ai4snews summary (paragraph 5) has the rotations
calibrated once and then fixed, which for a real model means one per layer.
Each case fills caches through the C ABI and compares with the fp64 oracle
(orc_encode_modes, the same chain written out step by step):
  * every code, FP8 scale/min and BF16 coefficient bit for bit (strict --
    no tolerated difference -- where the rotation is off, since then both
    sides round the very same fp64 values);
  * attention for the loops the decode kernels serve: every loop under the
    shared reference; the first loop (anchor record and its tail) and
    every later loop (anchor plus the chain of residual records) under the
    chained one.
"""
import numpy as np
import pytest

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _check(bt, strict, loops, layer=0):
    cfg = bt.cfg
    for kv in (0, 1):
        r = H.compare_records(bt, layer, 0, kv)
        assert r["mismatch"] == 0, (kv, r)
        assert r["compared"] > 0
        if strict:
            assert r["tolerated"] == 0, (kv, r)
        g, o = H.mse_check(bt, layer, 0, kv)
        assert abs(g / o - 1.0) <= H.MSE_REL_TOL, (kv, g, o)
    for loop in loops:
        q = synth.queries(bt.seed, layer, loop, 0, cfg.batch, cfg.num_q_heads)
        out = bt.cache.decode(layer, loop, q, out=H.guarded_out((cfg.batch, cfg.num_q_heads, 128))).cpu().numpy()
        ref = H.oracle_decode(bt, layer, loop, q)
        rel, mx = H.attn_errors(out, ref, cfg.num_q_heads // cfg.num_kv_heads)
        assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
    bt.cache.check()


@pytest.mark.parametrize("scale_mode", [rq.SCALE_NORM_RATIO, rq.SCALE_NONE])
@pytest.mark.parametrize("rotate", [True, False])
def test_scaling_modes_shared_anchor(scale_mode, rotate):
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=200, H=2, Hq=4, n_tail=1, rotate=rotate, seed=0x5EEDB000 + scale_mode,
                 scale_mode=scale_mode)
    _check(bt, strict=not rotate, loops=range(4))
    bt.cache.close()


def test_per_layer_rotations():
    """Two layers with the same inputs: each layer's records follow its own
    rotation (seed + layer * 2^32), so their residual codes differ."""
    bt = H.build(layers=2, loops=4, Lg=4, B=1, T=150, H=2, Hq=2, n_tail=1, seed=0x5EEDB100, rotation_per_layer=True)
    for layer in range(2):
        _check(bt, strict=False, loops=range(4), layer=layer)
    # the same K/V in both layers would give different residual codes
    K, V = bt.inputs[(0, 0)]
    bt2 = H.build(layers=2, loops=4, Lg=4, B=1, T=64, H=1, Hq=1, seed=0x5EEDB101, rotation_per_layer=True,
                  only_layers=[0])
    H.fill_group(bt2, 1, 0, [k[:, :64, :1].contiguous() for k in bt2.inputs[(0, 0)][0]],
                 [v[:, :64, :1].contiguous() for v in bt2.inputs[(0, 0)][1]], chunk=64)
    c0, _, _ = bt2.cache.export(0, 0)
    c1, _, _ = bt2.cache.export(1, 0)
    assert not np.array_equal(c0, c1)
    bt.cache.close()
    bt2.cache.close()


@pytest.mark.parametrize("scale_mode", [rq.SCALE_LEAST_SQUARES, rq.SCALE_NORM_RATIO, rq.SCALE_NONE])
@pytest.mark.parametrize("rotate", [True, False])
def test_chained_reference_records(scale_mode, rotate):
    """Previous-loop (chained) reference: loop 0 in the anchor record, loop
    l >= 1 a residual against the reconstruction of loop l - 1."""
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=170, H=2, Hq=4, n_tail=1, rotate=rotate,
                 seed=0x5EEDB200 + scale_mode, anchor_mode=rq.ANCHOR_CHAINED, scale_mode=scale_mode)
    _check(bt, strict=not rotate, loops=range(4))
    # records read per decode call grow along the chain: anchor, then 1, 2, 3 residuals
    per = [bt.cache.decode_bytes(0, loop) for loop in range(4)]
    assert per[0] < per[1] < per[2] < per[3]
    bt.cache.close()


@pytest.mark.parametrize("T,Hq", [(1000, 2), (3000, 8)])
def test_chained_reference_longer(T, Hq):
    """Longer caches (several splits, a ragged last tile) and GQA 4."""
    bt = H.build(layers=1, loops=4, Lg=4, B=1, T=T, H=2, Hq=Hq, n_tail=2, chunk=256, seed=0x5EEDB300 + T,
                 anchor_mode=rq.ANCHOR_CHAINED)
    _check(bt, strict=False, loops=range(4))
    bt.cache.close()
