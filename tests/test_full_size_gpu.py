"""Parity at the full sizes of the benchmarked workloads, in the launch
configuration the bench uses (the library picks the same split-KV partition
for the same shape), on sampled (sequence, kv head) units that the fp64
oracle can compute one by one:

  * Ouro-1.4B-shaped decode: 4 loops (loop 4 INT4 anchor), H = 16, d = 128,
    T = 8192, batch 4;
  * long context: T = 16384 at batch 2 and batch 4;
  * deep recurrence: 32 loops in 8 groups of 4, H = 40, T = 4096, batch 8
    (two of the eight groups are filled and checked);
  * format variants of the batch sweep (group 32, rotation off, uniform INT2)
    at T = 8192.

One layer is filled: every layer of the benchmark issues the same call.
Each check: records bit-exact (oracle-flagged boundary values excepted),
attention within relative L2 1e-3 / max abs 2e-3 against the oracle fed the
GPU's own records, for every loop.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _check(bt, groups, sel, loops_to_check=None):
    cfg = bt.cfg
    Lg = cfg.loops_per_group
    for grp in groups:
        for kv in (0, 1):
            r = H.compare_records(bt, 0, grp, kv, sel)
            assert r["mismatch"] == 0, r
            assert r["tolerated"] == 0, r   # none on the synthetic workloads (reported when nonzero)
        loops = loops_to_check if loops_to_check is not None else range(grp * Lg, grp * Lg + Lg)
        for loop in loops:
            q = synth.queries(bt.seed, 0, loop, 0, cfg.batch, cfg.num_q_heads)
            out = bt.cache.decode(0, loop, q, out=H.guarded_out((cfg.batch, cfg.num_q_heads, 128))).cpu().numpy()
            ref = H.oracle_decode(bt, 0, loop, q, sel)
            rel, mx = H.attn_errors(out, ref, cfg.num_q_heads // cfg.num_kv_heads)
            assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
    bt.cache.check()


def test_ouro_8k_batch4():
    bt = H.build(layers=1, loops=4, Lg=4, B=4, T=8192, H=16, Hq=16, n_tail=1, chunk=512, seed=0x5EED0001)
    _check(bt, [0], [(0, 3), (3, 12)])
    bt.cache.close()


@pytest.mark.parametrize("B", [2, 4])
def test_long_16k(B):
    bt = H.build(layers=1, loops=4, Lg=4, B=B, T=16384, H=16, Hq=16, n_tail=1, chunk=1024, seed=0x5EED0002)
    _check(bt, [0], [(B - 1, 7)])
    bt.cache.close()


def test_deep_recurrence_full_shape():
    bt = H.build(layers=1, loops=32, Lg=4, B=8, T=4096, H=40, Hq=40, n_tail=1, chunk=1024,
                 sigma=(0.1, 0.25, 0.4), seed=0x5EED0003, only_groups=[0, 7])
    _check(bt, [0, 7], [(5, 39)])
    bt.cache.close()


@pytest.mark.parametrize("g,ba,br,rotate", [(32, 4, 2, True), (16, 4, 2, False), (16, 2, 2, True)])
def test_sweep_format_variants_8k(g, ba, br, rotate):
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=8192, H=16, Hq=16, g=g, ba=ba, br=br, rotate=rotate, n_tail=1,
                 chunk=1024, seed=0x5EED0004 + g + ba)
    _check(bt, [0], [(1, 9)])
    bt.cache.close()
