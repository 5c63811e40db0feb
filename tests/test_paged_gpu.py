"""Paged caches on the GPU: records in a pool of blocks reached through a
per-sequence block table (the layout of a serving engine's paged KV cache;
the ai4snews summary, paragraph 4, runs the method inside vLLM).

Through the C ABI, against the fp64 oracle and against contiguous caches:
  * a paged cache with a shuffled free list (every sequence's blocks
    scattered over the pool) holds records bit-identical to the oracle's and
    to a contiguous cache fed the same inputs, and decodes to the same
    outputs, bit for bit (same splits; the ring items follow the block
    grid, which changes no summation order), with ragged per-sequence
    lengths;
  * forking a sequence shares its blocks; the first append into a shared
    block copies it (copy-on-write), leaving the other sequence's records
    untouched;
  * an exhausted pool refuses an append without changing anything, and
    truncation returns blocks to it;
  * the Ouro-1.4B-shaped workload (batch 4, T = 8192, 16 heads) in 128-token
    blocks, on sampled (sequence, head) units.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _shuffled(seed):
    return lambda cache: cache.shuffle_free_blocks(seed)


def _check(bt, sel=None, loops=range(4)):
    cfg = bt.cfg
    for kv in (0, 1):
        r = H.compare_records(bt, 0, 0, kv, sel)
        assert r["mismatch"] == 0 and r["tolerated"] == 0, (kv, r)
    outs = {}
    for loop in loops:
        q = synth.queries(bt.seed, 0, loop, 0, cfg.batch, cfg.num_q_heads)
        out = bt.cache.decode(0, loop, q, out=H.guarded_out((cfg.batch, cfg.num_q_heads, 128)))
        ref = H.oracle_decode(bt, 0, loop, q, sel)
        rel, mx = H.attn_errors(out.cpu().numpy(), ref, cfg.num_q_heads // cfg.num_kv_heads)
        assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
        outs[loop] = out
    bt.cache.check()
    return outs


@pytest.mark.parametrize("bt_tokens", [128, 256])
def test_paged_equals_contiguous_and_oracle(bt_tokens):
    kw = dict(layers=1, loops=4, Lg=4, B=3, T=700, H=2, Hq=4, n_tail=1, chunk=100, seed=0x5EEDC000 + bt_tokens)
    paged = H.build(block_tokens=bt_tokens, num_blocks=40, prepare=_shuffled(5), **kw)
    flat = H.build(**kw)
    blocks = paged.cache.seq_blocks(0)
    assert len(blocks) == (700 + bt_tokens - 1) // bt_tokens
    assert any(b2 != b1 + 1 for b1, b2 in zip(blocks, blocks[1:]))    # scattered over the pool
    out_p = _check(paged)
    for loop in range(4):
        a = paged.cache.export(0, loop)
        b = flat.cache.export(0, loop)
        for x, y in zip(a, b):
            assert (x is None and y is None) or np.array_equal(x, y)
        q = synth.queries(paged.seed, 0, loop, 0, 3, 4)
        assert torch.equal(out_p[loop], flat.cache.decode(0, loop, q))
    paged.cache.close()
    flat.cache.close()


def test_paged_ragged_and_truncation_returns_blocks():
    bt = H.build(layers=1, loops=4, Lg=4, B=3, T=600, H=2, Hq=2, n_tail=0, chunk=128, seed=0x5EEDC100,
                 max_tokens=640, block_tokens=128, num_blocks=20, prepare=_shuffled(6))
    c = bt.cache
    free0 = c.free_blocks()
    assert free0 == 20 - 3 * 5
    c.truncate_seq(0, 0, 1, 130)        # sequence 1 keeps 2 blocks
    c.truncate_seq(0, 0, 2, 0)          # sequence 2 keeps none
    assert c.free_blocks() == free0 + 3 + 5
    assert len(c.seq_blocks(1)) == 2 and c.seq_blocks(2) == []
    # decode attends to each sequence's own tokens
    cfg = bt.cfg
    for loop in range(4):
        q = synth.queries(bt.seed, 0, loop, 0, 3, 2)
        out = c.decode(0, loop, q).cpu().numpy()
        for b, Tb in ((0, 600), (1, 130)):
            bt.T = Tb
            bt.recon.clear()
            ref = H.oracle_decode(bt, 0, loop, q, [(b, h) for h in range(2)])
            rel, mx = H.attn_errors(out, ref, 1)
            assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, b, rel, mx)
        assert (out[2] == 0).all()
    # appends continue after each sequence's own last token, taking blocks again
    K, V = synth.group_kv(77, 0, 0, 4, (0.1, 0.2, 0.3), 3, 5, 2, device="cuda")
    for j in range(4):
        c.append(0, j, K[j], V[j])
    assert [c.length_seq(0, 0, b) for b in range(3)] == [605, 135, 5]
    assert len(c.seq_blocks(2)) == 1
    c.check()
    c.close()


def test_fork_shares_blocks_and_copies_on_write():
    """Sequence 1 is forked from sequence 0 at T = 300 (a partly filled third
    block); both then append 40 tokens of their own.  Records at positions
    below 300 are those of sequence 0's inputs for both, later ones their
    own; the shared partial block was copied once."""
    T0, n1, Hh = 300, 40, 2
    cfg = rq.make_config(num_layers=1, num_loops=4, loops_per_group=4, batch=2, max_tokens=T0 + n1,
                         max_tail_tokens=128, num_kv_heads=Hh, num_q_heads=Hh, block_tokens=128, num_blocks=12)
    c = rq.Cache(cfg)
    c.shuffle_free_blocks(9)
    K, V = synth.group_kv(0x5EEDC200, 0, 0, 4, (0.1, 0.2, 0.3), 2, T0 + n1, Hh, device="cuda")
    # sequence 1 starts as a copy of sequence 0
    K = [torch.cat([k[:1], torch.cat([k[:1, :T0], k[1:, T0:]], 1)]) for k in K]
    V = [torch.cat([v[:1], torch.cat([v[:1, :T0], v[1:, T0:]], 1)]) for v in V]
    bt = H.Built(c, cfg, 0x5EEDC200, T0 + n1, 0)
    bt.inputs[(0, 0)] = (K, V)
    for t0 in range(0, T0, 100):
        for j in range(4):
            c.append(0, j, K[j][:, t0:t0 + 100].contiguous(), V[j][:, t0:t0 + 100].contiguous())
    c.truncate_seq(0, 0, 1, 0)            # sequence 1 empty, its blocks back in the pool
    free_before = c.free_blocks()
    c.fork_seq(0, 1)
    assert c.seq_blocks(1) == c.seq_blocks(0) and c.free_blocks() == free_before
    assert c.length_seq(0, 0, 1) == T0
    for j in range(4):
        c.append(0, j, K[j][:, T0:].contiguous(), V[j][:, T0:].contiguous())
    b0, b1 = c.seq_blocks(0), c.seq_blocks(1)
    assert b0[:2] == b1[:2] and b0[2] != b1[2]      # full blocks shared, the written one copied
    assert c.free_blocks() == free_before - 1
    _check(bt)
    c.close()


def test_pool_exhaustion_refuses_and_changes_nothing():
    cfg = rq.make_config(num_layers=1, num_loops=4, loops_per_group=4, batch=2, max_tokens=1024,
                         max_tail_tokens=256, num_kv_heads=1, num_q_heads=1, block_tokens=128, num_blocks=3)
    c = rq.Cache(cfg)
    K, V = synth.group_kv(1, 0, 0, 4, (0.1, 0.2, 0.3), 2, 200, 1, device="cuda")
    for j in range(3):
        c.append(0, j, K[j], V[j])
    with pytest.raises(rq.RQError) as e:
        c.append(0, 3, K[3], V[3])          # 2 sequences x 2 blocks > 3
    assert e.value.status == rq.RQ_ERR_CAPACITY
    assert c.length(0, 0) == 0 and c.free_blocks() == 3 and c.tail_length(0, 0) == 200
    c.close()


def test_paged_chained_reference():
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=400, H=2, Hq=4, n_tail=1, chunk=200, seed=0x5EEDC300,
                 block_tokens=128, num_blocks=16, prepare=_shuffled(11), anchor_mode=rq.ANCHOR_CHAINED)
    _check(bt)
    bt.cache.close()


def test_paged_ouro_8k_batch4_sampled():
    bt = H.build(layers=1, loops=4, Lg=4, B=4, T=8192, H=16, Hq=16, n_tail=1, chunk=1024, seed=0x5EED0001,
                 block_tokens=128, num_blocks=4 * 64 + 8, prepare=_shuffled(12))
    _check(bt, sel=[(0, 3), (3, 12)])
    bt.cache.close()


@pytest.mark.parametrize("bt_tokens", [128, 256])
def test_paged_prefill_equals_contiguous(bt_tokens):
    """rq_prefill_attn on a paged cache (blocks scattered over the pool) gives
    the contiguous cache's outputs bit for bit, with the new tokens in a
    residual loop's tail and committed at the anchor loop: the same records,
    splits and steps (a 32-token step lies inside one block)."""
    B, Hkv, Hq, T, n = 3, 2, 4, 700, 24
    kw = dict(layers=1, loops=4, Lg=4, B=B, T=T, H=Hkv, Hq=Hq, n_tail=0, chunk=100,
              seed=0x5EEDC400 + bt_tokens, max_tokens=T + n)
    paged = H.build(block_tokens=bt_tokens, num_blocks=40, prepare=_shuffled(9), **kw)
    flat = H.build(**kw)
    blocks = paged.cache.seq_blocks(1)
    assert any(b2 != b1 + 1 for b1, b2 in zip(blocks, blocks[1:]))    # scattered over the pool
    g = torch.Generator(device="cuda").manual_seed(bt_tokens)
    K = torch.randn((4, B, n, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((4, B, n, Hkv, 128), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((B, n, Hq, 128), generator=g, device="cuda").to(torch.bfloat16)
    for bt in (paged, flat):
        bt.cache.append(0, 0, K[0], V[0])
    outs = [bt.cache.prefill(0, 0, q) for bt in (paged, flat)]
    assert torch.equal(outs[0], outs[1])
    for bt in (paged, flat):
        for j in range(1, 4):
            bt.cache.append(0, j, K[j], V[j])
    outs = [bt.cache.prefill(0, 3, q) for bt in (paged, flat)]
    assert torch.equal(outs[0], outs[1])
    paged.cache.check()
    flat.cache.check()
