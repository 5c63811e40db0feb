"""rq_decode_attn_noalloc: decode attention that allocates nothing.

Some callers may not allocate device memory once they are running -- a plugin
inside a host framework that owns every device byte and offers no allocator,
a serving loop whose memory is planned at start-up, or work issued while a
stream is being captured.  For them the library keeps the split-combine
scratch of this entry point in a fixed device array of its own (8 MiB per
GPU).  This file checks, through the C ABI, that it returns what
rq_decode_attn (and the fp64 oracle) return (within the parity tolerance) on
two calls in a row, that a call captured into a CUDA graph after a first
eager call replays correctly, and that it refuses, without enqueuing work, a
call whose scratch would not fit.  It is named to run last so that a failure here cannot hide the other
tests' results.
"""
import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

import rqharness as H

pytestmark = pytest.mark.gpu


def _errors(a: torch.Tensor, b: torch.Tensor):
    a64 = a.double().cpu().numpy()
    b64 = b.double().cpu().numpy()
    rel = float(np.linalg.norm(a64 - b64) / max(np.linalg.norm(b64), 1e-300))
    return rel, float(np.abs(a64 - b64).max())


def test_noalloc_matches_rq_decode_attn_twice():
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=700, H=4, Hq=8, n_tail=2, seed=0x5EEDA000)
    cfg = bt.cfg
    for loop in (0, 2, 3):          # residual loops with BF16 tail tokens, and the anchor loop
        q = synth.queries(bt.seed, 0, loop, 0, cfg.batch, cfg.num_q_heads)
        ref = bt.cache.decode(0, loop, q)
        orc_ref = H.oracle_decode(bt, 0, loop, q)
        for _ in range(2):
            out = torch.full_like(ref, float("nan"))
            st = rq.rq_decode_attn_noalloc(bt.cache.h, 0, loop, q, out)
            assert st == rq.RQ_OK, rq.rq_status_string(st)
            torch.cuda.synchronize()
            rel, mx = _errors(out, ref)
            assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
            # and against the fp64 oracle over the same records
            rel, mx = H.attn_errors(out.cpu().numpy(), orc_ref, cfg.num_q_heads // cfg.num_kv_heads)
            assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (loop, rel, mx)
    bt.cache.check()


def test_noalloc_inside_stream_capture():
    """After one eager call (which looks up the scratch address), a call
    captured into a CUDA graph on a side stream allocates nothing and replays
    with the same results, twice."""
    bt = H.build(layers=1, loops=4, Lg=4, B=2, T=500, H=2, Hq=4, n_tail=1, seed=0x5EEDA100)
    cfg = bt.cfg
    loop = 1
    q = synth.queries(bt.seed, 0, loop, 0, cfg.batch, cfg.num_q_heads)
    ref = bt.cache.decode(0, loop, q)
    out = torch.zeros_like(ref)
    assert rq.rq_decode_attn_noalloc(bt.cache.h, 0, loop, q, out) == rq.RQ_OK
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            st = rq.rq_decode_attn_noalloc(bt.cache.h, 0, loop, q, out, 0.0, side)
    assert st == rq.RQ_OK, rq.rq_status_string(st)
    for _ in range(2):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        rel, mx = _errors(out, ref)
        assert rel <= H.REL_L2_TOL and mx <= H.MAX_ABS_TOL, (rel, mx)
    del g
    bt.cache.check()


def test_noalloc_rejects_scratch_beyond_its_limit():
    # 128 sequences x 128 query heads x 1 split x 132 floats > 2^21 floats
    cfg = rq.make_config(num_layers=1, num_loops=1, loops_per_group=1, batch=128, max_tokens=64,
                         max_tail_tokens=0, num_kv_heads=128, num_q_heads=128)
    c = rq.Cache(cfg)
    k = torch.randn((128, 1, 128, 128), device="cuda").to(torch.bfloat16)
    c.append(0, 0, k, k)
    q = torch.randn((128, 128, 128), device="cuda").to(torch.bfloat16)
    out = torch.zeros((128, 128, 128), dtype=torch.float32, device="cuda")
    assert rq.rq_decode_attn_noalloc(c.h, 0, 0, q, out) == rq.RQ_ERR_CAPACITY
    torch.cuda.synchronize()
    assert (out == 0).all()                      # nothing was enqueued
    c.decode(0, 0, q, out)                       # the allocating path still serves it
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    c.check()
    c.close()


def test_noalloc_wrong_format_and_arguments():
    cfg = rq.make_config(num_layers=1, num_loops=1, loops_per_group=1, batch=1, max_tokens=64,
                         max_tail_tokens=0, num_kv_heads=1, num_q_heads=1, format=rq.RQ_FMT_BF16)
    c = rq.Cache(cfg)
    q = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    assert rq.rq_decode_attn_noalloc(c.h, 0, 0, q, out) == rq.RQ_ERR_STATE
    assert rq.rq_decode_attn_noalloc(c.h, 1, 0, q, out) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_decode_attn_noalloc(None, 0, 0, None, None, 0.0, None) == rq.RQ_ERR_INVALID
    c.close()
