"""Failure detection on the GPU without a GPU fault: a bounded wait that runs
out is reported, and the library recovers.

Every mbarrier wait of the decode kernel gives up after a limit (1 s in the
shipped library), sets the cache's error word, and lets the CTA finish
without touching further data; rq_check then returns RQ_ERR_TIMEOUT and
clears the error word and the split-combine counters.  This test builds a
test-only variant of the library (in a temporary directory) with a 0.2 s
limit and a hook that makes the next decode launch leave one ring item's
mbarrier unarmed -- no copy is issued for it, so nothing ever completes
that phase -- and checks, through the C ABI:
  * the call itself is enqueued (RQ_OK) and returns; nothing hangs;
  * rq_check reports RQ_ERR_TIMEOUT once, then RQ_OK;
  * the next call's output equals the output before the fault, bit for bit
    (the counters and the error word were cleaned up).
The injected failure is a wait that runs out; nothing traps or faults.
"""
import ctypes
import importlib.util
import os

import numpy as np
import pytest
import torch

import decode_attention_14_b200 as rq
import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fault_lib(tmp_path_factory):
    d = tmp_path_factory.mktemp("rq_fault_build")
    spec = importlib.util.spec_from_file_location("_rq_fault_build", os.path.join(ROOT, "decode_attention_14_b200",
                                                                                 "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.OBJ = str(d / "obj")
    b.LIB = str(d / "librq_fault.so")
    b.build(force=True, extra=["-DRQ_WAIT_NS=200000000ull", "-DRQ_FAULT_INJECT=1"])
    L = ctypes.CDLL(b.LIB)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    L.rq_cache_create.restype = i32
    L.rq_cache_create.argtypes = [ctypes.POINTER(rq.rq_config), vp, ctypes.c_size_t, ctypes.POINTER(vp)]
    L.rq_cache_destroy.argtypes = [vp]
    L.rq_append.restype = i32
    L.rq_append.argtypes = [vp, i32, i32, vp, vp, i32, vp]
    L.rq_decode_attn.restype = i32
    L.rq_decode_attn.argtypes = [vp, i32, i32, vp, vp, ctypes.c_float, vp]
    L.rq_check.restype = i32
    L.rq_check.argtypes = [vp]
    L.rq_test_arm_fault.restype = i32
    return L


def test_bounded_wait_runs_out_and_the_library_recovers(fault_lib):
    L = fault_lib
    B, T, Hkv = 1, 1000, 2
    cfg = rq.make_config(num_layers=1, num_loops=4, loops_per_group=4, batch=B, max_tokens=T, max_tail_tokens=256,
                         num_kv_heads=Hkv, num_q_heads=Hkv)
    h = ctypes.c_void_p()
    assert L.rq_cache_create(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == rq.RQ_OK
    K, V = synth.group_kv(0x5EEDD000, 0, 0, 4, (0.1, 0.2, 0.3), B, T, Hkv, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    for t0 in range(0, T, 250):
        for j in range(4):
            k = K[j][:, t0:t0 + 250].contiguous()
            v = V[j][:, t0:t0 + 250].contiguous()
            assert L.rq_append(h, 0, j, k.data_ptr(), v.data_ptr(), 250, st) == rq.RQ_OK
    q = synth.queries(1, 0, 1, 0, B, Hkv)
    ref = torch.empty((B, Hkv, 128), dtype=torch.float32, device="cuda")
    out = torch.empty_like(ref)
    assert L.rq_decode_attn(h, 0, 1, q.data_ptr(), ref.data_ptr(), 0.0, st) == rq.RQ_OK
    assert L.rq_check(h) == rq.RQ_OK

    assert L.rq_test_arm_fault() == 0
    assert L.rq_decode_attn(h, 0, 1, q.data_ptr(), out.data_ptr(), 0.0, st) == rq.RQ_OK
    assert L.rq_check(h) == rq.RQ_ERR_TIMEOUT          # the wait ran out and was reported
    assert L.rq_check(h) == rq.RQ_OK                   # ... once

    out.fill_(float("nan"))
    assert L.rq_decode_attn(h, 0, 1, q.data_ptr(), out.data_ptr(), 0.0, st) == rq.RQ_OK
    assert L.rq_check(h) == rq.RQ_OK
    assert torch.equal(out, ref)
    L.rq_cache_destroy(h)
