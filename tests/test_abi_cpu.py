"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every entry point include/rq.h declares, validates configurations, and its
byte accounting reproduces the 80.7% storage reduction of the ResidualQuant
abstract / ai4snews summary (paragraph 2)."""
import json
import os
import re

import pytest
import torch

import decode_attention_14_b200 as rq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "rq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t)\s*(rq_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(rq.lib, n), n


def _cfg(**kw):
    base = dict(num_layers=24, num_loops=4, loops_per_group=4, batch=4, max_tokens=8192, max_tail_tokens=4,
                num_kv_heads=16, num_q_heads=16)
    base.update(kw)
    return rq.make_config(**base)


def test_config_validation():
    assert rq.rq_config_check(_cfg()) == rq.RQ_OK
    assert rq.rq_config_check(_cfg(head_dim=64)) == rq.RQ_ERR_UNSUPPORTED
    assert rq.rq_config_check(_cfg(group_size=8)) == rq.RQ_ERR_UNSUPPORTED
    assert rq.rq_config_check(_cfg(anchor_bits=3)) == rq.RQ_ERR_UNSUPPORTED
    assert rq.rq_config_check(_cfg(num_loops=6)) == rq.RQ_ERR_INVALID
    assert rq.rq_config_check(_cfg(num_q_heads=24)) == rq.RQ_ERR_INVALID
    assert rq.rq_config_check(_cfg(num_q_heads=48)) == rq.RQ_ERR_UNSUPPORTED   # 3 q heads per kv head
    assert rq.rq_config_check(_cfg(batch=0)) == rq.RQ_ERR_INVALID
    assert rq.rq_config_check(_cfg(max_tail_tokens=0)) == rq.RQ_ERR_INVALID
    assert rq.rq_config_check(_cfg(loops_per_group=1, max_tail_tokens=0)) == rq.RQ_OK
    assert rq.rq_config_check(_cfg(format=rq.RQ_FMT_BF16, group_size=0)) == rq.RQ_OK
    assert rq.rq_cache_required_bytes(_cfg(head_dim=64)) == 0
    # at most 256 split partials of at most 1024 tokens per (sequence, head)
    assert rq.rq_config_check(_cfg(batch=1, max_tokens=262144)) == rq.RQ_OK
    assert rq.rq_config_check(_cfg(batch=1, max_tokens=262145)) == rq.RQ_ERR_UNSUPPORTED
    # sequences' lengths travel in the launch arguments: at most 256 per cache
    assert rq.rq_config_check(_cfg(batch=256, max_tokens=64)) == rq.RQ_OK
    assert rq.rq_config_check(_cfg(batch=257, max_tokens=64)) == rq.RQ_ERR_UNSUPPORTED


def test_token_bytes_reproduce_storage_reduction():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "storage_fraction.json")))
    bf16 = rq.rq_cache_token_bytes(_cfg(format=rq.RQ_FMT_BF16))
    assert bf16 == 24 * 4 * 16 * 2 * 128 * 2
    g32 = rq.rq_cache_token_bytes(_cfg(group_size=32))
    g16 = rq.rq_cache_token_bytes(_cfg(group_size=16))
    assert g32 / bf16 == 0.193359375
    assert g16 / bf16 == 0.224609375
    assert round(100 * (1 - g32 / bf16), g["printed_decimals"]) == g["reduction_percent"]
    # uniform INT2 (anchor at 2 bits too) and the deep-recurrence grouping
    u = rq.rq_cache_token_bytes(_cfg(anchor_bits=2))
    assert u / bf16 == (48 + 3 * 50) / (4 * 256)
    deep = rq.make_config(num_layers=4, num_loops=32, loops_per_group=4, batch=8, max_tokens=4096,
                          max_tail_tokens=1, num_kv_heads=40, num_q_heads=40)
    assert rq.rq_cache_token_bytes(deep) == 4 * 40 * 2 * 8 * (80 + 3 * 50)


def test_required_bytes_cover_records():
    c = _cfg()
    need = rq.rq_cache_required_bytes(c)
    per_seq = rq.rq_cache_token_bytes(c) * 8192      # token bytes are per sequence
    assert need >= per_seq * c.batch
    assert need % 256 == 0
    assert need < per_seq * c.batch * 1.05


def test_status_strings():
    for s in range(-7, 1):
        assert rq.rq_status_string(s) and rq.rq_status_string(s) != "unknown status"
    assert rq.rq_status_string(-99) == "unknown status"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_create_without_device_reports_cuda_error():
    h = rq.ctypes.c_void_p()
    st = rq.lib.rq_cache_create(rq.ctypes.byref(_cfg(num_layers=1, max_tokens=64)), None, 0, rq.ctypes.byref(h))
    assert st in (rq.RQ_ERR_CUDA, rq.RQ_ERR_NOMEM)
    assert not h.value


def test_null_arguments_rejected_without_device():
    assert rq.lib.rq_append(None, 0, 0, None, None, 1, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_decode_attn(None, 0, 0, None, None, 0.0, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_decode_attn_bf16(None, 0, 0, None, None, 0.0, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_prefill_attn(None, 0, 0, None, 4, None, 0.0, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_append_decode_attn(None, 0, 0, None, None, 1, None, None, 0.0, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_decode_attn_noalloc(None, 0, 0, None, None, 0.0, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_cache_truncate_seq(None, 0, 0, 0, 0) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_cache_export(None, 0, 0, None, None, None, None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_cache_truncate(None, 0, 0, 0) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_check(None) == rq.RQ_ERR_INVALID
    assert rq.lib.rq_cache_destroy(None) == rq.RQ_OK
    assert rq.lib.rq_decode_bytes(None, 0, 0) == 0
