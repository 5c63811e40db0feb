"""Python binding of the ResidualQuant decode-attention library (``librq.so``,
C ABI in include/rq.h).

Argument marshalling only: every step of the method runs in the library's
CUDA kernels.  Device buffers are torch tensors (PyTorch supplies device
memory and streams); the binding passes their raw pointers.  There is no
CPU or PyTorch fallback: if ``librq.so`` is missing or fails to load, import
fails.

The function names mirror the C ABI: ``rq_cache_create``, ``rq_append``,
``rq_decode_attn``, ``rq_decode_attn_bf16``, ... ; :class:`Cache` wraps
them for convenience.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librq.so")

RQ_OK = 0
RQ_ERR_INVALID = -1
RQ_ERR_UNSUPPORTED = -2
RQ_ERR_NOMEM = -3
RQ_ERR_CAPACITY = -4
RQ_ERR_STATE = -5
RQ_ERR_CUDA = -6
RQ_ERR_TIMEOUT = -7

RQ_FMT_RESIDUAL = 0
RQ_FMT_BF16 = 1

HEAD_DIM = 128


class rq_config(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int32),
        ("num_loops", ctypes.c_int32),
        ("loops_per_group", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("max_tokens", ctypes.c_int32),
        ("max_tail_tokens", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("group_size", ctypes.c_int32),
        ("anchor_bits", ctypes.c_int32),
        ("resid_bits", ctypes.c_int32),
        ("rotate", ctypes.c_int32),
        ("format", ctypes.c_int32),
        ("seed", ctypes.c_uint64),
        ("scale_mode", ctypes.c_int32),
        ("anchor_mode", ctypes.c_int32),
        ("rotation_per_layer", ctypes.c_int32),
        ("block_tokens", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m decode_attention_14_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, cfgp = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(rq_config)
    L.rq_status_string.restype = ctypes.c_char_p
    L.rq_status_string.argtypes = [i32]
    L.rq_config_check.restype = i32
    L.rq_config_check.argtypes = [cfgp]
    L.rq_cache_required_bytes.restype = ctypes.c_size_t
    L.rq_cache_required_bytes.argtypes = [cfgp]
    L.rq_cache_token_bytes.restype = ctypes.c_size_t
    L.rq_cache_token_bytes.argtypes = [cfgp]
    L.rq_cache_create.restype = i32
    L.rq_cache_create.argtypes = [cfgp, vp, ctypes.c_size_t, ctypes.POINTER(vp)]
    L.rq_cache_destroy.restype = i32
    L.rq_cache_destroy.argtypes = [vp]
    L.rq_append.restype = i32
    L.rq_append.argtypes = [vp, i32, i32, vp, vp, i32, vp]
    L.rq_decode_attn.restype = i32
    L.rq_decode_attn.argtypes = [vp, i32, i32, vp, vp, ctypes.c_float, vp]
    L.rq_append_decode_attn.restype = i32
    L.rq_append_decode_attn.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, ctypes.c_float, vp]
    L.rq_decode_attn_bf16.restype = i32
    L.rq_decode_attn_bf16.argtypes = [vp, i32, i32, vp, vp, ctypes.c_float, vp]
    L.rq_prefill_attn.restype = i32
    L.rq_prefill_attn.argtypes = [vp, i32, i32, vp, i32, vp, ctypes.c_float, vp]
    L.rq_decode_attn_noalloc.restype = i32
    L.rq_decode_attn_noalloc.argtypes = [vp, i32, i32, vp, vp, ctypes.c_float, vp]
    L.rq_cache_length.restype = i32
    L.rq_cache_length.argtypes = [vp, i32, i32, ctypes.POINTER(i32)]
    L.rq_cache_tail_length.restype = i32
    L.rq_cache_tail_length.argtypes = [vp, i32, i32, ctypes.POINTER(i32)]
    L.rq_cache_truncate.restype = i32
    L.rq_cache_truncate.argtypes = [vp, i32, i32, i32]
    L.rq_cache_truncate_seq.restype = i32
    L.rq_cache_truncate_seq.argtypes = [vp, i32, i32, i32, i32]
    L.rq_cache_length_seq.restype = i32
    L.rq_cache_length_seq.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i32)]
    L.rq_cache_export.restype = i32
    L.rq_cache_export.argtypes = [vp, i32, i32, vp, vp, vp, vp]
    L.rq_decode_bytes.restype = ctypes.c_size_t
    L.rq_decode_bytes.argtypes = [vp, i32, i32]
    L.rq_check.restype = i32
    L.rq_check.argtypes = [vp]
    L.rq_cache_fork_seq.restype = i32
    L.rq_cache_fork_seq.argtypes = [vp, i32, i32, vp]
    L.rq_cache_shuffle_free_blocks.restype = i32
    L.rq_cache_shuffle_free_blocks.argtypes = [vp, ctypes.c_uint64]
    L.rq_cache_free_blocks.restype = i32
    L.rq_cache_free_blocks.argtypes = [vp, ctypes.POINTER(i32)]
    L.rq_cache_seq_blocks.restype = i32
    L.rq_cache_seq_blocks.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int32), i32, ctypes.POINTER(i32)]
    return L


lib = _load()


class RQError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {lib.rq_status_string(status).decode()} ({status})")


def _ok(status: int, what: str) -> None:
    if status != RQ_OK:
        raise RQError(status, what)


SCALE_LEAST_SQUARES, SCALE_NORM_RATIO, SCALE_NONE = 0, 1, 2
ANCHOR_LAST, ANCHOR_CHAINED = 0, 1


def make_config(*, num_layers: int, num_loops: int, loops_per_group: int, batch: int, max_tokens: int,
                max_tail_tokens: int, num_kv_heads: int, num_q_heads: int, head_dim: int = HEAD_DIM,
                group_size: int = 16, anchor_bits: int = 4, resid_bits: int = 2, rotate: bool = True,
                format: int = RQ_FMT_RESIDUAL, seed: int = 0xA11CE, scale_mode: int = SCALE_LEAST_SQUARES,
                anchor_mode: int = ANCHOR_LAST, rotation_per_layer: bool = False, block_tokens: int = 0,
                num_blocks: int = 0) -> rq_config:
    return rq_config(num_layers, num_loops, loops_per_group, batch, max_tokens, max_tail_tokens,
                     num_kv_heads, num_q_heads, head_dim, group_size, anchor_bits, resid_bits,
                     int(bool(rotate)), format, seed, scale_mode, anchor_mode, int(bool(rotation_per_layer)),
                     block_tokens, num_blocks)


def layer_seed(cfg: rq_config, layer: int) -> int:
    """The rotation seed of a layer (seed + layer * 2^32 with per-layer rotations)."""
    return (cfg.seed + (layer << 32 if cfg.rotation_per_layer else 0)) & ((1 << 64) - 1)


# ------------------------------------------------------------ C-ABI mirrors
def rq_status_string(status: int) -> str:
    return lib.rq_status_string(status).decode()


def rq_config_check(cfg: rq_config) -> int:
    return lib.rq_config_check(ctypes.byref(cfg))


def rq_cache_required_bytes(cfg: rq_config) -> int:
    return int(lib.rq_cache_required_bytes(ctypes.byref(cfg)))


def rq_cache_token_bytes(cfg: rq_config) -> int:
    return int(lib.rq_cache_token_bytes(ctypes.byref(cfg)))


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def _check_dev(t, dtype_name: str, shape, what: str):
    import torch
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{what} must be a contiguous CUDA tensor")
    if t.dtype != getattr(torch, dtype_name):
        raise ValueError(f"{what} must be {dtype_name}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def rq_cache_create(cfg: rq_config, arena=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    nbytes = 0 if arena is None else arena.numel() * arena.element_size()
    _ok(lib.rq_cache_create(ctypes.byref(cfg), ctypes.c_void_p(_ptr(arena)), nbytes, ctypes.byref(h)),
        "rq_cache_create")
    return h


def rq_cache_destroy(h) -> None:
    _ok(lib.rq_cache_destroy(h), "rq_cache_destroy")


def rq_append(h, layer: int, loop: int, k, v, n_tokens: int, stream=None) -> int:
    return lib.rq_append(h, layer, loop, ctypes.c_void_p(_ptr(k)), ctypes.c_void_p(_ptr(v)), n_tokens,
                         ctypes.c_void_p(_stream(stream)))


def rq_decode_attn(h, layer: int, loop: int, q, out, softmax_scale: float = 0.0, stream=None) -> int:
    return lib.rq_decode_attn(h, layer, loop, ctypes.c_void_p(_ptr(q)), ctypes.c_void_p(_ptr(out)),
                              softmax_scale, ctypes.c_void_p(_stream(stream)))


def rq_append_decode_attn(h, layer: int, loop: int, k, v, n_tokens: int, q, out, softmax_scale: float = 0.0,
                          stream=None) -> int:
    return lib.rq_append_decode_attn(h, layer, loop, ctypes.c_void_p(_ptr(k)), ctypes.c_void_p(_ptr(v)), n_tokens,
                                     ctypes.c_void_p(_ptr(q)), ctypes.c_void_p(_ptr(out)), softmax_scale,
                                     ctypes.c_void_p(_stream(stream)))


def rq_decode_attn_bf16(h, layer: int, loop: int, q, out, softmax_scale: float = 0.0, stream=None) -> int:
    return lib.rq_decode_attn_bf16(h, layer, loop, ctypes.c_void_p(_ptr(q)), ctypes.c_void_p(_ptr(out)),
                                   softmax_scale, ctypes.c_void_p(_stream(stream)))


def rq_prefill_attn(h, layer: int, loop: int, q, n_tokens: int, out, softmax_scale: float = 0.0,
                    stream=None) -> int:
    return lib.rq_prefill_attn(h, layer, loop, ctypes.c_void_p(_ptr(q)), n_tokens, ctypes.c_void_p(_ptr(out)),
                               softmax_scale, ctypes.c_void_p(_stream(stream)))


def rq_decode_attn_noalloc(h, layer: int, loop: int, q, out, softmax_scale: float = 0.0, stream=None) -> int:
    return lib.rq_decode_attn_noalloc(h, layer, loop, ctypes.c_void_p(_ptr(q)), ctypes.c_void_p(_ptr(out)),
                                      softmax_scale, ctypes.c_void_p(_stream(stream)))


def rq_cache_length(h, layer: int, group: int) -> int:
    n = ctypes.c_int(0)
    _ok(lib.rq_cache_length(h, layer, group, ctypes.byref(n)), "rq_cache_length")
    return n.value


def rq_cache_tail_length(h, layer: int, loop: int) -> int:
    n = ctypes.c_int(0)
    _ok(lib.rq_cache_tail_length(h, layer, loop, ctypes.byref(n)), "rq_cache_tail_length")
    return n.value


def rq_cache_truncate(h, layer: int, group: int, new_len: int) -> int:
    return lib.rq_cache_truncate(h, layer, group, new_len)


def rq_cache_truncate_seq(h, layer: int, group: int, seq: int, new_len: int) -> int:
    return lib.rq_cache_truncate_seq(h, layer, group, seq, new_len)


def rq_cache_length_seq(h, layer: int, group: int, seq: int) -> int:
    n = ctypes.c_int(0)
    _ok(lib.rq_cache_length_seq(h, layer, group, seq, ctypes.byref(n)), "rq_cache_length_seq")
    return n.value


def rq_decode_bytes(h, layer: int, loop: int) -> int:
    return int(lib.rq_decode_bytes(h, layer, loop))


def rq_check(h) -> int:
    return lib.rq_check(h)


def rq_cache_fork_seq(h, src: int, dst: int, stream=None) -> int:
    return lib.rq_cache_fork_seq(h, src, dst, ctypes.c_void_p(_stream(stream)))


def rq_cache_shuffle_free_blocks(h, seed: int) -> int:
    return lib.rq_cache_shuffle_free_blocks(h, seed)


def rq_cache_free_blocks(h) -> int:
    n = ctypes.c_int(0)
    _ok(lib.rq_cache_free_blocks(h, ctypes.byref(n)), "rq_cache_free_blocks")
    return n.value


def rq_cache_seq_blocks(h, seq: int) -> list:
    n = ctypes.c_int(0)
    _ok(lib.rq_cache_seq_blocks(h, seq, None, 0, ctypes.byref(n)), "rq_cache_seq_blocks")
    buf = (ctypes.c_int32 * max(n.value, 1))()
    _ok(lib.rq_cache_seq_blocks(h, seq, buf, n.value, ctypes.byref(n)), "rq_cache_seq_blocks")
    return list(buf[:n.value])


# ------------------------------------------------------------ convenience
class Cache:
    """Owns one rq_cache handle (and its arena, a torch uint8 tensor, unless
    ``library_alloc`` asks the library to cudaMalloc it)."""

    def __init__(self, cfg: rq_config, device=None, library_alloc: bool = False, arena=None):
        """arena: an optional caller-owned uint8 CUDA tensor of at least
        rq_cache_required_bytes(cfg) bytes, 256-byte aligned (for example a
        view into a larger buffer); by default one is allocated."""
        import torch
        self.cfg = cfg
        self.B, self.H, self.Hq = cfg.batch, cfg.num_kv_heads, cfg.num_q_heads
        self.Lg = cfg.loops_per_group
        _ok(rq_config_check(cfg), "rq_config_check")
        self.nbytes = rq_cache_required_bytes(cfg)
        self.arena = arena
        if arena is None and not library_alloc:
            self.arena = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        self.h = rq_cache_create(cfg, self.arena)

    def close(self):
        if getattr(self, "h", None):
            rq_cache_destroy(self.h)
            self.h = None
            self.arena = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def append(self, layer: int, loop: int, k, v, stream=None) -> None:
        n = k.shape[1]
        shape = (self.B, n, self.H, HEAD_DIM)
        _check_dev(k, "bfloat16", shape, "k")
        _check_dev(v, "bfloat16", shape, "v")
        _ok(rq_append(self.h, layer, loop, k, v, n, stream), "rq_append")

    def decode(self, layer: int, loop: int, q, out=None, scale: float = 0.0, stream=None, bf16: bool = False):
        import torch
        _check_dev(q, "bfloat16", (self.B, self.Hq, HEAD_DIM), "q")
        if out is None:
            out = torch.empty((self.B, self.Hq, HEAD_DIM), dtype=torch.float32, device=q.device)
        _check_dev(out, "float32", (self.B, self.Hq, HEAD_DIM), "out")
        fn = rq_decode_attn_bf16 if bf16 else rq_decode_attn
        _ok(fn(self.h, layer, loop, q, out, scale, stream), fn.__name__)
        return out

    def prefill(self, layer: int, loop: int, q, out=None, scale: float = 0.0, stream=None):
        """rq_prefill_attn: causal attention of the n most recent tokens,
        q [batch][n][num_q_heads][128] bf16 -> fp32 of the same shape."""
        import torch
        n = q.shape[1]
        _check_dev(q, "bfloat16", (self.B, n, self.Hq, HEAD_DIM), "q")
        if out is None:
            out = torch.empty((self.B, n, self.Hq, HEAD_DIM), dtype=torch.float32, device=q.device)
        _check_dev(out, "float32", (self.B, n, self.Hq, HEAD_DIM), "out")
        _ok(rq_prefill_attn(self.h, layer, loop, q, n, out, scale, stream), "rq_prefill_attn")
        return out

    def append_decode(self, layer: int, loop: int, k, v, q, out=None, scale: float = 0.0, stream=None):
        """rq_append then rq_decode_attn, fused into one launch where possible."""
        import torch
        n = k.shape[1]
        shape = (self.B, n, self.H, HEAD_DIM)
        _check_dev(k, "bfloat16", shape, "k")
        _check_dev(v, "bfloat16", shape, "v")
        _check_dev(q, "bfloat16", (self.B, self.Hq, HEAD_DIM), "q")
        if out is None:
            out = torch.empty((self.B, self.Hq, HEAD_DIM), dtype=torch.float32, device=q.device)
        _check_dev(out, "float32", (self.B, self.Hq, HEAD_DIM), "out")
        _ok(rq_append_decode_attn(self.h, layer, loop, k, v, n, q, out, scale, stream), "rq_append_decode_attn")
        return out

    def length(self, layer: int, group: int) -> int:
        return rq_cache_length(self.h, layer, group)

    def tail_length(self, layer: int, loop: int) -> int:
        return rq_cache_tail_length(self.h, layer, loop)

    def truncate(self, layer: int, group: int, new_len: int) -> None:
        _ok(rq_cache_truncate(self.h, layer, group, new_len), "rq_cache_truncate")

    def truncate_seq(self, layer: int, group: int, seq: int, new_len: int) -> None:
        _ok(rq_cache_truncate_seq(self.h, layer, group, seq, new_len), "rq_cache_truncate_seq")

    def length_seq(self, layer: int, group: int, seq: int) -> int:
        return rq_cache_length_seq(self.h, layer, group, seq)

    def decode_bytes(self, layer: int, loop: int) -> int:
        return rq_decode_bytes(self.h, layer, loop)

    def check(self) -> None:
        _ok(rq_check(self.h), "rq_check")

    def fork_seq(self, src: int, dst: int, stream=None) -> None:
        _ok(rq_cache_fork_seq(self.h, src, dst, stream), "rq_cache_fork_seq")

    def shuffle_free_blocks(self, seed: int) -> None:
        _ok(rq_cache_shuffle_free_blocks(self.h, seed), "rq_cache_shuffle_free_blocks")

    def free_blocks(self) -> int:
        return rq_cache_free_blocks(self.h)

    def seq_blocks(self, seq: int) -> list:
        return rq_cache_seq_blocks(self.h, seq)

    def export(self, layer: int, loop: int, stream=None):
        """Logical records of (layer, loop) as numpy arrays:
        codes [2][B][H][len][bytes], meta [2][B][H][len][2d/g], coef [2][B][H][len] (uint16, residual loops)."""
        cfg = self.cfg
        j = loop % self.Lg
        # the anchor record holds the group's last loop, or its first under the chained reference
        anchor = j == (0 if cfg.anchor_mode else self.Lg - 1)
        n = self.length(layer, loop // self.Lg)
        bits = cfg.anchor_bits if anchor else cfg.resid_bits
        codes = np.zeros((2, self.B, self.H, n, HEAD_DIM * bits // 8), np.uint8)
        meta = np.zeros((2, self.B, self.H, n, 2 * HEAD_DIM // cfg.group_size), np.uint8)
        coef = None if anchor else np.zeros((2, self.B, self.H, n), np.uint16)
        _ok(lib.rq_cache_export(self.h, layer, loop, codes.ctypes.data_as(ctypes.c_void_p),
                                meta.ctypes.data_as(ctypes.c_void_p),
                                None if coef is None else coef.ctypes.data_as(ctypes.c_void_p),
                                ctypes.c_void_p(_stream(stream))), "rq_cache_export")
        return codes, meta, coef
