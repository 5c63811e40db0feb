"""ctypes front end of the fp64 CPU oracle (``rq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It never
imports the CUDA package and the CUDA package never imports it.

All arrays are numpy; floating point is float64; BF16 inputs are passed as
their uint16 bit patterns, exactly as the GPU holds them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rq_oracle.c")
_LIB = os.path.join(_HERE, "librq_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``rq_oracle.c`` into ``librq_oracle.so`` (plain gcc, IEEE fp:
    no fast-math and no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        L.orc_fp8_value.restype = ctypes.c_double
        L.orc_fp8_value.argtypes = [ctypes.c_uint8]
        L.orc_fp8_round.restype = ctypes.c_uint8
        L.orc_fp8_round.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_int)]
        L.orc_bf16_value.restype = ctypes.c_double
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_bf16_round.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_int)]
        L.orc_splitmix64.restype = ctypes.c_uint64
        L.orc_splitmix64.argtypes = [ctypes.c_uint64]
        L.orc_rotation_signs.restype = None
        L.orc_rotation_signs.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
        L.orc_rotation_scale.restype = ctypes.c_double
        L.orc_rotation_scale.argtypes = [ctypes.c_int, ctypes.c_int]
        L.orc_rotation_matrix.restype = None
        L.orc_rotation_matrix.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.orc_quantize_group.restype = None
        L.orc_quantize_group.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p, u8p, u8p, ctypes.c_void_p, u8p]
        L.orc_pack.restype = None
        L.orc_pack.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.orc_unpack.restype = None
        L.orc_unpack.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.orc_dequant.restype = None
        L.orc_dequant.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_void_p]
        L.orc_encode.restype = None
        L.orc_encode.argtypes = [ctypes.c_int] * 7 + [ctypes.c_uint64] + [ctypes.c_void_p] * 11
        L.orc_reconstruct.restype = None
        L.orc_reconstruct.argtypes = [ctypes.c_int] * 7 + [ctypes.c_uint64] + [ctypes.c_void_p] * 6
        L.orc_attention.restype = None
        L.orc_attention.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [ctypes.c_void_p] * 4 + [ctypes.c_int]
        L.orc_mse.restype = ctypes.c_double
        L.orc_mse.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t]
        L.orc_encode_modes.restype = None
        L.orc_encode_modes.argtypes = [ctypes.c_int] * 7 + [ctypes.c_uint64] + [ctypes.c_int] * 2 + \
            [ctypes.c_void_p] * 11
        L.orc_reconstruct_modes.restype = None
        L.orc_reconstruct_modes.argtypes = [ctypes.c_int] * 7 + [ctypes.c_uint64] + [ctypes.c_int] + \
            [ctypes.c_void_p] * 6
        L.orc_encode_ablation.restype = None
        L.orc_encode_ablation.argtypes = [ctypes.c_int] * 7 + [ctypes.c_uint64] + [ctypes.c_int] * 2 + \
            [ctypes.c_void_p] * 4
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalars
def fp8_value(code: int) -> float:
    return lib().orc_fp8_value(code)


def fp8_round(v: float) -> tuple[int, bool]:
    near = ctypes.c_int(0)
    c = lib().orc_fp8_round(float(v), ctypes.byref(near))
    return int(c), bool(near.value)


def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(bits)


def bf16_round(v: float) -> tuple[int, bool]:
    near = ctypes.c_int(0)
    c = lib().orc_bf16_round(float(v), ctypes.byref(near))
    return int(c), bool(near.value)


def splitmix64(x: int) -> int:
    return int(lib().orc_splitmix64(x))


def rotation_signs(seed: int, d: int) -> np.ndarray:
    out = np.zeros(d, np.float64)
    lib().orc_rotation_signs(seed, d, _p(out))
    return out


def rotation_scale(d: int, rotate: bool = True) -> float:
    """The scalar c of R = c * H diag(sigma): 1/sqrt(d), correctly rounded."""
    return float(lib().orc_rotation_scale(d, int(rotate)))


def rotation_matrix(seed: int, d: int, rotate: bool = True) -> np.ndarray:
    R = np.zeros((d, d), np.float64)
    lib().orc_rotation_matrix(seed, d, int(rotate), _p(R))
    return R


# ---------------------------------------------------------------- quantizer
def quantize_group(x: np.ndarray, bits: int):
    """Returns (codes[g], scale_code, min_code, elem_flags[g], meta_flag)."""
    x = np.ascontiguousarray(x, np.float64)
    g = x.size
    codes = np.zeros(g, np.uint8)
    ef = np.zeros(g, np.uint8)
    s8 = ctypes.c_uint8(0)
    m8 = ctypes.c_uint8(0)
    mf = ctypes.c_uint8(0)
    lib().orc_quantize_group(_p(x), g, bits, _p(codes), ctypes.byref(s8), ctypes.byref(m8),
                             _p(ef), ctypes.byref(mf))
    return codes, int(s8.value), int(m8.value), ef, int(mf.value)


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.zeros(codes.size * bits // 8, np.uint8)
    lib().orc_pack(_p(codes), codes.size, bits, _p(out))
    return out


def unpack(packed: np.ndarray, d: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    out = np.zeros(d, np.uint8)
    lib().orc_unpack(_p(packed), d, bits, _p(out))
    return out


def dequant(packed: np.ndarray, meta: np.ndarray, d: int, g: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    meta = np.ascontiguousarray(meta, np.uint8)
    out = np.zeros(d, np.float64)
    lib().orc_dequant(_p(packed), _p(meta), d, g, bits, _p(out))
    return out


# ---------------------------------------------------------------- records
class Encoded:
    """Logical records of one loop group for n token-heads (see rq_oracle.c)."""

    def __init__(self, n, L, d, g, ba, br):
        G = d // g
        self.n, self.L, self.d, self.g, self.ba, self.br = n, L, d, g, ba, br
        self.a_codes = np.zeros((n, d * ba // 8), np.uint8)
        self.a_meta = np.zeros((n, 2 * G), np.uint8)
        self.r_codes = np.zeros((L - 1, n, d * br // 8), np.uint8)
        self.r_meta = np.zeros((L - 1, n, 2 * G), np.uint8)
        self.r_coef = np.zeros((L - 1, n), np.uint16)
        self.a_eflag = np.zeros((n, d), np.uint8)
        self.a_mflag = np.zeros((n, G), np.uint8)
        self.r_eflag = np.zeros((L - 1, n, d), np.uint8)
        self.r_mflag = np.zeros((L - 1, n, G), np.uint8)
        self.r_cflag = np.zeros((L - 1, n), np.uint8)


def encode(x_bf16: np.ndarray, g: int, ba: int, br: int, rotate: bool, seed: int) -> Encoded:
    """x_bf16: uint16 [L][n][d] (loop L-1 is the anchor)."""
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    L, n, d = x_bf16.shape
    e = Encoded(n, L, d, g, ba, br)
    lib().orc_encode(n, L, d, g, ba, br, int(rotate), seed, _p(x_bf16),
                     _p(e.a_codes), _p(e.a_meta), _p(e.r_codes), _p(e.r_meta), _p(e.r_coef),
                     _p(e.a_eflag), _p(e.a_mflag), _p(e.r_eflag), _p(e.r_mflag), _p(e.r_cflag))
    return e


def reconstruct(a_codes, a_meta, r_codes, r_meta, r_coef, L: int, d: int, g: int,
                ba: int, br: int, rotate: bool, seed: int) -> np.ndarray:
    """Returns float64 [L][n][d]."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    a_meta = np.ascontiguousarray(a_meta, np.uint8)
    n = a_codes.shape[0]
    if L > 1:
        r_codes = np.ascontiguousarray(r_codes, np.uint8)
        r_meta = np.ascontiguousarray(r_meta, np.uint8)
        r_coef = np.ascontiguousarray(r_coef, np.uint16)
    else:
        r_codes = np.zeros(1, np.uint8)
        r_meta = np.zeros(1, np.uint8)
        r_coef = np.zeros(1, np.uint16)
    out = np.zeros((L, n, d), np.float64)
    lib().orc_reconstruct(n, L, d, g, ba, br, int(rotate), seed, _p(a_codes), _p(a_meta),
                          _p(r_codes), _p(r_meta), _p(r_coef), _p(out))
    return out


def encode_modes(x_bf16: np.ndarray, g: int, ba: int, br: int, rotate: bool, seed: int, anchor_mode: int,
                 scale_mode: int) -> Encoded:
    """Records of the ablation modes in the library's layout (orc_encode_modes):
    x_bf16 uint16 [L][n][d] in loop order."""
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    L, n, d = x_bf16.shape
    e = Encoded(n, L, d, g, ba, br)
    lib().orc_encode_modes(n, L, d, g, ba, br, int(rotate), seed, int(anchor_mode), int(scale_mode), _p(x_bf16),
                           _p(e.a_codes), _p(e.a_meta), _p(e.r_codes), _p(e.r_meta), _p(e.r_coef),
                           _p(e.a_eflag), _p(e.a_mflag), _p(e.r_eflag), _p(e.r_mflag), _p(e.r_cflag))
    return e


def reconstruct_modes(a_codes, a_meta, r_codes, r_meta, r_coef, L: int, d: int, g: int, ba: int, br: int,
                      rotate: bool, seed: int, anchor_mode: int) -> np.ndarray:
    """float64 [L][n][d] in loop order, from records as encode_modes lays them out."""
    if anchor_mode == 0:
        return reconstruct(a_codes, a_meta, r_codes, r_meta, r_coef, L, d, g, ba, br, rotate, seed)
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    a_meta = np.ascontiguousarray(a_meta, np.uint8)
    r_codes = np.ascontiguousarray(r_codes, np.uint8)
    r_meta = np.ascontiguousarray(r_meta, np.uint8)
    r_coef = np.ascontiguousarray(r_coef, np.uint16)
    n = a_codes.shape[0]
    out = np.zeros((L, n, d), np.float64)
    lib().orc_reconstruct_modes(n, L, d, g, ba, br, int(rotate), seed, int(anchor_mode), _p(a_codes), _p(a_meta),
                                _p(r_codes), _p(r_meta), _p(r_coef), _p(out))
    return out


ANCHOR_LAST, ANCHOR_PREVIOUS = 0, 1
SCALE_LEAST_SQUARES, SCALE_NORM_RATIO, SCALE_NONE = 0, 1, 2


def encode_ablation(x_bf16: np.ndarray, g: int, ba: int, br: int, rotate: bool, seed: int,
                    anchor_mode: int, scale_mode: int):
    """Ablation encoders of one loop group (orc_encode_ablation): x_bf16
    uint16 [L][n][d] -> (reconstruction float64 [L][n][d], stored
    coefficients float64 [L][n], records read to rebuild each loop [L])."""
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    L, n, d = x_bf16.shape
    xhat = np.zeros((L, n, d), np.float64)
    coef = np.zeros((L, n), np.float64)
    reads = np.zeros(L, np.int32)
    lib().orc_encode_ablation(n, L, d, g, ba, br, int(rotate), seed, int(anchor_mode), int(scale_mode),
                              _p(x_bf16), _p(xhat), _p(coef), _p(reads))
    return xhat, coef, reads


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, threads: int = 1) -> np.ndarray:
    """q [B][Hq][d], k/v [B][T][Hkv][d] float64 -> out [B][Hq][d] float64."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    B, Hq, d = q.shape
    _, T, Hkv, _ = k.shape
    out = np.zeros((B, Hq, d), np.float64)
    lib().orc_attention(B, Hq, Hkv, d, T, float(scale), _p(q), _p(k), _p(v), _p(out), int(threads))
    return out


def mse(a: np.ndarray, b: np.ndarray) -> float:
    a = np.ascontiguousarray(a, np.float64)
    b = np.ascontiguousarray(b, np.float64)
    assert a.size == b.size
    return float(lib().orc_mse(_p(a), _p(b), a.size))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float64 (exact)."""
    u = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
