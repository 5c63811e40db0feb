"""Test harness: builds caches on the GPU through the C ABI from seeded
synthetic inputs, and checks the GPU results against the fp64 oracle.

Parity contract (stated for the ResidualQuant hot path):
  * every packed code, FP8 scale/min and BF16 coefficient is compared and
    must be bit-exact; a difference is tolerated (and counted) only at a
    value the oracle flags as lying within 1e-6 (relative) of a rounding
    boundary, exact ties included.  A tolerated difference excludes what
    depends on it: a scale/min its group's codes, a coefficient its residual
    record, an anchor record the token-head's residual records;
  * attention output against the oracle fed the GPU's own records: relative
    L2 error <= 1e-3 and max abs error <= 2e-3;
  * reconstruction MSE of the GPU's records within 1% of the oracle's.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import decode_attention_14_b200 as rq
import synth
from oracle import oracle as orc

REL_L2_TOL = 1e-3
MAX_ABS_TOL = 2e-3
MSE_REL_TOL = 0.01
D = 128


# ------------------------------------------------------------------ guard bands
# Every cache the harness creates lives in the middle of a larger buffer
# whose margins hold a fixed byte pattern, and decode outputs get the same;
# an autouse fixture (conftest.py) checks after each GPU test that no margin
# changed -- a write outside the arena or past an output row would.
GUARD = 4096
GUARD_BYTE = 0xA5
_guarded = []


def guarded_buffer(nbytes: int, dtype=torch.uint8, device="cuda"):
    """A tensor view of nbytes (256-byte aligned) inside a buffer with
    GUARD_BYTE margins of GUARD bytes on both sides."""
    big = torch.full((nbytes + 2 * GUARD,), GUARD_BYTE, dtype=torch.uint8, device=device)
    _guarded.append((big, GUARD, nbytes))
    return big[GUARD:GUARD + nbytes].view(dtype)


def guarded_out(shape):
    n = int(np.prod(shape))
    return guarded_buffer(4 * n, torch.float32).view(*shape)


def check_guards():
    """Asserts that no margin changed; forgets the buffers."""
    bad = []
    for big, off, n in _guarded:
        host = big.cpu().numpy()
        if not ((host[:off] == GUARD_BYTE).all() and (host[off + n:] == GUARD_BYTE).all()):
            bad.append(n)
    _guarded.clear()
    assert not bad, f"guard bands overwritten around buffers of {bad} bytes"


def guarded_cache(cfg) -> rq.Cache:
    return rq.Cache(cfg, arena=guarded_buffer(rq.rq_cache_required_bytes(cfg)))


@dataclass
class Built:
    cache: rq.Cache
    cfg: object
    seed: int
    T: int
    n_tail: int
    # inputs[layer][group] = (K list of Lg bf16 [B][T+n_tail][H][d], V list)
    inputs: dict = field(default_factory=dict)
    # memoised oracle reconstructions of the GPU records (keyed by what they depend on)
    recon: dict = field(default_factory=dict)


def scale32() -> float:
    return float(np.float32(1.0 / math.sqrt(D)))


def build(*, layers=1, loops=4, Lg=4, B=1, T=256, H=4, Hq=8, g=16, ba=4, br=2, rotate=True,
          n_tail=0, seed=0x5EED0000, sigma=(0.1, 0.2, 0.3), chunk=128, fmt=rq.RQ_FMT_RESIDUAL,
          only_layers=None, only_groups=None, max_tokens=None, prepare=None, **modes) -> Built:
    """Fills `layers` x (loops/Lg) groups with T committed tokens (appended in
    chunks through the tail), then n_tail in-flight tokens on every
    non-anchor loop."""
    tail_cap = max(chunk, n_tail, 1)
    cfg = rq.make_config(num_layers=layers, num_loops=loops, loops_per_group=Lg, batch=B,
                         max_tokens=max_tokens or max(T, 1), max_tail_tokens=tail_cap, num_kv_heads=H,
                         num_q_heads=Hq, group_size=g, anchor_bits=ba, resid_bits=br, rotate=rotate,
                         format=fmt, seed=0xA11CE, **modes)
    cache = guarded_cache(cfg)
    if prepare is not None:
        prepare(cache)
    bt = Built(cache, cfg, seed, T, n_tail)
    for layer in range(layers):
        if only_layers is not None and layer not in only_layers:
            continue
        for grp in range(loops // Lg):
            if only_groups is not None and grp not in only_groups:
                continue
            K, V = synth.group_kv(seed, layer, grp, Lg, sigma, B, T + n_tail, H, device="cuda")
            fill_group(bt, layer, grp, K, V, chunk)
    torch.cuda.synchronize()
    return bt


def fill_group(bt: Built, layer: int, grp: int, K, V, chunk: int = 128) -> None:
    """Appends the given K/V of one loop group (lists of Lg BF16 CUDA tensors
    [B][T + n_tail][H][d], index Lg - 1 the anchor): the first bt.T tokens
    committed in chunks through the tails, the rest left in the tails."""
    cache, T, Lg = bt.cache, bt.T, bt.cfg.loops_per_group
    bt.inputs[(layer, grp)] = (K, V)
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        for j in range(Lg):
            cache.append(layer, grp * Lg + j, K[j][:, t0:t1].contiguous(), V[j][:, t0:t1].contiguous())
    if bt.n_tail and bt.cfg.format == rq.RQ_FMT_RESIDUAL:
        for j in range(Lg - 1):
            cache.append(layer, grp * Lg + j, K[j][:, T:].contiguous(), V[j][:, T:].contiguous())


def build_from(K, V, *, Hq: int, g=16, ba=4, br=2, rotate=True, T: int, n_tail=0, chunk=128,
               seed=0) -> Built:
    """A one-layer, one-group cache holding the given K/V (lists of Lg BF16
    CUDA tensors [B][T + n_tail][H][d]; index Lg - 1 is the anchor)."""
    Lg = len(K)
    B, _, Hkv, _ = K[0].shape
    cfg = rq.make_config(num_layers=1, num_loops=Lg, loops_per_group=Lg, batch=B, max_tokens=max(T, 1),
                         max_tail_tokens=max(chunk, n_tail, 1), num_kv_heads=Hkv, num_q_heads=Hq, group_size=g,
                         anchor_bits=ba, resid_bits=br, rotate=rotate, seed=0xA11CE)
    bt = Built(guarded_cache(cfg), cfg, seed, T, n_tail)
    fill_group(bt, 0, 0, K, V, chunk)
    torch.cuda.synchronize()
    return bt


# ------------------------------------------------------------------ records
def oracle_encode(bt: Built, layer: int, grp: int, kv: int, bh_sel=None) -> orc.Encoded:
    """Oracle encoding of the committed tokens of one group and side.
    Token-heads ordered (b, h, t) like the export; bh_sel restricts to a list
    of (b, h)."""
    K, V = bt.inputs[(layer, grp)]
    X = K if kv == 0 else V
    Lg = len(X)
    T = bt.T
    arrs = []
    for j in range(Lg):
        u = synth.bf16_to_u16(X[j][:, :T])            # [B][T][H][d]
        u = np.ascontiguousarray(u.transpose(0, 2, 1, 3))   # [B][H][T][d]
        if bh_sel is not None:
            u = np.stack([u[b, h] for (b, h) in bh_sel])     # [nsel][T][d]
        arrs.append(u.reshape(-1, D))
    x = np.stack(arrs)
    cfg = bt.cfg
    seed = rq.layer_seed(cfg, layer)
    if cfg.anchor_mode or cfg.scale_mode:
        return orc.encode_modes(x, cfg.group_size, cfg.anchor_bits, cfg.resid_bits, bool(cfg.rotate), seed,
                                cfg.anchor_mode, cfg.scale_mode)
    return orc.encode(x, cfg.group_size, cfg.anchor_bits, cfg.resid_bits, bool(cfg.rotate), seed)


def anchor_loop(cfg, grp: int) -> int:
    """The loop whose K/V the anchor record holds (the last of the group;
    the first with the chained reference)."""
    return grp * cfg.loops_per_group + (0 if cfg.anchor_mode else cfg.loops_per_group - 1)


def residual_loop(cfg, grp: int, j: int) -> int:
    """The loop whose K/V residual record j holds."""
    return grp * cfg.loops_per_group + (j + 1 if cfg.anchor_mode else j)


def gpu_records(bt: Built, layer: int, loop: int, kv: int, bh_sel=None):
    codes, meta, coef = bt.cache.export(layer, loop)
    c, m = codes[kv], meta[kv]
    f = None if coef is None else coef[kv]
    if bh_sel is not None:
        c = np.stack([c[b, h] for (b, h) in bh_sel])
        m = np.stack([m[b, h] for (b, h) in bh_sel])
        if f is not None:
            f = np.stack([f[b, h] for (b, h) in bh_sel])
    c = c.reshape(-1, c.shape[-1])
    m = m.reshape(-1, m.shape[-1])
    if f is not None:
        f = f.reshape(-1)
    return c, m, f


def _elem_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    per = 8 // bits
    return np.stack([(packed >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], -1).reshape(
        packed.shape[0], -1)


def compare_records(bt: Built, layer: int, grp: int, kv: int, bh_sel=None):
    """Compares every code, FP8 scale/min and BF16 coefficient.  A difference
    at a value the oracle flags as within 1e-6 (relative) of a rounding
    boundary (exact ties included) is tolerated and counted; a tolerated
    difference in an anchor record or a coefficient excludes the records that
    depend on it (the token-head's residuals / that residual record).  Any
    other difference is a mismatch.  Returns counts."""
    cfg = bt.cfg
    Lg = cfg.loops_per_group
    e = oracle_encode(bt, layer, grp, kv, bh_sel)
    res = dict(mismatch=0, tolerated=0, flagged=0, excluded=0, compared=0)
    gc, gm, _ = gpu_records(bt, layer, anchor_loop(cfg, grp), kv, bh_sel)
    grp_of = np.arange(D) // cfg.group_size

    def cmp(gpu_c, gpu_m, orc_c, orc_m, eflag, mflag, bits, skip_rows):
        """returns per-row bool: some tolerated difference in this record"""
        ge, oe = _elem_codes(gpu_c, bits), _elem_codes(orc_c, bits)
        live = ~skip_rows[:, None]
        # meta
        sc_diff = (gpu_m[:, 0::2] != orc_m[:, 0::2]) & live
        mn_diff = (gpu_m[:, 1::2] != orc_m[:, 1::2]) & live
        sc_flag = (mflag & 1) != 0
        mn_flag = (mflag & 2) != 0
        res["mismatch"] += int((sc_diff & ~sc_flag).sum() + (mn_diff & ~mn_flag).sum())
        meta_tol = (sc_diff & sc_flag) | (mn_diff & mn_flag)             # [rows][groups]
        # codes: a group whose meta legitimately differs is excluded
        excl = meta_tol[:, grp_of] | skip_rows[:, None]
        diff = (ge != oe) & ~excl
        fl = eflag.astype(bool)
        res["mismatch"] += int((diff & ~fl).sum())
        res["tolerated"] += int((diff & fl).sum() + meta_tol.sum())
        res["flagged"] += int((fl & ~excl).sum() + ((sc_flag | mn_flag) & live).sum())
        res["excluded"] += int(excl.sum())
        res["compared"] += int((~excl).sum())
        return (diff & fl).any(1) | meta_tol.any(1)

    a_tol = cmp(gc, gm, e.a_codes, e.a_meta, e.a_eflag, e.a_mflag, cfg.anchor_bits, np.zeros(len(gc), bool))
    for j in range(Lg - 1):
        rc, rm, rf = gpu_records(bt, layer, residual_loop(cfg, grp, j), kv, bh_sel)
        cdiff = (rf != e.r_coef[j]) & ~a_tol
        cflag = e.r_cflag[j] != 0
        res["mismatch"] += int((cdiff & ~cflag).sum())
        res["tolerated"] += int((cdiff & cflag).sum())
        cmp(rc, rm, e.r_codes[j], e.r_meta[j], e.r_eflag[j], e.r_mflag[j], cfg.resid_bits, a_tol | cdiff)
    return res


def reconstruct_gpu(bt: Built, layer: int, grp: int, kv: int, bh_sel=None) -> np.ndarray:
    """Oracle reconstruction of the GPU's exported records: [Lg][n][d]."""
    key = (layer, grp, kv, None if bh_sel is None else tuple(bh_sel), bt.T)
    if key not in bt.recon:
        bt.recon[key] = _reconstruct_gpu(bt, layer, grp, kv, bh_sel)
    return bt.recon[key]


def _reconstruct_gpu(bt: Built, layer: int, grp: int, kv: int, bh_sel=None) -> np.ndarray:
    cfg = bt.cfg
    Lg = cfg.loops_per_group
    ac, am, _ = gpu_records(bt, layer, anchor_loop(cfg, grp), kv, bh_sel)
    if Lg > 1:
        rs = [gpu_records(bt, layer, residual_loop(cfg, grp, j), kv, bh_sel) for j in range(Lg - 1)]
        rc = np.stack([r[0] for r in rs])
        rm = np.stack([r[1] for r in rs])
        rf = np.stack([r[2] for r in rs])
    else:
        rc = rm = rf = None
    return orc.reconstruct_modes(ac, am, rc, rm, rf, Lg, D, cfg.group_size, cfg.anchor_bits, cfg.resid_bits,
                                 bool(cfg.rotate), rq.layer_seed(cfg, layer), cfg.anchor_mode)


def mse_check(bt: Built, layer: int, grp: int, kv: int, bh_sel=None):
    cfg = bt.cfg
    e = oracle_encode(bt, layer, grp, kv, bh_sel)
    Lg = cfg.loops_per_group
    mine = orc.reconstruct_modes(e.a_codes, e.a_meta, e.r_codes if Lg > 1 else None,
                                 e.r_meta if Lg > 1 else None, e.r_coef if Lg > 1 else None, Lg, D,
                                 cfg.group_size, cfg.anchor_bits, cfg.resid_bits, bool(cfg.rotate),
                                 rq.layer_seed(cfg, layer), cfg.anchor_mode)
    gpu = reconstruct_gpu(bt, layer, grp, kv, bh_sel)
    K, V = bt.inputs[(layer, grp)]
    X = K if kv == 0 else V
    xs = []
    for j in range(Lg):
        u = synth.bf16_to_u16(X[j][:, :bt.T]).transpose(0, 2, 1, 3)
        if bh_sel is not None:
            u = np.stack([u[b, h] for (b, h) in bh_sel])
        xs.append(orc.bf16_bits_to_f64(np.ascontiguousarray(u).reshape(-1, D)))
    x = np.stack(xs)
    return orc.mse(gpu, x), orc.mse(mine, x)


# ------------------------------------------------------------------ attention
def oracle_decode(bt: Built, layer: int, loop: int, q_bf16: torch.Tensor, bh_sel=None, bf16_cache=False):
    """Oracle attention for (layer, loop), keys/values from the GPU's own
    records (or, for the BF16 format, the BF16 inputs).  Returns
    [len(bh_sel) or B*Hq ...] as [B][Hq][d] restricted to selected (b, kv)."""
    cfg = bt.cfg
    Lg = cfg.loops_per_group
    grp, j = loop // Lg, loop % Lg
    B, H, Hq = cfg.batch, cfg.num_kv_heads, cfg.num_q_heads
    Gq = Hq // H
    K, V = bt.inputs[(layer, grp)]
    sel = bh_sel if bh_sel is not None else [(b, h) for b in range(B) for h in range(H)]
    n_tail = bt.n_tail if (j != Lg - 1 and not bf16_cache) else 0
    T = bt.T
    qf = orc.bf16_bits_to_f64(synth.bf16_to_u16(q_bf16))          # [B][Hq][d]
    kv_vals = []
    for kv, X in ((0, K), (1, V)):
        if bf16_cache:
            u = synth.bf16_to_u16(X[j][:, :T]).transpose(0, 2, 1, 3)
            vals = orc.bf16_bits_to_f64(np.stack([u[b, h] for (b, h) in sel]))     # [nsel][T][d]
        else:
            # exported records span the group's longest sequence; keep the first T tokens
            rec = reconstruct_gpu(bt, layer, grp, kv, sel)[j].reshape(len(sel), -1, D)
            vals = rec[:, :T]
        if n_tail:
            tu = synth.bf16_to_u16(X[j][:, T:T + n_tail]).transpose(0, 2, 1, 3)
            tv = orc.bf16_bits_to_f64(np.stack([tu[b, h] for (b, h) in sel]))
            vals = np.concatenate([vals, tv], axis=1)
        kv_vals.append(vals)
    out = {}
    for i, (b, h) in enumerate(sel):
        q = qf[b:b + 1, h * Gq:(h + 1) * Gq]                       # [1][Gq][d]
        k = kv_vals[0][i][None, :, None, :]
        v = kv_vals[1][i][None, :, None, :]
        o = orc.attention(q, k, v, scale32())
        out[(b, h)] = o[0]                                          # [Gq][d]
    return out


def attn_errors(gpu_out: np.ndarray, ref: dict, Gq: int):
    g, r = [], []
    for (b, h), o in ref.items():
        g.append(gpu_out[b, h * Gq:(h + 1) * Gq])
        r.append(o)
    g = np.concatenate(g).astype(np.float64)
    r = np.concatenate(r)
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    mx = float(np.abs(g - r).max())
    return rel, mx
