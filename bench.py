"""Benchmark of the ResidualQuant decode step on B200.

A step is one decode step of a looped Transformer over a cache already
holding T-1 committed tokens per sequence: for every loop (outer) and layer
(inner) it appends the new token's K/V and runs single-token decode attention
over T keys: rq_append_decode_attn, one launch for loops 1..L-1 (the decode
kernel writes the tail row), the fp64 encode + commit and then the decode at
the anchor loop (--separate-append: rq_append and rq_decode_attn as two calls).  The metric is decode-attention
tokens/s = batch / step time (whole job: all ranks' sequences / max-over-ranks
time), plus achieved HBM GB/s of the decode calls over their algorithmic
compressed bytes.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
Multi-GPU: launched by torchrun, one rank per GPU; every rank owns its own
batch (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

CONFIGS = {
    # name: (layers, loops, loops_per_group, batch, T, H_kv, H_q, g, ba, br, sigma by distance)
    "tiny": dict(layers=1, loops=4, Lg=4, B=1, T=256, H=4, Hq=8, g=16, ba=4, br=2, sigma=(0.1, 0.2, 0.3)),
    "ouro8k_b4": dict(layers=24, loops=4, Lg=4, B=4, T=8192, H=16, Hq=16, g=16, ba=4, br=2, sigma=(0.1, 0.2, 0.3)),
    "long16k_b2": dict(layers=24, loops=4, Lg=4, B=2, T=16384, H=16, Hq=16, g=16, ba=4, br=2, sigma=(0.1, 0.2, 0.3)),
    "long16k_b4": dict(layers=24, loops=4, Lg=4, B=4, T=16384, H=16, Hq=16, g=16, ba=4, br=2, sigma=(0.1, 0.2, 0.3)),
    "deep": dict(layers=4, loops=32, Lg=4, B=8, T=4096, H=40, Hq=40, g=16, ba=4, br=2, sigma=(0.1, 0.25, 0.4)),
}
CONFIG_SEED = {"tiny": 0x5EED0000, "ouro8k_b4": 0x5EED0001, "long16k_b2": 0x5EED0002,
               "long16k_b4": 0x5EED0002, "deep": 0x5EED0003}
FILL_CHUNK = 512


KERNEL_SOURCES = ["decode_attention_14_b200/csrc/decode_rq.cu", "decode_attention_14_b200/csrc/combine.cuh",
                  "decode_attention_14_b200/csrc/common.cuh", "decode_attention_14_b200/csrc/rq_internal.h"]


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(config_name: str):
    """DRAM bytes (read + write) per decode launch from the committed ncu
    summary, only if it was taken on the kernel sources as they are now."""
    p = os.path.join(ROOT, "profiles", "decode_rq_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("sources_sha256") != kernel_sources_sha256():
        return None
    return j.get("bytes_per_launch", {}).get(config_name)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling (every 50 ms) around the
    timed region; summarise() keeps only the samples taken inside a host
    wall-clock window."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, path: str = ""):
        import tempfile
        self.index = index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), f"rq_clocks_rank{index}.csv")

    def start(self):
        if os.path.dirname(self.path):
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()

    def summarise(self, t0: float, t1: float):
        import datetime
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for n, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": max(r[2] for r in inside),
                "samples": len(inside), "reasons": sorted(reasons)}


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings (all ranks must call it).  With
    one process (no process group) the values come back unchanged."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_rate(world: int, per_rank_items: int, steps: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput: every rank processes its own per_rank_items per
    step; the job's time is the slowest rank's."""
    return world * per_rank_items * steps / (max_elapsed_ms / 1e3)


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own sequences (independent batches, no data-path exchange)."""
    return base + 1000 * rank


# ---------------------------------------------------------------- our arm
def run_ours(args, cfgd, rank, world, local_rank):
    import torch
    import decode_attention_14_b200 as rq
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    name = args.config
    layers = args.layers or cfgd["layers"]
    loops, Lg, B, T, H, Hq = cfgd["loops"], cfgd["Lg"], cfgd["B"], cfgd["T"], cfgd["H"], cfgd["Hq"]
    seed = rank_seed(CONFIG_SEED[name], rank)
    fmt = rq.RQ_FMT_BF16 if args.bf16 else rq.RQ_FMT_RESIDUAL
    paging = {}
    if args.paged:
        # 128-token blocks, the pool sized to the batch, allocation scattered over it
        paging = dict(block_tokens=128, num_blocks=B * ((T + 127) // 128) + 8)
    cfg = rq.make_config(num_layers=layers, num_loops=loops, loops_per_group=Lg, batch=B, max_tokens=T,
                         max_tail_tokens=FILL_CHUNK, num_kv_heads=H, num_q_heads=Hq, group_size=cfgd["g"],
                         anchor_bits=cfgd["ba"], resid_bits=cfgd["br"], rotate=True, format=fmt, seed=0xA11CE,
                         anchor_mode=rq.ANCHOR_CHAINED if args.chained else rq.ANCHOR_LAST, **paging)
    cache = rq.Cache(cfg, device=dev)
    if args.paged:
        cache.shuffle_free_blocks(0x5EED)
    T0 = T - 1
    groups = loops // Lg
    stream = torch.cuda.current_stream(dev)

    # ---- fill: T-1 committed tokens per (layer, group) (untimed)
    for layer in range(layers):
        for grp in range(groups):
            for t0 in range(0, T0, FILL_CHUNK):
                n = min(FILL_CHUNK, T0 - t0)
                Kg, Vg = synth.group_kv(seed, layer, grp, Lg, cfgd["sigma"], B, n, H, t0=t0, device=dev)
                for j in range(Lg):
                    cache.append(layer, grp * Lg + j, Kg[j], Vg[j])
                del Kg, Vg
    torch.cuda.synchronize(dev)

    # ---- per-step inputs: the new token of every (layer, loop), one query each
    gen = torch.Generator(device=dev)
    gen.manual_seed(synth.mix_seed(seed, 99))
    new_k = torch.randn((layers, loops, B, 1, H, 128), generator=gen, device=dev).to(torch.bfloat16)
    new_v = torch.randn((layers, loops, B, 1, H, 128), generator=gen, device=dev).to(torch.bfloat16)
    qs = torch.stack([torch.stack([synth.queries(seed, l, lp, 0, B, Hq, device=dev) for lp in range(loops)])
                      for l in range(layers)])
    outs = torch.empty((layers, loops, B, Hq, 128), dtype=torch.float32, device=dev)

    decode = rq.rq_decode_attn_bf16 if args.bf16 else rq.rq_decode_attn
    h = cache.h

    def reset():
        # host-side only: roll every (layer, group) back to T-1 committed tokens
        n_groups = loops if args.bf16 else groups
        for layer in range(layers):
            for grp in range(n_groups):
                cache.truncate(layer, grp, T0)

    fused = not args.bf16 and not args.separate_append

    def step(k=None, v=None, q=None, out=None):
        k = new_k if k is None else k
        v = new_v if v is None else v
        q = qs if q is None else q
        o = outs if out is None else out
        reset()
        cur = torch.cuda.current_stream(dev)
        sptr = int(cur.cuda_stream)
        for lp in range(loops):
            for layer in range(layers):
                if fused:
                    st = rq.rq_append_decode_attn(h, layer, lp, k[layer, lp], v[layer, lp], 1, q[layer, lp],
                                                  o[layer, lp], 0.0, sptr)
                    if st != 0:
                        raise rq.RQError(st, "rq_append_decode_attn")
                    continue
                st = rq.rq_append(h, layer, lp, k[layer, lp], v[layer, lp], 1, sptr)
                if st != 0:
                    raise rq.RQError(st, "rq_append")
                st = decode(h, layer, lp, q[layer, lp], o[layer, lp], 0.0, sptr)
                if st != 0:
                    raise rq.RQError(st, "rq_decode_attn")

    # algorithmic bytes of each decode call during a step (lengths as in the step)
    reset()
    call_bytes = []
    for lp in range(loops):
        for layer in range(layers):
            rq.rq_append(h, layer, lp, new_k[layer, lp], new_v[layer, lp], 1, int(stream.cuda_stream))
            call_bytes.append(cache.decode_bytes(layer, lp))
    torch.cuda.synchronize(dev)
    step_decode_bytes = sum(call_bytes)

    # The timed region replays one CUDA graph holding K identical steps (the
    # host-side state is reset to T-1 committed tokens before each captured
    # step, so every step launches the same work).  A second graph holds only
    # the K x (loops x layers) decode calls of those steps, with the same
    # arguments (the appends that set the cache state run eagerly on a side
    # stream while it is captured); replayed between two events it gives the
    # average decode-call duration for the roofline.
    ncalls = loops * layers
    for _ in range(2):
        step()   # eager warm-up before capture
    torch.cuda.synchronize(dev)
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        step()
    gK = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gK):
        for s_ in range(args.steps):
            step()
    side = torch.cuda.Stream(dev)
    gD = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gD, capture_error_mode="relaxed"):
        cur = torch.cuda.current_stream(dev)
        for s_ in range(args.steps):
            reset()
            for lp in range(loops):
                for layer in range(layers):
                    st = rq.rq_append(h, layer, lp, new_k[layer, lp], new_v[layer, lp], 1, int(side.cuda_stream))
                    if st != 0:
                        raise rq.RQError(st, "rq_append")
                    st = decode(h, layer, lp, qs[layer, lp], outs[layer, lp], 0.0, int(cur.cuda_stream))
                    if st != 0:
                        raise rq.RQError(st, "rq_decode_attn")
    side.synchronize()
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        g1.replay()
    torch.cuda.synchronize(dev)

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    sampler = ClockSampler(local_rank, args.clocks_csv) if rank == 0 and not args.no_clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    w0 = time.time()
    if args.profile:
        torch.cuda.cudart().cudaProfilerStart()   # ncu --profile-from-start off captures this region only
    t_start.record(stream)
    gK.replay()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if args.profile:
        torch.cuda.cudart().cudaProfilerStop()
    w1 = time.time()
    clocks = None
    if sampler:
        clock_src = "timed region"
        probe_until = w1
        if (w1 - w0) < 1.0:
            # too short for the sampler: replay the same graph for ~1.5 s more
            # (after the timed region, same load) and take the clocks there
            clock_src = "replays of the timed graph right after the timed region"
            pw0 = time.time()
            while time.time() - pw0 < 1.5:
                gK.replay()
                torch.cuda.synchronize(dev)
            probe_until = time.time()
            sampler.stop()
            clocks = sampler.summarise(pw0, probe_until)
        else:
            sampler.stop()
            clocks = sampler.summarise(w0, w1)
        if clocks is not None:
            clocks["sampled_during"] = clock_src
    elapsed_ms = t_start.elapsed_time(t_end)
    # average decode-call duration: the decode-only graph, right after the timed region
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    gD.replay()
    d1.record(stream)
    torch.cuda.synchronize(dev)
    dec_ms = d0.elapsed_time(d1)
    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], dev)

    # ---- end to end through the C ABI with host buffers
    # Every step copies its inputs in from pinned host memory and reads its
    # outputs back, through the public API, as a serving loop would: on a copy
    # stream, step s + 1's inputs go in while step s computes and step s's
    # outputs come out while step s + 1 computes (two buffer sets, ordered by
    # events).  The timed region runs from before the first copy in to after
    # the last copy out has landed.
    e2e = None
    if not args.no_e2e:
        hk = new_k.cpu().pin_memory()
        hv = new_v.cpu().pin_memory()
        hq = qs.cpu().pin_memory()
        ho = [torch.empty(outs.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        dk = [torch.empty_like(new_k) for _ in range(2)]
        dv = [torch.empty_like(new_v) for _ in range(2)]
        dq = [torch.empty_like(qs) for _ in range(2)]
        do = [torch.empty_like(outs) for _ in range(2)]
        h2d = hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 2
        d2h = ho[0].numel() * 4
        cs = torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the buffer set copied in
        ev_done = [torch.cuda.Event() for _ in range(2)]   # its step computed

        def copy_in(i):
            b = i % 2
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(ev_done[b])   # step i - 2 has read this set
                dk[b].copy_(hk, non_blocking=True)
                dv[b].copy_(hv, non_blocking=True)
                dq[b].copy_(hq, non_blocking=True)
                ev_in[b].record(cs)

        def run(nsteps):
            copy_in(0)
            for i in range(nsteps):
                b = i % 2
                if i + 1 < nsteps:
                    copy_in(i + 1)
                stream.wait_event(ev_in[b])   # (its outputs of step i - 2 were copied out before: same copy stream)
                step(k=dk[b], v=dv[b], q=dq[b], out=do[b])
                ev_done[b].record(stream)
                with torch.cuda.stream(cs):
                    cs.wait_event(ev_done[b])
                    ho[b].copy_(do[b], non_blocking=True)
            stream.wait_stream(cs)

        run(args.warmup)
        torch.cuda.synchronize(dev)
        if dist:
            tdist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run(args.steps)
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks([a.elapsed_time(b)], dev)[0]
        # every step computes the same outputs: the last one read back equals
        # the device-timed run's, bit for bit
        assert torch.equal(ho[(args.steps - 1) % 2], outs.cpu()), "end-to-end outputs differ"
        e2e = {"value": weak_scaling_rate(world, B, args.steps, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": "inputs of step s + 1 copied in and outputs of step s read back during compute"}
    cache.check()

    ms_step = elapsed_ms / args.steps
    value = weak_scaling_rate(world, B, args.steps, elapsed_ms)
    dec_ms_call = dec_ms / (args.steps * ncalls)
    achieved = step_decode_bytes * args.steps / (dec_ms / 1e3) / 1e9
    peak, peak_kind = _peaks()
    bf16_bytes = None
    res = {
        "metric": "decode-attention tokens/s (" + ("BF16 cache" if args.bf16 else "INT4 anchor/INT2 resid") + ")",
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("u4/u2 codes, int32 dp4a/dp2a dot products, fp32 softmax" if not args.bf16
                  else "bf16 in, fp32 math"),
        "data": "synthetic (seeded; anchor N(0,1) with 4 outlier channels x10, loops c*anchor+sigma*N(0,1))",
        "config": dict(workload_config(name, cfgd, layers, world), **{
                   "paged": "128-token blocks, shuffled pool" if args.paged else None,
                   "reference": "chained (previous loop)" if args.chained else "shared (last loop)",
                   "step_calls": ("rq_append + rq_decode_attn_bf16" if args.bf16 else
                                  "rq_append + rq_decode_attn" if args.separate_append else "rq_append_decode_attn"),
                   "l2": "inputs larger than L2: %.1f GB of records read per step, loop-major over %d layers"
                         % (step_decode_bytes / 1e9, layers)}),
        "decode_attn": {"ms_per_step": round(dec_ms / args.steps, 4), "us_per_call": round(dec_ms_call * 1e3, 3),
                        "timing": "CUDA events around a graph of the timed steps' decode calls only",
                        "bytes_per_step": int(step_decode_bytes), "gbs": round(achieved, 1),
                        "tokens_per_s_decode_only": round(world * B * args.steps / (dec_ms / 1e3), 2)},
        "append": {"ms_per_step_est": round(max(ms_step - dec_ms / args.steps, 0.0), 4)},
        # records each loop's decode reads per token-head and K|V side: the anchor alone,
        # or the anchor and residuals (one for the shared reference, the chain for the other)
        "records_read_per_loop": [1 if args.bf16 else lp % Lg + 1 if args.chained else 2 if lp % Lg < Lg - 1 else 1
                                  for lp in range(loops)],
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": measured_traffic(name) if not args.bf16 else None,
                     "algorithmic_bytes_per_launch": int(step_decode_bytes / ncalls),
                     "kernel": "rq_decode_attn call (split kernel + combine)", "peak_kind": peak_kind},
        "e2e": e2e,
        # per (layer, loop): the fused call is one kernel for a non-anchor loop and the encoder +
        # decode kernel at the anchor loop; separate calls add the tail-copy kernel; the BF16
        # path is store + decode + combine
        "gpu_launches": int(args.steps * layers * (3 * loops if args.bf16 else
                                                    2 * loops if args.separate_append else loops + groups)),
        "clocks": clocks,
    }
    return res, cache, call_bytes


# ---------------------------------------------------------------- cpu baseline (oracle)
class OracleUnits:
    """Records of a few (sequence, kv head) units at full T, encoded by the
    oracle from CPU-generated synthetic inputs (setup, untimed)."""

    def __init__(self, cfgd, seed, n_units: int, T: int | None = None):
        import torch
        import synth
        from oracle import oracle as orc
        from concurrent.futures import ThreadPoolExecutor
        self.cfgd, self.T = cfgd, T or cfgd["T"]
        Lg = cfgd["Lg"]
        inputs = []
        for u in range(n_units):
            Kg, Vg = synth.group_kv(seed + u, 0, 0, Lg, cfgd["sigma"], 1, self.T, 1, device="cpu")
            xs = [np.stack([synth.bf16_to_u16(X[j]).reshape(-1, 128) for j in range(Lg)]) for X in (Kg, Vg)]
            q = torch.randn((1, 1, 128), generator=torch.Generator().manual_seed(seed + u)).to(torch.bfloat16)
            inputs.append((xs, orc.bf16_bits_to_f64(synth.bf16_to_u16(q))))
        # encode the units' records concurrently (the oracle's C calls release the interpreter lock)
        with ThreadPoolExecutor(max_workers=2 * n_units) as ex:
            recs = list(ex.map(lambda x: orc.encode(x, cfgd["g"], cfgd["ba"], cfgd["br"], True, 0xA11CE),
                               [x for xs, _ in inputs for x in xs]))
        self.units = [(recs[2 * u:2 * u + 2], inputs[u][1]) for u in range(n_units)]

    def decode_seconds(self, u: int, loop: int) -> float:
        """One decode call of one unit, timed: reconstruct the loop's K and V
        from its two reads (anchor + the loop's residual; the anchor alone for
        the anchor loop) and run the direct fp64 softmax."""
        from oracle import oracle as orc
        c = self.cfgd
        Lg = c["Lg"]
        recs, qf = self.units[u % len(self.units)]
        t0 = time.perf_counter()
        kv = []
        for e in recs:
            if loop == Lg - 1:
                x = orc.reconstruct(e.a_codes, e.a_meta, None, None, None, 1, 128, c["g"], c["ba"], c["br"], True,
                                    0xA11CE)[0]
            else:
                x = orc.reconstruct(e.a_codes, e.a_meta, e.r_codes[loop:loop + 1], e.r_meta[loop:loop + 1],
                                    e.r_coef[loop:loop + 1], 2, 128, c["g"], c["ba"], c["br"], True, 0xA11CE)[0]
            kv.append(x)
        orc.attention(qf, kv[0][None, :, None, :], kv[1][None, :, None, :], 1 / math.sqrt(128))
        return time.perf_counter() - t0


def calls_per_step(cfgd) -> int:
    return cfgd["layers"] * cfgd["loops"] * cfgd["B"] * cfgd["H"]   # (unit, loop) decodes per step


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_round(ou: "OracleUnits", threads: int, first: int) -> float:
    """Wall seconds of `threads` unit-loop decodes run at once, one per host
    thread (the oracle's C calls release the interpreter lock): unit-loop i
    is unit i // Lg, loop i % Lg, for i = first .. first + threads - 1."""
    from concurrent.futures import ThreadPoolExecutor
    Lg = ou.cfgd["Lg"]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda i: ou.decode_seconds(i // Lg, i % Lg), range(first, first + threads)))
    return time.perf_counter() - t0


def cpu_baseline(cfgd, seed, budget_s: float = 15.0):
    """The oracle as it stands on all host cores, on a bounded sample of the
    workload: rounds of one unit-loop decode per core ((sequence, kv head)
    units at full T, every loop in turn), scaled to a decode step."""
    threads = host_cores()
    ou = OracleUnits(cfgd, seed, min(4, threads))
    Lg = cfgd["Lg"]
    walls, done, t_start = [], 0, time.perf_counter()
    while time.perf_counter() - t_start < budget_s or done < Lg:
        walls.append(oracle_round(ou, threads, done))
        done += threads
        if len(walls) >= 64:
            break
    rate = done / sum(walls)                      # unit-loop decodes per second, all cores
    step_s = calls_per_step(cfgd) / rate
    return {"value": round(cfgd["B"] / step_s, 6), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} unit-loop decodes in {len(walls)} round(s) of {threads} concurrent ones (one per "
                      f"host core; {len(ou.units)} distinct (sequence, kv head) units at T={cfgd['T']}, all {Lg} loops "
                      f"in turn; reconstruct from records + fp64 softmax), {sum(walls):.1f} s, scaled to "
                      f"{calls_per_step(cfgd)} unit-loops per decode step (extrapolated)"}


def workload_config(name: str, cfgd, layers: int, world: int) -> dict:
    """The `config` keys both arms report for a workload."""
    return {"workload": name, "layers": layers, "loops": cfgd["loops"], "loops_per_group": cfgd["Lg"],
            "batch": cfgd["B"], "seq_len": cfgd["T"], "kv_heads": cfgd["H"], "q_heads": cfgd["Hq"], "head_dim": 128,
            "group": cfgd["g"], "anchor_bits": cfgd["ba"], "resid_bits": cfgd["br"],
            "parallelism": f"replicas x{world}"}


def run_reference(args, cfgd):
    """The oracle, timed as it stands on all host cores: each step is a
    bounded sample -- one round of unit-loop decodes, one per host core
    ((sequence, kv head) units at full T, loops in turn; reconstruct from
    records + direct fp64 softmax) -- scaled to the workload's decode step."""
    seed = CONFIG_SEED[args.config]
    threads = host_cores()
    ou = OracleUnits(cfgd, seed, min(4, threads))
    for w in range(args.warmup):
        oracle_round(ou, threads, w * threads)
    walls = [oracle_round(ou, threads, (args.warmup + s) * threads) for s in range(args.steps)]
    rate = threads * args.steps / sum(walls)
    step_s = calls_per_step(cfgd) / rate
    value = cfgd["B"] / step_s
    sample = (f"per step: {threads} concurrent unit-loop decodes (one per host core, loops in turn) at "
              f"T={cfgd['T']} (oracle reconstruct + fp64 softmax, {np.mean(walls):.3f} s per round), scaled to "
              f"{calls_per_step(cfgd)} unit-loops per decode step")
    return {
        "impl": "reference",
        "metric": "decode-attention tokens/s (INT4 anchor/INT2 resid)",
        "value": round(value, 6), "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, CPU generator)",
        "config": dict(workload_config(args.config, cfgd, cfgd["layers"], int(os.environ.get("WORLD_SIZE", "1"))),
                       host=f"the oracle on {threads} host cores (rank 0)"),
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- batch / format sweep
SWEEP_FORMATS = [
    # name, (group, anchor bits, residual bits, rotate) or None for the BF16 cache
    ("mixed_g16", (16, 4, 2, True)),
    ("mixed_g32", (32, 4, 2, True)),
    ("mixed_g16_rotation_off", (16, 4, 2, False)),
    ("uniform_int2_g16", (16, 2, 2, True)),
    ("bf16", None),
]


def run_sweep(args):
    """Ouro-1.4B shape at T = 8192: for each format, batch 1, 2, 4, ... up
    to the largest power of two whose 24-layer cache fits in free device
    memory (at most 128).  Each row times the decode calls of one filled
    layer (every layer issues the same calls) and scales to the 24 x 4 calls
    of a decode step: tokens/s = batch / step time; GB/s over the calls'
    algorithmic bytes."""
    import torch
    import decode_attention_14_b200 as rq
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = CONFIGS["ouro8k_b4"]
    loops, Lg, T, H, Hq, layers = base["loops"], base["Lg"], base["T"], base["H"], base["Hq"], base["layers"]
    peak, peak_kind = _peaks()
    reps = 20
    rows = []
    for name, fmt in SWEEP_FORMATS:
        kw = dict(num_layers=layers, num_loops=loops, loops_per_group=Lg, max_tokens=T, max_tail_tokens=FILL_CHUNK,
                  num_kv_heads=H, num_q_heads=Hq, seed=0xA11CE)
        if fmt is None:
            kw.update(format=rq.RQ_FMT_BF16)
        else:
            kw.update(group_size=fmt[0], anchor_bits=fmt[1], resid_bits=fmt[2], rotate=fmt[3])
        free, _ = torch.cuda.mem_get_info(dev)
        token_bytes = rq.rq_cache_token_bytes(rq.make_config(batch=1, **kw))
        bf16_token_bytes = rq.rq_cache_token_bytes(rq.make_config(batch=1, **dict(kw, format=rq.RQ_FMT_BF16)))
        # the largest batch whose full cache (24 layers, a decode-time tail of
        # 8 tokens per loop) fits in free device memory
        fit = 0
        b = 1
        while b <= 128 and rq.rq_cache_required_bytes(rq.make_config(batch=b, **dict(kw, max_tail_tokens=8))) <= free:
            fit = b
            b *= 2
        b = 1
        while b <= fit:
            cfg = rq.make_config(batch=b, **dict(kw, num_layers=1))
            cache = rq.Cache(cfg, device=dev)
            seed = 0x5EED0005 + b
            for t0 in range(0, T, FILL_CHUNK):
                n = min(FILL_CHUNK, T - t0)
                Kg, Vg = synth.group_kv(seed, 0, 0, Lg, base["sigma"], b, n, H, t0=t0, device=dev)
                for j in range(Lg):
                    cache.append(0, j, Kg[j], Vg[j])
                del Kg, Vg
            torch.cuda.synchronize(dev)
            q = synth.queries(seed, 0, 0, 0, b, Hq, device=dev)
            out = torch.empty((b, Hq, 128), dtype=torch.float32, device=dev)
            fn = rq.rq_decode_attn_bf16 if fmt is None else rq.rq_decode_attn
            us, byt = [], []
            for lp in range(loops):
                for _ in range(3):
                    assert fn(cache.h, 0, lp, q, out, 0.0) == 0
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for _ in range(reps):
                        st = fn(cache.h, 0, lp, q, out, 0.0)
                        if st != 0:
                            raise rq.RQError(st, fn.__name__)
                g.replay()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize(dev)
                us.append(e0.elapsed_time(e1) * 1e3 / reps)
                byt.append(cache.decode_bytes(0, lp))
                del g
            cache.check()
            cache.close()
            step_us = layers * sum(us)
            gbs = sum(byt) / (sum(us) * 1e-6) / 1e9
            row = {"sweep": "ouro8k", "format": name, "batch": b, "seq_len": T,
                   "tokens_per_s": round(b / (step_us * 1e-6), 2), "decode_step_ms": round(step_us / 1e3, 4),
                   "us_per_call": [round(x, 2) for x in us], "gbs": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                   "peak": peak, "peak_kind": peak_kind, "largest_batch_fits": fit,
                   "cache_bytes_per_token": token_bytes, "vs_bf16_bytes": round(token_bytes / bf16_token_bytes, 4),
                   "timing": "CUDA graph of %d calls per loop on one filled layer, scaled to %d layers" % (reps, layers)}
            rows.append(row)
            print(json.dumps(row), flush=True)
            b *= 2
    return rows


def _bf16_peak():
    """Dense BF16 tensor-core peak (TFLOP/s): the measured burst figure, else
    the pool's earlier measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        if "bf16_tflops" in j:
            return float(j["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def prefill_mma_flops(n, G, B, H, T, resid):
    """Tensor-core FLOPs rq_prefill_attn issues.  A CTA takes 64 query rows
    and steps over 32 committed tokens at a time: 9 logit MMAs of 64x32x16
    and 2 value MMAs of 128x136x16 (the probabilities' high and low parts
    stacked) on the anchor side, and at a residual loop as many again on the
    residual side with the logit MMAs also at M = 128 (Rq's high and low
    parts stacked).  At a residual loop the n new tokens sit in the BF16
    tail, which the last split takes as anchor-side steps."""
    units = B * H * ((n * G + 63) // 64)
    anchor = 9 * 2 * 64 * 32 * 16 + 2 * 2 * 128 * 136 * 16
    residual = 9 * 2 * 128 * 32 * 16 + 2 * 2 * 128 * 136 * 16
    committed = units * ((T + 31) // 32) * (anchor + (residual if resid else 0))
    tail = units * ((n + 31) // 32) * anchor if resid else 0
    return committed + tail


def run_prefill(args):
    """rq_prefill_attn on the Ouro-1.4B-shaped cache (B = 4, T = 8192, H = 16;
    with --paged in 128-token blocks scattered over the pool):
    n new tokens per sequence, timed at a residual loop (the chunk in the BF16
    tail) and at the anchor loop (the chunk committed).  One JSON line per
    (n, loop kind).  FLOPs counted: 2 x 128 for q.k and 2 x 128 for p v per
    (query row, committed token), against the dense BF16 tensor peak; the
    line also gives the tensor FLOPs the kernel issues (hi/lo operand
    splits, minimum columns, rows padded to 64)."""
    import torch
    import decode_attention_14_b200 as rq
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = CONFIGS["ouro8k_b4"]
    loops, Lg, T, H, Hq, B = base["loops"], base["Lg"], base["T"], base["H"], base["Hq"], base["B"]
    reps = 10
    rows = []
    for n in [int(x) for x in args.prefill.split(",")]:
        paging = {}
        if args.paged:   # 128-token blocks, allocation scattered over the pool
            paging = dict(block_tokens=128, num_blocks=B * ((T + n + 127) // 128) + 8)
        cfg = rq.make_config(num_layers=1, num_loops=loops, loops_per_group=Lg, batch=B, max_tokens=T + n,
                             max_tail_tokens=max(FILL_CHUNK, n), num_kv_heads=H, num_q_heads=Hq, seed=0xA11CE,
                             **paging)
        cache = rq.Cache(cfg, device=dev)
        if args.paged:
            cache.shuffle_free_blocks(0x5EED)
        seed = 0x5EED0007 + n
        for t0 in range(0, T, FILL_CHUNK):
            Kg, Vg = synth.group_kv(seed, 0, 0, Lg, base["sigma"], B, FILL_CHUNK, H, t0=t0, device=dev)
            for j in range(Lg):
                cache.append(0, j, Kg[j], Vg[j])
        Kn, Vn = synth.group_kv(seed, 0, 0, Lg, base["sigma"], B, n, H, t0=T, device=dev)
        q = torch.randn((B, n, Hq, 128), generator=torch.Generator(device=dev).manual_seed(seed), device=dev)
        q = q.to(torch.bfloat16)
        out = torch.empty((B, n, Hq, 128), dtype=torch.float32, device=dev)
        for kind in ("residual", "anchor"):
            if kind == "residual":
                cache.append(0, 0, Kn[0], Vn[0])
                loop = 0
            else:
                for j in range(1, Lg):
                    cache.append(0, j, Kn[j], Vn[j])
                loop = Lg - 1
            for _ in range(3):
                assert rq.rq_prefill_attn(cache.h, 0, loop, q, n, out, 0.0) == 0
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(reps):
                    st = rq.rq_prefill_attn(cache.h, 0, loop, q, n, out, 0.0)
                    if st != 0:
                        raise rq.RQError(st, "rq_prefill_attn")
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            us = e0.elapsed_time(e1) * 1e3 / reps
            del g
            committed = T if kind == "residual" else T + n
            flops = 4.0 * 128 * n * Hq * B * committed
            tflops = flops / (us * 1e-6) / 1e12
            mma = prefill_mma_flops(n, Hq // H, B, H, committed, kind == "residual")
            peak, peak_kind = _bf16_peak()
            row = {"prefill": "ouro8k_b4", "n_tokens": n, "loop": kind, "batch": B, "seq_len": committed,
                   "paged": "128-token blocks, shuffled pool" if args.paged else None,
                   "us_per_call": round(us, 1), "query_tokens_per_s": round(B * n / (us * 1e-6), 1),
                   "decode_bytes_per_call": cache.decode_bytes(0, loop),
                   "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak, "unit": "TFLOP/s",
                                "frac": round(tflops / peak, 4), "peak_kind": peak_kind + " dense bf16 (burst)",
                                "achieved_counts": "4 x 128 flops per (query row, committed token)",
                                "mma_tflops": round(mma / (us * 1e-6) / 1e12, 2),
                                "mma_flops_per_call": mma},
                   "timing": "CUDA graph of %d calls (attention kernel + split combine), CUDA events" % reps}
            rows.append(row)
            print(json.dumps(row), flush=True)
        cache.check()
        cache.close()
    return rows


def run_all_configs(args):
    """One JSON line per workload on one GPU, each measured as the headline
    is (same step, timed graph, decode-only graph): the compressed cache and
    the BF16 comparison cache for Ouro 8k b4 and 16k b2/b4, the deep
    recurrence, and the Ouro 8k b4 step on a paged cache and with the
    chained reference."""
    import copy
    runs = [("ouro8k_b4", {}), ("ouro8k_b4", {"bf16": True}), ("long16k_b2", {}), ("long16k_b2", {"bf16": True}),
            ("long16k_b4", {}), ("deep", {}), ("ouro8k_b4", {"paged": True}), ("ouro8k_b4", {"chained": True})]
    for name, flags in runs:
        a = copy.copy(args)
        a.config, a.bf16, a.paged, a.chained = name, False, False, False
        a.no_e2e, a.no_clocks = True, True
        for k, v in flags.items():
            setattr(a, k, v)
        res, cache, _ = run_ours(a, CONFIGS[name], 0, 1, 0)
        print(json.dumps(res), flush=True)
        cache.close()
        del cache
        import torch
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="ouro8k_b4", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--bf16", action="store_true", help="time the uncompressed BF16 comparison kernel")
    ap.add_argument("--separate-append", action="store_true",
                    help="rq_append then rq_decode_attn instead of the fused rq_append_decode_attn")
    ap.add_argument("--layers", type=int, default=0, help="override layer count (profiling runs only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--clocks-csv", default="", help="where the raw nvidia-smi samples go (default: a temp file)")
    ap.add_argument("--json-out", default="")
    ap.add_argument("--sweep", action="store_true",
                    help="batch x format sweep of the Ouro shape at T=8192 (one JSON line per row)")
    ap.add_argument("--prefill", default="",
                    help="comma-separated chunk sizes: time rq_prefill_attn on the Ouro shape instead")
    ap.add_argument("--paged", action="store_true", help="records in a pool of 128-token blocks (block tables)")
    ap.add_argument("--chained", action="store_true",
                    help="the chained (previous-loop) reference of the ablation instead of the shared anchor")
    ap.add_argument("--all-configs", action="store_true",
                    help="one JSON line per workload (Ouro 8k b4, 16k b2/b4, deep; compressed and BF16; paged; "
                         "chained) instead of the single headline line")
    ap.add_argument("--profile", action="store_true",
                    help="bracket the timed region with cudaProfilerStart/Stop (for ncu --profile-from-start off)")
    args = ap.parse_args()
    if args.warmup < 3 and not args.layers:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    cfgd = CONFIGS[args.config]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.sweep:
        run_sweep(args)
        return
    if args.all_configs:
        run_all_configs(args)
        return
    if args.prefill:
        run_prefill(args)
        return
    if args.impl == "reference":
        if rank == 0:
            res = run_reference(args, cfgd)
            print(json.dumps(res))
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    res, cache, _ = run_ours(args, cfgd, rank, world, local_rank)
    if rank == 0 and not args.no_cpu_baseline and not args.layers:
        res["cpu_baseline"] = cpu_baseline(cfgd, CONFIG_SEED[args.config])
    if rank == 0:
        line = json.dumps(res)
        print(line)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(line + "\n")
    cache.close()
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
