#!/usr/bin/env python
"""Throughput of the separator-sparse attention hot path on B200; prints one JSON line.

A step is one pass of every hot-path row over one batch of synthetic input:
  sep_mask_build -> sep_attn_fwd -> sep_attn_bwd on the Pythia-160m training attention shape
  (B=8, H=12/12, L=2048, d=64, a=4, n=64, Geometric(mean 10) separator segments), then
  sepcache_update -> sepcache_decode for one new token of 64 SepCache sequences
  (Hq=32, Hkv=8, d=128, c=800 = 4+64+732, theta=5e5) held at full occupancy.
Each step is one CUDA-graph replay. The metric is kept-pair attention TFLOP/s: FLOPs are
counted on kept (query, key) pairs only (4*d per pair forward, 2.5x that backward, 4*d per
retained slot and query head in decode), summed over the step and divided by its device time.

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
--workload picks a single-row run instead (llama-prefill, long-context, long-context-dense,
decode, ...) for the other configurations; llama-train adds the backward to the Llama-3-8B
prefill shape (a small d = 128 backward case for profiler captures).
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no data-path collective);
time is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "kept-pair attention TFLOP/s fwd/bwd + SepCache decode GB/s, % of B200 roofline"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in self.rows for k in range(4) if r[5 + k] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


# ---------------------------------------------------------------------------- ranks
# Weak scaling: every rank runs the whole step on its own inputs (no data-path collective);
# only the timing is combined, as the max over ranks.
def rank_seed(seed, rank):
    """Seed of a rank's synthetic inputs: the workload's seed for rank 0, distinct per rank."""
    return seed + 1000 * rank


def max_over_ranks(x, device, world):
    """Max of a per-rank float over all ranks (the step time the whole job waits for)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step_per_rank, world, steps, max_ms):
    """Whole-job rate: the units all ranks processed divided by the slowest rank's time."""
    return units_per_step_per_rank * world * steps / (max_ms * 1e-3)


# ---------------------------------------------------------------------------- native arm
class TrainDecodeStep:
    """Buffers and one CUDA graph for the default step (training attention + decode)."""

    def __init__(self, S, dev, rank):
        self.S = S
        cfg = workloads.PYTHIA160M
        self.cfg = cfg
        inp = workloads.attn_inputs(dataclasses.replace(cfg, seed=rank_seed(cfg.seed, rank)))
        self.host = {k: inp[k].pin_memory() for k in ("sep", "q", "k", "v", "do")}
        self.dev = {k: v.to(dev) for k, v in inp.items() if v is not None}
        d = self.dev
        self.mask = S.sep_mask_build(d["sep"], cfg.a, cfg.n)
        self.o, self.lse = S.sep_attn_fwd(d["q"], d["k"], d["v"], self.mask)
        self.ws_f = torch.empty(S.sep_attn_fwd_workspace_size(cfg.B, cfg.L, cfg.Hkv, cfg.d),
                                dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(S.sep_attn_bwd_workspace_size(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d),
                                dtype=torch.uint8, device=dev)
        self.grads = tuple(torch.empty_like(d[x]) for x in ("q", "k", "v"))
        # decode: cache held at full occupancy; a pool of step inputs cycled through
        dc = workloads.SEPCACHE_DECODE
        self.dc = dc
        self.cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, dc.s, dc.w, dc.theta, device=dev)
        fill = dc.c + 100
        dc_r = dataclasses.replace(dc, seed=rank_seed(dc.seed, rank))
        ch = workloads.decode_chunk(dc_r, 0, fill, device=dev)
        for t in range(fill):
            self.cache.sepcache_update(ch["k"][t], ch["v"][t], ch["sep"][t])
        self.pool = workloads.decode_chunk(dc_r, fill, 64, device=dev)
        self.host_dec = {k: v[0].cpu().pin_memory() for k, v in self.pool.items()}
        self.step_in = {k: v[0].clone() for k, v in self.pool.items()}
        self.o_dec = torch.empty_like(self.step_in["q"])
        torch.cuda.synchronize()
        kept = int(self.mask.kept.sum())
        self.kept = kept
        self.flops_fwd = 4.0 * cfg.d * kept * cfg.Hq
        self.flops_bwd = 2.5 * self.flops_fwd
        occ = dc.c
        self.flops_dec = 4.0 * dc.d * occ * dc.Hq * dc.S
        # decode bytes: retained K and V rows, the query and output, the new slot written
        self.bytes_dec = (occ * dc.Hkv * dc.d * 2 * 2 + 2 * dc.Hq * dc.d * 2 + dc.Hkv * dc.d * 2 * 2) * dc.S
        self.flops = self.flops_fwd + self.flops_bwd + self.flops_dec
        self.launches = 11  # mask 2, fwd 2, bwd 5 (prep, schedule, dQ, dK/dV, combine), update 1, decode 1

    def run(self):
        S, d, cfg = self.S, self.dev, self.cfg
        S.sep_mask_build(d["sep"], cfg.a, cfg.n, out=self.mask)
        S.sep_attn_fwd(d["q"], d["k"], d["v"], self.mask, out=self.o, lse=self.lse,
                       workspace=self.ws_f)
        S.sep_attn_bwd(d["q"], d["k"], d["v"], self.o, self.lse, d["do"], self.mask,
                       workspace=self.ws_b, grads=self.grads)
        x = self.step_in
        self.cache.sepcache_update(x["k"], x["v"], x["sep"])
        self.cache.sepcache_decode(x["q"], out=self.o_dec)

    def next_inputs(self, i):
        for k in self.step_in:
            self.step_in[k].copy_(self.pool[k][i % self.pool[k].shape[0]])

    # one-pass components, for the per-kernel breakdown
    def components(self):
        S, d, cfg = self.S, self.dev, self.cfg
        x = self.step_in
        return {
            "mask_build": lambda: S.sep_mask_build(d["sep"], cfg.a, cfg.n, out=self.mask),
            "fwd_compact": lambda: S.sep_attn_fwd(d["q"], d["k"], d["v"], self.mask, out=self.o,
                                                  lse=self.lse, workspace=self.ws_f, stage=0),
            "fwd_kernel": lambda: S.sep_attn_fwd(d["q"], d["k"], d["v"], self.mask, out=self.o,
                                                 lse=self.lse, workspace=self.ws_f, stage=1),
            "bwd_prep": lambda: S.sep_attn_bwd(d["q"], d["k"], d["v"], self.o, self.lse, d["do"],
                                               self.mask, workspace=self.ws_b, grads=self.grads,
                                               stage=0),
            "bwd_dq": lambda: S.sep_attn_bwd(d["q"], d["k"], d["v"], self.o, self.lse, d["do"],
                                             self.mask, workspace=self.ws_b, grads=self.grads,
                                             stage=1),
            "bwd_dkdv": lambda: S.sep_attn_bwd(d["q"], d["k"], d["v"], self.o, self.lse, d["do"],
                                               self.mask, workspace=self.ws_b, grads=self.grads,
                                               stage=2),
            "decode_update": lambda: self.cache.sepcache_update(x["k"], x["v"], x["sep"]),
            "decode_attention": lambda: self.cache.sepcache_decode(x["q"], out=self.o_dec),
        }


def capture(fn, reps=1):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the launch path outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def flush_l2(buf):
    buf.add_(1)  # writes a buffer larger than L2


def time_graph(g, iters, flush):
    """Average device time of one replay (CUDA events on the replay stream), L2 flushed between."""
    times = []
    st = torch.cuda.current_stream()
    for _ in range(iters):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        g.replay()
        e1.record(st)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.mean(times)


def native(args, rank, world, dev):
    from kv_cache_compression_sep_b200 import sepattn as S
    peaks, peak_src = load_peaks()
    flush = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    step = TrainDecodeStep(S, dev, rank)
    graph = capture(step.run)
    assert S.sep_last_device_error() == 0

    # clocks sampled from the warm-up on, through the timed steps and the per-pass rows
    clk = ClockSampler(dev.index).__enter__()
    try:
        for i in range(args.warmup):
            flush_l2(flush)
            graph.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        torch.cuda.nvtx.range_push("timed")
        for i in range(args.steps):
            flush_l2(flush)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        max_ms = max_over_ranks(sum(step_ms), dev, world)
        value = job_throughput(step.flops, world, args.steps, max_ms) / 1e12
        assert S.sep_last_device_error() == 0

        if args.quick:  # timed step only (used under ncu)
            clk.__exit__(None, None, None)
            return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                    "steps": args.steps, "ms_per_step": max_ms / args.steps, "quick": True}
        # ---- end to end through the public API: host inputs in pinned memory, copies timed
        e2e = e2e_run(step, args, dev, world)

        # ---- per-kernel breakdown (each pass alone, CUDA-graph replays of 20 launches)
        comps = {}
        for name, fn in step.components().items():
            g = capture(fn, reps=20)
            comps[name] = time_graph(g, 5, flush) / 20.0
            del g
        # the decode row needs the cache at full occupancy: update/decode advance it, which is fine
        comp_out = train_components(step, comps, peaks, peak_src)
        # dominant kernel of the step by device time
        shares = {"fwd_kernel": comps["fwd_kernel"], "bwd_dq": comps["bwd_dq"],
                  "bwd_dkdv": comps["bwd_dkdv"], "decode_attention": comps["decode_attention"]}
        dom = max(shares, key=shares.get)
        roof = roofline_for(dom, comps, step, peaks, peak_src)
        # ---- the other configurations (same kernels), one row each
        configs = {}
        if not args.no_configs and rank == 0:
            configs = config_rows(S, dev, flush, peaks)
    finally:
        clk.__exit__(None, None, None)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, separator flags as configured)",
        "config": step_config(world, "flushed between timed steps (256 MiB write)",
                              "one CUDA graph: mask build, fwd, bwd, cache update, decode"),
        "roofline": roof,
        "components": comp_out,
        "configs": configs,
        "e2e": e2e,
        "gpu_launches": step.launches * args.steps,
        "clocks": {**clk.summary(), "window": "warm-up, timed steps, e2e and per-pass rows"},
        "peaks": {"source": peak_src, **peaks},
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return line


def train_components(step, comps, peaks, peak_src):
    """Per-pass rows of the default step: time, kept-pair TFLOP/s, tensor and combined roofline
    fractions, and the pair slots the kernels compute per kept pair."""
    cfg = step.cfg
    slots = pair_slots(step.mask.gather_end.cpu(), cfg.L, cfg.n)
    slots_fwd = pair_slots(step.mask.gather_end.cpu(), cfg.L, cfg.n,
                           step.mask.anchor_bits.cpu().numpy())
    computed_over_kept = slots / step.kept
    rows = {}
    for name, flops, sl in (("fwd_kernel", step.flops_fwd, slots_fwd),
                            ("bwd_dq", 1.5 * step.flops_fwd, slots_fwd),
                            ("bwd_dkdv", 2.0 * step.flops_fwd, slots)):
        r = roofline_for(name, comps, step, peaks, peak_src)
        rows[name] = {"us": comps[name] * 1e3, "tflops": r["achieved"], "frac_bf16_peak": r["frac"],
                      "algorithmic_flops": flops, "algorithmic_bytes": r["algorithmic_bytes_per_launch"],
                      "combined_frac": r["combined_frac"], "combined_bound": r["combined_bound"],
                      "computed_pairs_over_kept": sl / step.kept}
    bwd_ms = comps["bwd_prep"] + comps["bwd_dq"] + comps["bwd_dkdv"]
    dec = roofline_for("decode_attention", comps, step, peaks, peak_src)
    return {
        "mask_build_us": comps["mask_build"] * 1e3,
        "fwd": {"us": (comps["fwd_compact"] + comps["fwd_kernel"]) * 1e3,
                "compact_us": comps["fwd_compact"] * 1e3, **rows["fwd_kernel"]},
        "bwd": {"us": bwd_ms * 1e3, "prep_us": comps["bwd_prep"] * 1e3,
                "tflops": step.flops_bwd / (bwd_ms * 1e-3) / 1e12,
                "frac_bf16_peak": step.flops_bwd / (bwd_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "dq": rows["bwd_dq"], "dkdv": rows["bwd_dkdv"]},
        "decode": {"update_us": comps["decode_update"] * 1e3,
                   "attention_us": comps["decode_attention"] * 1e3,
                   "gbs": dec["achieved"], "frac_hbm": dec["frac"],
                   "algorithmic_bytes": step.bytes_dec},
        "kept_pairs": step.kept,
        "kept_over_dense_causal": step.kept / (cfg.B * cfg.L * (cfg.L + 1) / 2),
        "computed_pairs_over_kept": computed_over_kept,
    }


def device_attn_inputs(cfg, dev, n=None, with_do=True):
    """A configuration's inputs drawn on the device generator (seeded; the same distributions
    and flag recipe as workloads.attn_inputs, which draws on the CPU for the parity tests)."""
    g = torch.Generator(device=dev).manual_seed(cfg.seed)
    if cfg.flags == "bernoulli":
        sep = (torch.rand(cfg.B, cfg.L, generator=g, device=dev) < cfg.p).to(torch.uint8)
    else:
        sep = workloads.separator_flags(torch.Generator().manual_seed(cfg.seed), cfg.B, cfg.L,
                                        cfg.flags, cfg.p).to(dev)
    if cfg.force0:
        sep[:, 0] = 0

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    q = randn(cfg.B, cfg.L, cfg.Hq, cfg.d)
    k = randn(cfg.B, cfg.L, cfg.Hkv, cfg.d)
    v = randn(cfg.B, cfg.L, cfg.Hkv, cfg.d)
    do = randn(cfg.B, cfg.L, cfg.Hq, cfg.d) if with_do else None
    return dict(sep=sep, q=q, k=k, v=v, do=do)


def attn_row(S, cfg, dev, flush, peaks, n, bwd, iters):
    """Forward (and backward) of one attention configuration: device time per call, kept-pair
    TFLOP/s, tensor and combined roofline fractions, computed pair slots per kept pair."""
    d = device_attn_inputs(cfg, dev, with_do=bwd)
    mask = S.sep_mask_build(d["sep"], cfg.a, n)
    o, lse = S.sep_attn_fwd(d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    kept = int(mask.kept.sum())
    fl = 4.0 * cfg.d * kept * cfg.Hq
    slots = pair_slots(mask.gather_end.cpu(), cfg.L, n, mask.anchor_bits.cpu().numpy())
    ws = torch.empty(S.sep_attn_fwd_workspace_size(cfg.B, cfg.L, cfg.Hkv, cfg.d),
                     dtype=torch.uint8, device=dev)
    g = capture(lambda: S.sep_attn_fwd(d["q"], d["k"], d["v"], mask, out=o, lse=lse,
                                       workspace=ws))
    ms = time_graph(g, iters, flush)
    del g
    fb = attn_pass_bytes(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d, "fwd_kernel")
    t_f = max(fl / (peaks["bf16_tflops"] * 1e12), fb / (peaks["hbm_gbs"] * 1e9))
    row = {"B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "L": cfg.L, "d": cfg.d, "a": cfg.a, "n": n,
           "kept_pairs": kept, "kept_over_dense_causal": kept / (cfg.B * cfg.L * (cfg.L + 1) / 2),
           "fwd_computed_pairs_over_kept": slots / kept,
           "fwd_ms": ms, "fwd_tflops": fl / (ms * 1e-3) / 1e12,
           "fwd_frac_bf16_peak": fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "fwd_combined_frac": t_f / (ms * 1e-3)}
    if bwd:
        wsb = torch.empty(S.sep_attn_bwd_workspace_size(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d),
                          dtype=torch.uint8, device=dev)
        grads = tuple(torch.empty_like(d[x]) for x in ("q", "k", "v"))
        g = capture(lambda: S.sep_attn_bwd(d["q"], d["k"], d["v"], o, lse, d["do"], mask,
                                           workspace=wsb, grads=grads))
        ms = time_graph(g, iters, flush)
        del g, wsb, grads
        row.update({"bwd_ms": ms, "bwd_tflops": 2.5 * fl / (ms * 1e-3) / 1e12,
                    "bwd_frac_bf16_peak": 2.5 * fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"]})
    assert S.sep_last_device_error() == 0
    return row


def decode_loop_row(S, dev, peaks, first=2048, steps=63488, chunk=1024):
    """The SepCache decode configuration as a stream: 64 sequences, steps first..first+steps-1
    of the 65536-step run (the cache is full from then on), update + decode per step, chunk
    steps per CUDA-graph replay on the device-drawn input stream; steps run back to back."""
    dc = workloads.SEPCACHE_DECODE
    cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, dc.s, dc.w, dc.theta, device=dev)
    o = torch.empty(dc.S, dc.Hq, dc.d, dtype=torch.bfloat16, device=dev)
    # steps 0 .. first - chunk - 1 directly, the chunk before `first` through the capture's own
    # warm-up call, then the timed chunks replay the graph on their inputs
    for c0 in range(0, first - chunk, chunk):
        x = workloads.decode_chunk(dc, c0, chunk, device=dev)
        for t in range(chunk):
            cache.sepcache_update(x["k"][t], x["v"][t], x["sep"][t])
            cache.sepcache_decode(x["q"][t], out=o)
    buf = workloads.decode_chunk(dc, first - chunk, chunk, device=dev)

    def run():
        for t in range(chunk):
            cache.sepcache_update(buf["k"][t], buf["v"][t], buf["sep"][t])
            cache.sepcache_decode(buf["q"][t], out=o)
    g = capture(run)
    m = cache.meta.cpu()
    occ = (m[:, 1] + m[:, 3] + m[:, 5]).tolist()
    full = all(v == dc.c for v in occ)
    total_ms = 0.0
    st = torch.cuda.current_stream()
    for c0 in range(first, first + steps, chunk):
        x = workloads.decode_chunk(dc, c0, chunk, device=dev)
        for key in buf:
            buf[key].copy_(x[key])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        g.replay()
        e1.record(st)
        e1.synchronize()
        total_ms += e0.elapsed_time(e1)
    assert S.sep_last_device_error() == 0
    us = total_ms * 1e3 / steps
    byts = dc.S * (dc.c * dc.Hkv * dc.d * 2 * 2 + 2 * dc.Hq * dc.d * 2 + dc.Hkv * dc.d * 2 * 2)
    return {"sequences": dc.S, "steps_timed": steps, "first_step": first, "occupancy": dc.c,
            "cache_full_at_first_step": full, "us_per_step": us,
            "tokens_per_s": dc.S / (us * 1e-6), "bytes_per_step": byts,
            "gbs": byts / (us * 1e-6) / 1e9, "frac_hbm": byts / (us * 1e-6) / 1e9 / peaks["hbm_gbs"],
            "l2": "steps back to back (the 210 MB cache exceeds the 126 MB L2)"}


def config_rows(S, dev, flush, peaks):
    """The other configurations through the same kernels, one row each."""
    rows = {}
    rows["llama3-8b-prefill"] = attn_row(S, workloads.LLAMA3_8B_PREFILL, dev, flush, peaks,
                                         workloads.LLAMA3_8B_PREFILL.n, False, 10)
    torch.cuda.empty_cache()
    lc = workloads.LONG_CONTEXT
    rows["long-context"] = attn_row(S, lc, dev, flush, peaks, lc.n, True, 3)
    torch.cuda.empty_cache()
    rows["long-context-all-keep"] = attn_row(S, lc, dev, flush, peaks, lc.L, True, 2)
    torch.cuda.empty_cache()
    rows["sepcache-decode-stream"] = decode_loop_row(S, dev, peaks)
    torch.cuda.empty_cache()
    for r in rows.values():
        r["inputs"] = "seeded, drawn on the device generator"
    return rows


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "dram_traffic.json")
CSRC = os.path.join(ROOT, "kv_cache_compression_sep_b200", "csrc")


def source_digest(fname):
    """sha256 (first 16 hex digits) of one kernel source file of the library."""
    import hashlib
    with open(os.path.join(CSRC, fname), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def load_traffic(name):
    """DRAM bytes per launch of a pass (dram__bytes_read.sum + dram__bytes_write.sum) from the
    committed ncu capture table, or None when no capture covers the pass or the kernel's source
    file changed after the capture (the counters then describe another kernel)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    with open(TRAFFIC_JSON) as fh:
        table = json.load(fh)
    e = table.get("passes", {}).get(name)
    if not e:
        return None
    try:
        if source_digest(e["source"]) != e["source_sha256"]:
            return None
    except OSError:
        return None
    return int(e["bytes_per_launch"])


def attn_pass_bytes(B, L, Hq, Hkv, d, name):
    """Algorithmic HBM bytes of one attention pass: every input read once, every output written
    once (bf16 tensors, fp32 LSE and Delta); scratch traffic is not counted."""
    q = B * L * Hq * d * 2
    kv = B * L * Hkv * d * 2
    st = B * Hq * L * 4
    return {"fwd_kernel": q + 2 * kv + q + st,             # Q, K, V -> O, LSE
            "bwd_dq": 2 * q + 2 * kv + 2 * st + q,         # Q, dO, K, V, LSE, Delta -> dQ
            "bwd_dkdv": 2 * q + 2 * kv + 2 * st + 2 * kv}[name]  # ... -> dK, dV


def pair_slots(gather_end, L, n, anchor_bits=None):
    """Query-key pair slots the attention kernels compute per head (summed over the batch):
    every query tile t runs whole 128 x 128 tiles over its window key tiles lo(t)..t and over
    ceil(gather_end[t] / 128) compacted anchor chunks (the dK/dV pass, which visits these
    (query tile, key unit) pairs key-major).
    With anchor_bits ([B, W] anchor flags), the count of the forward and dQ passes: a query
    tile whose oldest
    window tile's lower 64 keys lie outside every row's band (128 t - n + 1 >= 128 lo + 64)
    gathers their anchors too (G = gather_end + their count), and the first 64 gathered anchors
    fill that half of the tile, so ceil(max(0, G - 64) / 128) chunks follow."""
    import numpy as np
    ge = np.asarray(gather_end, dtype=np.int64)
    T = ge.shape[-1]
    t = np.arange(T)
    lo = np.maximum(0, 128 * t - n + 1) // 128
    chunks = (ge + 127) // 128
    if anchor_bits is not None:
        half = (lo < t) & (128 * t - n + 1 >= 128 * lo + 64)
        bits = np.asarray(anchor_bits).astype(np.int64) & 0xFFFFFFFF
        w0 = np.minimum(4 * lo, bits.shape[-1] - 1)
        w1 = np.minimum(4 * lo + 1, bits.shape[-1] - 1)

        def popc(x):
            return np.array([[bin(int(v)).count("1") for v in row] for row in x], dtype=np.int64)

        extra = popc(bits[:, w0]) + popc(bits[:, w1])
        g = ge + extra * half[None, :]
        chunks = np.where(half[None, :], (np.maximum(0, g - 64) + 127) // 128, chunks)
    tiles = (t - lo + 1)[None, :] + chunks
    return int(tiles.sum()) * 128 * 128


def roofline_for(name, comps, step, peaks, peak_src):
    ms = comps[name]
    traffic = load_traffic(name)
    if name == "decode_attention":
        ach = step.bytes_dec / (ms * 1e-3) / 1e9
        return {"kernel": "sepcache_decode_kernel", "bound": "hbm", "achieved": ach,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                "traffic": traffic, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": step.bytes_dec}
    flops = {"fwd_kernel": step.flops_fwd, "bwd_dq": 1.5 * step.flops_fwd,
             "bwd_dkdv": 2.0 * step.flops_fwd}[name]
    kname = {"fwd_kernel": "sep_attn_fwd_kernel", "bwd_dq": "sep_attn_bwd_dq_kernel",
             "bwd_dkdv": "sep_attn_bwd_dkv_kernel"}[name]
    ach = flops / (ms * 1e-3) / 1e12
    out = {"kernel": kname, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
           "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"], "traffic": traffic,
           "peak_source": peak_src, "algorithmic_flops_per_launch": flops}
    cfg = getattr(step, "cfg", None)
    if cfg is not None:
        byts = attn_pass_bytes(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d, name)
        t_min = max(flops / (peaks["bf16_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9))
        out.update({"algorithmic_bytes_per_launch": byts,
                    "combined_frac": t_min / (ms * 1e-3),
                    "combined_bound": "hbm" if byts / (peaks["hbm_gbs"] * 1e9) >
                    flops / (peaks["bf16_tflops"] * 1e12) else "tensor"})
    return out


def e2e_run(step, args, dev, world):
    """Same step through the public API with host buffers: every step copies its inputs in from
    pinned host memory and its results (dQ, dK, dV and the decode output) back out, all inside
    the timed region. The copies of neighbouring steps overlap the compute: step k+1's inputs
    go in on one stream and step k-1's results come out on another while step k computes on a
    third (device inputs and outputs double-buffered)."""
    S, cfg = step.S, step.cfg
    h, hd = step.host, step.host_dec
    x_in = [({k: torch.empty_like(step.dev[k]) for k in h},
             {k: torch.empty_like(step.step_in[k]) for k in hd}) for _ in range(2)]
    y_dev = [tuple(torch.empty_like(g) for g in step.grads) + (torch.empty_like(step.o_dec),)
             for _ in range(2)]
    y_host = [tuple(torch.empty_like(t, device="cpu").pin_memory() for t in y) for y in y_dev]
    h2d = sum(t.numel() * t.element_size() for t in list(h.values()) + list(hd.values()))
    d2h = sum(t.numel() * t.element_size() for t in y_host[0])
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def compute(b):
        xa, xd = x_in[b]
        dq, dk, dv, od = y_dev[b]
        S.sep_mask_build(xa["sep"], cfg.a, cfg.n, out=step.mask)
        S.sep_attn_fwd(xa["q"], xa["k"], xa["v"], step.mask, out=step.o, lse=step.lse,
                       workspace=step.ws_f)
        S.sep_attn_bwd(xa["q"], xa["k"], xa["v"], step.o, step.lse, xa["do"], step.mask,
                       workspace=step.ws_b, grads=(dq, dk, dv))
        step.cache.sepcache_update(xd["k"], xd["v"], xd["sep"])
        step.cache.sepcache_decode(xd["q"], out=od)

    def pipeline(n, e_start=None, e_end=None):
        started = [False, False]
        for i in range(n + 2):
            if i < n:  # inputs of step i into buffer i % 2, once step i-2 has finished with it
                b = i % 2
                with torch.cuda.stream(s_in):
                    if started[b]:
                        s_in.wait_event(comp_done[b])
                    if i == 0 and e_start is not None:
                        e_start.record(s_in)
                    for k in h:
                        x_in[b][0][k].copy_(h[k], non_blocking=True)
                    for k in hd:
                        x_in[b][1][k].copy_(hd[k], non_blocking=True)
                    in_done[b].record(s_in)
            if 1 <= i <= n:  # compute step i-1, once its inputs are in and buffer's results out
                b = (i - 1) % 2
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(in_done[b])
                    if started[b]:
                        s_comp.wait_event(out_done[b])
                    compute(b)
                    comp_done[b].record(s_comp)
                started[b] = True
            if i >= 2:  # results of step i-2 out
                b = (i - 2) % 2
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[b])
                    for src, dst in zip(y_dev[b], y_host[b]):
                        dst.copy_(src, non_blocking=True)
                    out_done[b].record(s_out)
        if e_end is not None:
            e_end.record(s_out)

    n = max(3, min(args.steps, 20))
    pipeline(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(n, e0, e1)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / n
    torch.cuda.synchronize()
    ms = max_over_ranks(ms, dev, world)
    return {"value": job_throughput(step.flops, world, 1, ms) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "overlap": "H2D of step k+1 and D2H of step k-1 overlap step k"}


# ---------------------------------------------------------------------------- oracle arm
def oracle_sample(H=4, ndec=4):
    """One bounded sample of the workload on the oracle; returns (kept-pair FLOPs, seconds).

    Sample: forward + backward of query heads 0..H-1 of batch 0 of the Pythia-160m shape (full
    L=2048 masked oracle) and ndec decode steps of one SepCache sequence at full occupancy.
    """
    import numpy as np
    import oracle
    cfg = workloads.PYTHIA160M
    inp = workloads.attn_inputs(cfg)
    q = inp["q"][:1, :, :H].float().numpy()
    k = inp["k"][:1, :, :H].float().numpy()
    v = inp["v"][:1, :, :H].float().numpy()
    do = inp["do"][:1, :, :H].float().numpy()
    sep = inp["sep"][:1].numpy()
    kept = int(oracle.kept_pairs_closed_form(sep, cfg.a, cfg.n)[0])
    dc = workloads.SEPCACHE_DECODE
    rng = np.random.default_rng(0)
    kr = rng.standard_normal((dc.c, dc.Hkv, dc.d))
    vr = rng.standard_normal((dc.c, dc.Hkv, dc.d))
    qd = rng.standard_normal((dc.Hq, dc.d))
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, sep, cfg.a, cfg.n, cfg.scale)
    oracle.attn_bwd(q, k, v, do, sep, cfg.a, cfg.n, cfg.scale)
    for _ in range(ndec):
        oracle.decode_attention(qd, kr, vr, dc.theta, dc.scale)
    dt = time.perf_counter() - t0
    flops = 3.5 * 4.0 * cfg.d * kept * H + ndec * 4.0 * dc.d * dc.c * dc.Hq
    return flops, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((x.get("num_threads", 1) for x in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(seconds):
    flops, dt = 0.0, 0.0
    n = 0
    while dt < seconds or n == 0:
        f, t = oracle_sample()
        flops += f
        dt += t
        n += 1
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "sample": (f"{n} x [fwd+bwd of 4 query heads of batch 0, "
                                          "Pythia-160m shape, full fp64 masked oracle; 4 decode "
                                          "steps of one 800-slot SepCache sequence]"),
            "seconds": dt}


def step_config(world, l2, step):
    """The default step's configuration, shared by both arms (the reference arm runs a sample
    of the same step)."""
    return {"workload": "pythia160m-train-attention + sepcache-decode step",
            "train": {"B": 8, "Hq": 12, "Hkv": 12, "L": 2048, "d": 64, "a": 4, "n": 64,
                      "flags": "geometric(mean 10) segments"},
            "decode": {"S": 64, "Hq": 32, "Hkv": 8, "d": 128, "c": 800, "a": 4, "s": 64,
                       "w": 732, "theta": 5e5, "occupancy": 800},
            "global_batch": 8 * world, "seq_len": 2048, "parallelism": f"dp{world}",
            "l2": l2, "step": step}


def reference(args, rank, world):
    if rank != 0:
        return None
    # sample per step sized so that warm-up + steps stay within a few minutes
    H = max(1, min(4, 120 // max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(H, 1)
    flops, dt = 0.0, 0.0
    for _ in range(args.steps):
        f, t = oracle_sample(H, 1)
        flops += f
        dt += t
    value = flops / dt / 1e12
    cores = blas_threads()
    sample = (f"per step: fwd+bwd of {H} query head(s) of batch 0 (Pythia-160m shape, fp64 "
              "masked oracle) + 1 decode step of one 800-slot SepCache sequence")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(world, "host CPU run (no GPU L2)",
                                  "a bounded sample of the step on the host cores "
                                  "(cpu_baseline.sample)"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------- single rows
def single_row(args, dev):
    """Other configurations, one row at a time (fwd/bwd TFLOP/s or decode GB/s)."""
    from kv_cache_compression_sep_b200 import sepattn as S
    peaks, peak_src = load_peaks()
    flush = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    out = {"workload": args.workload, "peaks": peaks, "peak_source": peak_src}
    if args.workload == "decode":
        step = TrainDecodeStep.__new__(TrainDecodeStep)
        dc = workloads.SEPCACHE_DECODE
        cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, dc.s, dc.w, dc.theta, device=dev)
        pool = workloads.decode_chunk(dc, 0, 1024, device=dev)
        o = torch.empty_like(pool["q"][0])
        for t in range(1024):
            cache.sepcache_update(pool["k"][t], pool["v"][t], pool["sep"][t])
        x = {k: v[0].clone() for k, v in pool.items()}
        g = capture(lambda: (cache.sepcache_update(x["k"], x["v"], x["sep"]),
                             cache.sepcache_decode(x["q"], out=o)), reps=50)
        ms = time_graph(g, args.steps, flush) / 50
        occ = dc.c
        byts = (occ * dc.Hkv * dc.d * 4 + 4 * dc.Hq * dc.d + 4 * dc.Hkv * dc.d) * dc.S
        out.update({"us_per_step": ms * 1e3, "tokens_per_s": dc.S / (ms * 1e-3),
                    "gbs_update_plus_decode": byts / (ms * 1e-3) / 1e9})
        del step
        return out
    if args.workload == "decode-past":
        # SepCache with a Past Window: a=4, s=64, w=256, compressed when the usage reaches
        # c=800; R consecutive steps (distinct inputs) replayed from the same starting state
        dc, R, c_use, w_p = workloads.SEPCACHE_DECODE, 512, 800, 256
        cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, dc.s, w_p, dc.theta, device=dev,
                           c=c_use)
        warm = workloads.decode_chunk(dc, 0, 2048, device=dev)
        for t in range(2048):
            cache.sepcache_update(warm["k"][t], warm["v"][t], warm["sep"][t])
        pool = workloads.decode_chunk(dc, 2048, R, device=dev)
        o = torch.empty_like(pool["q"][0])
        state0 = cache.state_dict()
        occ = []
        for t in range(R):  # untimed pass: the occupancy each step reads
            cache.sepcache_update(pool["k"][t], pool["v"][t], pool["sep"][t])
            cache.sepcache_decode(pool["q"][t], out=o)
            m = cache.meta.cpu()
            occ.append(int((m[:, 1] + m[:, 3] + m[:, 5] + m[:, 6]).sum()))

        def steps():
            for t in range(R):
                cache.sepcache_update(pool["k"][t], pool["v"][t], pool["sep"][t])
                cache.sepcache_decode(pool["q"][t], out=o)
        cache.load_state_dict(state0)
        g = capture(steps)
        times = []
        st = torch.cuda.current_stream()
        for _ in range(max(3, args.steps)):
            cache.load_state_dict(state0)  # also evicts the cache lines of the previous replay
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            g.replay()
            e1.record(st)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.mean(times) / R
        byts = (sum(occ) / R * dc.Hkv * dc.d * 4 + dc.S * (4 * dc.Hq * dc.d + 4 * dc.Hkv * dc.d))
        out.update({"a": dc.a, "s": dc.s, "w": w_p, "c": c_use,
                    "mean_occupancy": sum(occ) / R / dc.S, "us_per_step": ms * 1e3,
                    "tokens_per_s": dc.S / (ms * 1e-3), "gbs_update_plus_decode": byts / (ms * 1e-3) / 1e9})
        return out
    if args.workload == "decode-noshift":
        # training-free use without positional shifting: initial a=4, every separator (s large)
        # and the n=256 neighbours, keys at their original positions; 64 sequences seeded from
        # 8192-token prompts, then steady decode steps
        dc, Lp, n_win, s_all = workloads.SEPCACHE_DECODE, 8192, 256, 2048
        cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, s_all, n_win, dc.theta, device=dev,
                           original_positions=True)
        g0 = torch.Generator(device=dev).manual_seed(dc.seed)
        k = torch.randn(dc.S, Lp, dc.Hkv, dc.d, generator=g0, device=dev).to(torch.bfloat16)
        v = torch.randn(dc.S, Lp, dc.Hkv, dc.d, generator=g0, device=dev).to(torch.bfloat16)
        sep = (torch.rand(dc.S, Lp, generator=g0, device=dev) < dc.p).to(torch.uint8)
        cache.sepcache_prefill(k, v, sep)
        del k, v
        pool = workloads.decode_chunk(dc, 0, 64, device=dev)
        o = torch.empty_like(pool["q"][0])
        x = {kk: vv[0].clone() for kk, vv in pool.items()}
        x["sep"].zero_()  # steady state: the window slides, the separator set stays as prompted
        g = capture(lambda: (cache.sepcache_update(x["k"], x["v"], x["sep"]),
                             cache.sepcache_decode(x["q"], out=o)), reps=50)
        ms = time_graph(g, args.steps, flush) / 50
        m = cache.meta.cpu()
        occ = int((m[:, 1] + m[:, 3] + m[:, 5]).sum())
        T = int(m[:, 0].float().mean())
        byts = occ * dc.Hkv * dc.d * 4 + dc.S * (4 * dc.Hq * dc.d + 4 * dc.Hkv * dc.d)
        out.update({"a": dc.a, "n": n_win, "prompt_len": Lp, "mean_occupancy": occ / dc.S,
                    "r_kv": occ / dc.S / T, "us_per_step": ms * 1e3,
                    "tokens_per_s": dc.S / (ms * 1e-3), "gbs_update_plus_decode": byts / (ms * 1e-3) / 1e9})
        return out
    if args.workload == "cache-prefill":
        # seed 64 caches (the decode configuration's capacities) from 8192-token prompts
        dc, Lp = workloads.SEPCACHE_DECODE, 8192
        cache = S.SepCache(dc.S, dc.Hq, dc.Hkv, dc.d, dc.a, dc.s, dc.w, dc.theta, device=dev)
        g0 = torch.Generator(device=dev).manual_seed(dc.seed)
        k = torch.randn(dc.S, Lp, dc.Hkv, dc.d, generator=g0, device=dev).to(torch.bfloat16)
        v = torch.randn(dc.S, Lp, dc.Hkv, dc.d, generator=g0, device=dev).to(torch.bfloat16)
        sep = (torch.rand(dc.S, Lp, generator=g0, device=dev) < dc.p).to(torch.uint8)
        g = capture(lambda: cache.sepcache_prefill(k, v, sep), reps=20)
        ms = time_graph(g, args.steps, flush) / 20
        occ = int(cache.state_dict()["meta"][:, 1:6:2].sum())  # initial + separators + window
        byts = occ * dc.Hkv * dc.d * 2 * 2 * 2 + dc.S * Lp  # K/V rows read and written, flags
        out.update({"prompt_len": Lp, "us": ms * 1e3, "occupied_slots": occ,
                    "gbs": byts / (ms * 1e-3) / 1e9,
                    "frac_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
        return out
    cfg = {"llama-prefill": workloads.LLAMA3_8B_PREFILL, "llama-train": workloads.LLAMA3_8B_PREFILL,
           "long-context": workloads.LONG_CONTEXT,
           "long-context-dense": workloads.LONG_CONTEXT,
           "pythia-train": workloads.PYTHIA160M}[args.workload]
    n = cfg.L if args.workload == "long-context-dense" else cfg.n
    inp = workloads.attn_inputs(cfg, with_do=args.workload != "llama-prefill")
    d = {k: v.to(dev) for k, v in inp.items() if v is not None}
    mask = S.sep_mask_build(d["sep"], cfg.a, n)
    o, lse = S.sep_attn_fwd(d["q"], d["k"], d["v"], mask)
    torch.cuda.synchronize()
    kept = int(mask.kept.sum())
    fl = 4.0 * cfg.d * kept * cfg.Hq
    ws = torch.empty(S.sep_attn_fwd_workspace_size(cfg.B, cfg.L, cfg.Hkv, cfg.d), dtype=torch.uint8, device=dev)
    g = capture(lambda: S.sep_attn_fwd(d["q"], d["k"], d["v"], mask, out=o, lse=lse, workspace=ws))
    ms = time_graph(g, args.steps, flush)
    out.update({"kept_pairs": kept, "kept_over_dense": kept / (cfg.B * cfg.L * (cfg.L + 1) / 2),
                "fwd_ms": ms, "fwd_tflops": fl / (ms * 1e-3) / 1e12})
    out["fwd_frac"] = out["fwd_tflops"] / peaks["bf16_tflops"]
    if d.get("do") is not None:
        wsb = torch.empty(S.sep_attn_bwd_workspace_size(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.d), dtype=torch.uint8, device=dev)
        grads = tuple(torch.empty_like(d[x]) for x in ("q", "k", "v"))
        g = capture(lambda: S.sep_attn_bwd(d["q"], d["k"], d["v"], o, lse, d["do"], mask,
                                           workspace=wsb, grads=grads))
        ms = time_graph(g, max(3, args.steps // 2), flush)
        out.update({"bwd_ms": ms, "bwd_tflops": 2.5 * fl / (ms * 1e-3) / 1e12})
        out["bwd_frac"] = out["bwd_tflops"] / peaks["bf16_tflops"]
    assert S.sep_last_device_error() == 0
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="train-decode",
                    choices=["train-decode", "pythia-train", "llama-prefill", "llama-train",
                             "long-context",
                             "long-context-dense", "decode", "decode-past", "decode-noshift",
                             "cache-prefill"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the Llama prefill, long-context and decode-stream rows")
    ap.add_argument("--quick", action="store_true",
                    help="timed step only: no e2e, breakdown or CPU baseline (for ncu runs)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        if args.workload != "train-decode":
            line = single_row(args, dev)
        else:
            line = native(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
