#!/usr/bin/env python
"""Benchmark of the Hymba hybrid-head layer hot path on B200.

One step = the whole hot path over one batch of synthetic input:
  * prefill of two consecutive sliding-window layers sharing one K/V (layer 2
    reuses layer 1's K/V), bf16, batch 128, 8192 real tokens + 128 meta tokens,
    window 1024, 1.5B widths (d_model 1600, 25/5 heads, d_inner 3200, state 16):
    the two layers' meta-token caches are computed (batch 1, the meta rows being the
    same in every sequence), then the real rows of both layers are prefilled from them;
    the same prefill without the meta cache is timed beside it for comparison;
  * one decode step of a 32-layer stack at the same widths, batch 128, 8k
    context: global attention in layers 0, 15, 31, window 1024 + 128 meta
    elsewhere, K/V shared by consecutive sliding-window layers, N(0,1) caches.
`value` is prefill throughput in real tokens per second (B * 8192 tokens through
both layers per step, whole job over all ranks); decode tokens/s is reported
beside it.  Inputs are resident in HBM before the timed region; inputs are far
larger than L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own replica (weak scaling, no collective on
the data path) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "hybrid-layer prefill tok/s @B=128,L=8k bf16 + decode tok/s; % of roofline"
UNIT = "tok/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one in_proj launch from an ncu capture of the current kernel
# (dram__bytes_{read,write}.sum of the in_proj launch of `bench.py --case b32`), scaled by
# rows to one producer launch of the headline's concurrent prefill (a batch chunk, 32 x 8192
# = 262,144 real rows); None while the kernel has changed since the last capture.
IN_PROJ_TRAFFIC = 5.53e9
IN_PROJ_TRAFFIC_BASIS = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of the in_proj launch of "
                         "`bench.py --case b32 --branch-chunks 0` (778 MB, 36,864 rows), scaled by rows to one "
                         "launch of the concurrent prefill (a chunk of 32 sequences x 8192 rows)")


def max_over_ranks(vals, device, world: int):
    """This rank's device times -> the slowest rank's, elementwise (one MAX all-reduce)."""
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_rate(units_per_rank_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units every replica processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / (ms / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------------------------
# clocks sampled with nvidia-smi during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except FileNotFoundError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[3]))
            except ValueError:
                pass
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(pw) if pw else None}


# ---------------------------------------------------------------------------------------------
# our path
# ---------------------------------------------------------------------------------------------
BRANCH_CHUNKS = 4  # batch chunks of the concurrent prefill (the two branches side by side)


class Prefill:
    """The two KV-sharing prefill layers of the headline workload.  A step computes the
    two layers' meta-token caches (batch 1: the m meta rows are the same in every sequence,
    Hymba §2.3) and then prefills the B x n real rows of both layers from them.  The
    layers exist twice over the same weights: with the concurrent schedule (the timed step)
    and with the serial one (the per-kernel figures, each kernel alone on the GPU)."""

    def __init__(self, w, dev, branch_chunks=BRANCH_CHUNKS):
        import hybrid_attention_ssm_head_b200 as hy
        import synth
        self.hy = hy
        self.w = w
        self.branch_chunks = branch_chunks
        d = w.dims
        B, L, n = w.batch, w.seq_rows, w.n_tokens
        self.B, self.L, self.n = B, L, n
        self.wts, self.handles, self.handles_serial = [], [], []
        for layer, consumer in ((0, False), (1, True)):
            wt = {k: v.contiguous() for k, v in
                  synth.configs.layer_weights(w, layer, consumer=consumer, device=dev).items()}
            self.wts.append(wt)
            for hs, chunks in ((self.handles, branch_chunks), (self.handles_serial, 0)):
                cfg = hy.make_config(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim_qk, d.d_inner, d.d_state,
                                     d.d_conv, d.rank, w.n_meta, w.window, False, "bf16",
                                     branch_chunks=chunks)
                hs.append(hy.hymba_layer_create(cfg, hy.make_weights(wt)))
        hy.hymba_kv_share_bind(self.handles[1], self.handles[0])
        hy.hymba_kv_share_bind(self.handles_serial[1], self.handles_serial[0])
        m = w.n_meta
        self.m = m
        self.meta_x = synth.configs.meta_tokens(w, device=dev)          # R [m, d]
        self.x = synth.configs.real_rows(w, device=dev).contiguous()     # X [B, n, d]
        self.y1 = torch.empty_like(self.x)
        self.y2 = torch.empty_like(self.x)
        self.k = torch.empty(B, L, d.n_kv_heads * d.head_dim_qk, dtype=torch.bfloat16, device=dev)
        self.v = torch.empty(B, L, d.n_kv_heads * d.head_dim_v, dtype=torch.bfloat16, device=dev)
        self.kv = hy.hymba_kv_seq(self.k.data_ptr(), self.v.data_ptr(), 0, 0, 0)
        # meta caches of the two layers (the consumer's K/V are its producer's)
        self.meta_bufs, self.metas = [], []
        for layer in range(2):
            bufs = dict(h=torch.empty(d.d_inner, d.d_state, dtype=torch.float32, device=dev),
                        conv=torch.empty(d.d_conv - 1, d.d_inner, dtype=torch.bfloat16, device=dev),
                        y=torch.empty(m, d.d_model, dtype=torch.bfloat16, device=dev))
            if layer == 0:
                bufs["k"] = torch.empty(m, d.n_kv_heads * d.head_dim_qk, dtype=torch.bfloat16, device=dev)
                bufs["v"] = torch.empty(m, d.n_kv_heads * d.head_dim_v, dtype=torch.bfloat16, device=dev)
            self.meta_bufs.append(bufs)
            self.metas.append(hy.hymba_meta_cache(
                bufs["k"].data_ptr() if layer == 0 else None, bufs["v"].data_ptr() if layer == 0 else None,
                bufs["h"].data_ptr(), bufs["conv"].data_ptr(), bufs["y"].data_ptr(), 0))
        nb = max(max(hy.hymba_layer_prefill_cached_workspace(h, B, n), hy.hymba_layer_meta_workspace(h))
                 for h in self.handles + self.handles_serial)
        self.ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        self._full = None

    def run(self, stream, x=None, y=None, serial=False):
        """One step: both layers' meta caches, then both layers over the real rows."""
        hy = self.hy
        x = self.x if x is None else x
        y = self.y2 if y is None else y
        hs = self.handles_serial if serial else self.handles
        hy.hymba_layer_meta_precompute(hs[0], self.meta_x, self.metas[0], None, self.ws,
                                       self.ws.numel(), stream)
        hy.hymba_layer_meta_precompute(hs[1], self.meta_bufs[0]["y"], self.metas[1], self.metas[0],
                                       self.ws, self.ws.numel(), stream)
        hy.hymba_layer_prefill_cached(hs[0], self.B, self.n, x, self.y1, self.metas[0], self.kv, None,
                                      None, self.ws, self.ws.numel(), stream)
        hy.hymba_layer_prefill_cached(hs[1], self.B, self.n, self.y1, y, self.metas[1], self.kv, None,
                                      None, self.ws, self.ws.numel(), stream)

    def run_full(self, stream):
        """The same two layers without the meta cache: every sequence's L = m + n rows."""
        hy = self.hy
        if self._full is None:
            import synth
            xf = synth.configs.x_tilde(self.w, device=self.x.device)
            nb = max(hy.hymba_layer_prefill_workspace(h, self.B, self.n) for h in self.handles)
            self._full = dict(x=xf, y1=torch.empty_like(xf), y2=torch.empty_like(xf),
                              ws=torch.empty(nb, dtype=torch.uint8, device=self.x.device))
        f = self._full
        hy.hymba_layer_prefill(self.handles[0], self.B, self.n, f["x"], f["y1"], self.kv, None, None,
                               f["ws"], f["ws"].numel(), stream)
        hy.hymba_layer_prefill(self.handles[1], self.B, self.n, f["y1"], f["y2"], self.kv, None, None,
                               f["ws"], f["ws"].numel(), stream)

    def release_full(self):
        self._full = None

    def flops(self):
        """Algorithmic FLOPs of one step (both layers): the meta rows once and the real rows of
        every sequence; attention counted on visible pairs only."""
        d, w = self.w.dims, self.w
        M = self.B * self.n + self.m
        E, H = d.d_inner, d.n_heads
        meta_pairs = visible_pairs(self.m, w.n_meta, w.window, False)
        real_pairs = visible_pairs(self.L, w.n_meta, w.window, False) - meta_pairs
        f = 0.0
        for consumer in (False, True):
            P = d.in_width(consumer)
            f += 2.0 * M * P * d.d_model                       # in_proj
            f += 2.0 * M * d.xproj_width * E                   # x_proj
            f += 2.0 * M * E * d.rank                          # dt_proj
            f += 2.0 * M * d.d_model * E                       # out_proj
            f += H * 2.0 * (d.head_dim_qk + d.head_dim_v) * (self.B * real_pairs + meta_pairs)  # attention
        return f

    def in_proj_flops(self):
        """Per launch over the real rows: [producer, consumer]."""
        d = self.w.dims
        M = self.B * self.n
        return [2.0 * M * d.in_width(False) * d.d_model, 2.0 * M * d.in_width(True) * d.d_model]


def visible_pairs(L, m, W, is_global):
    tot = 0
    for i in range(L):
        if is_global:
            tot += i + 1
        else:
            tot += min(i + 1, m) + max(0, i - max(m, i - W + 1) + 1)
    return tot


class Decode:
    """One decode step of the 32-layer stack (one new token per sequence)."""

    def __init__(self, w, dev, branch_chunks=BRANCH_CHUNKS):
        import hybrid_attention_ssm_head_b200 as hy
        import synth
        self.hy = hy
        self.w = w
        d = w.dims
        B = w.batch
        self.B = B
        self.pos = w.n_meta + w.n_tokens
        layout = synth.configs.stack_layout(w.n_layers)
        self.layers = []
        for l, (is_global, producer) in enumerate(layout):
            consumer = producer is not None
            wt = {k: v.contiguous() for k, v in
                  synth.configs.layer_weights(w, l, consumer=consumer, device=dev).items()}
            cfg = hy.make_config(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim_qk, d.d_inner, d.d_state,
                                 d.d_conv, d.rank, w.n_meta, w.window, is_global, "bf16",
                                 branch_chunks=branch_chunks)
            h = hy.hymba_layer_create(cfg, hy.make_weights(wt))
            cap = self.pos + 1 if is_global else w.n_meta + w.window
            caches = synth.configs.decode_caches(w, l, cap, consumer, device=dev)
            caches = {k: v.contiguous() for k, v in caches.items()}
            ent = dict(handle=h, wt=wt, caches=caches, is_global=is_global, producer=producer, cap=cap)
            ent["ssm"] = hy.hymba_ssm_cache(caches["ssm"].data_ptr(), caches["conv"].data_ptr())
            if not consumer:
                ent["kvc"] = hy.hymba_kv_cache(caches["k"].data_ptr(), caches["v"].data_ptr(), B, cap, 0)
            else:
                hy.hymba_kv_share_bind(h, self.layers[producer]["handle"])
            self.layers.append(ent)
        self.x = synth.configs.decode_tokens(w, device=dev)
        self.ys = [torch.empty_like(self.x) for _ in range(2)]
        nb = max(hy.hymba_layer_decode_workspace(e["handle"], B, self.pos) for e in self.layers)
        self.ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        self.graph = None

    def run(self, stream, x=None, y_out=None):
        hy = self.hy
        cur = self.x if x is None else x
        for l, e in enumerate(self.layers):
            out = self.ys[l % 2] if (l + 1 < len(self.layers) or y_out is None) else y_out
            kvc = e["kvc"] if e["producer"] is None else self.layers[e["producer"]]["kvc"]
            hy.hymba_layer_decode_step(e["handle"], self.B, self.pos, cur, out, kvc, e["ssm"],
                                       self.ws, self.ws.numel(), stream)
            cur = out
        return cur

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(s)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(torch.cuda.current_stream())
        self.graph = g

    def hbm_bytes(self):
        """Minimum HBM traffic of one decode step (bytes)."""
        d = self.w.dims
        B = self.B
        tot = 0
        for e in self.layers:
            for k, v in e["wt"].items():
                tot += v.numel() * v.element_size()
            tot += 2 * e["caches"]["ssm"].numel() * 4                 # SSM state read + write
            tot += 2 * e["caches"]["conv"].numel() * 2
            if e["is_global"]:
                keys = self.pos + 1
            else:
                keys = self.w.n_meta + self.w.window
            tot += B * d.n_kv_heads * keys * (d.head_dim_qk + d.head_dim_v) * 2  # K/V read
        return tot


MUFU_OPS_PER_CLK_SM = 16  # MUFU (ex2/rcp/lg2) results per clock per SM on sm_100
SCAN_MUFU_PER_CHANNEL_STEP = 16  # the 16 decays exp2(delta A) (the gate SiLU(z) comes precomputed)


def kernel_fractions(pre, dec, prof, dprof, peaks, sm_mhz, sms, layer_calls):
    """Each hot kernel's achieved rate against its bound: algorithmic FLOPs (tensor-bound
    kernels) or bytes (memory-bound kernels) of one layer over the CUDA-event time the
    library's profiler measured for it (summed over a layer's batch chunks; `layer_calls`
    layer prefills were profiled).  The scan is also reported against its MUFU floor (its
    16 MUFU operations per channel-step at the sampled SM clock)."""
    d, w = pre.w.dims, pre.w
    B, L = pre.B, pre.L
    M = B * pre.n  # the prefill's main launches run over the real rows (the meta rows are cached)
    E, H, R, N = d.d_inner, d.n_heads, d.rank, d.d_state
    hbm = peaks.get("hbm_gbs", 6650.0)
    tens = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1400.0))
    pm = {n: ms / layer_calls for n, c, _, ms in prof if c}
    out = {}

    def tensor(name, flops):
        if name in pm:
            a = flops / (pm[name] / 1e3) / 1e12
            out[name] = {"bound": "tensor", "achieved": a, "peak": tens, "unit": "TFLOP/s", "frac": a / tens,
                         "ms": pm[name]}

    def mem(name, nbytes, table=None, extra=None):
        t = (table or pm)
        if name in t:
            a = nbytes / (t[name] / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
                         "ms": t[name]}
            if extra:
                out[name].update(extra)

    fl_in = sum(pre.in_proj_flops()) / 2.0
    tensor("in_proj", fl_in)
    tensor("out_proj", 2.0 * M * d.d_model * E)
    tensor("attention", B * H * 2.0 * (d.head_dim_qk + d.head_dim_v) *
           (visible_pairs(L, w.n_meta, w.window, False) - visible_pairs(w.n_meta, w.n_meta, w.window, False)))
    mem("conv", 2.0 * M * E * 2)
    mem("x_proj", M * E * 2 + M * (R + 2 * N) * 4)
    mem("dt_proj", M * (R + 2 * N) * 4 + M * E * 2)
    mem("fuse", 3.0 * M * E * 2)
    if "scan" in pm and sm_mhz:
        floor_ms = M * E * SCAN_MUFU_PER_CHANNEL_STEP / (MUFU_OPS_PER_CLK_SM * sms * sm_mhz * 1e6) * 1e3
        mem("scan", 4.0 * M * E * 2 + M * 2 * N * 4,
            extra={"mufu_floor_ms": floor_ms, "mufu_frac": floor_ms / pm["scan"]})
    # decode, per layer (the stack's 32 layers averaged)
    dm = {n: ms / c for n, c, _, ms in dprof if c}
    nl = len(dec.layers)
    wbytes = lambda key: sum(e["wt"][key].numel() * e["wt"][key].element_size() for e in dec.layers) / nl  # noqa: E731
    kv_bytes = 0
    for e in dec.layers:
        keys = dec.pos + 1 if e["is_global"] else dec.w.n_meta + dec.w.window
        kv_bytes += dec.B * d.n_kv_heads * keys * (d.head_dim_qk + d.head_dim_v) * 2
    mem("dec_in_proj", wbytes("w_in"), dm)
    mem("dec_out_proj", wbytes("w_out"), dm)
    mem("dec_attention", kv_bytes / nl, dm)
    mem("dec_ssm", 2.0 * dec.B * E * N * 4 + wbytes("w_x") + wbytes("w_dt") + 2.0 * dec.B * (d.d_conv - 1) * E * 2,
        dm)
    return out


def run_ours(args, rank, world, dev):
    import hybrid_attention_ssm_head_b200 as hy
    import synth
    torch.cuda.set_device(dev)
    w3, w4 = synth.configs.CFG3, synth.configs.CFG4
    t_setup = time.time()
    pre = Prefill(w3, dev, branch_chunks=args.branch_chunks)
    # the decode stack in the serial order: the side-by-side decode measured the same step
    # time (5.057 against 5.059 ms), and the serial one gives per-kernel events that are not
    # stretched by the other branch's kernels running beside them
    dec = Decode(w4, dev, branch_chunks=0)
    torch.cuda.synchronize()
    setup_s = time.time() - t_setup
    stream = torch.cuda.current_stream()

    # warm-up (also first-use costs: function attributes, tensor maps)
    for _ in range(args.warmup):
        pre.run(stream)
        dec.run(stream)
    hy.hymba_stream_status(stream)
    dec.capture()
    dec.graph.replay()
    hy.hymba_stream_status(stream)

    # timed region: K steps, prefill (eager, per-kernel events on) + decode (graph)
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(torch.cuda.current_device())
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    hy.hymba_profile_enable(True)
    hy.hymba_profile_collect()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 1)]
    ev[0].record(stream)
    for s in range(args.steps):
        pre.run(stream)
        ev[2 * s + 1].record(stream)
        dec.graph.replay()
        ev[2 * s + 2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    prof = hy.hymba_profile_collect()
    hy.hymba_profile_enable(False)
    clocks = sampler.stop() if rank == 0 else None
    # the serial schedule (every kernel alone on the GPU): per-kernel figures and step time
    steps_serial = max(1, min(args.steps, 3))
    pre.run(stream, serial=True)
    torch.cuda.synchronize()
    sampler_s = ClockSampler(torch.cuda.current_device())
    if rank == 0:
        sampler_s.start()
        time.sleep(0.3)
    hy.hymba_profile_enable(True)
    hy.hymba_profile_collect()
    es0, es1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es0.record(stream)
    for _ in range(steps_serial):
        pre.run(stream, serial=True)
    es1.record(stream)
    torch.cuda.synchronize()
    sprof = hy.hymba_profile_collect()
    hy.hymba_profile_enable(False)
    clocks_serial = sampler_s.stop() if rank == 0 else None
    serial_ms = max_over_ranks([es0.elapsed_time(es1) / steps_serial], dev, world)[0]
    # for comparison: the same two layers without the meta cache (every sequence's m + n rows)
    steps_full = max(1, min(args.steps, 3))
    pre.run_full(stream)
    torch.cuda.synchronize()
    ef0, ef1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ef0.record(stream)
    for _ in range(steps_full):
        pre.run_full(stream)
    ef1.record(stream)
    torch.cuda.synchronize()
    full_ms = max_over_ranks([ef0.elapsed_time(ef1) / steps_full], dev, world)[0]
    pre.release_full()
    hy.hymba_stream_status(stream)
    pre_ms = sum(ev[2 * s].elapsed_time(ev[2 * s + 1]) for s in range(args.steps))
    dec_ms = sum(ev[2 * s + 1].elapsed_time(ev[2 * s + 2]) for s in range(args.steps))
    tot_ms = ev[0].elapsed_time(ev[-1])
    pre_ms, dec_ms, tot_ms = max_over_ranks([pre_ms, dec_ms, tot_ms], dev, world)

    # kernel launches of this library in the timed region: prefill launches are counted by the
    # profiler; the decode graph holds a fixed number per step (counted once below, eagerly)
    pre_launches = sum(k for _, _, k, _ in prof)
    hy.hymba_profile_enable(True)
    hy.hymba_profile_collect()
    # a device-side delay first, so that the host has enqueued the whole eager step before the
    # GPU reaches it and the events time the kernels, not the host's launch latency
    torch.cuda._sleep(50_000_000)
    dec.run(stream)
    dprof = hy.hymba_profile_collect()
    hy.hymba_profile_enable(False)
    dec_kernels_per_step = sum(k for _, _, k, _ in dprof)

    tokens = w3.batch * w3.n_tokens
    value = job_rate(tokens, args.steps, world, pre_ms)
    dec_tok_s = job_rate(w4.batch, args.steps, world, dec_ms)

    # roofline of the dominant kernel: the input projection GEMM (tensor-bound)
    pmap = {n: (c, ms) for n, c, _, ms in prof}
    c_in, ms_in = pmap.get("in_proj", (0, 0.0))
    # (the concurrent schedule launches it once per batch chunk: the FLOPs of all its launches
    # in the timed region over the sum of their CUDA-event durations)
    fl = pre.in_proj_flops()
    achieved = (sum(fl) * args.steps) / (ms_in / 1e3) / 1e12 if ms_in > 0 else None
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    # the same kernel in the serial pass (alone on the GPU, no scan beside it)
    smap = {n: (c, ms) for n, c, _, ms in sprof}
    _, ms_alone = smap.get("in_proj", (0, 0.0))
    alone = (sum(fl) * steps_serial) / (ms_alone / 1e3) / 1e12 if ms_alone > 0 else None
    roof = {"kernel": "in_proj (gemm_tc_kernel<256,bf16>)", "bound": "tensor",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": (achieved / peak) if achieved else None, "traffic": IN_PROJ_TRAFFIC,
            "traffic_basis": IN_PROJ_TRAFFIC_BASIS,
            "peak_source": f"{peak_src} bf16_tflops_sustained",
            "timing": "timed region: the concurrent step, the scan of the previous batch chunk "
                      "running beside this kernel",
            "alone": {"achieved": alone, "frac": (alone / peak) if alone else None,
                      "timing": "the serial pass after the timed region"}}
    step_flops = pre.flops()
    dec_bytes = dec.hbm_bytes()

    # end to end through the C ABI with host buffers: every step copies its X~ in from pinned
    # host memory and its Y back out.  The copies run on their own streams, double-buffered on
    # the device, so step i+1's input and step i-1's output cross PCIe while step i computes;
    # the timed region runs from before the first input copy to the end of the last output
    # copy.
    e2e = None
    if not args.no_e2e:
        xh = torch.empty(pre.x.shape, dtype=pre.x.dtype, pin_memory=True)
        xh.copy_(pre.x)
        yh = torch.empty_like(xh, pin_memory=True)
        xt_h = torch.empty(dec.x.shape, dtype=dec.x.dtype, pin_memory=True)
        xt_h.copy_(dec.x)
        yt_h = torch.empty_like(xt_h, pin_memory=True)
        xd = [pre.x, torch.empty_like(pre.x)]
        yd = [pre.y2, torch.empty_like(pre.x)]
        xtd = torch.empty_like(dec.x)
        ytd = torch.empty_like(dec.x)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        torch.cuda.synchronize()
        steps_e2e = args.steps
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        in_ready = [ev(), ev()]
        done = [ev(), ev()]
        out_done = [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(steps_e2e):
            j = i % 2
            if i >= 2:
                s_in.wait_event(done[j])          # step i-2 has consumed xd[j]
            with torch.cuda.stream(s_in):
                xd[j].copy_(xh, non_blocking=True)
            in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if i >= 2:
                stream.wait_event(out_done[j])    # step i-2's Y has left yd[j]
            pre.run(stream, x=xd[j], y=yd[j])
            done[j].record(stream)
            s_out.wait_event(done[j])
            with torch.cuda.stream(s_out):
                yh.copy_(yd[j], non_blocking=True)
            out_done[j].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        pre_e2e_ms = t0.elapsed_time(t1)
        ed0, ed1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dec_e2e_ms = 0.0
        for _ in range(steps_e2e):
            ed0.record(stream)
            xtd.copy_(xt_h, non_blocking=True)
            dec.run(stream, x=xtd, y_out=ytd)
            yt_h.copy_(ytd, non_blocking=True)
            ed1.record(stream)
            torch.cuda.synchronize()
            dec_e2e_ms += ed0.elapsed_time(ed1)
        pre_e2e_ms, dec_e2e_ms = max_over_ranks([pre_e2e_ms, dec_e2e_ms], dev, world)
        e2e = {"value": job_rate(tokens, steps_e2e, world, pre_e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": xh.numel() * 2 + xt_h.numel() * 2,
               "d2h_bytes_per_step": yh.numel() * 2 + yt_h.numel() * 2,
               "decode_tok_s": job_rate(w4.batch, steps_e2e, world, dec_e2e_ms),
               "copies": "overlapped with compute on two copy streams, device buffers double-buffered"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample()

    sm_mhz = clocks.get("sm_mhz") if clocks else None
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kernels = kernel_fractions(pre, dec, prof, dprof, peaks, sm_mhz, sms, 2 * args.steps)
    kernels_serial = kernel_fractions(pre, dec, sprof, dprof, peaks, sm_mhz, sms, 2 * steps_serial)

    if rank != 0:
        return None
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "prefill: 2 KV-sharing SWA layers, B=128, 8192+128 meta rows, W=1024, "
                               "1.5B widths, meta rows computed once per step (batch 1) and the "
                               "real rows prefilled from them; decode: 32-layer stack, B=128, 8k context",
                   "prefill": w3.name, "decode": w4.name, "global_batch": w3.batch * world,
                   "seq_len": w3.seq_rows, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (no flush)"},
        "prefill_ms_per_step": pre_ms / args.steps,
        "prefill_without_meta_cache_ms_per_step": full_ms,
        "prefill_serial_ms_per_step": serial_ms,
        "clocks_serial": clocks_serial,
        "branch_chunks": pre.branch_chunks,
        "decode_ms_per_step": dec_ms / args.steps,
        "decode_tok_s": dec_tok_s,
        "prefill_tflops": step_flops * args.steps / (pre_ms / 1e3) / 1e12,
        "prefill_roofline_frac": (step_flops / (peaks.get("bf16_tflops_sustained", 1400) * 1e12))
                                 / (pre_ms / args.steps / 1e3),
        "decode_hbm_gbs": dec_bytes * args.steps / (dec_ms / 1e3) / 1e9,
        "decode_roofline_frac": (dec_bytes / (peaks.get("hbm_gbs", 6650) * 1e9)) / (dec_ms / args.steps / 1e3),
        "roofline": roof,
        "steps_profile": {n: {"calls": c, "kernels": k, "ms_per_call": ms / c if c else None}
                          for n, c, k, ms in prof},
        "decode_steps_profile": {n: {"calls": c, "kernels": k, "ms_per_call": ms / c if c else None}
                                 for n, c, k, ms in dprof},
        "kernels": kernels,
        "kernels_serial": kernels_serial,
        "steps_profile_serial": {n: {"calls": c, "kernels": k, "ms_per_call": ms / c if c else None}
                                 for n, c, k, ms in sprof},
        "gpu_launches": pre_launches + dec_kernels_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "setup_s": setup_s,
    }
    return out


# ---------------------------------------------------------------------------------------------
# CPU baseline: the oracle as it stands on the host cores, on a bounded sample
# ---------------------------------------------------------------------------------------------
CPU_SAMPLE_TOKENS = 2048


def cpu_baseline_sample(tokens: int = CPU_SAMPLE_TOKENS):
    import numpy as np
    import synth
    from oracle import hymba_oracle as O
    w = synth.configs.CFG3
    d = w.dims
    spec = O.Spec(d_model=d.d_model, n_heads=d.n_heads, n_kv_heads=d.n_kv_heads,
                  head_dim_qk=d.head_dim_qk, head_dim_v=d.head_dim_v, d_inner=d.d_inner,
                  d_state=d.d_state, d_conv=d.d_conv, dt_rank=d.rank, n_meta=w.n_meta,
                  window=w.window, is_global=False)
    x = synth.configs.x_tilde(w, batch_index=0)[: w.n_meta + tokens]
    w0 = {k: v.double().numpy() for k, v in synth.configs.layer_weights(w, 0).items()}
    w1 = {k: v.double().numpy() for k, v in synth.configs.layer_weights(w, 1, consumer=True).items()}
    xt = x.double().numpy()
    t0 = time.perf_counter()
    r0 = O.layer_prefill(xt, w0, spec)
    O.layer_prefill(r0["Y"], w1, spec, kv_from=r0)
    dt = time.perf_counter() - t0
    cores = torch.get_num_threads()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max([i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"] or [cores])
    except Exception:
        pass
    return {"value": tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"one sequence (batch row 0) of the prefill workload, first {tokens} real "
                      f"tokens + {w.n_meta} meta rows, both KV-sharing layers, fp64 numpy",
            "seconds": dt}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    samples = []
    for _ in range(args.warmup):
        cpu_baseline_sample(512)
    for _ in range(args.steps):
        samples.append(cpu_baseline_sample(512))
    secs = sum(s["seconds"] for s in samples)
    value = 512 * args.steps / secs
    s0 = samples[0]
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "prefill: 2 KV-sharing SWA layers, B=128, 8192+128 meta rows, "
                                   "W=1024, 1.5B widths (oracle on a bounded sample per step)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": s0["cores"], "kind": "oracle",
                             "sample": s0["sample"].replace("2048", "512")},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(args, dev):
    """A smaller workload for profiling: one prefill layer of the given config, or the decode
    stack alone; prints the per-step profile."""
    import hybrid_attention_ssm_head_b200 as hy
    import synth
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    if args.case in ("decode", "decode-b32"):
        from dataclasses import replace as _replace
        w4 = synth.configs.CFG4 if args.case == "decode" else \
            _replace(synth.configs.CFG4, name="decode_b32", batch=32)
        dec = Decode(w4, dev, branch_chunks=args.branch_chunks)
        run = lambda: dec.run(stream)  # noqa: E731
    elif args.case == "prefill":
        # the headline prefill step alone (both layers, meta caches + real rows)
        pre = Prefill(synth.configs.CFG3, dev, branch_chunks=args.branch_chunks)
        run = lambda: pre.run(stream, serial=args.branch_chunks < 2)  # noqa: E731
    else:
        from dataclasses import replace as _replace
        w = {"cfg1": synth.configs.CFG1, "cfg2": synth.configs.CFG2,
             # prefill layer at the headline widths, batch 32, 1024 tokens: every kernel in the
             # single-pass configuration of the headline run, with a few GB on the device
             "b32": _replace(synth.configs.CFG3, name="b32_n1024", batch=32, n_tokens=1024,
                             n_layers=1, kv_shared_pair=False)}[args.case]
        d = w.dims
        wt = {k: v.contiguous() for k, v in synth.configs.layer_weights(w, 0, device=dev).items()}
        cfg = hy.make_config(d.d_model, d.n_heads, d.n_kv_heads, d.head_dim_qk, d.d_inner, d.d_state,
                             d.d_conv, d.rank, w.n_meta, w.window, w.window <= 0, "bf16",
                             branch_chunks=args.branch_chunks)
        h = hy.hymba_layer_create(cfg, hy.make_weights(wt))
        B, L = w.batch, w.seq_rows
        x = synth.configs.x_tilde(w, device=dev)
        y = torch.empty_like(x)
        k = torch.empty(B, L, d.n_kv_heads * d.head_dim_qk, dtype=torch.bfloat16, device=dev)
        v = torch.empty(B, L, d.n_kv_heads * d.head_dim_v, dtype=torch.bfloat16, device=dev)
        kv = hy.hymba_kv_seq(k.data_ptr(), v.data_ptr(), 0, 0, 0)
        ws = torch.empty(hy.hymba_layer_prefill_workspace(h, B, w.n_tokens), dtype=torch.uint8, device=dev)
        run = lambda: hy.hymba_layer_prefill(h, B, w.n_tokens, x, y, kv, None, None, ws,  # noqa: E731
                                             ws.numel(), stream)
    for _ in range(args.warmup):
        run()
    hy.hymba_stream_status(stream)
    hy.hymba_profile_enable(True)
    hy.hymba_profile_collect()
    torch.cuda._sleep(50_000_000)  # the host gets ahead of the device: events time the kernels
    for _ in range(args.steps):
        run()
    prof = hy.hymba_profile_collect()
    hy.hymba_profile_enable(False)
    hy.hymba_stream_status(stream)
    out = {"case": args.case, "steps": args.steps, "profile": {
        n: {"calls": c, "kernels": kk, "ms_per_call": ms / c} for n, c, kk, ms in prof}}
    if args.case in ("decode", "decode-b32"):
        # the step as the headline times it: one CUDA graph replay per step
        dec.capture()
        for _ in range(3):
            dec.graph.replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record()
        for _ in range(args.steps):
            dec.graph.replay()
        t1.record()
        torch.cuda.synchronize()
        hy.hymba_stream_status(stream)
        out["graph_ms_per_step"] = t0.elapsed_time(t1) / args.steps
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--branch-chunks", type=int, default=BRANCH_CHUNKS,
                    help="batch chunks of the concurrent prefill (0: serial schedule)")
    ap.add_argument("--case", choices=["headline", "prefill", "cfg1", "cfg2", "b32", "decode", "decode-b32"],
                    default="headline",
                    help="headline: the benchmark; others: a smaller run for profiling")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    if args.case != "headline":
        run_case(args, dev)
        return
    out = run_ours(args, rank, world, dev)
    if out is not None:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
