#!/usr/bin/env python
"""Benchmark of the DSA layer stack under IndexCache on B200.

Metric (one JSON line on rank 0): prefill tokens/s of a 16-layer stack at
L = 200,000 with one F layer in four (FSSS x 4), plus decode ms/step of a
48-layer 1/4-F stack with 8 sequences at 200,000 cached tokens, both with
k = 2048, 64 indexer heads of dim 128 and MLA attention (128 heads, 576-wide
latent, 512 value columns).  Inputs are seeded synthetic tensors generated on
the device; every input of the timed region is larger than L2 (126 MB), so no
flush is needed.  A prefill step runs, per layer, the indexer (F layers) and
the sparse attention through the C ABI with CUDA events between launches;
the e2e figure runs the public indexcache_forward() with inputs copied from
pinned host memory every step and the final output copied back (double
buffered on the device, so that one step's copies overlap the neighbouring
steps' compute; every copy stays inside the timed region).  The decode
step is timed as replays of one CUDA graph holding the whole 48-layer step
(per-kernel times come from separate eager steps with events).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dsa|reference]
Multi-GPU: launched by torchrun, one independent replica per rank (weak scaling;
no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s and decode ms/step at 200K ctx, 1/4-F IndexCache stack"

PREFILL = dict(B=1, L=200000, layers=16, ratio=4, H_I=64, d_I=128, k=2048, n_h=128, D_qk=576, D_v=512)
DECODE = dict(B=8, ctx=200000, layers=48, ratio=4, H_I=64, d_I=128, k=2048, n_h=128, D_qk=576, D_v=512)
SEED = 1234


WORKLOAD = ("prefill: B=1, L=200000, 16 layers FSSS x4 (1/4 F), H_I=64 d_I=128 k=2048, MLA 128 heads "
            "576/512; decode: B=8, ctx 200000, 48 layers 1/4 F")


def config_of(world, shard_mode="replicas"):
    """The `config` object of the JSON line (the same for both arms)."""
    zig = shard_mode == "zigzag" and world > 1
    return {"workload": WORKLOAD, "global_batch": 1 if zig else world, "seq_len": PREFILL["L"],
            "parallelism": (f"one sequence, zig-zag query chunks over {world} ranks" if zig
                            else f"dp{world} (independent replicas)"),
            "l2": "inputs larger than L2 (126 MB) every step; no flush"}


def pattern_of(layers, ratio):
    return "".join("F" if l % ratio == 0 else "S" for l in range(layers))


# ----------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.uuid and self.uuid not in parts[1]:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def reduce_max(x, world, device):
    """Max of a per-rank scalar over all ranks (every rank gets the result);
    timings are reported as the slowest rank's."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank runs its own replica)."""
    return units_per_rank * world / (ms_max / 1e3)


def pipelined_e2e(torch, dev, stream, h2d_pairs, forward, d2h_pairs, steps):
    """End-to-end steps with host buffers, double-buffered on the device.

    Step i computes on device buffer set i % 2 (forward(set) enqueues it on
    `stream`) while a copy stream loads step i + 1's inputs from pinned host
    memory into the other set, and a third stream copies step i - 1's result
    back to the host.  Every step's host-to-device inputs and device-to-host
    result are inside the timed region, which ends when the last result is on
    the host.  h2d_pairs[set] and d2h_pairs[set] are lists of (device tensor,
    pinned host tensor).  Returns milliseconds per step."""
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    h2d_done, comp_done, d2h_done = [None, None], [None, None], [None, None]

    def load(b):
        with torch.cuda.stream(s_in):
            if comp_done[b] is not None:
                s_in.wait_event(comp_done[b])  # the step that last used set b is done
            for d, h in h2d_pairs[b]:
                d.copy_(h, non_blocking=True)
            h2d_done[b] = torch.cuda.Event()
            h2d_done[b].record(s_in)

    load(0)
    for i in range(steps):
        b, nb = i % 2, (i + 1) % 2
        if i + 1 < steps:
            load(nb)
        stream.wait_event(h2d_done[b])
        if d2h_done[b] is not None:
            stream.wait_event(d2h_done[b])  # set b's previous result has been read back
        forward(b)
        comp_done[b] = torch.cuda.Event()
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for d, h in d2h_pairs[b]:
                h.copy_(d, non_blocking=True)
            d2h_done[b] = torch.cuda.Event()
            d2h_done[b].record(s_out)
    for ev in d2h_done:
        if ev is not None:
            stream.wait_event(ev)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / steps


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1400.0, "fallback"


def traffic_for(kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    src = os.path.join(ROOT, "sparse_attention_13_b200", "csrc", d["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != d["sha256_16"]:
            return None
    return d["bytes_per_launch"]


def attn_units(Lq, start_pos, k, B=1):
    # selected (t, r) pairs: min(t, k) per query row
    if start_pos == 0:
        n_short = min(Lq, k)
        return B * (n_short * (n_short - 1) // 2 + max(0, Lq - n_short) * k)
    return B * Lq * min(start_pos, k)


def indexer_pairs(Lq, start_pos, B=1):
    if start_pos == 0:
        return B * Lq * (Lq - 1) // 2
    return B * Lq * start_pos


# ----------------------------------------------------------------- GPU arm
def time_stack(torch, dsa, stream, pat, layer_in, idx, ws, k, scale, D_v, steps, warmup, start_pos=0):
    """Runs the layer loop `pat` eagerly through the C ABI (indexer on F
    layers, attention on every layer) with CUDA events around each launch.
    layer_in[l] holds q, kv, out and, on F layers, q_idx, k_idx, w.  Returns
    (ms per step over `steps` timed steps, mean indexer ms per launch, mean
    attention ms per launch, indexer ms per step)."""
    def step(ev=None):
        for l, role in enumerate(pat):
            t = layer_in[l]
            if role == "F":
                if ev is not None:
                    ev["idx"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                    ev["idx"][-1][0].record(stream)
                dsa.indexer_topk(t["q_idx"], t["k_idx"], t["w"], k, start_pos=start_pos, out=idx, ws=ws)
                if ev is not None:
                    ev["idx"][-1][1].record(stream)
            if ev is not None:
                ev["attn"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                ev["attn"][-1][0].record(stream)
            dsa.sparse_attn(t["q"], t["kv"], t["kv"], idx, scale, D_v=D_v, start_pos=start_pos, out=t["out"], ws=ws)
            if ev is not None:
                ev["attn"][-1][1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = {"idx": [], "attn": []}
    t0, t1 = torch.cuda.Event(True), torch.cuda.Event(True)
    t0.record(stream)
    for _ in range(steps):
        step(ev)
    t1.record(stream)
    torch.cuda.synchronize()
    dsa.check_device_errors()
    idx_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["idx"]) if ev["idx"] else 0.0
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["attn"])
    idx_per_step = sum(a.elapsed_time(b) for a, b in ev["idx"]) / steps
    return t0.elapsed_time(t1) / steps, idx_ms, attn_ms, idx_per_step


def run_dsa(args):
    import torch
    import torch.distributed as dist

    from sparse_attention_13_b200 import dsa, shard, synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=600))
    dev = torch.device("cuda", local)
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    seed = SEED + 1000 * rank

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    result = {}
    # ---------------------------------------------------------------- prefill
    P = dict(PREFILL)
    if args.seq:
        P["L"] = args.seq
    L, k, pat = P["L"], P["k"], pattern_of(P["layers"], P["ratio"])
    nF = pat.count("F")
    bf, f32 = torch.bfloat16, torch.float32
    q_idx, k_idx, w = {}, {}, {}
    for l, role in enumerate(pat):
        if role == "F":
            q_idx[l] = torch.empty((1, L, P["H_I"], P["d_I"]), dtype=bf, device=dev)
            k_idx[l] = torch.empty((1, L, P["d_I"]), dtype=bf, device=dev)
            w[l] = torch.empty((1, L, P["H_I"]), dtype=f32, device=dev)
            synth.fill_cuda(q_idx[l], seed, synth.Q_IDX, synth.INT9, l)
            synth.fill_cuda(k_idx[l], seed, synth.K_IDX, synth.INT9, l)
            synth.fill_cuda(w[l], seed, synth.W, synth.POW2W, l)
    kv = []
    for l in range(len(pat)):
        t = torch.empty((1, L, P["D_qk"]), dtype=bf, device=dev)
        synth.fill_cuda(t, seed, synth.KV, synth.NORMAL, l, sigma=0.5)
        kv.append(t)
    q = torch.empty((1, L, P["n_h"], P["D_qk"]), dtype=bf, device=dev)
    synth.fill_cuda(q, seed, synth.Q, synth.NORMAL, 0, sigma=0.5)
    out = torch.empty((1, L, P["n_h"], P["D_v"]), dtype=bf, device=dev)
    idx = torch.empty((1, L, k), dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(P["D_qk"])
    dims = dsa.make_dims(B=1, Lq=L, Lk=L, start_pos=0, H_I=P["H_I"], d_I=P["d_I"], k=k,
                         n_h=P["n_h"], D_qk=P["D_qk"], D_v=P["D_v"], scale=scale,
                         k_row_stride=P["D_qk"], v_row_stride=P["D_qk"])
    # Query rows this rank computes: the whole sequence (independent
    # replicas), or its two zig-zag chunks of the one sequence, each run as a
    # chunked prefill (start_pos = the chunk's first row) over the full caches.
    zig = args.shard == "zigzag" and world > 1
    chunks = shard.zigzag_chunks(L, world, rank) if zig else [(0, L)]

    def chunk_dims(s, n):
        return dsa.make_dims(B=1, Lq=n, Lk=L, start_pos=s, H_I=P["H_I"], d_I=P["d_I"], k=k,
                             n_h=P["n_h"], D_qk=P["D_qk"], D_v=P["D_v"], scale=scale,
                             k_row_stride=P["D_qk"], v_row_stride=P["D_qk"])

    ws = torch.empty(max(dsa.indexcache_forward_workspace(chunk_dims(s, n)) for s, n in chunks),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        for l, role in enumerate(pat):
            if role == "F":
                if events is not None:
                    events["idx"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                    events["idx"][-1][0].record(stream)
                for s, n in chunks:
                    dsa.indexer_topk(q_idx[l][:, s:s + n], k_idx[l], w[l][:, s:s + n], k, start_pos=s,
                                     out=idx[:, s:s + n], ws=ws)
                if events is not None:
                    events["idx"][-1][1].record(stream)
            if events is not None:
                events["attn"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                events["attn"][-1][0].record(stream)
            for s, n in chunks:
                dsa.sparse_attn(q[:, s:s + n], kv[l], kv[l], idx[:, s:s + n], scale, D_v=P["D_v"], start_pos=s,
                                out=out[:, s:s + n], ws=ws)
            if events is not None:
                events["attn"][-1][1].record(stream)

    for _ in range(args.warmup):
        step()
    dsa.check_device_errors()
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(uuid)
    clocks.start()
    ev = {"idx": [], "attn": []}
    t0, t1 = torch.cuda.Event(True), torch.cuda.Event(True)
    t0.record(stream)
    for _ in range(args.steps):
        step(ev)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier()
    dsa.check_device_errors()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    idx_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["idx"])
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["attn"])
    # this rank's work per layer (its chunks; the whole sequence for replicas)
    a_units = sum(shard.attention_rows(s, n, k) for s, n in chunks)
    i_pairs = sum(shard.indexer_pairs(s, n) for s, n in chunks)
    attn_flops = a_units * 2 * P["n_h"] * (P["D_qk"] + P["D_v"])
    idx_flops = i_pairs * 2 * P["H_I"] * P["d_I"]
    job_tokens = L if zig else L * world  # one sequence split, or one per rank
    result["prefill"] = dict(
        ms_per_step=ms, tokens_per_s=job_tokens / (ms / 1e3), idx_ms=idx_ms, attn_ms=attn_ms,
        indexer_share=nF * idx_ms / (nF * idx_ms + len(pat) * attn_ms),
        attn_tflops=attn_flops / attn_ms / 1e9, idx_tflops=idx_flops / idx_ms / 1e9,
        attn_flops=attn_flops, idx_flops=idx_flops, clocks=clk, chunks=chunks,
        scaling="strong" if zig else "weak",
        launches=args.steps * len(chunks) * (nF + len(pat)))

    # The ratio sweep of the long prefill (1/1 and 1/2 beside the 1/4 stack
    # timed above): the same 16 layers and shapes, with an indexer on every
    # layer, or on every other layer.  Extra F layers get their own indexer
    # inputs.  Kernels are warm; one warm-up step and a short timed region.
    sweep = {}
    if not args.no_sweep and not zig:
        extra = []
        for l in range(len(pat)):
            if l not in q_idx:
                q_idx[l] = torch.empty((1, L, P["H_I"], P["d_I"]), dtype=bf, device=dev)
                k_idx[l] = torch.empty((1, L, P["d_I"]), dtype=bf, device=dev)
                w[l] = torch.empty((1, L, P["H_I"]), dtype=f32, device=dev)
                synth.fill_cuda(q_idx[l], seed, synth.Q_IDX, synth.INT9, l)
                synth.fill_cuda(k_idx[l], seed, synth.K_IDX, synth.INT9, l)
                synth.fill_cuda(w[l], seed, synth.W, synth.POW2W, l)
                extra.append(l)
        sw_steps = max(1, min(args.steps, 2))
        runs = {}
        for ratio in (1, 2):
            spat = pattern_of(P["layers"], ratio)
            lin = [dict(q=q, kv=kv[l], out=out, q_idx=q_idx.get(l), k_idx=k_idx.get(l), w=w.get(l))
                   for l in range(len(spat))]
            barrier()
            runs[ratio] = (spat,) + time_stack(torch, dsa, stream, spat, lin, idx, ws, k, scale, P["D_v"],
                                               sw_steps, 1)
        runs[P["ratio"]] = (pat, ms, idx_ms, attn_ms, idx_ms * nF)
        all_f_idx = runs[1][4]
        for ratio in sorted(runs):
            spat, sms, sidx, sattn, sidx_step = runs[ratio]
            sms = max_over_ranks(sms)
            m = spat.count("F")
            sweep[f"1/{ratio}"] = dict(
                pattern=spat, ms_per_step=sms, tokens_per_s=job_rate(L, world, sms),
                indexer_ms_per_step=sidx_step, attn_ms_per_step=sattn * len(spat),
                indexer_share=sidx_step / (sidx_step + sattn * len(spat)),
                indexer_ms_expected=m / len(spat) * all_f_idx,
                indexer_launches_per_step=m,
                steps=sw_steps if ratio != P["ratio"] else args.steps,
                warmup=1 if ratio != P["ratio"] else args.warmup)
        for l in extra:
            del q_idx[l], k_idx[l], w[l]
        del lin
        torch.cuda.empty_cache()
    result["prefill"]["sweep"] = sweep

    # The low-precision selector ([IDX] §5.4) on the first F layer's inputs,
    # timed per launch beside the bf16 indexer (the call quantises q_idx and
    # k_idx into its workspace, included in the time).
    lowprec = {}
    if not args.no_sweep and not zig:
        for fmt in ("e4m3", "e2m1"):
            lws = torch.empty(dsa.indexer_topk_lowprec_workspace(1, L, L, 0, P["H_I"], P["d_I"], k, fmt),
                              dtype=torch.uint8, device=dev)
            run = lambda: dsa.indexer_topk_lowprec(q_idx[0], k_idx[0], w[0], k, fmt=fmt, out=idx, ws=lws)  # noqa: E731
            run()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
            e0.record(stream)
            for _ in range(2):
                run()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            lms = max_over_ranks(e0.elapsed_time(e1) / 2)
            lowprec[fmt] = {"ms_per_launch": lms, "speedup_vs_bf16": idx_ms / lms,
                            "tflops_equiv": idx_flops / lms / 1e9}
            del lws
        dsa.check_device_errors()
    result["prefill"]["lowprec"] = lowprec

    # e2e through the public API with host buffers: every step copies in the
    # caches and this rank's query-side rows, and copies its output rows back
    host_in = []
    for l in sorted(q_idx):
        host_in += [(k_idx[l], None)] + [(q_idx[l][:, s:s + n], None) for s, n in chunks] + \
                   [(w[l][:, s:s + n], None) for s, n in chunks]
    host_in += [(t, None) for t in kv] + [(q[:, s:s + n], None) for s, n in chunks]
    host_in = [(d, torch.empty(d.shape, dtype=d.dtype, pin_memory=True)) for d, _ in host_in]
    for d, h in host_in:
        h.copy_(d)
    out_dev = [out[:, s:s + n] for s, n in chunks]
    out_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in out_dev]
    h2d = sum(d.numel() * d.element_size() for d, _ in host_in)
    d2h = sum(o.numel() * o.element_size() for o in out_dev)
    # a second device set of every input and of the output (double buffering)
    set_dev = [[d for d, _ in host_in], [torch.empty_like(d) for d, _ in host_in]]
    set_out = [out_dev, [torch.empty_like(o) for o in out_dev]]
    pos = {id(d): i for i, (d, _) in enumerate(host_in)}

    def layers_of(b, c):
        # the layer list of chunk c on device set b
        sel = lambda d: set_dev[b][pos[id(d)]]  # noqa: E731
        res = []
        for l, role in enumerate(pat):
            L_ = dict(q=sel(q_views[c]), kbuf=sel(kv[l]), vbuf=sel(kv[l]), out=set_out[b][c])
            if role == "F":
                L_.update(q_idx=sel(qi_views[l][c]), k_idx=sel(k_idx[l]), w=sel(w_views[l][c]))
            res.append(L_)
        return res

    # the views registered in host_in, by chunk
    q_views = [host_in[len(host_in) - len(chunks) + c][0] for c in range(len(chunks))]
    qi_views, w_views = {}, {}
    base = 0
    for l in sorted(q_idx):
        qi_views[l] = [host_in[base + 1 + c][0] for c in range(len(chunks))]
        w_views[l] = [host_in[base + 1 + len(chunks) + c][0] for c in range(len(chunks))]
        base += 1 + 2 * len(chunks)
    set_layers = [[layers_of(b, c) for c in range(len(chunks))] for b in range(2)]
    h2d_pairs = [[(d, h) for d, (_, h) in zip(set_dev[b], host_in)] for b in range(2)]
    d2h_pairs = [[(set_out[b][c], out_h[c]) for c in range(len(chunks))] for b in range(2)]
    cdims = [chunk_dims(s, n) for s, n in chunks]
    cidx = [idx[:, s:s + n] for s, n in chunks]

    def e2e_forward(b):
        for c in range(len(chunks)):
            dsa.indexcache_forward(pat, set_layers[b][c], cdims[c], cidx[c], ws=ws)

    pipelined_e2e(torch, dev, stream, h2d_pairs, e2e_forward, d2h_pairs, args.warmup)
    barrier()
    e2e_ms = max_over_ranks(pipelined_e2e(torch, dev, stream, h2d_pairs, e2e_forward, d2h_pairs, args.steps))
    barrier()
    dsa.check_device_errors()
    result["prefill"]["e2e"] = {"value": job_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del host_in, out_h, q_idx, k_idx, w, kv, q, out, idx, ws, set_dev, set_out, set_layers, h2d_pairs, d2h_pairs
    del out_dev, q_views, qi_views, w_views, cidx, pos
    d = h = t = None  # loop variables above still name device tensors
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    assert torch.cuda.memory_allocated(dev) < (1 << 30), "prefill buffers still referenced"

    # ---------------------------------------------------------------- decode
    D = dict(DECODE)
    B, ctx, kd = D["B"], D["ctx"], D["k"]
    dpat = pattern_of(D["layers"], D["ratio"])
    dq_idx, dk_idx, dw, dq, dkv = {}, {}, {}, [], []
    for l, role in enumerate(dpat):
        if role == "F":
            dq_idx[l] = torch.empty((B, 1, D["H_I"], D["d_I"]), dtype=bf, device=dev)
            dk_idx[l] = torch.empty((B, ctx, D["d_I"]), dtype=bf, device=dev)
            dw[l] = torch.empty((B, 1, D["H_I"]), dtype=f32, device=dev)
            synth.fill_cuda(dq_idx[l], seed + 7, synth.Q_IDX, synth.INT9, l)
            synth.fill_cuda(dk_idx[l], seed + 7, synth.K_IDX, synth.INT9, l)
            synth.fill_cuda(dw[l], seed + 7, synth.W, synth.POW2W, l)
        t = torch.empty((B, 1, D["n_h"], D["D_qk"]), dtype=bf, device=dev)
        synth.fill_cuda(t, seed + 7, synth.Q, synth.NORMAL, l, sigma=0.5)
        dq.append(t)
        t = torch.empty((B, ctx, D["D_qk"]), dtype=bf, device=dev)
        synth.fill_cuda(t, seed + 7, synth.KV, synth.NORMAL, l, sigma=0.5)
        dkv.append(t)
    dout = torch.empty((B, 1, D["n_h"], D["D_v"]), dtype=bf, device=dev)
    didx = torch.empty((B, 1, kd), dtype=torch.int32, device=dev)
    ddims = dsa.make_dims(B=B, Lq=1, Lk=ctx, start_pos=ctx, H_I=D["H_I"], d_I=D["d_I"], k=kd,
                          n_h=D["n_h"], D_qk=D["D_qk"], D_v=D["D_v"], scale=scale,
                          k_row_stride=D["D_qk"], v_row_stride=D["D_qk"])
    dws = torch.empty(dsa.indexcache_forward_workspace(ddims), dtype=torch.uint8, device=dev)

    def dstep(events=None):
        for l, role in enumerate(dpat):
            if role == "F":
                if events is not None:
                    events["idx"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                    events["idx"][-1][0].record(stream)
                dsa.indexer_topk(dq_idx[l], dk_idx[l], dw[l], kd, start_pos=ctx, out=didx, ws=dws)
                if events is not None:
                    events["idx"][-1][1].record(stream)
            if events is not None:
                events["attn"].append((torch.cuda.Event(True), torch.cuda.Event(True)))
                events["attn"][-1][0].record(stream)
            dsa.sparse_attn(dq[l], dkv[l], dkv[l], didx, scale, D_v=D["D_v"], start_pos=ctx,
                            out=dout, ws=dws)
            if events is not None:
                events["attn"][-1][1].record(stream)

    for _ in range(max(args.warmup, 3)):
        dstep()
    barrier()
    torch.cuda.synchronize(dev)
    # per-kernel breakdown: eager steps with events between the calls
    dev_ev = {"idx": [], "attn": []}
    for _ in range(3):
        dstep(dev_ev)
    torch.cuda.synchronize(dev)
    d_idx_ms = statistics.mean(a.elapsed_time(b) for a, b in dev_ev["idx"])
    d_attn_ms = statistics.mean(a.elapsed_time(b) for a, b in dev_ev["attn"])
    # the timed decode step is one CUDA graph of the whole 48-layer step (the
    # way a decode loop replays it); several seconds of replays, so that the
    # clock record holds many samples
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        dstep()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dstep()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    dsa.check_device_errors()
    dsteps = args.decode_steps
    barrier()
    torch.cuda.synchronize(dev)
    dclocks = ClockSampler(uuid)
    dclocks.start()
    t0.record(stream)
    for _ in range(dsteps):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    dclk = dclocks.stop()
    barrier()
    dsa.check_device_errors()
    dms = max_over_ranks(t0.elapsed_time(t1) / dsteps)
    del graph
    nFd = dpat.count("F")
    idx_bytes = B * ctx * D["d_I"] * 2 + B * D["H_I"] * D["d_I"] * 2 + B * kd * 4
    attn_bytes = B * kd * D["D_qk"] * 2 + B * D["n_h"] * (D["D_qk"] + D["D_v"]) * 2 + B * kd * 4
    step_bytes = nFd * idx_bytes + len(dpat) * attn_bytes
    # e2e: new query tokens in, final output out; caches stay resident
    hq = [(t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True)) for t in dq]
    hqi = [(dq_idx[l], torch.empty(dq_idx[l].shape, dtype=bf, pin_memory=True)) for l in sorted(dq_idx)]
    hw = [(dw[l], torch.empty(dw[l].shape, dtype=f32, pin_memory=True)) for l in sorted(dw)]
    for d_, h_ in hq + hqi + hw:
        h_.copy_(d_)
    hout = torch.empty(dout.shape, dtype=bf, pin_memory=True)
    pairs0 = hq + hqi + hw
    dset = [[d_ for d_, _ in pairs0], [torch.empty_like(d_) for d_, _ in pairs0]]
    dset_out = [dout, torch.empty_like(dout)]

    def dlayers_of(b):
        dmap = {id(d0): d1 for d0, d1 in zip(dset[0], dset[b])}
        res = []
        for l, role in enumerate(dpat):
            L_ = dict(q=dmap[id(dq[l])], kbuf=dkv[l], vbuf=dkv[l], out=dset_out[b])
            if role == "F":
                L_.update(q_idx=dmap[id(dq_idx[l])], k_idx=dk_idx[l], w=dmap[id(dw[l])])
            res.append(L_)
        return res

    dset_layers = [dlayers_of(0), dlayers_of(1)]
    dh2d_pairs = [[(d_, h_) for d_, (_, h_) in zip(dset[b], pairs0)] for b in range(2)]
    dd2h_pairs = [[(dset_out[b], hout)] for b in range(2)]

    def de2e_forward(b):
        dsa.indexcache_forward(dpat, dset_layers[b], ddims, didx, ws=dws)

    pipelined_e2e(torch, dev, stream, dh2d_pairs, de2e_forward, dd2h_pairs, 3)
    barrier()
    de2e_ms = max_over_ranks(pipelined_e2e(torch, dev, stream, dh2d_pairs, de2e_forward, dd2h_pairs, 20))
    barrier()
    dsa.check_device_errors()
    dh2d = sum(d_.numel() * d_.element_size() for d_, _ in hq + hqi + hw)
    result["decode"] = dict(ms_per_step=dms, idx_ms=d_idx_ms, attn_ms=d_attn_ms,
                            step_bytes=step_bytes, clocks=dclk,
                            e2e={"value": de2e_ms, "unit": "ms/step", "h2d_bytes_per_step": dh2d,
                                 "d2h_bytes_per_step": hout.numel() * 2})
    # per step: score + top-k kernels per F layer, attention + split merge per layer
    result["decode"]["launches"] = dsteps * (2 * nFd + 2 * len(dpat))
    del dq_idx, dk_idx, dw, dq, dkv, dset, dset_out, dset_layers, dh2d_pairs, dd2h_pairs, hq, hqi, hw, hout
    torch.cuda.empty_cache()
    if not args.no_sweep:
        result["config2"] = run_config2(torch, dsa, synth, dev, stream, seed, max_over_ranks)
        result["config3"] = run_config3(torch, dsa, synth, dev, stream, seed, max_over_ranks, world, barrier)
    result["peaks"] = (hbm_peak, tc_peak, peak_kind)
    result["world"] = world
    if world > 1:
        dist.destroy_process_group()
    return result


CONFIG2 = dict(B=1, L=16384, H_I=64, d_I=128, k=2048)
CONFIG3 = dict(B=1, L=32768, pattern="FSSSFSSS", H_I=64, d_I=128, k=2048, n_h=128, D_qk=576, D_v=512)


def run_config2(torch, dsa, synth, dev, stream, seed, max_over_ranks, reps=20):
    """One F layer's indexer + top-k alone (B = 1, L = 16,384, 64 heads x 128,
    k = 2048, integer inputs), `reps` launches after 3 warm-up launches.  The
    kernel is timed on its own, so its roofline uses the burst bf16 peak."""
    C = CONFIG2
    L = C["L"]
    qi = torch.empty((1, L, C["H_I"], C["d_I"]), dtype=torch.bfloat16, device=dev)
    ki = torch.empty((1, L, C["d_I"]), dtype=torch.bfloat16, device=dev)
    wi = torch.empty((1, L, C["H_I"]), dtype=torch.float32, device=dev)
    synth.fill_cuda(qi, seed + 2, synth.Q_IDX, synth.INT9, 0)
    synth.fill_cuda(ki, seed + 2, synth.K_IDX, synth.INT9, 0)
    synth.fill_cuda(wi, seed + 2, synth.W, synth.POW2W, 0)
    out = torch.empty((1, L, C["k"]), dtype=torch.int32, device=dev)
    ws = torch.empty(dsa.indexer_topk_workspace(1, L, L, 0, C["H_I"], C["d_I"], C["k"]), dtype=torch.uint8,
                     device=dev)
    for _ in range(3):
        dsa.indexer_topk(qi, ki, wi, C["k"], out=out, ws=ws)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(True), torch.cuda.Event(True)
    t0.record(stream)
    for _ in range(reps):
        dsa.indexer_topk(qi, ki, wi, C["k"], out=out, ws=ws)
    t1.record(stream)
    torch.cuda.synchronize()
    dsa.check_device_errors()
    ms = max_over_ranks(t0.elapsed_time(t1) / reps)
    flops = indexer_pairs(L, 0) * 2 * C["H_I"] * C["d_I"]
    burst = measured_burst_tflops()
    return {"workload": f"B=1, L={L}, one F layer (indexer + top-k), H_I=64 d_I=128 k=2048, integer "
                        "q/k in [-4,4], w = +-2^-m", "ms_per_launch": ms, "launches": reps,
            "roofline": {"bound": "tensor", "kernel": "indexer_topk", "achieved": flops / ms / 1e9,
                         "peak": burst[0], "unit": "TFLOP/s", "frac": flops / ms / 1e9 / burst[0],
                         "peak_kind": f"{burst[1]} bf16 burst (kernel timed alone)",
                         "per_launch_flops": flops}}


def run_config3(torch, dsa, synth, dev, stream, seed, max_over_ranks, world, barrier, steps=5):
    """The eight-layer FSSSFSSS stack (B = 1, L = 32,768, k = 2048, MLA 128
    heads 576/512, correlated layers), `steps` timed steps after 3 warm-up
    steps.  Each layer has its own query and latent cache; the layers share
    one output buffer."""
    C = CONFIG3
    L, pat = C["L"], C["pattern"]
    bf = torch.bfloat16
    lin = []
    out = torch.empty((1, L, C["n_h"], C["D_v"]), dtype=bf, device=dev)
    for l, role in enumerate(pat):
        t = dict(q=torch.empty((1, L, C["n_h"], C["D_qk"]), dtype=bf, device=dev),
                 kv=torch.empty((1, L, C["D_qk"]), dtype=bf, device=dev), out=out)
        synth.fill_cuda(t["q"], seed + 3, synth.Q, synth.NORMAL, l, sigma=0.5, corr=True)
        synth.fill_cuda(t["kv"], seed + 3, synth.KV, synth.NORMAL, l, sigma=0.5, corr=True)
        if role == "F":
            t["q_idx"] = torch.empty((1, L, C["H_I"], C["d_I"]), dtype=bf, device=dev)
            t["k_idx"] = torch.empty((1, L, C["d_I"]), dtype=bf, device=dev)
            t["w"] = torch.empty((1, L, C["H_I"]), dtype=torch.float32, device=dev)
            synth.fill_cuda(t["q_idx"], seed + 3, synth.Q_IDX, synth.INT9, l, corr=True)
            synth.fill_cuda(t["k_idx"], seed + 3, synth.K_IDX, synth.INT9, l, corr=True)
            synth.fill_cuda(t["w"], seed + 3, synth.W, synth.POW2W, l)
        lin.append(t)
    idx = torch.empty((1, L, C["k"]), dtype=torch.int32, device=dev)
    dims = dsa.make_dims(B=1, Lq=L, Lk=L, start_pos=0, H_I=C["H_I"], d_I=C["d_I"], k=C["k"], n_h=C["n_h"],
                         D_qk=C["D_qk"], D_v=C["D_v"], scale=1 / math.sqrt(C["D_qk"]), k_row_stride=C["D_qk"],
                         v_row_stride=C["D_qk"])
    ws = torch.empty(dsa.indexcache_forward_workspace(dims), dtype=torch.uint8, device=dev)
    barrier()
    ms, idx_ms, attn_ms, idx_step = time_stack(torch, dsa, stream, pat, lin, idx, ws, C["k"],
                                               1 / math.sqrt(C["D_qk"]), C["D_v"], steps, 3)
    ms = max_over_ranks(ms)
    a_flops = attn_units(L, 0, C["k"]) * 2 * C["n_h"] * (C["D_qk"] + C["D_v"])
    i_flops = indexer_pairs(L, 0) * 2 * C["H_I"] * C["d_I"]
    return {"workload": f"B=1, L={L}, 8 layers {pat}, H_I=64 d_I=128 k=2048, MLA 128 heads 576/512, "
                        "correlated layers", "ms_per_step": ms, "tokens_per_s": job_rate(L, world, ms),
            "steps": steps, "warmup": 3, "indexer_ms": idx_ms, "attn_ms": attn_ms,
            "indexer_share": idx_step / ms,
            "attn_tflops": a_flops / attn_ms / 1e9, "indexer_tflops": i_flops / idx_ms / 1e9,
            "step_flops": 2 * i_flops + 8 * a_flops}


def measured_burst_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f).get("bf16_tflops", 1590.0), "measured"
    return 1590.0, "fallback"


# ----------------------------------------------------------------- CPU oracle
_ORACLE_KEYS = {}


def _oracle_keys(seed, B, L, d):
    # indexer keys of sequence 0, layer 0 (host copy for the oracle sample)
    import numpy as np

    from sparse_attention_13_b200 import synth
    key = (seed, B, L, d)
    if key not in _ORACLE_KEYS:
        _ORACLE_KEYS[key] = synth.rows(seed, synth.K_IDX, synth.INT9, 0, (B, L, d), np.arange(L))
    return _ORACLE_KEYS[key]


def _par_init():
    import oracle
    oracle.build()
    _oracle_keys(SEED, 1, PREFILL["L"], PREFILL["d_I"])


def _par_indexer_row(t):
    """One oracle indexer + top-k row of the prefill stack (worker process)."""
    import numpy as np

    import oracle
    from sparse_attention_13_b200 import synth
    P = PREFILL
    k_h = _oracle_keys(SEED, 1, P["L"], P["d_I"])
    qr = synth.rows(SEED, synth.Q_IDX, synth.INT9, 0, (1, P["L"], P["H_I"], P["d_I"]),
                    np.arange(P["H_I"]) + t * P["H_I"])
    wr = synth.rows(SEED, synth.W, synth.POW2W, 0, (1, P["L"], P["H_I"]), [t], bf16=False)[0]
    return oracle.topk_row(oracle.indexer_row(qr, k_h, wr, t), t, P["k"])


def _par_attn_row(args):
    """One oracle attention row of the prefill stack (worker process)."""
    import numpy as np

    import oracle
    from sparse_attention_13_b200 import synth
    t, sel = args
    P = PREFILL
    valid = sel[sel >= 0]
    rows_kv = synth.rows(SEED, synth.KV, synth.NORMAL, 0, (1, P["L"], P["D_qk"]), valid, sigma=0.5)
    q_r = synth.rows(SEED, synth.Q, synth.NORMAL, 0, (1, P["L"], P["n_h"], P["D_qk"]),
                     np.arange(P["n_h"]) + t * P["n_h"], sigma=0.5)
    a = time.perf_counter()
    oracle.sparse_attn_row(q_r, rows_kv, rows_kv, np.arange(len(valid), dtype=np.int32),
                           1 / math.sqrt(P["D_qk"]), Dv=P["D_v"])
    return time.perf_counter() - a


def oracle_parallel_sample(procs):
    """The same oracle routines run row-parallel: `procs` spawned processes
    (one single-threaded oracle each), one stratified indexer row and one
    attention row per process; wall time of each batch, extrapolated to the
    stack like the single-threaded sample."""
    import multiprocessing as mp
    P = PREFILL
    L = P["L"]
    nF = pattern_of(P["layers"], P["ratio"]).count("F")
    ts = [int(L * (2 * j + 1) / (2 * procs)) for j in range(procs)]
    with mp.get_context("spawn").Pool(procs, initializer=_par_init) as pool:
        pool.map(_par_indexer_row, [1] * procs, chunksize=1)   # workers up, keys built
        a = time.perf_counter()
        sels = pool.map(_par_indexer_row, ts, chunksize=1)
        w_idx = time.perf_counter() - a
        a = time.perf_counter()
        pool.map(_par_attn_row, list(zip(ts, sels)), chunksize=1)
        w_attn = time.perf_counter() - a
    per_tok = nF * w_idx / procs + P["layers"] * w_attn / procs
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "processes": procs,
            "kind": "oracle, row-parallel",
            "sample": f"{procs} spawned single-threaded oracle processes, one indexer row each at "
                      f"stratified t, then one attention row each; wall time per batch, extrapolated "
                      f"by rows x layers", "seconds": w_idx + w_attn}


def oracle_sample(budget_rows=4, decode=True):
    """Times the CPU oracle (single thread, as it stands) on a bounded sample
    of the prefill and decode workloads and extrapolates to the metric."""
    import numpy as np

    import oracle
    from sparse_attention_13_b200 import synth

    oracle.build()
    P = PREFILL
    L, k = P["L"], P["k"]
    nF = pattern_of(P["layers"], P["ratio"]).count("F")
    seed = SEED
    k_h = _oracle_keys(seed, 1, L, P["d_I"])[None]
    ts = [int(L * (2 * j + 1) / (2 * budget_rows)) for j in range(budget_rows)]
    t_idx, t_attn = [], []
    for t in ts:
        qr = synth.rows(seed, synth.Q_IDX, synth.INT9, 0, (1, L, P["H_I"], P["d_I"]),
                        np.arange(P["H_I"]) + t * P["H_I"])
        wr = synth.rows(seed, synth.W, synth.POW2W, 0, (1, L, P["H_I"]), [t], bf16=False)[0]
        a = time.perf_counter()
        I = oracle.indexer_row(qr, k_h[0], wr, t)
        sel = oracle.topk_row(I, t, k)
        t_idx.append(time.perf_counter() - a)
        valid = sel[sel >= 0]
        rows_kv = synth.rows(seed, synth.KV, synth.NORMAL, 0, (1, L, P["D_qk"]), valid, sigma=0.5)
        q_r = synth.rows(seed, synth.Q, synth.NORMAL, 0, (1, L, P["n_h"], P["D_qk"]),
                         np.arange(P["n_h"]) + t * P["n_h"], sigma=0.5)
        a = time.perf_counter()
        oracle.sparse_attn_row(q_r, rows_kv, rows_kv, np.arange(len(valid), dtype=np.int32),
                               1 / math.sqrt(P["D_qk"]), Dv=P["D_v"])
        t_attn.append(time.perf_counter() - a)
    # per token of the stack: nF indexer rows (work ~ t, sampled at mean t) + all layers' attention
    per_tok = nF * statistics.mean(t_idx) + P["layers"] * statistics.mean(t_attn)
    res = {"prefill_tokens_per_s": 1.0 / per_tok,
           "sample": f"{budget_rows} indexer rows (t = {ts}) and {budget_rows} attention rows "
                     f"(k = {k}) of the L = {L} stack, single-threaded, extrapolated by "
                     f"rows x layers (indexer work is linear in t; mean of stratified t)",
           "seconds": sum(t_idx) + sum(t_attn)}
    if decode:
        Dd = DECODE
        ctx = Dd["ctx"]
        kd_h = _oracle_keys(seed + 7, Dd["B"], ctx, Dd["d_I"])
        qr = synth.rows(seed + 7, synth.Q_IDX, synth.INT9, 0, (Dd["B"], 1, Dd["H_I"], Dd["d_I"]),
                        np.arange(Dd["H_I"]))
        wr = synth.rows(seed + 7, synth.W, synth.POW2W, 0, (Dd["B"], 1, Dd["H_I"]), [0], bf16=False)[0]
        a = time.perf_counter()
        I = oracle.indexer_row(qr, kd_h, wr, ctx)
        sel = oracle.topk_row(I, ctx, Dd["k"])
        ti = time.perf_counter() - a
        valid = sel[sel >= 0]
        rows_kv = synth.rows(seed + 7, synth.KV, synth.NORMAL, 0, (Dd["B"], ctx, Dd["D_qk"]), valid, sigma=0.5)
        q_r = synth.rows(seed + 7, synth.Q, synth.NORMAL, 0, (Dd["B"], 1, Dd["n_h"], Dd["D_qk"]),
                         np.arange(Dd["n_h"]), sigma=0.5)
        a = time.perf_counter()
        oracle.sparse_attn_row(q_r, rows_kv, rows_kv, np.arange(len(valid), dtype=np.int32),
                               1 / math.sqrt(Dd["D_qk"]), Dv=Dd["D_v"])
        ta = time.perf_counter() - a
        nFd = pattern_of(Dd["layers"], Dd["ratio"]).count("F")
        res["decode_ms_per_step"] = 1e3 * Dd["B"] * (nFd * ti + Dd["layers"] * ta)
        res["decode_sample"] = (f"1 indexer row over {ctx} keys and 1 attention row, sequence 0, "
                                f"single-threaded, extrapolated x {Dd['B']} sequences x layers")
        res["seconds"] += ti + ta
    return res


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    P = PREFILL
    # each step: a bounded sample (one stratified indexer row + one attention row)
    for _ in range(args.warmup):
        oracle_sample(budget_rows=1, decode=False)
    vals = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        vals.append(oracle_sample(budget_rows=1, decode=False)["prefill_tokens_per_s"])
    elapsed = time.perf_counter() - t_all
    v = statistics.mean(vals)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(args.gpus, args.shard),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "host_cores": os.cpu_count() or 1,
                             "kind": "oracle",
                             "sample": f"per step: 1 indexer row at t = L/2 (the mean causal row) and "
                                       f"1 attention row of the L = {P['L']} prefill stack, single host "
                                       f"thread, extrapolated to the 16-layer stack (prefill metric only)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def kernel_case(name, seq, reps):
    """Runs one kernel on a small case (inputs of a few GB, larger than L2) for
    profiling: `reps` launches after one warm-up launch."""
    import torch

    from sparse_attention_13_b200 import dsa, synth
    dev = torch.device("cuda", 0)
    bf = torch.bfloat16
    if name in ("indexer", "decode_idx", "indexer_tail"):
        # indexer_tail: the last `seq` query rows of a 200,000-token prefill
        B, Lq, Lk, sp = {"indexer": (1, seq, seq, 0), "decode_idx": (8, 1, 200000, 200000),
                         "indexer_tail": (1, seq, 200000, 200000 - seq)}[name]
        q = torch.empty((B, Lq, 64, 128), dtype=bf, device=dev)
        kk = torch.empty((B, Lk, 128), dtype=bf, device=dev)
        w = torch.empty((B, Lq, 64), dtype=torch.float32, device=dev)
        synth.fill_cuda(q, SEED, synth.Q_IDX, synth.INT9, 0)
        synth.fill_cuda(kk, SEED, synth.K_IDX, synth.INT9, 0)
        synth.fill_cuda(w, SEED, synth.W, synth.POW2W, 0)
        out = torch.empty((B, Lq, 2048), dtype=torch.int32, device=dev)
        ws = torch.empty(dsa.indexer_topk_workspace(B, Lq, Lk, sp, 64, 128, 2048), dtype=torch.uint8, device=dev)
        run = lambda: dsa.indexer_topk(q, kk, w, 2048, start_pos=sp, out=out, ws=ws)
    elif name in ("attn", "decode_attn", "attn_tail"):
        # attn_tail: the last `seq` rows of a 200,000-token prefill against the
        # full latent cache (the long-context gather regime on a few GB)
        B, Lq, Lk, sp = {"attn": (1, seq, seq, 0), "decode_attn": (8, 1, 200000, 200000),
                         "attn_tail": (1, seq, 200000, 200000 - seq)}[name]
        q = torch.empty((B, Lq, 128, 576), dtype=bf, device=dev)
        kv = torch.empty((B, Lk, 576), dtype=bf, device=dev)
        synth.fill_cuda(q, SEED, synth.Q, synth.NORMAL, 0, sigma=0.5)
        synth.fill_cuda(kv, SEED, synth.KV, synth.NORMAL, 0, sigma=0.5)
        # every row selects min(t, k) distinct positions below t (strided pattern)
        r = torch.arange(2048, device=dev, dtype=torch.int64)[None, :]
        t = torch.arange(Lq, device=dev, dtype=torch.int64)[:, None] + sp
        pos = (r * 7919) % t.clamp(min=1)
        idx = torch.where(r < t, pos, torch.full_like(pos, -1)).to(torch.int32)[None].expand(B, Lq, 2048).contiguous()
        out = torch.empty((B, Lq, 128, 512), dtype=bf, device=dev)
        run = lambda: dsa.sparse_attn(q, kv, kv, idx, 1 / math.sqrt(576), D_v=512, start_pos=sp, out=out)
    elif name == "decode_step":
        # the whole decode step (48 layers, 1/4 F, B = 8 at 200,000 cached
        # tokens), eager, for launch lists: `reps` steps after one warm-up step
        D = DECODE
        B, ctx, kd = D["B"], D["ctx"], D["k"]
        dpat = pattern_of(D["layers"], D["ratio"])
        qi, ki, wi, qs, kvs = {}, {}, {}, [], []
        for l, role in enumerate(dpat):
            if role == "F":
                qi[l] = torch.empty((B, 1, D["H_I"], D["d_I"]), dtype=bf, device=dev)
                ki[l] = torch.empty((B, ctx, D["d_I"]), dtype=bf, device=dev)
                wi[l] = torch.empty((B, 1, D["H_I"]), dtype=torch.float32, device=dev)
                synth.fill_cuda(qi[l], SEED, synth.Q_IDX, synth.INT9, l)
                synth.fill_cuda(ki[l], SEED, synth.K_IDX, synth.INT9, l)
                synth.fill_cuda(wi[l], SEED, synth.W, synth.POW2W, l)
            t = torch.empty((B, 1, D["n_h"], D["D_qk"]), dtype=bf, device=dev)
            synth.fill_cuda(t, SEED, synth.Q, synth.NORMAL, l, sigma=0.5)
            qs.append(t)
            t = torch.empty((B, ctx, D["D_qk"]), dtype=bf, device=dev)
            synth.fill_cuda(t, SEED, synth.KV, synth.NORMAL, l, sigma=0.5)
            kvs.append(t)
        dout = torch.empty((B, 1, D["n_h"], D["D_v"]), dtype=bf, device=dev)
        didx = torch.empty((B, 1, kd), dtype=torch.int32, device=dev)
        dws = torch.empty(max(dsa.indexer_topk_workspace(B, 1, ctx, ctx, D["H_I"], D["d_I"], kd),
                              dsa.sparse_attn_workspace(B, 1, D["n_h"], D["D_v"], kd)), dtype=torch.uint8, device=dev)
        scale = 1 / math.sqrt(D["D_qk"])

        def run():
            for l, role in enumerate(dpat):
                if role == "F":
                    dsa.indexer_topk(qi[l], ki[l], wi[l], kd, start_pos=ctx, out=didx, ws=dws)
                dsa.sparse_attn(qs[l], kvs[l], kvs[l], didx, scale, D_v=D["D_v"], start_pos=ctx, out=dout, ws=dws)
    else:
        raise SystemExit(f"unknown kernel case {name}")
    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    dsa.check_device_errors()
    print(f"{name} seq={seq}: {e0.elapsed_time(e1) / reps:.3f} ms/launch", flush=True)


def lowprec_case(seq, kk=2048, reps=2):
    """The low-precision selector ([IDX] §5.4) against the exact one on
    normal inputs (B = 1, L = seq, 64 indexer heads x 128, k = kk): Recall@k
    of each format's selection over the rows t >= k, and CUDA-event times of
    the bf16 indexer and of both formats.  Prints one JSON line."""
    import torch

    from sparse_attention_13_b200 import dsa, synth
    dev = torch.device("cuda", 0)
    L = seq
    q = torch.empty((1, L, 64, 128), dtype=torch.bfloat16, device=dev)
    kt = torch.empty((1, L, 128), dtype=torch.bfloat16, device=dev)
    w = torch.empty((1, L, 64), dtype=torch.float32, device=dev)
    synth.fill_cuda(q, SEED, synth.Q_IDX, synth.NORMAL, 0, sigma=1.0)
    synth.fill_cuda(kt, SEED, synth.K_IDX, synth.NORMAL, 0, sigma=1.0)
    synth.fill_cuda(w, SEED, synth.W, synth.NORMAL, 0, sigma=1.0)
    w = w.abs() / 64.0  # positive head weights (the softmax-normalised gates of the pages' indexer)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        e0.record()
        for _ in range(reps):
            r = fn()
        e1.record()
        torch.cuda.synchronize()
        return r, e0.elapsed_time(e1) / reps

    ws = torch.empty(dsa.indexer_topk_workspace(1, L, L, 0, 64, 128, kk), dtype=torch.uint8, device=dev)
    exact, t_exact = timed(lambda: dsa.indexer_topk(q, kt, w, kk, ws=ws))
    exact = exact.clone()
    res = {"tool": "lowprec_selector", "workload": f"B=1, L={L}, H_I=64, d_I=128, k={kk}, normal q/k (sigma 1), "
           "positive head weights", "data": "synthetic", "bf16_ms": t_exact}
    for fmt in ("e4m3", "e2m1"):
        lws = torch.empty(dsa.indexer_topk_lowprec_workspace(1, L, L, 0, 64, 128, kk, fmt), dtype=torch.uint8,
                          device=dev)
        sel, t = timed(lambda: dsa.indexer_topk_lowprec(q, kt, w, kk, fmt=fmt, ws=lws))
        inter = dsa.index_overlap(exact[:, kk:].contiguous(), sel[:, kk:].contiguous())
        res[fmt] = {"ms": t, "speedup_vs_bf16": t_exact / t,
                    "recall_at_k": float(inter.float().mean()) / kk}
    dsa.check_device_errors()
    print(json.dumps(res), flush=True)


def csa_layer(seq, kk=512, m=4, reps=2):
    """One CSA-style layer ([IDX] §5.2, the V4 settings of §5.3: m = 4, 64
    indexer heads x 128, k = 512) at B = 1, L = seq: the indexer over the
    floor(t/m) visible compressed blocks with top-k, then MLA attention over
    the selected compressed entries.  Synthetic compressed keys and latent
    entries (the gated compression needs weights).  Prints one JSON line with
    CUDA-event times per call and the tensor-pipe roofline of each."""
    import torch

    from sparse_attention_13_b200 import dsa, synth
    dev = torch.device("cuda", 0)
    bf = torch.bfloat16
    L, H, dI = seq, 64, 128
    N = L // m
    qi = torch.empty((1, L, H, dI), dtype=bf, device=dev)
    kc = torch.empty((1, N, dI), dtype=bf, device=dev)
    w = torch.empty((1, L, H), dtype=torch.float32, device=dev)
    synth.fill_cuda(qi, SEED, synth.Q_IDX, synth.INT9, 0)
    synth.fill_cuda(kc, SEED, synth.K_IDX, synth.INT9, 0)
    synth.fill_cuda(w, SEED, synth.W, synth.POW2W, 0)
    idx = torch.empty((1, L, kk), dtype=torch.int32, device=dev)
    ws = torch.empty(dsa.csa_indexer_topk_workspace(1, L, N, 0, m, H, dI, kk), dtype=torch.uint8, device=dev)
    q = torch.empty((1, L, 128, 576), dtype=bf, device=dev)
    c = torch.empty((1, N, 576), dtype=bf, device=dev)
    synth.fill_cuda(q, SEED, synth.Q, synth.NORMAL, 0, sigma=0.5)
    synth.fill_cuda(c, SEED, synth.KV, synth.NORMAL, 0, sigma=0.5)
    out = torch.empty((1, L, 128, 512), dtype=bf, device=dev)
    aws = torch.empty(max(dsa.sparse_attn_workspace(1, L, 128, 512, kk), 16), dtype=torch.uint8, device=dev)
    scale = 1 / math.sqrt(576)
    run_idx = lambda: dsa.csa_indexer_topk(qi, kc, w, kk, m=m, out=idx, ws=ws)
    run_attn = lambda: dsa.csa_sparse_attn(q, c, idx, scale, m=m, D_v=512, out=out, ws=aws)

    def ms_of(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    t_idx, t_attn = ms_of(run_idx), ms_of(run_attn)
    dsa.check_device_errors()
    peak = measured_peaks()[1]
    pairs = sum(t // m for t in range(L))
    idx_flops = 2 * H * dI * pairs
    attn_flops = 2 * 128 * (576 + 512) * sum(min(t // m, kk) for t in range(L))
    print(json.dumps({
        "tool": "csa_layer", "workload": f"B=1, L={L}, m={m}, N_cmp={N}, k={kk}, indexer H_I=64 d_I=128, "
        "MLA 128 heads 576/512 over compressed entries", "data": "synthetic",
        "indexer_ms": t_idx, "attn_ms": t_attn,
        "indexer_roofline": {"bound": "tensor", "achieved": idx_flops / t_idx / 1e9, "unit": "TFLOP/s",
                             "peak": peak, "frac": idx_flops / t_idx / 1e9 / peak},
        "attn_roofline": {"bound": "tensor", "achieved": attn_flops / t_attn / 1e9, "unit": "TFLOP/s",
                          "peak": peak, "frac": attn_flops / t_attn / 1e9 / peak}}), flush=True)


def selection_quality(seq, layers=4, kk=2048):
    """The selection-quality tools of [IDX] §8 on a short correlated synthetic
    stack (B = 1, L = seq, `layers` layers, k = kk): per layer, the indexer's
    own selection S^(l), the oracle selection TopK over the head-averaged
    dense weights, CapturedMass@k and Recall@k of S^(l) and of the reused
    S^(0), and the adjacent-layer overlap |S^(l-1) & S^(l)| / k, both with
    the head weights redrawn per layer (the input recipe) and held at layer
    0's.  Prints one
    JSON line with the means (over rows t >= k, where selection matters) and
    each tool kernel's CUDA-event time."""
    import torch

    from sparse_attention_13_b200 import dsa, synth
    dev = torch.device("cuda", 0)
    bf = torch.bfloat16
    L, H, dI, n_h, Dqk = seq, 64, 128, 128, 576
    scale = 1 / math.sqrt(Dqk)
    times = {"dense_weights": 0.0, "topk_rows": 0.0, "index_overlap": 0.0, "captured_mass": 0.0}

    def timed(name, fn):
        e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
        e0.record()
        r = fn()
        e1.record()
        e1.synchronize()
        times[name] += e0.elapsed_time(e1)
        return r

    rows = slice(kk, L)               # rows whose selection is a real choice
    n_sel = float(kk)
    res = []
    prev = first = prev_held = w0 = None
    ws = torch.empty(dsa.indexer_topk_workspace(1, L, L, 0, H, dI, kk), dtype=torch.uint8, device=dev)
    for l in range(layers):
        qi = torch.empty((1, L, H, dI), dtype=bf, device=dev)
        ki = torch.empty((1, L, dI), dtype=bf, device=dev)
        w = torch.empty((1, L, H), dtype=torch.float32, device=dev)
        q = torch.empty((1, L, n_h, Dqk), dtype=bf, device=dev)
        kv = torch.empty((1, L, Dqk), dtype=bf, device=dev)
        synth.fill_cuda(qi, SEED, synth.Q_IDX, synth.INT9, l, corr=True)
        synth.fill_cuda(ki, SEED, synth.K_IDX, synth.INT9, l, corr=True)
        synth.fill_cuda(w, SEED, synth.W, synth.POW2W, l)
        synth.fill_cuda(q, SEED, synth.Q, synth.NORMAL, l, sigma=0.5, corr=True)
        synth.fill_cuda(kv, SEED, synth.KV, synth.NORMAL, l, sigma=0.5, corr=True)
        own = dsa.indexer_topk(qi, ki, w, kk, ws=ws)
        first = own if first is None else first
        lse_d, mw = timed("dense_weights", lambda: dsa.dense_weights(q, kv, scale=scale))
        s_or = timed("topk_rows", lambda: dsa.topk_rows(mw, kk))
        entry = {"layer": l}
        for tag, sel in (("own", own), ("reused", first)):
            lse_s = torch.empty_like(lse_d)
            dsa.sparse_attn(q, kv, kv, sel, scale, D_v=512, lse=lse_s)
            mass = timed("captured_mass", lambda: dsa.captured_mass(lse_s, lse_d))
            inter = timed("index_overlap", lambda: dsa.index_overlap(s_or, sel))
            entry[f"captured_mass_{tag}"] = float(mass[0, rows].mean())
            entry[f"recall_{tag}"] = float(inter[0, rows].float().mean()) / n_sel
        if prev is not None:
            inter = timed("index_overlap", lambda: dsa.index_overlap(prev, own))
            entry["overlap_prev"] = float(inter[0, rows].float().mean()) / n_sel
        # the same layer with layer 0's head weights: the overlap then follows
        # the 0.9 correlation of q_idx and k_idx alone
        held = own if l == 0 else dsa.indexer_topk(qi, ki, w0, kk, ws=ws)
        if prev_held is not None:
            inter = timed("index_overlap", lambda: dsa.index_overlap(prev_held, held))
            entry["overlap_prev_w_held"] = float(inter[0, rows].float().mean()) / n_sel
        prev, prev_held = own, held
        w0 = w if l == 0 else w0
        res.append(entry)
    dsa.check_device_errors()
    flops = 2 * 2 * n_h * Dqk * (L * (L - 1) // 2)   # two passes of logits per dense call
    fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12          # FMA units x 2 flop x max clock
    dw_ms = times["dense_weights"] / layers
    print(json.dumps({
        "tool": "selection_quality", "workload": f"B=1, L={L}, {layers} correlated layers, k={kk}, "
        "indexer H_I=64 d_I=128, MLA 128 heads 576/512", "data": "synthetic",
        "per_layer": res, "ms_per_layer": {k: v / layers for k, v in times.items()},
        "dense_weights_roofline": {"bound": "alu", "achieved": flops / dw_ms / 1e9, "unit": "TFLOP/s",
                                   "peak": fp32_peak, "frac": flops / dw_ms / 1e9 / fp32_peak,
                                   "peak_kind": "fp32 FMA issue at 1965 MHz (derived)"}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--seq", type=int, default=0, help="override the prefill length (testing)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", default="",
                    help="profiling: indexer|indexer_tail|attn|attn_tail|decode_idx|decode_attn|decode_step; "
                         "quality runs the selection-quality tools, csa one CSA-style layer, "
                         "lowprec the low-precision selector's recall and times")
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--decode-steps", type=int, default=2000,
                    help="CUDA-graph replays in the decode timed region")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "zigzag"],
                    help="N > 1: independent replicas (weak scaling) or one sequence split into zig-zag "
                         "query chunks across the ranks (strong scaling)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the ratio sweep and the config-2/config-3 lines (short runs)")
    args = ap.parse_args()
    if args.kernel_case == "quality":
        selection_quality(args.seq or 8192)
        return
    if args.kernel_case == "lowprec":
        lowprec_case(args.seq or 65536, reps=args.reps)
        return
    if args.kernel_case == "csa":
        csa_layer(args.seq or 200000, reps=args.reps)
        return
    if args.kernel_case:
        kernel_case(args.kernel_case, args.seq or 16384, args.reps)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
        return
    rank, world, _ = dist_env()
    res = run_dsa(args)
    if rank != 0:
        return
    hbm_peak, tc_peak, peak_kind = res["peaks"]
    pf, dc = res["prefill"], res["decode"]
    attn_tr = traffic_for("mla_sparse_attn")
    idx_tr = traffic_for("indexer_topk")
    line = {
        "metric": METRIC, "value": pf["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": pf["ms_per_step"],
        "higher_is_better": True, "scaling": pf["scaling"], "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(world, args.shard),
        "roofline": {"bound": "tensor", "kernel": "mla_sparse_attn", "achieved": pf["attn_tflops"],
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": pf["attn_tflops"] / tc_peak,
                     "traffic": attn_tr, "peak_kind": f"{peak_kind} bf16 sustained",
                     "per_launch_flops": pf["attn_flops"], "avg_launch_ms": pf["attn_ms"]},
        "roofline_indexer": {"bound": "tensor", "kernel": "indexer_topk", "achieved": pf["idx_tflops"],
                             "peak": tc_peak, "unit": "TFLOP/s", "frac": pf["idx_tflops"] / tc_peak,
                             "traffic": idx_tr, "per_launch_flops": pf["idx_flops"],
                             "avg_launch_ms": pf["idx_ms"]},
        "indexer_share": pf["indexer_share"],
        "lowprec": {"workload": "one F layer of the prefill (L=200000, 64 x 128, k=2048), MX operands "
                                "quantised inside the call, bf16 scores; 1 warm-up + 2 launches",
                    "bf16_ms_per_launch": pf["idx_ms"], "formats": pf["lowprec"]},
        "sweep": {"workload": "prefill B=1, L=200000, 16 layers, F ratios 1/1 (F x16), 1/2 (FS x8), "
                              "1/4 (FSSS x4); indexer_ms_expected = M/N x the all-F indexer time per step",
                  "ratios": pf["sweep"]},
        "decode": {"ms_per_step": dc["ms_per_step"], "higher_is_better": False,
                   "timing": f"CUDA graph of the 48-layer step, {args.decode_steps} replays",
                   "gpu_launches": dc["launches"],
                   "idx_launch_ms": dc["idx_ms"], "attn_launch_ms": dc["attn_ms"],
                   "roofline": {"bound": "hbm", "achieved": dc["step_bytes"] / dc["ms_per_step"] / 1e6,
                                "peak": hbm_peak, "unit": "GB/s",
                                "frac": dc["step_bytes"] / dc["ms_per_step"] / 1e6 / hbm_peak,
                                "traffic": None, "per_step_bytes": dc["step_bytes"]},
                   "e2e": dc["e2e"], "clocks": dc["clocks"]},
        "e2e": pf["e2e"],
        "gpu_launches": pf["launches"],
        "clocks": pf["clocks"],
    }
    if "config2" in res:
        line["config2"] = res["config2"]
        line["config3"] = res["config3"]
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample()
        host_cores = os.cpu_count() or 1
        line["cpu_baseline"] = {"value": cb["prefill_tokens_per_s"], "unit": "tokens/s", "cores": 1,
                                "host_cores": host_cores,
                                "kind": "oracle", "sample": cb["sample"],
                                "decode_ms_per_step": cb["decode_ms_per_step"],
                                "decode_sample": cb["decode_sample"]}
        if host_cores > 1:
            line["cpu_baseline"]["row_parallel"] = oracle_parallel_sample(min(host_cores, 16))
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
