#!/usr/bin/env python
"""Benchmark of the B200 NSA forward pass.

Headline: NSA prefill of one 131,072-token video sequence (2048 frames x 64 tokens,
Hq=28, Hkv=4, d=128, l=32, s=16, l'=64, n=16, w=512, per-frame correlated keys) in
video tokens/s, with attended TFLOP/s against the measured bf16 peak; the 64 x 128K
decode's HBM GB/s is reported beside it. One step = one nsa_prefill call over inputs
already resident in HBM (every kernel of the path: pooling, compressed branch with
block scores, top-n, selected branch, window + gated combine). L2 is flushed (a
256 MiB write) before every timed step, outside the step's events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

With --gpus N > 1 and no launcher environment, the script starts N ranks itself
(torch.distributed.run on 127.0.0.1); under torchrun WORLD_SIZE must equal N. Each rank
runs its own sequence on its own GPU (independent problems, no collective on the data
path): value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_long_fwd_b200 import dist as dist_helpers  # noqa: E402
from sparse_attention_long_fwd_b200 import nsa  # noqa: E402
from sparse_attention_long_fwd_b200.inputs import (WORKLOADS, decode_inputs, gate_weights, phi_weights,  # noqa: E402
                                                   prefill_inputs)

METRIC = "NSA prefill video tokens/s at 128K & TFLOP/s vs peak; decode HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures, reported beside the measured-peak fractions: dense bf16 tensor
# throughput (the 2:4-sparse figure halved) and HBM3e bandwidth
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
PREFILL_STAGES = ["pool", "cmp_attn_scores", "topn", "sel_bucket", "sel_tile", "win", "sel_merge_combine",
                  "dense_text"]
# kernels of ours launched per prefill step: pool, compressed tile, top-n, bucket count / scan / scatter,
# selected tiles, window tile, merge + gated combine (+ the dense text tile)
PREFILL_KERNELS = 9
# DRAM bytes per launch of a stage's kernel on the 128K workload, from one ncu capture of the
# current kernel version (the full-size traffic summary kept with the profiles); an entry is
# removed when its kernel changes, and the roofline then reports traffic null.
STAGE_TRAFFIC_V128K = {"cmp_attn_scores": 4065668352}
DECODE_STAGES = ["dec_cmp_and_window", "dec_select", "dec_selected_and_combine"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------- work counts

def prefill_counts(w):
    """Attended keys per head for every query row, from the definition (no GPU output)."""
    t = np.arange(w.n_video, dtype=np.int64)
    nc = np.where(t + 1 >= w.cmp_len, (t + 1 - w.cmp_len) // w.cmp_stride + 1, 0)
    jt = t // w.sel_len
    nblk = np.minimum(w.top_n, jt + 1)
    sel = (nblk - 1) * w.sel_len + (t % w.sel_len) + 1
    win = np.minimum(w.window, t + 1)
    text = np.arange(w.n_video, w.n_tokens, dtype=np.int64) + 1
    per_key = 4.0 * w.d * w.hq  # QK^T and PV multiply-adds, 2 flops each
    return {
        "cmp_flops": per_key * nc.sum(), "sel_flops": per_key * sel.sum(), "win_flops": per_key * win.sum(),
        "text_flops": per_key * text.sum(),
        "keys_per_head": {"cmp": int(nc.sum()), "sel": int(sel.sum()), "win": int(win.sum()),
                          "text": int(text.sum())},
        "dense_causal_pairs": int(w.n_tokens) * (int(w.n_tokens) + 1) // 2,
    }


def decode_bytes(w, seq_lens, sel):
    """Algorithmic HBM bytes of one decode step: visible compressed K/V, the union of selected
    and window tokens of every (sequence, group), q, gates and the bf16 output."""
    row = w.d * 2
    total = 0
    for b in range(w.batch):
        L = int(seq_lens[b])
        nc = (L - w.cmp_len) // w.cmp_stride + 1 if L >= w.cmp_len else 0
        total += nc * w.hkv * row * 2
        for g in range(w.hkv):
            toks = np.zeros(L, dtype=bool)
            toks[max(0, L - w.window):] = True
            for j in sel[b, g]:
                if j >= 0:
                    toks[j * w.sel_len: min(L, (j + 1) * w.sel_len)] = True
            total += int(toks.sum()) * row * 2
    total += w.batch * w.hq * (w.d * 2 + 3 * 4 + w.d * 2)
    return total


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    FIELDS = ["pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device: int):
        self.bus = None
        try:
            pr = torch.cuda.get_device_properties(device)
            self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            pass
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = self.rows
        if self.bus is not None:
            mine = [r for r in rows if r[0].upper().endswith(self.bus[-12:])]
            rows = mine or rows
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


# ---------------------------------------------------------------------------- helpers

def dist_setup():
    world, rank, local = dist_helpers.rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    dist_helpers.init("nccl", 120, torch.device("cuda", local) if world > 1 else None)
    return world, rank, local


def barrier(world):
    dist_helpers.barrier(world)


def max_over_ranks(x: float, world: int) -> float:
    return dist_helpers.max_over_ranks(x, world, device="cuda")


def timed_steps(fn, steps, warmup, flush, n_stage_events):
    """Run warmup + timed steps; per step: flush L2 (untimed), events around fn()."""
    for _ in range(warmup):
        flush.zero_()
        fn(None)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_stage_events)] for _ in range(steps)]
    for ev in stage_ev:  # torch creates the CUDA event on its first record: do that before handing it over
        for e in ev:
            e.record()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record()
        fn(stage_ev[i])
        ends[i].record()
    torch.cuda.synchronize()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return step_ms, stage_ev


def stage_times(stage_ev, names, nrec):
    """Average duration of each recorded stage over the timed steps."""
    out = {}
    for j in range(min(nrec, len(names))):
        ms = [ev[j].elapsed_time(ev[j + 1]) for ev in stage_ev]
        out[names[j]] = sum(ms) / len(ms)
    return out


# ---------------------------------------------------------------------------- arms

def measure_prefill(w, q, k, v, g, args, world, peaks, peaks_src, flush, dev):
    """Time one nsa_prefill per step on workload w (inputs resident, L2 flushed before every
    step); returns the line's timing, stage times and the dominant stage's roofline."""
    counts = prefill_counts(w)
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_BF16)
    ws = nsa.alloc_workspace(p, False, dev)
    out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    has_text = w.n_tokens > w.n_video
    n_stages = (7 if w.n_video > 0 else 0) + (1 if has_text else 0)
    stage_names = (PREFILL_STAGES[:7] if w.n_video > 0 else []) + (["dense_text"] if has_text else [])

    def step(events):
        nsa.nsa_profile_stages(events or [])
        rc = nsa.nsa_prefill(q, k, v, g, p, out, None, ws, ws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_prefill")

    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    clocks.start()
    step_ms, stage_ev = timed_steps(step, args.steps, args.warmup, flush, n_stages + 1)
    clk = clocks.stop()
    nsa.nsa_profile_stages([])
    barrier(world)
    assert nsa.nsa_get_device_error(clear=True) == 0, "device error word set during the benchmark"
    ms_per_step = max_over_ranks(sum(step_ms), world) / args.steps
    stages = stage_times(stage_ev, stage_names, n_stages)
    flops = counts["cmp_flops"] + counts["sel_flops"] + counts["win_flops"] + counts["text_flops"]
    tflops = flops / (sum(step_ms) / args.steps / 1e3) / 1e12
    # the step lasts tens of milliseconds and the timed loop well under a second: the burst peak
    peak_t, peak_name = peaks["bf16_tflops"], "bf16_tflops (burst: the step is short)"
    dom = max(stages, key=stages.get)
    stage_flops = {"cmp_attn_scores": counts["cmp_flops"], "sel_tile": counts["sel_flops"],
                   "win": counts["win_flops"], "dense_text": counts["text_flops"]}
    if dom in stage_flops:
        ach = stage_flops[dom] / (stages[dom] / 1e3) / 1e12
        traffic = STAGE_TRAFFIC_V128K.get(dom) if w.name == "v128k" else None
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 2), "peak": peak_t, "unit": "TFLOP/s",
                    "frac": round(ach / peak_t, 4), "traffic": traffic,
                    "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, one full-size launch"
                    if traffic else None,
                    "peak_source": f"{peaks_src} {peak_name}",
                    "frac_of_datasheet": round(ach / DATASHEET["bf16_tflops"], 4),
                    "datasheet_peak": DATASHEET["bf16_tflops"],
                    "algorithmic": f"{stage_flops[dom]:.4e} FLOP per launch (attended keys only)"}
    else:
        roofline = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": None, "traffic": None}
    del ws, out
    return {"ms_per_step": ms_per_step, "stages": stages, "roofline": roofline, "clocks": clk, "counts": counts,
            "tflops": tflops, "peak_t": peak_t, "n_kernels": PREFILL_KERNELS * (w.n_video > 0) + has_text}


def measure_graph_replay(make_call, args, world, flush):
    """The same call captured once in a CUDA graph (after one direct call, which sets the kernels'
    attributes) and replayed once per step: the launch-bound small workloads lose their
    per-launch host cost. Returns ms per step, or None with the reason if capture fails."""
    call = make_call()
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(graph):
            call()
    except Exception as e:  # pragma: no cover - reported in the line instead
        return None, f"capture failed: {type(e).__name__}: {e}"
    barrier(world)
    step_ms, _ = timed_steps(lambda ev: graph.replay(), args.steps, args.warmup, flush, 0)
    torch.cuda.synchronize()
    del graph
    return max_over_ranks(sum(step_ms), world) / args.steps, None


def run_config_lines(args, dev, peaks, peaks_src, flush, world, rank):
    """The small prefill workloads, timed like the headline: the 2,048-token tiny case and
    the 36K hybrid (its 256 trailing text rows run the dense stage)."""
    lines = []
    for name in ("tiny", "qwen36k_hybrid"):
        w = WORKLOADS[name]
        q, k, v, g = prefill_inputs(w, seed=10 + rank, device=dev)
        m = measure_prefill(w, q, k, v, g, args, world, peaks, peaks_src, flush, dev)

        def make_call(w=w, q=q, k=k, v=v, g=g):
            p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len,
                                w.top_n, w.window, out_dtype=nsa.NSA_OUT_BF16)
            ws = nsa.alloc_workspace(p, False, dev)
            out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)

            def call():
                rc = nsa.nsa_prefill(q, k, v, g, p, out, None, ws, ws.numel())
                if rc != nsa.NSA_OK:
                    raise nsa.NsaError(rc, "nsa_prefill")
            return call

        gms, gerr = measure_graph_replay(make_call, args, world, flush)
        graph = ({"ms_per_step": round(gms, 4), "value": round(w.n_video * world / (gms / 1e3), 1),
                  "form": "one nsa_prefill call captured in a CUDA graph, replayed once per step"}
                 if gms is not None else {"unavailable": gerr})
        lines.append({
            "workload": name, "n_tokens": w.n_tokens, "n_video": w.n_video, "hq": w.hq, "hkv": w.hkv, "d": w.d,
            "top_n": w.top_n, "window": w.window, "ms_per_step": round(m["ms_per_step"], 4),
            "value": round(w.n_video * world / (m["ms_per_step"] / 1e3), 1), "unit": "video tokens/s",
            "all_tokens_per_s": round(w.n_tokens * world / (m["ms_per_step"] / 1e3), 1),
            "attended_tflops": round(m["tflops"], 2), "attended_frac_of_peak": round(m["tflops"] / m["peak_t"], 4),
            "stages_ms": {kk: round(vv, 4) for kk, vv in m["stages"].items()}, "roofline": m["roofline"],
            "graph_replay": graph,
            "launches": m["n_kernels"] * args.steps * (2 if gms is not None else 1)})
        del q, k, v, g
    return lines


VARLEN_KERNELS = 11  # table and gather kernels, then the nine NSA stages (all-video batch: no text stage)


def run_varlen(args, dev, peaks, flush, world, rank):
    """A serving batch: 64 all-video clips of 2,048 tokens packed back to back, one
    nsa_prefill_varlen call per step (every stage launched once for the whole batch)."""
    B, L = 64, 2048
    w = WORKLOADS["v128k"]
    from sparse_attention_long_fwd_b200.inputs import scaled
    wb = scaled(w, n_tokens=B * L, n_video=B * L)
    q, k, v, g = prefill_inputs(wb, seed=30 + rank, device=dev)
    cu = [b * L for b in range(B + 1)]
    nvs = [L] * B
    p = nsa.make_params(B * L, 0, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n, w.window,
                        out_dtype=nsa.NSA_OUT_BF16)
    need = nsa.nsa_prefill_varlen_workspace_size(p, cu, nvs)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    out = torch.empty((B * L, w.hq, w.d), dtype=torch.bfloat16, device=dev)

    def step(events):
        rc = nsa.nsa_prefill_varlen(q, k, v, g, cu, nvs, p, out, None, ws, need)
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_prefill_varlen")

    barrier(world)
    step_ms, _ = timed_steps(step, args.steps, args.warmup, flush, 0)
    assert nsa.nsa_get_device_error(clear=True) == 0, "device error word set during the varlen run"
    ms = max_over_ranks(sum(step_ms), world) / args.steps
    # attended FLOPs: each clip counted as its own 2,048-token sequence
    c = prefill_counts(scaled(w, n_tokens=L, n_video=L))
    flops = B * (c["cmp_flops"] + c["sel_flops"] + c["win_flops"])
    tf = flops / (ms / 1e3) / 1e12
    del ws, out, q, k, v, g
    return {"workload": f"{B} clips x {L} video tokens packed back to back (nsa_prefill_varlen), Hq={w.hq}, "
                        f"Hkv={w.hkv}, d={w.d}, n={w.top_n}, w={w.window}",
            "ms_per_step": round(ms, 4), "value": round(B * L * world / (ms / 1e3), 1), "unit": "video tokens/s",
            "attended_tflops": round(tf, 2), "attended_frac_of_peak": round(tf / peaks["bf16_tflops"], 4),
            "launches_per_step": VARLEN_KERNELS, "steps": args.steps, "warmup": args.warmup}


def run_b200(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peaks_src = load_peaks()
    w = WORKLOADS[args.workload]
    q, k, v, g = prefill_inputs(w, seed=2 + rank, device=dev)
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_BF16)
    ws = nsa.alloc_workspace(p, False, dev)
    out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n_kernels = PREFILL_KERNELS + (1 if w.n_tokens > w.n_video else 0)

    def step(events):
        nsa.nsa_profile_stages(events or [])
        rc = nsa.nsa_prefill(q, k, v, g, p, out, None, ws, ws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_prefill")

    m = measure_prefill(w, q, k, v, g, args, world, peaks, peaks_src, flush, dev)
    ms_per_step, stages, counts, peak_t = m["ms_per_step"], m["stages"], m["counts"], m["peak_t"]
    tokens = w.n_video * world
    value = dist_helpers.aggregate_rate(w.n_video, world, ms_per_step / 1e3)
    tflops = m["tflops"]

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "video tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: one {w.n_tokens}-token sequence ({w.n_tokens // 64} frames x 64 tokens), "
                               f"Hq={w.hq}, Hkv={w.hkv}, d={w.d}, l={w.cmp_len}, s={w.cmp_stride}, l'={w.sel_len}, "
                               f"n={w.top_n}, w={w.window}, bf16 in/out", "n_tokens": w.n_tokens,
                   "n_video": w.n_video, "top_n": w.top_n, "window": w.window,
                   "l2": "flushed (256 MiB write) before every timed step; inputs also exceed L2",
                   "parallelism": f"independent sequence per rank x{world}"},
        "attended_tflops": round(tflops, 2), "attended_frac_of_peak": round(tflops / peak_t, 4),
        "attended_frac_of_datasheet": round(tflops / DATASHEET["bf16_tflops"], 4),
        "attended_keys_per_head": counts["keys_per_head"],
        "attended_fraction_of_dense_pairs": round(sum(counts["keys_per_head"].values()) / counts["dense_causal_pairs"], 4),
        "stages_ms": {kk: round(vv, 4) for kk, vv in stages.items()},
        "roofline": m["roofline"], "clocks": m["clocks"], "gpu_launches": n_kernels * args.steps,
    }

    # end to end through the public call: pinned host inputs in, bf16 output back, every step.
    # Serving-style pipeline: while step i computes, step i+1's inputs upload on one copy stream
    # and step i-1's output downloads on another (two device buffer sets). Every step's bytes
    # cross PCIe inside the timed region; only their overlap with neighbouring steps differs
    # from the serial form, which is reported too.
    qh, kh, vh, gh = (t.cpu().pin_memory() for t in (q, k, v, g))
    outh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, gh))
    d2h = outh[0].numel() * outh[0].element_size()
    bufs = [(q, k, v, g, out), tuple(torch.empty_like(t) for t in (q, k, v, g, out))]
    comp = torch.cuda.current_stream()

    def e2e_serial_step(events):
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        g.copy_(gh, non_blocking=True)
        step(None)
        outh[0].copy_(out, non_blocking=True)

    barrier(world)
    e2e_ms, _ = timed_steps(e2e_serial_step, args.steps, min(args.warmup, 3), flush, 0)
    barrier(world)
    serial_total = max_over_ranks(sum(e2e_ms), world)

    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined(nsteps):
        ready = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        drained = [torch.cuda.Event() for _ in range(2)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(up)
        for i in range(nsteps):
            b = i % 2
            qd, kd, vd, gd, od = bufs[b]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[b])  # step i-2 has finished reading these inputs
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                gd.copy_(gh, non_blocking=True)
                ready[b].record(up)
            comp.wait_event(ready[b])
            if i >= 2:
                comp.wait_event(drained[b])  # step i-2's output has left this buffer
            rc = nsa.nsa_prefill(qd, kd, vd, gd, p, od, None, ws, ws.numel(), stream=comp.cuda_stream)
            if rc != nsa.NSA_OK:
                raise nsa.NsaError(rc, "nsa_prefill")
            computed[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                outh[b].copy_(od, non_blocking=True)
                drained[b].record(down)
        t1.record(down)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    barrier(world)
    pipelined(min(args.warmup, 3))
    pipe_ms = max_over_ranks(pipelined(args.steps), world)
    barrier(world)
    result["e2e"] = {"value": round(tokens / (pipe_ms / args.steps / 1e3), 1), "unit": "video tokens/s",
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                     "ms_per_step": round(pipe_ms / args.steps, 3),
                     "form": "pipelined: step i+1 uploads and step i-1 downloads while step i computes",
                     "serial": {"value": round(tokens / (serial_total / args.steps / 1e3), 1),
                                "ms_per_step": round(serial_total / args.steps, 3)}}
    result["gpu_launches_e2e"] = n_kernels * args.steps
    del qh, kh, vh, gh, outh, bufs

    if not args.no_sweep and w.name == "v128k":
        result["sweep"] = run_sweep(args, dev, q, k, v, g, flush, peak_t, world)
        result["gpu_launches"] += PREFILL_KERNELS * args.steps * len(result["sweep"]["points"])

    if not args.no_configs:
        result["configs"] = run_config_lines(args, dev, peaks, peaks_src, flush, world, rank)
        result["gpu_launches"] += sum(c["launches"] for c in result["configs"])
        result["varlen"] = run_varlen(args, dev, peaks, flush, world, rank)
        result["gpu_launches"] += VARLEN_KERNELS * args.steps

    if not args.no_decode:
        result["decode"] = run_decode(args, dev, peaks, peaks_src, flush, world)
        # the direct and the graph-replay timed loops
        result["gpu_launches"] += len(DECODE_STAGES) * result["decode"]["steps"] * (
            2 if "ms_per_step" in result["decode"]["graph_replay"] else 1)

    if not args.no_gates and w.name == "v128k":
        result["gates_and_phi"] = run_gates(args, dev, q, k, v, g, peaks, peaks_src, flush, world)
        result["gpu_launches"] += result["gates_and_phi"]["launches"]

    if not args.no_backward and w.n_video == w.n_tokens:
        result["backward"] = run_backward(args, dev, w, q, k, v, g, peaks, flush, world)
        result["gpu_launches"] += result["backward"]["launches"]

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, q, k, v, g, args.cpu_seconds)
    return result


SWEEP_POINTS = ("sweep128k_n4_w256", "sweep128k_n16_w512", "sweep128k_n48_w1024")


def run_sweep(args, dev, q, k, v, g, flush, peak_t, world):
    """Attended-key budget sweep at 128K: the same inputs, each (n, w) point timed like the headline."""
    ws = None
    points = []
    for name in SWEEP_POINTS:
        w = WORKLOADS[name]
        p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                            w.window, out_dtype=nsa.NSA_OUT_BF16)
        need = nsa.nsa_workspace_size(p, False)
        if ws is None or ws.numel() < need:
            ws = None
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
        out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)

        def step(events, p=p, out=out):
            rc = nsa.nsa_prefill(q, k, v, g, p, out, None, ws, ws.numel())
            if rc != nsa.NSA_OK:
                raise nsa.NsaError(rc, "nsa_prefill")

        barrier(world)
        step_ms, _ = timed_steps(step, args.steps, args.warmup, flush, 0)
        assert nsa.nsa_get_device_error(clear=True) == 0, "device error word set during the sweep"
        ms = max_over_ranks(sum(step_ms), world) / args.steps
        c = prefill_counts(w)
        flops = c["cmp_flops"] + c["sel_flops"] + c["win_flops"] + c["text_flops"]
        tf = flops / (ms / 1e3) / 1e12
        budget = sum(c["keys_per_head"].values()) / c["dense_causal_pairs"]
        points.append({"workload": name, "top_n": w.top_n, "window": w.window, "ms_per_step": round(ms, 4),
                       "value": round(w.n_video * world / (ms / 1e3), 1), "unit": "video tokens/s",
                       "attended_tflops": round(tf, 2), "attended_frac_of_peak": round(tf / peak_t, 4),
                       "attended_fraction_of_dense_pairs": round(budget, 4)})
        del out
    return {"points": points, "inputs": "the headline 128K tensors (same seed); only n and w change",
            "l2": "flushed before every timed step", "steps": args.steps, "warmup": args.warmup}


def run_gates(args, dev, q, k, v, g, peaks, peaks_src, flush, world):
    """The gate network over the 128K queries (one row per token and head) and the prefill
    with the learnable compression, on the headline tensors."""
    w = WORKLOADS["v128k"]
    rows, dim = w.n_tokens * w.hq, w.d
    w1, b1, w2, b2 = gate_weights(dim, seed=21, device=dev)
    gates = torch.empty((rows, 3), dtype=torch.float32, device=dev)

    def gate_step(events):
        rc = nsa.nsa_gate_mlp(q, w1, b1, w2, b2, rows, dim, gates)
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_gate_mlp")

    barrier(world)
    gms, _ = timed_steps(gate_step, args.steps, args.warmup, flush, 0)
    gate_ms = max_over_ranks(sum(gms), world) / args.steps
    gate_bytes = rows * dim * 2 + rows * 3 * 4 + w1.numel() * 2 + (b1.numel() + w2.numel() + b2.numel()) * 4
    gate_gbs = gate_bytes / (gate_ms / 1e3) / 1e9

    B, T, H = 1, w.n_tokens, w.hq
    pooled = torch.empty((B, 1, H, 3), dtype=torch.float32, device=dev)
    pws_n = nsa.nsa_gate_mlp_pooled_workspace_size(B, T, H, dim)
    pws = torch.empty(pws_n, dtype=torch.uint8, device=dev)

    def pooled_step(events):
        rc = nsa.nsa_gate_mlp_pooled(q, w1, b1, w2, b2, B, T, H, dim, 1, pooled, pws, pws_n)
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_gate_mlp_pooled")

    barrier(world)
    pms, _ = timed_steps(pooled_step, args.steps, args.warmup, flush, 0)
    pooled_ms = max_over_ranks(sum(pms), world) / args.steps
    pooled_gbs = rows * dim * 2 / (pooled_ms / 1e3) / 1e9

    phi = phi_weights(w.hkv, w.cmp_len, seed=22, device=dev)
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_BF16)
    ws = nsa.alloc_workspace(p, False, dev)
    out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)

    def phi_step(events):
        rc = nsa.nsa_prefill_phi(q, k, v, g, phi[0], phi[1], p, out, None, ws, ws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_prefill_phi")

    barrier(world)
    fms, _ = timed_steps(phi_step, args.steps, args.warmup, flush, 0)
    assert nsa.nsa_get_device_error(clear=True) == 0, "device error word set during the gate / phi runs"
    phi_ms = max_over_ranks(sum(fms), world) / args.steps
    hbm = peaks["hbm_gbs"]
    del ws, out, gates
    return {
        "gate_mlp": {"workload": f"{rows} rows (131,072 tokens x 28 heads) of d={dim}: W1 {dim // 2}x{dim} on the "
                                 "tensor cores, GELU, W2 3x{0}, softmax".format(dim // 2),
                     "ms": round(gate_ms, 4),
                     "roofline": {"bound": "hbm", "achieved": round(gate_gbs, 1), "peak": hbm, "unit": "GB/s",
                                  "frac": round(gate_gbs / hbm, 4), "peak_source": f"{peaks_src} hbm_gbs",
                                  "algorithmic": f"{gate_bytes} bytes per launch (x read once, gates written)"}},
        "gate_mlp_pooled": {"workload": "mean over 131,072 tokens per head (28 heads), then the MLP in fp64",
                            "ms": round(pooled_ms, 4), "hbm_gbs": round(pooled_gbs, 1),
                            "frac": round(pooled_gbs / hbm, 4)},
        "prefill_phi": {"workload": "the headline 128K prefill with the learnable compression",
                        "ms_per_step": round(phi_ms, 4),
                        "value": round(w.n_video * world / (phi_ms / 1e3), 1), "unit": "video tokens/s"},
        "steps": args.steps, "warmup": args.warmup, "l2": "flushed before every timed step",
        "launches": args.steps * (1 + 2 + PREFILL_KERNELS),
    }


# 128K, no text rows, the forward's statistics kept: pool, statistics, 3 bucket kernels, the
# selected key pass, the row pass, the selected dq merge, 2 key passes, pool backward
BACKWARD_KERNELS = 11


def run_backward(args, dev, w, q, k, v, g, peaks, flush, world):
    """nsa_backward on the prefill's tensors (the headline 128K ones by default; --workload v16k
    gives a small case for profiler captures), with the selection of one forward call and a
    N(0,1) dL/dout."""
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_BF16, keep_branch_stats=True)
    ws = nsa.alloc_workspace(p, False, dev)
    out = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((w.n_video, w.hkv, w.top_n), dtype=torch.int32, device=dev)

    def fwd(events):
        rc = nsa.nsa_prefill(q, k, v, g, p, out, sel, ws, ws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_prefill")

    # the forward that keeps every branch's statistics, timed too (its cost over the plain forward)
    fwd_ms, _ = timed_steps(fwd, args.steps, args.warmup, flush, 0)
    fwd_keep_ms = max_over_ranks(sum(fwd_ms), world) / args.steps
    del out  # ws keeps the forward's statistics
    gen = torch.Generator(device=dev).manual_seed(31)
    d_out = torch.randn((w.n_tokens, w.hq, w.d), generator=gen, device=dev).to(torch.bfloat16)
    dq = torch.empty((w.n_tokens, w.hq, w.d), dtype=torch.float32, device=dev)
    dk = torch.empty((w.n_tokens, w.hkv, w.d), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    dgates = torch.empty((w.n_tokens, w.hq, 3), dtype=torch.float32, device=dev)
    bws = torch.empty(nsa.nsa_backward_workspace_size(p), dtype=torch.uint8, device=dev)

    def step(events):
        rc = nsa.nsa_backward(q, k, v, g, d_out, sel, ws, ws.numel(), None, None, p, dq, dk, dv, dgates, bws,
                              bws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_backward")

    barrier(world)
    step_ms, _ = timed_steps(step, args.steps, args.warmup, flush, 0)
    assert nsa.nsa_get_device_error(clear=True) == 0, "device error word set during the backward"
    ms = max_over_ranks(sum(step_ms), world) / args.steps
    c = prefill_counts(w)
    # QK^T, dO V^T, P^T dO, dS K and dS^T Q against the forward's QK^T and PV: 2.5x its FLOPs
    flops = 2.5 * (c["cmp_flops"] + c["sel_flops"] + c["win_flops"] + c["text_flops"])
    tf = flops / (ms / 1e3) / 1e12
    # a step is tens of milliseconds and the timed loop well under a second, at the full SM clock:
    # the burst peak, as for the prefill
    peak = peaks["bf16_tflops"]
    del bws, dq, dk, dv, dgates, d_out, ws
    return {"workload": f"{w.name} backward: dq, dk, dv and the gates' gradient of the prefill "
                        "(its forward's selection held constant; every branch's statistics kept by that "
                        "forward and reused)",
            "forward_keeping_statistics_ms": round(fwd_keep_ms, 3),
            "ms_per_step": round(ms, 3), "value": round(w.n_video * world / (ms / 1e3), 1),
            "unit": "video tokens/s", "steps": args.steps, "warmup": args.warmup,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4),
                         "peak_source": "measured bf16_tflops (burst: sub-second timed loop)",
                         "frac_of_datasheet": round(tf / DATASHEET["bf16_tflops"], 4),
                         "algorithmic": f"{flops:.4e} FLOP per step (2.5x the forward's attended FLOPs)"},
            "launches": BACKWARD_KERNELS * args.steps}


def run_decode(args, dev, peaks, peaks_src, flush, world):
    w = WORKLOADS["decode64x128k"]
    if args.decode_batch != w.batch:
        from sparse_attention_long_fwd_b200.inputs import scaled
        w = scaled(w, batch=args.decode_batch)
    q, kc, vc, g, sl = decode_inputs(w, seed=4, device=dev)
    kcmp, vcmp = nsa.compress(kc, vc)
    p = nsa.make_params(w.n_tokens, w.n_tokens, w.hq, w.hkv, w.d, top_n=w.top_n, window=w.window,
                        out_dtype=nsa.NSA_OUT_BF16, batch=w.batch)
    ws = nsa.alloc_workspace(p, True, dev)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((w.batch, w.hkv, w.top_n), dtype=torch.int32, device=dev)

    def step(events):
        nsa.nsa_profile_stages(events or [])
        rc = nsa.nsa_decode(q, kc, vc, kcmp, vcmp, sl, g, p, out, sel, ws, ws.numel())
        if rc != nsa.NSA_OK:
            raise nsa.NsaError(rc, "nsa_decode")

    steps = max(args.steps, 20)
    # the step time is taken without stage events (an event between two kernels would hold
    # back the next kernel's early launch); a second pass records the stage boundaries
    step_ms, _ = timed_steps(lambda ev: step(None), steps, args.warmup, flush, 0)
    _, stage_ev = timed_steps(step, steps, 1, flush, len(DECODE_STAGES) + 1)
    nsa.nsa_profile_stages([])
    assert nsa.nsa_get_device_error(clear=True) == 0
    total = max_over_ranks(sum(step_ms), world)
    ms = total / steps
    nbytes = decode_bytes(w, sl.cpu().numpy(), sel.cpu().numpy())
    gbs = nbytes / (ms / 1e3) / 1e9
    stages = stage_times(stage_ev, DECODE_STAGES, len(DECODE_STAGES))

    def make_call():
        def call():
            rc = nsa.nsa_decode(q, kc, vc, kcmp, vcmp, sl, g, p, out, sel, ws, ws.numel())
            if rc != nsa.NSA_OK:
                raise nsa.NsaError(rc, "nsa_decode")
        return call

    gargs = argparse.Namespace(steps=steps, warmup=args.warmup)
    gms, gerr = measure_graph_replay(make_call, gargs, world, flush)
    graph = ({"ms_per_step": round(gms, 4), "hbm_gbs": round(nbytes / (gms / 1e3) / 1e9 * world, 1),
              "frac_of_peak": round(nbytes / (gms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
              "form": "one nsa_decode call captured in a CUDA graph (its dependent launches included), replayed "
                      "once per step"} if gms is not None else {"unavailable": gerr})
    assert nsa.nsa_get_device_error(clear=True) == 0
    # first kernel: the compressed cache read once, plus the window branch's K/V (its own CTAs)
    cmp_bytes = w.batch * ((w.n_tokens - 32) // 16 + 1) * w.hkv * w.d * 2 * 2
    cmp_bytes += w.batch * min(w.window, w.n_tokens) * w.hkv * w.d * 2 * 2
    cmp_gbs = cmp_bytes / (stages["dec_cmp_and_window"] / 1e3) / 1e9
    del kc, vc
    return {"workload": f"decode{w.batch}x128k: {w.batch} sequences x 131,072-token bf16 cache, Hq=28, Hkv=4, "
                        f"d=128, n=16, w=512",
            "ms_per_step": round(ms, 4), "hbm_gbs": round(gbs * world, 1), "unit": "GB/s",
            "algorithmic_bytes_per_step": nbytes, "frac_of_peak": round(gbs / peaks["hbm_gbs"], 4),
            "frac_of_datasheet": round(gbs / DATASHEET["hbm_gbs"], 4), "datasheet_gbs": DATASHEET["hbm_gbs"],
            "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peaks_src} hbm_gbs",
            "steps": steps, "stages_ms": {kk: round(vv, 4) for kk, vv in stages.items()},
            "graph_replay": graph,
            "dec_cmp_roofline": {"bound": "hbm", "achieved": round(cmp_gbs, 1), "peak": peaks["hbm_gbs"],
                                 "unit": "GB/s", "frac": round(cmp_gbs / peaks["hbm_gbs"], 4),
                                 "algorithmic": f"{cmp_bytes} bytes per launch (compressed K and V read once, "
                                                f"window K and V)"}}


def cpu_baseline(w, q, k, v, g, seconds):
    """The fp64 oracle, as it stands, on this host's cores over a stratified row sample."""
    from oracle import oracle as orc  # test infrastructure: the CPU baseline only
    from sparse_attention_long_fwd_b200.inputs import bf16_bits

    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    gh = g.cpu().numpy()
    cfg = orc.OracleConfig(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                           w.window)
    t0 = time.perf_counter()
    kc, vc = orc.compress(kb[: w.n_video]), orc.compress(vb[: w.n_video])
    t_cmp = time.perf_counter() - t0
    # probe, then size the sample for roughly `seconds` of work
    probe = np.linspace(0, w.n_video - 1, 32).astype(np.int32)
    t0 = time.perf_counter()
    orc.prefill_rows(cfg, qb, kb, vb, gh, probe, kc=kc, vc=vc, want=())
    t_probe = time.perf_counter() - t0
    nrows = int(min(w.n_video, max(64, 32 * seconds / max(t_probe, 1e-3))))
    rows = np.linspace(0, w.n_video - 1, nrows).astype(np.int32)
    t0 = time.perf_counter()
    orc.prefill_rows(cfg, qb, kb, vb, gh, rows, kc=kc, vc=vc, want=())
    t_rows = time.perf_counter() - t0
    est = t_cmp + t_rows * w.n_video / nrows
    return {"value": round(w.n_video / est, 2), "unit": "video tokens/s", "cores": orc.max_threads(), "kind": "oracle",
            "sample": f"{nrows} query rows evenly spaced over the {w.n_video}-token workload (all heads, all "
                      f"branches) plus the full compression; time extrapolated by rows",
            "seconds_measured": round(t_cmp + t_rows, 2)}


def run_reference(args, world, rank):
    """Reference arm: the fp64 oracle on the host cores, same workload and metric."""
    if rank != 0:
        return None
    from oracle import oracle as orc
    from sparse_attention_long_fwd_b200.inputs import bf16_bits

    w = WORKLOADS[args.workload]
    q, k, v, g = prefill_inputs(w, seed=2, device="cpu")
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    gh = g.numpy()
    cfg = orc.OracleConfig(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                           w.window)
    t0 = time.perf_counter()
    kc, vc = orc.compress(kb[: w.n_video]), orc.compress(vb[: w.n_video])
    t_cmp = time.perf_counter() - t0
    rows_per_step = 256
    rng = np.random.default_rng(0)
    times = []
    for i in range(args.warmup + args.steps):
        # stratified: one row from each of rows_per_step equal slices of the sequence
        edges = np.linspace(0, w.n_video, rows_per_step + 1).astype(np.int64)
        rows = np.array([rng.integers(a, max(a + 1, b)) for a, b in zip(edges[:-1], edges[1:])], dtype=np.int32)
        t0 = time.perf_counter()
        orc.prefill_rows(cfg, qb, kb, vb, gh, rows, kc=kc, vc=vc, want=())
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = statistics.mean(times) * w.n_video / rows_per_step + t_cmp
    value = w.n_video / per_step
    cores = orc.max_threads()
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "video tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{w.name}: one {w.n_tokens}-token sequence, Hq={w.hq}, Hkv={w.hkv}, d={w.d}, "
                               f"n={w.top_n}, w={w.window}", "n_tokens": w.n_tokens},
        "cpu_baseline": {"value": round(value, 2), "unit": "video tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {rows_per_step} rows, one per equal slice of the sequence, "
                                   f"extrapolated to all {w.n_video} rows, plus the full compression"},
        "e2e": {"value": round(value, 2), "unit": "video tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def relaunch_ranks(n: int) -> int:
    """Run this command again as n ranks on this node (torch.distributed.run, rendezvous on
    127.0.0.1); rank 0 prints the JSON line. Returns the launcher's exit status."""
    import socket

    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        port = sck.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="v128k", choices=[k for k, v in WORKLOADS.items() if not v.is_decode])
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 128K (n, w) budget sweep")
    ap.add_argument("--no-gates", action="store_true", help="skip the gate-network and learnable-compression lines")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-configs", action="store_true", help="skip the tiny and 36K-hybrid prefill lines")
    ap.add_argument("--decode-batch", type=int, default=64,
                    help="sequences of the decode line (a smaller batch for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "b200":
        ap.error("--warmup must be >= 3")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the ranks here when no launcher did
        sys.exit(relaunch_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} does not match the launcher's WORLD_SIZE={world}")
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    world, rank, local = dist_setup()
    try:
        res = run_b200(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
