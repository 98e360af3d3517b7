#!/usr/bin/env python
"""Benchmark of the gradient-compression hot path on B200.

Workload: a flat fp32 gradient of 2^30 entries (4 GiB) per worker, Laplace(0, 1e-3) with 0.1%
Laplace(0, 1e-1) outliers, W = 2 workers resident on one GPU, residual carried from step to step.
One step:
  per worker: residual top-k at a 99% drop (keep 1/100), which first applies the previous step's
              quantisation error to the residual -> 2-bit quantisation (its error kept as a list for
              the next step) -> Golomb encode (b* = 6) -> Golomb decode
  then, per worker (the receive side): the worker-ordered sum G of the W decoded updates combined
              with the worker's own gradient, out_w = G + g_w, in one fused pass that never writes G
Metric: gradient GB/s compressed = W * 4 * n bytes per step / step time (whole job over all
ranks), with the residual-top-k call's share of HBM bandwidth reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--drop 0.99]
  python bench.py --exchange [--gpus N] ...   one worker per GPU, payloads all-gathered (NCCL)

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica of the step:
the path has no exchange on one node's simulated workers, so there is no collective in the data
path; the barrier and the max-over-ranks reduction use NCCL. Rank 0 prints one JSON line.
The reference arm is the CPU oracle (single thread) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "gradient GB/s compressed (top-1% residual select+compact)"
UNIT = "GB/s"
PROFILE = os.path.join(ROOT, "profiles", "pass1_ring_kernel_flat_fp32.md")
FALLBACK_HBM_GBS = 6650.0


def workload_config(n, workers, drop, b, extra=None):
    cfg = {"workload": f"flat fp32 gradient of {n} entries per worker, Laplace(0,1e-3) with 0.1% "
                       f"Laplace(0,1e-1) outliers, {workers} workers on one GPU, residual carried",
           "n": n, "workers": workers, "drop": drop, "keep": f"1/{round(1 / (1 - drop))}",
           "golomb_b": b, "step": "per worker: topk+quantise+golomb enc/dec; per worker: fused accumulate+combine",
           "l2": "inputs larger than L2 (8 GiB of gradients + 8 GiB of residuals per step)"}
    if extra:
        cfg.update(extra)
    return cfg


def keep_of(drop):
    den = round(1.0 / (1.0 - drop))
    return (1, den)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_text(src):
    """CUDA source with its comments and blank lines removed: edits to comments alone leave the
    compiled kernel, and so its counters, unchanged."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())


def source_sha():
    """First 16 hex digits of the sha256 of the code of select.cu followed by common.cuh."""
    h = hashlib.sha256()
    for f in ("select.cu", "common.cuh"):
        src = open(os.path.join(ROOT, "compressed_sgd_b200", "csrc", f)).read()
        h.update(code_text(src).encode())
    return h.hexdigest()[:16]


def profiled_traffic(n):
    """Per-launch DRAM bytes of the pass-1 kernel from the committed ncu summary, scaled to n
    entries; None if the summary is missing or the kernel source (select.cu and the shared
    common.cuh) changed since the capture."""
    try:
        text = open(PROFILE).read()
        sha = source_sha()
        m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
        m_b = re.search(r"dram_bytes_per_entry:\s*([0-9.]+)", text)
        if not m_sha or not m_b or m_sha.group(1) != sha:
            return None
        return float(m_b.group(1)) * n
    except Exception:
        return None


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = f"/tmp/gsparse_clocks_{os.getpid()}.csv"

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.index)], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.remove(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, dist, device):
    """Element-wise maximum of a list of floats over all ranks (every rank gets the result); a
    None entry (a leg that did not run) stays None. With dist None: the values themselves."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor([-1.0 if v is None else float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [None if v is None else float(x) for v, x in zip(values, t.tolist())]


# ---------------------------------------------------------------------------------------------
# our arm

def run_ours(args, rank, world, dist):
    import torch
    import compressed_sgd_b200 as gs
    import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    n, W = args.n, args.workers
    keep = keep_of(args.drop)
    b = gs.golomb_b_star(1.0 - args.drop)
    cap = gs.k_for(n, keep)
    chunk = gs.golomb_chunk_hint(cap)

    # inputs: generated on the host (pinned, for the end-to-end leg), copied once to the device
    g_host = []
    for w in range(W):
        t = torch.empty(n, dtype=torch.float32, pin_memory=True)
        t.numpy()[:] = synth.laplace_outliers(w + 2 * rank, n)
        g_host.append(t)
    g = [t.to(dev) for t in g_host]
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)]
    mom = args.momentum
    u = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if mom is not None else None
    # sent lists alternate between two buffers: step t applies step t-1's quantisation error
    idx2 = [[torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(W)] for _ in range(2)]
    val2 = [[torch.empty(cap, dtype=torch.float32, device=dev) for _ in range(W)] for _ in range(2)]
    fb2 = [[torch.empty(cap, dtype=torch.float32, device=dev) for _ in range(W)] for _ in range(2)]
    off2 = [[torch.zeros(2, dtype=torch.int64, device=dev) for _ in range(W)] for _ in range(2)]
    pend2 = [[gs.make_pending(idx2[p][w], fb2[p][w], off2[p][w][1:2], capacity=cap) for w in range(W)]
             for p in range(2)]
    parity = [0]
    sb = [torch.empty((cap + 31) // 32, dtype=torch.int32, device=dev) for _ in range(W)]
    means = [torch.empty(2, dtype=torch.float32, device=dev) for _ in range(W)]
    nwords = gs.golomb_word_capacity(cap, b, n)
    words = [torch.empty(nwords, dtype=torch.int32, device=dev) for _ in range(W)]
    nbits = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(W)]
    table = [torch.empty(((cap + chunk - 1) // chunk, 2), dtype=torch.int64, device=dev) for _ in range(W)]
    dec = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(W)]
    out = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    ws_t = [torch.empty(gs.residual_topk_workspace_size(n, 1, keep), dtype=torch.uint8, device=dev) for _ in range(W)]
    ws_q = [torch.empty(gs.lib().gsparse_quantize_workspace_size(cap), dtype=torch.uint8, device=dev) for _ in range(W)]
    ws_g = [torch.empty(gs.lib().gsparse_golomb_encode_workspace_size(cap), dtype=torch.uint8, device=dev)
            for _ in range(W)]
    ws_s = torch.empty(gs.lib().gsparse_accumulate_combine_workspace_size(W, n), dtype=torch.uint8, device=dev)
    st = gs.status_tensor(dev)
    lists2 = [[gs.make_list(dec[w], off2[p][w][1:2], val=val2[p][w], capacity=cap) for w in range(W)]
              for p in range(2)]
    # payload read back in the end-to-end leg: Golomb words, sign bits, means, bit count
    payload = [(words[w], sb[w], means[w], nbits[w], off2[0][w], off2[1][w]) for w in range(W)]
    payload_host = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in p] for p in payload]
    d2h_bytes = sum(t.numel() * t.element_size() for p in payload for t in p)
    h2d_bytes = W * n * 4

    stage_names = ["residual_topk", "quantize", "golomb_encode", "golomb_decode"]
    stage_ms = {k: [] for k in stage_names + ["receive"]}
    pass1_ms = []

    def step(events=None, p1=None):
        e = iter(events) if events is not None else None
        rec = (lambda: next(e).record()) if e is not None else (lambda: None)
        cur, prev = parity[0], 1 - parity[0]
        parity[0] = prev
        for w in range(W):
            idx, val, off, fb = idx2[cur][w], val2[cur][w], off2[cur][w], fb2[cur][w]
            end = off[1:2]
            rec()
            gs.residual_topk(g[w], r[w], keep, out_idx=idx, out_val=val, out_offsets=off, workspace=ws_t[w],
                             d_status=st, capacity=cap, pending=pend2[prev][w],
                             momentum=None if u is None else (u[w], mom),
                             pass_events=None if p1 is None else (p1[w][0], p1[w][1]))
            rec()
            gs.quantize(idx, val, end, write_dequantized=True, feedback_out=fb, sign_bits=sb[w], means=means[w],
                        workspace=ws_q[w], d_status=st, capacity=cap)
            rec()
            gs.golomb_encode(idx, end, b, n, chunk=chunk, words=words[w], nbits=nbits[w], table=table[w],
                             workspace=ws_g[w], d_status=st, capacity=cap)
            rec()
            gs.golomb_decode(words[w], nbits[w], end, cap, b, table=table[w], chunk=chunk, n_limit=n,
                             out_idx=dec[w], d_status=st)
        rec()
        for w in range(W):
            gs.accumulate_combine(lists2[cur], n, g[w], out=out[w], workspace=ws_s, d_status=st)
        rec()

    n_ev = 4 * W + 2

    def new_events(k):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
        for ev in evs:
            ev.record()       # materialise the CUDA event before handing it to the library
        return evs

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after warm-up")

    K = args.steps
    ev = [new_events(n_ev) for _ in range(K)]
    p1 = [[new_events(2) for _ in range(W)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(dev.index if dev.index is not None else 0)
    barrier()
    clocks.start()
    t0.record()
    for k in range(K):
        step(ev[k], p1[k])
    t1.record()
    barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / K
    for k in range(K):
        e = ev[k]
        for w in range(W):
            for s, name in enumerate(stage_names):
                stage_ms[name].append(e[4 * w + s].elapsed_time(e[4 * w + s + 1]))
            pass1_ms.append(p1[k][w][0].elapsed_time(p1[k][w][1]))
        stage_ms["receive"].append(e[4 * W].elapsed_time(e[4 * W + 1]))
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the timed region")
    if getattr(args, "step_hook", None) is not None:
        args.step_hook(step, dev)

    # kernels of this library launched per step, counted by the CUDA profiler on one extra step
    launches_per_step = None
    if not args.no_launch_count:
      try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize(dev)
        names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
        launches_per_step = len([x for x in names if "gs::" in x])
      except Exception:
        launches_per_step = None

    # end-to-end through the public API: pinned host gradients in, compressed payload out
    e2e_ms = None
    if args.e2e_steps > 0:
        def e2e_step():
            for w in range(W):
                g[w].copy_(g_host[w], non_blocking=True)
            step()
            for w in range(W):
                for src, dst in zip(payload[w], payload_host[w]):
                    dst.copy_(src, non_blocking=True)
        e2e_step()
        barrier()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        z.record()
        barrier()
        e2e_ms = a.elapsed_time(z) / args.e2e_steps

    # max over ranks
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], dist if world > 1 else None, dev)

    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    grad_bytes = world * W * 4 * n
    value = grad_bytes / (ms * 1e-3) / 1e9
    p1 = statistics.mean(pass1_ms)
    per_entry = 12 if mom is None else 20     # g, r read + r written (+ u read and written)
    p1_bytes = per_entry * n
    achieved = p1_bytes / (p1 * 1e-3) / 1e9
    topk_ms = statistics.mean(stage_ms["residual_topk"])
    topk_bytes = per_entry * n + 8 * cap
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(n, W, args.drop, b, {"parallelism": f"replicas x{world}"}
                                  if mom is None else {"parallelism": f"replicas x{world}", "momentum": mom}),
        "roofline": {"bound": "hbm", "kernel": "pass1_ring_kernel<1, " + ("momentum" if mom is not None else "two streams") + "> (streaming pass of residual top-k)",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": profiled_traffic(n) if mom is None else None,
                     "algorithmic_bytes_per_launch": p1_bytes, "launch_ms": round(p1, 4)},
        "residual_topk_call": {"ms": round(topk_ms, 4), "algorithmic_bytes": topk_bytes,
                               "gbs": round(topk_bytes / (topk_ms * 1e-3) / 1e9, 1),
                               "frac_of_peak": round(topk_bytes / (topk_ms * 1e-3) / 1e9 / peak, 4),
                               "frac_of_8000": round(topk_bytes / (topk_ms * 1e-3) / 1e9 / 8000.0, 4),
                               "gradient_gbs": round(4 * n / (topk_ms * 1e-3) / 1e9, 1)},
        "stages_ms": {k: round(statistics.median(v), 4) for k, v in stage_ms.items()},
        "gpu_launches": (launches_per_step * K) if launches_per_step is not None else None,
        "gpu_launches_per_step": launches_per_step,
        "clocks": clk,
    }
    if e2e_ms is not None:
        line["e2e"] = {"value": round(grad_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
                       "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                       "ms_per_step": round(e2e_ms, 3)}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args, args.cpu_n)
    return line


# ---------------------------------------------------------------------------------------------
# exchange between ranks: one worker per GPU

def run_exchange(args, rank, world, dist):
    """One worker per rank. Step per rank: residual top-k (with the previous step's quantisation
    error as pending writes) -> 2-bit quantisation (dequantised values sent) -> Golomb encode ->
    all-gather of the fixed-capacity payloads (NCCL; lengths travel in a device header, no host
    synchronisation) -> decode of every rank's stream -> fused receive of all ranks' updates in
    rank order combined with the rank's own gradient."""
    import torch
    import compressed_sgd_b200 as gs
    from compressed_sgd_b200 import exchange
    import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    n = args.n
    keep = keep_of(args.drop)
    b = gs.golomb_b_star(1.0 - args.drop)
    cap = gs.k_for(n, keep)
    chunk = gs.golomb_chunk_hint(cap)
    nch = (cap + chunk - 1) // chunk
    nwords = gs.golomb_word_capacity(cap, b, n)
    g = torch.from_numpy(synth.laplace_outliers(rank, n)).to(dev)
    r = torch.zeros(n, dtype=torch.float32, device=dev)
    out = torch.empty(n, dtype=torch.float32, device=dev)
    # two sets of send buffers: step t applies step t-1's quantisation error
    idx = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(2)]
    val = [torch.empty(cap, dtype=torch.float32, device=dev) for _ in range(2)]
    fb = [torch.empty(cap, dtype=torch.float32, device=dev) for _ in range(2)]
    # header: [0] stream bits (written by the encoder), [1:3] the top-k's offsets {0, K}
    meta = [torch.zeros(3, dtype=torch.int64, device=dev) for _ in range(2)]
    words = [torch.zeros(nwords, dtype=torch.int32, device=dev) for _ in range(2)]
    table = [torch.zeros(nch * 2, dtype=torch.int64, device=dev) for _ in range(2)]
    pend = [gs.make_pending(idx[p], fb[p], meta[p][2:3], capacity=cap) for p in range(2)]
    sb = torch.empty((cap + 31) // 32, dtype=torch.int32, device=dev)
    means = torch.empty(2, dtype=torch.float32, device=dev)
    ws_t = torch.empty(gs.residual_topk_workspace_size(n, 1, keep), dtype=torch.uint8, device=dev)
    ws_q = torch.empty(gs.lib().gsparse_quantize_workspace_size(cap), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(gs.lib().gsparse_golomb_encode_workspace_size(cap), dtype=torch.uint8, device=dev)
    ws_s = torch.empty(gs.lib().gsparse_accumulate_combine_workspace_size(world, n), dtype=torch.uint8,
                       device=dev)
    st = gs.status_tensor(dev)
    dec = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(world)]
    recv = [exchange.gather_buffers([words[p], table[p], val[p], meta[p]], world) for p in range(2)]
    parity = [0]

    def step(ev=None):
        rec = (lambda k: ev[k].record()) if ev is not None else (lambda k: None)
        cur, prev = parity[0], 1 - parity[0]
        parity[0] = prev
        rec(0)
        gs.residual_topk(g, r, keep, out_idx=idx[cur], out_val=val[cur], out_offsets=meta[cur][1:3],
                         workspace=ws_t, d_status=st, capacity=cap, pending=pend[prev])
        end = meta[cur][2:3]
        gs.quantize(idx[cur], val[cur], end, write_dequantized=True, feedback_out=fb[cur], sign_bits=sb,
                    means=means, workspace=ws_q, d_status=st, capacity=cap)
        gs.golomb_encode(idx[cur], end, b, n, chunk=chunk, words=words[cur], nbits=meta[cur][0:1],
                         table=table[cur].view(nch, 2), workspace=ws_g, d_status=st, capacity=cap)
        rec(1)
        rows = exchange.all_gather_fixed([words[cur], table[cur], val[cur], meta[cur]],
                                         dist if world > 1 else None, out=recv[cur])
        rec(2)
        lists = []
        for q in range(world):
            w_q, t_q, v_q, m_q = rows[q]
            gs.golomb_decode(w_q, m_q[0:1], m_q[2:3], cap, b, table=t_q.view(nch, 2), chunk=chunk, n_limit=n,
                             out_idx=dec[q], d_status=st)
            lists.append(gs.make_list(dec[q], m_q[2:3], val=v_q, capacity=cap))
        rec(3)
        gs.accumulate_combine(lists, n, g, out=out, workspace=ws_s, d_status=st)
        rec(4)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after warm-up")
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(dev.index if dev.index is not None else 0)
    barrier()
    clocks.start()
    t0.record()
    for k in range(K):
        step(evs[k])
    t1.record()
    barrier()
    clk = clocks.stop()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the timed region")
    ms = t0.elapsed_time(t1) / K
    names = ["compress", "all_gather", "decode", "receive"]
    stages = {nm: statistics.median(e[i].elapsed_time(e[i + 1]) for e in evs) for i, nm in enumerate(names)}
    # bytes of this rank's payload (used part) and of the padded buffers that cross the interconnect
    p = 1 - parity[0]
    m = [int(x) for x in meta[p].tolist()]
    used = ((m[0] + 31) // 32) * 4 + ((m[2] + chunk - 1) // chunk) * 16 + m[2] * 4 + 24
    padded = sum(t.numel() * t.element_size() for t in (words[p], table[p], val[p], meta[p]))
    vals = max_over_ranks([ms] + [stages[nm] for nm in names], dist if world > 1 else None, dev)
    if rank != 0:
        return None
    ms = vals[0]
    grad_bytes = world * 4 * n
    return {"metric": METRIC, "mode": "exchange", "value": round(grad_bytes / (ms * 1e-3) / 1e9, 2), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"flat fp32 gradient of {n} entries per rank (one worker per GPU), Laplace(0,1e-3) "
                                   f"with 0.1% Laplace(0,1e-1) outliers, residual carried",
                       "n": n, "drop": args.drop, "keep": f"1/{keep[1]}", "golomb_b": b,
                       "step": "per rank: topk+quantise+golomb encode; all-gather of fixed-capacity payloads; decode "
                               "of every rank's stream; fused receive of all ranks' updates + own gradient",
                       "parallelism": f"data parallel x{world}, NCCL all-gather" if world > 1 else "one rank"},
            "stages_ms": {nm: round(v, 4) for nm, v in zip(names, vals[1:])},
            "payload_bytes_per_rank": used, "padded_bytes_per_rank": padded,
            "clocks": clk}


# ---------------------------------------------------------------------------------------------
# the other workloads (one JSON line each; not the default line)

WORKLOADS = {
    "flat2e20": "flat fp32 gradient of 2^20 entries (95% N(0,1e-4^2), 5% N(0,1e-2^2)), 1 worker, global 99% "
                "drop; step: residual top-k, Golomb encode/decode (b*=6), scatter-accumulate",
    "mlp": "3-layer MNIST MLP gradient (1,863,690 entries, 6 tensors), 4 workers, per-tensor 99% drop; step per "
           "worker: residual top-k, 2-bit quantisation per tensor with error feedback; then scatter-accumulate",
    "nmt": "NMT-shaped gradient (147,337,216 entries), 4 workers, global 99% drop; step per worker: residual "
           "top-k; then per worker the fused receive (sum of the 4 updates + own gradient)",
    "resnet50": "ResNet-50-shaped gradient (25,557,032 entries, 161 tensors), 8 workers; round per worker: 9 "
                "accumulate-only steps, sparse binarisation p=0.001, Golomb encode/decode (b*=9); then "
                "scatter-accumulate of the 8 binarised updates",
}


def workload_oracle(name, g_host, n, seg, keep, b):
    """One step of a smaller workload through the CPU oracle (zero starting residual)."""
    import numpy as np
    import oracle
    oracle.build()
    W = len(g_host)
    T = 1 if seg is None else len(seg) - 1
    lists_h = []
    for w in range(W):
        rr = np.zeros(n, np.float32)
        if name == "resnet50":
            for _ in range(9):
                _, _, _, rr = oracle.residual_topk(g_host[w], rr, (0, 1))
            oi, ov, _, oo, rr = oracle.binarize(g_host[w], rr, keep)
        else:
            oi, ov, oo, rr = oracle.residual_topk(g_host[w], rr, keep, seg=seg)
        if name == "mlp":
            for s_ in range(T):
                bb, ee = int(oo[s_]), int(oo[s_ + 1])
                _, _, ov[bb:ee], rr = oracle.quantize(oi[bb:ee], ov[bb:ee], residual=rr, write_dequantized=True)
        if name in ("flat2e20", "resnet50"):
            ww, nb_, _ = oracle.golomb_encode(oi, b, chunk=64)
            oi = oracle.golomb_decode(ww, nb_, oi.size, b, n_limit=n)
        lists_h.append((oi, ov))
    dense_h, _, _ = oracle.scatter_accumulate(lists_h, n, merged=False)
    outs = [oracle.combine_local(dense_h, g_host[w]) for w in range(W)] if name == "nmt" else None
    return dense_h, outs


def run_workload(args):
    """Times one of the smaller workloads on cuda:0 and the oracle on the same step."""
    import numpy as np
    import torch
    import compressed_sgd_b200 as gs
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    name = args.workload
    keep = (1, 100)
    seg = None
    if name == "flat2e20":
        n, W = 1 << 20, 1
        gen = lambda w: synth.flat_mixture(n, seed=w)
    elif name == "mlp":
        seg = synth.offsets(synth.mlp_layout())
        n, W = int(seg[-1]), 4
        gen = lambda w: synth.mlp_gradient(w, 0)
    elif name == "nmt":
        n, W = int(synth.offsets(synth.nmt_layout())[-1]), 4
        gen = lambda w: synth.nmt_gradient(w, 0)
    else:
        n, W = int(synth.offsets(synth.resnet50_layout())[-1]), 8
        keep = (1, 1000)
        gen = lambda w: synth.resnet50_gradient(w, 0)
    T = 1 if seg is None else len(seg) - 1
    seg_d = None if seg is None else torch.from_numpy(seg).to(dev)
    b = gs.golomb_b_star(keep[0] / keep[1])
    cap = gs.k_for(n, keep) + (T if T > 1 else 0)
    g_host = [gen(w) for w in range(W)]
    g = [torch.from_numpy(x).to(dev) for x in g_host]
    r = [torch.zeros(n, device=dev) for _ in range(W)]
    st = gs.status_tensor(dev)
    idx = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(W)]
    val = [torch.empty(cap, device=dev) for _ in range(W)]
    off = [torch.zeros(T + 1, dtype=torch.int64, device=dev) for _ in range(W)]
    mean = [torch.zeros(T, device=dev) for _ in range(W)]
    words = [torch.empty(gs.golomb_word_capacity(cap, b, n), dtype=torch.int32, device=dev) for _ in range(W)]
    nbits = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(W)]
    chunk = gs.golomb_chunk_hint(cap)
    table = [torch.empty(((cap + chunk - 1) // chunk, 2), dtype=torch.int64, device=dev) for _ in range(W)]
    dec = [torch.empty(cap, dtype=torch.int32, device=dev) for _ in range(W)]
    out = [torch.empty(n, device=dev) for _ in range(W)]
    dense = torch.empty(n, device=dev)
    ws_t = torch.empty(max(gs.residual_topk_workspace_size(n, T, keep), gs.residual_topk_workspace_size(n, T, (0, 1)),
                           gs.binarize_workspace_size(n, 1, keep)), dtype=torch.uint8, device=dev)
    none_i = torch.empty(1, dtype=torch.int32, device=dev)
    none_v = torch.empty(1, device=dev)
    none_o = torch.zeros(2, dtype=torch.int64, device=dev)
    ws_q = torch.empty(gs.lib().gsparse_quantize_segments_workspace_size(cap, T), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(gs.lib().gsparse_golomb_encode_workspace_size(cap), dtype=torch.uint8, device=dev)
    ws_s = torch.empty(max(gs.lib().gsparse_scatter_accumulate_workspace_size(W, n),
                           gs.lib().gsparse_accumulate_combine_workspace_size(W, n)), dtype=torch.uint8, device=dev)
    sb = [torch.empty((cap + 31) // 32, dtype=torch.int32, device=dev) for _ in range(W)]
    means = [torch.empty(2 * T, device=dev) for _ in range(W)]

    def step(ev=None):
        rec = (lambda k: ev[k].record()) if ev is not None else (lambda k: None)
        rec(0)
        for w in range(W):
            if name == "resnet50":
                for _ in range(9):
                    gs.residual_topk(g[w], r[w], (0, 1), out_idx=none_i, out_val=none_v, out_offsets=none_o,
                                     workspace=ws_t, d_status=st, capacity=0)
                gs.binarize(g[w], r[w], keep, out_idx=idx[w], out_val=val[w], mean=mean[w], out_offsets=off[w],
                            workspace=ws_t, d_status=st, capacity=cap)
            else:
                gs.residual_topk(g[w], r[w], keep, seg_offsets=seg_d, out_idx=idx[w], out_val=val[w],
                                 out_offsets=off[w], workspace=ws_t, d_status=st, capacity=cap)
            if name == "mlp":
                # per-tensor means, all tensors in one call
                gs.quantize_segments(idx[w], val[w], off[w], residual=r[w], write_dequantized=True, sign_bits=sb[w],
                                     means=means[w], workspace=ws_q, d_status=st, capacity=cap)
            if name in ("flat2e20", "resnet50"):
                end = off[w][T:T + 1]
                gs.golomb_encode(idx[w], end, b, n, chunk=chunk, words=words[w], nbits=nbits[w], table=table[w],
                                 workspace=ws_g, d_status=st, capacity=cap)
                gs.golomb_decode(words[w], nbits[w], end, cap, b, table=table[w], chunk=chunk, n_limit=n,
                                 out_idx=dec[w], d_status=st)
        rec(1)
        src = dec if name in ("flat2e20", "resnet50") else idx
        lists = [gs.make_list(src[w], off[w][T:T + 1], val=val[w], capacity=cap) for w in range(W)]
        if name == "nmt":
            for w in range(W):
                gs.accumulate_combine(lists, n, g[w], out=out[w], workspace=ws_s, d_status=st)
        else:
            gs.scatter_accumulate(lists, n, dense_out=dense, workspace=ws_s, d_status=st, device=dev)
        rec(2)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(K):
        step(evs[k])
    t1.record()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())}")
    ms = t0.elapsed_time(t1) / K
    compress = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    receive = statistics.median(e[1].elapsed_time(e[2]) for e in evs)

    # the same step captured once as a CUDA graph and replayed (no host work per step)
    graph_ms = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(K):
            graph.replay()
        g1.record()
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} (graph replay)")
        graph_ms = g0.elapsed_time(g1) / K
        del graph

    # the oracle on the same step (first step, zero residual), single thread
    t = time.perf_counter()
    if not args.no_oracle:
        workload_oracle(name, g_host, n, seg, keep, b)
    oms = (time.perf_counter() - t) * 1e3
    grad = W * 4 * n
    # algorithmic HBM bytes of the step: every residual pass reads g and r and writes r (12 B per
    # entry); the receive writes the dense sum (scatter) or reads L and writes out per worker
    # (combine); the lists themselves are < 1% of that and left out
    passes = 10 if name == "resnet50" else 1
    algo = W * passes * 12 * n + (W * 8 * n if name == "nmt" else 4 * n)
    peak, peak_kind = measured_peaks()
    ach = algo / (ms * 1e-3) / 1e9
    return {"metric": METRIC, "workload": name, "description": WORKLOADS[name], "n": n, "workers": W,
            "value": round(grad / (ms * 1e-3) / 1e9, 2), "unit": UNIT, "ms_per_step": round(ms, 4),
            "roofline": {"bound": "hbm", "scope": "whole step", "achieved": round(ach, 1), "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach / peak, 4),
                         "algorithmic_bytes_per_step": algo},
            "stages_ms": {"compress": round(compress, 4), "receive": round(receive, 4)}, "steps": K,
            "graph": None if graph_ms is None else {
                "ms_per_step": round(graph_ms, 4), "value": round(grad / (graph_ms * 1e-3) / 1e9, 2),
                "what": "the same step captured once as a CUDA graph and replayed"},
            "oracle": None if args.no_oracle else {
                "ms_per_step": round(oms, 1), "value": round(grad / (oms * 1e-3) / 1e9, 4), "cores": 1,
                "sample": "the same step on the full workload, zero residual, single-threaded C++ oracle"}}


# ---------------------------------------------------------------------------------------------
# the CPU oracle (reference arm and cpu_baseline)

def oracle_step(gs_list, rs, keep, b, n, us=None, mom=None):
    import oracle
    lists = []
    for w, (g, r) in enumerate(zip(gs_list, rs)):
        if us is None:
            idx, val, off, r2 = oracle.residual_topk(g, r, keep)
        else:
            idx, val, off, r2, u2 = oracle.residual_topk_momentum(g, us[w], mom, r, keep)
            us[w][:] = u2
        bits, means, val, r2 = oracle.quantize(idx, val, residual=r2, write_dequantized=True)
        words, nb, table = oracle.golomb_encode(idx, b, chunk=64)
        dec = oracle.golomb_decode(words, nb, idx.size, b, n_limit=n)
        lists.append((dec, val))
        r[:] = r2
    dense, _, _ = oracle.scatter_accumulate(lists, n, merged=False)
    for g in gs_list:
        oracle.combine_local(dense, g)


def cpu_baseline(args, n_s):
    import oracle
    import synth
    oracle.build()
    keep = keep_of(args.drop)
    b = oracle.golomb_b_star(1.0 - args.drop)
    gsl = [synth.laplace_outliers(w, n_s) for w in range(args.workers)]
    rs = [np.zeros(n_s, np.float32) for _ in range(args.workers)]
    us = None if args.momentum is None else [np.zeros(n_s, np.float32) for _ in range(args.workers)]
    oracle_step(gsl, rs, keep, b, n_s, us, args.momentum)          # warm
    t = time.perf_counter()
    reps = 0
    while True:
        oracle_step(gsl, rs, keep, b, n_s, us, args.momentum)
        reps += 1
        if time.perf_counter() - t > 8.0 or reps >= 5:
            break
    dt = (time.perf_counter() - t) / reps
    return {"value": round(args.workers * 4 * n_s / dt / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"the same step on {n_s} entries per worker ({args.workers} workers), {reps} timed steps, "
                      f"single-threaded C++ oracle", "host_cpus": os.cpu_count()}


def run_reference(args):
    import oracle
    import synth
    oracle.build()
    keep = keep_of(args.drop)
    b = oracle.golomb_b_star(1.0 - args.drop)
    n_s = args.ref_n
    gsl = [synth.laplace_outliers(w, n_s) for w in range(args.workers)]
    rs = [np.zeros(n_s, np.float32) for _ in range(args.workers)]
    us = None if args.momentum is None else [np.zeros(n_s, np.float32) for _ in range(args.workers)]
    for _ in range(args.warmup):
        oracle_step(gsl, rs, keep, b, n_s, us, args.momentum)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(gsl, rs, keep, b, n_s, us, args.momentum)
    dt = (time.perf_counter() - t) / args.steps
    value = round(args.workers * 4 * n_s / dt / 1e9, 4)
    sample = (f"each step the full hot path on {n_s} entries per worker ({args.workers} workers) instead of "
              f"{args.n}; single-threaded C++ oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(args.n, args.workers, args.drop, b, {"sample_n": n_s}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--drop", type=float, default=0.99)
    ap.add_argument("--n", type=int, default=1 << 30)
    ap.add_argument("--workers", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-launch-count", action="store_true", help="skip the profiler-based kernel count")
    ap.add_argument("--cpu-n", type=int, default=1 << 24)
    ap.add_argument("--ref-n", type=int, default=1 << 20)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help="time one of the smaller workloads instead of the default flat 2^30 line")
    ap.add_argument("--no-oracle", action="store_true", help="with --workload: skip the oracle timing")
    ap.add_argument("--momentum", type=float, default=None,
                    help="momentum correction and masking in the residual top-k (e.g. 0.9); off by default")
    ap.add_argument("--no-graph", action="store_true", help="with --workload: skip the CUDA-graph replay leg")
    ap.add_argument("--exchange", action="store_true",
                    help="one worker per GPU with the compressed payloads all-gathered between ranks")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.workload is not None:
        if rank == 0:
            print(json.dumps(run_workload(args)), flush=True)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        line = run_exchange(args, rank, world, dist) if args.exchange else run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
