#!/usr/bin/env python
"""Gated decode throughput of SP-KV on B200: tokens/s and effective KV GB/s at 32K context.

Workload (decode32k): batch 8, 32 query / 8 key-value heads, head_dim 128,
d_model 4096, utility perceptron 4096 -> 128 -> 8, window 128, tau 0.5, 32 layers,
32768 tokens already processed per row (per-head keep rates drawn in [5%, 50%]).
One step = one decode token for every batch row through all 32 layers: per layer
score the new token (a1), retire token t-128 into the gated cache if its gate is 1
and store the new token in the ring (a2, a3), and gated decode attention with the
split merge (a4, a5); by default the attention runs first, on the state before the
step's update (the new rows passed in), and a1-a3 follow on a second stream.  Steps are real consecutive decode steps (positions 32768,
32769, ...), each captured once in a CUDA graph; every step reads ~9.5 GB of K/V,
far more than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spkv|reference]

Under torchrun rank r serves its own batch shard, global rows 8r .. 8r+7 of a batch
of 8N (every input drawn by global row index; batch rows and key heads are independent:
no collective on the data path); the elapsed time is the max over ranks and ``value``
counts every rank's tokens.  ``--impl reference`` times the
fp64 CPU oracle on bounded samples of the same workload on rank 0.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated decode tokens/s and effective KV GB/s (% HBM peak) at 32K ctx"
WORKLOAD = "decode32k"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- distributed ----

def _dist_init():
    from sparse_decode_attention_spkv_b200 import dist as D
    return D.init("nccl")


def _barrier(world):
    from sparse_decode_attention_spkv_b200 import dist as D
    D.barrier(world)


def _max_over_ranks(x: float, world: int) -> float:
    from sparse_decode_attention_spkv_b200 import dist as D
    return D.max_over_ranks(x, world, device="cuda")


# ----------------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            pass
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "20"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # the timed region starts once the sampler is running (its first line is out)
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 3.0:
            if os.path.getsize(self.out.name) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.01)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------- GPU arm -------

def _code_hash(paths) -> str:
    """Hash of source files' code, line comments and blank lines left out (so that a
    comment edit does not orphan a profile taken on the same code)."""
    h = hashlib.sha256()
    for path in paths:
        with open(path) as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def _kernel_source_hash() -> str:
    """_code_hash of the decode kernels' sources."""
    return _code_hash(os.path.join(ROOT, "sparse_decode_attention_spkv_b200", "csrc", name)
                      for name in ("decode.cu", "decode_tc.cu", "common.cuh"))


def _profiled_traffic(launch_bytes: float):
    """DRAM bytes per decode launch from the committed ncu capture's key file
    (profiles/decode_attn_decode32k.json), if the capture was taken on the current
    kernel source (else None).  The capture is one layer of the same workload; its
    traffic is scaled to this launch by the algorithmic bytes."""
    path = os.path.join(ROOT, "profiles", "decode_attn_decode32k.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        key = json.load(f)
    if key.get("source_hash") != _kernel_source_hash() or "traffic_bytes_per_launch" not in key:
        return None
    traffic = float(key["traffic_bytes_per_launch"])
    if key.get("algorithmic_bytes_per_launch"):
        traffic *= launch_bytes / float(key["algorithmic_bytes_per_launch"])
    return traffic


def run_gpu(args, world, rank, local):
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import workloads as W

    device = torch.device("cuda", local)
    wl = W.WORKLOADS[WORKLOAD]
    layers = wl.layers
    K, Wm = args.steps, args.warmup
    R = 4  # steps with per-layer events, after the timed and end-to-end steps
    if Wm + K + R > wl.decode_steps:
        raise SystemExit(f"warmup+steps must be <= {wl.decode_steps - R}")
    E = max(0, min(args.e2e_steps, wl.decode_steps - R - Wm - K))  # what is left of the steps
    steps_total = Wm + K + E + R
    from sparse_decode_attention_spkv_b200.states import (DecodeStep, build_decode_state, kv_bytes,
                                                          kv_bytes_layers)
    # rank r: global batch rows r*B .. r*B + B-1 (disjoint shards, drawn by global row)
    p, Ls, inp = build_decode_state(wl, layers, steps_total, device, row0=rank * wl.B)
    T0 = wl.ctx[0]
    step = DecodeStep(p, Ls, device, split=args.decode_step != "fused",
                      attn_first=args.decode_step == "attn-first")

    # one eager decode-attention call per layer sets kernel attributes before capture
    for l, L in enumerate(Ls):
        S.spkv_decode_attn(p, L.cache, L.ring, inp["q"][0, l], inp["t"][0], step.o[l], step.lse[l], L.ws)
    torch.cuda.synchronize()

    # one graph per step; the timed steps carry no event inside (an event between two
    # launches keeps the second from starting before the first ends, so every layer
    # keeps its programmatic overlap).  The roofline divides the step time by the 32
    # decode-attention calls on the main stream; the last R steps, after the timed and
    # end-to-end ones, bracket the call of every 4th layer with events (each such call
    # then runs without overlap: the isolated duration, reported beside it).
    timed_layers = list(range(0, layers, 4))
    graphs = []
    for i in range(Wm + K):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.launch(inp["h"][i], inp["q"][i], inp["k"][i], inp["v"][i], inp["t"][i])
        graphs.append(g)
    torch.cuda.synchronize()

    for i in range(Wm):
        graphs[i].replay()
    torch.cuda.synchronize()
    bytes_before = kv_bytes(p, Ls, T0 + Wm)
    lbytes_before = kv_bytes_layers(p, Ls, T0 + Wm)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    with clocks:
        _barrier(world)
        torch.cuda.synchronize()
        start.record()
        for i in range(Wm, Wm + K):
            graphs[i].replay()
        end.record()
        torch.cuda.synchronize()
        _barrier(world)
    elapsed_ms = start.elapsed_time(end)
    bytes_after = kv_bytes(p, Ls, T0 + Wm + K - 1)
    lbytes_after = kv_bytes_layers(p, Ls, T0 + Wm + K - 1)
    step_bytes = 0.5 * (bytes_before + bytes_after)
    # algorithmic bytes of an average decode-attention call of the timed steps, and the
    # call's average duration in the pipeline (timed-step time / calls per step)
    launch_bytes = sum(0.5 * (lbytes_before[l] + lbytes_after[l]) for l in range(layers)) / layers
    elapsed_max = _max_over_ranks(elapsed_ms, world)
    attn_avg_ms = elapsed_max / K / layers
    for L in Ls:
        status, flags = S.spkv_cache_check(L.cache)
        if status != S.OK:
            raise RuntimeError(f"device error after timing: {S.status_str(status)} flags={flags}")
    if not torch.isfinite(step.o.float()).all():
        raise RuntimeError("non-finite decode output")

    # ---- end to end: host inputs in, host outputs back, every step -------------------
    # Two input/output buffer sets, each with its own captured step: step j's inputs are
    # copied in (pinned host memory, a copy stream) while step j-1 computes, and step j's
    # output is read back (another copy stream) while step j+1 computes.  A buffer set is
    # rewritten only after the step that used it has finished and its output is back.
    e2e = None
    if E > 0:
        keys = ("h", "q", "k", "v", "t")
        host = {k: inp[k][Wm + K:].cpu().pin_memory() for k in keys}
        o_host = torch.empty((E,) + tuple(step.o.shape), dtype=step.o.dtype).pin_memory()
        steps2 = [step, DecodeStep(p, Ls, device, split=step.split, attn_first=step.attn_first)]
        bufs = [{k: torch.empty_like(inp[k][0]) for k in keys} for _ in range(2)]
        g2 = []
        for b in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                steps2[b].launch(*(bufs[b][k] for k in keys))
            g2.append(g)
        torch.cuda.synchronize()
        comp = torch.cuda.current_stream()
        copy_in, copy_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(E)]
        ev_done = [torch.cuda.Event() for _ in range(E)]
        ev_out = [torch.cuda.Event() for _ in range(E)]
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _barrier(world)
        torch.cuda.synchronize()
        s0.record(comp)
        copy_in.wait_stream(comp)
        for j in range(E):
            b = j % 2
            with torch.cuda.stream(copy_in):
                if j >= 2:
                    copy_in.wait_event(ev_done[j - 2])  # the step that read bufs[b] is done
                for k_ in keys:
                    bufs[b][k_].copy_(host[k_][j], non_blocking=True)
                ev_in[j].record(copy_in)
            comp.wait_event(ev_in[j])
            if j >= 2:
                comp.wait_event(ev_out[j - 2])  # steps2[b].o of step j-2 is back on the host
            g2[b].replay()
            ev_done[j].record(comp)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(ev_done[j])
                o_host[j].copy_(steps2[b].o, non_blocking=True)
                ev_out[j].record(copy_out)
        comp.wait_event(ev_out[E - 1])
        s1.record(comp)
        torch.cuda.synchronize()
        _barrier(world)
        e2e_ms = _max_over_ranks(s0.elapsed_time(s1), world)
        h2d = sum(host[k_][0].numel() * host[k_][0].element_size() for k_ in host)
        d2h = step.o.numel() * step.o.element_size()
        if not torch.isfinite(o_host.float()).all():
            raise RuntimeError("non-finite decode output read back")
        e2e = {"value": world * p.B * E / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": E,
               "overlap": "inputs of step j copied in during step j-1, output of step j read "
                          "back during step j+1 (two buffer sets, pinned host memory)"}
        del g2
    del graphs

    # ---- isolated call timing: events around the call of every 4th layer ---------------
    i0 = Wm + K + E
    lb_iso = kv_bytes_layers(p, Ls, T0 + i0)
    iso = []
    for i in range(i0, i0 + R):
        ev = {l: (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True)) for l in timed_layers}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.launch(inp["h"][i], inp["q"][i], inp["k"][i], inp["v"][i], inp["t"][i], ev)
        g.replay()
        torch.cuda.synchronize()
        iso += [ev[l][0].elapsed_time(ev[l][1]) for l in timed_layers]
        del g
    iso_ms = sum(iso) / len(iso)
    iso_bytes = sum(lb_iso[l] for l in timed_layers) / len(timed_layers)

    peak, peak_kind = _peaks()
    achieved = launch_bytes / (attn_avg_ms / 1e3) / 1e9
    traffic = _profiled_traffic(launch_bytes)
    tokens_s = world * p.B * K / (elapsed_max / 1e3)
    ms_step = elapsed_max / K
    live = sum(int(L.cache.count.sum().item()) for L in Ls)
    heads = layers * p.B * p.Hkv
    out = {
        "metric": METRIC, "value": tokens_s, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode32k: batch 8 x 32 layers, 32q/8kv heads, head_dim 128, "
                               "d_model 4096, utility MLP 4096->128->8, w=128, tau=0.5, 32768-token "
                               "context, per-head keep U[5%,50%], per-token retirement",
                   "decode_step": args.decode_step,
                   "global_batch": world * p.B, "seq_len": T0, "layers": layers,
                   "parallelism": f"batch shards x{world}: rank r serves global rows "
                                  f"{wl.B}r..{wl.B}r+{wl.B - 1} (no data-path collective)",
                   "l2": "inputs larger than L2 (every step reads all live K/V, ~GBs)"},
        "kv_gbs_effective": step_bytes / (ms_step / 1e3) / 1e9,
        "kv_bytes_per_step": step_bytes,
        "kv_density_nonlocal": (live / heads) / (T0 - p.window),
        "decode_attn_ms_avg": attn_avg_ms,
        "decode_attn_ms_isolated": iso_ms,
        "roofline": {"bound": "hbm", "kernel": "decode_attn", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": traffic, "algorithmic_bytes_per_launch": launch_bytes,
                     "timed_launches": f"the {layers} decode-attention calls (decode + merge) of "
                                       f"each timed step, back to back on the main stream: CUDA "
                                       f"events on that stream around the {K} timed steps, "
                                       f"duration per call = step time / {layers} (launch gaps "
                                       f"and the step's end included)",
                     "isolated": {"ms": iso_ms, "achieved": iso_bytes / (iso_ms / 1e3) / 1e9,
                                  "frac": iso_bytes / (iso_ms / 1e3) / 1e9 / peak,
                                  "how": f"events around the call of layers {timed_layers[0]},"
                                         f"{timed_layers[1] if len(timed_layers) > 1 else ''}.."
                                         f"{timed_layers[-1]} in {R} further steps (each such "
                                         f"call starts only after the previous kernel ends)"}},
        "gpu_launches": (DecodeStep.LAUNCHES_PER_LAYER + (1 if step.split else 0) + 1) * layers * K,
        "clocks": clocks.summary(),
        "e2e": e2e,
    }
    del Ls, inp, step
    torch.cuda.empty_cache()
    if not args.no_aux and world == 1:  # per-GPU kernel measurements: once, at N = 1
        out["aux"] = {"prefill16k": measure_prefill(device, reps=3),
                      "rethreshold_decode32k": measure_rethreshold(device),
                      "soft_attn_16k": measure_soft(device),
                      "hybrid_3to1_decode32k": measure_hybrid(device),
                      "ragged128k": measure_ragged(device),
                      "seqsplit_ragged128k": measure_seqsplit(device),
                      "serving_e2e": measure_serving(device)}
    return out


def measure_seqsplit(device, reps=20):
    """Secondary measurement: the sequence-split decode (f4) on one GPU.  The ragged128k
    state (one layer) is cut by position into two slices (split_bounds: the first slice
    the older rows, the second the newer rows and the window); each slice's attention
    (spkv_decode_attn_partial, fp32 o and lse) and the merge of the two
    (spkv_decode_merge) are timed against the unsplit attention of the same state
    (spkv_decode_attn).  Every call reads its slice's live K/V from HBM (286 MB in all,
    more than L2).  With one slice per GPU, a rank's share of a step is its slice's
    partial, the exchange of B x Hq x (head_dim + 1) floats, and the merge; the exchange
    is not measured here (one GPU)."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import seqsplit as SS
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    from sparse_decode_attention_spkv_b200.states import build_decode_state, kv_bytes

    wl = W.small_case("ragged128k", layers=1)
    (lo0, hi0), (lo1, hi1) = SS.split_bounds(wl.ctx, 2, wl.window)
    p, (LA,), inp = build_decode_state(wl, 1, 1, device, pos_range=(lo0, hi0), with_ring=False)
    _, (LB,), _ = build_decode_state(wl, 1, 1, device, pos_range=(lo1, hi1))
    _, (LF,), _ = build_decode_state(wl, 1, 1, device)
    t = inp["t"][0]
    h, q, k, v = inp["h"][0][0], inp["q"][0][0], inp["k"][0][0], inp["v"][0][0]
    R.decode_step(LF, t, h, q, k, v)  # the step's update; then only attention is timed
    u_t, z_t = R.score(LB, h, p.B)
    S.spkv_decode_append(p, LB.cache, LB.ring, t, k, v, z_t, u_t, 1)
    sls = [SS.SliceDecode(p, LA.cache, None, False, device),
           SS.SliceDecode(p, LB.cache, LB.ring, True, device)]
    o = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=device)
    o_parts = torch.empty((2, p.B, p.Hq, p.head_dim), dtype=torch.float32, device=device)
    lse_parts = torch.empty((2, p.B, p.Hq), dtype=torch.float32, device=device)

    def timed(fn):
        # the calls captured in one CUDA graph, so that the figure is device time, not the
        # host's launch rate (a merge is far shorter than a call from Python)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps

    unsplit = timed(lambda: S.spkv_decode_attn(p, LF.cache, LF.ring, q, t, o, lse, LF.ws))
    part = [timed(lambda i=i: S.spkv_decode_attn_partial(p, sls[i].cache, sls[i].ring, q, t,
                                                         sls[i].flags, o_parts[i], lse_parts[i],
                                                         sls[i].ws)) for i in range(2)]
    merge = timed(lambda: S.spkv_decode_merge(p, 2, o_parts, lse_parts, o, lse))
    both = timed(lambda: SS.merge_local(p, sls, q, t, o, lse))
    for L in (LA, LB, LF):
        status, flags = S.spkv_cache_check(L.cache)
        if status != S.OK:
            raise RuntimeError(f"seqsplit measurement: cache error {flags}")
    nbytes = kv_bytes(p, [LF], int(t.min().item()))
    peak, peak_kind = _peaks()
    return {"unit": "ms", "unsplit_ms": unsplit, "slice_ms": part, "merge_ms": merge,
            "two_slices_one_gpu_ms": both, "per_rank_compute_ms": max(part) + merge,
            "kv_bytes": nbytes, "unsplit_frac_of_hbm_peak": nbytes / (unsplit / 1e3) / 1e9 / peak,
            "peak_kind": peak_kind, "slices": [[lo0, hi0], [lo1, hi1]],
            "how": f"{reps} calls per figure captured in one CUDA graph, CUDA events around a "
                   f"replay; inputs larger than L2"}


def measure_prefill(device, reps=3):
    """Secondary measurement: the prefill16k chunked prefill (4 chunks of 4096: score,
    compact, gated prefill attention, ring update) timed end to end with CUDA events,
    and the prefill-attention kernel alone.  FLOPs are the live (query, key) pairs of
    Eq. (4): 4 * head_dim * Hq * sum_t |S(t)| (QK^T and PV, multiply-add = 2)."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen
    from sparse_decode_attention_spkv_b200.inputs import workloads as W

    wl = W.WORKLOADS["prefill16k"]
    T, chunk = wl.ctx[0], wl.chunk
    bf = torch.bfloat16
    p = S.make_params(1, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    L = R.Layer.create(p, torch.from_numpy(wl.w1(0)).to(bf).to(device),
                       torch.from_numpy(wl.b1(0)).to(device), torch.from_numpy(wl.w2(0)).to(device),
                       torch.from_numpy(wl.b2(0)).to(device), num_pages=wl.Hkv * R.pages_for(T),
                       max_pages_per_head=R.pages_for(T), device=device)
    Tt = wl.T_total
    n_ch = T // chunk
    hs = [torch.empty((1, chunk, wl.d_model), dtype=bf, device=device) for _ in range(n_ch)]
    qs = [torch.empty((1, chunk, wl.Hq, wl.head_dim), dtype=bf, device=device) for _ in range(n_ch)]
    ks = [torch.empty((1, chunk, wl.Hkv, wl.head_dim), dtype=bf, device=device) for _ in range(n_ch)]
    vs = [torch.empty_like(k) for k in ks]
    for i in range(n_ch):
        c0 = i * chunk
        D.fill_normal(hs[i], wl.key(0, gen.T_H), 1.0, offset=c0 * wl.d_model)
        D.fill_rope(qs[i], wl.key(0, gen.T_Q), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_rope(ks[i], wl.key(0, gen.T_K), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_normal(vs[i], wl.key(0, gen.T_V), wl.qkv_scale, offset=c0 * wl.Hkv * wl.head_dim)
    o = torch.empty((1, chunk, wl.Hq, wl.head_dim), dtype=bf, device=device)
    lse = torch.empty((1, chunk, wl.Hq), dtype=torch.float32, device=device)
    u = torch.empty((chunk, wl.Hkv), dtype=torch.float32, device=device)
    z = torch.empty((chunk, wl.Hkv), dtype=torch.uint8, device=device)
    src = [torch.full((1,), i * chunk, dtype=torch.int32, device=device) for i in range(n_ch)]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)

    def run(evs=None):
        for i in range(n_ch):
            S.spkv_score(p, hs[i], chunk, L.W1, L.b1, L.W2, L.b2, u, z)
            S.spkv_write_compact(p, L.cache, L.ring, S.SRC_CHUNK, ks[i], vs[i], z, u, src[i], chunk,
                                 chunk)
            if evs:
                evs[i][0].record()
            S.spkv_prefill_attn(p, L.cache, L.ring, qs[i], ks[i], vs[i], i * chunk, chunk, o, lse,
                                L.pf_ws)
            if evs:
                evs[i][1].record()
            S.spkv_ring_write(p, L.ring, ks[i], vs[i], z, u, chunk, src[i], chunk, chunk)

    totals, attn = [], []
    for r in range(reps + 1):
        S.spkv_cache_reset(p, L.cache, L.ring)
        flush.zero_()  # L2 flush: the chunk working set fits in L2
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_ch)]
        a, bE = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run(evs)
        bE.record()
        torch.cuda.synchronize()
        if r:  # the first pass is a warm-up
            totals.append(a.elapsed_time(bE))
            attn.append(sum(e0.elapsed_time(e1) for e0, e1 in evs))
    status, flags = S.spkv_cache_check(L.cache)
    if status != S.OK:
        raise RuntimeError(f"prefill measurement: {S.status_str(status)} flags={flags}")
    # live pairs: every query sees min(w, t+1) window keys and the cached keys with pos <= t-w
    pos = []
    for lst in R.cache_lists(L):
        pos.append(lst.astype("int64"))
    w = wl.window
    pairs_win = sum(min(w, t + 1) for t in range(T))
    pairs_cache = sum(int(np.maximum(0, T - (pp + w)).sum()) for pp in pos)
    flops = 4.0 * wl.head_dim * wl.G * (pairs_win * wl.Hkv + pairs_cache)
    # tile FLOPs: every 128-query x 128-key block the kernel computes (masked entries
    # included): per chunk, query tile and key head, the window band (from 128 keys
    # before the tile to its last query) and the cache blocks (two pages each) holding a
    # row with pos <= last query - w at the time of that chunk (its own rows included)
    qt, kb = 128, 128
    blocks = 0
    for c0 in range(0, T, chunk):
        for t0 in range(c0, c0 + chunk, qt):
            wfirst = t0 - w if t0 >= w else t0
            nwin = (t0 + qt - wfirst) // kb
            for pp in pos:
                n_any = int(np.sum(pp[pp < c0 + chunk] <= t0 + qt - 1 - w))
                blocks += nwin + (n_any + kb - 1) // kb
    tile_flops = 4.0 * wl.head_dim * wl.G * blocks * qt * kb
    t_total = statistics.median(totals) / 1e3
    t_attn = statistics.median(attn) / 1e3
    import json as _json
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) if os.path.exists(
            os.path.join(ROOT, "MEASURED_PEAKS.json")) else open(os.devnull) as f:
        txt = f.read()
    peak_tf = float(_json.loads(txt)["bf16_tflops"]) if txt else 1590.0
    return {"unit": "TFLOP/s", "live_pair_flops": flops, "ms_total": t_total * 1e3,
            "ms_prefill_attn": t_attn * 1e3, "tflops_total": flops / t_total / 1e12,
            "tflops_prefill_attn": flops / t_attn / 1e12, "tile_flops": tile_flops,
            "tile_tflops_prefill_attn": tile_flops / t_attn / 1e12,
            "roofline": {"bound": "tensor", "kernel": "prefill_attn",
                         "achieved": flops / t_attn / 1e12, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": flops / t_attn / 1e12 / peak_tf,
                         "peak_kind": "measured (burst)" if txt else "fallback"},
            "density_nonlocal": float(sum(len(pp) for pp in pos)) / (wl.Hkv * T),
            "l2": "512 MB buffer written before each repetition"}


def measure_rethreshold(device, reps=3):
    """Secondary measurement: post-hoc re-threshold (in-place stable compaction of every
    key head's cache by the stored utilities) of one decode32k layer at 32768-token
    context from tau = 0.5 to the median stored utility (about half the rows stay).
    The cache is restored from a device copy before each repetition (which also evicts
    it from L2).  Algorithmic bytes: every stored row read once (K, V, position,
    utility) and every kept row written once."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.states import build_decode_state
    from sparse_decode_attention_spkv_b200.inputs import workloads as W

    wl = W.small_case("decode32k", layers=1)
    p, Ls, _ = build_decode_state(wl, 1, 1, device, store_u=True)
    L = Ls[0]
    c = L.cache
    saved = {k: getattr(c, k).clone() for k in ("K_pool", "V_pool", "pos_pool", "u_pool",
                                                  "count", "count_prev", "page_table")}
    z_saved = L.ring.z_win.clone()
    # median utility of the stored rows (setup on the host side of the measurement)
    n_rows = c.count.tolist()
    vals = []
    table = c.page_table.cpu()
    for bh, n in enumerate(n_rows):
        idx = torch.arange(n)
        vals.append(c.u_pool[table[bh, idx // S.PAGE_ROWS].to(device).long(), (idx % S.PAGE_ROWS).to(device)])
    tau_new = float(torch.cat(vals).median().item())
    ws = S.alloc_rethreshold_workspace(p, c)
    times = []
    rows_before = int(saved["count"].sum().item())
    rows_after = 0
    for r in range(reps + 1):
        for k, v in saved.items():
            getattr(c, k).copy_(v)
        L.ring.z_win.copy_(z_saved)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        S.spkv_cache_rethreshold(p, c, L.ring, tau_new, ws)
        b.record()
        torch.cuda.synchronize()
        if r:
            times.append(a.elapsed_time(b))
        rows_after = int(c.count.sum().item())
    status, flags = S.spkv_cache_check(c)
    if status != S.OK:
        raise RuntimeError(f"rethreshold measurement: {S.status_str(status)} flags={flags}")
    row = 2 * p.head_dim * 2 + 8
    nbytes = rows_before * row + rows_after * row
    t = statistics.median(times) / 1e3
    peak, peak_kind = _peaks()
    return {"unit": "GB/s", "tau": [p.tau, tau_new], "rows_before": rows_before,
            "rows_after": rows_after, "ms": t * 1e3, "algorithmic_bytes": nbytes,
            "roofline": {"bound": "hbm", "kernel": "cache_rethreshold", "achieved": nbytes / t / 1e9,
                         "peak": peak, "unit": "GB/s", "frac": nbytes / t / 1e9 / peak,
                         "peak_kind": peak_kind}}


def measure_soft(device, reps=3, beta=0.01, c=1e6):
    """Secondary measurement: soft-gated training-time attention (Eqs. (5)-(6)) over one
    16384-token sequence with the prefill16k shapes (32 query / 8 key heads, head_dim
    128, RoPE'd q/k), the utilities from the utility perceptron of that workload.
    FLOPs: every (query, key <= query) pair of every query head, QK^T and PV:
    4 * head_dim * Hq * T (T + 1) / 2."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen
    from sparse_decode_attention_spkv_b200.inputs import workloads as W

    wl = W.WORKLOADS["prefill16k"]
    T = wl.ctx[0]
    bf = torch.bfloat16
    p = S.make_params(1, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    h = torch.empty((T, wl.d_model), dtype=bf, device=device)
    q = torch.empty((1, T, wl.Hq, wl.head_dim), dtype=bf, device=device)
    k = torch.empty((1, T, wl.Hkv, wl.head_dim), dtype=bf, device=device)
    v = torch.empty_like(k)
    D.fill_normal(h, wl.key(0, gen.T_H), 1.0)
    D.fill_rope(q, wl.key(0, gen.T_Q), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_rope(k, wl.key(0, gen.T_K), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_normal(v, wl.key(0, gen.T_V), wl.qkv_scale)
    W1 = torch.from_numpy(wl.w1(0)).to(bf).to(device)
    u = torch.empty((T, wl.Hkv), dtype=torch.float32, device=device)
    z = torch.empty((T, wl.Hkv), dtype=torch.uint8, device=device)
    S.spkv_score(p, h, T, W1, torch.from_numpy(wl.b1(0)).to(device),
                 torch.from_numpy(wl.w2(0)).to(device), torch.from_numpy(wl.b2(0)).to(device), u, z)
    o = torch.empty_like(q)
    lse = torch.empty((1, T, wl.Hq), dtype=torch.float32, device=device)
    ws = torch.empty(S.spkv_soft_attn_workspace_bytes(p, T), dtype=torch.uint8, device=device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    times = []
    for r in range(reps + 1):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        S.spkv_soft_attn(p, q, k, v, u, T, beta, c, o, lse, ws)
        b.record()
        torch.cuda.synchronize()
        if r:
            times.append(a.elapsed_time(b))
    if not torch.isfinite(o.float()).all():
        raise RuntimeError("soft attention: non-finite output")
    flops = 4.0 * wl.head_dim * wl.Hq * T * (T + 1) / 2
    t = statistics.median(times) / 1e3
    peak_tf = _bf16_peak()
    return {"unit": "TFLOP/s", "seq_len": T, "beta": beta, "c": c, "flops": flops,
            "ms": t * 1e3, "roofline": {"bound": "tensor", "kernel": "soft_attn",
                                        "achieved": flops / t / 1e12, "peak": peak_tf[0],
                                        "unit": "TFLOP/s", "frac": flops / t / 1e12 / peak_tf[0],
                                        "peak_kind": peak_tf[1]},
            "l2": "512 MB buffer written before each repetition"}


def _bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    return 1590.0, "fallback"


def measure_hybrid(device, steps=10, warmup=3, period=4):
    """Secondary measurement: per-token decode over a 32-layer hybrid local/global stack
    (SP-KV page §3.3 "Hybrids"): every 4th layer global with the decode32k gated cache
    (32768-token context; the 8 global layers are decode32k layers 0-7), the other 24
    local (window of 128, no cache).  Same batch, heads and step as the headline
    workload; graph-replayed steps timed with CUDA events."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    from sparse_decode_attention_spkv_b200.states import HybridStep, build_decode_state

    wl = W.WORKLOADS[WORKLOAD]
    n_layers = wl.layers
    n_glob = n_layers // period
    p, G, inp = build_decode_state(wl, n_glob, warmup + steps, device)
    loc = []
    for l in range(n_layers - n_glob):
        L = R.Layer.create_local(p, device)
        D.fill_normal(L.ring.K_win, wl.key(l, gen.T_K), wl.qkv_scale)
        D.fill_normal(L.ring.V_win, wl.key(l, gen.T_V), wl.qkv_scale)
        loc.append(L)
    step = HybridStep(p, G, loc, period, device)
    graphs = []
    for i in range(warmup + steps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.launch(inp["h"][i], inp["q"][i], inp["k"][i], inp["v"][i], inp["t"][i])
        graphs.append(g)
    torch.cuda.synchronize()
    for i in range(warmup):
        graphs[i].replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(warmup, warmup + steps):
        graphs[i].replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    for L in G:
        status, flags = S_check(L)
        if status:
            raise RuntimeError(f"hybrid measurement: cache error {flags}")
    del graphs
    # kernels per layer: decode + merge, the update, and (global layers) the scoring or
    # the fused score + update
    per_glob, per_loc = (4, 3) if step.attn_first else (3, 3)
    return {"unit": "tokens/s", "value": p.B / (ms / 1e3), "ms_per_step": ms,
            "layers": {"global": n_glob, "local": n_layers - n_glob, "period": period},
            "order": "attn-first" if step.attn_first else "update first",
            "launches_per_step": per_glob * n_glob + per_loc * (n_layers - n_glob)}


def measure_ragged(device, warmup=3, one_stream=True):
    """Secondary measurement: ragged128k (batch 4, contexts 128K / 96K / 64K / 32K, one
    layer, per-head keep 60% / 2% / 5-15%) per-token decode over the workload's 64 steps:
    every step attends (on the state before its update), then scores the new token,
    retires t - 128 and stores the new token (one_stream: one fused launch on the same
    stream, as a single layer's next attention needs the update anyway; else the
    retirement and the scoring on a second stream).  The timed steps are one CUDA graph
    (inputs drawn ahead in HBM; consecutive steps overlap through the programmatic
    launches, as a multi-layer model's do); the same steps replayed one graph per step
    are reported beside it.  Effective GB/s = live K/V bytes read per step / step time."""
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    from sparse_decode_attention_spkv_b200.states import DecodeStep, build_decode_state, kv_bytes

    wl = W.WORKLOADS["ragged128k"]
    steps = wl.decode_steps - warmup
    p, Ls, inp = build_decode_state(wl, 1, wl.decode_steps, device, store_u=False)
    L = Ls[0]
    state = [L.cache.K_pool, L.cache.V_pool, L.cache.pos_pool, L.cache.page_table, L.cache.count,
             L.cache.count_prev, L.cache.pool_top, L.cache.err_flag, L.ring.K_win, L.ring.V_win,
             L.ring.z_win]
    snap = [x.clone() for x in state]
    step = DecodeStep(p, Ls, device, split=not one_stream, attn_first=True,
                      inputs_settled=True)  # inputs drawn ahead in HBM
    S_ = __import__("sparse_decode_attention_spkv_b200.spkv", fromlist=["spkv"])
    S_.spkv_decode_attn(p, L.cache, L.ring, inp["q"][0][0], inp["t"][0], step.o[0], step.lse[0],
                        L.ws)  # kernel attributes, before capture
    torch.cuda.synchronize()

    def graph(i0, i1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(i0, i1):
                step.launch(inp["h"][i], inp["q"][i], inp["k"][i], inp["v"][i], inp["t"][i])
        return g

    g_warm, g_all = graph(0, warmup), graph(warmup, wl.decode_steps)
    g_each = [graph(i, i + 1) for i in range(warmup, wl.decode_steps)]
    torch.cuda.synchronize()
    results = {}
    for mode in ("one_graph", "graph_per_step"):
        for x, y in zip(state, snap):
            x.copy_(y)
        g_warm.replay()
        torch.cuda.synchronize()
        b0 = kv_bytes(p, Ls, min(wl.ctx) + warmup)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if mode == "one_graph":
            g_all.replay()
        else:
            for g in g_each:
                g.replay()
        b.record()
        torch.cuda.synchronize()
        b1 = kv_bytes(p, Ls, min(wl.ctx) + wl.decode_steps - 1)
        status, flags = S_check(L)
        if status:
            raise RuntimeError(f"ragged measurement: cache error {flags}")
        results[mode] = (a.elapsed_time(b) / steps, 0.5 * (b0 + b1))
    del g_warm, g_all, g_each
    peak, peak_kind = _peaks()
    ms, nbytes = results["one_graph"]
    ms1, nbytes1 = results["graph_per_step"]
    return {"unit": "tokens/s", "value": p.B / (ms / 1e3), "ms_per_step": ms, "steps": steps,
            "kv_bytes_per_step": nbytes, "kv_gbs": nbytes / (ms / 1e3) / 1e9,
            "frac_of_hbm_peak": nbytes / (ms / 1e3) / 1e9 / peak, "peak_kind": peak_kind,
            "timing": f"the {steps} timed steps in one CUDA graph (state restored first)",
            "step": "attention, then fused score + update on one stream" if one_stream else
                    "attention, then update and score on a second stream",
            "graph_per_step": {"value": p.B / (ms1 / 1e3), "ms_per_step": ms1,
                               "kv_gbs": nbytes1 / (ms1 / 1e3) / 1e9,
                               "frac_of_hbm_peak": nbytes1 / (ms1 / 1e3) / 1e9 / peak}}


def measure_serving(device, reps=3):
    """Secondary measurement: serving (batch 32, contexts U[8K, 64K], one layer, keep
    U[5%, 25%]) end to end over its 256 decode steps: tokens enter the window ungated,
    and every 128 steps the 128 buffered tokens of every row are scored and their gated
    rows compacted from the window into the cache, then decoding goes on.  The whole run
    is one CUDA graph; the cache and ring are snapshotted before it and restored after
    every replay, so each timed replay starts from the same state (one untimed replay
    first).  tokens/s = 32 x 256 / the run's device time (median over `reps`); the K/V
    bytes per step count every head's live cache rows (pos <= t - w) and window rows,
    averaged over the first and last step."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    from sparse_decode_attention_spkv_b200.states import build_decode_state

    wl = W.WORKLOADS["serving"]
    steps, bulk = wl.decode_steps, wl.bulk
    p, Ls, inp = build_decode_state(wl, 1, steps, device, compact_window=True)
    L = Ls[0]
    o = torch.empty((p.B, p.Hq, p.head_dim), dtype=torch.bfloat16, device=device)
    lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=device)
    h_rows = inp["h_layer_row"][0]                      # [B][steps][d_model]
    starts = [inp["t"][i0].clone() for i0 in range(0, steps, bulk)]
    h_bufs = [h_rows[:, i0:i0 + bulk].contiguous() for i0 in range(0, steps, bulk)]
    state = [x for x in (L.cache.K_pool, L.cache.V_pool, L.cache.pos_pool, L.cache.page_table,
                         L.cache.count, L.cache.count_prev, L.cache.pool_top, L.cache.err_flag,
                         L.cache.u_pool, L.ring.K_win, L.ring.V_win, L.ring.z_win, L.ring.u_win)
             if x is not None]
    snap = [x.clone() for x in state]

    def run():
        for i in range(steps):
            R.decode_step(L, inp["t"][i], None, inp["q"][i][0], inp["k"][i][0], inp["v"][i][0],
                          retire=False, o=o, lse=lse)
            if (i + 1) % bulk == 0:
                R.bulk_compact(L, h_bufs[i // bulk], starts[i // bulk])

    def restore():
        for x, y in zip(state, snap):
            x.copy_(y)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    torch.cuda.synchronize()
    bytes_first = _live_kv_bytes(p, L, inp["t"][0])
    g.replay()  # untimed
    torch.cuda.synchronize()
    status, flags = S_check(L)
    if status:
        raise RuntimeError(f"serving measurement: cache error {flags}")
    bytes_last = _live_kv_bytes(p, L, inp["t"][steps - 1])
    restore()
    times = []
    for _ in range(reps):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
        status, flags = S_check(L)
        if status:
            raise RuntimeError(f"serving measurement: cache error {flags}")
        restore()
    del g
    ms = statistics.median(times)
    step_bytes = 0.5 * (bytes_first + bytes_last)
    peak, peak_kind = _peaks()
    gbs = step_bytes / (ms / steps / 1e3) / 1e9
    return {"unit": "tokens/s", "value": p.B * steps / (ms / 1e3), "ms_total": ms,
            "ms_runs": times, "steps": steps, "bulk": bulk,
            "kv_bytes_per_step": step_bytes, "kv_gbs": gbs, "frac_of_hbm_peak": gbs / peak,
            "peak_kind": peak_kind,
            "l2": "the state restore between replays writes GBs (larger than L2)"}


def _live_kv_bytes(p, L, t):
    """K/V bytes one decode step reads at query positions t [B]: per head, the cache
    rows with pos <= t - w plus min(w, t + 1) window rows (K and V, bf16)."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    count = L.cache.count.long()
    table = L.cache.page_table.long()
    idx = torch.arange(table.shape[1] * S.PAGE_ROWS, device=table.device)
    pages = table[:, idx // S.PAGE_ROWS].clamp(min=0)
    pos = L.cache.pos_pool[pages, idx % S.PAGE_ROWS]
    th = t.long().repeat_interleave(p.Hkv)
    live = ((pos <= (th - p.window)[:, None]) & (idx[None, :] < count[:, None])).sum(1)
    nw = torch.clamp(th + 1, max=p.window)
    return float((live + nw).sum().item()) * 2 * p.head_dim * 2


def S_check(L):
    from sparse_decode_attention_spkv_b200 import spkv as S
    status, flags = S.spkv_cache_check(L.cache)
    return (0 if status == S.OK else status), flags


# -------------------------------------------------------------- CPU oracle arm -----

_ORACLE_INPUTS = {}


def _host_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def _oracle_inputs(name: str, T: int, seed: int = 0):
    """Random fp64 inputs with a workload's shapes (the oracle's work does not depend on
    the values): perceptron weights, one query row, K/V and gates of T positions (keep
    27.5%, about the decode32k mean), hidden states of 256 tokens.  Drawn once per
    (workload, length) per process."""
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    key = (name, T, seed)
    if key not in _ORACLE_INPUTS:
        wl = W.WORKLOADS[name]
        rng = np.random.default_rng(seed)
        sd = 1.0 / math.sqrt(wl.head_dim)
        reps = (T + 4095) // 4096  # one 4096-position block of K/V repeated (values are moot)

        def kv():
            blk = rng.standard_normal((4096, wl.Hkv, wl.head_dim)) * sd
            return np.ascontiguousarray(np.tile(blk, (reps, 1, 1))[:T])
        _ORACLE_INPUTS[key] = dict(
            W1=rng.standard_normal((wl.hid, wl.d_model)) * 0.02, b1=rng.standard_normal(wl.hid) * 0.02,
            W2=rng.standard_normal((wl.Hkv, wl.hid)) * 0.02, b2=np.zeros(wl.Hkv),
            Q=rng.standard_normal((1, wl.Hq, wl.head_dim)) * sd, K=kv(), V=kv(),
            z=(rng.random((T, wl.Hkv)) < 0.275).astype(np.uint8),
            h=rng.standard_normal((256, wl.d_model)))
    return W.WORKLOADS[name], _ORACLE_INPUTS[key]


def _oracle_query(wl, x, t, n_tok=1):
    """The oracle's work for one query position t of one batch row: the utility and gate
    of n_tok new tokens (Eqs. (1)-(2)) and Eqs. (3)-(4) for every query head over the
    keys 0..t."""
    from oracle import spkv_oracle as O
    O.gate(O.utility(x["h"][:n_tok], x["W1"], x["b1"], x["W2"], x["b2"]), wl.tau)
    O.gated_attention(x["Q"], x["K"][:t + 1], x["V"][:t + 1], x["z"][:t + 1], wl.window, [t])


def oracle_decode_sample(units: int, seed: int = 0):
    """Time the fp64 oracle on `units` (layer, batch row) units of the decode32k step at
    t = 32768: the utility of the row's new token and Eqs. (3)-(4) for its 32 query heads
    over 32769 keys.  Returns (seconds per unit, threads available)."""
    wl, x = _oracle_inputs(WORKLOAD, W_CTX_DECODE + 1, seed)
    t0 = time.perf_counter()
    for _ in range(units):
        _oracle_query(wl, x, W_CTX_DECODE)
    return (time.perf_counter() - t0) / units, _host_threads()


W_CTX_DECODE = 32768


def _oracle_config_rate(name: str, budget_s: float):
    """The oracle's rate on a bounded sample of one workload, in its unit:
    decode32k / ragged128k / serving: tokens/s of whole decode steps (every batch row's
    query, its new token's utility; serving adds the bulk scoring of 128 buffered tokens
    per row every 128 steps, i.e. one token per row per step); prefill16k: tokens/s of the
    whole chunked prefill (every position's utility and attention).  Query positions are
    sampled across the workload's rows (the oracle's cost grows with the context), and the
    sample is scaled to the workload; `budget_s` bounds the sample's time."""
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    wl = W.WORKLOADS[name]
    if name == "decode32k":
        ctx = [W_CTX_DECODE] * wl.B
        per_step_rows = wl.B * wl.layers
        tokens_per_step = wl.B
    elif name == "ragged128k":
        ctx, per_step_rows, tokens_per_step = list(wl.ctx), wl.B, wl.B
    elif name == "serving":
        ctx, per_step_rows, tokens_per_step = list(wl.ctx), wl.B, wl.B
    elif name == "prefill16k":
        T = wl.ctx[0]
        ctx = [int((k + 0.5) * T / 64) for k in range(64)]  # 64 positions across the sequence
        per_step_rows, tokens_per_step = T, T
    else:
        raise ValueError(name)
    wl_, x = _oracle_inputs(name, max(ctx) + 1)
    t_start = time.perf_counter()
    spent, n = 0.0, 0
    i = 0
    # the rows' query positions in turn (round robin), until the budget is spent
    while n < len(ctx) or spent < budget_s:
        t = ctx[i % len(ctx)]
        a = time.perf_counter()
        _oracle_query(wl_, x, t)
        spent += time.perf_counter() - a
        n += 1
        i += 1
        if spent >= budget_s and n >= min(len(ctx), 4):
            break
    per_query = spent / n
    # a row sampled unevenly is corrected by the mean context of the sample vs the rows'
    mean_ctx_sample = sum(ctx[k % len(ctx)] for k in range(n)) / n
    mean_ctx = sum(ctx) / len(ctx)
    per_query *= mean_ctx / mean_ctx_sample
    step_s = per_query * per_step_rows
    return {"value": tokens_per_step / step_s, "unit": "tokens/s",
            "s_per_step" if name != "prefill16k" else "s_whole_prefill": step_s,
            "sample": f"{n} query positions ({spent:.1f} s), scaled to "
                      f"{per_step_rows} per {'step' if name != 'prefill16k' else 'prefill'}",
            "wall_s": time.perf_counter() - t_start}


def cpu_baseline(units: int, per_config_budget_s: float = 2.5):
    """The oracle as it stands on the host cores: the headline (decode32k, all cores) and,
    per workload, a single-thread and an all-core figure on bounded samples."""
    per_unit, threads = oracle_decode_sample(units)
    wl_units = 32 * 8  # (layer, batch row) units in one decode32k step
    step_s = per_unit * wl_units
    out = {"value": 8 / step_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{units} of the 256 (layer, batch row) units of one decode32k step at "
                     f"t=32768 (fp64 numpy oracle: utility + Eqs. (3)-(4) for 32 query heads "
                     f"over 32769 keys), {per_unit * 1e3:.1f} ms per unit, extrapolated to the "
                     f"full step"}
    per = {}
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        threadpool_limits = None
    for name in ("decode32k", "prefill16k", "ragged128k", "serving"):
        per[name] = {"all_cores": dict(_oracle_config_rate(name, per_config_budget_s),
                                       cores=threads)}
        if threadpool_limits is not None:
            with threadpool_limits(limits=1):
                per[name]["1_core"] = dict(_oracle_config_rate(name, per_config_budget_s),
                                           cores=1)
        _ORACLE_INPUTS.clear()  # the long-context inputs are GBs of host memory
    out["per_config"] = per
    return out


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle on the host cores, on the decode32k workload.
    One step of this arm is the oracle over `units` of the 256 (layer, batch row) units of a
    decode32k token step (8 tokens over 32 layers); ms_per_step is the time of those units,
    so ms_per_step x steps is the timed run, and value is tokens/s at that rate
    (tokens_per_step = 8 x units / 256)."""
    if rank != 0:
        return None
    # bounded work: about 600 oracle units (~1 minute on the host) over all timed steps
    units = max(1, min(args.cpu_units, 600 // max(1, args.steps)))
    for _ in range(args.warmup):
        oracle_decode_sample(1)
    times = []
    threads = _host_threads()
    for _ in range(args.steps):
        per_unit, threads = oracle_decode_sample(units)
        times.append(per_unit * units)
    step_s = sum(times) / len(times)
    tokens_per_step = 8.0 * units / 256
    value = tokens_per_step / step_s
    cb = {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
          "sample": f"each step: {units} of the 256 (layer, batch row) units of one decode32k "
                    f"token step (fp64 numpy oracle)"}
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "tokens_per_step": tokens_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "decode32k (see the spkv arm); one step of this arm = "
                                   f"{units} of the 256 (layer, batch row) units of a token step",
                       "global_batch": 8, "seq_len": 32768, "layers": 32,
                       "parallelism": "host cores"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="spkv", choices=["spkv", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-units", type=int, default=48)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-aux", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--decode-step", default="attn-first", choices=["attn-first", "split", "fused"],
                    help="attn-first: per layer the attention on the state before the step's "
                         "update (new rows passed in), then retirement, ring write and scoring "
                         "on a second stream; split: retirement and ring write, attention, "
                         "scoring on a second stream; fused: score, retirement and ring write "
                         "in one launch, then the attention")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed steps; the line reports the count run
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = _dist_init()
    out = run_gpu(args, world, rank, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(args.cpu_units)
        else:
            out["cpu_baseline"] = None
        print(json.dumps(out), flush=True)
    from sparse_decode_attention_spkv_b200 import dist as D
    D.finalize(world)


if __name__ == "__main__":
    main()
