#!/usr/bin/env python
"""Decode throughput of the 48-layer mixer-only stack, one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload stack48|attn_fa|attn_swa|prefill_fa|prefill_swa|decode_kda|
                                decode_gdn|prefill_kda|prefill_gdn|sweep]

Default workload ("stack48"): 48 layers, placement 12 FA / 12 SWA (w=4096) / 12 KDA / 12 GDN
randomly interleaved (seed 0), B=64 sequences at context 32768, H=32 query/delta heads, 8 KV
heads, d=128, bf16 activations and KV, fp32 states. A step decodes one token for every sequence
through all 48 layers; the metric is tokens/s = B / step time. Every layer's working set is
larger than L2 (state 128 MiB, KV >= 1 GiB) and a step touches ~122 GB, so no L2 flush is needed.

Multi-GPU (torchrun): replicas only -- every rank runs its own copy of the workload on its own
caches (weak scaling, no collective on the data path); value = all ranks' tokens / the slowest
rank's time.

The headline is timed as K CUDA-graph replays of the 48-layer step with nothing else on the
stream. At one GPU the line also carries, each measured after the headline:
  per_mixer          each mixer's layer time inside the stack (CUDA-graph replays of that
                     kind's layers, and its marginal cost in the interleaved step) and its
                     fraction of the HBM roofline;
  placement_switch   the first step after a placement switch against a steady step;
  prefill, decode    tokens/s of each mixer at its own configuration (KDA/GDN prefill B=4,
                     H=16, T=4096; FA/SWA prefill B=2, T=8192; KDA/GDN decode B=64, H=32;
                     FA/SWA decode B=32, ctx 8192), each with its roofline and the fp64
                     oracle's tokens/s on a bounded sample of the same work on the host's cores;
  oracle_check       the fp32 GDN configuration (B=1, H=2, d=64, T=128) against the oracle;
  context_sweep      decode tok/s of all-FA and the hybrid placements at 8k and 128k context
                     (B=16, 48 layers) and each one's speedup over all-FA;
  speculative,       self-speculative decoding (drafter all-GDN, k = 3) and one mixed batch of
  mixed_batch        two placements on the stack, each with its roofline.

--impl reference times the fp64 CPU oracle (the only other implementation of the method) on a
bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hybrid_mixer_decoding_b200 import inputs as I  # noqa: E402

METRIC = "decode tok/s per placement (BxCtx) and % of HBM roofline per mixer kernel"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# nominal peaks, for context beside the measured ones: HBM3e 8 TB/s, dense bf16 2.25 PFLOP/s
NOMINAL = {"GB/s": 8000.0, "TFLOP/s": 2250.0}


def with_nominal(roof: dict) -> dict:
    """The roofline object with the achieved figure also as a fraction of the nominal peak."""
    nom = NOMINAL.get(roof.get("unit"))
    if nom is not None and roof.get("achieved") is not None:
        roof = dict(roof, nominal_peak=nom, frac_of_nominal=round(roof["achieved"] / nom, 4))
    return roof


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def stack_placement():
    return I.placement({I.FA: 12, I.SWA: 12, I.KDA: 12, I.GDN: 12}, seed=0)


WORKLOADS = {
    "stack48": dict(B=64, ctx=32768, H=32, Hkv=8, d=128, window=4096),
}


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# replicas: every rank runs its own copy of the workload; the job's time is the slowest rank's
# ------------------------------------------------------------------------------------------
def max_over_ranks(ms: float, dist=None, device="cpu") -> float:
    """The largest of every rank's device time (ms); the local value without a process group."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms * 1e-3)


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
def traffic_for(kernel_key: str):
    """dram bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        tab = json.load(f)
    ent = tab.get(kernel_key)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if sha != ent.get("source_sha"):
        return None
    return ent.get("bytes_per_launch")


def run_ours(args, rank, world, local_rank):
    import torch

    import hybrid_mixer_decoding_b200 as hmd
    from hybrid_mixer_decoding_b200.stack import MixerStack, StackShape, layer_bytes

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    cfg = WORKLOADS["stack48"]
    shape = StackShape(cfg["B"], cfg["H"], cfg["Hkv"], cfg["d"], cfg["ctx"], cfg["window"])
    pl = stack_placement()
    # a second placement on the same caches (every layer as GDN), for the switch latency
    st = MixerStack({"hybrid": pl, "all_gdn": np.full(len(pl), I.GDN, np.int8)}, shape, seed=0,
                    io_sets=2)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        st.step("hybrid")
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    # one step = one CUDA-graph replay of the 48 mixer_decode_step calls (per io set)
    graphs = [st.capture(lambda b_=b_: st.step("hybrid", io_set=b_), warmup=1) for b_ in range(2)]
    for _ in range(args.warmup):
        graphs[0].replay()
    torch.cuda.synchronize()

    # ---- the timed region: K replays, nothing else on the stream ----------------------------
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clk.start()
    t0.record()
    for _ in range(args.steps):
        graphs[0].replay()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    assert hmd.hmd_device_errors(clear=True) == 0
    ms = max_over_ranks(t0.elapsed_time(t1), dist, "cuda")
    ms_per_step = ms / args.steps
    tokens = shape.B * args.steps * world
    value = job_throughput(shape.B * args.steps, world, ms)

    # ---- per-mixer figures: CUDA-graph replays, no events inside a replay --------------------
    # (1) each kind's layers of the stack alone, back to back, as one graph: layer time = replay
    #     time / layers; (2) the kind's marginal cost inside the interleaved step: the 48-layer
    #     replay minus a replay of the same step without that kind's layers, per layer.
    n_layers = st.n_layers
    n_rep = max(5, min(args.steps, 20))

    def graph_ms(layers):
        g = st.capture(lambda: st.step("hybrid", layers=layers), warmup=1)
        for _ in range(2):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(n_rep):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / n_rep

    full_ms = graph_ms(list(range(n_layers)))
    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    per_kind = {}
    for kind in (I.FA, I.SWA, I.KDA, I.GDN):
        layers = [l for l in range(n_layers) if pl[l] == kind]
        if not layers:
            continue
        mean_ms = graph_ms(layers) / len(layers)
        rest = [l for l in range(n_layers) if pl[l] != kind]
        marg_ms = (full_ms - graph_ms(rest)) / len(layers)
        gbs = layer_bytes(kind, shape) / (mean_ms * 1e-3) / 1e9
        per_kind[I.KIND_NAMES[kind]] = {"layer_us": round(mean_ms * 1e3, 2),
                                        "achieved_gbs": round(gbs, 1),
                                        "frac": round(gbs / hbm, 4),
                                        "frac_nominal_8tbs": round(gbs / 8000.0, 4),
                                        "marginal_layer_us": round(marg_ms * 1e3, 2),
                                        "bytes_per_layer": layer_bytes(kind, shape),
                                        "decode_tok_s_per_layer": round(shape.B / (mean_ms * 1e-3), 1)}
    assert hmd.hmd_device_errors(clear=True) == 0
    per_kind["measured"] = (f"separate pass after the timed region: layer_us = one CUDA-graph "
                            f"replay of that kind's layers of the stack (same caches and inputs), "
                            f"back to back, / layers, mean of {n_rep} replays timed "
                            f"with CUDA events around the replays only; marginal_layer_us = (the "
                            f"48-layer replay, {full_ms:.3f} ms, minus a replay of the step "
                            f"without that kind's layers) / that kind's layers")
    dom = per_kind["FA"]
    roofline = {"bound": "hbm", "achieved": dom["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                "frac": dom["frac"], "traffic": traffic_for("attn_fa_stack48"),
                "kernel": "attn_decode FA layer (attn_split_kernel<128> + attn_combine_kernel)",
                "peak_source": pk_kind,
                "algorithmic_bytes_per_launch": dom["bytes_per_layer"],
                "timing": "CUDA-graph replays of the stack's FA layers (events around replays only)"}
    switch = placement_switch(st, args.warmup)
    assert hmd.hmd_device_errors(clear=True) == 0

    # ---- end to end through the C ABI from pinned host buffers ----------------------------
    # Every step copies that step's inputs host->device and reads every layer's output
    # device->host. A copy stream moves the next step's inputs into the other buffer set while
    # the current step computes (one graph replay of the 48 C-ABI calls on that set), and drains
    # the current step's outputs once it is done (events order every reuse of a buffer).
    host_in, dev_in, dev_out = [], [[], []], [[], []]
    for l in range(n_layers):
        names = ["q", "k", "v", "beta", "lg_s" if pl[l] == I.GDN else "lg_c"] \
            if pl[l] in (I.GDN, I.KDA) else ["q", "nk", "nv"]
        for nm in names:
            src = st.input_sets[0][l][nm]
            host_in.append(torch.empty_like(src, device="cpu").pin_memory().copy_(src))
            for b_ in range(2):
                dev_in[b_].append(st.input_sets[b_][l][nm])
        for b_ in range(2):
            dev_out[b_].append(st.input_sets[b_][l]["o"])
    host_out = [[torch.empty_like(o, device="cpu").pin_memory() for o in dev_out[b_]]
                for b_ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out[0])
    comp, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_run(n_steps, e0=None, e1=None):
        with torch.cuda.stream(copy):
            if e0 is not None:
                e0.record(copy)
            for h, d in zip(host_in, dev_in[0]):
                d.copy_(h, non_blocking=True)
            ev_in[0].record(copy)
        for k in range(n_steps):
            b_ = k % 2
            comp.wait_event(ev_in[b_])
            graphs[b_].replay()
            ev_done[b_].record(comp)
            with torch.cuda.stream(copy):
                if k + 1 < n_steps:
                    if k >= 1:
                        copy.wait_event(ev_done[1 - b_])
                    for h, d in zip(host_in, dev_in[1 - b_]):
                        d.copy_(h, non_blocking=True)
                    ev_in[1 - b_].record(copy)
                copy.wait_event(ev_done[b_])
                for d, h in zip(dev_out[b_], host_out[b_]):
                    h.copy_(d, non_blocking=True)
        with torch.cuda.stream(copy):
            if e1 is not None:
                e1.record(copy)

    e2e_run(max(2, args.warmup // 2))
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize()
    barrier()
    assert hmd.hmd_device_errors(clear=True) == 0
    ems = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    e2e = {"value": round(tokens / (ems * 1e-3), 2), "unit": "tok/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "how": "per step: pinned host inputs -> device, one graph replay of the 48 C-ABI "
                  "calls, every layer's output -> pinned host; copies overlap the other buffer "
                  "set's step"}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init caches, no weights)",
        "config": {"workload": "stack48: 48-layer mixer-only decode, 12 FA / 12 SWA(w=4096) / "
                               "12 KDA / 12 GDN interleaved (seed 0), B=64, ctx=32768, H=32, "
                               "Hkv=8, d=128, bf16 act/KV, fp32 state",
                   "global_batch": shape.B * world, "seq_len": shape.ctx,
                   "parallelism": f"replicas x{world}",
                   "timed": "K CUDA-graph replays of the 48-layer step, no other work on the "
                            "stream",
                   "l2": "working set per step ~122 GB >> L2 (126 MB); no flush",
                   "aliased_kv": st.aliased},
        "roofline": with_nominal(roofline),
        "per_mixer": per_kind,
        "placement_switch": switch,
        "e2e": e2e,
        "gpu_launches": st.launches_per_step("hybrid") * args.steps,
        "clocks": clocks,
    }
    del graphs
    st.free()
    del st
    torch.cuda.empty_cache()
    if rank == 0 and not args.skip_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(shape, pl, budget_s=args.cpu_budget)
    if dist is not None:
        dist.destroy_process_group()
    return out


def placement_switch(st, warmup: int) -> dict:
    """Latency of a placement switch on a registered stack. Each placement's step is one CUDA-graph
    replay of its 48 mixer_decode_step calls (captured on the same caches), so the steps are
    GPU-bound; steady replays of each placement are timed, then alternating replays (each one
    the first step after a switch), all with CUDA events around every step. A switch passes
    another placement array: no cache is copied or reloaded, so the first step after a switch
    should cost what a steady step of its placement costs."""
    import torch

    graphs = {nm: st.capture(nm, warmup=1) for nm in ("hybrid", "all_gdn")}

    def timed_steps(names):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in names]
        for (a, b), nm in zip(evs, names):
            a.record()
            graphs[nm].replay()
            b.record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    for nm in graphs:
        for _ in range(max(1, warmup // 2)):
            graphs[nm].replay()
    n = 6
    steady_h = timed_steps(["hybrid"] * n)[1:]
    steady_g = timed_steps(["all_gdn"] * n)[1:]
    alt = timed_steps(["hybrid", "all_gdn"] * n)
    to_h = alt[0::2][1:]  # every hybrid step here directly follows an all-GDN step
    to_g = alt[1::2]
    del graphs
    sh, sg = float(np.median(steady_h)), float(np.median(steady_g))
    fh, fg = float(np.median(to_h)), float(np.median(to_g))
    return {"steady_step_ms": {"hybrid": round(sh, 4), "all_gdn": round(sg, 4)},
            "first_step_after_switch_ms": {"to_hybrid": round(fh, 4), "to_all_gdn": round(fg, 4)},
            "switch_cost_us": {"to_hybrid": round((fh - sh) * 1e3, 1),
                               "to_all_gdn": round((fg - sg) * 1e3, 1)},
            "how": "medians of CUDA-graph replays of each placement's step timed with CUDA "
                   "events; a switch is a replay of the other placement's graph on the same "
                   "registered caches (nothing is copied or reloaded)"}


# ------------------------------------------------------------------------------------------
# the oracle on host cores (reported baseline / the reference arm)
# ------------------------------------------------------------------------------------------
def _oracle_layer_inputs(kind, shape, n_seq, seed):
    """Host inputs for one layer of the stack workload restricted to n_seq sequences."""
    if kind in (I.GDN, I.KDA):
        d = I.delta_inputs(kind, n_seq, 1, shape.H, shape.d, shape.d, dtype="bf16", seed=seed,
                           state0="randn")
        return d
    w = shape.window if kind == I.SWA else 0
    return I.attn_inputs(kind, n_seq, shape.H, shape.Hkv, shape.d, shape.ctx, window=w,
                         seed=seed)


def _oracle_layer_time(O, kind, inp, threads):
    t0 = time.perf_counter()
    if kind in (I.GDN, I.KDA):
        O.delta_recurrent(kind, inp.q, inp.k, inp.v, inp.beta, inp.log_gate, inp.state0,
                          n_threads=threads)
    else:
        O.attn_decode(kind, inp.window, inp.q, inp.new_k, inp.new_v, inp.k_pool, inp.v_pool,
                      inp.page_table, inp.seq_lens, n_threads=threads)
    return time.perf_counter() - t0


def cpu_baseline(shape, pl, budget_s=15.0, n_seq=2):
    from oracle import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    per_kind = {}
    for kind in (I.FA, I.SWA, I.KDA, I.GDN):
        inp = _oracle_layer_inputs(kind, shape, n_seq, seed=kind)
        ts = []
        t_start = time.perf_counter()
        while True:
            ts.append(_oracle_layer_time(O, kind, inp, cores))
            if time.perf_counter() - t_start > budget_s / 4 or len(ts) >= 50:
                break
        per_kind[kind] = float(np.median(ts))
    step_s = sum(per_kind[int(k)] for k in pl)  # one token for n_seq sequences, 48 layers
    # the same sample on one host thread (each kind timed once), for the per-core figure
    one = {kind: _oracle_layer_time(O, kind, _oracle_layer_inputs(kind, shape, 1, seed=kind), 1)
           for kind in (I.FA, I.SWA, I.KDA, I.GDN)}
    one_s = sum(one[int(k)] for k in pl)
    return {"value": round(n_seq / step_s, 4), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "one_thread_tok_s": round(1.0 / one_s, 4),
            "sample": f"fp64 C oracle, {n_seq} sequences at the stack's per-layer shapes "
                      f"(H=32, Hkv=8, d=128, ctx 32768, w=4096); each mixer kind timed on one "
                      f"layer, summed over the placement's 48 layers; tokens/s = "
                      f"{n_seq} / summed time; one_thread_tok_s: one sequence on one thread",
            "per_layer_s": {I.KIND_NAMES[k]: round(v, 5) for k, v in per_kind.items()}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from oracle import oracle as O
    from hybrid_mixer_decoding_b200.stack import StackShape
    O.build()
    cfg = WORKLOADS["stack48"]
    shape = StackShape(cfg["B"], cfg["H"], cfg["Hkv"], cfg["d"], cfg["ctx"], cfg["window"])
    pl = stack_placement()
    cores = len(os.sched_getaffinity(0))
    n_seq = 1
    inputs = {k: _oracle_layer_inputs(k, shape, n_seq, seed=k) for k in (I.FA, I.SWA, I.KDA, I.GDN)}

    def step():
        # one token for n_seq sequences through the 48 layers (each kind's layer inputs reused)
        for kind in pl:
            _oracle_layer_time(O, int(kind), inputs[int(kind)], cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = n_seq * args.steps / el
    sample = (f"fp64 C oracle on {cores} host threads, {n_seq} sequence(s) of the stack48 "
              f"workload per step (all 48 layers at ctx 32768)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": "stack48 (oracle sample)", "global_batch": n_seq,
                       "seq_len": shape.ctx, "parallelism": "host threads"},
            "cpu_baseline": {"value": round(value, 4), "unit": "tok/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------------------
# single-kernel workloads (the per-mixer configurations) and the context sweep
# ------------------------------------------------------------------------------------------
def _events_time(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps * 1e-3  # seconds per launch


def measure_workload(w: str, steps: int, warmup: int) -> dict:
    """One mixer kernel at its configuration:
    attn_fa / attn_swa: B=32, Hq=32, Hkv=8, d=128, context 8192, SWA w=4096, paged bf16 KV
      (pages of 64, random page permutation), one new token per sequence;
    prefill_fa / prefill_swa: B=2, T=8192, Hq=32, Hkv=8, d=128, SWA w=4096, prompts written into
      an empty paged cache;
    decode_kda / decode_gdn: one decode step at the stack's layer shape (B=64, H=32, d=128),
      rotating over 4 state buffers (512 MiB) so every launch streams from HBM;
    prefill_kda / prefill_gdn: B=4, H=16, d=128, T=4096, chunk 64, bf16 q/k/v, fp32 state."""
    import torch

    import hybrid_mixer_decoding_b200 as hmd
    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    dev = "cuda"
    bf = torch.bfloat16
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    extra = {}
    if w in ("attn_fa", "attn_swa"):
        kind = I.FA if w == "attn_fa" else I.SWA
        B, Hq, Hkv, d, L, win = 32, 32, 8, 128, 8192, 4096
        pps = L // 64 if kind == I.FA else win // 64
        P = B * pps
        kp = torch.randn(P, Hkv, 64, d, device=dev, dtype=bf, generator=g)
        vp = torch.randn(P, Hkv, 64, d, device=dev, dtype=bf, generator=g)
        table = torch.randperm(P, device=dev, generator=g).to(torch.int32).view(B, pps).contiguous()
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        q = torch.randn(B, Hq, d, device=dev, dtype=bf, generator=g)
        nk = torch.randn(B, Hkv, d, device=dev, dtype=bf, generator=g)
        nv = torch.randn(B, Hkv, d, device=dev, dtype=bf, generator=g)
        o = torch.empty(B, Hq, d, device=dev, dtype=bf)
        ws = torch.empty(hmd.attn_decode_workspace_size(kind, win, B, Hq, Hkv, d, 64, L),
                         dtype=torch.uint8, device=dev)

        def fn():
            hmd.attn_decode(kind, win, q, nk, nv, kp, vp, table, lens, L, o, ws)
        sec = _events_time(fn, steps, warmup)
        keys = L if kind == I.FA else win
        byts = B * (keys * Hkv * d * 4 + 2 * Hq * d * 2 + 2 * Hkv * d * 2)
        value, unit = B / sec, "tok/s"
        desc = (f"{'FA' if kind == I.FA else 'SWA(w=4096)'} decode: B=32, Hq=32, Hkv=8, d=128, "
                f"ctx 8192, paged bf16 KV (64-token pages, random permutation)")
        roof = {"bound": "hbm", "achieved": round(byts / sec / 1e9, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(byts / sec / 1e9 / hbm, 4),
                "traffic": traffic_for(w), "algorithmic_bytes": byts}
        launches = 2
    elif w in ("verify_fa", "verify_swa"):
        kind = I.FA if w == "verify_fa" else I.SWA
        B, Hq, Hkv, d, L, win, nq_max = 32, 32, 8, 128, 8192, 4096, 4
        ring = -(-(win + nq_max - 1) // 64)
        pps = L // 64 if kind == I.FA else ring
        P = B * pps
        kp = torch.randn(P, Hkv, 64, d, device=dev, dtype=bf, generator=g)
        vp = torch.randn(P, Hkv, 64, d, device=dev, dtype=bf, generator=g)
        table = torch.randperm(P, device=dev, generator=g).to(torch.int32).view(B, pps).contiguous()
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        per_nq = {}
        for nq in range(1, nq_max + 1):
            q = torch.randn(B, nq, Hq, d, device=dev, dtype=bf, generator=g)
            nk = torch.randn(B, nq, Hkv, d, device=dev, dtype=bf, generator=g)
            nv = torch.randn(B, nq, Hkv, d, device=dev, dtype=bf, generator=g)
            o = torch.empty(B, nq, Hq, d, device=dev, dtype=bf)
            ws = torch.empty(hmd.attn_verify_workspace_size(kind, win, nq, B, Hq, Hkv, d, 64, L),
                             dtype=torch.uint8, device=dev)

            def fn():
                hmd.attn_verify(kind, win, ring, q, nk, nv, kp, vp, table, lens, L, o, ws)
            per_nq[nq] = _events_time(fn, steps, warmup)
        sec = per_nq[nq_max]
        keys = L if kind == I.FA else win + nq_max - 1
        byts = B * (keys * Hkv * d * 4 + nq_max * (2 * Hq * d * 2 + 2 * Hkv * d * 2))
        value, unit = B * nq_max / sec, "tok/s"
        desc = (f"{'FA' if kind == I.FA else 'SWA(w=4096, ring 65 pages)'} verification pass of "
                f"4 new tokens per sequence: B=32, Hq=32, Hkv=8, d=128, ctx 8192 counting them, "
                f"paged bf16 KV (64-token pages, random permutation); value = tokens checked/s")
        roof = {"bound": "hbm", "achieved": round(byts / sec / 1e9, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(byts / sec / 1e9 / hbm, 4),
                "traffic": traffic_for(w), "algorithmic_bytes": byts}
        extra["verify"] = {"us_per_pass_by_n_q": {str(n): round(t * 1e6, 2) for n, t in per_nq.items()},
                           "cost_vs_one_token": round(per_nq[nq_max] / per_nq[1], 4)}
        launches = 2
    elif w in ("prefill_fa", "prefill_swa"):
        kind = I.FA if w == "prefill_fa" else I.SWA
        B, T, Hq, Hkv, d, win = 2, 8192, 32, 8, 128, 4096
        pps = T // 64 if kind == I.FA else win // 64
        P = B * pps
        kp = torch.empty(P, Hkv, 64, d, device=dev, dtype=bf)
        vp = torch.empty(P, Hkv, 64, d, device=dev, dtype=bf)
        table = torch.randperm(P, device=dev, generator=g).to(torch.int32).view(B, pps).contiguous()
        q = torch.randn(B, T, Hq, d, device=dev, dtype=bf, generator=g)
        k = torch.randn(B, T, Hkv, d, device=dev, dtype=bf, generator=g)
        v = torch.randn(B, T, Hkv, d, device=dev, dtype=bf, generator=g)
        o = torch.empty(B, T, Hq, d, device=dev, dtype=bf)

        def fn():
            hmd.attn_prefill(kind, win, q, k, v, kp, vp, table, o)
        sec = _events_time(fn, steps, warmup)
        keys = sum(min(t + 1, win) if kind == I.SWA else t + 1 for t in range(T))
        flops = 4 * d * Hq * B * keys  # S = q K^T and O = P V over the attended keys
        tf = float(pk["bf16_tflops"])
        value, unit = B * T / sec, "tok/s"
        desc = (f"{'FA' if kind == I.FA else 'SWA(w=4096)'} prefill from an empty cache: B=2, "
                f"T=8192, Hq=32, Hkv=8, d=128, K/V written to a paged bf16 cache "
                f"(64-token pages, random permutation)")
        roof = {"bound": "tensor", "achieved": round(flops / sec / 1e12, 2), "peak": tf,
                "unit": "TFLOP/s", "frac": round(flops / sec / 1e12 / tf, 5),
                "traffic": traffic_for(w), "algorithmic_flops": flops}
        launches = 1
    elif w in ("decode_kda", "decode_gdn"):
        kind = I.KDA if w == "decode_kda" else I.GDN
        B, H, d = 64, 32, 128
        states = [torch.randn(B, H, d, d, device=dev, generator=g) / math.sqrt(d) for _ in range(4)]
        q = torch.randn(B, H, d, device=dev, dtype=bf, generator=g)
        k = torch.nn.functional.normalize(torch.randn(B, H, d, device=dev, generator=g), dim=-1).to(bf)
        v = torch.randn(B, H, d, device=dev, dtype=bf, generator=g)
        beta = torch.sigmoid(torch.randn(B, H, device=dev, generator=g))
        lg = (-0.05 * torch.rand(B, H, d, device=dev, generator=g) if kind == I.KDA
              else -0.1 * torch.rand(B, H, device=dev, generator=g))
        o = torch.empty(B, H, d, device=dev, dtype=bf)
        it = [0]

        def fn():
            hmd.delta_rule_decode(kind, q, k, v, beta, lg, states[it[0] % 4], o)
            it[0] += 1
        sec = _events_time(fn, steps, warmup)
        byts = B * H * (2 * d * d * 4 + 4 * d * 2 + 4 + (4 * d if kind == I.KDA else 4))
        value, unit = B / sec, "tok/s"
        desc = f"{I.KIND_NAMES[kind]} decode step, B=64, H=32, d=128, bf16 act, fp32 state"
        roof = {"bound": "hbm", "achieved": round(byts / sec / 1e9, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(byts / sec / 1e9 / hbm, 4),
                "traffic": traffic_for(w), "algorithmic_bytes": byts}
        launches = 1
    elif w in ("prefill_kda", "prefill_gdn"):
        kind = I.KDA if w == "prefill_kda" else I.GDN
        B, T, H, d = 4, 4096, 16, 128
        q = torch.randn(B, T, H, d, device=dev, dtype=bf, generator=g)
        k = torch.nn.functional.normalize(torch.randn(B, T, H, d, device=dev, generator=g), dim=-1).to(bf)
        v = torch.randn(B, T, H, d, device=dev, dtype=bf, generator=g)
        beta = torch.sigmoid(torch.randn(B, T, H, device=dev, generator=g))
        lg = (-0.05 * torch.rand(B, T, H, d, device=dev, generator=g) if kind == I.KDA
              else -0.1 * torch.rand(B, T, H, device=dev, generator=g))
        st = torch.zeros(B, H, d, d, device=dev)
        o = torch.empty(B, T, H, d, device=dev, dtype=bf)

        def fn():
            hmd.delta_rule_prefill_chunked(kind, q, k, v, beta, lg, st, o)
        sec = _events_time(fn, steps, warmup)
        per_tok = 768 + 256 + 4 + (512 if kind == I.KDA else 4)
        byts = B * T * H * per_tok + 2 * B * H * d * d * 4
        flops = B * T * H * (10 * 64 * d + 6 * d * d)
        tf = float(pk["bf16_tflops"])
        value, unit = B * T / sec, "tok/s"
        desc = f"{I.KIND_NAMES[kind]} chunked prefill: B=4, H=16, d=128, T=4096, chunk 64"
        roof = {"bound": "hbm", "achieved": round(byts / sec / 1e9, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(byts / sec / 1e9 / hbm, 5),
                "traffic": traffic_for(w), "algorithmic_bytes": byts}
        extra["tensor"] = {"achieved_tflops": round(flops / sec / 1e12, 3), "peak": tf,
                           "frac": round(flops / sec / 1e12 / tf, 5), "algorithmic_flops": flops}
        launches = 2  # chunk-parallel pass + state scan
    else:
        raise SystemExit(f"unknown workload {w}")
    assert hmd.hmd_device_errors(clear=True) == 0
    out = {"value": round(value, 2), "unit": unit, "ms_per_step": round(sec * 1e3, 4),
           "workload": f"{w}: {desc}", "roofline": with_nominal(roof),
           "launches_per_step": launches}
    out.update(extra)
    return out


def run_kernel_workload(args):
    """One mixer kernel at its configuration as the JSON line (see measure_workload). Its timed
    region lasts milliseconds, shorter than the clock sampler's period, so the line carries no
    clock record; the default stack line does."""
    m = measure_workload(args.workload, args.steps, args.warmup)
    out = {"metric": METRIC, "value": m.pop("value"), "unit": m.pop("unit"), "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.pop("ms_per_step"),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded)", "config": {"workload": m.pop("workload")},
           "roofline": m.pop("roofline"),
           "gpu_launches": m.pop("launches_per_step") * args.steps}
    out.update(m)
    if not args.skip_cpu_baseline and args.workload in ORACLE_SAMPLES:
        out["cpu_baseline"] = workload_cpu_baseline(args.workload, args.cpu_budget / 4)
    return out


# ------------------------------------------------------------------------------------------
# the oracle on a bounded sample of each per-mixer workload (reported baseline, not a target)
# ------------------------------------------------------------------------------------------
# workload -> (mixer, sample description); the sample's oracle time is scaled to the workload
ORACLE_SAMPLES = {
    "prefill_kda": (I.KDA, "sequence 0 of 4 (all 16 heads, T=4096, d=128), token by token"),
    "prefill_gdn": (I.GDN, "sequence 0 of 4 (all 16 heads, T=4096, d=128), token by token"),
    "prefill_fa": (I.FA, "the last 128 prompt tokens of sequence 0, kv-head group 0 (4 of 32 "
                         "query heads) of B=2, T=8192; time scaled by the workload's attended "
                         "query-key pairs over the sample's"),
    "prefill_swa": (I.SWA, "the last 128 prompt tokens of sequence 0, kv-head group 0 (4 of 32 "
                           "query heads) of B=2, T=8192, w=4096; time scaled by the workload's "
                           "attended query-key pairs over the sample's"),
    "decode_kda": (I.KDA, "2 of 64 sequences (all 32 heads, d=128), one token"),
    "decode_gdn": (I.GDN, "2 of 64 sequences (all 32 heads, d=128), one token"),
    "attn_fa": (I.FA, "2 of 32 sequences (32 query / 8 kv heads, ctx 8192), one token"),
    "attn_swa": (I.SWA, "2 of 32 sequences (32 query / 8 kv heads, ctx 8192, w=4096), one token"),
}


def _repeat_time(fn, budget_s: float) -> float:
    """Median seconds of fn() over repetitions until budget_s has passed (at least 2)."""
    ts = []
    t_start = time.perf_counter()
    while len(ts) < 2 or (time.perf_counter() - t_start < budget_s and len(ts) < 50):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return float(np.median(ts))


def workload_cpu_baseline(w: str, budget_s: float = 2.0) -> dict:
    """The fp64 oracle, as it stands, on the host's cores, on a bounded sample of workload w;
    value in the workload's unit (tok/s)."""
    from oracle import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    kind, sample = ORACLE_SAMPLES[w]
    if w in ("prefill_kda", "prefill_gdn"):
        T, H = 4096, 16
        x = I.delta_inputs(kind, 1, T, H, 128, 128, dtype="bf16", seed=7)
        sec = _repeat_time(lambda: O.delta_recurrent(kind, x.q, x.k, x.v, x.beta, x.log_gate,
                                                     x.state0, n_threads=cores), budget_s)
        value = T / sec  # the sample is one whole sequence of the workload
    elif w in ("prefill_fa", "prefill_swa"):
        T, n_q, win, Hq = 8192, 128, 4096, 4
        window = win if kind == I.SWA else 0
        x = I.verify_inputs(kind, 1, n_q, Hq, 1, 128, T, window=window, seed=7)
        sec = _repeat_time(lambda: O.attn_verify(kind, window, x.ring_pages, x.q, x.new_k,
                                                 x.new_v, x.k_pool, x.v_pool, x.page_table,
                                                 x.seq_lens, n_threads=cores), budget_s)
        keys = (lambda t: min(t + 1, win)) if kind == I.SWA else (lambda t: t + 1)
        pairs_full = 2 * 32 * sum(keys(t) for t in range(T))   # B=2, Hq=32
        pairs_sample = Hq * sum(keys(t) for t in range(T - n_q, T))
        value = 2 * T / (sec * pairs_full / pairs_sample)
    elif w in ("decode_kda", "decode_gdn"):
        n = 2
        x = I.delta_inputs(kind, n, 1, 32, 128, 128, dtype="bf16", seed=7, state0="randn")
        sec = _repeat_time(lambda: O.delta_recurrent(kind, x.q, x.k, x.v, x.beta, x.log_gate,
                                                     x.state0, n_threads=cores), budget_s)
        value = n / sec
    else:  # attn_fa, attn_swa (config 3)
        n = 2
        window = 4096 if kind == I.SWA else 0
        x = I.attn_inputs(kind, n, 32, 8, 128, 8192, window=window, seed=7)
        sec = _repeat_time(lambda: O.attn_decode(kind, window, x.q, x.new_k, x.new_v, x.k_pool,
                                                 x.v_pool, x.page_table, x.seq_lens,
                                                 n_threads=cores), budget_s)
        value = n / sec
    return {"value": round(value, 3), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 C oracle on {cores} host threads: {sample}; median of repeats",
            "sample_s": round(sec, 4)}


def oracle_check_config1() -> dict:
    """The single-layer GDN oracle check: B=1, H=2, d_k=d_v=64, T=128, fp32 (q, v ~ N(0,1),
    k ~ N(0,1) L2-normalised, beta = sigmoid(N(0,1)), log g ~ U(-0.1, 0), S0 = 0, seed 0), run
    on the GPU as 128 decode steps and as one chunked prefill (chunk 64), both against the fp64
    recurrence at the fp32 tolerance 1e-4; the oracle's own time on the host is reported."""
    import torch

    import hybrid_mixer_decoding_b200 as hmd
    from oracle import oracle as O
    O.build()
    x = I.delta_inputs(I.GDN, 1, 128, 2, 64, 64, dtype="f32", seed=0)
    dev = "cuda"

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q, k, v, beta, lg = t(x.q), t(x.k), t(x.v), t(x.beta), t(x.log_gate)
    # 128 decode steps
    state = t(x.state0).clone()
    o_dec = torch.empty(1, 128, 2, 64, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(128):
        hmd.delta_rule_decode(I.GDN, q[:, i].contiguous(), k[:, i].contiguous(),
                              v[:, i].contiguous(), beta[:, i].contiguous(),
                              lg[:, i].contiguous(), state, o_dec[:, i])
    e1.record()
    torch.cuda.synchronize()
    dec_ms = e0.elapsed_time(e1)
    st_dec = state.cpu().numpy()
    # one chunked prefill
    state_p = t(x.state0).clone()
    o_pre = torch.empty(1, 128, 2, 64, device=dev)
    hmd.delta_rule_prefill_chunked(I.GDN, q, k, v, beta, lg, state_p, o_pre)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    cores = len(os.sched_getaffinity(0))
    o_ref, s_ref = O.delta_recurrent(I.GDN, x.q, x.k, x.v, x.beta, x.log_gate, x.state0)
    sec = _repeat_time(lambda: O.delta_recurrent(I.GDN, x.q, x.k, x.v, x.beta, x.log_gate,
                                                 x.state0, n_threads=cores), 1.0)
    errs = {"decode_o": O.rel_err(o_dec.cpu().numpy(), o_ref),
            "decode_state": O.rel_err(st_dec, s_ref),
            "prefill_o": O.rel_err(o_pre.cpu().numpy(), o_ref),
            "prefill_state": O.rel_err(state_p.cpu().numpy(), s_ref)}
    return {"config": "GDN B=1, H=2, d=64, T=128, fp32, S0=0, seed 0",
            "rel_err": {k_: float(f"{v_:.3e}") for k_, v_ in errs.items()}, "tol": 1e-4,
            "pass": all(v_ <= 1e-4 for v_ in errs.values()),
            "gpu_decode_tok_s": round(128 / (dec_ms * 1e-3), 1),
            "cpu_baseline": {"value": round(128 / sec, 1), "unit": "tok/s", "cores": cores,
                             "kind": "oracle", "sample": "the whole config (128 tokens)"}}


PREFILL_WORKLOADS = {"KDA": "prefill_kda", "GDN": "prefill_gdn", "FA": "prefill_fa",
                     "SWA": "prefill_swa"}
DECODE_WORKLOADS = {"KDA": "decode_kda", "GDN": "decode_gdn", "FA": "attn_fa", "SWA": "attn_swa"}


def per_mixer_lines(args) -> dict:
    """Prefill and decode tokens/s of each mixer at its configuration (bench steps/warmup),
    each with its roofline and the oracle's throughput on a bounded sample of the same work."""
    import torch
    out = {}
    for key, table in (("prefill", PREFILL_WORKLOADS), ("decode", DECODE_WORKLOADS)):
        out[key] = {}
        for mixer, w in table.items():
            m = measure_workload(w, max(5, args.steps), args.warmup)
            torch.cuda.empty_cache()
            if not args.skip_cpu_baseline:
                m["cpu_baseline"] = workload_cpu_baseline(w, budget_s=1.5)
            out[key][mixer] = m
    return out




def run_spec(args):
    """Self-speculative decoding on the 48-layer mixer-only stack: B=32, context 32768, H=32,
    Hkv=8, d=128, target placement 12 FA / 12 SWA(w=4096) / 12 KDA / 12 GDN (the stack48
    placement), drafter all-GDN, k=3 drafts per round (4 positions verified), each draft kept
    with probability 0.8 until the first rejection (seeded). Every round is two CUDA-graph
    replays (draft, verify); the plain decode step of the target placement is timed alongside."""
    import torch

    import hybrid_mixer_decoding_b200 as hmd
    from hybrid_mixer_decoding_b200.spec import SpecStack, make_schedule
    from hybrid_mixer_decoding_b200.stack import StackShape, layer_bytes

    pk, _ = peaks()
    hbm = float(pk["hbm_gbs"])
    k, alpha = 3, 0.8
    shape = StackShape(B=32, H=32, Hkv=8, d=128, ctx=32768, window=4096)
    rounds = args.warmup + args.steps
    target = stack_placement()
    sp = SpecStack(target, shape, k, max_rounds=rounds + 2)
    sched = make_schedule(shape.B, k, rounds, sp.L0, alpha, seed=1)
    slots_dev = torch.from_numpy(sched.slots).cuda()
    lens_dev = torch.from_numpy(sched.lens).cuda()
    g_draft, g_verify, g_plain = sp.capture(sp.draft), sp.capture(sp.verify), sp.capture(sp.plain_step)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for i in range(n):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    for _ in range(args.warmup):
        g_plain.replay()
    plain_s = timed(lambda i: g_plain.replay(), args.steps) / args.steps
    # phase times (on the first round's chain; the work does not depend on it)
    sp.set_round(sched, 0, slots_dev, lens_dev)
    draft_s = timed(lambda i: g_draft.replay(), args.steps) / args.steps
    verify_s = timed(lambda i: g_verify.replay(), args.steps) / args.steps

    def round_(r):
        sp.set_round(sched, r, slots_dev, lens_dev)
        g_draft.replay()
        g_verify.replay()
    for r in range(args.warmup):
        round_(r)
    spec_s = timed(lambda i: round_(args.warmup + i), args.steps)
    assert hmd.hmd_device_errors(clear=True) == 0
    tokens = int(sched.tokens[args.warmup:].sum())
    value = tokens / spec_s
    plain_tok_s = shape.B / plain_s
    # algorithmic bytes of one round: the drafter's k+1 steps, the target's verify pass
    B, H, Hkv, d, ctx, w = shape.B, shape.H, shape.Hkv, shape.d, shape.ctx, shape.window
    nq = k + 1
    lin = lambda kind: layer_bytes(kind, shape)  # noqa: E731
    draft_bytes = nq * sum(lin(int(x)) for x in sp.drafter)
    attn = lambda keys: B * (keys * Hkv * d * 4 + nq * (2 * H * d * 2 + 2 * Hkv * d * 2))  # noqa: E731
    # a GDN/KDA layer of the target reads its state once and stores it after each of the nq
    # positions (delta_rule_decode_chain): state (1 + nq) times, activations nq times
    state_b = B * H * d * d * 4

    def chain_bytes(kind):
        return (1 + nq) * state_b + nq * (lin(kind) - 2 * state_b)
    verify_bytes = sum(attn(ctx) if x == I.FA else attn(w + k) if x == I.SWA else
                       chain_bytes(int(x)) for x in target)
    round_s = spec_s / args.steps
    byts = draft_bytes + verify_bytes
    la = sp.launches()
    sp.free()
    return {"metric": METRIC, "value": round(value, 2), "unit": "tok/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(round_s * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded); acceptance drawn from a seeded model, not a sampler",
            "config": {"workload": ("spec_stack: self-speculative decode on the 48-layer "
                                    "mixer-only stack, B=32, ctx 32768, H=32, Hkv=8, d=128; "
                                    "target 12 FA/12 SWA(w=4096)/12 KDA/12 GDN, drafter all-GDN, "
                                    "k=3 drafts, acceptance 0.8 per draft; a step is one round"),
                       "inputs": "KV larger than L2 (48 GiB), states 22 GiB"},
            "roofline": with_nominal({"bound": "hbm", "achieved": round(byts / round_s / 1e9, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(byts / round_s / 1e9 / hbm, 4),
                         "traffic": None, "algorithmic_bytes": byts,
                         "scope": "whole round (draft + verify kernels)"}),
            "spec": {"k": k, "alpha": alpha,
                     "mean_drafts_kept": round(float(sched.accepted[args.warmup:].mean()), 4),
                     "tokens_per_round": round(tokens / args.steps, 3),
                     "round_ms": round(round_s * 1e3, 4), "draft_ms": round(draft_s * 1e3, 4),
                     "verify_ms": round(verify_s * 1e3, 4),
                     "plain_step_ms": round(plain_s * 1e3, 4), "plain_tok_s": round(plain_tok_s, 2),
                     "speedup_vs_plain": round(value / plain_tok_s, 4)},
            "gpu_launches": (la["draft"] + la["verify"]) * args.steps}


def run_mixed(args):
    """Mixed placements in one batch on the 48-layer mixer-only stack: B=64, context 32768,
    H=32, Hkv=8, d=128; 32 sequences follow the 12 FA / 12 SWA / 12 KDA / 12 GDN placement and
    32 the all-GDN placement, in one mixed step per token (each layer runs each of its mixers
    over its group of sequences). The single-placement steps of the same stack at the same B
    are timed alongside. Each step is one CUDA-graph replay."""
    import torch

    import hybrid_mixer_decoding_b200 as hmd
    from hybrid_mixer_decoding_b200.stack import MixerStack, StackShape, layer_bytes

    pk, _ = peaks()
    hbm = float(pk["hbm_gbs"])
    shape = StackShape(B=64, H=32, Hkv=8, d=128, ctx=32768, window=4096)
    pls = {"hybrid": stack_placement(), "all_gdn": np.full(48, I.GDN, np.int8)}
    st = MixerStack(pls, shape, fill_kv=False)
    sp = np.array([0, 1] * 32, np.int32)  # interleaved: every other sequence on each preset
    plan = st.batch_plan(sp)
    graphs = {"mixed": st.capture(lambda: st.step_batch(plan)),
              "hybrid": st.capture("hybrid"), "all_gdn": st.capture("all_gdn")}
    sec = {}
    for name, g in graphs.items():
        sec[name] = _events_time(g.replay, args.steps, args.warmup)
    assert hmd.hmd_device_errors(clear=True) == 0
    half = StackShape(B=32, H=32, Hkv=8, d=128, ctx=32768, window=4096)
    byts = sum(layer_bytes(int(k), half) for k in pls["hybrid"]) + \
        sum(layer_bytes(int(k), half) for k in pls["all_gdn"])
    launches = sum((2 if plan.group(l, k).size and k in (I.FA, I.SWA) else
                    1 if plan.group(l, k).size else 0)
                   for l in range(48) for k in (I.FA, I.SWA, I.KDA, I.GDN))
    aliased = st.aliased
    plan.free()
    st.free()
    t = sec["mixed"]
    return {"metric": METRIC, "value": round(shape.B / t, 2), "unit": "tok/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random-init caches, no weights)",
            "config": {"workload": ("mixed_stack: one batch of 64 sequences at ctx 32768 on the "
                                    "48-layer mixer-only stack, 32 on the 12 FA/12 SWA/12 KDA/"
                                    "12 GDN placement and 32 on all-GDN, one mixed step per token"),
                       "kv_aliased": aliased,
                       "inputs": "KV and states larger than L2"},
            "roofline": with_nominal({"bound": "hbm", "achieved": round(byts / t / 1e9, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(byts / t / 1e9 / hbm, 4), "traffic": None,
                         "algorithmic_bytes": byts, "scope": "whole mixed step"}),
            "mixed": {"mixed_ms": round(t * 1e3, 4),
                      "hybrid_B64_ms": round(sec["hybrid"] * 1e3, 4),
                      "all_gdn_B64_ms": round(sec["all_gdn"] * 1e3, 4),
                      "half_of_each_ms": round((sec["hybrid"] + sec["all_gdn"]) / 2 * 1e3, 4)},
            "gpu_launches": launches * args.steps}


SWEEP_CTX = (4096, 16384, 65536, 131072)


def sweep_placements():
    return {
        "all-FA": np.full(48, I.FA, np.int8),
        "24FA+24GDN": I.placement({I.FA: 24, I.GDN: 24}, seed=0),
        "8FA+20KDA+20GDN": I.placement({I.FA: 8, I.KDA: 20, I.GDN: 20}, seed=0),
        "all-GDN": np.full(48, I.GDN, np.int8),
        "all-KDA": np.full(48, I.KDA, np.int8),
    }


PURE = {I.FA: "all-FA", I.KDA: "all-KDA", I.GDN: "all-GDN"}


def linear_cost_model(pls, res):
    """The pages' cost model: a placement's step time is the sum of its layers' costs. Per-layer
    costs come from the single-kind placements (step / 48); the mixed placements are predicted
    from their mixer counts and compared with their measured step times."""
    per_layer = {k: res[name]["ms_per_step"] / len(pls[name]) for k, name in PURE.items()}
    out = {"per_layer_us": {I.KIND_NAMES[k]: round(v * 1e3, 2) for k, v in per_layer.items()},
           "predicted_ms": {}, "error_pct": {}}
    for name, pl in pls.items():
        if name in PURE.values():
            continue
        pred = sum(per_layer[int(k)] for k in pl)
        out["predicted_ms"][name] = round(pred, 3)
        out["error_pct"][name] = round(100.0 * (res[name]["ms_per_step"] / pred - 1.0), 2)
    return out


def run_sweep(args, ctxs=SWEEP_CTX, steps=None):
    """Context sweep: B=16, ctx in {4k, 16k, 64k, 128k} (or `ctxs`), 48-layer stack, placements
    all-FA, 24 FA + 24 GDN, 8 FA + 40 (20 KDA + 20 GDN), all-GDN, all-KDA; decode tok/s, speedup
    over all-FA, and the linear per-layer cost model checked against the mixed placements.
    KV pools are zero-filled (timing only); FA layers share physical pools round-robin when the
    placement's KV exceeds device memory (each layer still streams its own full context)."""
    import torch

    from hybrid_mixer_decoding_b200.stack import MixerStack, StackShape, layer_bytes
    pls = sweep_placements()
    steps = args.steps if steps is None else steps
    rows = []
    for ctx in ctxs:
        shape = StackShape(16, 32, 8, 128, ctx, 4096)
        st = MixerStack(pls, shape, seed=0, fill_kv=False)
        res = {}
        graphs = {name: st.capture(name) for name in pls}
        for name in pls:
            sec = _events_time(graphs[name].replay, steps, args.warmup)
            byts = sum(layer_bytes(int(k), shape) for k in pls[name])
            res[name] = {"tok_s": round(16 / sec, 1), "ms_per_step": round(sec * 1e3, 3),
                         "achieved_gbs": round(byts / sec / 1e9, 1)}
        fa_bytes = sum(layer_bytes(int(k), shape) for k in pls["all-FA"])
        for name in pls:
            res[name]["speedup_vs_all_fa"] = round(res[name]["tok_s"] / res["all-FA"]["tok_s"], 3)
            res[name]["predicted_by_bytes"] = round(
                fa_bytes / sum(layer_bytes(int(k), shape) for k in pls[name]), 3)
        rows.append({"ctx": ctx, "aliased_fa_pools": st.n_fa_pools if st.aliased else None,
                     "placements": res, "linear_cost_model": linear_cost_model(pls, res)})
        del graphs
        st.free()
        del st
        torch.cuda.empty_cache()
    return {"metric": "decode tok/s per placement (BxCtx), context sweep", "workload":
            "sweep: 48-layer mixer-only stack, B=16, H=32, Hkv=8, d=128, SWA-free placements; "
            "each step one CUDA-graph replay of the 48 mixer_decode_step calls",
            "steps": steps, "warmup": args.warmup, "rows": rows}


def next_row_lines(args) -> dict:
    """Self-speculative decoding and a mixed-placement batch on the 48-layer stack (B=32 and
    B=64 at ctx 32768), each with its roofline, for the one-GPU bench line; the full lines are
    --workload spec_stack and mixed_stack. A failure is recorded in the line, not raised."""
    import argparse as _ap

    import torch
    short = _ap.Namespace(**{**vars(args), "steps": min(args.steps, 10)})
    keep = ("value", "unit", "ms_per_step", "roofline", "spec", "mixed", "config")
    out = {}
    for key, fn in (("speculative", run_spec), ("mixed_batch", run_mixed)):
        try:
            r = fn(short)
            out[key] = {k: r[k] for k in keep if k in r}
        except Exception as e:  # noqa: BLE001 - reported in the line
            out[key] = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def context_sweep_line(args) -> dict:
    """The hybrid placements' decode speedup over all-FA at 8k and 128k context (B=16, 48 layers,
    CUDA-graph replays), for the one-GPU bench line; the full sweep is --workload sweep."""
    r = run_sweep(args, ctxs=(8192, 131072), steps=min(args.steps, 10))
    return {"workload": r["workload"], "steps": r["steps"],
            "rows": [{"ctx": row["ctx"], "aliased_fa_pools": row["aliased_fa_pools"],
                      "tok_s": {n: v["tok_s"] for n, v in row["placements"].items()},
                      "speedup_vs_all_fa": {n: v["speedup_vs_all_fa"] for n, v in row["placements"].items()},
                      "predicted_by_bytes": {n: v["predicted_by_bytes"] for n, v in row["placements"].items()},
                      "achieved_gbs": {n: v["achieved_gbs"] for n, v in row["placements"].items()},
                      "linear_cost_model": row["linear_cost_model"]}
                     for row in r["rows"]]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (used for profiler runs)")
    ap.add_argument("--headline-only", action="store_true",
                    help="stack48: only the 48-layer line (no per-mixer prefill/decode lines)")
    ap.add_argument("--workload", default="stack48",
                    choices=["stack48", "attn_fa", "attn_swa", "prefill_fa", "prefill_swa",
                             "decode_kda", "decode_gdn",
                             "prefill_kda", "prefill_gdn", "verify_fa", "verify_swa",
                             "spec_stack", "mixed_stack", "sweep"])
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    elif args.workload == "stack48":
        out = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.headline_only:
            # per-mixer prefill and decode lines and the fp32 oracle check, on this rank's GPU
            out.update(per_mixer_lines(args))
            out["oracle_check"] = oracle_check_config1()
            out["context_sweep"] = context_sweep_line(args)
            out.update(next_row_lines(args))
    elif args.workload == "sweep":
        out = run_sweep(args)
    elif args.workload == "spec_stack":
        out = run_spec(args)
    elif args.workload == "mixed_stack":
        out = run_mixed(args)
    else:
        out = run_kernel_workload(args)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
