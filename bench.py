#!/usr/bin/env python
"""Decode throughput of the 48-layer mixer-only stack, one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload stack48|attn_fa|attn_swa|decode_kda|decode_gdn|prefill_kda|
                                prefill_gdn|sweep]

Default workload ("stack48"): 48 layers, placement 12 FA / 12 SWA (w=4096) / 12 KDA / 12 GDN
randomly interleaved (seed 0), B=64 sequences at context 32768, H=32 query/delta heads, 8 KV
heads, d=128, bf16 activations and KV, fp32 states. A step decodes one token for every sequence
through all 48 layers; the metric is tokens/s = B / step time. Every layer's working set is
larger than L2 (state 128 MiB, KV >= 1 GiB) and a step touches ~122 GB, so no L2 flush is needed.

Multi-GPU (torchrun): replicas only -- every rank runs its own copy of the workload on its own
caches (weak scaling, no collective on the data path); value = all ranks' tokens / the slowest
rank's time.

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
    st = MixerStack({"hybrid": pl}, shape, seed=0)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        st.step("hybrid")
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0

    # per-layer events for every layer (cheap: two event records per layer)
    n_layers = st.n_layers
    evs = [{l: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for l in range(n_layers)} for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clk.start()
    t0.record()
    for k in range(args.steps):
        st.step("hybrid", events=evs[k])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    ms = t0.elapsed_time(t1)
    if dist is not None:
        tt = torch.tensor([ms], device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    ms_per_step = ms / args.steps
    tokens = shape.B * args.steps * world
    value = tokens / (ms * 1e-3)

    # per-mixer achieved bandwidth from the per-layer events
    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    per_kind = {}
    for kind in (I.FA, I.SWA, I.KDA, I.GDN):
        layers = [l for l in range(n_layers) if pl[l] == kind]
        if not layers:
            continue
        durs = [evs[k][l][0].elapsed_time(evs[k][l][1]) for k in range(args.steps) for l in layers]
        mean_ms = float(np.mean(durs))
        gbs = layer_bytes(kind, shape) / (mean_ms * 1e-3) / 1e9
        per_kind[I.KIND_NAMES[kind]] = {"layer_us": round(mean_ms * 1e3, 2),
                                        "achieved_gbs": round(gbs, 1),
                                        "frac": round(gbs / hbm, 4),
                                        "frac_nominal_8tbs": round(gbs / 8000.0, 4),
                                        "bytes_per_layer": layer_bytes(kind, shape)}
    dom = per_kind["FA"]
    roofline = {"bound": "hbm", "achieved": dom["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                "frac": dom["frac"], "traffic": traffic_for("attn_fa_stack48"),
                "kernel": "attn_decode FA layer (attn_split_kernel<128> + attn_combine_kernel)",
                "peak_source": pk_kind}
    assert hmd.hmd_device_errors(clear=True) == 0

    # end to end through the C ABI from pinned host buffers: per step, copy every layer's
    # inputs host->device, run the step, copy every layer's output device->host
    host_in, dev_in, host_out = [], [], []
    for l in range(n_layers):
        t = st.inputs[l]
        names = ["q", "k", "v", "beta", "lg_s", "lg_c"] if pl[l] in (I.GDN, I.KDA) else ["q", "nk", "nv"]
        if pl[l] == I.GDN:
            names.remove("lg_c")
        if pl[l] == I.KDA:
            names.remove("lg_s")
        for nm in names:
            host_in.append(torch.empty_like(t[nm], device="cpu").pin_memory().copy_(t[nm]))
            dev_in.append(t[nm])
        host_out.append(torch.empty_like(t["o"], device="cpu").pin_memory())
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out)

    def e2e_step():
        for h, dv in zip(host_in, dev_in):
            dv.copy_(h, non_blocking=True)
        st.step("hybrid")
        for l in range(n_layers):
            host_out[l].copy_(st.inputs[l]["o"], non_blocking=True)

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    ems = e0.elapsed_time(e1)
    if dist is not None:
        tt = torch.tensor([ems], device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ems = float(tt.item())
    e2e = {"value": round(tokens / (ems * 1e-3), 2), "unit": "tok/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h}

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
                   "l2": "working set per step ~122 GB >> L2 (126 MB); no flush",
                   "aliased_kv": st.aliased},
        "roofline": roofline,
        "per_mixer": per_kind,
        "e2e": e2e,
        "gpu_launches": st.launches_per_step("hybrid") * args.steps,
        "clocks": clocks,
    }
    st.free()
    if rank == 0 and not args.skip_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(shape, pl, budget_s=args.cpu_budget)
    if dist is not None:
        dist.destroy_process_group()
    return out


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
    return {"value": round(n_seq / step_s, 4), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 C oracle, {n_seq} sequences at the stack's per-layer shapes "
                      f"(H=32, Hkv=8, d=128, ctx 32768, w=4096); each mixer kind timed on one "
                      f"layer, summed over the placement's 48 layers; tokens/s = "
                      f"{n_seq} / summed time",
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (used for profiler runs)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        out = run_ours(args, rank, world, local_rank)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
