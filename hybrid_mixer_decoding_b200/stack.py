"""A mixer-only decode stack: n_layers layers, each able to run any of the four mixers, driven
by a placement vector through mixer_decode_step.

The supernet's placements pick one mixer per layer and can be switched between requests without
reloading weights ("Super Apriel: One Checkpoint, Many Speeds", abstract; gist.science technical
summary, section 2d). Here the stack registers, for every layer, the caches of every mixer kind
that any of its placements can ask for (a recurrent-state block for GDN/KDA, a paged KV pool for
FA/SWA), together with per-layer inputs for each kind. Switching placement is then calling step()
with another name: nothing is copied or reallocated.

There are no projections or MLPs: each layer's q/k/v/gates are synthetic, drawn once on the
device from per-layer seeds, and every step decodes one token per sequence at a fixed context
length (the new token is written to position ctx-1 of every attention layer each step).

When the KV of all attention layers does not fit in device memory, FA-capable layers share
physical pools round-robin ("aliased"); each layer still streams its own full context from HBM,
so the traffic per step is unchanged.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib as L
from .inputs import FA, GDN, KDA, SWA, layer_seed

PAGE = 64


@dataclass
class StackShape:
    B: int
    H: int
    Hkv: int
    d: int
    ctx: int       # context length per sequence, including the token decoded by each step
    window: int    # SWA window


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return g


class MixerStack:
    def __init__(self, placements: dict[str, np.ndarray], shape: StackShape, seed: int = 0,
                 mem_fraction: float = 0.9, fill_kv: bool = True, io_sets: int = 1):
        """fill_kv=False leaves the KV pools zero-filled (as allocated), for timing runs whose
        results are not checked: the data does not change the work done. io_sets > 1 keeps
        that many independent sets of per-layer input/output buffers (same initial values), so
        a caller can copy the next step's inputs into one set while a step runs on another."""
        self.placements = {k: np.asarray(v, dtype=np.int8) for k, v in placements.items()}
        self.names = list(self.placements)
        self.n_layers = len(next(iter(self.placements.values())))
        assert all(len(p) == self.n_layers for p in self.placements.values())
        self.shape = s = shape
        B, H, Hkv, d = s.B, s.H, s.Hkv, s.d
        kinds_of = [set(int(p[l]) for p in self.placements.values()) for l in range(self.n_layers)]
        self.kinds_of = kinds_of

        # --- recurrent states: one [B,H,d,d] fp32 block per layer ------------------------------
        self.state = L.StateCache(self.n_layers, B, H, d, d)
        for l in range(self.n_layers):
            if kinds_of[l] & {GDN, KDA}:
                v = self.state.layer_view(l)
                v.normal_(0.0, 1.0 / math.sqrt(d), generator=_gen(layer_seed(l, 90) + seed))

        # --- paged KV pools -------------------------------------------------------------------
        self.pages_fa = B * (-(-s.ctx // PAGE))
        R = -(-s.window // PAGE)
        self.ring = R
        self.pages_swa = B * min(R, -(-s.ctx // PAGE))
        fa_layers = [l for l in range(self.n_layers) if FA in kinds_of[l]]
        swa_layers = [l for l in range(self.n_layers) if SWA in kinds_of[l] and FA not in kinds_of[l]]
        pool_bytes = lambda pages: 2 * pages * Hkv * PAGE * d * 2  # noqa: E731
        free, _total = torch.cuda.mem_get_info()
        budget = int(free * mem_fraction) - pool_bytes(self.pages_swa) * len(swa_layers) - (2 << 30)
        n_fa_pools = len(fa_layers)
        if fa_layers and pool_bytes(self.pages_fa) * n_fa_pools > budget:
            n_fa_pools = max(1, budget // pool_bytes(self.pages_fa))
        self.aliased = bool(fa_layers) and n_fa_pools < len(fa_layers)
        self.n_fa_pools = n_fa_pools
        self.kv_fa = self.kv_swa = None
        if fa_layers:
            lp = [-1] * self.n_layers
            for i, l in enumerate(fa_layers):
                lp[l] = i % n_fa_pools
            self.kv_fa = L.KVCache(lp, n_fa_pools, self.pages_fa, Hkv, d, PAGE)
        if swa_layers:
            lp = [-1] * self.n_layers
            for i, l in enumerate(swa_layers):
                lp[l] = i
            self.kv_swa = L.KVCache(lp, len(swa_layers), self.pages_swa, Hkv, d, PAGE)
        if fill_kv:
            self._fill_pools(fa_layers, swa_layers, seed)

        # page tables (a seeded random permutation of each pool's pages) and lengths
        dev = "cuda"
        self.table_fa = torch.randperm(self.pages_fa, generator=_gen(seed + 7), device=dev).to(
            torch.int32).view(B, -1).contiguous()
        if self.kv_swa is not None:
            self.table_swa = torch.randperm(self.pages_swa, generator=_gen(seed + 8),
                                            device=dev).to(torch.int32).view(B, -1).contiguous()
            if self.table_swa.shape[1] < R:
                pad = torch.full((B, R - self.table_swa.shape[1]), -1, dtype=torch.int32,
                                 device=dev)
                self.table_swa = torch.cat([self.table_swa, pad], 1).contiguous()
        # a FA-capable layer running as SWA uses the first R entries of its FA table
        self.table_fa_ring = self.table_fa[:, :min(R, self.table_fa.shape[1])].contiguous()
        self.seq_lens = torch.full((B,), s.ctx, dtype=torch.int32, device=dev)

        # --- per-layer inputs for every kind a layer can take ------------------------------------
        self.inputs = []
        self.io = []
        bf = torch.bfloat16
        for l in range(self.n_layers):
            t = {}
            t["q"] = torch.randn(B, H, d, generator=_gen(layer_seed(l, 0) + seed), device=dev).to(bf)
            t["o"] = torch.empty(B, H, d, device=dev, dtype=bf)
            if kinds_of[l] & {GDN, KDA}:
                kk = torch.randn(B, H, d, generator=_gen(layer_seed(l, 1) + seed), device=dev)
                t["k"] = torch.nn.functional.normalize(kk, dim=-1).to(bf)
                t["v"] = torch.randn(B, H, d, generator=_gen(layer_seed(l, 2) + seed), device=dev).to(bf)
                t["beta"] = torch.sigmoid(torch.randn(B, H, generator=_gen(layer_seed(l, 3) + seed),
                                                      device=dev))
                t["lg_s"] = -0.1 * torch.rand(B, H, generator=_gen(layer_seed(l, 4) + seed), device=dev)
                t["lg_c"] = -0.05 * torch.rand(B, H, d, generator=_gen(layer_seed(l, 5) + seed),
                                               device=dev)
            if kinds_of[l] & {FA, SWA}:
                t["nk"] = torch.randn(B, Hkv, d, generator=_gen(layer_seed(l, 6) + seed), device=dev).to(bf)
                t["nv"] = torch.randn(B, Hkv, d, generator=_gen(layer_seed(l, 7) + seed), device=dev).to(bf)
            self.inputs.append(t)
            self.io.append(self._make_io(l, t))
        # further buffer sets: copies of the same inputs, their own outputs
        self.input_sets = [self.inputs]
        self.io_sets = [self.io]
        for _ in range(1, io_sets):
            ts = [{k: v.clone() for k, v in t.items()} for t in self.inputs]
            self.input_sets.append(ts)
            self.io_sets.append([self._make_io(l, ts[l]) for l in range(self.n_layers)])
        ws_bytes = max(L.attn_decode_workspace_size(FA, 0, B, H, Hkv, d, PAGE, s.ctx),
                       L.attn_decode_workspace_size(SWA, s.window, B, H, Hkv, d, PAGE, s.ctx))
        self.ws = torch.empty(max(16, ws_bytes), dtype=torch.uint8, device=dev)
        self.c_placements = {k: (np.ctypeslib.as_ctypes(v)) for k, v in self.placements.items()}
        torch.cuda.synchronize()

    def _make_io(self, l: int, t: dict) -> dict:
        """hmd_decode_io_t for every kind layer l can take, pointing at the tensors in t."""
        s = self.shape
        ios = {}
        for kind in self.kinds_of[l]:
            io = L.DecodeIO(B=s.B, H=s.H, Hkv=s.Hkv, d=s.d, dtype=L.BF16)
            io.q, io.o, io.scale = t["q"].data_ptr(), t["o"].data_ptr(), 1.0
            if kind in (GDN, KDA):
                io.k, io.v = t["k"].data_ptr(), t["v"].data_ptr()
                io.beta = t["beta"].data_ptr()
                io.log_gate_scalar = t["lg_s"].data_ptr()
                io.log_gate_channel = t["lg_c"].data_ptr()
            else:
                io.k, io.v = t["nk"].data_ptr(), t["nv"].data_ptr()
                io.seq_lens, io.max_seq_len, io.window = self.seq_lens.data_ptr(), s.ctx, s.window
                tab = self.table_for(l, kind)
                io.page_table, io.max_pages = tab.data_ptr(), tab.shape[1]
            ios[kind] = io
        return ios

    def _fill_pools(self, fa_layers, swa_layers, seed):
        done = set()
        for cache, layers in ((self.kv_fa, fa_layers), (self.kv_swa, swa_layers)):
            if cache is None:
                continue
            for l in layers:
                kp, vp = cache.layer_pools(l)
                if kp.data_ptr() in done:
                    continue
                done.add(kp.data_ptr())
                kp.normal_(generator=_gen(layer_seed(l, 10) + seed))
                vp.normal_(generator=_gen(layer_seed(l, 11) + seed))

    def table_for(self, layer: int, kind: int) -> torch.Tensor:
        if FA in self.kinds_of[layer]:
            return self.table_fa if kind == FA else self.table_fa_ring
        return self.table_swa

    def kv_for(self, layer: int):
        if FA in self.kinds_of[layer]:
            return self.kv_fa
        if SWA in self.kinds_of[layer]:
            return self.kv_swa
        return None

    def pools_for(self, layer: int):
        return self.kv_for(layer).layer_pools(layer)

    def step(self, name: str, events: dict | None = None, io_set: int = 0,
             layers=None) -> None:
        """One decode token for every sequence through all layers under placement `name`,
        reading and writing the per-layer buffers of set `io_set`.
        events: optional {layer: (start_event, end_event)} recorded around that layer.
        layers: optional subset of the layer indices to run (in order); default all."""
        pl = self.placements[name]
        cpl = self.c_placements[name]
        ios = self.io_sets[io_set]
        for l in (range(self.n_layers) if layers is None else layers):
            kind = int(pl[l])
            ev = events.get(l) if events else None
            if ev:
                ev[0].record()
            L.mixer_decode_step(cpl, l, ios[l][kind], self.state,
                                self.kv_for(l) if kind in (FA, SWA) else None,
                                self.ws if kind in (FA, SWA) else None)
            if ev:
                ev[1].record()

    def batch_plan(self, seq_placement) -> "L.BatchPlan":
        """A mixed-batch plan: sequence b follows placement names[seq_placement[b]] (names in
        the order of self.names). Grows the attention workspace to what the plan needs."""
        pl = np.stack([self.placements[n] for n in self.names])
        plan = L.BatchPlan(pl, seq_placement)
        s = self.shape
        need = plan.workspace_size(s.window, s.H, s.Hkv, s.d, PAGE, s.ctx)
        if need > self.ws.numel():
            self.ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        return plan

    def step_batch(self, plan: "L.BatchPlan", io_set: int = 0) -> None:
        """One decode token for every sequence of a mixed batch: layer by layer, each mixer
        runs over the sequences whose placement picks it there (mixer_decode_step_batch)."""
        ios = self.io_sets[io_set]
        for l in range(self.n_layers):
            L.mixer_decode_step_batch(plan, l, ios[l], self.state, self.kv_for(l), self.ws)

    def capture(self, name, warmup: int = 2) -> "torch.cuda.CUDAGraph":
        """Capture one step into a CUDA graph (the library's calls allocate nothing and never
        synchronise, so the whole 48-layer step is one graph launch). name: a placement name,
        or a callable that runs one step."""
        fn = name if callable(name) else (lambda: self.step(name))
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g

    def launches_per_step(self, name: str) -> int:
        pl = self.placements[name]
        return int(sum(2 if k in (FA, SWA) else 1 for k in pl))

    def free(self):
        for c in (self.kv_fa, self.kv_swa):
            if c is not None:
                c.free()
        self.state.free()
        torch.cuda.synchronize()


def layer_bytes(kind: int, shape: StackShape) -> int:
    """Algorithmic HBM bytes of one layer's decode step (what the method must move).
    GDN/KDA: the fp32 state read and written, q/k/v/o in bf16, beta and gates in fp32.
    FA/SWA: the K and V of every attended key (ctx, or the window for SWA) in bf16, q and o,
    and the appended token's k and v."""
    B, H, Hkv, d = shape.B, shape.H, shape.Hkv, shape.d
    if kind in (GDN, KDA):
        gate = 4 if kind == GDN else 4 * d
        return B * H * (2 * d * d * 4 + 4 * d * 2 + 4 + gate)
    keys = shape.ctx if kind == FA else min(shape.window, shape.ctx)
    return B * (keys * Hkv * d * 2 * 2 + 2 * H * d * 2 + 2 * Hkv * d * 2)
