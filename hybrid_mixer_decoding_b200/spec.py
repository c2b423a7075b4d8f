"""Self-speculative decoding on the mixer-only stack: a cheap placement of the supernet drafts k
tokens, the target placement checks all k + 1 positions in one pass.

The pages present the supernet's placements as speed/quality presets of one checkpoint, switched
without reloading weights, and name speculative decoding with a cheaper preset as a use of it
("Super Apriel: One Checkpoint, Many Speeds", abstract; gist.science technical summary,
sections 1 and 4). This module is the decode-side machinery of that loop for the token mixers,
with no projections, MLPs or sampler (so no tokens): per round, for every sequence,

  draft:  the drafter placement (all GDN by default) runs k + 1 decode steps on its inputs
          x_0, d_1, ..., d_k; step t reads state slot s_t and writes s_{t+1}
          (delta_rule_decode_to), so every intermediate state is kept;
  verify: the target placement checks the k + 1 positions at once: its attention layers in one
          attn_verify pass (n_q = k + 1 query rows per sequence), its GDN/KDA layers in one
          delta_rule_decode_chain launch (the state read once, the state after each position
          stored along the same slot chain);
  accept: j_b of the k drafts are kept (plus the target's own token): the drafter's and the
          target's recurrent state are then slot s_{j_b + 1}, chosen without copying, and the
          attention caches keep L_b + j_b + 1 positions (the rejected ones are overwritten
          later; the SWA ring holds window + k positions, so they never clobber a live key).

Acceptance is an input: without weights there is no distribution to sample, so j_b is drawn
from a seeded model (each draft kept with probability alpha until the first rejection), and the
report states alpha. Each round's kernels are one CUDA graph; the slot chains and lengths of
every round are precomputed on the host and copied device-to-device before each replay.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib as L
from .inputs import FA, GDN, KDA, SWA, layer_seed, rng
from .stack import StackShape, _gen

PAGE = 64


def accept_counts(g: np.random.Generator, B: int, k: int, alpha: float) -> np.ndarray:
    """Drafts kept per sequence: the number of leading successes of k Bernoulli(alpha) trials."""
    ok = g.random((B, k)) < alpha
    first_reject = np.where(~ok, np.arange(k)[None, :], k).min(axis=1)
    return first_reject.astype(np.int32)


def chain_slots(cur: np.ndarray, k: int) -> np.ndarray:
    """Slot of chain position t for sequence b, [k + 2][B] int32: each sequence owns k + 2
    consecutive slots used as a ring starting at its current position cur[b]."""
    n = k + 2
    B = len(cur)
    t = np.arange(n)[:, None]
    return (np.arange(B)[None, :] * n + (cur[None, :] + t) % n).astype(np.int32)


@dataclass
class Schedule:
    slots: np.ndarray     # [rounds][k + 2][B] int32
    lens: np.ndarray      # [rounds][B] int32: attention lengths of each verify pass (L + k + 1)
    accepted: np.ndarray  # [rounds][B] int32: drafts kept in each round
    tokens: np.ndarray    # [rounds] int: tokens produced by each round (sum over b of j_b + 1)


def make_schedule(B: int, k: int, rounds: int, L0: int, alpha: float, seed: int = 0) -> Schedule:
    """The host side of `rounds` speculative rounds starting from L0 cached positions."""
    g = rng(seed)
    cur = np.zeros(B, np.int32)
    L = np.full(B, L0, np.int32)
    slots = np.empty((rounds, k + 2, B), np.int32)
    lens = np.empty((rounds, B), np.int32)
    acc = np.empty((rounds, B), np.int32)
    for r in range(rounds):
        slots[r] = chain_slots(cur, k)
        lens[r] = L + k + 1
        j = accept_counts(g, B, k, alpha)
        acc[r] = j
        cur = ((cur + j + 1) % (k + 2)).astype(np.int32)
        L = L + j + 1
    return Schedule(slots, lens, acc, (acc + 1).sum(axis=1))


class SpecStack:
    def __init__(self, target: np.ndarray, shape: StackShape, k: int, max_rounds: int,
                 drafter: np.ndarray | None = None, seed: int = 0, fill: bool = False):
        """target / drafter: placement vectors (drafter defaults to all GDN). shape.ctx bounds
        every length reached: the caches start with ctx - (k + 1) * max_rounds positions.
        fill=False leaves the KV pools zero (timing runs; the data does not change the work)."""
        self.target = np.asarray(target, np.int8)
        self.n_layers = nl = len(self.target)
        self.drafter = (np.full(nl, GDN, np.int8) if drafter is None
                        else np.asarray(drafter, np.int8))
        assert set(self.drafter.tolist()) <= {GDN, KDA}, "the drafter runs recurrent mixers only"
        self.shape = s = shape
        self.k, self.n_q = k, k + 1
        B, H, Hkv, d = s.B, s.H, s.Hkv, s.d
        assert self.n_q * (H // Hkv) <= 16, "k + 1 query rows per kv-head must fit 16"
        n_chain = k + 2
        self.L0 = s.ctx - self.n_q * max_rounds
        assert self.L0 >= 1
        dev = "cuda"
        bf = torch.bfloat16

        # recurrent states: k + 2 slots per sequence for every GDN/KDA layer
        self.t_lin = [l for l in range(nl) if self.target[l] in (GDN, KDA)]
        self.t_state = L.StateCache(max(1, len(self.t_lin)), B * n_chain, H, d, d)
        self.d_state = L.StateCache(nl, B * n_chain, H, d, d)
        for i, l in enumerate(self.t_lin):
            self.t_state.layer_view(i).normal_(0.0, 1.0 / math.sqrt(d),
                                               generator=_gen(layer_seed(l, 90) + seed))
        for l in range(nl):
            self.d_state.layer_view(l).normal_(0.0, 1.0 / math.sqrt(d),
                                               generator=_gen(layer_seed(l, 91) + seed))

        # paged KV: FA covers ctx; SWA keeps a ring of window + k positions
        self.ring = -(-(s.window + k) // PAGE)
        self.fa = [l for l in range(nl) if self.target[l] == FA]
        self.swa = [l for l in range(nl) if self.target[l] == SWA]
        pps_fa = -(-s.ctx // PAGE)
        self.kv_fa = self.kv_swa = None
        if self.fa:
            lp = [self.fa.index(l) if l in self.fa else -1 for l in range(nl)]
            self.kv_fa = L.KVCache(lp, len(self.fa), B * pps_fa, Hkv, d, PAGE)
            self.table_fa = torch.randperm(B * pps_fa, generator=_gen(seed + 7), device=dev).to(
                torch.int32).view(B, pps_fa).contiguous()
        if self.swa:
            lp = [self.swa.index(l) if l in self.swa else -1 for l in range(nl)]
            self.kv_swa = L.KVCache(lp, len(self.swa), B * self.ring, Hkv, d, PAGE)
            self.table_swa = torch.randperm(B * self.ring, generator=_gen(seed + 8),
                                            device=dev).to(torch.int32).view(B, self.ring).contiguous()
        if fill:
            for cache, layers in ((self.kv_fa, self.fa), (self.kv_swa, self.swa)):
                for l in layers:
                    kp, vp = cache.layer_pools(l)
                    kp.normal_(generator=_gen(layer_seed(l, 10) + seed))
                    vp.normal_(generator=_gen(layer_seed(l, 11) + seed))

        # per-layer inputs (resident; each round reads the same values)
        nq = self.n_q

        def lin_inputs(l, kind, tag, seq_major):
            """[nq][B][...] for the drafter's token-by-token steps; [B][nq][...] for the
            target's chain launches (plus token 0 alone, for its plain decode step)."""
            shp = (B, nq) if seq_major else (nq, B)
            t = {}
            t["q"] = torch.randn(*shp, H, d, generator=_gen(layer_seed(l, tag) + seed), device=dev).to(bf)
            kk = torch.randn(*shp, H, d, generator=_gen(layer_seed(l, tag + 1) + seed), device=dev)
            t["k"] = torch.nn.functional.normalize(kk, dim=-1).to(bf)
            t["v"] = torch.randn(*shp, H, d, generator=_gen(layer_seed(l, tag + 2) + seed), device=dev).to(bf)
            t["beta"] = torch.sigmoid(torch.randn(*shp, H, generator=_gen(layer_seed(l, tag + 3) + seed),
                                                  device=dev))
            if kind == KDA:
                t["lg"] = -0.05 * torch.rand(*shp, H, d, generator=_gen(layer_seed(l, tag + 4) + seed),
                                             device=dev)
            else:
                t["lg"] = -0.1 * torch.rand(*shp, H, generator=_gen(layer_seed(l, tag + 4) + seed),
                                            device=dev)
            t["o"] = torch.empty(*shp, H, d, device=dev, dtype=bf)
            if seq_major:
                for x in ("q", "k", "v", "beta", "lg", "o"):
                    t[x + "1"] = t[x][:, 0].contiguous()
            return t

        self.t_in, self.d_in = [], []
        for l in range(nl):
            kind = int(self.target[l])
            if kind in (GDN, KDA):
                self.t_in.append(lin_inputs(l, kind, 20, seq_major=True))
            else:
                t = {"q": torch.randn(B, nq, H, d, generator=_gen(layer_seed(l, 0) + seed), device=dev).to(bf),
                     "nk": torch.randn(B, nq, Hkv, d, generator=_gen(layer_seed(l, 6) + seed), device=dev).to(bf),
                     "nv": torch.randn(B, nq, Hkv, d, generator=_gen(layer_seed(l, 7) + seed), device=dev).to(bf),
                     "o": torch.empty(B, nq, H, d, device=dev, dtype=bf)}
                # one-token copies for the plain decode step of the target placement
                t["q1"], t["nk1"], t["nv1"] = (t[x][:, :1].contiguous() for x in ("q", "nk", "nv"))
                t["o1"] = torch.empty(B, 1, H, d, device=dev, dtype=bf)
                self.t_in.append(t)
            self.d_in.append(lin_inputs(l, int(self.drafter[l]), 40, seq_major=False))

        ws = max([L.attn_verify_workspace_size(FA, 0, nq, B, H, Hkv, d, PAGE, s.ctx),
                  L.attn_verify_workspace_size(SWA, s.window, nq, B, H, Hkv, d, PAGE, s.ctx)])
        self.ws = torch.empty(max(16, ws), dtype=torch.uint8, device=dev)
        # per-round device state: the slot chain and the attention lengths
        self.slot_buf = torch.zeros(n_chain, B, dtype=torch.int32, device=dev)
        self.lens_v = torch.full((B,), self.L0 + nq, dtype=torch.int32, device=dev)
        self.lens_1 = torch.full((B,), self.L0 + 1, dtype=torch.int32, device=dev)
        self.slot_buf.copy_(torch.from_numpy(chain_slots(np.zeros(B, np.int32), k)))
        torch.cuda.synchronize()

    # ---- the three phases ------------------------------------------------------------------
    def _lin_step(self, kind, t_in, state, t, src, dst):
        L.delta_rule_decode_to(kind, t_in["q"][t], t_in["k"][t], t_in["v"][t], t_in["beta"][t],
                               t_in["lg"][t], state, t_in["o"][t], src, dst)

    def draft(self):
        for t in range(self.n_q):
            for l in range(self.n_layers):
                self._lin_step(int(self.drafter[l]), self.d_in[l], self.d_state.layer_view(l), t,
                               self.slot_buf[t], self.slot_buf[t + 1])

    def _attn(self, l, kind, q, nk, nv, o, lens):
        cache, table = (self.kv_fa, self.table_fa) if kind == FA else (self.kv_swa, self.table_swa)
        kp, vp = cache.layer_pools(l)
        L.attn_verify(kind, self.shape.window, self.ring, q, nk, nv, kp, vp, table, lens,
                      self.shape.ctx, o, self.ws)

    def verify(self):
        for l in range(self.n_layers):
            kind, t_in = int(self.target[l]), self.t_in[l]
            if kind in (FA, SWA):
                self._attn(l, kind, t_in["q"], t_in["nk"], t_in["nv"], t_in["o"], self.lens_v)
            else:  # k + 1 tokens in one launch: the state read once, each step stored
                st = self.t_state.layer_view(self.t_lin.index(l))
                L.delta_rule_decode_chain(kind, t_in["q"], t_in["k"], t_in["v"], t_in["beta"],
                                          t_in["lg"], st, t_in["o"], self.slot_buf)

    def plain_step(self):
        """One ordinary decode token of the target placement (its states updated in place)."""
        for l in range(self.n_layers):
            kind, t_in = int(self.target[l]), self.t_in[l]
            if kind in (FA, SWA):
                self._attn(l, kind, t_in["q1"], t_in["nk1"], t_in["nv1"], t_in["o1"], self.lens_1)
            else:
                st = self.t_state.layer_view(self.t_lin.index(l))
                L.delta_rule_decode_to(kind, t_in["q1"], t_in["k1"], t_in["v1"], t_in["beta1"],
                                       t_in["lg1"], st, t_in["o1"], self.slot_buf[0],
                                       self.slot_buf[0])

    def set_round(self, sched: Schedule, r: int, slots_dev: torch.Tensor, lens_dev: torch.Tensor):
        """Stream-ordered device-to-device copies of round r's slot chain and lengths."""
        self.slot_buf.copy_(slots_dev[r], non_blocking=True)
        self.lens_v.copy_(lens_dev[r], non_blocking=True)

    def capture(self, fn) -> torch.cuda.CUDAGraph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g

    def launches(self) -> dict:
        n_lin_t = len(self.t_lin)
        n_att = self.n_layers - n_lin_t
        return {"draft": self.n_q * self.n_layers,
                "verify": 2 * n_att + n_lin_t,
                "plain": 2 * n_att + n_lin_t}

    def free(self):
        for c in (self.kv_fa, self.kv_swa, self.t_state, self.d_state):
            if c is not None:
                c.free()
        torch.cuda.synchronize()
