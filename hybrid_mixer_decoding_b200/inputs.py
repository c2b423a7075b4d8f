"""Seeded synthetic inputs for the four token mixers.

This module draws random numbers and lays them out in the tensor layouts the library uses.
It performs none of the mixers' arithmetic, so both the CUDA path (through the tests and the
benchmark) and the fp64 oracle (through the tests) can take their inputs from it without sharing
any computation.

Distributions follow the workloads the Super Apriel pages measure on (the supernet's 48 decoder
layers, each with FA / SWA / KDA / GDN mixers; abstract of "Super Apriel: One Checkpoint, Many
Speeds"), with the shapes and value ranges of the mixer-level workloads:

* delta-rule mixers (GDN, KDA): q, v ~ N(0,1); k ~ N(0,1) then L2-normalised per token-head in
  fp32 (before any bf16 rounding); beta = sigmoid(N(0,1)); log-gates ~ U(lo, 0) with lo = -0.1
  for a GDN scalar gate per token-head and lo = -0.05 for a KDA per-channel gate;
* attention mixers (FA, SWA): a paged bf16 KV pool filled with N(0,1), pages of 64 tokens, page
  ids a seeded random permutation of the pool; q and the new token's k, v ~ N(0,1).

bf16 tensors are produced by round-to-nearest-even from fp32 on the host, so the oracle and the
GPU see identical bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Mixer kinds, as numbered by the C ABI (hmd_kind_t).
FA, SWA, KDA, GDN = 0, 1, 2, 3
KIND_NAMES = {FA: "FA", SWA: "SWA", KDA: "KDA", GDN: "GDN"}


def rng(seed: int) -> np.random.Generator:
    """A numpy PCG64 generator; every input is drawn from one of these."""
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even. Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded (RNE) to the nearest bf16 value, returned as fp32."""
    return (bf16_bits(x).astype(np.uint32) << 16).view(np.float32)


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    # Part of the input recipe ("k ~ N(0,1) then L2-normalised"), done in fp32.
    n = np.sqrt(np.sum(x.astype(np.float32) ** 2, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-6))).astype(np.float32)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


@dataclass
class DeltaInputs:
    """Inputs of a GDN or KDA mixer over T tokens (T=1 for one decode step).

    Layouts: q, k [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H]; log_gate [B,T,H] for GDN or
    [B,T,H,dk] for KDA; state0 [B,H,dk,dv] (fp32, the d_k x d_v state of each head).
    When dtype is "bf16", q/k/v hold bf16-representable fp32 values.
    """
    kind: int
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    beta: np.ndarray
    log_gate: np.ndarray
    state0: np.ndarray


def delta_inputs(kind: int, B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                 seed: int = 0, gate_lo: float | None = None, state0: str = "zero",
                 beta_override: float | None = None) -> DeltaInputs:
    """Draw one seeded set of delta-rule inputs (see the module docstring for the recipe)."""
    assert kind in (KDA, GDN) and dtype in ("bf16", "f32")
    g = rng(seed)
    q = g.standard_normal((B, T, H, dk), dtype=np.float32)
    k = _l2_normalise(g.standard_normal((B, T, H, dk), dtype=np.float32))
    v = g.standard_normal((B, T, H, dv), dtype=np.float32)
    beta = _sigmoid(g.standard_normal((B, T, H), dtype=np.float32))
    if beta_override is not None:
        beta = np.full((B, T, H), beta_override, dtype=np.float32)
    if gate_lo is None:
        gate_lo = -0.1 if kind == GDN else -0.05
    gshape = (B, T, H) if kind == GDN else (B, T, H, dk)
    log_gate = g.uniform(gate_lo, 0.0, size=gshape).astype(np.float32)
    if state0 == "zero":
        s0 = np.zeros((B, H, dk, dv), dtype=np.float32)
    elif state0 == "randn":
        s0 = (g.standard_normal((B, H, dk, dv), dtype=np.float32) / np.float32(math.sqrt(dk)))
    else:
        raise ValueError(state0)
    if dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    return DeltaInputs(kind, B, T, H, dk, dv, dtype, q, k, v, beta, log_gate,
                       s0.astype(np.float32))


@dataclass
class DeltaRawInputs:
    """Raw projection outputs for the fused-activation entry points of GDN/KDA.

    q_raw, k_raw [B,T,H,dk] ~ 2 N(0,1) (norms far from 1); v [B,T,H,dv] ~ N(0,1);
    beta_logit [B,T,H] ~ N(0,1); gate_logit [B,T,H] (GDN) or [B,T,H,dk] (KDA) ~ N(0,1);
    A_log [H] = log U(0.5, 2); dt_bias [H] (GDN) or [H,dk] (KDA) ~ U(-5, -3), so that the
    per-token log-gates land near -0.02 as in the configured workloads; state0 [B,H,dk,dv].
    bf16 values are bf16-representable fp32 (the raw q, k, v only).
    """
    kind: int
    dtype: str
    q_raw: np.ndarray
    k_raw: np.ndarray
    v: np.ndarray
    beta_logit: np.ndarray
    gate_logit: np.ndarray
    A_log: np.ndarray
    dt_bias: np.ndarray
    state0: np.ndarray


def delta_raw_inputs(kind: int, B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                     seed: int = 0) -> DeltaRawInputs:
    assert kind in (KDA, GDN) and dtype in ("bf16", "f32")
    g = rng(seed)
    q = 2.0 * g.standard_normal((B, T, H, dk), dtype=np.float32)
    k = 2.0 * g.standard_normal((B, T, H, dk), dtype=np.float32)
    v = g.standard_normal((B, T, H, dv), dtype=np.float32)
    bl = g.standard_normal((B, T, H), dtype=np.float32)
    gl = g.standard_normal((B, T, H) if kind == GDN else (B, T, H, dk), dtype=np.float32)
    A_log = np.log(g.uniform(0.5, 2.0, size=H)).astype(np.float32)
    dt_bias = g.uniform(-5.0, -3.0, size=(H,) if kind == GDN else (H, dk)).astype(np.float32)
    s0 = (g.standard_normal((B, H, dk, dv), dtype=np.float32) / np.float32(math.sqrt(dk)))
    if dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    return DeltaRawInputs(kind, dtype, q, k, v, bl, gl, A_log, dt_bias, s0)


@dataclass
class AttnInputs:
    """Inputs of one FA or SWA decode step over a paged bf16 KV cache.

    k_pool, v_pool: uint16 bf16 bits [P][Hkv][page_tokens][d].
    page_table: int32 [B][max_pages]; entry c is the physical page of logical page c (FA) or of
    ring page c (SWA, ring of R = ceil(window / page_tokens) pages); unused entries are -1.
    seq_lens: int32 [B], the context length including the token being decoded.
    q: bf16 bits [B][Hq][d]; new_k, new_v: bf16 bits [B][Hkv][d] (the decoded token's k and v,
    which the decode step appends to the cache at position seq_len - 1).
    """
    kind: int
    window: int
    B: int
    Hq: int
    Hkv: int
    d: int
    page_tokens: int
    k_pool: np.ndarray
    v_pool: np.ndarray
    page_table: np.ndarray
    seq_lens: np.ndarray
    q: np.ndarray
    new_k: np.ndarray
    new_v: np.ndarray


def pages_per_sequence(kind: int, max_ctx: int, window: int, page_tokens: int) -> int:
    """Pages one sequence occupies: ceil(ctx/64) for FA; for SWA at most the ring's
    R = ceil(window/64) pages."""
    n = -(-max_ctx // page_tokens)
    if kind == SWA:
        n = min(n, -(-window // page_tokens))
    return max(n, 1)


def attn_inputs(kind: int, B: int, Hq: int, Hkv: int, d: int, ctx: int, window: int = 0,
                page_tokens: int = 64, seed: int = 0, permute: bool = True,
                seq_lens: np.ndarray | None = None, extra_pages: int = 0) -> AttnInputs:
    """Draw one seeded paged-KV decode problem (see the module docstring for the recipe).

    ctx is the largest sequence length (including the new token); seq_lens defaults to ctx for
    every sequence. For SWA the ring holds R = ceil(window/64) pages (fewer when every sequence
    is shorter than the window, in which case no slot is ever reused).
    """
    assert kind in (FA, SWA)
    g = rng(seed)
    if seq_lens is None:
        seq_lens = np.full(B, ctx, dtype=np.int32)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    if kind == SWA:
        assert window >= 1
        max_pages = -(-window // page_tokens)   # ring geometry: R pages per sequence
    else:
        max_pages = -(-int(seq_lens.max()) // page_tokens)
    pps = pages_per_sequence(kind, int(seq_lens.max()), window, page_tokens)
    P = B * pps + extra_pages
    perm = g.permutation(P).astype(np.int32) if permute else np.arange(P, dtype=np.int32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    for b in range(B):
        table[b, :pps] = perm[b * pps:(b + 1) * pps]
    shape = (P, Hkv, page_tokens, d)
    k_pool = bf16_bits(g.standard_normal(shape, dtype=np.float32))
    v_pool = bf16_bits(g.standard_normal(shape, dtype=np.float32))
    q = bf16_bits(g.standard_normal((B, Hq, d), dtype=np.float32))
    new_k = bf16_bits(g.standard_normal((B, Hkv, d), dtype=np.float32))
    new_v = bf16_bits(g.standard_normal((B, Hkv, d), dtype=np.float32))
    return AttnInputs(kind, window, B, Hq, Hkv, d, page_tokens, k_pool, v_pool, table,
                      seq_lens, q, new_k, new_v)


@dataclass
class AttnVerifyInputs:
    """Inputs of one FA or SWA verification pass: n_q new tokens per sequence on top of a paged
    cache that already holds positions 0..seq_len-n_q-1.

    q: bf16 bits [B][n_q][Hq][d]; new_k, new_v: bf16 bits [B][n_q][Hkv][d].
    k_pool, v_pool: bf16 bits [P][Hkv][page_tokens][d], N(0,1) in every slot (the cached
    positions are whatever the slot mapping reads there). page_table: int32 [B][max_pages]
    (FA: ceil(ctx/64) pages; SWA: ring_pages), a seeded permutation of the pool when permute.
    seq_lens: int32 [B], counting the n_q new tokens.
    """
    kind: int
    window: int
    ring_pages: int
    n_q: int
    B: int
    Hq: int
    Hkv: int
    d: int
    page_tokens: int
    k_pool: np.ndarray
    v_pool: np.ndarray
    page_table: np.ndarray
    seq_lens: np.ndarray
    q: np.ndarray
    new_k: np.ndarray
    new_v: np.ndarray


def verify_inputs(kind: int, B: int, n_q: int, Hq: int, Hkv: int, d: int, ctx: int,
                  window: int = 0, ring_pages: int = 0, page_tokens: int = 64, seed: int = 0,
                  permute: bool = True, seq_lens: np.ndarray | None = None) -> AttnVerifyInputs:
    """Draw one seeded verification problem (same distributions as attn_inputs). ctx is the
    longest sequence length counting the new tokens; for SWA ring_pages (0: the smallest ring a
    verifier of n_q tokens may use, ceil((window + n_q - 1) / 64)) sets the pages per sequence."""
    assert kind in (FA, SWA) and n_q >= 1
    g = rng(seed)
    if seq_lens is None:
        seq_lens = np.full(B, ctx, dtype=np.int32)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    assert int(seq_lens.min()) >= n_q
    if kind == SWA:
        assert window >= 1
        if ring_pages == 0:
            ring_pages = -(-(window + n_q - 1) // page_tokens)
        max_pages = ring_pages
    else:
        max_pages = -(-int(seq_lens.max()) // page_tokens)
    P = B * max_pages
    perm = g.permutation(P).astype(np.int32) if permute else np.arange(P, dtype=np.int32)
    table = perm.reshape(B, max_pages).copy()
    shape = (P, Hkv, page_tokens, d)
    k_pool = bf16_bits(g.standard_normal(shape, dtype=np.float32))
    v_pool = bf16_bits(g.standard_normal(shape, dtype=np.float32))
    q = bf16_bits(g.standard_normal((B, n_q, Hq, d), dtype=np.float32))
    new_k = bf16_bits(g.standard_normal((B, n_q, Hkv, d), dtype=np.float32))
    new_v = bf16_bits(g.standard_normal((B, n_q, Hkv, d), dtype=np.float32))
    return AttnVerifyInputs(kind, window, ring_pages, n_q, B, Hq, Hkv, d, page_tokens, k_pool,
                            v_pool, table, seq_lens, q, new_k, new_v)


@dataclass
class AttnPrefillInputs:
    """Inputs of one FA or SWA prefill of T prompt tokens per sequence into an empty cache.

    q: bf16 bits [B][T][Hq][d]; k, v: bf16 bits [B][T][Hkv][d].
    page_table: int32 [B][max_pages] (FA: ceil(T/64) pages per sequence; SWA: the ring's
    R = ceil(window/64) pages), physical ids a seeded permutation of the pool when permute.
    n_pages: pool size (the caller allocates [n_pages][Hkv][page_tokens][d] pools).
    """
    kind: int
    window: int
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    page_tokens: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    page_table: np.ndarray
    n_pages: int


def attn_prefill_inputs(kind: int, B: int, T: int, Hq: int, Hkv: int, d: int, window: int = 0,
                        page_tokens: int = 64, seed: int = 0,
                        permute: bool = True) -> AttnPrefillInputs:
    """Draw one seeded attention-prefill problem: q, k, v ~ N(0, 1) rounded to bf16."""
    assert kind in (FA, SWA)
    g = rng(seed)
    max_pages = -(-window // page_tokens) if kind == SWA else -(-T // page_tokens)
    max_pages = max(max_pages, 1)
    P = B * max_pages
    perm = g.permutation(P).astype(np.int32) if permute else np.arange(P, dtype=np.int32)
    table = perm.reshape(B, max_pages).copy()
    q = bf16_bits(g.standard_normal((B, T, Hq, d), dtype=np.float32))
    k = bf16_bits(g.standard_normal((B, T, Hkv, d), dtype=np.float32))
    v = bf16_bits(g.standard_normal((B, T, Hkv, d), dtype=np.float32))
    return AttnPrefillInputs(kind, window, B, T, Hq, Hkv, d, page_tokens, q, k, v, table, P)


def placement(counts: dict[int, int], seed: int = 0) -> np.ndarray:
    """A placement vector (int8, one mixer kind per layer) with the given count of each kind,
    positions shuffled by a seeded permutation ("randomly interleaved")."""
    layers = []
    for kind in (FA, SWA, KDA, GDN):
        layers += [kind] * int(counts.get(kind, 0))
    arr = np.array(layers, dtype=np.int8)
    return arr[rng(seed).permutation(len(arr))]


def layer_seed(layer: int, tensor_id: int) -> int:
    """Per-layer seed, 1000*layer + tensor_id."""
    return 1000 * layer + tensor_id
