"""GPU parity of attn_prefill (FA and SWA prefill from an empty paged cache) against the fp64
oracle, through the C ABI: outputs within 2e-2 (bf16), the cache slots bit for bit, and a
decode step after the prefill equal to the prefill over one more token.
"""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu
SENTINEL = 0x3F80  # bf16 1.0: fills the pools so that untouched slots are recognisable


def _bits_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


def _bits_host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_prefill(a: I.AttnPrefillInputs):
    kp = torch.full((a.n_pages, a.Hkv, a.page_tokens, a.d), SENTINEL, dtype=torch.int16,
                    device="cuda").view(torch.bfloat16)
    vp = kp.clone()
    o = torch.empty(a.B, a.T, a.Hq, a.d, dtype=torch.bfloat16, device="cuda")
    table = torch.from_numpy(a.page_table).cuda()
    hmd.attn_prefill(a.kind, a.window, _bits_dev(a.q), _bits_dev(a.k), _bits_dev(a.v), kp, vp,
                     table, o)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    return o, kp, vp


def expected_pools(O, a: I.AttnPrefillInputs):
    """The pools as T decode steps would leave them: position t at its slot (FA: every t; SWA:
    the ring keeps the latest position of each slot); every other slot keeps the sentinel."""
    kp = np.full((a.n_pages, a.Hkv, a.page_tokens, a.d), SENTINEL, np.uint16)
    vp = kp.copy()
    for b in range(a.B):
        for t in range(a.T):
            pg, off = O.kv_slot(a.kind, a.window, a.page_tokens, a.page_table[b], t)
            kp[pg, :, off] = a.k[b, t]
            vp[pg, :, off] = a.v[b, t]
    return kp, vp


CASES = [  # kind, window, B, T, Hq, Hkv, d
    (I.FA, 0, 2, 1, 8, 2, 128),
    (I.FA, 0, 2, 1, 8, 2, 64),
    (I.FA, 0, 1, 300, 16, 1, 64),     # G = 16 at d = 64
    (I.FA, 0, 2, 63, 8, 2, 128),
    (I.FA, 0, 2, 200, 8, 2, 128),
    (I.FA, 0, 1, 130, 8, 8, 128),     # G = 1: 128 tokens per block
    (I.FA, 0, 2, 70, 16, 1, 128),     # G = 16: 8 tokens per block
    (I.FA, 0, 2, 150, 8, 2, 64),
    (I.SWA, 64, 2, 200, 8, 2, 128),
    (I.SWA, 100, 2, 300, 8, 2, 128),  # ring of 2 pages wraps
    (I.SWA, 1, 2, 90, 8, 2, 128),
    (I.SWA, 500, 1, 130, 8, 4, 64),   # window longer than the prompt
]


@pytest.mark.parametrize("kind,window,B,T,Hq,Hkv,d", CASES)
def test_prefill_matches_oracle_and_writes_the_cache(oracle_mod, kind, window, B, T, Hq, Hkv, d):
    O = oracle_mod
    a = I.attn_prefill_inputs(kind, B, T, Hq, Hkv, d, window=window, seed=T + Hq + d)
    o, kp, vp = run_prefill(a)
    ref = O.attn_prefill(kind, window, O.bf16_bits_to_f64(a.q), O.bf16_bits_to_f64(a.k),
                         O.bf16_bits_to_f64(a.v))
    assert O.rel_err(o.float().cpu().numpy(), ref) < 2e-2
    ek, ev = expected_pools(O, a)
    np.testing.assert_array_equal(_bits_host(kp), ek)
    np.testing.assert_array_equal(_bits_host(vp), ev)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 100)])
def test_decode_after_prefill_equals_longer_prefill(oracle_mod, kind, window):
    """Prefill T tokens, then one attn_decode step with the (T+1)-th token: its output equals
    row T of the oracle's prefill over T + 1 tokens."""
    O = oracle_mod
    B, T, Hq, Hkv, d = 2, 250, 8, 2, 128
    full = I.attn_prefill_inputs(kind, B, T + 1, Hq, Hkv, d, window=window, seed=77)
    head = I.AttnPrefillInputs(kind, window, B, T, Hq, Hkv, d, 64, full.q[:, :T], full.k[:, :T],
                               full.v[:, :T], full.page_table, full.n_pages)
    _, kp, vp = run_prefill(head)
    o1 = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), T + 1, dtype=torch.int32, device="cuda")
    ws = torch.empty(hmd.attn_decode_workspace_size(kind, window, B, Hq, Hkv, d, 64, T + 1),
                     dtype=torch.uint8, device="cuda")
    hmd.attn_decode(kind, window, _bits_dev(full.q[:, T]), _bits_dev(full.k[:, T]),
                    _bits_dev(full.v[:, T]), kp, vp, torch.from_numpy(full.page_table).cuda(),
                    lens, T + 1, o1, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    ref = O.attn_prefill(kind, window, O.bf16_bits_to_f64(full.q), O.bf16_bits_to_f64(full.k),
                         O.bf16_bits_to_f64(full.v))[:, T]
    assert O.rel_err(o1.float().cpu().numpy(), ref) < 2e-2


def host_cache_before(O, a: I.AttnPrefillInputs, t: int):
    """Pools and table holding positions 0..t-1 as t decode steps leave them, built on the host
    from the prompt (FA: every position; SWA: the ring's latest position per slot)."""
    R = -(-a.window // a.page_tokens) if a.kind == I.SWA else -(-max(t, 1) // a.page_tokens)
    table = np.arange(a.B * R, dtype=np.int32).reshape(a.B, R)
    kp = np.zeros((a.B * R, a.Hkv, a.page_tokens, a.d), np.uint16)
    vp = np.zeros_like(kp)
    first = max(0, t - R * a.page_tokens)  # older positions are overwritten in a ring
    for b in range(a.B):
        for p in range(first, t):
            pg, off = O.kv_slot(a.kind, a.window, a.page_tokens, table[b], p)
            kp[pg, :, off], vp[pg, :, off] = a.k[b, p], a.v[b, p]
    return kp, vp, table


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 4096)])
def test_full_size_sampled_rows(oracle_mod, kind, window):
    """The benchmark's prefill shape (B=2, T=8192, Hq=32, Hkv=8, d=128, SWA w=4096), checked on
    sampled token positions (each against the oracle's decode step with L = t + 1 over a cache
    built on the host from the prompt, not from the GPU's pools) and on every pool slot."""
    O = oracle_mod
    B, T, Hq, Hkv, d = 2, 8192, 32, 8, 128
    a = I.attn_prefill_inputs(kind, B, T, Hq, Hkv, d, window=window, seed=5)
    o, kp, vp = run_prefill(a)
    got = o.float().cpu().numpy()
    for t in (0, 1, 63, 64, 4095, 4096, 5000, T - 1):
        hk, hv, table = host_cache_before(O, a, t)
        ref = O.attn_decode(kind, window, a.q[:, t], a.k[:, t], a.v[:, t], hk, hv, table,
                            np.full(B, t + 1, np.int32))
        assert O.rel_err(got[:, t], ref) < 2e-2, t
    ek, ev = expected_pools(O, a)
    np.testing.assert_array_equal(_bits_host(kp), ek)
    np.testing.assert_array_equal(_bits_host(vp), ev)


# ---- prefill after a cached prefix (chunked prefill) ----------------------------------------

def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_prefill_ext(a: I.AttnVerifyInputs, T):
    """attn_prefill_ext of the T tokens in a (q, new_k, new_v as the prompt) after prefixes of
    seq_lens - T positions, on device copies of a's pools."""
    kp, vp = _bits_dev(a.k_pool), _bits_dev(a.v_pool)
    o = torch.empty(a.B, T, a.Hq, a.d, dtype=torch.bfloat16, device="cuda")
    pre = (a.seq_lens - T).astype(np.int32)
    hmd.attn_prefill_ext(a.kind, a.window, _bits_dev(a.q), _bits_dev(a.new_k), _bits_dev(a.new_v),
                         torch.from_numpy(pre).cuda(), int(pre.max()), kp, vp,
                         torch.from_numpy(a.page_table).cuda(), o)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    return o, kp, vp


def expected_pools_after_prefix(O, a: I.AttnVerifyInputs, T):
    """The pools after the prompt's K/V are written: FA every position L0 + t, SWA the positions
    its ring keeps (the last R*64 of the prompt); other slots unchanged."""
    ek, ev = a.k_pool.copy(), a.v_pool.copy()
    R64 = a.ring_pages * a.page_tokens
    for b in range(a.B):
        L0 = int(a.seq_lens[b]) - T
        for t in range(T):
            if a.kind == I.SWA and t < T - R64:
                continue
            pg, off = O.kv_slot_ring(a.kind, a.ring_pages, a.page_tokens, a.page_table[b], L0 + t)
            ek[pg, :, off], ev[pg, :, off] = a.new_k[b, t], a.new_v[b, t]
    return ek, ev


PREFIX_CASES = [  # kind, window, T, Hq, Hkv, prefix lengths (multiples of 64), d
    (I.FA, 0, 200, 8, 2, [0, 64, 640], 128),
    (I.FA, 0, 1, 8, 2, [128, 0, 64], 128),
    (I.FA, 0, 130, 8, 8, [64, 192], 128),      # G = 1
    (I.FA, 0, 70, 16, 1, [256, 64], 128),      # G = 16
    (I.SWA, 100, 150, 8, 2, [0, 64, 640], 128),  # ring of 2 pages, prompt longer than the ring
    (I.SWA, 64, 40, 8, 2, [128, 64], 128),
    (I.SWA, 300, 500, 32, 8, [320, 1024], 128),
    (I.FA, 0, 200, 8, 2, [0, 64, 640], 64),
    (I.SWA, 100, 150, 8, 4, [0, 128, 640], 64),
]


@pytest.mark.parametrize("kind,window,T,Hq,Hkv,prefixes,d", PREFIX_CASES)
def test_prefill_after_prefix_matches_oracle(oracle_mod, kind, window, T, Hq, Hkv, prefixes, d):
    O = oracle_mod
    pre = np.array(prefixes, np.int32)
    lens = pre + T
    ring = -(-window // 64) if kind == I.SWA else 0
    a = I.verify_inputs(kind, len(pre), T, Hq, Hkv, d, int(lens.max()), window=window,
                        ring_pages=ring, seed=int(lens.sum()) + T, seq_lens=lens)
    o, kp, vp = run_prefill_ext(a, T)
    ref = O.attn_verify(kind, window, a.ring_pages, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool,
                        a.page_table, a.seq_lens)
    assert O.rel_err(o.float().cpu().numpy(), ref) < 2e-2
    ek, ev = expected_pools_after_prefix(O, a, T)
    np.testing.assert_array_equal(_bits(kp), ek)
    np.testing.assert_array_equal(_bits(vp), ev)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 200)])
def test_two_chunks_equal_one_prefill(oracle_mod, kind, window):
    """A prompt prefilled as 256 tokens, then 190 more after that cached prefix, gives the second
    chunk the rows of the oracle's prefill over all 446 tokens."""
    O = oracle_mod
    B, T1, T2, Hq, Hkv, d = 2, 256, 190, 8, 2, 128
    full = I.attn_prefill_inputs(kind, B, T1 + T2, Hq, Hkv, d, window=window, seed=91)
    head = I.AttnPrefillInputs(kind, window, B, T1, Hq, Hkv, d, 64, full.q[:, :T1],
                               full.k[:, :T1], full.v[:, :T1], full.page_table, full.n_pages)
    _, kp, vp = run_prefill(head)
    o2 = torch.empty(B, T2, Hq, d, dtype=torch.bfloat16, device="cuda")
    hmd.attn_prefill_ext(kind, window, _bits_dev(full.q[:, T1:]), _bits_dev(full.k[:, T1:]),
                         _bits_dev(full.v[:, T1:]), torch.full((B,), T1, dtype=torch.int32,
                                                               device="cuda"),
                         T1, kp, vp, torch.from_numpy(full.page_table).cuda(), o2)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    ref = O.attn_prefill(kind, window, O.bf16_bits_to_f64(full.q), O.bf16_bits_to_f64(full.k),
                         O.bf16_bits_to_f64(full.v))
    assert O.rel_err(o2.float().cpu().numpy(), ref[:, T1:]) < 2e-2
    # and the cache then holds what one prefill of all 446 tokens leaves
    ek, ev = expected_pools(O, full)
    np.testing.assert_array_equal(_bits_host(kp), ek)
    np.testing.assert_array_equal(_bits_host(vp), ev)
