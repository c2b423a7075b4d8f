"""Pins of the fp64 oracle against facts other than itself (CPU only).

Each check is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign, a
transposed state, the gate applied after instead of before the delta correction, an off-by-one
in a window or a page index) fails at least one of them:

* hand-worked two-token examples (tests/golden/delta_hand_examples.json);
* closed forms: beta=0 & g=1 is the identity; beta=0 is pure decay; the delta-rule write
  M_t^T k_t = (1-beta) M'^T k_t + beta v_t for unit k; orthonormal keys store and retrieve
  values; one token from a zero state gives o = beta (k.q) v;
* KDA with a uniform per-channel gate equals GDN (two differently oriented formulas);
* the chunked UT-transform form equals the token-by-token recurrence (any chunk size, ragged T);
* FA equals torch's scaled_dot_product_attention and a numpy softmax(QK^T/sqrt(d))V in fp64;
  SWA with w >= L equals FA; w = 1 and L = 1 return the new token's value;
* paged indexing: bijectivity of the FA map, injectivity of the SWA ring over every window,
  and a new token's ring slot never holding a position inside the window.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from hybrid_mixer_decoding_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _hand():
    with open(os.path.join(GOLD, "delta_hand_examples.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_hand_worked_example(oracle_mod, kind):
    O = oracle_mod
    ex = _hand()
    key = "gdn" if kind == I.GDN else "kda"
    inp = ex["inputs"]
    k = np.array(inp["k"])[None, :, None, :]
    v = np.array(inp["v"])[None, :, None, :]
    q = np.array(inp["q"])[None, :, None, :]
    beta = np.array(inp["beta"])[None, :, None]
    gate = np.array(ex[key]["gate"], dtype=np.float64)
    log_gate = np.log(gate)[None, :, None] if kind == I.GDN else np.log(gate)[None, :, None, :]
    s0 = np.zeros((1, 1, 2, 2))
    for fn in (lambda: O.delta_recurrent(kind, q, k, v, beta, log_gate, s0),
               lambda: O.delta_chunked(kind, q, k, v, beta, log_gate, s0, chunk=2),
               lambda: O.delta_chunked(kind, q, k, v, beta, log_gate, s0, chunk=1)):
        o, st = fn()
        np.testing.assert_allclose(o[0, :, 0, :], np.array(ex[key]["o"]), atol=1e-12)
        np.testing.assert_allclose(st[0, 0], np.array(ex[key]["final_state_M"]), atol=1e-12)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_identity_when_beta0_g1(oracle_mod, kind):
    """beta = 0 and g = 1 leave the state unchanged, and o = M0^T q."""
    O = oracle_mod
    d = I.delta_inputs(kind, 2, 7, 3, 8, 5, dtype="f32", seed=1, state0="randn")
    lg = np.zeros_like(d.log_gate)
    o, st = O.delta_recurrent(kind, d.q, d.k, d.v, np.zeros_like(d.beta), lg, d.state0)
    np.testing.assert_array_equal(st, d.state0.astype(np.float64))
    expect = np.einsum("bthi,bhij->bthj", d.q.astype(np.float64), d.state0.astype(np.float64))
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_pure_decay_when_beta0(oracle_mod, kind):
    """beta = 0: M_T = Diag(prod_t a_t) M0 (scalar product for GDN)."""
    O = oracle_mod
    d = I.delta_inputs(kind, 1, 9, 2, 6, 4, dtype="f32", seed=2, state0="randn")
    _, st = O.delta_recurrent(kind, d.q, d.k, d.v, np.zeros_like(d.beta), d.log_gate, d.state0)
    tot = np.exp(d.log_gate.astype(np.float64).sum(axis=1))  # [B,H] or [B,H,dk]
    if kind == I.GDN:
        expect = tot[:, :, None, None] * d.state0
    else:
        expect = tot[:, :, :, None] * d.state0
    np.testing.assert_allclose(st, expect, rtol=1e-12)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_delta_rule_write(oracle_mod, kind):
    """After each token, M_t^T k_t = (1-beta) (Diag(a_t) M_{t-1})^T k_t + beta v_t (unit k)."""
    O = oracle_mod
    d = I.delta_inputs(kind, 1, 6, 2, 8, 5, dtype="f32", seed=3, state0="randn")
    k = d.k.astype(np.float64)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)  # exactly unit in fp64
    st = d.state0.astype(np.float64)
    for t in range(d.T):
        sl = slice(t, t + 1)
        lg = d.log_gate[:, sl]
        _, st_new = O.delta_recurrent(kind, d.q[:, sl], k[:, sl], d.v[:, sl], d.beta[:, sl], lg,
                                      st)
        a = np.exp(lg[0, 0].astype(np.float64))  # [H] or [H,dk]
        for h in range(d.H):
            ah = a[h] if kind == I.GDN else a[h][:, None]
            Mp = ah * st[0, h]
            b = float(d.beta[0, t, h])
            lhs = st_new[0, h].T @ k[0, t, h]
            rhs = (1 - b) * (Mp.T @ k[0, t, h]) + b * d.v[0, t, h].astype(np.float64)
            np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
        st = st_new


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_orthonormal_keys_store_and_retrieve(oracle_mod, kind):
    """k_t = e_t, beta = 1, g = 1, M0 = 0: M_T = sum_t e_t v_t^T, so q = e_t returns v_t."""
    O = oracle_mod
    dk, dv, T = 6, 4, 6
    rs = np.random.default_rng(4)
    k = np.eye(dk)[None, :, None, :]
    v = rs.standard_normal((1, T, 1, dv))
    q = np.eye(dk)[None, :, None, :]  # token t queries e_t after writing it
    beta = np.ones((1, T, 1))
    lg = np.zeros((1, T, 1)) if kind == I.GDN else np.zeros((1, T, 1, dk))
    o, st = O.delta_recurrent(kind, q, k, v, beta, lg, np.zeros((1, 1, dk, dv)))
    np.testing.assert_allclose(st[0, 0], v[0, :, 0, :], atol=1e-14)
    np.testing.assert_allclose(o[0, :, 0, :], v[0, :, 0, :], atol=1e-14)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_single_token_from_zero(oracle_mod, kind):
    """One token from a zero state: o = scale * beta (k.q) v, state = beta k v^T."""
    O = oracle_mod
    d = I.delta_inputs(kind, 2, 1, 3, 8, 5, dtype="f32", seed=5)
    o, st = O.delta_recurrent(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0, scale=0.25)
    q, k, v, b = (x.astype(np.float64) for x in (d.q, d.k, d.v, d.beta))
    kq = np.einsum("bthi,bthi->bth", k, q)
    np.testing.assert_allclose(o, 0.25 * (b * kq)[..., None] * v, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(st, np.einsum("bth,bthi,bthj->bhij", b, k, v), rtol=1e-13)


def test_kda_uniform_gate_equals_gdn(oracle_mod):
    O = oracle_mod
    d = I.delta_inputs(I.GDN, 2, 20, 3, 8, 6, dtype="f32", seed=6, state0="randn")
    o_g, s_g = O.delta_recurrent(I.GDN, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)
    lg_k = np.repeat(d.log_gate[..., None], d.dk, axis=-1)
    o_k, s_k = O.delta_recurrent(I.KDA, d.q, d.k, d.v, d.beta, lg_k, d.state0)
    assert O.rel_err(o_k, o_g) < 1e-12 and O.rel_err(s_k, s_g) < 1e-12


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
@pytest.mark.parametrize("T,C", [(37, 1), (37, 2), (37, 16), (200, 64), (64, 64), (37, 37),
                                 (130, 64)])
def test_chunked_equals_recurrent(oracle_mod, kind, T, C):
    O = oracle_mod
    d = I.delta_inputs(kind, 1, T, 2, 16, 8, dtype="f32", seed=7 + T + C, state0="randn")
    o_r, s_r = O.delta_recurrent(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)
    o_c, s_c = O.delta_chunked(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0, chunk=C)
    assert O.rel_err(o_c, o_r) < 1e-12
    assert O.rel_err(s_c, s_r) < 1e-12


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_chunked_equals_recurrent_under_strong_decay(oracle_mod, kind):
    # log-gates down to -30 per token: over a chunk of 64 the cumulative gate reaches about
    # -1000, beyond fp64's e^{+-709}, so e^{G} and e^{-G} formed separately would underflow /
    # overflow; the chunked form must still equal the recurrence
    O = oracle_mod
    d = I.delta_inputs(kind, 1, 150, 2, 16, 8, dtype="f32", seed=31, gate_lo=-30.0,
                       state0="randn")
    o_r, s_r = O.delta_recurrent(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)
    o_c, s_c = O.delta_chunked(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0, chunk=64)
    assert np.isfinite(o_c).all() and np.isfinite(s_c).all()
    assert O.rel_err(o_c, o_r) < 1e-12
    assert O.rel_err(s_c, s_r) < 1e-12


def test_oracle_thread_count_invariance(oracle_mod):
    O = oracle_mod
    d = I.delta_inputs(I.KDA, 2, 30, 4, 8, 8, dtype="f32", seed=8, state0="randn")
    a = O.delta_recurrent(I.KDA, d.q, d.k, d.v, d.beta, d.log_gate, d.state0, n_threads=1)
    b = O.delta_recurrent(I.KDA, d.q, d.k, d.v, d.beta, d.log_gate, d.state0, n_threads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_oracle_rejects_bad_kind(oracle_mod):
    O = oracle_mod
    d = I.delta_inputs(I.GDN, 1, 2, 1, 4, 4, dtype="f32", seed=9)
    with pytest.raises(ValueError):
        O.delta_recurrent(I.FA, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)


# --------------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------------

def _logical_kv(a: I.AttnInputs, O):
    """Logical K/V [B][L][Hkv][d] for an identity page table (reshape, no oracle indexing)."""
    B, PT = a.B, a.page_tokens
    P = a.k_pool.shape[0]
    pps = P // B
    K = O.bf16_bits_to_f64(a.k_pool).reshape(B, pps, a.Hkv, PT, a.d).transpose(0, 1, 3, 2, 4)
    V = O.bf16_bits_to_f64(a.v_pool).reshape(B, pps, a.Hkv, PT, a.d).transpose(0, 1, 3, 2, 4)
    return K.reshape(B, pps * PT, a.Hkv, a.d), V.reshape(B, pps * PT, a.Hkv, a.d)


def _brute(a: I.AttnInputs, O, lo_fn):
    K, V = _logical_kv(a, O)
    q = O.bf16_bits_to_f64(a.q)
    nk, nv = O.bf16_bits_to_f64(a.new_k), O.bf16_bits_to_f64(a.new_v)
    out = np.zeros((a.B, a.Hq, a.d))
    grp = a.Hq // a.Hkv
    for b in range(a.B):
        L = int(a.seq_lens[b])
        Kb, Vb = K[b, :L].copy(), V[b, :L].copy()
        Kb[L - 1], Vb[L - 1] = nk[b], nv[b]
        lo = lo_fn(L)
        for h in range(a.Hq):
            s = Kb[lo:L, h // grp] @ q[b, h] / math.sqrt(a.d)
            p = np.exp(s - s.max())
            out[b, h] = (p / p.sum()) @ Vb[lo:L, h // grp]
    return out


def test_fa_matches_brute_force_and_torch_sdpa(oracle_mod):
    O = oracle_mod
    a = I.attn_inputs(I.FA, 3, 8, 2, 16, 150, page_tokens=16, seed=10, permute=False,
                      seq_lens=np.array([150, 1, 77]))
    o = O.attn_decode(I.FA, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                      a.seq_lens)
    ref = _brute(a, O, lambda L: 0)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    # torch's fp64 CPU attention on the same logical sequences
    K, V = _logical_kv(a, O)
    q = O.bf16_bits_to_f64(a.q)
    for b in range(a.B):
        L = int(a.seq_lens[b])
        Kb, Vb = K[b, :L].copy(), V[b, :L].copy()
        Kb[L - 1], Vb[L - 1] = O.bf16_bits_to_f64(a.new_k)[b], O.bf16_bits_to_f64(a.new_v)[b]
        Kt = torch.from_numpy(np.repeat(Kb.transpose(1, 0, 2), a.Hq // a.Hkv, axis=0))
        Vt = torch.from_numpy(np.repeat(Vb.transpose(1, 0, 2), a.Hq // a.Hkv, axis=0))
        qt = torch.from_numpy(q[b][:, None, :])
        st = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)
        np.testing.assert_allclose(o[b], st[:, 0, :].numpy(), rtol=1e-12, atol=1e-13)


def test_fa_page_permutation_invariance(oracle_mod):
    """Same logical data under a permuted page table gives the same result."""
    O = oracle_mod
    a = I.attn_inputs(I.FA, 2, 4, 2, 8, 100, page_tokens=16, seed=11, permute=False)
    o1 = O.attn_decode(I.FA, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                       a.seq_lens)
    perm = np.random.default_rng(0).permutation(a.k_pool.shape[0])
    inv = np.argsort(perm)
    kp, vp = a.k_pool[perm], a.v_pool[perm]  # physical page x holds old page perm[x]
    table = inv[a.page_table].astype(np.int32)
    o2 = O.attn_decode(I.FA, 0, a.q, a.new_k, a.new_v, kp, vp, table, a.seq_lens)
    np.testing.assert_array_equal(o1, o2)


def test_swa_wide_window_equals_fa(oracle_mod):
    O = oracle_mod
    a = I.attn_inputs(I.FA, 2, 4, 1, 8, 90, page_tokens=16, seed=12)
    o_fa = O.attn_decode(I.FA, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                         a.seq_lens)
    for w in (90, 91, 500):
        # a ring of R >= ceil(L/PT) pages never wraps, so the FA table is a valid ring table
        R = -(-w // 16)
        table = np.full((a.B, R), -1, np.int32)
        table[:, :a.page_table.shape[1]] = a.page_table
        o_swa = O.attn_decode(I.SWA, w, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, table,
                              a.seq_lens)
        np.testing.assert_array_equal(o_swa, o_fa)


def test_swa_matches_brute_force_window(oracle_mod):
    O = oracle_mod
    w = 40
    # contiguous layout long enough to hold every position, so the brute force can index it
    a = I.attn_inputs(I.FA, 2, 4, 2, 8, 130, page_tokens=16, seed=13, permute=False)
    ref = _brute(a, O, lambda L: max(0, L - w))
    # build the SWA ring (R = 3 pages of 16) holding positions of the last window
    R, PT = 3, 16
    P = a.B * R
    kp = np.zeros((P, a.Hkv, PT, a.d), np.uint16)
    vp = np.zeros_like(kp)
    table = np.arange(P, dtype=np.int32).reshape(a.B, R)[:, ::-1].copy()
    for b in range(a.B):
        L = int(a.seq_lens[b])
        for j in range(max(0, L - R * PT), L - 1):
            src_pg, src_off = b * (a.k_pool.shape[0] // a.B) + j // PT, j % PT
            r = j % (R * PT)
            kp[table[b, r // PT], :, r % PT] = a.k_pool[src_pg, :, src_off]
            vp[table[b, r // PT], :, r % PT] = a.v_pool[src_pg, :, src_off]
    o = O.attn_decode(I.SWA, w, a.q, a.new_k, a.new_v, kp, vp, table, a.seq_lens)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_degenerate_attention(oracle_mod):
    O = oracle_mod
    # L = 1 (FA) and w = 1 (SWA): output is the new token's value
    a = I.attn_inputs(I.FA, 2, 4, 2, 8, 50, page_tokens=16, seed=14,
                      seq_lens=np.array([1, 50]))
    o = O.attn_decode(I.FA, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                      a.seq_lens)
    nv = O.bf16_bits_to_f64(a.new_v)
    np.testing.assert_allclose(o[0], np.repeat(nv[0], 2, axis=0), rtol=1e-15)
    s = I.attn_inputs(I.SWA, 2, 4, 2, 8, 50, window=1, page_tokens=16, seed=15)
    o1 = O.attn_decode(I.SWA, 1, s.q, s.new_k, s.new_v, s.k_pool, s.v_pool, s.page_table,
                       s.seq_lens)
    np.testing.assert_allclose(o1, np.repeat(O.bf16_bits_to_f64(s.new_v), 2, axis=1),
                               rtol=1e-15)
    # all keys equal: output is the mean of the values
    e = I.attn_inputs(I.FA, 1, 2, 1, 8, 20, page_tokens=16, seed=16, permute=False)
    e.k_pool[:] = e.k_pool[0, 0, 0]
    e.new_k[:] = e.k_pool[0, 0, 0]
    o2 = O.attn_decode(I.FA, 0, e.q, e.new_k, e.new_v, e.k_pool, e.v_pool, e.page_table,
                       e.seq_lens)
    vals = np.concatenate([O.bf16_bits_to_f64(e.v_pool)[0, 0, :16],
                           O.bf16_bits_to_f64(e.v_pool)[1, 0, :3],
                           O.bf16_bits_to_f64(e.new_v)[0]], axis=0)
    np.testing.assert_allclose(o2[0, 0], vals.mean(axis=0), rtol=1e-13, atol=1e-15)


def test_attention_hand_example(oracle_mod):
    """q = (1,1), keys (0,0) and (1,1), values (1,0) and (0,2), d = 2:
    scores (0, sqrt 2), so o = ((1, 0) + e^sqrt2 (0, 2)) / (1 + e^sqrt2)."""
    O = oracle_mod
    one, two = I.bf16_bits(np.array([1.0], np.float32))[0], I.bf16_bits(np.array([2.0], np.float32))[0]
    kp = np.zeros((1, 1, 4, 2), np.uint16)
    vp = np.zeros((1, 1, 4, 2), np.uint16)
    vp[0, 0, 0, 0] = one
    q = np.array([[[one, one]]], np.uint16)
    nk = np.array([[[one, one]]], np.uint16)
    nv = np.array([[[0, two]]], np.uint16)
    o = O.attn_decode(I.FA, 0, q, nk, nv, kp, vp, np.array([[0]], np.int32),
                      np.array([2], np.int32))
    e = math.exp(math.sqrt(2.0))
    np.testing.assert_allclose(o[0, 0], [1 / (1 + e), 2 * e / (1 + e)], rtol=1e-15)


def test_fa_index_map_is_a_bijection(oracle_mod):
    O = oracle_mod
    PT, n = 16, 7
    row = np.random.default_rng(1).permutation(40)[:n].astype(np.int32)
    seen = set()
    for pos in range(n * PT):
        pg, off = O.kv_slot(I.FA, 0, PT, row, pos)
        assert pg in set(row.tolist()) and 0 <= off < PT
        seen.add((pg, off))
    assert len(seen) == n * PT  # every (page, offset) of the sequence used exactly once


@pytest.mark.parametrize("w", [1, 15, 16, 17, 40, 48])
def test_swa_ring_injective_over_every_window(oracle_mod, w):
    O = oracle_mod
    PT = 16
    R = -(-w // PT)
    row = np.random.default_rng(w).permutation(50)[:R].astype(np.int32)
    slots = [O.kv_slot(I.SWA, w, PT, row, p) for p in range(300)]
    for L in range(1, 300):
        lo = max(0, L - w)
        win = slots[lo:L]
        assert len(set(win)) == len(win)  # the window's positions never share a slot
        if L >= 2:
            # the new token (position L-1) overwrites a slot whose previous occupant, if any,
            # is older than the window
            prev = [p for p in range(L - 1) if slots[p] == slots[L - 1]]
            assert all(p < lo for p in prev)


# ---- attention prefill from an empty cache (token t attends [lo_t, t]) ------------------------

def _prefill_qkv(B, T, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, Hq, d)), rng.standard_normal((B, T, Hkv, d)),
            rng.standard_normal((B, T, Hkv, d)))


def _masked_softmax_attention(q, k, v, window):
    """Brute force with an explicit T x T mask: allowed[t, j] = j <= t and t - j < window."""
    B, T, Hq, d = q.shape
    grp = Hq // k.shape[2]
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    allowed = (j <= t) & (t - j < window)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            s = (q[b, :, h] @ k[b, :, h // grp].T) / math.sqrt(d)
            s = np.where(allowed, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            out[b, :, h] = (p / p.sum(axis=1, keepdims=True)) @ v[b, :, h // grp]
    return out


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 5), (I.SWA, 16)])
def test_prefill_attention_matches_masked_softmax_and_sdpa(oracle_mod, kind, window):
    O = oracle_mod
    q, k, v = _prefill_qkv(2, 37, 4, 2, 8, seed=30 + window)
    o = O.attn_prefill(kind, window, q, k, v)
    ref = _masked_softmax_attention(q, k, v, window if kind == I.SWA else 10 ** 9)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    if kind == I.FA:  # torch's fp64 causal attention on the same data
        qt = torch.from_numpy(q.transpose(0, 2, 1, 3))
        kt = torch.from_numpy(np.repeat(k, 2, axis=2).transpose(0, 2, 1, 3))
        vt = torch.from_numpy(np.repeat(v, 2, axis=2).transpose(0, 2, 1, 3))
        st = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        np.testing.assert_allclose(o, st.numpy().transpose(0, 2, 1, 3), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 7)])
def test_prefill_rows_equal_decode_steps(oracle_mod, kind, window):
    """Row t of the prefill is the decode step with L = t + 1 over a paged cache holding tokens
    0..t-1 (the decode oracle is pinned on its own above)."""
    O = oracle_mod
    B, T, Hq, Hkv, d, PT = 2, 21, 4, 2, 8, 4
    bits = lambda x: I.bf16_bits(x)
    q, k, v = _prefill_qkv(B, T, Hq, Hkv, d, seed=41)
    qb, kb, vb = bits(q), bits(k), bits(v)
    o = O.attn_prefill(kind, window, O.bf16_bits_to_f64(qb), O.bf16_bits_to_f64(kb),
                       O.bf16_bits_to_f64(vb))
    n_pg = -(-T // PT) if kind == I.FA else -(-window // PT)  # FA pages / SWA ring pages
    table = np.arange(B * n_pg, dtype=np.int32).reshape(B, n_pg)
    for t in range(T):
        # the cache as t decode steps leave it: positions 0..t-1 written in order at their
        # slots (for SWA the ring keeps the latest position of each slot)
        kp = np.zeros((B * n_pg, Hkv, PT, d), np.uint16)
        vp = np.zeros_like(kp)
        for b in range(B):
            for p in range(t):
                pg, off = O.kv_slot(kind, window, PT, table[b], p)
                kp[pg, :, off], vp[pg, :, off] = kb[b, p], vb[b, p]
        dec = O.attn_decode(kind, window, qb[:, t], kb[:, t], vb[:, t], kp, vp, table,
                            np.full(B, t + 1, np.int32))
        np.testing.assert_allclose(o[:, t], dec, rtol=1e-12, atol=1e-13)


def test_prefill_attention_closed_forms(oracle_mod):
    O = oracle_mod
    q, k, v = _prefill_qkv(2, 12, 4, 1, 8, seed=50)
    # the first token sees only itself; a window of 1 gives every token its own value
    o = O.attn_prefill(I.FA, 0, q, k, v)
    np.testing.assert_array_equal(o[:, 0], np.repeat(v[:, 0], 4, axis=1))
    o1 = O.attn_prefill(I.SWA, 1, q, k, v)
    np.testing.assert_array_equal(o1, np.repeat(v, 4, axis=2))
    # a window covering the whole prompt is FA, bit for bit
    np.testing.assert_array_equal(O.attn_prefill(I.SWA, 12, q, k, v), o)
    np.testing.assert_array_equal(O.attn_prefill(I.SWA, 500, q, k, v), o)
    # equal keys: uniform weights, so each row is the mean of the values in its window
    ke = np.repeat(k[:, :1], 12, axis=1)
    w = 3
    oe = O.attn_prefill(I.SWA, w, q, ke, v)
    for t in range(12):
        lo = max(0, t + 1 - w)
        np.testing.assert_allclose(oe[:, t], np.repeat(v[:, lo:t + 1].mean(axis=1), 4, axis=1),
                                   rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------------------------
# verification pass (speculative decoding): n_q new tokens, each a decode step
# --------------------------------------------------------------------------------------------

def _verify_brute(a: I.AttnVerifyInputs, O):
    """Brute force over the logical sequence: positions below L - n_q are gathered from the
    pools with the slot formula written out here (ring index p mod (R * PT) for SWA), the
    last n_q are the new tokens; row i attends [lo, L - n_q + i]."""
    PT, R = a.page_tokens, a.ring_pages
    q = O.bf16_bits_to_f64(a.q)
    nk, nv = O.bf16_bits_to_f64(a.new_k), O.bf16_bits_to_f64(a.new_v)
    kp, vp = O.bf16_bits_to_f64(a.k_pool), O.bf16_bits_to_f64(a.v_pool)
    grp = a.Hq // a.Hkv
    out = np.zeros(q.shape)
    for b in range(a.B):
        L = int(a.seq_lens[b])
        first = L - a.n_q
        K = np.zeros((L, a.Hkv, a.d))
        V = np.zeros_like(K)
        for p in range(first):
            r = p % (R * PT) if a.kind == I.SWA else p
            pg = a.page_table[b, r // PT]
            K[p], V[p] = kp[pg, :, r % PT], vp[pg, :, r % PT]
        K[first:], V[first:] = nk[b], nv[b]
        for i in range(a.n_q):
            P_ = first + i
            lo = max(0, P_ + 1 - a.window) if a.kind == I.SWA else 0
            for h in range(a.Hq):
                s = K[lo:P_ + 1, h // grp] @ q[b, i, h] / math.sqrt(a.d)
                w = np.exp(s - s.max())
                out[b, i, h] = (w / w.sum()) @ V[lo:P_ + 1, h // grp]
    return out


@pytest.mark.parametrize("kind,window,n_q,ring_extra", [
    (I.FA, 0, 1, 0), (I.FA, 0, 3, 0), (I.FA, 0, 4, 0),
    (I.SWA, 9, 1, 0), (I.SWA, 9, 4, 0), (I.SWA, 8, 3, 0), (I.SWA, 5, 2, 2), (I.SWA, 1, 4, 0)])
def test_verify_matches_brute_force(oracle_mod, kind, window, n_q, ring_extra):
    O = oracle_mod
    PT = 4
    ring = -(-(window + n_q - 1) // PT) + ring_extra if kind == I.SWA else 0
    a = I.verify_inputs(kind, 3, n_q, 4, 2, 8, 30, window=window, ring_pages=ring,
                        page_tokens=PT, seed=60 + n_q, seq_lens=np.array([30, n_q, 17]))
    o = O.attn_verify(kind, window, a.ring_pages, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool,
                      a.page_table, a.seq_lens)
    np.testing.assert_allclose(o, _verify_brute(a, O), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 9)])
def test_verify_single_token_is_the_decode_step(oracle_mod, kind, window):
    O = oracle_mod
    PT = 4
    a = I.verify_inputs(kind, 3, 1, 4, 2, 8, 30, window=window,
                        ring_pages=-(-window // PT) if kind == I.SWA else 0, page_tokens=PT,
                        seed=70, seq_lens=np.array([30, 1, 13]))
    o = O.attn_verify(kind, window, a.ring_pages, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool,
                      a.page_table, a.seq_lens)
    dec = O.attn_decode(kind, window, a.q[:, 0], a.new_k[:, 0], a.new_v[:, 0], a.k_pool,
                        a.v_pool, a.page_table, a.seq_lens)
    np.testing.assert_allclose(o[:, 0], dec, rtol=1e-12, atol=1e-13)


def test_verify_rows_equal_successive_decode_steps(oracle_mod):
    """FA: row i of a verify pass is the decode step of token i after tokens 0..i-1 have been
    appended at their slots (the decode oracle is pinned on its own)."""
    O = oracle_mod
    PT, n_q = 4, 4
    a = I.verify_inputs(I.FA, 2, n_q, 4, 2, 8, 23, page_tokens=PT, seed=71,
                        seq_lens=np.array([23, 9]))
    o = O.attn_verify(I.FA, 0, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                      a.seq_lens)
    kp, vp = a.k_pool.copy(), a.v_pool.copy()
    for i in range(n_q):
        L_i = a.seq_lens - n_q + i + 1
        dec = O.attn_decode(I.FA, 0, a.q[:, i], a.new_k[:, i], a.new_v[:, i], kp, vp,
                            a.page_table, L_i)
        np.testing.assert_allclose(o[:, i], dec, rtol=1e-12, atol=1e-13)
        for b in range(a.B):  # append token i for the next step
            pg, off = O.kv_slot(I.FA, 0, PT, a.page_table[b], int(L_i[b]) - 1)
            kp[pg, :, off], vp[pg, :, off] = a.new_k[b, i], a.new_v[b, i]


def test_verify_from_empty_cache_is_prefill(oracle_mod):
    """FA with L = n_q (nothing cached): the verify pass is the prefill of those n_q tokens."""
    O = oracle_mod
    n_q = 5
    a = I.verify_inputs(I.FA, 2, n_q, 4, 2, 8, n_q, page_tokens=4, seed=72)
    o = O.attn_verify(I.FA, 0, 0, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool, a.page_table,
                      a.seq_lens)
    pre = O.attn_prefill(I.FA, 0, O.bf16_bits_to_f64(a.q), O.bf16_bits_to_f64(a.new_k),
                         O.bf16_bits_to_f64(a.new_v))
    np.testing.assert_allclose(o, pre, rtol=1e-12, atol=1e-13)


def test_ring_slot_formula_cases(oracle_mod):
    """kv_slot_ring: FA ignores the ring; SWA wraps at ring_pages * PT; the default ring of
    ceil(w / PT) pages agrees with kv_slot."""
    O = oracle_mod
    row = np.array([7, 3, 9, 1, 4], np.int32)
    assert O.kv_slot_ring(I.FA, 2, 4, row, 13) == (1, 1)   # page 13 // 4 = 3
    assert O.kv_slot_ring(I.SWA, 2, 4, row, 13) == (3, 1)   # 13 mod 8 = 5: page 1, offset 1
    assert O.kv_slot_ring(I.SWA, 3, 4, row, 13) == (7, 1)   # 13 mod 12 = 1
    assert O.kv_slot_ring(I.SWA, 5, 4, row, 19) == (4, 3)
    for w in (1, 4, 5, 9):
        for p in range(40):
            assert O.kv_slot_ring(I.SWA, -(-w // 4), 4, row, p) == O.kv_slot(I.SWA, w, 4, row, p)


# --------------------------------------------------------------------------------------------
# input activations of the delta-rule mixers (raw projections -> q, k, beta, log-gates)
# --------------------------------------------------------------------------------------------

@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_activations_closed_forms(oracle_mod, kind):
    O = oracle_mod
    rng = np.random.default_rng(80)
    N, H, dk = 5, 3, 8
    qr, kr = rng.standard_normal((N, H, dk)) * 3, rng.standard_normal((N, H, dk)) * 0.1
    gshape = (N, H) if kind == I.GDN else (N, H, dk)
    bshape = (H,) if kind == I.GDN else (H, dk)
    q, k, beta, lg = O.delta_activations(kind, qr, kr, np.zeros((N, H)), np.zeros(gshape),
                                         np.zeros(H), np.zeros(bshape), eps=0.0)
    # eps = 0: unit L2 norm, direction kept
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(k, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(q * np.linalg.norm(qr, axis=-1, keepdims=True), qr, rtol=1e-13)
    # sigmoid(0) = 1/2; A_log = 0, logit + bias = 0: log gate = -log 2
    np.testing.assert_array_equal(beta, 0.5)
    np.testing.assert_allclose(lg, -math.log(2.0), rtol=1e-15)
    # a large logit: softplus(x) -> x, so log gate -> -exp(A_log) * (x + b)
    A = np.log(np.arange(1, H + 1, dtype=np.float64))
    big = np.full(gshape, 40.0)
    bias = np.full(bshape, 2.0)
    _, _, _, lg2 = O.delta_activations(kind, qr, kr, np.zeros((N, H)), big, A, bias)
    expect = -np.exp(A)[:, None] * 42.0 if kind == I.KDA else -np.exp(A)[None, :] * 42.0
    np.testing.assert_allclose(lg2, np.broadcast_to(expect, gshape), rtol=1e-14)
    # eps > 0 shrinks the norm: |q| = sqrt(s / (s + eps))
    q3, _, b3, _ = O.delta_activations(kind, qr, kr, np.full((N, H), 2.0), np.zeros(gshape),
                                       np.zeros(H), np.zeros(bshape), eps=0.5)
    s2 = (qr ** 2).sum(-1)
    np.testing.assert_allclose(np.linalg.norm(q3, axis=-1), np.sqrt(s2 / (s2 + 0.5)), rtol=1e-13)
    np.testing.assert_allclose(b3, 1.0 / (1.0 + math.exp(-2.0)), rtol=1e-15)


def test_activations_gate_is_per_head_and_per_channel(oracle_mod):
    """GDN: one gate per (token, head) with the head's A_log and dt_bias; KDA: one per channel
    with the channel's dt_bias: permuting heads / channels of every input permutes the gate."""
    O = oracle_mod
    rng = np.random.default_rng(81)
    N, H, dk = 4, 3, 6
    qr, kr = rng.standard_normal((N, H, dk)), rng.standard_normal((N, H, dk))
    bl = rng.standard_normal((N, H))
    A = rng.standard_normal(H) * 0.3
    for kind, gl, db in ((I.GDN, rng.standard_normal((N, H)), rng.standard_normal(H)),
                         (I.KDA, rng.standard_normal((N, H, dk)), rng.standard_normal((H, dk)))):
        _, _, _, lg = O.delta_activations(kind, qr, kr, bl, gl, A, db)
        perm = np.array([2, 0, 1])
        _, _, _, lgp = O.delta_activations(kind, qr[:, perm], kr[:, perm], bl[:, perm],
                                           gl[:, perm], A[perm], db[perm])
        np.testing.assert_allclose(lgp, lg[:, perm], rtol=1e-15)
        # softplus > 0 and exp(A_log) > 0: every log gate is negative
        assert (lg < 0).all()
