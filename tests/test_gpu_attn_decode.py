"""GPU parity of attn_decode (FA, SWA over the paged bf16 KV cache) against the fp64 oracle,
through the C ABI. Outputs are bf16 (tolerance 2e-2 normwise); the KV append is checked
bit-exact against the oracle's index map, and every other pool byte must be unchanged.
"""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _bits_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _i32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def run_gpu(a: I.AttnInputs, max_seq_len=None):
    kp, vp = _bits_dev(a.k_pool), _bits_dev(a.v_pool)
    q, nk, nv = _bits_dev(a.q), _bits_dev(a.new_k), _bits_dev(a.new_v)
    table, lens = _i32(a.page_table), _i32(a.seq_lens)
    msl = int(max_seq_len or a.seq_lens.max())
    ws = torch.empty(hmd.attn_decode_workspace_size(a.kind, a.window, a.B, a.Hq, a.Hkv, a.d,
                                                    a.page_tokens, msl),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty(a.B, a.Hq, a.d, device="cuda", dtype=torch.bfloat16)
    hmd.attn_decode(a.kind, a.window, q, nk, nv, kp, vp, table, lens, msl, o, ws)
    torch.cuda.synchronize()
    return (o.float().cpu().numpy(), kp.view(torch.int16).cpu().numpy().view(np.uint16),
            vp.view(torch.int16).cpu().numpy().view(np.uint16))


def check(a: I.AttnInputs, O, tol=2e-2):
    o, kp, vp = run_gpu(a)
    ref = O.attn_decode(a.kind, a.window, a.q, a.new_k, a.new_v, a.k_pool, a.v_pool,
                        a.page_table, a.seq_lens)
    err = O.rel_err(o, ref)
    assert err < tol, err
    # the append: position L-1 of every (sequence, kv-head) holds the new token, bit-exact
    exp_k, exp_v = a.k_pool.copy(), a.v_pool.copy()
    for b in range(a.B):
        pg, off = O.kv_slot(a.kind, a.window, a.page_tokens, a.page_table[b],
                            int(a.seq_lens[b]) - 1)
        exp_k[pg, :, off] = a.new_k[b]
        exp_v[pg, :, off] = a.new_v[b]
    np.testing.assert_array_equal(kp, exp_k)
    np.testing.assert_array_equal(vp, exp_v)
    return o


@pytest.mark.parametrize("kind", [I.FA, I.SWA])
@pytest.mark.parametrize("d,Hq,Hkv", [(128, 8, 2), (64, 4, 4), (128, 16, 1), (64, 32, 2)])
def test_small_ragged(oracle_mod, kind, d, Hq, Hkv):
    lens = np.array([1, 63, 64, 65, 150, 257, 300], np.int32)
    w = 100 if kind == I.SWA else 0
    a = I.attn_inputs(kind, len(lens), Hq, Hkv, d, int(lens.max()), window=w, seed=d + Hq,
                      seq_lens=lens, extra_pages=3)
    check(a, oracle_mod)


@pytest.mark.parametrize("w", [1, 63, 64, 65, 128, 1000])
def test_swa_windows_and_ring_wrap(oracle_mod, w):
    lens = np.array([1, 2, 64, 65, 127, 128, 129, 500, 700], np.int32)
    a = I.attn_inputs(I.SWA, len(lens), 4, 1, 128, int(lens.max()), window=w, seed=w,
                      seq_lens=lens)
    check(a, oracle_mod)


def test_swa_wide_window_equals_fa_on_gpu():
    lens = np.array([5, 64, 200], np.int32)
    a = I.attn_inputs(I.FA, 3, 8, 2, 128, 200, seed=3, seq_lens=lens)
    o_fa, _, _ = run_gpu(a)
    R = -(-1000 // 64)
    table = np.full((3, R), -1, np.int32)
    table[:, :a.page_table.shape[1]] = a.page_table
    s = I.AttnInputs(I.SWA, 1000, a.B, a.Hq, a.Hkv, a.d, 64, a.k_pool, a.v_pool, table,
                     a.seq_lens, a.q, a.new_k, a.new_v)
    o_swa, _, _ = run_gpu(s)
    np.testing.assert_array_equal(o_fa, o_swa)


def test_page_permutation_invariance_bitwise():
    a = I.attn_inputs(I.FA, 4, 8, 2, 128, 400, seed=5, permute=False,
                      seq_lens=np.array([400, 17, 128, 333], np.int32))
    o1, _, _ = run_gpu(a)
    perm = np.random.default_rng(1).permutation(a.k_pool.shape[0])
    inv = np.argsort(perm)
    b = I.AttnInputs(I.FA, 0, a.B, a.Hq, a.Hkv, a.d, 64, a.k_pool[perm].copy(),
                     a.v_pool[perm].copy(), inv[a.page_table].astype(np.int32), a.seq_lens, a.q,
                     a.new_k, a.new_v)
    o2, _, _ = run_gpu(b)
    np.testing.assert_array_equal(o1, o2)


def test_longer_max_seq_len_bound_changes_nothing():
    a = I.attn_inputs(I.FA, 3, 8, 2, 128, 300, seed=6)
    o1, _, _ = run_gpu(a)
    # a larger bound needs a table wide enough for it (unused entries -1) and changes the plan
    wide = np.full((a.B, -(-5000 // 64)), -1, np.int32)
    wide[:, :a.page_table.shape[1]] = a.page_table
    a.page_table = wide
    o2, _, _ = run_gpu(a, max_seq_len=5000)
    assert np.max(np.abs(o1 - o2)) <= 2e-2 * np.max(np.abs(o1))


def test_bad_page_id_sets_device_error():
    hmd.hmd_device_errors(clear=True)
    a = I.attn_inputs(I.FA, 2, 4, 1, 128, 130, seed=7)
    a.page_table[1, 1] = 10_000  # beyond the pool
    run_gpu(a)
    assert hmd.hmd_device_errors(clear=True) & hmd.DEVERR_PAGE


def test_deterministic():
    a = I.attn_inputs(I.SWA, 5, 8, 2, 128, 900, window=300, seed=8)
    o1, _, _ = run_gpu(a)
    o2, _, _ = run_gpu(a)
    np.testing.assert_array_equal(o1, o2)


@pytest.mark.parametrize("kind", [I.FA, I.SWA])
def test_config3_full_size(oracle_mod, kind):
    """B=32, Hq=32, Hkv=8, d=128, context 8192 (including the new token), SWA window 4096,
    pages of 64 tokens under a random page permutation: every output checked."""
    w = 4096 if kind == I.SWA else 0
    a = I.attn_inputs(kind, 32, 32, 8, 128, 8192, window=w, seed=2)
    check(a, oracle_mod)


@pytest.mark.parametrize("kind", [I.FA, I.SWA])
def test_long_context_128k(oracle_mod, kind):
    """The context sweep's longest context: B=2, Hq=32, Hkv=8, d=128, one sequence at 131072
    tokens and one ragged at 100033 (the split plan's longest key ranges, and a last page that
    holds only the new token), SWA window 4096, random page permutation: every output and the
    append checked."""
    w = 4096 if kind == I.SWA else 0
    a = I.attn_inputs(kind, 2, 32, 8, 128, 131072, window=w, seed=5,
                      seq_lens=np.array([131072, 100033], np.int32))
    check(a, oracle_mod)
