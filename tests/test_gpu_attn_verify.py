"""GPU parity of attn_verify (the verification pass of speculative decoding: n_q new tokens per
sequence in one pass) against the fp64 oracle, through the C ABI. Outputs are bf16 (2e-2
normwise); the n_q appended tokens are checked bit-exact at the slots of the oracle's index map,
and every other pool byte must be unchanged.
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


def _host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_verify(a: I.AttnVerifyInputs, kp=None, vp=None):
    kp = _bits_dev(a.k_pool) if kp is None else kp
    vp = _bits_dev(a.v_pool) if vp is None else vp
    msl = int(a.seq_lens.max())
    ws = torch.empty(hmd.attn_verify_workspace_size(a.kind, a.window, a.n_q, a.B, a.Hq, a.Hkv,
                                                    a.d, a.page_tokens, msl),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty(a.B, a.n_q, a.Hq, a.d, device="cuda", dtype=torch.bfloat16)
    hmd.attn_verify(a.kind, a.window, a.ring_pages, _bits_dev(a.q), _bits_dev(a.new_k),
                    _bits_dev(a.new_v), kp, vp, _i32(a.page_table), _i32(a.seq_lens), msl, o, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    return o, kp, vp


def expected_pools(O, a: I.AttnVerifyInputs):
    ek, ev = a.k_pool.copy(), a.v_pool.copy()
    for b in range(a.B):
        for i in range(a.n_q):
            pos = int(a.seq_lens[b]) - a.n_q + i
            pg, off = O.kv_slot_ring(a.kind, a.ring_pages, a.page_tokens, a.page_table[b], pos)
            ek[pg, :, off], ev[pg, :, off] = a.new_k[b, i], a.new_v[b, i]
    return ek, ev


def check(O, a: I.AttnVerifyInputs):
    o, kp, vp = run_verify(a)
    ref = O.attn_verify(a.kind, a.window, a.ring_pages, a.q, a.new_k, a.new_v, a.k_pool,
                        a.v_pool, a.page_table, a.seq_lens)
    err = O.rel_err(o.float().cpu().numpy(), ref)
    assert err < 2e-2, err
    ek, ev = expected_pools(O, a)
    np.testing.assert_array_equal(_host_bits(kp), ek)
    np.testing.assert_array_equal(_host_bits(vp), ev)
    return o


CASES = [  # kind, window, n_q, Hq, Hkv, d, seq_lens (each >= n_q)
    (I.FA, 0, 2, 8, 2, 128, [2, 63, 64, 65, 129, 300]),
    (I.FA, 0, 4, 8, 2, 128, [4, 66, 128, 130, 257, 500]),   # new tokens straddle pages
    (I.FA, 0, 4, 32, 8, 64, [5, 64, 191, 260]),
    (I.FA, 0, 16, 4, 4, 128, [16, 70, 200]),                # G = 1: 16 tokens per pass
    (I.FA, 0, 8, 4, 2, 128, [8, 64, 300]),                  # G = 2: 8 tokens
    (I.SWA, 100, 4, 8, 2, 128, [4, 90, 103, 104, 300, 777]),  # smallest ring (2 pages), wraps
    (I.SWA, 64, 3, 8, 2, 128, [3, 65, 66, 200, 401]),
    (I.SWA, 1, 4, 8, 2, 64, [4, 70, 129]),
    (I.SWA, 4096, 2, 32, 8, 128, [2, 4097, 5000]),
]


@pytest.mark.parametrize("kind,window,n_q,Hq,Hkv,d,lens", CASES)
def test_verify_matches_oracle_and_appends(oracle_mod, kind, window, n_q, Hq, Hkv, d, lens):
    lens = np.array(lens, np.int32)
    a = I.verify_inputs(kind, len(lens), n_q, Hq, Hkv, d, int(lens.max()), window=window,
                        seed=int(lens.sum()) + n_q, seq_lens=lens)
    check(oracle_mod, a)


def test_verify_with_a_larger_ring(oracle_mod):
    lens = np.array([4, 200, 390], np.int32)
    a = I.verify_inputs(I.SWA, 3, 4, 8, 2, 128, 390, window=100, ring_pages=5, seed=5,
                        seq_lens=lens)
    check(oracle_mod, a)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 300)])
def test_one_token_is_the_decode_step_bitwise(kind, window):
    a = I.verify_inputs(kind, 6, 1, 32, 8, 128, 1000, window=window,
                        ring_pages=-(-window // 64) if kind == I.SWA else 0, seed=9,
                        seq_lens=np.array([1, 64, 65, 300, 999, 1000]))
    o, kp, vp = run_verify(a)
    kp2, vp2 = _bits_dev(a.k_pool), _bits_dev(a.v_pool)
    msl = int(a.seq_lens.max())
    ws = torch.empty(hmd.attn_decode_workspace_size(kind, window, a.B, a.Hq, a.Hkv, a.d, 64, msl),
                     dtype=torch.uint8, device="cuda")
    o2 = torch.empty(a.B, a.Hq, a.d, device="cuda", dtype=torch.bfloat16)
    hmd.attn_decode(kind, window, _bits_dev(a.q[:, 0]), _bits_dev(a.new_k[:, 0]),
                    _bits_dev(a.new_v[:, 0]), kp2, vp2, _i32(a.page_table), _i32(a.seq_lens),
                    msl, o2, ws)
    torch.cuda.synchronize()
    assert torch.equal(o[:, 0].view(torch.int16), o2.view(torch.int16))
    assert torch.equal(kp.view(torch.int16), kp2.view(torch.int16))
    assert torch.equal(vp.view(torch.int16), vp2.view(torch.int16))


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 200)])
def test_verify_equals_successive_one_token_passes(oracle_mod, kind, window):
    """n_q tokens in one pass leave the same cache, bit for bit, as n_q one-token passes on the
    same ring, and give the same outputs within the bf16 tolerance."""
    n_q = 4
    lens = np.array([4, 100, 257, 640], np.int32)
    a = I.verify_inputs(kind, 4, n_q, 16, 4, 128, 640, window=window, seed=11, seq_lens=lens)
    o, kp, vp = run_verify(a)
    kp2, vp2 = _bits_dev(a.k_pool), _bits_dev(a.v_pool)
    outs = []
    for i in range(n_q):
        step = I.AttnVerifyInputs(kind, window, a.ring_pages, 1, a.B, a.Hq, a.Hkv, a.d, 64,
                                  a.k_pool, a.v_pool, a.page_table, lens - n_q + i + 1,
                                  a.q[:, i:i + 1], a.new_k[:, i:i + 1], a.new_v[:, i:i + 1])
        oi, kp2, vp2 = run_verify(step, kp2, vp2)
        outs.append(oi[:, 0].float().cpu().numpy())
    assert torch.equal(kp.view(torch.int16), kp2.view(torch.int16))
    assert torch.equal(vp.view(torch.int16), vp2.view(torch.int16))
    seq = np.stack(outs, axis=1)
    assert oracle_mod.rel_err(o.float().cpu().numpy(), seq) < 2e-2


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 4096)])
def test_full_size_verify(oracle_mod, kind, window):
    """B=32, Hq=32, Hkv=8, d=128, context 8192 counting 4 new tokens per sequence, pages of 64
    under a random permutation (SWA: window 4096 on the smallest ring, 65 pages)."""
    a = I.verify_inputs(kind, 32, 4, 32, 8, 128, 8192, window=window, seed=12)
    check(oracle_mod, a)
