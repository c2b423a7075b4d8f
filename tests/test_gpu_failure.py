"""Failure detection on the GPU without a fault: every wait on a copy barrier is bounded.

hmd_test_arm_copy_skip makes one CTA of the next launch arm its copy barrier without issuing
the copy, with a 1 ms wait limit. That CTA's wait runs out, the whole CTA gives up together,
reports HMD_DEVERR_TIMEOUT and writes nothing; nothing invalid is accessed. The tests check the
error bit, that the CTA's outputs are untouched, that every other output equals an unarmed run
of the same call bit for bit, and that the next call on the same context runs cleanly.
"""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import _lib
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu
WAIT_NS = 1_000_000  # 1 ms
SENTINEL = 7.0


def _dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def _bits(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_delta_decode_wait_times_out_cleanly(kind):
    B, H, d = 2, 2, 128
    x = I.delta_inputs(kind, B, 1, H, d, d, dtype="bf16", seed=31, state0="randn")
    bf = torch.bfloat16
    args = (_dev(x.q[:, 0], bf), _dev(x.k[:, 0], bf), _dev(x.v[:, 0], bf), _dev(x.beta[:, 0]),
            _dev(x.log_gate[:, 0]))
    s0 = _dev(x.state0)
    assert hmd.hmd_device_errors(clear=True) == 0

    # unarmed run: the reference for every CTA that is not disturbed
    s_ref = s0.clone()
    o_ref = torch.full((B, H, d), SENTINEL, device="cuda", dtype=bf)
    hmd.delta_rule_decode(kind, *args, s_ref, o_ref)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0

    # grid: (sequence, head, 32-column slice) -> CTA 5 is sequence 0, head 1, columns 32..63
    s = s0.clone()
    o = torch.full((B, H, d), SENTINEL, device="cuda", dtype=bf)
    hmd.hmd_test_arm_copy_skip(_lib.TEST_DELTA_DECODE, 5, WAIT_NS)
    hmd.delta_rule_decode(kind, *args, s, o)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) & hmd.DEVERR_TIMEOUT

    untouched = (0, 1, slice(None), slice(32, 64))
    assert torch.equal(s[untouched], s0[untouched])
    assert (o[0, 1, 32:64].float() == SENTINEL).all()
    mask = torch.ones_like(s, dtype=torch.bool)
    mask[untouched] = False
    assert torch.equal(s[mask], s_ref[mask])
    omask = torch.ones_like(o, dtype=torch.bool)
    omask[0, 1, 32:64] = False
    assert torch.equal(o[omask], o_ref[omask])

    # the context is still usable: the same call again, unarmed, reproduces the reference
    s2 = s0.clone()
    o2 = torch.empty_like(o)
    hmd.delta_rule_decode(kind, *args, s2, o2)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    assert torch.equal(s2, s_ref) and torch.equal(o2, o_ref)


@pytest.mark.parametrize("kind,window", [(I.FA, 0), (I.SWA, 200)])
def test_attn_split_wait_times_out_cleanly(kind, window):
    B, Hq, Hkv, d, ctx = 2, 8, 2, 128, 300
    a = I.attn_inputs(kind, B, Hq, Hkv, d, ctx, window=window, seed=32)
    q, nk, nv = _bits(a.q), _bits(a.new_k), _bits(a.new_v)
    table = _dev(a.page_table, torch.int32)
    lens = _dev(a.seq_lens, torch.int32)
    ws = torch.empty(hmd.attn_decode_workspace_size(kind, window, B, Hq, Hkv, d, 64, ctx),
                     dtype=torch.uint8, device="cuda")
    assert hmd.hmd_device_errors(clear=True) == 0

    kp_ref, vp_ref = _bits(a.k_pool), _bits(a.v_pool)
    o_ref = torch.full((B, Hq, d), SENTINEL, device="cuda", dtype=torch.bfloat16)
    hmd.attn_decode(kind, window, q, nk, nv, kp_ref, vp_ref, table, lens, ctx, o_ref, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0

    # CTA 0 is the first key range of sequence 0, kv-head 0 (query heads 0..3); with five
    # one-page ranges here it does not hold the new token, so every append still happens
    kp, vp = _bits(a.k_pool), _bits(a.v_pool)
    o = torch.full((B, Hq, d), SENTINEL, device="cuda", dtype=torch.bfloat16)
    hmd.hmd_test_arm_copy_skip(_lib.TEST_ATTN_SPLIT, 0, WAIT_NS)
    hmd.attn_decode(kind, window, q, nk, nv, kp, vp, table, lens, ctx, o, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) & hmd.DEVERR_TIMEOUT
    G = Hq // Hkv
    assert (o[0, :G].float() == SENTINEL).all()  # the combine left the affected heads alone
    assert torch.equal(o[0, G:], o_ref[0, G:]) and torch.equal(o[1], o_ref[1])
    assert torch.equal(kp, kp_ref) and torch.equal(vp, vp_ref)

    o2 = torch.empty_like(o)
    kp2, vp2 = _bits(a.k_pool), _bits(a.v_pool)
    hmd.attn_decode(kind, window, q, nk, nv, kp2, vp2, table, lens, ctx, o2, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    assert torch.equal(o2, o_ref)
