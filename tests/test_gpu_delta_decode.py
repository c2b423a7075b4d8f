"""GPU parity of delta_rule_decode (GDN, KDA) against the fp64 oracle, through the C ABI.

Tolerances (normwise max|x - y| / max|y| per output tensor): 1e-4 when activations are fp32,
2e-2 when they are bf16 (both the outputs and the fp32 states of a bf16 call).
"""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def _run_decode_steps(d: I.DeltaInputs, slots=None, n_slots=None):
    """Feed the T tokens of d one decode step at a time through the C ABI."""
    act = torch.bfloat16 if d.dtype == "bf16" else torch.float32
    n_slots = n_slots or d.B
    state = torch.zeros(n_slots, d.H, d.dk, d.dv, device="cuda")
    sl = np.arange(d.B) if slots is None else np.asarray(slots)
    state[torch.from_numpy(sl).long().cuda()] = _dev(d.state0)
    slots_t = None if slots is None else _dev(sl.astype(np.int32), torch.int32)
    outs = []
    for t in range(d.T):
        q, k, v = (_dev(x[:, t], act) for x in (d.q, d.k, d.v))
        beta = _dev(d.beta[:, t])
        lg = _dev(d.log_gate[:, t])
        o = torch.empty(d.B, d.H, d.dv, device="cuda", dtype=act)
        hmd.delta_rule_decode(d.kind, q, k, v, beta, lg, state, o, slots=slots_t)
        outs.append(o.float())
    torch.cuda.synchronize()
    o = torch.stack(outs, dim=1).cpu().numpy()
    return o, state[torch.from_numpy(sl).long().cuda()].cpu().numpy()


def test_config1_gdn_fp32_128_steps(oracle_mod):
    """GDN, B=1, H=2, d_k=d_v=64, T=128, fp32, S0=0, seed 0: token-by-token decode."""
    O = oracle_mod
    d = I.delta_inputs(I.GDN, 1, 128, 2, 64, 64, dtype="f32", seed=0)
    o, st = _run_decode_steps(d)
    o_ref, st_ref = O.delta_recurrent(I.GDN, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)
    assert O.rel_err(o, o_ref) < TOL["f32"]
    assert O.rel_err(st, st_ref) < TOL["f32"]


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 64), (128, 128), (64, 40), (256, 32)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_matches_oracle(oracle_mod, kind, dk, dv, dtype):
    O = oracle_mod
    d = I.delta_inputs(kind, 3, 6, 4, dk, dv, dtype=dtype, seed=100 + dk + dv, state0="randn")
    slots = [5, 0, 2]  # sequences in non-identity slots
    o, st = _run_decode_steps(d, slots=slots, n_slots=7)
    o_ref, st_ref = O.delta_recurrent(kind, d.q, d.k, d.v, d.beta, d.log_gate, d.state0)
    assert O.rel_err(o, o_ref) < TOL[dtype]
    assert O.rel_err(st, st_ref) < TOL[dtype]


def test_decode_scale_and_other_slots_untouched(oracle_mod):
    O = oracle_mod
    d = I.delta_inputs(I.KDA, 2, 1, 2, 64, 64, dtype="f32", seed=7, state0="randn")
    state = torch.randn(4, 2, 64, 64, device="cuda")
    before = state.clone()
    state[1] = _dev(d.state0[0])
    state[3] = _dev(d.state0[1])
    slots = _dev(np.array([1, 3], np.int32), torch.int32)
    o = torch.empty(2, 2, 64, device="cuda")
    hmd.delta_rule_decode(I.KDA, _dev(d.q[:, 0]), _dev(d.k[:, 0]), _dev(d.v[:, 0]),
                          _dev(d.beta[:, 0]), _dev(d.log_gate[:, 0]), state, o, slots=slots,
                          scale=0.125)
    torch.cuda.synchronize()
    o_ref, st_ref = O.delta_recurrent(I.KDA, d.q, d.k, d.v, d.beta, d.log_gate, d.state0,
                                      scale=0.125)
    assert O.rel_err(o.cpu().numpy(), o_ref[:, 0]) < 1e-4
    assert O.rel_err(state[[1, 3]].cpu().numpy(), st_ref) < 1e-4
    assert torch.equal(state[0], before[0]) and torch.equal(state[2], before[2])


def test_decode_bad_slot_sets_device_error():
    hmd.hmd_device_errors(clear=True)
    B, H, d = 2, 2, 64
    state = torch.zeros(2, H, d, d, device="cuda")
    x = torch.randn(B, H, d, device="cuda")
    slots = torch.tensor([0, 5], dtype=torch.int32, device="cuda")  # 5 is out of range
    o = torch.zeros(B, H, d, device="cuda")
    hmd.delta_rule_decode(I.GDN, x, x, x, torch.rand(B, H, device="cuda"),
                          -torch.rand(B, H, device="cuda"), state, o, slots=slots)
    bits = hmd.hmd_device_errors(clear=True)
    assert bits & hmd.DEVERR_SLOT
    assert hmd.hmd_device_errors(clear=True) == 0


def test_decode_is_deterministic():
    d = I.delta_inputs(I.KDA, 4, 1, 8, 128, 128, dtype="bf16", seed=3, state0="randn")
    res = []
    for _ in range(2):
        state = _dev(d.state0)
        o = torch.empty(4, 8, 128, device="cuda", dtype=torch.bfloat16)
        hmd.delta_rule_decode(I.KDA, _dev(d.q[:, 0], torch.bfloat16), _dev(d.k[:, 0], torch.bfloat16),
                              _dev(d.v[:, 0], torch.bfloat16), _dev(d.beta[:, 0]),
                              _dev(d.log_gate[:, 0]), state, o)
        res.append((o.clone(), state.clone()))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_full_size_stack_layer_sampled(oracle_mod, kind):
    """One decode step at the 48-layer stack's per-layer shape (B=64, H=32, d=128, bf16,
    random fp32 state), checked on a sample of (sequence, head) pairs."""
    O = oracle_mod
    B, H, dd = 64, 32, 128
    d = I.delta_inputs(kind, B, 1, H, dd, dd, dtype="bf16", seed=11, state0="randn")
    state = _dev(d.state0)
    o = torch.empty(B, H, dd, device="cuda", dtype=torch.bfloat16)
    hmd.delta_rule_decode(kind, _dev(d.q[:, 0], torch.bfloat16), _dev(d.k[:, 0], torch.bfloat16),
                          _dev(d.v[:, 0], torch.bfloat16), _dev(d.beta[:, 0]),
                          _dev(d.log_gate[:, 0]), state, o)
    torch.cuda.synchronize()
    rs = np.random.default_rng(0)
    for b in rs.choice(B, 6, replace=False):
        sl = slice(b, b + 1)
        o_ref, st_ref = O.delta_recurrent(kind, d.q[sl], d.k[sl], d.v[sl], d.beta[sl],
                                          d.log_gate[sl], d.state0[sl])
        assert O.rel_err(o[b].float().cpu().numpy(), o_ref[0, 0]) < 2e-2
        assert O.rel_err(state[b].cpu().numpy(), st_ref[0]) < 2e-2


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
def test_out_of_place_draft_chain_and_rollback(oracle_mod, kind):
    """A speculative draft of 3 tokens steps slots s0 -> s1 -> s2 -> s3 with
    delta_rule_decode_to: each slot holds the state after its token, bit-identical to the
    in-place path, the source slots are never written, and every slot matches the oracle's
    recurrence after that many tokens (so rejecting tokens is a choice of slot)."""
    O = oracle_mod
    B, T, H, dkv = 3, 3, 4, 128
    d = I.delta_inputs(kind, B, T, H, dkv, dkv, dtype="bf16", seed=31, state0="randn")
    act = torch.bfloat16
    n_slots = B * (T + 1)
    chain = torch.zeros(n_slots, H, dkv, dkv, device="cuda")
    slot_of = lambda t: np.arange(B, dtype=np.int32) * (T + 1) + t  # sequence b, step t
    chain[torch.from_numpy(slot_of(0)).long().cuda()] = _dev(d.state0)
    inplace = torch.zeros(B, H, dkv, dkv, device="cuda")
    inplace[:] = _dev(d.state0)
    for t in range(T):
        q, k, v = (_dev(x[:, t], act) for x in (d.q, d.k, d.v))
        beta, lg = _dev(d.beta[:, t]), _dev(d.log_gate[:, t])
        src_before = chain[torch.from_numpy(slot_of(t)).long().cuda()].clone()
        o1 = torch.empty(B, H, dkv, device="cuda", dtype=act)
        hmd.delta_rule_decode_to(kind, q, k, v, beta, lg, chain, o1,
                                 _dev(slot_of(t), torch.int32), _dev(slot_of(t + 1), torch.int32))
        o2 = torch.empty_like(o1)
        hmd.delta_rule_decode(kind, q, k, v, beta, lg, inplace, o2)
        torch.cuda.synchronize()
        assert hmd.hmd_device_errors(clear=True) == 0
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        assert torch.equal(chain[torch.from_numpy(slot_of(t + 1)).long().cuda()], inplace)
        assert torch.equal(chain[torch.from_numpy(slot_of(t)).long().cuda()], src_before)
        _, st_ref = O.delta_recurrent(kind, d.q[:, :t + 1], d.k[:, :t + 1], d.v[:, :t + 1],
                                      d.beta[:, :t + 1], d.log_gate[:, :t + 1], d.state0)
        got = chain[torch.from_numpy(slot_of(t + 1)).long().cuda()].cpu().numpy()
        assert O.rel_err(got, st_ref) < TOL["bf16"]


def test_out_of_place_bad_destination_sets_device_error():
    d = I.delta_inputs(I.GDN, 2, 1, 2, 64, 64, dtype="bf16", seed=32)
    state = torch.zeros(4, 2, 64, 64, device="cuda")
    before = state.clone()
    o = torch.empty(2, 2, 64, device="cuda", dtype=torch.bfloat16)
    hmd.delta_rule_decode_to(I.GDN, _dev(d.q[:, 0], torch.bfloat16), _dev(d.k[:, 0], torch.bfloat16),
                             _dev(d.v[:, 0], torch.bfloat16), _dev(d.beta[:, 0]),
                             _dev(d.log_gate[:, 0]), state, o, _dev(np.array([0, 1], np.int32), torch.int32),
                             _dev(np.array([2, 4], np.int32), torch.int32))
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) & hmd.DEVERR_SLOT
    # sequence 0 (valid destination) was written to slot 2; sequence 1 skipped entirely
    assert torch.equal(state[[0, 1, 3]], before[[0, 1, 3]])


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chain_launch_equals_steps_and_oracle(oracle_mod, kind, dtype):
    """delta_rule_decode_chain over 4 tokens: every chain slot and output is bit-identical to
    4 delta_rule_decode_to steps along the same chain, the first slot is never written, and the
    slots match the oracle's recurrence after 1..4 tokens."""
    O = oracle_mod
    B, nq, H, dk, dv = 3, 4, 4, 128, 64
    d = I.delta_inputs(kind, B, nq, H, dk, dv, dtype=dtype, seed=50, state0="randn")
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    chain = (np.arange(B)[None, :] * (nq + 1) + np.arange(nq + 1)[:, None]).astype(np.int32)
    n_slots = B * (nq + 1)
    st1 = torch.zeros(n_slots, H, dk, dv, device="cuda")
    st1[torch.from_numpy(chain[0]).long().cuda()] = _dev(d.state0)
    st2 = st1.clone()
    o1 = torch.empty(B, nq, H, dv, device="cuda", dtype=act)
    hmd.delta_rule_decode_chain(kind, _dev(d.q, act), _dev(d.k, act), _dev(d.v, act),
                                _dev(d.beta), _dev(d.log_gate), st1, o1,
                                _dev(chain, torch.int32))
    outs = []
    for t in range(nq):
        o2 = torch.empty(B, H, dv, device="cuda", dtype=act)
        hmd.delta_rule_decode_to(kind, _dev(d.q[:, t], act), _dev(d.k[:, t], act),
                                 _dev(d.v[:, t], act), _dev(d.beta[:, t]), _dev(d.log_gate[:, t]),
                                 st2, o2, _dev(chain[t], torch.int32), _dev(chain[t + 1], torch.int32))
        outs.append(o2)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    assert torch.equal(st1, st2)
    assert torch.equal(o1.view(torch.int16) if act == torch.bfloat16 else o1,
                       (torch.stack(outs, 1).view(torch.int16) if act == torch.bfloat16
                        else torch.stack(outs, 1)))
    np.testing.assert_array_equal(st1[torch.from_numpy(chain[0]).long().cuda()].cpu().numpy(),
                                  d.state0)
    for t in range(nq):
        _, s_ref = O.delta_recurrent(kind, d.q[:, :t + 1], d.k[:, :t + 1], d.v[:, :t + 1],
                                     d.beta[:, :t + 1], d.log_gate[:, :t + 1], d.state0)
        got = st1[torch.from_numpy(chain[t + 1]).long().cuda()].cpu().numpy()
        assert O.rel_err(got, s_ref) < TOL[dtype]


def test_state_cache_save_and_restore_round_trip():
    """state_cache_save copies slots out bit for bit; state_cache_reset(init=...) puts them back
    (a preempted request's recurrent state set aside and restored)."""
    sc = hmd.StateCache(2, 5, 3, 64, 32)
    view = sc.layer_view(1)
    view.normal_()
    orig = view.clone()
    out = torch.empty(2, 3, 64, 32, device="cuda")
    sc.save(1, [3, 0], out)
    torch.cuda.synchronize()
    assert torch.equal(out[0], orig[3]) and torch.equal(out[1], orig[0])
    sc.reset(1, [3, 0])
    torch.cuda.synchronize()
    assert not view[3].any() and not view[0].any()
    sc.reset(1, [3, 0], init=out)
    torch.cuda.synchronize()
    assert torch.equal(view, orig)
    sc.free()
