"""GPU parity of the fused input activations (raw q, k L2-normalised, beta sigmoid, log-gate
-exp(A_log) softplus(logit + dt_bias)) in the delta-rule decode and chunked-prefill kernels,
against the fp64 oracle's activations followed by its token-by-token recurrence."""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-4, "bf16": 2e-2}


def _dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(dtype)


def _reference(O, r: I.DeltaRawInputs, eps):
    q, k, beta, lg = O.delta_activations(r.kind, r.q_raw, r.k_raw, r.beta_logit, r.gate_logit,
                                         r.A_log, r.dt_bias, eps=eps)
    return O.delta_recurrent(r.kind, q, k, r.v, beta, lg, r.state0)


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_act_steps_match_oracle(oracle_mod, kind, dtype):
    O = oracle_mod
    B, T, H, dk, dv = 3, 6, 4, 128, 64
    r = I.delta_raw_inputs(kind, B, T, H, dk, dv, dtype=dtype, seed=40)
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    state = _dev(r.state0)
    A, db = _dev(r.A_log), _dev(r.dt_bias)
    outs = []
    for t in range(T):
        o = torch.empty(B, H, dv, device="cuda", dtype=act)
        hmd.delta_rule_decode_act(kind, _dev(r.q_raw[:, t], act), _dev(r.k_raw[:, t], act),
                                  _dev(r.v[:, t], act), _dev(r.beta_logit[:, t]),
                                  _dev(r.gate_logit[:, t]), A, db, state, o, eps=1e-6)
        outs.append(o.float())
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    o_ref, s_ref = _reference(O, r, 1e-6)
    assert O.rel_err(torch.stack(outs, 1).cpu().numpy(), o_ref) < TOL[dtype]
    assert O.rel_err(state.cpu().numpy(), s_ref) < TOL[dtype]


@pytest.mark.parametrize("kind", [I.GDN, I.KDA])
@pytest.mark.parametrize("T", [1, 64, 200])
def test_prefill_act_matches_oracle(oracle_mod, kind, T):
    O = oracle_mod
    B, H, d = 2, 3, 128
    r = I.delta_raw_inputs(kind, B, T, H, d, d, dtype="bf16", seed=41 + T)
    state = _dev(r.state0)
    o = torch.empty(B, T, H, d, device="cuda", dtype=torch.bfloat16)
    hmd.delta_rule_prefill_chunked_act(kind, _dev(r.q_raw, torch.bfloat16),
                                       _dev(r.k_raw, torch.bfloat16), _dev(r.v, torch.bfloat16),
                                       _dev(r.beta_logit), _dev(r.gate_logit), _dev(r.A_log),
                                       _dev(r.dt_bias), state, o, eps=1e-6)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    o_ref, s_ref = _reference(O, r, 1e-6)
    assert O.rel_err(o.float().cpu().numpy(), o_ref) < 2e-2
    assert O.rel_err(state.cpu().numpy(), s_ref) < 2e-2


def test_prefill_act_then_decode_act_continue_the_recurrence(oracle_mod):
    """A prefill of 100 raw tokens followed by 3 raw decode steps equals the oracle over 103."""
    O = oracle_mod
    kind, B, T, H, d = I.KDA, 2, 103, 2, 128
    r = I.delta_raw_inputs(kind, B, T, H, d, d, dtype="bf16", seed=43)
    bf = torch.bfloat16
    state = _dev(r.state0)
    A, db = _dev(r.A_log), _dev(r.dt_bias)
    o = torch.empty(B, 100, H, d, device="cuda", dtype=bf)
    hmd.delta_rule_prefill_chunked_act(kind, _dev(r.q_raw[:, :100], bf), _dev(r.k_raw[:, :100], bf),
                                       _dev(r.v[:, :100], bf), _dev(r.beta_logit[:, :100]),
                                       _dev(r.gate_logit[:, :100]), A, db, state, o)
    tail = []
    for t in range(100, T):
        ot = torch.empty(B, H, d, device="cuda", dtype=bf)
        hmd.delta_rule_decode_act(kind, _dev(r.q_raw[:, t], bf), _dev(r.k_raw[:, t], bf),
                                  _dev(r.v[:, t], bf), _dev(r.beta_logit[:, t]),
                                  _dev(r.gate_logit[:, t]), A, db, state, ot)
        tail.append(ot.float())
    torch.cuda.synchronize()
    o_ref, s_ref = _reference(O, r, 1e-6)
    assert O.rel_err(o.float().cpu().numpy(), o_ref[:, :100]) < 2e-2
    assert O.rel_err(torch.stack(tail, 1).cpu().numpy(), o_ref[:, 100:]) < 2e-2
    assert O.rel_err(state.cpu().numpy(), s_ref) < 2e-2
