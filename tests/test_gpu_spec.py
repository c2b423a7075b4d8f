"""GPU check of one self-speculative round on a 4-layer stack (FA, SWA, KDA, GDN target; all-GDN
drafter): the verify pass matches the fp64 oracle on the cache as it stood, and each slot of
the recurrent-state chain (one delta_rule_decode_chain launch per GDN/KDA layer) holds exactly
the state of that many in-place decode steps."""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I
from hybrid_mixer_decoding_b200.spec import SpecStack, make_schedule
from hybrid_mixer_decoding_b200.stack import StackShape

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_one_round(oracle_mod):
    O = oracle_mod
    k = 3
    shape = StackShape(B=3, H=8, Hkv=2, d=128, ctx=420, window=100)
    target = np.array([I.FA, I.SWA, I.KDA, I.GDN], np.int8)
    sp = SpecStack(target, shape, k, max_rounds=4, fill=True, seed=5)
    sched = make_schedule(shape.B, k, 4, sp.L0, 0.6, seed=2)
    slots_dev = torch.from_numpy(sched.slots).cuda()
    lens_dev = torch.from_numpy(sched.lens).cuda()
    sp.set_round(sched, 0, slots_dev, lens_dev)
    # the caches and states before the round
    pools0 = {l: tuple(_bits(p) for p in (sp.kv_fa if target[l] == I.FA else sp.kv_swa).layer_pools(l))
              for l in (0, 1)}
    st0 = {l: sp.t_state.layer_view(sp.t_lin.index(l)).clone() for l in (2, 3)}
    sp.draft()
    sp.verify()
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0

    lens = sched.lens[0]
    for l in (0, 1):
        t = sp.t_in[l]
        table = (sp.table_fa if target[l] == I.FA else sp.table_swa).cpu().numpy()
        ref = O.attn_verify(int(target[l]), shape.window, sp.ring, _bits(t["q"]), _bits(t["nk"]),
                            _bits(t["nv"]), pools0[l][0], pools0[l][1], table, lens)
        assert O.rel_err(t["o"].float().cpu().numpy(), ref) < 2e-2

    chain = sched.slots[0]  # [k + 2][B]
    for l in (2, 3):
        t = sp.t_in[l]
        st = st0[l][torch.from_numpy(chain[0]).long().cuda()].clone()  # [B, H, d, d]
        for step in range(k + 1):
            x = {n: t[n][:, step].contiguous() for n in ("q", "k", "v", "beta", "lg", "o")}
            o = torch.empty_like(x["o"])
            hmd.delta_rule_decode(int(target[l]), x["q"], x["k"], x["v"], x["beta"], x["lg"], st, o)
            got = sp.t_state.layer_view(sp.t_lin.index(l))[torch.from_numpy(chain[step + 1]).long().cuda()]
            assert torch.equal(got, st), (l, step)
            assert torch.equal(o.view(torch.int16), x["o"].view(torch.int16))
    sp.free()


def test_rounds_run_as_graphs_without_errors():
    k = 3
    shape = StackShape(B=4, H=8, Hkv=2, d=128, ctx=700, window=128)
    target = np.array([I.FA, I.GDN, I.SWA, I.KDA, I.FA, I.GDN], np.int8)
    sp = SpecStack(target, shape, k, max_rounds=8)
    sched = make_schedule(shape.B, k, 8, sp.L0, 0.8, seed=4)
    slots_dev = torch.from_numpy(sched.slots).cuda()
    lens_dev = torch.from_numpy(sched.lens).cuda()
    gd, gv, gp = sp.capture(sp.draft), sp.capture(sp.verify), sp.capture(sp.plain_step)
    for r in range(8):
        sp.set_round(sched, r, slots_dev, lens_dev)
        gd.replay()
        gv.replay()
    gp.replay()
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    sp.free()
