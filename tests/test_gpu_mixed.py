"""GPU check of mixed placements in one batch: one layer whose sequences use FA, SWA, KDA and
GDN at once. Each group's results (outputs, appended KV, states) equal, bit for bit, those of
running that group alone as its own batch through the single-mixer entry points, and match
the fp64 oracle."""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import _lib as L
from hybrid_mixer_decoding_b200 import inputs as I

pytestmark = pytest.mark.gpu
bf = torch.bfloat16


def test_mixed_layer_equals_each_group_alone(oracle_mod):
    O = oracle_mod
    B, H, Hkv, d, ctx, w = 7, 8, 2, 128, 300, 100
    # four placements of a 1-layer stack; sequence b follows placement sp[b]
    placements = np.array([[I.FA], [I.SWA], [I.KDA], [I.GDN]], np.int8)
    sp = np.array([2, 0, 3, 1, 0, 2, 3], np.int32)
    lens = np.array([300, 130, 7, 200, 65, 299, 1], np.int32)
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    # one pool shared by the layer's FA and SWA sequences; table rows of ceil(ctx/64) pages
    pps = -(-ctx // 64)
    kc = L.KVCache([0], 1, B * pps, Hkv, d, 64)
    kp, vp = kc.layer_pools(0)
    kp.normal_(generator=g)
    vp.normal_(generator=g)
    table = torch.randperm(B * pps, generator=g, device="cuda").to(torch.int32).view(B, pps).contiguous()
    ring = table[:, :-(-w // 64)].contiguous()
    seq_lens = torch.from_numpy(lens).cuda()
    sc = L.StateCache(1, B, H, d, d)
    state = sc.layer_view(0)
    state.normal_(0.0, 0.05, generator=g)
    q = torch.randn(B, H, d, generator=g, device="cuda").to(bf)
    k = torch.nn.functional.normalize(torch.randn(B, H, d, generator=g, device="cuda"), dim=-1).to(bf)
    v = torch.randn(B, H, d, generator=g, device="cuda").to(bf)
    beta = torch.sigmoid(torch.randn(B, H, generator=g, device="cuda"))
    lg_s = -0.1 * torch.rand(B, H, generator=g, device="cuda")
    lg_c = -0.05 * torch.rand(B, H, d, generator=g, device="cuda")
    nk = torch.randn(B, Hkv, d, generator=g, device="cuda").to(bf)
    nv = torch.randn(B, Hkv, d, generator=g, device="cuda").to(bf)
    o = torch.zeros(B, H, d, device="cuda", dtype=bf)

    def io(kind):
        x = L.DecodeIO(B=B, H=H, Hkv=Hkv, d=d, dtype=L.BF16)
        x.q, x.o, x.scale = q.data_ptr(), o.data_ptr(), 1.0
        if kind in (I.GDN, I.KDA):
            x.k, x.v, x.beta = k.data_ptr(), v.data_ptr(), beta.data_ptr()
            x.log_gate_scalar, x.log_gate_channel = lg_s.data_ptr(), lg_c.data_ptr()
        else:
            tab = table if kind == I.FA else ring
            x.k, x.v = nk.data_ptr(), nv.data_ptr()
            x.page_table, x.max_pages = tab.data_ptr(), tab.shape[1]
            x.seq_lens, x.max_seq_len, x.window = seq_lens.data_ptr(), ctx, w
        return x

    ios = {kind: io(kind) for kind in (I.FA, I.SWA, I.KDA, I.GDN)}
    plan = L.BatchPlan(placements, sp)
    ws = torch.empty(plan.workspace_size(w, H, Hkv, d, 64, ctx), dtype=torch.uint8, device="cuda")
    # references: each group alone, on copies of the pool and the state
    kp_ref, vp_ref, st_ref = kp.clone(), vp.clone(), state.clone()
    kp0, vp0, st0 = kp.clone(), vp.clone(), state.clone()
    o_ref = torch.zeros_like(o)
    for kind in (I.FA, I.SWA, I.KDA, I.GDN):
        r = torch.from_numpy(plan.group(0, kind)).long().cuda()
        assert list(r.cpu().numpy()) == [b for b in range(B) if placements[sp[b], 0] == kind]
        n = r.numel()
        if kind in (I.GDN, I.KDA):
            og = torch.empty(n, H, d, device="cuda", dtype=bf)
            hmd.delta_rule_decode(kind, q[r].contiguous(), k[r].contiguous(), v[r].contiguous(),
                                  beta[r].contiguous(),
                                  (lg_s if kind == I.GDN else lg_c)[r].contiguous(), st_ref, og,
                                  slots=r.to(torch.int32).contiguous())
        else:
            tab = (table if kind == I.FA else ring)[r].contiguous()
            og = torch.empty(n, H, d, device="cuda", dtype=bf)
            wsr = torch.empty(hmd.attn_decode_workspace_size(kind, w, n, H, Hkv, d, 64, ctx),
                              dtype=torch.uint8, device="cuda")
            hmd.attn_decode(kind, w, q[r].contiguous(), nk[r].contiguous(), nv[r].contiguous(),
                            kp_ref, vp_ref, tab, seq_lens[r].contiguous(), ctx, og, wsr)
        o_ref[r] = og
    hmd.mixer_decode_step_batch(plan, 0, ios, sc, kc, ws)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(kp.view(torch.int16), kp_ref.view(torch.int16))
    assert torch.equal(vp.view(torch.int16), vp_ref.view(torch.int16))
    assert torch.equal(state, st_ref)
    # and against the oracle, group by group
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
    for kind in (I.FA, I.SWA):
        r = plan.group(0, kind)
        tab = (table if kind == I.FA else ring).cpu().numpy()[r]
        ref = O.attn_decode(kind, w, bits(q[r]), bits(nk[r]), bits(nv[r]), bits(kp0), bits(vp0),
                            tab, lens[r])
        assert O.rel_err(o[torch.from_numpy(r).long().cuda()].float().cpu().numpy(), ref) < 2e-2
    for kind in (I.KDA, I.GDN):
        r = plan.group(0, kind)
        rt = torch.from_numpy(r).long().cuda()
        lg = (lg_s if kind == I.GDN else lg_c)[rt]
        o_or, s_or = O.delta_recurrent(kind, q[rt].float().cpu().numpy()[:, None],
                                       k[rt].float().cpu().numpy()[:, None],
                                       v[rt].float().cpu().numpy()[:, None],
                                       beta[rt].cpu().numpy()[:, None], lg.cpu().numpy()[:, None],
                                       st0[rt].cpu().numpy())
        assert O.rel_err(o[rt].float().cpu().numpy(), o_or[:, 0]) < 2e-2
        assert O.rel_err(state[rt].cpu().numpy(), s_or) < 2e-2
    plan.free()
    kc.free()
    sc.free()


def test_mixed_stack_step_in_a_graph():
    from hybrid_mixer_decoding_b200.stack import MixerStack, StackShape
    shape = StackShape(B=6, H=8, Hkv=2, d=128, ctx=400, window=128)
    pls = {"hybrid": np.array([I.FA, I.SWA, I.KDA, I.GDN, I.FA, I.GDN], np.int8),
           "linear": np.array([I.GDN, I.KDA, I.GDN, I.KDA, I.GDN, I.GDN], np.int8)}
    st = MixerStack(pls, shape, seed=1)
    plan = st.batch_plan(np.array([0, 1, 1, 0, 1, 0], np.int32))
    graph = st.capture(lambda: st.step_batch(plan))
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    plan.free()
    st.free()
