"""The placement dispatcher on the GPU: a mixer-only stack decoded through mixer_decode_step,
layer by layer against the fp64 oracle, with placements switched between steps on the same
registered caches (no reallocation, no copy).
"""
import numpy as np
import pytest
import torch

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I
from hybrid_mixer_decoding_b200.stack import MixerStack, StackShape

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def snapshot(st: MixerStack, layer: int, kind: int, seqs):
    """Host copy of what layer `layer` reads under `kind`, for sequences `seqs`, taken before
    the step (the oracle gets each sequence's pages with an identity table)."""
    t = st.inputs[layer]
    snap = {"q": t["q"][seqs].float().cpu().numpy()}
    if kind in (I.GDN, I.KDA):
        snap["k"] = t["k"][seqs].float().cpu().numpy()
        snap["v"] = t["v"][seqs].float().cpu().numpy()
        snap["beta"] = t["beta"][seqs].cpu().numpy()
        snap["lg"] = (t["lg_s"] if kind == I.GDN else t["lg_c"])[seqs].cpu().numpy()
        snap["state"] = st.state.layer_view(layer)[seqs].cpu().numpy()
    else:
        kp, vp = st.pools_for(layer)
        tab = st.table_for(layer, kind)[seqs]  # [n, max_pages]
        n, mp = tab.shape
        valid = (tab >= 0)
        idx = tab.clamp(min=0).long()
        snap["k_pool"] = _bits(kp[idx.view(-1)]).reshape(n * mp, *kp.shape[1:])
        snap["v_pool"] = _bits(vp[idx.view(-1)]).reshape(n * mp, *vp.shape[1:])
        table = np.arange(n * mp, dtype=np.int32).reshape(n, mp)
        table[~valid.cpu().numpy()] = -1
        snap["table"] = table
        snap["q_bits"] = _bits(t["q"][seqs])
        snap["nk"], snap["nv"] = _bits(t["nk"][seqs]), _bits(t["nv"][seqs])
        snap["lens"] = st.seq_lens[seqs].cpu().numpy()
    return snap


def oracle_layer(O, st: MixerStack, kind, snap):
    if kind in (I.GDN, I.KDA):
        o, s = O.delta_recurrent(kind, snap["q"][:, None], snap["k"][:, None], snap["v"][:, None],
                                 snap["beta"][:, None], snap["lg"][:, None], snap["state"])
        return o[:, 0], s
    return O.attn_decode(kind, st.shape.window, snap["q_bits"], snap["nk"], snap["nv"],
                         snap["k_pool"], snap["v_pool"], snap["table"], snap["lens"]), None


def check_step(O, st, name, seqs):
    pl = st.placements[name]
    snaps = [snapshot(st, l, int(pl[l]), seqs) for l in range(st.n_layers)]
    st.step(name)
    torch.cuda.synchronize()
    assert hmd.hmd_device_errors(clear=True) == 0
    for l in range(st.n_layers):
        kind = int(pl[l])
        ref, ref_state = oracle_layer(O, st, kind, snaps[l])
        got = st.inputs[l]["o"][seqs].float().cpu().numpy()
        assert O.rel_err(got, ref) < 2e-2, (name, l, kind)
        if ref_state is not None:
            new_state = st.state.layer_view(l)[seqs].cpu().numpy()
            assert O.rel_err(new_state, ref_state) < 2e-2, (name, l, kind)


def test_small_stack_and_placement_switch(oracle_mod):
    O = oracle_mod
    shape = StackShape(B=3, H=8, Hkv=2, d=128, ctx=300, window=100)
    hybrid = I.placement({I.FA: 2, I.SWA: 2, I.KDA: 2, I.GDN: 2}, seed=0)
    # the other placement swaps every layer to a different kind
    alt = np.array([{I.FA: I.GDN, I.SWA: I.KDA, I.KDA: I.FA, I.GDN: I.SWA}[int(k)]
                    for k in hybrid], np.int8)
    st = MixerStack({"hybrid": hybrid, "alt": alt}, shape, seed=3)
    seqs = torch.arange(3, device="cuda")
    check_step(O, st, "hybrid", seqs)
    free0 = torch.cuda.mem_get_info()[0]
    check_step(O, st, "alt", seqs)          # switch: same caches, nothing reallocated
    check_step(O, st, "hybrid", seqs)       # and back, continuing from the updated caches
    assert torch.cuda.mem_get_info()[0] == free0
    st.free()


def test_stack48_full_size_sampled(oracle_mod):
    """The benchmark's workload (48 layers, 12 FA / 12 SWA w=4096 / 12 KDA / 12 GDN shuffled,
    B=64, ctx 32768, H=32, Hkv=8, d=128), one step, checked on every layer for a sample of
    three sequences."""
    O = oracle_mod
    shape = StackShape(B=64, H=32, Hkv=8, d=128, ctx=32768, window=4096)
    pl = I.placement({I.FA: 12, I.SWA: 12, I.KDA: 12, I.GDN: 12}, seed=0)
    st = MixerStack({"hybrid": pl}, shape, seed=0)
    seqs = torch.tensor([0, 31, 63], device="cuda")
    check_step(O, st, "hybrid", seqs)
    st.free()


def test_graph_replay_matches_eager_step():
    """A CUDA graph of the 48-call step (as the sweep replays it) reproduces the eager step
    bit for bit, starting from the same caches."""
    shape = StackShape(B=3, H=8, Hkv=2, d=128, ctx=300, window=100)
    pl = I.placement({I.FA: 2, I.SWA: 2, I.KDA: 2, I.GDN: 2}, seed=1)
    st = MixerStack({"p": pl}, shape, seed=4)
    g = st.capture("p")  # capture runs two warm-up steps first

    def snap():
        states = [st.state.layer_view(l).clone() for l in range(st.n_layers)]
        pools = [tuple(p.clone() for p in st.pools_for(l)) if pl[l] in (I.FA, I.SWA) else None
                 for l in range(st.n_layers)]
        return states, pools

    def restore(s):
        for l in range(st.n_layers):
            st.state.layer_view(l).copy_(s[0][l])
            if s[1][l] is not None:
                kp, vp = st.pools_for(l)
                kp.copy_(s[1][l][0])
                vp.copy_(s[1][l][1])

    s0 = snap()
    st.step("p")
    torch.cuda.synchronize()
    eager = [st.inputs[l]["o"].clone() for l in range(st.n_layers)]
    eager_state = [st.state.layer_view(l).clone() for l in range(st.n_layers)]
    restore(s0)
    g.replay()
    torch.cuda.synchronize()
    for l in range(st.n_layers):
        assert torch.equal(st.inputs[l]["o"], eager[l]), l
        assert torch.equal(st.state.layer_view(l), eager_state[l]), l
    del g
    st.free()
