"""Mixed placements in one batch, host side (CPU only): the per-layer grouping of sequences by
the mixer their placement picks, and its argument checks."""
import numpy as np

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import inputs as I

ARG = 1


def _brute(placements, seq_placement):
    n_l = placements.shape[1]
    groups = []
    for l in range(n_l):
        groups.append({k: [b for b, p in enumerate(seq_placement) if placements[p, l] == k]
                       for k in (I.FA, I.SWA, I.KDA, I.GDN)})
    return groups


def test_grouping_matches_brute_force():
    g = I.rng(7)
    for trial in range(20):
        n_p, n_l, B = int(g.integers(1, 5)), int(g.integers(1, 49)), int(g.integers(1, 70))
        pl = g.integers(0, 4, size=(n_p, n_l)).astype(np.int8)
        sp = g.integers(0, n_p, size=B).astype(np.int32)
        rows, offs = hmd.group_sequences(pl, sp)
        ref = _brute(pl, sp)
        for l in range(n_l):
            assert sorted(rows[l]) == list(range(B))  # every sequence exactly once per layer
            for k in (I.FA, I.SWA, I.KDA, I.GDN):
                assert list(rows[l, offs[l, k]:offs[l, k + 1]]) == ref[l][k], (trial, l, k)
            assert offs[l, 0] == 0 and offs[l, 4] == B


def test_one_placement_is_the_plain_step():
    pl = I.placement({I.FA: 12, I.SWA: 12, I.KDA: 12, I.GDN: 12}, seed=0)[None, :]
    rows, offs = hmd.group_sequences(pl, np.zeros(9, np.int32))
    for l in range(48):
        k = int(pl[0, l])
        assert offs[l, k + 1] - offs[l, k] == 9 and list(rows[l]) == list(range(9))


def test_grouping_rejects_bad_arguments():
    L = hmd.lib()
    pl = np.array([[0, 1, 2, 3]], np.int8)
    sp = np.array([0, 0], np.int32)
    rows = np.zeros((4, 2), np.int32)
    offs = np.zeros((4, 5), np.int32)
    call = lambda p, s, B=2: L.hmd_group_sequences(4, p.shape[0], p.ctypes.data, B, s.ctypes.data,  # noqa: E731
                                                   rows.ctypes.data, offs.ctypes.data)
    assert call(pl, sp) == 0
    assert call(np.array([[0, 1, 5, 3]], np.int8), sp) == ARG       # not a mixer kind
    assert call(pl, np.array([0, 1], np.int32)) == ARG               # placement 1 does not exist
    assert call(pl, np.array([-1, 0], np.int32)) == ARG
    assert call(pl, sp, B=0) == ARG
    assert L.mixer_decode_step_batch(None, 0, None, None, None, None, 0, None) == ARG


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(st.data())
def test_grouping_properties(data):
    """For any placements and assignment: each layer's rows are a permutation of the batch,
    grouped by kind in FA, SWA, KDA, GDN order, increasing within a group, and each row sits
    in the group of the kind its placement picks at that layer."""
    n_p = data.draw(st.integers(1, 5))
    n_l = data.draw(st.integers(1, 12))
    B = data.draw(st.integers(1, 40))
    pl = np.array(data.draw(st.lists(st.lists(st.integers(0, 3), min_size=n_l, max_size=n_l),
                                     min_size=n_p, max_size=n_p)), np.int8)
    sp = np.array(data.draw(st.lists(st.integers(0, n_p - 1), min_size=B, max_size=B)), np.int32)
    rows, offs = hmd.group_sequences(pl, sp)
    for l in range(n_l):
        assert sorted(rows[l]) == list(range(B))
        assert list(offs[l]) == sorted(offs[l]) and offs[l, 0] == 0 and offs[l, 4] == B
        for k in range(4):
            grp = rows[l, offs[l, k]:offs[l, k + 1]]
            assert list(grp) == sorted(grp)
            assert all(pl[sp[b], l] == k for b in grp)
