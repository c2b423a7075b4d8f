"""Host logic of the speculative loop (CPU only): acceptance draws, slot chains, schedules."""
import numpy as np

from hybrid_mixer_decoding_b200 import inputs as I
from hybrid_mixer_decoding_b200.spec import accept_counts, chain_slots, make_schedule


def test_accept_counts_range_and_extremes():
    g = I.rng(0)
    j = accept_counts(g, 1000, 3, 0.8)
    assert j.min() >= 0 and j.max() <= 3
    assert (accept_counts(g, 50, 3, 1.0) == 3).all()
    assert (accept_counts(g, 50, 3, 0.0) == 0).all()
    # P(j >= i) = alpha^i: the mean is alpha + alpha^2 + alpha^3
    big = accept_counts(I.rng(1), 200000, 3, 0.8)
    assert abs(big.mean() - (0.8 + 0.64 + 0.512)) < 0.01


def test_chain_slots_are_private_rings():
    k, B = 3, 5
    cur = np.array([0, 1, 4, 2, 3], np.int32)
    s = chain_slots(cur, k)
    assert s.shape == (k + 2, B) and s.dtype == np.int32
    for b in range(B):
        assert sorted(s[:, b]) == list(range(b * (k + 2), (b + 1) * (k + 2)))
        assert s[0, b] == b * (k + 2) + cur[b]
        # consecutive chain positions are distinct slots (a step never writes its own source)
        assert all(s[t, b] != s[t + 1, b] for t in range(k + 1))


def test_schedule_keeps_the_accepted_slot_and_length():
    k, B, R, L0 = 3, 7, 40, 1000
    sch = make_schedule(B, k, R, L0, 0.7, seed=3)
    L = np.full(B, L0)
    for r in range(R):
        assert (sch.lens[r] == L + k + 1).all()
        j = sch.accepted[r]
        assert sch.tokens[r] == int((j + 1).sum())
        if r + 1 < R:
            # the state after x_0, d_1..d_j (chain position j + 1) starts the next round
            nxt = sch.slots[r][j + 1, np.arange(B)]
            assert (sch.slots[r + 1][0] == nxt).all()
        L = L + j + 1
    assert sch.slots.min() >= 0 and sch.slots.max() < B * (k + 2)


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 20), k=st.integers(1, 6), rounds=st.integers(1, 15),
       alpha=st.floats(0.0, 1.0), seed=st.integers(0, 1000))
def test_schedule_properties(B, k, rounds, alpha, seed):
    sch = make_schedule(B, k, rounds, 100, alpha, seed=seed)
    assert ((sch.accepted >= 0) & (sch.accepted <= k)).all()
    assert sch.slots.min() >= 0 and sch.slots.max() < B * (k + 2)
    for r in range(rounds):
        for b in range(B):  # a sequence's chain never leaves its own k + 2 slots
            assert set(sch.slots[r, :, b]) == set(range(b * (k + 2), (b + 1) * (k + 2)))
    # lengths grow by exactly the tokens each round produced
    grow = (sch.accepted + 1).cumsum(axis=0)
    assert (sch.lens[1:] - sch.lens[:-1] == sch.accepted[:-1] + 1).all()
    if rounds > 1:
        assert (sch.lens[-1] - sch.lens[0] == grow[-2]).all()
