"""Host-side logic of bench.py that needs no GPU: the sweep's placements and the linear
per-layer cost model the pages describe (a placement's cost is the sum of its layers' costs)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from hybrid_mixer_decoding_b200 import inputs as I  # noqa: E402


def test_sweep_placements_have_the_stated_mixer_counts():
    pls = bench.sweep_placements()
    want = {"all-FA": {I.FA: 48}, "24FA+24GDN": {I.FA: 24, I.GDN: 24},
            "8FA+20KDA+20GDN": {I.FA: 8, I.KDA: 20, I.GDN: 20}, "all-GDN": {I.GDN: 48},
            "all-KDA": {I.KDA: 48}}
    assert set(pls) == set(want)
    for name, counts in want.items():
        got = {int(k): int(n) for k, n in zip(*np.unique(pls[name], return_counts=True))}
        assert got == counts, name


def test_linear_cost_model_recovers_per_layer_costs_and_flags_nonlinearity():
    pls = bench.sweep_placements()
    cost = {I.FA: 0.25, I.KDA: 0.0131, I.GDN: 0.0127}  # ms per layer
    res = {n: {"ms_per_step": sum(cost[int(k)] for k in pl)} for n, pl in pls.items()}
    res["8FA+20KDA+20GDN"]["ms_per_step"] *= 1.05      # a 5% interaction
    m = bench.linear_cost_model(pls, res)
    assert m["per_layer_us"] == {"FA": 250.0, "KDA": 13.1, "GDN": 12.7}
    assert m["error_pct"]["24FA+24GDN"] == 0.0
    assert m["error_pct"]["8FA+20KDA+20GDN"] == 5.0
    assert m["predicted_ms"]["24FA+24GDN"] == round(24 * 0.25 + 24 * 0.0127, 3)
    assert set(m["error_pct"]) == {"24FA+24GDN", "8FA+20KDA+20GDN"}
