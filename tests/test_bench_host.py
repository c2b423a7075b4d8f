"""Host-side logic of bench.py that needs no GPU: the sweep's placements, the linear per-layer
cost model the pages describe (a placement's cost is the sum of its layers' costs), and the
committed DRAM-traffic figures with their source-hash guard."""
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


def test_committed_traffic_figures_match_the_current_kernel_sources():
    """Every DRAM-traffic entry was captured on the kernel source as it stands: its sha256 prefix
    matches, so bench.py reports it (a stale entry would silently turn into null)."""
    import json
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        tab = json.load(f)
    keys = [k for k in tab if not k.startswith("_")]
    assert keys
    for k in keys:
        assert bench.traffic_for(k) == tab[k]["bytes_per_launch"], k


def test_traffic_entry_is_ignored_once_its_source_changes(tmp_path, monkeypatch):
    import json
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_bytes(b"kernel v1\n")
    import hashlib
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"x": {"bytes_per_launch": 123, "source": "k.cu", "source_sha": sha}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("x") == 123
    assert bench.traffic_for("missing") is None
    src.write_bytes(b"kernel v2\n")
    assert bench.traffic_for("x") is None
