"""bench.py's host-side helpers (no GPU)."""
import json

import numpy as np

import bench
import oracle


def test_balance_log_matches_the_oracle_metrics(tmp_path):
    counts = np.array([[10, 2, 0, 4], [4, 4, 4, 4], [0, 0, 16, 0]])
    path = tmp_path / "bal.jsonl"
    bench.write_balance_log(str(path), counts, T=8, k=2, capacity=5)
    lines = [json.loads(l) for l in open(path)]
    assert [l["step"] for l in lines] == [0, 1, 2]
    for L, rec in zip(counts, lines):
        m = oracle.load_metrics(L, 5, 8, 2)
        assert rec["max_load"] == m["max_load"] and rec["dropped"] == m["dropped"]
        assert abs(rec["max_vio"] - m["max_vio"]) < 1e-6 and abs(rec["drop_rate"] - m["drop_rate"]) < 1e-8
    bench.write_balance_log(str(path), counts, T=8, k=2, capacity=None)
    assert "dropped" not in json.loads(open(path).readline())


def test_peaks_fall_back_without_the_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.peaks()
    assert p["src"] == "fallback" and p["hbm_gbs"] == bench.FALLBACK_HBM_GBS
