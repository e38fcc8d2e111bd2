"""The reference arm's JSON line carries the contract's keys (CPU only: the oracle sample is
replaced by a stub that takes no time, so only the line's shape is checked here)."""
import argparse
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_line_keys(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    calls = []

    def fake_sample(p, rows, cols=None):
        calls.append((rows, cols))
        return 0.5 if cols is None and rows == 1 else 0.01

    monkeypatch.setattr(bench, "_oracle_sample", fake_sample)
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(argparse.Namespace(steps=1500, warmup=300))
    lines = [l for l in out.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
              "cpu_baseline"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1500 and d["warmup"] == 300
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert "workload" in d["config"]
    # 1800 steps within the ~150 s budget: one full-width row (0.5 s here) is too much, so the
    # sample narrows to the first output features
    assert all(c is not None and c < 14336 for r, c in calls[1:])
