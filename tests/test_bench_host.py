"""bench.py's CPU baseline (the oracle timed on the host cores on a sample of the
workload), on tiny stand-in cases: the time it reports is positive and never
smaller than the sampled calls minus their one-row calls, also when a one-row
call happens to outlast its sampled call (the subtraction must not go negative:
the reference arm divides FLOPs by it)."""
import sys
from pathlib import Path

import pytest

sys.path.insert(0, str(Path(__file__).resolve().parents[1]))
import bench  # noqa: E402
from oracle import krea_oracle as ko  # noqa: E402
from synth import inputs as S  # noqa: E402


def tiny_cases():
    return [S.Case("t_dense", 1, 4, 2, 64, 16, 8, 8, dtype="bf16", mode="dense", seed=7, gate=True),
            S.Case("t_scan", 1, 4, 1, 64, 16, 8, 8, dtype="bf16", mode="scanline", seed=8, window=3)]


def test_oracle_sample_on_tiny_cases(monkeypatch):
    monkeypatch.setattr(bench, "step_cases", tiny_cases)
    flops, seconds, fixed, rows = bench.oracle_sample(rows_per_tile=2, tile_stride=1)
    assert rows > 0 and flops > 0
    assert seconds > 0 and fixed >= 0


def test_oracle_sample_keeps_whole_time_when_fixed_call_is_slower(monkeypatch):
    # a fake oracle whose one-row, one-head call takes longer than the sampled call
    monkeypatch.setattr(bench, "step_cases", tiny_cases)
    clock = {"t": 0.0}

    def fake_attention(c, q, k, v, g, rows=None, batches=None, heads=None):
        clock["t"] += 5.0 if heads == [0] else 1.0
        return {}

    monkeypatch.setattr(ko, "attention", fake_attention)
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock["t"])
    flops, seconds, fixed, rows = bench.oracle_sample(rows_per_tile=1, tile_stride=1)
    assert seconds == pytest.approx(2.0)  # each case keeps its sampled call's whole second
    assert fixed == 0.0
