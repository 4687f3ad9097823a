"""bench.py --impl reference (the oracle arm) keeps the JSON line contract.

Runs on host cores only; a bounded sample keeps it to a few seconds.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_line_on_c1():
    d = _run("--config", "c1", "--steps", "2", "--warmup", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def test_reference_line_on_the_video_workload():
    """The default workload (GNA video, stride 1): the oracle on sampled query tiles."""
    d = _run("--steps", "1", "--warmup", "0")
    assert d["impl"] == "reference" and d["value"] > 0
    assert "stride 1x1x1" in d["config"]["workload"]
    assert "query tiles" in d["cpu_baseline"]["sample"]


def test_oracle_sampler_credits_computed_blocks():
    """The sampled units credit exactly the computed-block FLOPs of their rows: summed over every
    unit of a workload, the credits equal the workload's total (arrow heads; GNA query tiles)."""
    import numpy as np

    import bench
    import workloads as W
    from oracle import masks as OM
    w = W.c1()
    units = bench._oracle_plan("c1", w, np.random.default_rng(0))
    total = sum(run() for run, _, _ in units)
    s = w["shape"]
    kept = int((OM.arrow_block_classes_all(s, w["head_mode"], w["window"]) > 0).sum())
    assert total == 4.0 * s.block_q * s.block_k * s.d * kept
    v = W.video_case(1, 1, 16, (4, 8, 8), (2, 4, 4), (3, 5, 5), (1, 1, 1), 64, 5)
    units = bench._oracle_plan("c5f", v, np.random.default_rng(0))
    lay = OM.GnaLayout(16, (4, 8, 8), (2, 4, 4), (3, 5, 5), (1, 1, 1))
    cls = OM.gna_block_classes_separable(lay)
    sampled = sum(run() for run, _, _ in units)
    assert len(units) == 2 and 0 < sampled <= 4.0 * lay.bs * lay.bs * 64 * 2 * cls.shape[0]


def test_hbm_phase_bytes_match_the_stated_traffic():
    import bench
    # pooled selection at the FLUX-2048-like size reads Q and K once: 2 x 103.8 MB
    assert bench.select_bytes(1, 24, 16896, 128) == 2 * 24 * 16896 * 128 * 2
    assert abs(bench.select_bytes(1, 24, 16896, 128) / 1e6 - 207.6) < 0.1
    # the video workload (256 text + 16x48x80, no padding): the forward permute of Q, K, V and
    # the inverse of O together move about 3.03 GB
    n = 256 + 16 * 48 * 80
    fw = bench.permute_bytes(1, 24, n, n, 128, 3)
    bw = bench.unpermute_bytes(1, 24, n, 128, 1)
    assert fw == 3 * 24 * 2 * n * 128 * 2 and bw == 24 * 2 * n * 128 * 2
    assert abs((fw + bw) / 1e9 - 3.03) < 0.01
    # padding rows are written by the forward permute but not read back by the inverse
    assert bench.permute_bytes(1, 1, 100, 128, 8, 1) == (100 + 128) * 8 * 2
    assert bench.unpermute_bytes(1, 1, 100, 8, 1) == 2 * 100 * 8 * 2


def test_phase_bandwidth_reports_median_and_fraction(monkeypatch):
    import bench
    import torch

    class FakeEvent:  # stands in for torch.cuda.Event: successive pairs are 2 ms apart
        t = 0.0

        def __init__(self, enable_timing=True):
            self.at = None

        def record(self):
            FakeEvent.t += 1.0
            self.at = FakeEvent.t

        def elapsed_time(self, other):
            return 2.0
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    calls = []
    out = bench.phase_bandwidth([("p", lambda: calls.append(1), 13_102_800)], torch.zeros(4), 6551.4, reps=5,
                                warmup=2)
    assert len(calls) == 7
    p = out["p"]
    assert p["ms"] == 2.0 and p["algorithmic_bytes"] == 13_102_800
    assert abs(p["gbs"] - 6.5514) < 1e-9 and abs(p["frac_of_hbm"] - 0.001) < 1e-12


def test_gna_useful_pairs_equal_the_token_mask():
    import bench
    from oracle import masks as OM
    cases = [(5, (3, 5, 6), (2, 2, 4), (2, 3, 3), (1, 1, 1)), (0, (7, 9), (4, 4), (3, 4), (1, 2)),
             (3, (10,), (4,), (4,), (2,)), (17, (4, 6, 10), (2, 4, 8), (4, 4, 8), (2, 4, 8)),
             (9, (6, 6), (4, 4), (6, 6), (3, 3))]
    for n_text, grid, tile, window, stride in cases:
        lay = OM.GnaLayout(n_text, grid, tile, window, stride)
        assert int(OM.gna_token_mask(lay).sum()) == bench.gna_useful_pairs(n_text, grid, window), grid
    # the video workload: 61,440 video queries x (3,072 + 256) keys + 256 text rows x 61,696
    assert 4 * 128 * 24 * bench.gna_useful_pairs(256, (16, 48, 80), (8, 16, 24)) == 2_706_634_702_848
