"""Host-side checks of bench.py that need no GPU: the reference arm's JSON
line (the CPU oracle timed on a small sample) carries every key of the
line format, and the committed DRAM-traffic summary is read only for its
own workload and kernel sources."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_complete_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--cpu-sample", "2", "--workload",
                          "lmhead_1024x4096x32768"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["config"]["workload"] == "lmhead_1024x4096x32768"
    assert d["config"]["tokens_per_step"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_sample_shrinks_with_the_step_count():
    # the default 200 + 10 steps take a few tokens per step; a short run the full 16
    assert bench.reference_tokens_per_step(200, 10, 256) == 4
    assert bench.reference_tokens_per_step(5, 1, 256) == 16
    assert bench.reference_tokens_per_step(5, 1, 2) == 2
    assert bench.reference_tokens_per_step(100000, 0, 256) == 1
    # a token of the large-vocabulary workload costs ~3.9x one of the mid-size one
    assert bench.reference_tokens_per_step(20, 5, 256, 4096, 128256) == 9


def test_default_workload_is_the_large_vocabulary_lm_head(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    args = bench.parse()
    assert args.workload == "lmhead_4096x4096x128256"
    cfg = bench.lmhead_config(args.workload)
    assert (cfg.M, cfg.K, cfg.V, cfg.ignore_frac) == (4096, 4096, 128256, 0.01)
    mid = bench.lmhead_config("lmhead_1024x4096x32768")
    assert (mid.M, mid.ignore_frac) == (1024, 0.02)
    other = bench.lmhead_config("lmhead_4096x4096x32768")
    assert (other.M, other.K, other.V, other.dist) == (4096, 4096, 32768, "normal")


def test_traffic_summary_is_tied_to_workload_and_sources():
    assert bench.committed_traffic("no_such_workload") == {}
    p = os.path.join(ROOT, "profiles", "traffic_lmhead_1024x4096x32768.md")
    txt = open(p).read()
    recorded = txt.rsplit("kernel-source-hash:", 1)[1].split()[0]
    got = bench.committed_traffic("lmhead_1024x4096x32768")
    if recorded == bench.kernel_source_hash():
        assert set(got) >= {"lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw"}
        assert all(v > 0 for v in got.values())
    else:
        assert got == {}
