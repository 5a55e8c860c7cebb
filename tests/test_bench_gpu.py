"""bench.py on the GPU, on small shapes: the default five-call line and the
vocabulary-parallel mode (one rank, so its collectives are skipped) each
print one complete JSON line whose kernels ran and whose numbers are
consistent (tokens per step over the timed device time)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    out = subprocess.run([sys.executable, "bench.py", "--steps", "3", "--warmup", "3",
                          "--no-cpu-baseline", *extra], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_bench_five_call_line_small_shape():
    d = _run("--workload", "lmhead_512x1024x8192")
    assert d["config"]["workload"] == "lmhead_512x1024x8192"
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["n_gpus"] == 1
    assert abs(d["value"] - 512 / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    assert set(d["kernels"]) == {"lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw"}
    assert d["roofline"]["kernel"] in d["kernels"] and d["roofline"]["frac"] > 0
    assert d["fused_step"]["value"] > 0 and d["e2e"]["value"] > 0
    assert d["e2e"]["d2h_bytes_per_step"] == 512 * 4 * 4 + 512 * 1024 * 4
    assert d["gpu_launches"] == 5 * 3


def test_bench_vocab_parallel_mode_one_rank():
    d = _run("--workload", "lmhead_256x512x4096", "--parallel", "vocab")
    assert d["scaling"] == "strong" and d["config"]["parallelism"] == "vocab1"
    assert d["config"]["vocab_rows_per_rank"] == 4096 and d["config"]["nccl_ranks"] == 1
    assert abs(d["value"] - 256 / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    assert d["roofline"]["kernel"] in ("lmhead_fwd", "lmhead_bwd_dx", "lmhead_bwd_dw",
                                       "ce_fwd_shard", "ce_bwd_shard")
    assert d["e2e"]["value"] > 0 and d["gpu_launches"] == 6 * 3
