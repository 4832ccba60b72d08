"""bench.py on the GPU at small sizes: the timed step's JSON line (the contract keys, a roofline
object for the W0' products, a live clock record) and the --vs-cublas comparison (the library's
block-diagonal and W0' products against cuBLAS on the same operands: block outputs bit-identical,
W0' outputs within bf16 rounding)."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=600, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout + out.stderr
    return json.loads(lines[0])


def test_bench_line_on_a_small_step():
    d = _bench("--workload", "llama1p3b_attn", "--tokens", "1024", "--steps", "3",
               "--warmup", "3", "--no-cpu-baseline")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "dtype", "config", "roofline", "e2e",
              "gpu_launches", "clocks"):
        assert k in d, k
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 3
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["achieved"] > 0 and r["launches"] == 2 * 3
    assert d["gpu_launches"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0


def test_vs_cublas_outputs_match():
    d = _bench("--vs-cublas", "--workload", "llama1p3b_attn", "--tokens", "2048", "--steps", "3",
               "--warmup", "1")
    assert d["mode"] == "vs_cublas"
    assert d["block_product_outputs_equal"] is True
    assert d["w0_outputs_max_rel_diff"] <= 1e-2
    for row in list(d["block_product"].values()) + list(d["w0_product"].values()):
        assert row["ms"] > 0
