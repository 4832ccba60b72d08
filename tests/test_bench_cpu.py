"""The benchmark's JSON contract, checked on CPU through its reference arm (the float64 oracle on
the host cores): one line with the required keys, the same `config` object the GPU arm prints for
the workload, and an end-to-end record that moves no bytes."""
import json
import os
import subprocess
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-tokens", "8", *extra],
                         capture_output=True, text=True, timeout=300, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_line_has_the_contract_keys():
    d = _run()
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "8 of its 16384 tokens" in cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_config_is_the_gpu_arms_config(capsys, monkeypatch):
    """The reference arm prints the `config` object the GPU arm builds for the same workload
    (one function builds both). The oracle step itself is stubbed here (its timing is not the
    point; the first test runs it for real)."""
    sys.path.insert(0, ROOT)
    import bench
    import poetx_workloads as W
    monkeypatch.setattr(bench, "oracle_step_sample", lambda wl, T, nlin=1: (1.0, None))
    for key in ("llama8b_up_proj", "llama13b_layers", "llama8b_decoder", "llama1p3b_attn"):
        capsys.readouterr()
        assert bench.main(["--impl", "reference", "--workload", key, "--steps", "1",
                           "--warmup", "0", "--ref-tokens", "8"]) == 0
        lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
        d = json.loads(lines[-1])
        args = types.SimpleNamespace(tokens=None, all_linears=True, xq=False, xq_staged=False)
        assert d["config"] == bench.workload_config(W.WORKLOADS[key], args, 1), key


def test_cpu_baseline_reports_one_thread_blas_and_merge_extrapolation():
    """The oracle baseline carries the BLAS library, a 1-thread figure of the same sample and,
    for a workload with a merge period, the step plus one merge_reinit spread over the period,
    labelled as an extrapolation."""
    sys.path.insert(0, ROOT)
    import bench
    import poetx_workloads as W
    wl = W.WORKLOADS["tiny_fp32"]   # merge_reinit every step
    cb = bench.cpu_baseline(wl, 16, 1)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["blas"]
    assert cb["one_thread"]["value"] > 0 and "1 BLAS thread" in cb["one_thread"]["sample"]
    ex = cb["extrapolated_with_merge"]
    assert ex["merge_reinit_s"] > 0 and "extrapolated" in ex["label"]
    assert 0 < ex["value"] < cb["value"]


def test_other_configs_reports_a_failing_workload_without_failing():
    """The default run's other_configs: each workload runs in a process of its own, and one that
    fails (here an unknown workload name, rejected by the argument parser) is reported with its
    exit status instead of ending the benchmark."""
    sys.path.insert(0, ROOT)
    import bench
    saved = bench.OTHER_WORKLOADS
    bench.OTHER_WORKLOADS = ("no_such_workload",)
    try:
        out = bench.other_configs(types.SimpleNamespace(steps=1, warmup=3))
    finally:
        bench.OTHER_WORKLOADS = saved
    assert set(out) == {"no_such_workload"}
    assert out["no_such_workload"]["error"].startswith("exit 2")
