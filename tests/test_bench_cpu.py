"""bench.py without a GPU: the module imports, and the reference arm (the
float64 oracle on the host cores) prints the contract's keys for the forward
and the backward pass on a small workload."""
import argparse
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    # imported under its own name, so that spawned oracle processes can import
    # the worker function the same way
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    return importlib.import_module("bench")


def test_forward_traffic_hash_is_computable(bench):
    assert len(bench.kernel_source_hash()) == 64
    bench.log("bench helpers load")


@pytest.mark.parametrize("pass_", ["forward", "backward"])
def test_reference_arm_line(bench, pass_):
    args = argparse.Namespace(gpus=1, steps=3, warmup=3, impl="reference",
                              workload="dcnv3_f32_1x14x14x64_g4", pass_=pass_)
    line = bench.run_reference(args)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert ("backward" in line["metric"]) == (pass_ == "backward")


def test_gpus_flag_never_silently_runs_one_rank(bench):
    import subprocess
    import sys
    import torch
    args = argparse.Namespace(gpus=2, steps=3, warmup=3, impl="b200",
                              workload="dcnv3_f32_1x14x14x64_g4", pass_="forward", algo="auto")
    cmd = bench.torchrun_command(args, 29511)
    assert "--nproc-per-node=2" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[cmd.index("--gpus") + 1] == "2"
    if torch.cuda.device_count() < 2:
        # without two GPUs the benchmark refuses instead of running one rank
        env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK")}
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                            "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                           env=env, timeout=300)
        assert r.returncode != 0
        assert "2 are needed" in r.stderr
        assert r.stdout.strip() == ""
        # a launcher that started a different number of ranks is refused too
        env["WORLD_SIZE"] = "1"
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                            "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                           env=env, timeout=300)
        assert r.returncode != 0 and "does not match" in r.stderr


def test_cpu_baseline_reports_single_and_all_core_rates(bench):
    import gen
    w = gen.WORKLOADS["dcnv3_f32_1x14x14x64_g4"]
    pool = bench.start_oracle_pool(2)
    try:
        line = bench.cpu_baseline(w, budget_s=0.4, pool=pool, cores=2)
    finally:
        pool.close()
        pool.join()
    assert line["cores"] == 2 and line["kind"] == "oracle"
    assert line["value"] == line["all_core_value"] > 0
    assert line["single_thread_value"] > 0
    assert "2 processes" in line["sample"]
