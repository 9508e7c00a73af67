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
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


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
