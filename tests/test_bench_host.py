"""Host-side logic of bench.py that needs no GPU: launch counts per step,
workload names, and the lookup of the profiled DRAM traffic, which must be
keyed to the kernel source it was taken on."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_launches_per_step(bench):
    assert bench.launches_per_step(1, 0) == 1   # in-kernel routing
    assert bench.launches_per_step(2, 1) == 1
    assert bench.launches_per_step(3, 0) == 7   # route, select, five streamed stages
    assert bench.launches_per_step(1, 2) == 7
    assert bench.launches_per_step(1, 0, d=4096) == 7  # the one-cluster reader runs d <= 2048


def test_workload_names(bench):
    assert bench.workload_name(1) == "qwen3_30b_a3b_layer_b1"
    assert bench.workload_name(16) == "qwen3_30b_a3b_layer_b16"


def test_traffic_is_keyed_to_the_source_hash(bench, monkeypatch):
    lines = [l for l in open(os.path.join(ROOT, "profiles", "traffic.txt")) if l.strip() and not l.startswith("#")]
    fields = dict(kv.split("=", 1) for kv in lines[0].split())
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: fields["source"])
    assert bench.profiled_traffic(fields["kernel"], fields["workload"]) == int(fields["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic(fields["kernel"], fields["workload"]) is None
    assert bench.profiled_traffic("no_such_kernel", fields["workload"]) is None
