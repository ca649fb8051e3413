"""The bench's CPU baseline times the oracle on a bounded sample, with all
host threads and with one.  CPU only, on the tiny workload."""

import bench
from mixture_experts_routed_03_b200 import workloads


def test_cpu_baseline_reports_all_threads_and_one():
    p = workloads.problem("tiny_bf16")
    d = workloads.make_inputs(p, seed=0, device="cpu")
    cb = bench.cpu_baseline(p, d, seconds=0.5)
    assert cb["kind"] == "oracle" and cb["unit"] == "routed_tokens/s"
    assert cb["value"] > 0 and cb["cores"] >= 1
    assert cb["one_thread"] is not None and cb["one_thread"]["cores"] == 1 and cb["one_thread"]["value"] > 0
