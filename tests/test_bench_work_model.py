"""The algorithmic work the bench divides by (its roofline numerator),
against figures derived by hand from the layer's definition.  CPU only."""

import bench
from mixture_experts_routed_03_b200 import workloads


def test_fp8_block_work():
    p = workloads.problem("fp8_block")          # M 256, H 2048, I 768, E 64, k 6
    w = bench.work_model(p, num_active=64)
    R = 256 * 6
    assert w["layer"]["flops"] == 6 * R * 2048 * 768                       # 14.5 GFLOP
    per_expert = (2 * 768 * 2048 + (2 * 768 // 128) * (2048 // 128) * 4    # W13 codes + FP32 block scales
                  + 2048 * 768 + (2048 // 128) * (768 // 128) * 4)         # W2 codes + scales
    x = 256 * (2048 + 2048 // 128 * 4)                                     # E4M3 x + per-128 FP32 scales
    out = 256 * 2048 * 2                                                    # BF16 out
    assert per_expert == 4_719_744
    assert w["layer"]["bytes"] == 64 * per_expert + x + out                 # 303.6 MB


def test_nvfp4_decode_work_counts_active_experts_only():
    p = workloads.problem("nvfp4_decode")       # M 64, H 7168, I 2048, E 256, k 8
    w10 = bench.work_model(p, num_active=10)
    w20 = bench.work_model(p, num_active=20)
    per_expert = (2 * 2048 * 7168 // 2 + 2 * 2048 * 7168 // 16               # W13 e2m1 + E4M3 per 16
                  + 7168 * 2048 // 2 + 7168 * 2048 // 16)                   # W2
    assert w20["layer"]["bytes"] - w10["layer"]["bytes"] == 10 * per_expert
    assert w10["layer"]["flops"] == 6 * 64 * 8 * 7168 * 2048


def test_routed_logits_are_counted():
    p = workloads.problem("fp8_prefill_routed")
    w = bench.work_model(p, num_active=128)
    q = dict(p, routing="given")
    wq = bench.work_model(q, num_active=128)
    assert w["layer"]["bytes"] - wq["layer"]["bytes"] == p["num_tokens"] * p["num_experts"] * 4
