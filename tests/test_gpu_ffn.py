"""GPU parity of the expert FFN (moe_ffn, moe_combine, moe_fused) against the
oracle, per format, on small problems that span several tiles with ragged
tails and on the full-size workloads (sampled tokens)."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import formats as F
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _small(fmt, M, H, I, E, k, routing="softmax", clamp=10.0):
    return dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k,
                format=fmt, routing=routing, activation_clamp=clamp)


def _weights(d):
    return {k: d.get(k) for k in ("w13", "w13_scale", "w2", "w2_scale", "gate_up_expert_scales",
                                  "down_expert_scales", "c_input_scales")}


SMALL = [
    # fmt, M, H, I, E, k
    ("bf16", 16, 256, 128, 8, 2),      # the tiny BF16 workload
    ("bf16", 300, 512, 384, 4, 2),     # several m tiles per expert, ragged tails
    ("fp8", 200, 512, 256, 6, 3),
    ("fp8", 256, 2048, 768, 64, 6),    # the FP8 block-scaled workload
    ("nvfp4", 200, 512, 256, 6, 3),
    ("nvfp4", 333, 1024, 512, 5, 2),
]


@pytest.mark.parametrize("fmt,M,H,I,E,k", SMALL)
def test_ffn_parity_small(fmt, M, H, I, E, k):
    p = _small(fmt, M, H, I, E, k)
    d, host = S.make(p, seed=1)
    L = layer.MoELayer(p, _weights(d), device=S.device())
    lay, acc, inter, out = S.run_unfused(L, d)
    assert L.status() == api.MOE_OK
    lay_h = lay.host()
    S.check_layout_exact(lay_h, O.permute(host["topk_idx"], E), M, k)
    stats = S.check_ffn_against_oracle(p, host, lay_h, acc, inter, out, np.arange(M), label=fmt)
    print(fmt, stats)
    # the one-call path gives the same result (up to FP32 summation order)
    out2 = L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"])
    torch.cuda.synchronize()
    a, b = S.bf16_to_np(out), S.bf16_to_np(out2)
    assert np.all(S.close_bf16(a, b, 1e-2 * S.rms(a)))


@pytest.mark.parametrize("regime", ["large_m", "small_m"])
@pytest.mark.parametrize("fmt,M,H,I,E,k", [c for c in SMALL if c[0] != "nvfp4"])
def test_ffn_parity_both_tile_regimes(fmt, M, H, I, E, k, regime):
    """Both GEMM tile regimes (128 routed rows x 256 weight rows, and the
    swapped operands with 32 routed rows) on every BF16 / FP8 case, through
    the unfused chain and the single launch."""
    p = _small(fmt, M, H, I, E, k)
    p["tile_regime"] = regime
    d, host = S.make(p, seed=3)
    L = layer.MoELayer(p, _weights(d), device=S.device())
    assert api.tile_regime(L.problem(M)) == regime
    lay, acc, inter, out = S.run_unfused(L, d)
    assert L.status() == api.MOE_OK
    lay_h = lay.host()
    S.check_layout_exact(lay_h, O.permute(host["topk_idx"], E), M, k)
    stats = S.check_ffn_against_oracle(p, host, lay_h, acc, inter, out, np.arange(M), label=f"{fmt}/{regime}")
    print(fmt, regime, stats)
    out2 = L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"])
    torch.cuda.synchronize()
    assert L.status() == api.MOE_OK
    a, b = S.bf16_to_np(out), S.bf16_to_np(out2)
    assert np.all(S.close_bf16(a, b, 1e-2 * S.rms(a)))


@pytest.mark.parametrize("fmt,regime", [("bf16", "large_m"), ("fp8", "large_m"), ("nvfp4", "large_m"),
                                        ("bf16", "small_m"), ("fp8", "small_m")])
def test_staged_mode_and_deterministic_combine(fmt, regime):
    M, H, I, E, k = 96, 512, 256, 4, 3
    p = _small(fmt, M, H, I, E, k)
    p["tile_regime"] = regime
    d, host = S.make(p, seed=2)
    L = layer.MoELayer(p, _weights(d), device=S.device())
    lay = L.permute(d["topk_idx"])
    staged, _ = L.ffn(d["x"], d.get("x_scale"), lay, d["topk_weights"], out_mode=api.MOE_OUT_STAGED)
    out_s = L.combine(lay, d["topk_weights"], staged, api.MOE_IN_STAGED, M)
    out_s2 = L.combine(lay, d["topk_weights"], staged, api.MOE_IN_STAGED, M)
    acc, _ = L.ffn(d["x"], d.get("x_scale"), lay, d["topk_weights"])
    out_a = L.combine(lay, None, acc, api.MOE_IN_ACCUMULATED, M)
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_s2)          # staged combine is deterministic
    a, s = S.bf16_to_np(out_a), S.bf16_to_np(out_s)
    assert np.all(S.close_bf16(a, s, 1e-2 * S.rms(a)))
    ref = O.moe_forward(p, host, host["topk_idx"], host["topk_weights"])
    want = F.bf16_decode(ref["out_bf16"])
    # loose end-to-end bound (re-quant flips may move a few tokens; the split
    # parity of the accumulate path above is the strict check)
    assert np.all(S.close_bf16(s, want, 3 * S.TOL[fmt] * S.rms(want)))


def test_clamp_active_bf16():
    """Large weights push > 20% of g and u past +-c; the clamp must match."""
    M, H, I, E, k = 64, 256, 128, 2, 1
    p = _small("bf16", M, H, I, E, k, clamp=0.1)
    d, host = S.make(p, seed=3)
    d["w13"] = (d["w13"].view(torch.bfloat16).float() * 40).to(torch.bfloat16).view(torch.int16)
    host["w13"] = d["w13"].cpu().view(torch.int16).numpy().view(np.uint16)
    L = layer.MoELayer(p, _weights(d), device=S.device())
    lay, acc, inter, out = S.run_unfused(L, d)
    xh = O.decode_x("bf16", host["x"], None, H)
    g = xh @ O.decode_weight("bf16", host["w13"], None, 0, 2 * I, H).T
    assert np.mean(np.abs(g) > 0.1) > 0.2
    S.check_ffn_against_oracle(p, host, lay.host(), acc, inter, out, np.arange(M), label="clamp")


def test_skipped_and_duplicate_slots():
    M, H, I, E, k = 40, 256, 128, 3, 3
    p = _small("bf16", M, H, I, E, k)
    d, host = S.make(p, seed=4)
    idx = host["topk_idx"].copy()
    idx[::3, 1] = -1
    idx[1::5, 2] = idx[1::5, 0]
    host["topk_idx"] = idx
    d["topk_idx"] = torch.from_numpy(idx).cuda()
    L = layer.MoELayer(p, _weights(d), device=S.device())
    lay, acc, inter, out = S.run_unfused(L, d)
    S.check_ffn_against_oracle(p, host, lay.host(), acc, inter, out, np.arange(M), label="skip/dup")


def test_all_tokens_one_expert_and_single_expert():
    for E, k in ((1, 1), (4, 1)):
        M, H, I = 260, 512, 256
        p = _small("nvfp4", M, H, I, E, k)
        d, host = S.make(p, seed=5)
        idx = np.zeros((M, k), np.int64)
        host["topk_idx"] = idx
        d["topk_idx"] = torch.from_numpy(idx).cuda()
        host["topk_weights"] = np.ones((M, k), np.float32)
        d["topk_weights"] = torch.ones((M, k), device="cuda")
        L = layer.MoELayer(p, _weights(d), device=S.device())
        lay, acc, inter, out = S.run_unfused(L, d)
        S.check_ffn_against_oracle(p, host, lay.host(), acc, inter, out, np.arange(M), label=f"E={E}")


@pytest.mark.parametrize("name,ntok", [("tiny_bf16", 16), ("fp8_block", 64), ("nvfp4_decode", 24),
                                       ("nvfp4_prefill", 12), ("fp8_prefill_routed", 12)])
def test_full_size_workloads_sampled(name, ntok):
    """The full-size workloads in the launch configuration the benchmark uses
    (moe_fused), checked on sampled tokens."""
    p = workloads.problem(name)
    d, host = S.make(p, seed=0, on_gpu_generation=True)
    L = layer.MoELayer(p, _weights(d), device=S.device())
    M, k = p["num_tokens"], p["num_topk"]
    if p["routing"] == "logits":
        idx, w = L.route(d["logits"], d["bias"])
        torch.cuda.synchronize()
        ridx, rw = O.route(host["logits"], host["bias"], k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        wg = w.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(wg - rw) <= 1e-6 * rw + 1e-7)
        d["topk_idx"], d["topk_weights"] = idx, w
        # the oracle keeps its own routing weights
        host["topk_idx"], host["topk_weights"] = ridx, rw.astype(np.float32)
        out_f = L.forward(d["x"], d.get("x_scale"), logits=d["logits"], bias=d["bias"])
    else:
        out_f = L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"])
    torch.cuda.synchronize()
    assert L.status() == api.MOE_OK
    lay, acc, inter, out = S.run_unfused(L, d)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(M, size=min(ntok, M), replace=False))
    stats = S.check_ffn_against_oracle(p, host, lay.host(), acc, inter, out, tokens, label=name)
    print(name, stats)
    a, b = S.bf16_to_np(out), S.bf16_to_np(out_f)
    assert np.all(S.close_bf16(a, b, 1e-2 * S.rms(a)))
