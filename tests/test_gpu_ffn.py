"""GPU parity of the expert FFN against the oracle, per format, through the
unfused chain (moe_permute / moe_ffn / moe_combine) and through the single
moe_fused launch -- whose layout, intermediate codes, FP32 accumulator and
output are read back from its workspace and held to the same split-parity
checks -- on small problems that span several tiles with ragged tails, and on
the full-size workloads in the launch configuration the benchmark times
(sampled tokens, plus whole-problem layout and routing checks)."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _small(fmt, M, H, I, E, k, routing="softmax", clamp=10.0, regime="auto"):
    return dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k,
                format=fmt, routing=routing, activation_clamp=clamp, tile_regime=regime)


def _check_both_paths(p, d, host, L, tokens, label):
    """The chain and the single launch, each against the oracle."""
    M, E, k = p["num_tokens"], p["num_experts"], p["num_topk"]
    ref_perm = O.permute(host["topk_idx"], E)
    ref = S.oracle_reference(p, host, tokens)
    chain = S.run_chain(L, d)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(chain.lay_h, ref_perm, M, k)
    st_c = S.check_against_oracle(p, host, chain, tokens, label=label + "/chain", ref=ref)
    fused = S.run_fused(L, d)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(fused.lay_h, ref_perm, M, k)
    st_f = S.check_against_oracle(p, host, fused, tokens, label=label + "/fused", ref=ref)
    print(label, "chain", st_c, "fused", st_f)
    return chain, fused


SMALL = [
    # fmt, M, H, I, E, k
    ("bf16", 16, 256, 128, 8, 2),      # the tiny BF16 workload
    ("bf16", 300, 512, 384, 4, 2),     # several m tiles per expert, ragged tails
    ("fp8", 200, 512, 256, 6, 3),
    ("fp8", 256, 2048, 768, 64, 6),    # the FP8 block-scaled workload
    ("fp8", 700, 1024, 384, 3, 2),     # several m and n tiles, ragged
    ("nvfp4", 200, 512, 256, 6, 3),
    ("nvfp4", 333, 1024, 512, 5, 2),
    ("mxfp8", 200, 512, 256, 6, 3),
    ("mxfp8", 700, 1024, 384, 3, 2),   # several m and n tiles, ragged
    ("fp8_tensor", 200, 512, 256, 6, 3),
    ("fp8_tensor", 700, 1024, 384, 3, 2),
]


@pytest.mark.parametrize("fmt,M,H,I,E,k", SMALL)
def test_ffn_parity_small(fmt, M, H, I, E, k):
    p = _small(fmt, M, H, I, E, k)
    d, host = S.make(p, seed=1)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    _check_both_paths(p, d, host, L, np.arange(M), fmt)


@pytest.mark.parametrize("regime", ["large_m", "small_m"])
@pytest.mark.parametrize("fmt,M,H,I,E,k", SMALL)
def test_ffn_parity_both_tile_regimes(fmt, M, H, I, E, k, regime):
    """Both GEMM tile regimes (128 routed rows x 256 weight rows, and the
    swapped operands with 32 routed rows) on every case of every format,
    through the chain and the single launch."""
    p = _small(fmt, M, H, I, E, k, regime=regime)
    d, host = S.make(p, seed=3)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    assert api.tile_regime(L.problem(M)) == regime
    _check_both_paths(p, d, host, L, np.arange(M), f"{fmt}/{regime}")


ALL_FMT_REGIMES = [(f, r) for r in ("large_m", "small_m") for f in ("bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor")]


@pytest.mark.parametrize("fmt,regime", ALL_FMT_REGIMES)
def test_staged_mode_and_deterministic_combine(fmt, regime):
    """Staged rows + the deterministic gather-combine meet the format's own
    tolerance; the combine gives the same bytes twice."""
    M, H, I, E, k = 96, 512, 256, 4, 3
    p = _small(fmt, M, H, I, E, k, regime=regime)
    d, host = S.make(p, seed=2)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    staged = S.run_chain(L, d, out_mode=api.MOE_OUT_STAGED)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(staged.lay_h, O.permute(host["topk_idx"], E), M, k)
    print(fmt, regime, "staged", S.check_against_oracle(p, host, staged, np.arange(M), label=f"staged/{fmt}"))
    lay = L.permute(d["topk_idx"])
    y, _ = L.ffn(d["x"], d.get("x_scale"), lay, d["topk_weights"], out_mode=api.MOE_OUT_STAGED)
    o1 = L.combine(lay, d["topk_weights"], y, api.MOE_IN_STAGED, M)
    o2 = L.combine(lay, d["topk_weights"], y, api.MOE_IN_STAGED, M)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("fmt,regime", ALL_FMT_REGIMES)
def test_clamp_active(fmt, regime):
    """Weights scaled up so that more than 20% of g and u pass +-c: the clamp
    is exercised in every format and tile regime, chain and single launch."""
    M, H, I, E, k = 160, 512, 256, 3, 2
    clamp = 0.5
    p = _small(fmt, M, H, I, E, k, clamp=clamp, regime=regime)
    d, host = S.make(p, seed=3)
    if fmt == "bf16":
        d["w13"] = (d["w13"].view(torch.bfloat16).float() * 60).to(torch.bfloat16).view(torch.int16)
        host["w13"] = d["w13"].cpu().view(torch.int16).numpy().view(np.uint16)
    elif fmt in ("fp8", "fp8_tensor"):
        d["w13_scale"] = d["w13_scale"] * 60
        host["w13_scale"] = d["w13_scale"].cpu().numpy()
    elif fmt == "mxfp8":
        d["w13_scale"] = d["w13_scale"] + 6        # x 64
        host["w13_scale"] = d["w13_scale"].cpu().numpy()
    else:
        d["gate_up_expert_scales"] = d["gate_up_expert_scales"] * 60
        host["gate_up_expert_scales"] = d["gate_up_expert_scales"].cpu().numpy()
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    # more than 20% of the gate and up values lie beyond the clamp
    xh = O.decode_x(fmt, host["x"], host.get("x_scale"), H)
    w13 = O.decode_weight(fmt, host["w13"], host.get("w13_scale"), 0, 2 * I, H)
    gu = xh @ w13.T
    if fmt == "nvfp4":
        gu = gu * float(host["gate_up_expert_scales"][0])
    assert np.mean(np.abs(gu[:, :I]) > clamp) > 0.2 and np.mean(np.abs(gu[:, I:]) > clamp) > 0.2
    _check_both_paths(p, d, host, L, np.arange(M), f"clamp/{fmt}/{regime}")


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor"])
def test_skipped_and_duplicate_slots(fmt):
    M, H, I, E, k = 40, 512, 256, 3, 3
    p = _small(fmt, M, H, I, E, k)
    d, host = S.make(p, seed=4)
    idx = host["topk_idx"].copy()
    idx[::3, 1] = -1
    idx[1::5, 2] = idx[1::5, 0]
    host["topk_idx"] = idx
    d["topk_idx"] = torch.from_numpy(idx).cuda()
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    _check_both_paths(p, d, host, L, np.arange(M), f"skip/dup/{fmt}")


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor"])
def test_all_tokens_one_expert_and_single_expert(fmt):
    for E, k in ((1, 1), (4, 1)):
        M, H, I = 260, 512, 256
        p = _small(fmt, M, H, I, E, k)
        d, host = S.make(p, seed=5)
        idx = np.zeros((M, k), np.int64)
        host["topk_idx"] = idx
        d["topk_idx"] = torch.from_numpy(idx).cuda()
        host["topk_weights"] = np.ones((M, k), np.float32)
        d["topk_weights"] = torch.ones((M, k), device="cuda")
        L = layer.MoELayer(p, S.weights_of(d), device=S.device())
        _check_both_paths(p, d, host, L, np.arange(M), f"one-expert/{fmt}/E={E}")


@pytest.mark.parametrize("name,ntok", [("tiny_bf16", 16), ("fp8_block", 96), ("nvfp4_decode", 24),
                                       ("nvfp4_prefill", 24), ("fp8_prefill_routed", 48),
                                       ("mxfp8_prefill_routed", 48), ("fp8_tensor_prefill_routed", 48)])
def test_full_size_workloads_sampled(name, ntok):
    """The full-size workloads through moe_fused, the launch the benchmark
    times: routing (in-kernel for the logits workload) and the whole layout
    bit-exact over all tokens, then split parity on sampled tokens; the chain
    gets the same split parity."""
    p = workloads.problem(name)
    d, host = S.make(p, seed=0, on_gpu_generation=True)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    M, E, k = p["num_tokens"], p["num_experts"], p["num_topk"]
    routed = p["routing"] == "logits"
    fused = S.run_fused(L, d, from_logits=routed)
    assert L.status() == api.MOE_OK
    if routed:
        ridx, rw = S.check_route(fused, host, k)
        # the oracle keeps its own routing; the chain runs on the same indices
        host["topk_idx"], host["topk_weights"] = ridx, rw.astype(np.float32)
        d["topk_idx"] = torch.from_numpy(ridx).cuda()
        d["topk_weights"] = torch.from_numpy(fused.route[1]).cuda()
    ref_perm = O.permute(host["topk_idx"], E)
    S.check_layout_exact(fused.lay_h, ref_perm, M, k)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(M, size=min(ntok, M), replace=False))
    ref = S.oracle_reference(p, host, tokens)
    st_f = S.check_against_oracle(p, host, fused, tokens, label=name + "/fused", ref=ref)
    chain = S.run_chain(L, d)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(chain.lay_h, ref_perm, M, k)
    st_c = S.check_against_oracle(p, host, chain, tokens, label=name + "/chain", ref=ref)
    print(name, "fused", st_f, "chain", st_c)
    # every token: the two paths agree (they differ only in FP32 summation order
    # and at rounding midpoints of the intermediate)
    a, b = chain.out, fused.out
    assert np.mean(~S.close_bf16(a, b, S.TOL[p["format"]] * S.rms(a))) < 1e-3


@pytest.mark.parametrize("fmt,regime", ALL_FMT_REGIMES)
def test_swigluoai_activation(fmt, regime):
    """The clamped swigluoai activation (Struct_mega_ffn_ep_combine_send,
    clamp_activation) with slope 1.702 and clamp 7, weights scaled so that
    the clamp is active: chain and single launch against the oracle."""
    M, H, I, E, k = 150, 512, 256, 4, 2
    p = dict(_small(fmt, M, H, I, E, k, clamp=7.0, regime=regime), activation="swigluoai",
             activation_alpha=1.702)
    d, host = S.make(p, seed=21)
    if fmt == "bf16":
        d["w13"] = (d["w13"].view(torch.bfloat16).float() * 40).to(torch.bfloat16).view(torch.int16)
        host["w13"] = d["w13"].cpu().view(torch.int16).numpy().view(np.uint16)
    elif fmt in ("fp8", "fp8_tensor"):
        d["w13_scale"] = d["w13_scale"] * 40
        host["w13_scale"] = d["w13_scale"].cpu().numpy()
    elif fmt == "mxfp8":
        d["w13_scale"] = d["w13_scale"] + 5        # x 32
        host["w13_scale"] = d["w13_scale"].cpu().numpy()
    else:
        d["gate_up_expert_scales"] = d["gate_up_expert_scales"] * 40
        host["gate_up_expert_scales"] = d["gate_up_expert_scales"].cpu().numpy()
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    assert api.tile_regime(L.problem(M)) == regime
    _check_both_paths(p, d, host, L, np.arange(M), f"swigluoai/{fmt}/{regime}")
