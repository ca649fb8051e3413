"""Per-token dynamic NVFP4 activations (EPConfig, nvfp4_dyn_global_scales):
the quantiser moe_quantize_nvfp4_rowwise against the oracle's, bit for bit,
and the layer fed with its codes, block scales and BF16 rowwise scales --
chain and single launch -- against the oracle's rowwise dequant."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import formats as F
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _bf16_activations(M, H, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((M, H), generator=g) * torch.exp(torch.randn((M, 1), generator=g) * 2)
    x[M // 3] = 0.0                       # an all-zero token
    x[M // 2, :H // 2] = 0.0              # zero blocks inside a token
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("M,H", [(37, 256), (300, 1024), (64, 7168)])
def test_quantizer_matches_oracle_bit_for_bit(M, H):
    x = _bf16_activations(M, H, seed=M + H)
    p = dict(num_tokens=M, hidden=H, intermediate_hidden=256, num_experts=4, num_topk=2, format="nvfp4",
             activation_clamp=10.0)
    dev = S.device()
    L = layer.MoELayer(p, dict(w13=torch.zeros((4, 512, H // 2), dtype=torch.uint8, device=dev),
                               w13_scale=torch.zeros((4, 512, H // 16), dtype=torch.uint8, device=dev),
                               w2=torch.zeros((4, H, 128), dtype=torch.uint8, device=dev),
                               w2_scale=torch.zeros((4, H, 16), dtype=torch.uint8, device=dev),
                               gate_up_expert_scales=torch.ones(4, device=dev),
                               down_expert_scales=torch.ones(4, device=dev),
                               c_input_scales=torch.ones(4, device=dev)), device=dev)
    codes, scales, rowwise = L.quantize_rowwise(x.to(dev))
    torch.cuda.synchronize()
    ref = O.quantize_nvfp4_rowwise(x.float().numpy())
    assert np.array_equal(scales.cpu().numpy(), ref["scales"])
    assert np.array_equal(rowwise.cpu().numpy().view(np.uint16), ref["rowwise"])
    got = codes.cpu().numpy()
    if not np.array_equal(got, ref["codes"]):
        # only a signed zero may differ: the same value
        g4, r4 = F.fp4_unpack(got, H), F.fp4_unpack(ref["codes"], H)
        diff = g4 != r4
        assert np.all(F.e2m1_decode(g4[diff]) == 0) and np.all(F.e2m1_decode(r4[diff]) == 0)


@pytest.mark.parametrize("name,M,regime", [("small", 200, "large_m"), ("small", 200, "small_m"),
                                           ("nvfp4_prefill", 512, "auto")])
def test_layer_with_rowwise_scales_matches_oracle(name, M, regime):
    if name == "small":
        p = dict(num_tokens=M, hidden=1024, intermediate_hidden=512, num_experts=6, num_topk=3, format="nvfp4",
                 routing="softmax", activation_clamp=10.0, tile_regime=regime)
    else:
        p = workloads.problem("nvfp4_prefill", num_tokens=M)
    d, host = S.make(p, seed=11)
    xb = _bf16_activations(M, p["hidden"], seed=5)
    ref_q = O.quantize_nvfp4_rowwise(xb.float().numpy())
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    codes, scales, rowwise = L.quantize_rowwise(xb.to(S.device()))
    torch.cuda.synchronize()
    d["x"], d["x_scale"], d["x_row_scale"] = codes, scales, rowwise
    host["x"], host["x_scale"], host["x_row_scale"] = ref_q["codes"], ref_q["scales"], ref_q["rowwise"]
    ref_perm = O.permute(host["topk_idx"], p["num_experts"])
    tokens = np.arange(M) if M <= 256 else np.sort(np.random.default_rng(0).choice(M, 48, replace=False))
    ref = S.oracle_reference(p, host, tokens)
    for run in (S.run_chain, S.run_fused):
        res = run(L, d)
        assert L.status() == api.MOE_OK
        S.check_layout_exact(res.lay_h, ref_perm, M, p["num_topk"])
        print(name, run.__name__, S.check_against_oracle(p, host, res, tokens, label=f"rowwise/{name}", ref=ref))


def test_rowwise_scale_rejected_for_other_formats():
    p = dict(num_tokens=16, hidden=256, intermediate_hidden=128, num_experts=4, num_topk=2, format="bf16",
             routing="softmax", activation_clamp=10.0)
    d, _ = S.make(p, seed=1)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    with pytest.raises(api.MoEError) as ei:
        L.forward(d["x"], None, topk_idx=d["topk_idx"], topk_weights=d["topk_weights"],
                  x_rowwise_scale=torch.ones(16, dtype=torch.int16, device="cuda"))
    assert ei.value.code == api.MOE_ERR_INVALID_ARG
