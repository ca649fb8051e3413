"""Edge cases of the CUDA path against the oracle: one layer (one workspace)
called with different token counts in turn, through the single launch and
the chain; tokens whose every slot is skipped (their output is exactly
zero); and the shared expert together with per-token NVFP4 activations."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _problem(fmt, M, H, I, E, k, **kw):
    p = dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k, format=fmt,
             routing="softmax", activation_clamp=10.0)
    p.update(kw)
    return p


def _slice(d, host, M):
    """The first M tokens of a drawn problem (x rows, scales, routing)."""
    dd, hh = dict(d), dict(host)
    for key in ("x", "topk_idx", "topk_weights", "x_row_scale"):
        if dd.get(key) is not None:
            dd[key] = dd[key][:M].contiguous()
            hh[key] = hh[key][:M]
    if dd.get("x_scale") is not None and dd["x_scale"].dim() == 2:
        dd["x_scale"] = dd["x_scale"][:M].contiguous()
        hh["x_scale"] = hh["x_scale"][:M]
    return dd, hh


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor"])
def test_one_workspace_for_several_token_counts(fmt):
    """A layer sized for 512 tokens serves 512, then 37, then 300, then 512
    again (the workspace layout moves with the count); every call matches
    the oracle, in the single launch and in the chain."""
    Mmax, H, I, E, k = 512, 512, 256, 6, 2
    p = _problem(fmt, Mmax, H, I, E, k)
    d, host = S.make(p, seed=41)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    for M in (512, 37, 300, 512):
        pm = dict(p, num_tokens=M)
        dm, hm = _slice(d, host, M)
        ref = S.oracle_reference(pm, hm, np.arange(M))
        fused = S.run_fused(L, dm)
        assert L.status() == api.MOE_OK
        S.check_layout_exact(fused.lay_h, O.permute(hm["topk_idx"], E), M, k)
        S.check_against_oracle(pm, hm, fused, np.arange(M), label=f"{fmt}/M={M}/fused", ref=ref)
        chain = S.run_chain(L, dm)
        assert L.status() == api.MOE_OK
        S.check_against_oracle(pm, hm, chain, np.arange(M), label=f"{fmt}/M={M}/chain", ref=ref)


@pytest.mark.parametrize("fmt,regime", [("bf16", "small_m"), ("fp8", "large_m"), ("nvfp4", "large_m"),
                                        ("mxfp8", "large_m"), ("nvfp4", "small_m"), ("mxfp8", "small_m"),
                                        ("fp8_tensor", "small_m")])
def test_tokens_with_every_slot_skipped_are_zero(fmt, regime):
    M, H, I, E, k = 96, 512, 256, 4, 3
    p = _problem(fmt, M, H, I, E, k, tile_regime=regime)
    d, host = S.make(p, seed=42)
    idx = host["topk_idx"].copy()
    idx[::7, :] = -1          # every slot of these tokens skipped
    idx[3::7, 1:] = -1        # all but one slot skipped
    host["topk_idx"] = idx
    d["topk_idx"] = torch.from_numpy(idx).cuda()
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    tokens = np.arange(M)
    ref = S.oracle_reference(p, host, tokens)
    for res in (S.run_fused(L, d), S.run_chain(L, d)):
        assert L.status() == api.MOE_OK
        assert np.all(res.out[::7] == 0.0)
        S.check_against_oracle(p, host, res, tokens, label=f"skipped/{fmt}", ref=ref)


def test_shared_expert_with_per_token_nvfp4_scales():
    """The shared expert and the rowwise NVFP4 activations together: the
    rowwise scale is looked up by token for the shared slot too."""
    M, H, I, E, k = 200, 512, 256, 5, 2
    p = _problem("nvfp4", M, H, I, E, k, shared_expert=1, act="bf16")
    d, host = S.make(p, seed=43)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    xb = d["x_bf16"].view(torch.bfloat16)
    codes, scales, rowwise = L.quantize_rowwise(xb)
    torch.cuda.synchronize()
    q = O.quantize_nvfp4_rowwise(S.bf16_to_np(xb))
    assert np.array_equal(codes.cpu().numpy(), q["codes"]) and np.array_equal(scales.cpu().numpy(), q["scales"])
    d["x"], d["x_scale"], d["x_row_scale"] = codes, scales, rowwise
    host["x"], host["x_scale"] = q["codes"], q["scales"]
    host["x_row_scale"] = rowwise.cpu().numpy().view(np.uint16)
    host["topk_idx"], host["topk_weights"] = O.shared_expert_slots(host["topk_idx"], host["topk_weights"], E)
    d["topk_idx"], d["topk_weights"] = L.shared_slots(d["topk_idx"], d["topk_weights"])
    tokens = np.arange(M)
    ref = S.oracle_reference(p, host, tokens)
    for res in (S.run_fused(L, d), S.run_chain(L, d)):
        assert L.status() == api.MOE_OK
        S.check_against_oracle(p, host, res, tokens, label="shared+rowwise", ref=ref)
