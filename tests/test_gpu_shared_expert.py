"""GPU parity of the fused shared expert (EPConfig fused_shared_expert;
DistributedEPCombine fused_shared_expert): the shared expert rides in the
same grouped GEMMs as one more expert that every token takes with weight 1.
Chain and single launch, every format and both tile regimes, against the
oracle with the split-parity checks; and in-kernel routing from logits,
which writes the shared column itself."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _problem(fmt, M, H, I, E, k, routing="softmax", regime="auto"):
    return dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k, format=fmt,
                routing=routing, activation_clamp=10.0, tile_regime=regime, shared_expert=1)


@pytest.mark.parametrize("fmt,M,H,I,E,k,regime", [
    ("bf16", 200, 512, 256, 6, 2, "large_m"),
    ("bf16", 40, 512, 256, 8, 2, "small_m"),
    ("fp8", 300, 1024, 384, 8, 3, "large_m"),
    ("fp8", 64, 1024, 384, 16, 4, "small_m"),
    ("nvfp4", 200, 512, 256, 6, 3, "large_m"),
    ("nvfp4", 48, 512, 256, 12, 3, "small_m"),
    ("mxfp8", 260, 1024, 384, 5, 2, "large_m"),
    ("mxfp8", 64, 1024, 384, 16, 2, "small_m"),
    ("fp8_tensor", 200, 512, 256, 6, 2, "large_m"),
    ("fp8_tensor", 40, 512, 256, 8, 2, "small_m"),
])
def test_shared_expert_parity(fmt, M, H, I, E, k, regime):
    p = _problem(fmt, M, H, I, E, k, regime=regime)
    d, host = S.make(p, seed=11)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    assert api.tile_regime(L.problem(M)) == regime
    # routing [M, k] -> [M, k + 1] with the shared column, on each side by its own code
    host["topk_idx"], host["topk_weights"] = O.shared_expert_slots(host["topk_idx"], host["topk_weights"], E)
    d["topk_idx"], d["topk_weights"] = L.shared_slots(d["topk_idx"], d["topk_weights"])
    assert np.array_equal(d["topk_idx"].cpu().numpy(), host["topk_idx"])
    ref_perm = O.permute(host["topk_idx"], E + 1)
    tokens = np.arange(M)
    ref = S.oracle_reference(p, host, tokens)
    chain = S.run_chain(L, d)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(chain.lay_h, ref_perm, M, k + 1)
    st_c = S.check_against_oracle(p, host, chain, tokens, label=f"shared/{fmt}/chain", ref=ref)
    fused = S.run_fused(L, d)
    assert L.status() == api.MOE_OK
    S.check_layout_exact(fused.lay_h, ref_perm, M, k + 1)
    st_f = S.check_against_oracle(p, host, fused, tokens, label=f"shared/{fmt}/fused", ref=ref)
    # the shared expert got every token
    assert int(fused.lay_h["expert_counts"][E]) == M
    print(fmt, regime, "chain", st_c, "fused", st_f)


def test_shared_expert_with_in_kernel_routing():
    M, H, I, E, k = 512, 1024, 384, 16, 4
    p = _problem("fp8", M, H, I, E, k, routing="logits")
    d, host = S.make(p, seed=12)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    fused = S.run_fused(L, d, from_logits=True)
    assert L.status() == api.MOE_OK
    ridx, rw = O.route(host["logits"], host["bias"], k)
    sidx, sw = O.shared_expert_slots(ridx, rw.astype(np.float32), E)
    gidx, gw = fused.route
    assert np.array_equal(gidx, sidx)
    assert np.all(np.abs(gw.astype(np.float64) - sw) <= 1e-6 * sw + 1e-7)
    host["topk_idx"], host["topk_weights"] = sidx, sw
    S.check_layout_exact(fused.lay_h, O.permute(sidx, E + 1), M, k + 1)
    tokens = np.arange(0, M, 3)
    print("shared/logits", S.check_against_oracle(p, host, fused, tokens, label="shared/logits"))
    # moe_route writes the same [M, k + 1] routing
    idx2, w2 = L.route(d["logits"], d["bias"])
    torch.cuda.synchronize()
    assert np.array_equal(idx2.cpu().numpy(), sidx)
    assert torch.equal(w2.cpu(), torch.from_numpy(gw))
