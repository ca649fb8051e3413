"""Pins of the oracle's fused shared expert (EPConfig fused_shared_expert;
DistributedEPCombine fused_shared_expert): one more expert after the routed
ones, which every token goes through with weight 1.  With all routed weights
zero the layer is the shared expert's dense FFN, computed here with torch's
own F.linear / F.silu on ml_dtypes-decoded BF16 operands; the shared term
adds to the routed layer; and a shared expert equal to a routed expert e
doubles the routed contribution of a token whose only routed slot is e."""

import ml_dtypes
import numpy as np
import torch
import torch.nn.functional as TF

from oracle import moe as O


def _bf16(a):
    return np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def _dec(a):
    return np.asarray(a).view(ml_dtypes.bfloat16).astype(np.float64)


def _problem(seed, M=10, H=256, I=128, E=4, k=2):
    rng = np.random.default_rng(seed)
    inp = dict(x=_bf16(rng.standard_normal((M, H)) * 0.5),
               w13=_bf16(rng.standard_normal((E + 1, 2 * I, H)) * 0.1),
               w2=_bf16(rng.standard_normal((E + 1, H, I)) * 0.1))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(M)]).astype(np.int64)
    w = rng.uniform(0.1, 1.0, (M, k)).astype(np.float32)
    p = dict(format="bf16", hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k, activation_clamp=10.0)
    return p, inp, idx, w


def test_slots_layout():
    idx = np.array([[2, 0], [1, -1]])
    w = np.array([[0.25, 0.75], [0.5, 0.0]], np.float32)
    si, sw = O.shared_expert_slots(idx, w, 3)
    assert np.array_equal(si, [[2, 0, 3], [1, -1, 3]])
    assert np.array_equal(sw, np.array([[0.25, 0.75, 1.0], [0.5, 0.0, 1.0]], np.float32))


def test_zero_routed_weights_give_the_dense_shared_ffn():
    p, inp, idx, w = _problem(1)
    M, H, I, E = inp["x"].shape[0], p["hidden"], p["intermediate_hidden"], p["num_experts"]
    si, sw = O.shared_expert_slots(idx, np.zeros_like(w), E)
    r = O.moe_forward(dict(p, shared_expert=1), inp, si, sw)
    x = torch.from_numpy(_dec(inp["x"]))
    a = TF.linear(x, torch.from_numpy(_dec(inp["w13"][E])))
    g, u = torch.clamp(a[:, :I], max=10.0), torch.clamp(a[:, I:], -10.0, 10.0)
    h = (TF.silu(g) * u).to(torch.float32).to(torch.bfloat16).to(torch.float64)
    ref = TF.linear(h, torch.from_numpy(_dec(inp["w2"][E]))).numpy()
    assert np.allclose(r["out_f64"], ref, rtol=1e-10, atol=1e-14)


def test_shared_term_adds_to_the_routed_layer():
    p, inp, idx, w = _problem(2)
    E = p["num_experts"]
    routed = O.moe_forward(p, inp, idx, w)["out_f64"]
    si, sw = O.shared_expert_slots(idx, w, E)
    both = O.moe_forward(dict(p, shared_expert=1), inp, si, sw)["out_f64"]
    si0, sw0 = O.shared_expert_slots(idx, np.zeros_like(w), E)
    shared = O.moe_forward(dict(p, shared_expert=1), inp, si0, sw0)["out_f64"]
    assert np.allclose(both, routed + shared, rtol=1e-12, atol=1e-14)


def test_shared_copy_of_a_routed_expert_doubles_it():
    p, inp, idx, w = _problem(3, k=1)
    E = p["num_experts"]
    e = int(idx[0, 0])
    inp = dict(inp)
    inp["w13"] = inp["w13"].copy()
    inp["w2"] = inp["w2"].copy()
    inp["w13"][E] = inp["w13"][e]
    inp["w2"][E] = inp["w2"][e]
    ones = np.ones_like(w)
    routed = O.moe_forward(p, inp, idx, ones)["out_f64"]
    si, sw = O.shared_expert_slots(idx, ones, E)
    both = O.moe_forward(dict(p, shared_expert=1), inp, si, sw)["out_f64"]
    assert np.allclose(both[0], 2.0 * routed[0], rtol=1e-12, atol=1e-14)
