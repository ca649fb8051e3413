"""Pins of the oracle's clamped "swigluoai" activation (Struct_mega_ffn_ep_
combine_send, clamp_activation): h = min(g, c) * sigmoid(alpha * min(g, c))
* (clamp(u, -c, c) + 1).  Checked against the already pinned clamped SwiGLU
(alpha = 1 splits into two of its values), special cases with exact results
(u = -1; the clamps), the large-alpha limit (the ReLU gate), and a dense FFN
built from torch's F.linear and F.silu, whose silu of alpha * g over alpha is
the gate's own sigmoid-weighted form."""

import ml_dtypes
import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import moe as O


def _vals(seed, n=4000, scale=4.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(n) * scale, rng.standard_normal(n) * scale


def test_up_minus_one_gives_zero():
    g, _ = _vals(1)
    assert np.array_equal(O.swigluoai(g, -np.ones_like(g), 10.0, 1.702), np.zeros_like(g))


def test_alpha_one_splits_into_clamped_swiglu_terms():
    """With alpha = 1 the +1 bias adds a second SwiGLU term with u = 1."""
    g, u = _vals(2)
    c = 3.0
    got = O.swigluoai(g, u, c, 1.0)
    want = O.clamped_swiglu(g, u, c) + O.clamped_swiglu(g, np.ones_like(u), c)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_clamps():
    g, u = _vals(3, scale=20.0)
    c = 5.0
    assert np.array_equal(O.swigluoai(g, u, c, 1.702),
                          O.swigluoai(np.minimum(g, c), np.clip(u, -c, c), np.inf, 1.702))
    # the gate is clamped from above only
    assert O.swigluoai(np.array([-30.0]), np.array([0.0]), c, 1.0)[0] == pytest.approx(-30.0 / (1 + np.exp(30.0)))


def test_large_alpha_is_a_relu_gate():
    g, u = _vals(4)
    g = g[np.abs(g) > 0.05]
    u = u[: g.shape[0]]
    c = 6.0
    got = O.swigluoai(g, u, c, 1e4)
    want = np.maximum(np.minimum(g, c), 0.0) * (np.clip(u, -c, c) + 1.0)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("alpha,clamp", [(1.702, 7.0), (0.5, 10.0), (3.0, float("inf"))])
def test_dense_ffn_special_case_with_torch(alpha, clamp):
    """E = 1, k = 1, BF16: the layer equals a dense FFN with the gate
    silu(alpha g) / alpha computed by torch."""
    rng = np.random.default_rng(5)
    M, H, I = 6, 256, 128
    bf = lambda a: np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)
    dec = lambda a: a.view(ml_dtypes.bfloat16).astype(np.float64)
    x, w13, w2 = bf(rng.standard_normal((M, H))), bf(rng.standard_normal((1, 2 * I, H)) * 0.15), \
        bf(rng.standard_normal((1, H, I)) * 0.1)
    p = dict(format="bf16", hidden=H, intermediate_hidden=I, num_experts=1, num_topk=1, activation_clamp=clamp,
             activation="swigluoai", activation_alpha=alpha)
    r = O.moe_forward(p, dict(x=x, w13=w13, w2=w2), np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32))
    a = TF.linear(torch.from_numpy(dec(x)), torch.from_numpy(dec(w13[0])))
    g, u = a[:, :I], a[:, I:]
    if np.isfinite(clamp):
        g, u = torch.clamp(g, max=clamp), torch.clamp(u, -clamp, clamp)
    h = (TF.silu(alpha * g) / alpha * (u + 1.0)).to(torch.float32).to(torch.bfloat16).to(torch.float64)
    ref = TF.linear(h, torch.from_numpy(dec(w2[0]))).numpy()
    assert np.allclose(r["out_f64"], ref, rtol=1e-9, atol=1e-12)
    # and it differs from the plain clamped SwiGLU
    plain = O.moe_forward(dict(p, activation="swiglu"), dict(x=x, w13=w13, w2=w2), np.zeros((M, 1), np.int64),
                          np.ones((M, 1), np.float32))
    assert not np.allclose(plain["out_f64"], r["out_f64"])
