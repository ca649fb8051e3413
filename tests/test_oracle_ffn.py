"""Pins of the oracle's expert FFN and combine.

Special cases reduce the routed layer to a dense FFN computed with torch's
own library routines (``F.linear``, ``F.silu``, dtype casts), which share no
code with the oracle; algebraic properties (linearity in the router weights,
token-order equivariance, skipped and duplicated slots) pin the combine.
"""

import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import formats as Fm
from oracle import moe as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _bf16(a):
    return np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def _prob(fmt, H, I, E, k, clamp=10.0):
    return dict(format=fmt, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k,
                activation_clamp=clamp)


def test_ffn_bf16_worked_example():
    ex = GOLDEN["ffn_bf16"]
    for case in ex["cases"]:
        p = _prob("bf16", 2, 1, 1, 1, case["clamp"])
        inp = dict(x=_bf16([ex["x"]]), w13=_bf16([ex["w13"]]), w2=_bf16([ex["w2"]]))
        r = O.moe_forward(p, inp, np.array([[0]]), np.array([[ex["weight"]]], np.float32))
        assert np.array_equal(r["out_f64"][0], np.array(case["out"]))
        assert np.array_equal(Fm.bf16_decode(r["out_bf16"][0]), np.array(case["out"]))


def _torch_dense_ffn(xhat, w13hat, w2hat, I, clamp, requant_fn):
    """Dense per-token FFN with torch library ops in float64."""
    x = torch.from_numpy(xhat)
    a = TF.linear(x, torch.from_numpy(w13hat))
    g, u = a[:, :I], a[:, I:]
    if np.isfinite(clamp):
        g = torch.clamp(g, max=clamp)
        u = torch.clamp(u, -clamp, clamp)
    h = (TF.silu(g) * u).to(torch.float32)
    hh = requant_fn(h)
    return TF.linear(hh, torch.from_numpy(w2hat)).numpy()


@pytest.mark.parametrize("clamp", [10.0, 0.05, float("inf")])
def test_bf16_topk1_equals_dense_ffn(clamp):
    """top_k = 1 with weight 1: every token gets the dense FFN of its expert."""
    rng = np.random.default_rng(0)
    M, H, I, E = 12, 256, 128, 3
    x = _bf16(rng.standard_normal((M, H)) * 0.5)
    w13 = _bf16(rng.standard_normal((E, 2 * I, H)) * 0.1)
    w2 = _bf16(rng.standard_normal((E, H, I)) * 0.1)
    idx = rng.integers(0, E, (M, 1))
    p = _prob("bf16", H, I, E, 1, clamp)
    r = O.moe_forward(p, dict(x=x, w13=w13, w2=w2), idx, np.ones((M, 1), np.float32))
    for t in range(M):
        e = idx[t, 0]
        xhat = x[t:t + 1].view(ml_dtypes.bfloat16).astype(np.float64)
        w13h = w13[e].view(ml_dtypes.bfloat16).astype(np.float64)
        w2h = w2[e].view(ml_dtypes.bfloat16).astype(np.float64)
        ref = _torch_dense_ffn(xhat, w13h, w2h, I, clamp,
                               lambda h: h.to(torch.bfloat16).to(torch.float64))
        assert np.allclose(r["out_f64"][t], ref[0], rtol=1e-10, atol=1e-14)


def test_clamp_is_active_in_test_data():
    """The clamp test above really clamps: with c = 0.05 the result differs from c = inf."""
    rng = np.random.default_rng(0)
    g = rng.standard_normal(1000) * 3
    u = rng.standard_normal(1000) * 3
    assert not np.allclose(O.clamped_swiglu(g, u, 0.05), O.clamped_swiglu(g, u, np.inf))
    # values inside +-c are untouched
    small = np.array([0.01, -0.02])
    assert np.array_equal(O.clamped_swiglu(small, small, 0.05), O.clamped_swiglu(small, small, np.inf))
    # the gate is clamped from above only
    assert O.clamped_swiglu(np.array([-20.0]), np.array([1.0]), 1.0)[0] == pytest.approx(-20.0 / (1 + np.exp(20.0)))


def test_fp8_dense_special_case_with_torch_decode():
    """E = 1, k = 1: the FP8 layer equals a dense FFN on torch-decoded weights."""
    rng = np.random.default_rng(4)
    M, H, I = 5, 256, 128
    x = torch.from_numpy(np.clip(rng.standard_normal((M, H)) * 60, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
    w13 = torch.from_numpy(np.clip(rng.standard_normal((1, 2 * I, H)) * 60, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
    w2 = torch.from_numpy(np.clip(rng.standard_normal((1, H, I)) * 60, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
    xs = rng.uniform(0.5, 1.5, (M, H // 128)).astype(np.float32) / 60
    w13s = rng.uniform(0.5, 1.5, (1, 2 * I // 128, H // 128)).astype(np.float32) * 0.02 / 60
    w2s = rng.uniform(0.5, 1.5, (1, H // 128, I // 128)).astype(np.float32) * 0.02 / 60
    inp = dict(x=x.view(torch.uint8).numpy(), x_scale=xs, w13=w13.view(torch.uint8).numpy(),
               w13_scale=w13s, w2=w2.view(torch.uint8).numpy(), w2_scale=w2s)
    p = _prob("fp8", H, I, 1, 1)
    r = O.moe_forward(p, inp, np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32))

    def expand(s, rows, cols):
        return np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)[:rows, :cols]
    xhat = x.to(torch.float64).numpy() * np.repeat(xs, 128, axis=1)
    w13h = w13[0].to(torch.float64).numpy() * expand(w13s[0], 2 * I, H)
    w2h = w2[0].to(torch.float64).numpy() * expand(w2s[0], H, I)

    def fp8_requant(h):
        # per 128 block: s = amax / 448, codes by torch's float8 cast of h / s
        hb = h.reshape(h.shape[0], -1, 128)
        s = hb.abs().amax(dim=2, keepdim=True) / 448.0
        q = (hb * (1.0 / s)).to(torch.float8_e4m3fn).to(torch.float64)
        return (q * s.to(torch.float64)).reshape(h.shape)
    ref = _torch_dense_ffn(xhat, w13h, w2h, I, 10.0, fp8_requant)
    assert np.allclose(r["out_f64"], ref, rtol=1e-9, atol=1e-12)


def test_nvfp4_dense_special_case_with_ml_dtypes_decode():
    """E = 1, k = 1: the NVFP4 layer equals a dense FFN on ml_dtypes-decoded operands."""
    rng = np.random.default_rng(8)
    M, H, I = 4, 256, 128
    x = rng.integers(0, 256, (M, H // 2), dtype=np.uint8)
    xs = np.array(rng.uniform(0.5, 1.5, (M, H // 16)), np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    w13 = rng.integers(0, 256, (1, 2 * I, H // 2), dtype=np.uint8)
    w13s = np.array(rng.uniform(0.5, 1.5, (1, 2 * I, H // 16)), np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    w2 = rng.integers(0, 256, (1, H, I // 2), dtype=np.uint8)
    w2s = np.array(rng.uniform(0.5, 1.5, (1, H, I // 16)), np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    a1, a2, G = np.float32(0.003), np.float32(0.02), np.float32(0.04)
    inp = dict(x=x, x_scale=xs, w13=w13, w13_scale=w13s, w2=w2, w2_scale=w2s,
               gate_up_expert_scales=np.array([a1]), down_expert_scales=np.array([a2]),
               c_input_scales=np.array([G]))
    p = _prob("nvfp4", H, I, 1, 1)
    r = O.moe_forward(p, inp, np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32))

    def dec4(packed, sc):
        nib = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)
        vals = nib.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        return vals * np.repeat(sc.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)
    xhat = dec4(x, xs)
    w13h = dec4(w13[0], w13s[0]) * float(a1)
    w2h = dec4(w2[0], w2s[0]) * float(a2)

    def nv_requant(h):
        hb = h.numpy().reshape(h.shape[0], -1, 16)
        amax = np.abs(hb).max(axis=2, keepdims=True)
        sf = (amax / np.float32(6 * G)).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float32)
        v = (hb * (np.float32(1) / (sf * G).astype(np.float32))).astype(np.float32)
        q = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
        return torch.from_numpy((q * sf.astype(np.float64)).reshape(h.shape))
    ref = _torch_dense_ffn(xhat, w13h, w2h, I, 10.0, nv_requant)
    assert np.allclose(r["out_f64"], ref, rtol=1e-9, atol=1e-12)


def _random_bf16_problem(seed, M=10, H=256, I=128, E=4, k=3):
    rng = np.random.default_rng(seed)
    inp = dict(x=_bf16(rng.standard_normal((M, H)) * 0.5),
               w13=_bf16(rng.standard_normal((E, 2 * I, H)) * 0.1),
               w2=_bf16(rng.standard_normal((E, H, I)) * 0.1))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(M)])
    w = rng.uniform(0.1, 1.0, (M, k)).astype(np.float32)
    return _prob("bf16", H, I, E, k), inp, idx, w


def test_combine_linear_in_router_weights():
    p, inp, idx, _ = _random_bf16_problem(1)
    rng = np.random.default_rng(2)
    # multiples of 1/64 keep every weight and every pairwise sum exact in FP32
    w = (rng.integers(1, 64, idx.shape) / 64.0).astype(np.float32)
    w2 = (rng.integers(1, 64, idx.shape) / 64.0).astype(np.float32)
    a = O.moe_forward(p, inp, idx, w)["out_f64"]
    b = O.moe_forward(p, inp, idx, w2)["out_f64"]
    c = O.moe_forward(p, inp, idx, w + w2)["out_f64"]
    assert np.allclose(a + b, c, rtol=1e-12, atol=1e-14)


def test_combine_token_permutation_equivariant():
    p, inp, idx, w = _random_bf16_problem(3)
    perm = np.random.default_rng(0).permutation(idx.shape[0])
    a = O.moe_forward(p, inp, idx, w)["out_bf16"]
    inp2 = dict(inp, x=inp["x"][perm])
    b = O.moe_forward(p, inp2, idx[perm], w[perm])["out_bf16"]
    assert np.array_equal(a[perm], b)


def test_skipped_slot_contributes_nothing():
    p, inp, idx, w = _random_bf16_problem(5)
    idx2 = idx.copy()
    idx2[2, 1] = -1
    w0 = w.copy()
    w0[2, 1] = 0.0
    a = O.moe_forward(p, inp, idx2, w)["out_f64"]
    b = O.moe_forward(p, inp, idx, w0)["out_f64"]
    assert np.array_equal(a, b)


def test_duplicate_expert_slots_add():
    p, inp, idx, w = _random_bf16_problem(6, k=2)
    idx2 = idx.copy()
    idx2[:, 1] = idx2[:, 0]
    a = O.moe_forward(p, inp, idx2, w)["out_f64"]
    wsum = (w[:, :1].astype(np.float64) + w[:, 1:]).astype(np.float32)
    b = O.moe_forward(dict(p, num_topk=1), inp, idx2[:, :1], wsum)["out_f64"]
    assert np.allclose(a, b, rtol=1e-6, atol=1e-12)


def test_gate_up_order():
    """Gate rows are W13[:I], up rows W13[I:]: with up weights making u = 1 exactly,
    the layer output is W2 . bf16(silu(g)); swapping the halves changes it."""
    rng = np.random.default_rng(12)
    H, I = 256, 128
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    x[0, 1:] = rng.standard_normal(H - 1) * 0.5
    w13 = np.zeros((1, 2 * I, H), np.float32)
    w13[0, :I, :] = rng.standard_normal((I, H)) * 0.1
    w13[0, I:, 0] = 1.0                                   # u = x[0] = 1
    w2 = (rng.standard_normal((1, H, I)) * 0.1).astype(np.float32)
    p = _prob("bf16", H, I, 1, 1, float("inf"))
    inp = dict(x=_bf16(x), w13=_bf16(w13), w2=_bf16(w2))
    r = O.moe_forward(p, inp, np.zeros((1, 1), np.int64), np.ones((1, 1), np.float32))
    xh = Fm.bf16_decode(inp["x"])
    g = xh @ Fm.bf16_decode(inp["w13"][0, :I]).T
    h = torch.from_numpy(TF.silu(torch.from_numpy(g)).numpy().astype(np.float32)).to(torch.bfloat16).double().numpy()
    ref = h @ Fm.bf16_decode(inp["w2"][0]).T
    assert np.allclose(r["out_f64"], ref, rtol=1e-10, atol=1e-14)
    swapped = dict(inp, w13=np.concatenate([inp["w13"][:, I:], inp["w13"][:, :I]], axis=1))
    r2 = O.moe_forward(p, swapped, np.zeros((1, 1), np.int64), np.ones((1, 1), np.float32))
    assert not np.allclose(r2["out_f64"], ref)


def test_token_subset_matches_full():
    p, inp, idx, w = _random_bf16_problem(7)
    full = O.moe_forward(p, inp, idx, w)
    sub = O.moe_forward(p, inp, idx, w, tokens=[7, 2, 5])
    assert np.array_equal(sub["out_bf16"], full["out_bf16"][[7, 2, 5]])


def test_hhat_override_reproduces_own_intermediate():
    p, inp, idx, w = _random_bf16_problem(8)
    full = O.moe_forward(p, inp, idx, w, keep_intermediate=True)
    inter = full["intermediate"]

    def override(e, t, j):
        return np.stack([Fm.bf16_decode(inter[(int(a), int(b))]["codes"]) for a, b in zip(t, j)])
    again = O.moe_forward(p, inp, idx, w, hhat_override=override)
    assert np.array_equal(again["out_f64"], full["out_f64"])
