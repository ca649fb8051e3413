"""Pins of the oracle's FP8 per-tensor format (MoEActivationPack: E4M3
values with one FP32 dequantisation scale for the tensor; one FP32 scale per
expert matrix; the intermediate re-quantised against the per-expert static
c_input_scales G).  Checked against ml_dtypes' E4M3 cast, an exhaustive
nearest-code search, saturation, an exact power-of-two rescaling of the
scales, and a dense FFN computed with torch."""

import ml_dtypes
import numpy as np
import torch
import torch.nn.functional as TF

from oracle import moe as O

E4M3_VALUES = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_requant_with_unit_scale_is_the_e4m3_cast():
    rng = np.random.default_rng(1)
    h = (rng.standard_normal((4, 256)) * 50).astype(np.float32)
    rq = O.requant("fp8_tensor", h, np.float32(1.0))
    want = h.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(rq["codes"], want)
    assert np.array_equal(rq["hhat"], want.view(ml_dtypes.float8_e4m3fn).astype(np.float64))


def test_requant_codes_are_nearest_by_exhaustive_search_and_saturate():
    rng = np.random.default_rng(2)
    G = np.float32(0.37)
    h = (rng.standard_normal((2, 128)) * 60).astype(np.float32)
    h[0, :4] = [1000.0, -1000.0, 448.0 * 0.37 * 1.05, 0.0]
    rq = O.requant("fp8_tensor", h, G)
    finite = np.isfinite(E4M3_VALUES)
    cand, vals = np.arange(256)[finite], E4M3_VALUES[finite]
    inv = np.float32(np.float32(1.0) / G)
    for r in range(2):
        for j in range(128):
            v = float(np.float32(h[r, j] * inv))
            d = np.abs(vals - np.clip(v, -448.0, 448.0))
            near = cand[d == d.min()]
            even = [c for c in near if (c & 1) == 0]
            assert E4M3_VALUES[rq["codes"][r, j]] == E4M3_VALUES[even[0] if even else near[0]]
    assert E4M3_VALUES[rq["codes"][0, 0]] == 448.0 and E4M3_VALUES[rq["codes"][0, 1]] == -448.0
    assert np.allclose(rq["hhat"], E4M3_VALUES[rq["codes"]] * float(G))


def _problem(rng, M=5, H=256, I=128, E=2):
    e4 = lambda shape: (rng.standard_normal(shape) * 64).clip(-448, 448).astype(np.float32) \
        .astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    inp = dict(x=e4((M, H)), x_scale=np.array([0.0137], np.float32),
               w13=e4((E, 2 * I, H)), w13_scale=rng.uniform(0.5, 1.5, E).astype(np.float32) * 3e-4,
               w2=e4((E, H, I)), w2_scale=rng.uniform(0.5, 1.5, E).astype(np.float32) * 3e-4,
               c_input_scales=rng.uniform(1.0, 1.2, E).astype(np.float32) * (100.0 / 448.0))
    p = dict(format="fp8_tensor", hidden=H, intermediate_hidden=I, num_experts=E, num_topk=1,
             activation_clamp=10.0)
    return p, inp


def test_power_of_two_rescaling_of_the_scales_is_exact():
    rng = np.random.default_rng(3)
    p, inp = _problem(rng)
    idx = rng.integers(0, 2, (5, 1))
    w = np.ones((5, 1), np.float32)
    a = O.moe_forward(p, inp, idx, w)["out_f64"]
    inp2 = dict(inp, x_scale=inp["x_scale"] * np.float32(4.0), w13_scale=inp["w13_scale"] * np.float32(0.25))
    assert np.array_equal(O.moe_forward(p, inp2, idx, w)["out_f64"], a)


def test_dense_special_case_with_torch():
    rng = np.random.default_rng(4)
    p, inp = _problem(rng, E=1)
    M, H, I = 5, 256, 128
    r = O.moe_forward(p, inp, np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32))
    dec = lambda c: c.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    xs, ws1, ws2, G = (float(inp["x_scale"][0]), float(inp["w13_scale"][0]), float(inp["w2_scale"][0]),
                       np.float32(inp["c_input_scales"][0]))
    a = TF.linear(torch.from_numpy(dec(inp["x"]) * xs), torch.from_numpy(dec(inp["w13"][0]) * ws1))
    g, u = torch.clamp(a[:, :I], max=10.0), torch.clamp(a[:, I:], -10.0, 10.0)
    h = (TF.silu(g) * u).to(torch.float32).numpy()
    q = (h * np.float32(np.float32(1.0) / G)).astype(np.float32).clip(-448, 448).astype(ml_dtypes.float8_e4m3fn)
    hh = q.astype(np.float64) * float(G)
    ref = TF.linear(torch.from_numpy(hh), torch.from_numpy(dec(inp["w2"][0]) * ws2)).numpy()
    assert np.allclose(r["out_f64"], ref, rtol=1e-9, atol=1e-12)
