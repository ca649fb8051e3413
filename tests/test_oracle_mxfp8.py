"""Pins of the oracle's MXFP8 format (MoEActivationPack: E4M3 values with
UE8M0 scales per 32 along K): the UE8M0 decode against ml_dtypes, the
intermediate's per-32 re-quant against closed forms and an exhaustive
nearest-code search, and the layer against a dense FFN computed with torch on
ml_dtypes-decoded operands."""

import ml_dtypes
import numpy as np
import torch
import torch.nn.functional as TF

from oracle import formats as Fm
from oracle import moe as O

E4M3_VALUES = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_ue8m0_decode_all_codes_match_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = Fm.ue8m0_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def _h(seed, rows=6, I=256):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((rows, I)) * np.exp(rng.uniform(-20, 20, (rows, I // 32))).repeat(32, axis=1)
    h[0, :32] = 0.0                      # an all-zero block
    h[1, 32:64] = 1e-40                  # a subnormal block: its exponent clamps at -127
    return h.astype(np.float32)


def test_requant_scale_is_floor_log2_amax_minus_8():
    h = _h(1)
    rq = O.requant("mxfp8", h)
    blk = np.abs(h.astype(np.float64)).reshape(h.shape[0], -1, 32).max(axis=2)
    X = np.where(blk > 0, np.floor(np.log2(np.where(blk > 0, blk, 1))) - 8, -127)
    assert np.array_equal(rq["scales"], np.clip(X, -127, 127).astype(np.int64) + 127)
    # the block's largest element lands in [256, 448] (448 when it saturates)
    codes = rq["codes"].reshape(h.shape[0], -1, 32)
    for r in range(h.shape[0]):
        for b in range(h.shape[1] // 32):
            if blk[r, b] >= 2.0 ** -100:
                mx = np.max(np.abs(E4M3_VALUES[codes[r, b]]))
                assert 256.0 <= mx <= 448.0


def test_requant_codes_are_nearest_by_exhaustive_search():
    h = _h(2, rows=3)
    rq = O.requant("mxfp8", h)
    finite = np.isfinite(E4M3_VALUES)
    cand = np.arange(256)[finite]
    vals = E4M3_VALUES[finite]
    for r in range(3):
        for b in range(h.shape[1] // 32):
            X = int(rq["scales"][r, b]) - 127
            for j in range(32):
                v = float(h[r, 32 * b + j]) * 2.0 ** -X
                d = np.abs(vals - np.clip(v, -448.0, 448.0))
                near = cand[d == d.min()]
                even = [c for c in near if (c & 1) == 0]
                want = E4M3_VALUES[even[0] if even else near[0]]
                assert E4M3_VALUES[rq["codes"][r, 32 * b + j]] == want, (r, b, j, v)


def test_zero_block():
    h = np.zeros((1, 64), np.float32)
    h[0, 40] = 3.0
    rq = O.requant("mxfp8", h)
    assert rq["scales"][0, 0] == 0 and not rq["codes"][0, :32].any()
    assert rq["scales"][0, 1] == 127 + 1 - 8   # floor(log2 3) = 1


def _mx(rng, shape):
    """Random MXFP8 operand: E4M3 codes and UE8M0 scales per 32."""
    codes = (rng.standard_normal(shape) * 64).clip(-448, 448).astype(np.float32).astype(ml_dtypes.float8_e4m3fn)
    sc = rng.integers(120, 126, shape[:-1] + (shape[-1] // 32,), dtype=np.uint8)
    return codes.view(np.uint8), sc


def test_mxfp8_dense_special_case_with_torch():
    """E = 1, k = 1: the MXFP8 layer equals a dense FFN on operands decoded
    with ml_dtypes, with the intermediate re-quantised per 32 by the closed
    form of the scale and ml_dtypes' E4M3 cast."""
    rng = np.random.default_rng(9)
    M, H, I = 4, 256, 128
    x, xs = _mx(rng, (M, H))
    w13, w13s = _mx(rng, (1, 2 * I, H))
    w2, w2s = _mx(rng, (1, H, I))
    inp = dict(x=x, x_scale=xs, w13=w13, w13_scale=w13s, w2=w2, w2_scale=w2s)
    p = dict(format="mxfp8", hidden=H, intermediate_hidden=I, num_experts=1, num_topk=1, activation_clamp=10.0)
    r = O.moe_forward(p, inp, np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32))

    def dec(c, s):
        v = c.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
        return v * np.repeat(s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64), 32, axis=-1)
    g_u = torch.from_numpy(dec(x, xs)) @ torch.from_numpy(dec(w13[0], w13s[0])).T
    g, u = g_u[:, :I], g_u[:, I:]
    h = (TF.silu(torch.clamp(g, max=10.0)) * torch.clamp(u, -10.0, 10.0)).float().numpy()
    hb = h.astype(np.float64).reshape(M, I // 32, 32)
    amax = np.abs(hb).max(axis=2, keepdims=True)
    X = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1))) - 8, -127)
    q = (hb * 2.0 ** -X).clip(-448, 448).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    hh = (q * 2.0 ** X).reshape(M, I)
    ref = torch.from_numpy(hh) @ torch.from_numpy(dec(w2[0], w2s[0])).T
    assert np.allclose(r["out_f64"], ref.numpy(), rtol=1e-9, atol=1e-12)
