"""Pins of the oracle's per-token dynamic NVFP4 quantisation (EPConfig,
nvfp4_dyn_global_scales: each token quantised against 2688 / rowmax, the
scale's BF16 inverse travelling with the token) and of the rowwise dequant in
the FFN.  Checked against closed forms, exhaustive nearest-code searches over
all 16 E2M1 and all 256 E4M3 codes decoded by ml_dtypes, and a dense FFN
computed with torch."""

import ml_dtypes
import numpy as np
import torch
import torch.nn.functional as TF

from oracle import formats as Fm
from oracle import moe as O

E2M1_VALUES = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64) \
    if hasattr(ml_dtypes, "float4_e2m1fn") else None
E4M3_VALUES = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def _bf16_vals(a):
    return np.asarray(a, np.float32).astype(ml_dtypes.bfloat16).astype(np.float32)


def _nearest_even(values, grid_codes, grid_vals, x):
    """Code of the nearest finite grid value to x (ties to the even code), by
    exhaustive search; values beyond the largest magnitude saturate."""
    finite = np.isfinite(grid_vals)
    cand = grid_codes[finite]
    vals = grid_vals[finite]
    d = np.abs(vals - x)
    best = d.min()
    ties = cand[d == best]
    # among equally near codes prefer the one with the even (zero) last mantissa bit
    even = [c for c in ties if (c & 1) == 0]
    return int(even[0] if even else ties[0])


def test_rowmax_element_is_six_with_block_scale_448():
    """Closed form: the token's largest magnitude sits in a block whose scale
    is e4m3(rowmax / (6 * rowmax / 2688)) = 448 and codes to +-6."""
    rng = np.random.default_rng(1)
    x = _bf16_vals(rng.standard_normal((8, 256)) * rng.uniform(0.01, 100, (8, 1)))
    q = O.quantize_nvfp4_rowwise(x)
    codes = Fm.fp4_unpack(q["codes"], 256)
    for t in range(8):
        i = int(np.argmax(np.abs(x[t])))
        assert q["scales"][t, i // 16] == 0x7E                       # 448
        assert Fm.e2m1_decode(codes[t, i]) == (6.0 if x[t, i] > 0 else -6.0)


def test_rowwise_scale_is_bf16_of_rowmax_over_2688():
    rng = np.random.default_rng(2)
    x = _bf16_vals(rng.standard_normal((16, 128)) * 3)
    q = O.quantize_nvfp4_rowwise(x)
    want = (np.abs(x).max(axis=1).astype(np.float32) / np.float32(2688.0)).astype(np.float32)
    assert np.array_equal(q["rowwise"], want.astype(ml_dtypes.bfloat16).view(np.uint16))
    assert 448.0 * 6.0 == O.NVFP4_ROW_RANGE


def test_codes_and_scales_are_nearest_by_exhaustive_search():
    """Every block scale is the nearest E4M3 value to amax / (6 G) and every
    element code the nearest E2M1 value to x / (sf G) (FP32 steps as stated),
    found by searching all codes decoded with ml_dtypes."""
    if E2M1_VALUES is None:
        return
    rng = np.random.default_rng(3)
    x = _bf16_vals(rng.standard_normal((4, 64)) * rng.uniform(0.1, 10, (4, 64)))
    q = O.quantize_nvfp4_rowwise(x)
    codes = Fm.fp4_unpack(q["codes"], 64)
    for t in range(4):
        G = np.float32(np.float32(np.abs(x[t]).max()) / np.float32(2688.0))
        for b in range(4):
            blk = x[t, 16 * b: 16 * b + 16]
            u = np.float32(np.float32(np.abs(blk).max()) / np.float32(np.float32(6.0) * G))
            sf_code = _nearest_even(None, np.arange(128, dtype=np.int64), E4M3_VALUES[:128], float(u))
            assert q["scales"][t, b] == sf_code
            sf = np.float32(E4M3_VALUES[sf_code])
            inv = np.float32(np.float32(1.0) / np.float32(sf * G))
            for j in range(16):
                v = float(np.float32(blk[j] * inv))
                c = _nearest_even(None, np.arange(16, dtype=np.int64), E2M1_VALUES, v)
                got = int(codes[t, 16 * b + j])
                # +0 and -0 are the same value
                assert E2M1_VALUES[got] == E2M1_VALUES[c], (t, b, j, v, got, c)


def test_round_trip_within_half_a_step():
    rng = np.random.default_rng(4)
    x = _bf16_vals(rng.standard_normal((32, 256)))
    q = O.quantize_nvfp4_rowwise(x)
    xhat = O.decode_x("nvfp4", q["codes"], q["scales"], 256, row_scale=q["rowwise"])
    G = np.abs(x).max(axis=1, keepdims=True) / 2688.0
    sf = np.repeat(Fm.e4m3_decode(q["scales"]), 16, axis=1)
    # half the largest E2M1 step (2, between 4 and 6) at the block's scale,
    # plus the BF16 rounding of the rowwise scale (2^-9 relative)
    bound = 1.0 * sf * G + np.abs(x) * 2.0 ** -8
    assert np.all(np.abs(xhat - x) <= bound + 1e-30)


def test_zero_token():
    x = np.zeros((2, 64), np.float32)
    x[1, 5] = 1.0
    q = O.quantize_nvfp4_rowwise(x)
    assert not q["codes"][0].any() and not q["scales"][0].any() and q["rowwise"][0] == 0
    assert q["rowwise"][1] != 0


def test_rowwise_dense_special_case_with_torch():
    """E = 1, k = 1 with per-token quantised activations: the layer equals a
    dense FFN on the ml_dtypes-decoded operands with each row times its
    rowwise scale."""
    if E2M1_VALUES is None:
        return
    rng = np.random.default_rng(5)
    M, H, I = 4, 256, 128
    xf = _bf16_vals(rng.standard_normal((M, H)))
    q = O.quantize_nvfp4_rowwise(xf)
    w13 = rng.integers(0, 256, (1, 2 * I, H // 2), dtype=np.uint8)
    w13s = np.array(rng.uniform(0.5, 1.5, (1, 2 * I, H // 16)), np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    w2 = rng.integers(0, 256, (1, H, I // 2), dtype=np.uint8)
    w2s = np.array(rng.uniform(0.5, 1.5, (1, H, I // 16)), np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    a1, a2, G = np.float32(0.003), np.float32(0.02), np.float32(0.04)
    inp = dict(x=q["codes"], x_scale=q["scales"], x_row_scale=q["rowwise"], w13=w13, w13_scale=w13s, w2=w2,
               w2_scale=w2s, gate_up_expert_scales=np.array([a1]), down_expert_scales=np.array([a2]),
               c_input_scales=np.array([G]))
    p = dict(format="nvfp4", hidden=H, intermediate_hidden=I, num_experts=1, num_topk=1, activation_clamp=10.0)
    r = O.moe_forward(p, inp, np.zeros((M, 1), np.int64), np.ones((M, 1), np.float32), keep_intermediate=True)

    def dec4(packed, sc):
        nib = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)
        vals = nib.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        return vals * np.repeat(sc.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)
    rs = q["rowwise"].view(ml_dtypes.bfloat16).astype(np.float64)[:, None]
    xhat = dec4(q["codes"], q["scales"]) * rs
    g_u = torch.from_numpy(xhat) @ torch.from_numpy(dec4(w13[0], w13s[0]) * float(a1)).T
    g, u = g_u[:, :I], g_u[:, I:]
    h = (TF.silu(torch.clamp(g, max=10.0)) * torch.clamp(u, -10.0, 10.0)).float()
    # the re-quantised intermediate the oracle used, fed to the down projection
    hh = np.stack([O.dequant_intermediate("nvfp4", r["intermediate"][(t, 0)]["codes"][None],
                                          r["intermediate"][(t, 0)]["scales"][None], I)[0] for t in range(M)])
    assert np.allclose(np.stack([r["intermediate"][(t, 0)]["h32"] for t in range(M)]), h.numpy(), rtol=1e-5, atol=1e-6)
    ref = torch.from_numpy(hh) @ torch.from_numpy(dec4(w2[0], w2s[0]) * float(a2)).T
    assert np.allclose(r["out_f64"], ref.numpy(), rtol=1e-9, atol=1e-12)
