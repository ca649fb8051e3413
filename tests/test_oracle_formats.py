"""Pins of the oracle's element codecs against independent implementations.

E4M3 / E2M1 / BF16 are checked exhaustively (every code) and on every
midpoint between neighbouring representable values against ml_dtypes and
torch casts, and against a brute-force nearest-value search -- none of which
shares code with ``oracle.formats``.
"""

import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _nearest_even(values, table_vals, table_codes, mant_bits_of_code):
    """Brute force: nearest entry of a finite code table, ties to the even mantissa."""
    out = []
    for v in values:
        d = np.abs(table_vals - v)
        best = np.min(d)
        cand = [c for c, dv in zip(table_codes, d) if dv == best]
        even = [c for c in cand if mant_bits_of_code(c) % 2 == 0]
        out.append((even or cand)[0])
    return np.array(out)


def test_e4m3_decode_all_codes_vs_ml_dtypes():
    c = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(c)
    ref = c.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    # the field decoder (small arrays) and the table path (large) agree
    assert np.array_equal(F.e4m3_decode(np.tile(c, 3))[:256][m], ours[m])
    assert F.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert F.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9


def test_e4m3_encode_midpoints_and_random_vs_casts():
    fin = np.unique(F.e4m3_decode(np.arange(256, dtype=np.uint8)))
    fin = fin[~np.isnan(fin)]
    mids = (fin[1:] + fin[:-1]) / 2
    rng = np.random.default_rng(7)
    vals = np.concatenate([fin, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                           rng.standard_normal(50000) * 60, rng.standard_normal(5000) * 1e-2])
    vals = vals.astype(np.float32)
    vals = vals[np.abs(vals) < 448]
    ours = F.e4m3_encode(vals)
    ref_ml = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    nz = vals != 0
    assert np.array_equal(ours[nz], ref_ml[nz])
    assert np.array_equal(ours[nz], ref_t[nz])


def test_e4m3_encode_saturates_and_nan():
    v = np.array([448.0, 449.0, 464.0, 500.0, 1e30, -1e30, np.inf, -np.inf], np.float32)
    assert list(F.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert F.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_e4m3_encode_brute_force_small():
    codes = [c for c in range(0x7F)]                       # positive finite codes
    vals = F.e4m3_decode(np.array(codes, np.uint8))
    rng = np.random.default_rng(3)
    probe = np.concatenate([rng.uniform(0, 448, 3000), rng.uniform(0, 0.05, 1000),
                            (vals[1:] + vals[:-1]) / 2]).astype(np.float32)
    bf = _nearest_even(probe.astype(np.float64), vals, codes, lambda c: c & 7)
    assert np.array_equal(F.e4m3_encode(probe), bf.astype(np.uint8))


def test_e2m1_decode_all_codes_vs_ml_dtypes():
    n = np.arange(16, dtype=np.uint8)
    ref = n.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(F.e2m1_decode(n), ref)
    assert np.array_equal(F.e2m1_decode(np.tile(n, 4))[:16], ref)


def test_e2m1_encode_vs_ml_dtypes_and_brute_force():
    mags = F.e2m1_decode(np.arange(8))
    mids = (mags[1:] + mags[:-1]) / 2
    rng = np.random.default_rng(5)
    vals = np.concatenate([mags, -mags, mids, -mids, rng.uniform(-6, 6, 20000),
                           np.nextafter(mids, 0), np.nextafter(mids, 10)]).astype(np.float32)
    ours = F.e2m1_encode(vals)
    ref = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(F.e2m1_decode(ours), F.e2m1_decode(ref))
    pos = vals[~np.signbit(vals)]
    bf = _nearest_even(pos.astype(np.float64), mags, list(range(8)), lambda c: c & 1)
    assert np.array_equal(F.e2m1_encode(pos), bf.astype(np.uint8))
    sat = F.e2m1_encode(np.array([6.0, 7.0, 100.0, -50.0], np.float32))
    assert list(F.e2m1_decode(sat)) == [6.0, 6.0, 6.0, -6.0]


def test_fp4_pack_roundtrip_low_nibble_first():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    packed = F.fp4_pack(codes)
    assert list(packed[0]) == [0x21, 0x43, 0x0F]
    assert np.array_equal(F.fp4_unpack(packed, 6), codes)


def test_bf16_vs_ml_dtypes_and_torch():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(100000), rng.standard_normal(1000) * 1e-30,
                        [0.0, -0.0, 1.0, 3.0e38]]).astype(np.float32)
    ours = F.bf16_encode(v)
    assert np.array_equal(ours, v.astype(ml_dtypes.bfloat16).view(np.uint16))
    assert np.array_equal(ours, torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(F.bf16_decode(ours), v.astype(ml_dtypes.bfloat16).astype(np.float64))


def test_requant_nvfp4_worked_example():
    ex = GOLDEN["requant_nvfp4"]
    h = np.array([ex["h"]], np.float32)
    rq = O.requant("nvfp4", h, ex["G"])
    assert F.e4m3_decode(rq["scales"])[0, 0] == ex["sf"]
    assert np.array_equal(rq["hhat"][0], np.array(ex["hhat"]))


def test_requant_fp8_worked_example():
    ex = GOLDEN["requant_fp8"]
    h = np.zeros((1, 128), np.float32)
    h[0, :4] = ex["h_head"]
    rq = O.requant("fp8", h, None)
    assert rq["scales"][0, 0] == ex["s"]
    assert np.array_equal(rq["hhat"][0, :4], np.array(ex["hhat_head"]))
    assert np.all(rq["hhat"][0, 4:] == 0)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_requant_nearest_code_brute_force(fmt):
    """Each code is the nearest representable value of h / scale (ties to even)."""
    rng = np.random.default_rng(2)
    I = 256
    h = (rng.standard_normal((4, I)) * rng.uniform(0.01, 30, (4, 1))).astype(np.float32)
    h[3, :128] = 0.0                                       # an all-zero block
    G = 0.37
    rq = O.requant(fmt, h, G)
    if fmt == "fp8":
        codes = list(range(0x7F))
        table = F.e4m3_decode(np.array(codes, np.uint8))
        blk = 128
        s = rq["scales"].astype(np.float32)
        for r in range(4):
            for b in range(I // blk):
                sl = slice(b * blk, (b + 1) * blk)
                if s[r, b] == 0:
                    assert np.all(rq["hhat"][r, sl] == 0)
                    continue
                v = (h[r, sl] * (np.float32(1) / s[r, b])).astype(np.float32)
                mag = _nearest_even(np.abs(v).astype(np.float64), table, codes, lambda c: c & 7)
                want = np.sign(v) * F.e4m3_decode(mag.astype(np.uint8)) * np.float64(s[r, b])
                assert np.array_equal(rq["hhat"][r, sl], want)
    else:
        mags = F.e2m1_decode(np.arange(8))
        sf = F.e4m3_decode(rq["scales"]).astype(np.float32)
        for r in range(4):
            for b in range(I // 16):
                sl = slice(b * 16, (b + 1) * 16)
                amax = np.max(np.abs(h[r, sl]))
                # the block scale is the E4M3 rounding of amax / (6 G)
                want_sf = F.e4m3_decode(F.e4m3_encode(np.float32(amax / np.float32(6 * np.float32(G)))))
                assert sf[r, b] == want_sf
                if sf[r, b] == 0:
                    assert np.all(rq["hhat"][r, sl] == 0)
                    continue
                v = (h[r, sl] * (np.float32(1) / np.float32(sf[r, b] * np.float32(G)))).astype(np.float32)
                mag = _nearest_even(np.abs(v).astype(np.float64), mags, list(range(8)), lambda c: c & 1)
                want = np.sign(v) * mags[mag] * np.float64(sf[r, b])
                assert np.array_equal(rq["hhat"][r, sl], want)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_requant_error_bound(fmt):
    """|h^ - h| stays within half a code step (relative 2^-4 for E4M3, 1/4 of a step for e2m1 top)."""
    rng = np.random.default_rng(9)
    h = (rng.standard_normal((8, 512)) * 3).astype(np.float32)
    G = 100.0 / 2688.0
    rq = O.requant(fmt, h, G)
    hh = rq["hhat"] * (G if fmt == "nvfp4" else 1.0)
    if fmt == "fp8":
        s = np.repeat(rq["scales"], 128, axis=1)
        # E4M3 normal spacing is 2^-3 relative, so RNE error <= 2^-4 |v| (+ subnormal quantum)
        assert np.all(np.abs(hh - h) <= np.abs(h) * 2 ** -4 + s * 2 ** -10 + 1e-30)
    else:
        sf = np.repeat(F.e4m3_decode(rq["scales"]), 16, axis=1) * G
        # the largest e2m1 step is 2 (between 4 and 6); the scale itself rounds by <= 2^-4
        amax = np.repeat(np.max(np.abs(h.reshape(8, -1, 16)), axis=2), 16, axis=1)
        assert np.all(np.abs(hh - h) <= sf * 1.0 + amax * 2 ** -4 * 1.0 + 1e-12)
