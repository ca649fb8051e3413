"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it with the oracle.  Test code only."""

import numpy as np
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import formats as F
from oracle import moe as O

TOL = {"bf16": 5e-3, "fp8": 2e-2, "nvfp4": 2e-2}


def device():
    return torch.device("cuda", 0)


def make(p, seed, on_gpu_generation=False):
    """Inputs on the GPU and the same bytes on the host (numpy)."""
    dev = device()
    if on_gpu_generation:
        d = workloads.make_inputs(p, seed=seed, device=dev)
        host = workloads.to_numpy(d)
    else:
        h = workloads.make_inputs(p, seed=seed, device="cpu")
        host = workloads.to_numpy(h)
        d = {k: (None if v is None else v.to(dev)) for k, v in h.items()}
    return d, host


def bf16_to_np(t):
    return F.bf16_decode(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def rms(a):
    return float(np.sqrt(np.mean(np.asarray(a, np.float64) ** 2)))


def bf16_half_ulp(v):
    """Half the BF16 spacing at |v| (8 significant bits): the most a correct
    round-to-nearest of v can move it."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def close_bf16(a, b, tol_abs):
    """|a - b| <= tol_abs + one BF16 half-ulp of each side (two roundings of
    nearly equal values may land on neighbouring BF16 numbers)."""
    return np.abs(a - b) <= tol_abs + bf16_half_ulp(a) + bf16_half_ulp(b)


def row_scale_positions(lay_h, r):
    """Expert e of row r and its padded scale row."""
    starts = lay_h["expert_start_indices"]
    e = int(np.searchsorted(starts, r, side="right") - 1)
    while starts[e + 1] == starts[e]:
        e += 1
    pr = int(lay_h["a_scale_offsets"][e] + (r - starts[e]))
    return e, pr


def decode_gpu_intermediate(p, inter, scale_off, lay_h, rows):
    """GPU re-quantised intermediate rows -> (codes, scales-in-oracle-layout, hhat float64)."""
    fmt, I = p["format"], p["intermediate_hidden"]
    buf = inter.cpu().numpy()
    R_total = p["num_tokens"] * p["num_topk"]
    out = {}
    if fmt == "bf16":
        codes = buf[: R_total * I * 2].view(np.uint16).reshape(R_total, I)
        for r in rows:
            out[r] = dict(codes=codes[r], scales=None, hhat=F.bf16_decode(codes[r]))
        return out
    if fmt == "fp8":
        codes = buf[: R_total * I].reshape(R_total, I)
        P = int(lay_h["a_scale_offsets"][p["num_experts"]])
        ld = (len(buf) - scale_off) // 4 // (I // 128)
        sc = buf[scale_off: scale_off + (I // 128) * ld * 4].view(np.float32).reshape(I // 128, ld)
        for r in rows:
            _, pr = row_scale_positions(lay_h, r)
            s = sc[:, pr].copy()
            out[r] = dict(codes=codes[r], scales=s,
                          hhat=O.dequant_intermediate("fp8", codes[r][None], s[None], I)[0])
        return out
    codes = buf[: R_total * I // 2].reshape(R_total, I // 2)
    kc = I // 64
    sfb = buf[scale_off:]
    for r in rows:
        _, pr = row_scale_positions(lay_h, r)
        j = np.arange(I // 16)
        off = ((pr >> 7) * kc + (j >> 2)) * 512 + (pr & 31) * 16 + ((pr >> 5) & 3) * 4 + (j & 3)
        s = sfb[off].copy()
        out[r] = dict(codes=codes[r], scales=s,
                      hhat=O.dequant_intermediate("nvfp4", codes[r][None], s[None], I)[0])
    return out


def check_layout_exact(lay_h, ref, M, k):
    R = int(ref["expert_start_indices"][-1])
    E = len(ref["expert_counts"])
    assert np.array_equal(lay_h["expert_counts"][:E], ref["expert_counts"])
    assert np.array_equal(lay_h["expert_start_indices"][:E + 1], ref["expert_start_indices"])
    assert np.array_equal(lay_h["src_info"][:R], ref["src_info"])
    assert np.array_equal(lay_h["slot_to_row"][:M * k], ref["slot_to_row"])
    assert np.array_equal(lay_h["expert_ids"][:E], ref["expert_ids"])
    assert int(lay_h["num_active"][0]) == ref["num_active"]
    assert np.array_equal(lay_h["a_scale_offsets"][:E + 1], ref["a_scale_offsets"])
    na = ref["num_active"]
    tiles = -(-ref["expert_counts"][ref["expert_ids"][:na]] // 128)
    assert np.array_equal(lay_h["tile_offsets"][:na + 1], np.concatenate([[0], np.cumsum(tiles)]))


def run_unfused(L, d, keep_intermediate=True):
    """permute -> ffn (accumulate, keeping the intermediate) -> combine."""
    M = d["x"].shape[0]
    lay = L.permute(d["topk_idx"])
    acc, inter = L.ffn(d["x"], d.get("x_scale"), lay, d["topk_weights"], keep_intermediate=keep_intermediate)
    out = L.combine(lay, None, acc, api.MOE_IN_ACCUMULATED, M)
    torch.cuda.synchronize()
    return lay, acc, inter, out


def check_ffn_against_oracle(p, host, lay_h, acc, inter, out_bf16, tokens, label=""):
    """Split parity for the tokens in `tokens`:
      (a) re-quantised codes equal the oracle's except near rounding midpoints,
      (b) L2 + combine recomputed by the oracle from the GPU's own codes match
          the GPU's FP32 accumulator to 1e-3 * rms,
      (c) end to end against the pure oracle within the format's tolerance,
          tokens that miss it being only ones whose codes flipped.
    Returns a dict of statistics."""
    fmt = p["format"]
    k = p["num_topk"]
    I = p["intermediate_hidden"]
    tokens = np.asarray(tokens)
    ref = O.moe_forward(p, host, host["topk_idx"], host["topk_weights"], tokens=tokens,
                        keep_intermediate=True)
    so = api.intermediate_size(api.problem_from_dict(p))[1]
    slot_to_row = lay_h["slot_to_row"]
    rows = []
    for t in tokens:
        for j in range(k):
            r = int(slot_to_row[t * k + j])
            if r >= 0:
                rows.append(r)
    gi = decode_gpu_intermediate(p, inter, so, lay_h, rows)

    # (a) codes
    flipped_tokens = set()
    n_vals = n_diff = 0
    for (t, j), it in ref["intermediate"].items():
        r = int(slot_to_row[t * k + j])
        g = gi[r]
        hh_o = O.dequant_intermediate(fmt, it["codes"][None], None if it["scales"] is None else it["scales"][None], I)[0]
        diff = np.abs(g["hhat"] - hh_o)
        scale = np.max(np.abs(hh_o)) + 1e-30
        bad = diff > 1e-6 * scale
        n_vals += bad.size
        n_diff += int(bad.sum())
        if bad.any():
            flipped_tokens.add(int(t))
    # (b) L2 + combine from the GPU codes
    def override(e, ts, js):
        return np.stack([gi[int(slot_to_row[int(a) * k + int(b)])]["hhat"] for a, b in zip(ts, js)])
    ref_g = O.moe_forward(p, host, host["topk_idx"], host["topk_weights"], tokens=tokens,
                          hhat_override=override)
    acc_h = acc.cpu().numpy()[tokens]
    r_ref = rms(ref_g["out_f64"])
    err_b = float(np.max(np.abs(acc_h - ref_g["out_f64"])))
    assert err_b <= 1e-3 * r_ref, f"{label} L2+combine from GPU codes: {err_b:.3e} > 1e-3*rms {r_ref:.3e}"
    # (c) end to end: the GPU's BF16 output against the oracle's unrounded
    # value, within the format's tolerance plus the output's own rounding
    got = bf16_to_np(out_bf16)[tokens]
    exact = ref["out_f64"]
    r = rms(exact)
    excess = np.abs(got - exact) - bf16_half_ulp(exact)
    per_tok = np.max(excess, axis=1)
    over = [int(tokens[i]) for i in np.nonzero(per_tok > TOL[fmt] * r)[0]]
    unexplained = [t for t in over if t not in flipped_tokens]
    assert not unexplained, (f"{label} end-to-end error {per_tok.max():.3e} > {TOL[fmt]}*rms {r:.3e} "
                             f"at tokens {unexplained} without code flips")
    # the code differences must be rare
    assert n_diff <= max(8, 1e-3 * n_vals), f"{label} {n_diff} of {n_vals} intermediate codes differ"
    plain = float(np.max(np.abs(got - F.bf16_decode(ref["out_bf16"]))) / r)
    return dict(max_err_rel=float(per_tok.max() / r), max_err_vs_bf16_oracle_rel=plain,
                tokens_over=len(over), code_diffs=n_diff,
                code_vals=n_vals, l2_err_rel=err_b / r_ref)
