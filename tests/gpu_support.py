"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
(the unfused chain or the single moe_fused launch), collect what it computed,
and compare it with the oracle.  Test code only."""

import numpy as np
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import formats as F
from oracle import moe as O

# max|err| bounds of the FFN output, relative to rms(oracle output)
TOL = {"bf16": 5e-3, "fp8": 2e-2, "nvfp4": 2e-2, "mxfp8": 2e-2, "fp8_tensor": 2e-2}
# An intermediate code may differ from the oracle's only if it is the correct
# rounding of a value within this distance of the oracle's pre-rounding FP32
# value, relative to that value (the kernel's FP32 h differs from the
# oracle's in its last bits, so a value that close to a rounding midpoint may
# round either way) ...
MID_REL = 1e-4
# ... plus this fraction of the block's magnitude (absolute error floor)
MID_ABS = 1e-5
# FP8 block scales are FP32 amax / 448 on both sides.
SCALE_REL = 1e-5
# A token whose intermediate codes flipped must still be within this multiple
# of the tolerance of the pure oracle (and within the plain tolerance of the
# oracle recomputed from the GPU's own codes).
FLIP_FACTOR = 3.0
# L2 + combine recomputed by the oracle from the GPU's codes vs the GPU's
# FP32 accumulator.
L2_REL = 1e-3


def k_all(p):
    """Slots per token after the routing (a shared expert adds one)."""
    return p["num_topk"] + int(p.get("shared_expert", 0))


def e_all(p):
    """Experts after the routing (a shared expert adds one)."""
    return p["num_experts"] + int(p.get("shared_expert", 0))


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


def weights_of(d):
    return {k: d.get(k) for k in ("w13", "w13_scale", "w2", "w2_scale", "gate_up_expert_scales",
                                  "down_expert_scales", "c_input_scales")}


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


# ------------------------------------------------------------------ code tables

def _round_to(fmt, v):
    """The format's round-to-nearest-even of v (the oracle's codecs), decoded."""
    if fmt == "bf16":
        return F.bf16_decode(F.bf16_encode(np.asarray(v, np.float64)))
    if fmt == "e4m3":
        return F.e4m3_decode(F.e4m3_encode(v))
    return F.e2m1_decode(F.e2m1_encode(v))


def rounding_of_nearby(fmt, got, pre, scale, rel=MID_REL, floor=MID_ABS):
    """True where `got` (a decoded GPU code) is the correct rounding of some
    value within rel * |pre| + floor * scale of `pre`, the oracle's value
    before rounding.  For an element near its block's magnitude this is the usual
    "a code may flip only at a rounding midpoint"; `scale` is the largest
    |pre| of the element's quantisation block, since the kernel's FP32 h
    differs from the oracle's by a few units in the last place of the block's
    large values (the dot product's rounding), so an element much smaller than
    its block may land several of its own code steps away."""
    pre = np.asarray(pre, np.float64)
    d = rel * np.abs(pre) + floor * np.asarray(scale, np.float64)
    lo, hi = _round_to(fmt, pre - d), _round_to(fmt, pre + d)   # rounding is monotonic
    got = np.asarray(got, np.float64)
    return (got >= lo) & (got <= hi)


def block_max(pre, block):
    """Per element, the largest |pre| of its block of `block` consecutive elements."""
    a = np.abs(np.asarray(pre, np.float64))
    return np.repeat(a.reshape(-1, block).max(axis=1), block)


# ------------------------------------------------------------------ GPU results

def row_scale_positions(lay_h, r):
    """Expert e of row r and its padded scale row."""
    starts = lay_h["expert_start_indices"]
    e = int(np.searchsorted(starts, r, side="right") - 1)
    while starts[e + 1] == starts[e]:
        e += 1
    pr = int(lay_h["a_scale_offsets"][e] + (r - starts[e]))
    return e, pr


class GpuResult:
    """What one run of the CUDA path computed: the layout (host arrays), the
    re-quantised intermediate (codes, then scales at scale_off; FP8 scales
    [I/128][scale_rows]), the FP32 accumulator (None in staged mode) and the
    BF16 output; route = (topk_idx, topk_weights) chosen in-kernel, if any."""

    def __init__(self, lay_h, codes, scales, scale_rows, acc, out, route=None):
        self.lay_h = lay_h
        self.codes = codes.cpu().numpy() if torch.is_tensor(codes) else codes
        self.scales = scales.cpu().numpy() if torch.is_tensor(scales) else scales
        self.scale_rows = int(scale_rows)
        self.acc = None if acc is None else acc.cpu().numpy()
        self.out = bf16_to_np(out)
        self.route = route

    def rows(self, p, rows, host=None):
        """GPU intermediate rows -> {row: dict(values, scales, hhat)}: values =
        decoded element codes (unscaled), scales = block scales (FP8 float32,
        NVFP4 E4M3 codes, MXFP8 UE8M0 codes), hhat = dequantised row (float64,
        the L2 input)."""
        fmt, I = p["format"], p["intermediate_hidden"]
        R_total = p["num_tokens"] * k_all(p)
        out = {}
        if fmt == "bf16":
            codes = self.codes[: R_total * I * 2].view(np.uint16).reshape(R_total, I)
            for r in rows:
                v = F.bf16_decode(codes[r])
                out[r] = dict(codes=codes[r], values=v, scales=None, hhat=v)
            return out
        if fmt == "fp8":
            codes = self.codes[: R_total * I].reshape(R_total, I)
            P = self.scale_rows
            sc = self.scales[: (I // 128) * P * 4].view(np.float32).reshape(I // 128, P)
            for r in rows:
                _, pr = row_scale_positions(self.lay_h, r)
                s = sc[:, pr].copy()
                out[r] = dict(codes=codes[r], values=F.e4m3_decode(codes[r]), scales=s,
                              hhat=O.dequant_intermediate("fp8", codes[r][None], s[None], I)[0])
            return out
        if fmt == "fp8_tensor":
            # one static scale per expert (an input, not in the workspace)
            codes = self.codes[: R_total * I].reshape(R_total, I)
            for r in rows:
                e, _ = row_scale_positions(self.lay_h, r)
                G = np.float32(host["c_input_scales"][e])
                out[r] = dict(codes=codes[r], values=F.e4m3_decode(codes[r]), scales=np.array([G]),
                              hhat=O.dequant_intermediate("fp8_tensor", codes[r][None], np.array([G]), I)[0])
            return out
        if fmt == "mxfp8":
            codes = self.codes[: R_total * I].reshape(R_total, I)
            kc = I // 128
            j = np.arange(I // 32)
            for r in rows:
                _, pr = row_scale_positions(self.lay_h, r)
                off = ((pr >> 7) * kc + (j >> 2)) * 512 + (pr & 31) * 16 + ((pr >> 5) & 3) * 4 + (j & 3)
                s = self.scales[off].copy()
                out[r] = dict(codes=codes[r], values=F.e4m3_decode(codes[r]), scales=s,
                              hhat=O.dequant_intermediate("mxfp8", codes[r][None], s[None], I)[0])
            return out
        codes = self.codes[: R_total * I // 2].reshape(R_total, I // 2)
        kc = I // 64
        j = np.arange(I // 16)
        for r in rows:
            _, pr = row_scale_positions(self.lay_h, r)
            off = ((pr >> 7) * kc + (j >> 2)) * 512 + (pr & 31) * 16 + ((pr >> 5) & 3) * 4 + (j & 3)
            s = self.scales[off].copy()
            out[r] = dict(codes=codes[r], values=F.e2m1_decode(F.fp4_unpack(codes[r][None], I)[0]),
                          scales=s, hhat=O.dequant_intermediate("nvfp4", codes[r][None], s[None], I)[0])
        return out


def run_chain(L, d, out_mode=api.MOE_OUT_ACCUMULATE):
    """moe_permute -> moe_ffn (keeping the intermediate) -> moe_combine."""
    M = d["x"].shape[0]
    prob = L.problem(M)
    lay = L.permute(d["topk_idx"])
    y, inter = L.ffn(d["x"], d.get("x_scale"), lay, d["topk_weights"], out_mode=out_mode, keep_intermediate=True,
                     x_rowwise_scale=d.get("x_row_scale"))
    if out_mode == api.MOE_OUT_ACCUMULATE:
        out = L.combine(lay, None, y, api.MOE_IN_ACCUMULATED, M)
    else:
        out = L.combine(lay, d["topk_weights"], y, api.MOE_IN_STAGED, M)
    torch.cuda.synchronize()
    so = api.intermediate_size(prob)[1]
    P = api.workspace_offsets(prob)["scale_rows"]
    return GpuResult(lay.host(), inter[:so], inter[so:], P,
                     y if out_mode == api.MOE_OUT_ACCUMULATE else None, out)


def run_fused(L, d, from_logits=False):
    """moe_fused, then what it left in the workspace."""
    M = d["x"].shape[0]
    if from_logits:
        out = L.forward(d["x"], d.get("x_scale"), logits=d["logits"], bias=d["bias"])
    else:
        out = L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"],
                        x_rowwise_scale=d.get("x_row_scale"))
    torch.cuda.synchronize()
    v = L.workspace_views(M)
    lay_h = {k: v[k].cpu().numpy() for k in ("expert_counts", "expert_start_indices", "src_info",
                                             "slot_to_row", "expert_ids", "num_active", "a_scale_offsets",
                                             "tile_offsets")}
    route = (v["topk_idx"].cpu().numpy(), v["topk_weights"].cpu().numpy()) if from_logits else None
    return GpuResult(lay_h, v["intermediate"], v["intermediate_scales"], v["scale_rows"], v["accumulator"],
                     out, route=route)


# ------------------------------------------------------------------ checks

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


def check_route(res, host, k):
    """In-kernel routing: indices bit-exact, weights to 1e-6 relative."""
    ridx, rw = O.route(host["logits"], host["bias"], k)
    gidx, gw = res.route
    assert np.array_equal(gidx, ridx)
    assert np.all(np.abs(gw.astype(np.float64) - rw) <= 1e-6 * rw + 1e-7)
    return ridx, rw


def _compare_codes(p, host, e, it, g, stats):
    """Tier (a) for one routed slot: the GPU's codes against the oracle's.
    Returns True if any code or scale differs (all at rounding midpoints)."""
    fmt, I = p["format"], p["intermediate_hidden"]
    pre = np.asarray(it["pre"], np.float64)
    ref_vals = None
    flipped = False
    if fmt == "bf16":
        table = "bf16"
        ref_vals = F.bf16_decode(it["codes"])
    elif fmt == "fp8":
        table = "e4m3"
        s_o = np.asarray(it["scales"], np.float64)
        s_g = np.asarray(g["scales"], np.float64)
        assert np.all(np.abs(s_g - s_o) <= SCALE_REL * np.abs(s_o)), \
            f"FP8 block scales differ: {s_g} vs {s_o}"
        ref_vals = F.e4m3_decode(it["codes"])
    elif fmt == "fp8_tensor":
        table = "e4m3"
        ref_vals = F.e4m3_decode(it["codes"]).astype(np.float64)
    elif fmt == "mxfp8":
        table = "e4m3"
        ref_vals = F.e4m3_decode(it["codes"]).astype(np.float64)
        sc_o = np.asarray(it["scales"], np.int64)
        sc_g = np.asarray(g["scales"], np.int64)
        sdiff = sc_o != sc_g
        if sdiff.any():
            # a scale may differ only by one step, where the block's amax is
            # within MID_REL of the power of two that separates the two
            amax = np.max(np.abs(np.asarray(it["h32"], np.float64).reshape(I // 32, 32)), axis=1)
            edge = np.ldexp(1.0, np.maximum(sc_o, sc_g) - 127 + 8)
            ok = (np.abs(sc_g - sc_o) == 1) & (np.abs(amax - edge) <= MID_REL * edge)
            ok = ok[sdiff]
            assert ok.all(), f"MXFP8 block scale differs beyond a power-of-two edge: {sc_g[sdiff][~ok]} vs {sc_o[sdiff][~ok]}"
            stats["scale_flips"] += int(sdiff.sum())
            flipped = True
            # the block's codes follow the GPU's scale: re-derive the oracle's
            h32 = np.asarray(it["h32"], np.float64).reshape(I // 32, 32)
            ref_vals = ref_vals.reshape(I // 32, 32).copy()
            pre = pre.reshape(I // 32, 32).copy()
            for b in np.nonzero(sdiff)[0]:
                v = h32[b] * np.ldexp(1.0, 127 - int(sc_g[b]))
                ref_vals[b] = F.e4m3_decode(F.e4m3_encode(v))
                pre[b] = v
            ref_vals = ref_vals.reshape(I)
            pre = pre.reshape(I)
    else:
        table = "e2m1"
        ref_vals = F.e2m1_decode(F.fp4_unpack(np.asarray(it["codes"])[None], I)[0]).astype(np.float64)
        sv_o = F.e4m3_decode(it["scales"])
        sv_g = F.e4m3_decode(g["scales"])
        sdiff = sv_o != sv_g
        if sdiff.any():
            ok = rounding_of_nearby("e4m3", sv_g[sdiff], it["pre_scale"][sdiff], np.max(np.abs(it["pre_scale"])))
            assert ok.all(), f"NVFP4 block scale is not a rounding of the oracle's value: " \
                             f"{sv_g[sdiff][~ok]} vs {sv_o[sdiff][~ok]}"
            stats["scale_flips"] += int(sdiff.sum())
            flipped = True
            # the block's codes are then those of the GPU's scale: re-derive
            # the oracle's codes for those blocks from its h with that scale
            G = np.float32(host["c_input_scales"][e])
            h32 = np.asarray(it["h32"], np.float32).reshape(I // 16, 16)
            ref_vals = ref_vals.reshape(I // 16, 16).copy()
            pre = pre.reshape(I // 16, 16).copy()
            for b in np.nonzero(sdiff)[0]:
                sg = np.float32(sv_g[b])
                if sg == 0:
                    ref_vals[b] = 0.0
                    pre[b] = 0.0
                    continue
                inv = np.float32(1.0) / np.float32(sg * G)
                v = (h32[b] * inv).astype(np.float32)
                ref_vals[b] = F.e2m1_decode(F.e2m1_encode(v))
                pre[b] = v
            ref_vals = ref_vals.reshape(I)
            pre = pre.reshape(I)
    got_vals = np.asarray(g["values"], np.float64)
    diff = got_vals != ref_vals
    stats["code_vals"] += diff.size
    if diff.any():
        # quantisation blocks: the whole row (BF16), 128 (FP8), 16 (NVFP4) or 32 (MXFP8) values
        scale = block_max(pre, {"bf16": I, "fp8": 128, "nvfp4": 16, "mxfp8": 32, "fp8_tensor": I}[fmt])
        ok = rounding_of_nearby(table, got_vals[diff], pre[diff], scale[diff])
        assert ok.all(), (f"{fmt} intermediate codes are not a rounding of the oracle's value: GPU "
                          f"{got_vals[diff][~ok][:8]} oracle {ref_vals[diff][~ok][:8]} "
                          f"pre-rounding {pre[diff][~ok][:8]}")
        stats["code_flips"] += int(diff.sum())
        flipped = True
    return flipped


def oracle_reference(p, host, tokens):
    """The pure oracle on `tokens`, keeping its intermediate (shareable between checks)."""
    return O.moe_forward(p, host, host["topk_idx"], host["topk_weights"], tokens=np.asarray(tokens),
                         keep_intermediate=True)


def check_against_oracle(p, host, res, tokens, label="", ref=None):
    """Split parity of one GPU result for the tokens in `tokens`:
      (a) every re-quantised intermediate code (and block scale) is the
          correct rounding of a value within MID_REL * |value| + MID_ABS *
          (the block's magnitude) of the oracle's pre-rounding value -- equal
          to the oracle's code except at rounding midpoints;
      (b) the oracle's L2 + combine recomputed from the GPU's own codes matches
          the GPU's FP32 accumulator to L2_REL * rms (when there is one);
      (c) end to end, |out - oracle| <= TOL * rms + the output's own half-ulp;
          a token with flipped codes may exceed it only if it meets that bound
          against the oracle recomputed from the GPU's codes AND stays within
          FLIP_FACTOR * TOL * rms of the pure oracle.
    Returns a dict of statistics (flip counts, errors relative to rms)."""
    fmt = p["format"]
    k = k_all(p)
    tokens = np.asarray(tokens)
    if ref is None:
        ref = oracle_reference(p, host, tokens)
    slot_to_row = res.lay_h["slot_to_row"]
    rows = [int(slot_to_row[t * k + j]) for t in tokens for j in range(k) if slot_to_row[t * k + j] >= 0]
    gi = res.rows(p, rows, host)

    # (a) codes
    stats = dict(code_flips=0, scale_flips=0, code_vals=0)
    flipped_tokens = set()
    for (t, j), it in ref["intermediate"].items():
        r = int(slot_to_row[t * k + j])
        assert r >= 0
        if _compare_codes(p, host, it["expert"], it, gi[r], stats):
            flipped_tokens.add(int(t))
    assert stats["code_flips"] <= max(8, 1e-3 * stats["code_vals"]), \
        f"{label}: {stats['code_flips']} of {stats['code_vals']} intermediate codes differ"

    # (b) L2 + combine from the GPU's codes
    def override(e, ts, js):
        return np.stack([gi[int(slot_to_row[int(a) * k + int(b)])]["hhat"] for a, b in zip(ts, js)])
    ref_g = O.moe_forward(p, host, host["topk_idx"], host["topk_weights"], tokens=tokens,
                          hhat_override=override)
    r_g = rms(ref_g["out_f64"])
    err_b = None
    if res.acc is not None:
        err_b = float(np.max(np.abs(res.acc[tokens] - ref_g["out_f64"])))
        assert err_b <= L2_REL * r_g, f"{label} L2+combine from GPU codes: {err_b:.3e} > {L2_REL}*rms {r_g:.3e}"

    # (c) end to end
    got = res.out[tokens]
    exact = ref["out_f64"]
    r = rms(exact)
    tol = TOL[fmt] * r
    per_tok = np.max(np.abs(got - exact) - bf16_half_ulp(exact), axis=1)
    over = [i for i in np.nonzero(per_tok > tol)[0]]
    for i in over:
        t = int(tokens[i])
        assert t in flipped_tokens, f"{label}: token {t} error {per_tok[i] / r:.3e}*rms > {TOL[fmt]} with no code flip"
        expl = float(np.max(np.abs(got[i] - ref_g["out_f64"][i]) - bf16_half_ulp(ref_g["out_f64"][i])))
        assert expl <= TOL[fmt] * r_g, f"{label}: token {t} not explained by its flipped codes ({expl / r_g:.3e}*rms)"
        assert per_tok[i] <= FLIP_FACTOR * tol, f"{label}: token {t} error {per_tok[i] / r:.3e}*rms > {FLIP_FACTOR}x tol"
    stats.update(max_err_rel=float(per_tok.max() / r), tokens_over=len(over), tokens_flipped=len(flipped_tokens),
                 l2_err_rel=None if err_b is None else err_b / r_g,
                 max_err_vs_bf16_oracle_rel=float(np.max(np.abs(got - F.bf16_decode(ref["out_bf16"]))) / r))
    return stats
