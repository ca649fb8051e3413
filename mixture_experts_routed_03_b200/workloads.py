"""Seeded synthetic inputs for the routed MoE FFN.

This module draws the *inputs* of the layer -- activations, expert weights,
their block scales, the per-expert scale arrays and the routing -- with
torch's seeded generators.  It holds none of the layer's own arithmetic:
codes are drawn directly (random bytes for packed e2m1, torch's float8 cast of
Gaussian draws for E4M3, torch's bfloat16 cast for BF16) and scales are drawn
as plain positive numbers.  Both the CUDA path and the CPU oracle consume
what it returns; neither is imported here.

The workloads follow the shapes and value structure of the routed-MoE
API pages (flashinfer.megamoe.MegaMoESymmBuffer staging views; Struct_mega_
ffn_ep_combine_send operands; flashinfer.fused_moe.MoEActivationPack
activation encodings and FromLogits routing):

  tiny_bf16        M=16    H=256  I=128  E=8   k=2  BF16, softmax top-2 routing
  fp8_block        M=256   H=2048 I=768  E=64  k=6  E4M3 + FP32 per-128 scales
  nvfp4_prefill    M=4096  H=7168 I=2048 E=32  k=8  NVFP4, uniform routing
  nvfp4_decode     M=64    H=7168 I=2048 E=256 k=8  NVFP4, Zipf(1.2) routing
  fp8_prefill_routed M=16384 H=4096 I=1536 E=128 k=8 E4M3, routing from logits
  nvfp4_prefill_rowwise  as nvfp4_prefill, with BF16 activations [M, H]
                     (x_bf16) for the per-token quantiser
  mxfp8_prefill_routed   the fp8_prefill_routed shapes in MXFP8: E4M3 with
                     UE8M0 scales per 32 (MoEActivationPack MXFP8)
  fp8_tensor_prefill_routed  the same shapes in FP8 per-tensor: E4M3 with
                     one FP32 scale per tensor (MoEActivationPack FP8
                     per-tensor)
"""

import math

import torch

WORKLOADS = {
    "tiny_bf16": dict(num_tokens=16, hidden=256, intermediate_hidden=128,
                      num_experts=8, num_topk=2, format="bf16", routing="softmax"),
    "fp8_block": dict(num_tokens=256, hidden=2048, intermediate_hidden=768,
                      num_experts=64, num_topk=6, format="fp8", routing="softmax"),
    "nvfp4_prefill": dict(num_tokens=4096, hidden=7168, intermediate_hidden=2048,
                          num_experts=32, num_topk=8, format="nvfp4", routing="uniform"),
    "nvfp4_decode": dict(num_tokens=64, hidden=7168, intermediate_hidden=2048,
                         num_experts=256, num_topk=8, format="nvfp4", routing="zipf"),
    "fp8_prefill_routed": dict(num_tokens=16384, hidden=4096, intermediate_hidden=1536,
                               num_experts=128, num_topk=8, format="fp8", routing="logits"),
    # the NVFP4 prefill with BF16 activations quantised per token by the
    # layer (EPConfig nvfp4_dyn_global_scales) instead of arriving quantised
    "nvfp4_prefill_rowwise": dict(num_tokens=4096, hidden=7168, intermediate_hidden=2048,
                                  num_experts=32, num_topk=8, format="nvfp4", routing="uniform",
                                  act="bf16"),
    # the FP8 prefill's shapes with the microscaling format's power-of-two
    # scales per 32 elements, which the tensor cores apply themselves
    "mxfp8_prefill_routed": dict(num_tokens=16384, hidden=4096, intermediate_hidden=1536,
                                 num_experts=128, num_topk=8, format="mxfp8", routing="logits"),
    # the same shapes with one FP32 scale per tensor: the tensor cores sum all
    # of K and the epilogue applies the scales once
    "fp8_tensor_prefill_routed": dict(num_tokens=16384, hidden=4096, intermediate_hidden=1536,
                                      num_experts=128, num_topk=8, format="fp8_tensor", routing="logits"),
}

# Typical magnitudes of the drawn values.
X_STD = 1.0          # activations
W_STD = 0.02         # expert weights
FP8_CODE_STD = 64.0  # spread of the drawn E4M3 codes (well inside +-448)
FP4_CODE_RMS = math.sqrt(68.5 / 8.0)   # rms of a uniformly drawn e2m1 code
BF16_X_STD = 0.02    # the BF16 workload draws x and W from N(0, 0.02)


def problem(name, **overrides):
    p = dict(WORKLOADS[name])
    p.setdefault("activation_clamp", 10.0)
    p.update(overrides)
    return p


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _uniform(shape, lo, hi, g, device):
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def _bf16_codes(shape, std, g, device):
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std
    return v.to(torch.bfloat16).view(torch.int16)


def _e4m3_codes(shape, g, device):
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * FP8_CODE_STD
    return v.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _e4m3_positive(shape, lo, hi, g, device):
    return _uniform(shape, lo, hi, g, device).to(torch.float8_e4m3fn).view(torch.uint8)


def _ue8m0_codes(shape, lo, hi, g, device):
    """UE8M0 scale codes drawn uniformly from the integers lo..hi (code c is 2^(c-127))."""
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def _fp4_bytes(shape, g, device):
    return torch.randint(0, 256, shape, generator=g, device=device, dtype=torch.uint8)


def _routing(p, g, device):
    M, E, k = p["num_tokens"], p["num_experts"], p["num_topk"]
    kind = p["routing"]
    out = {}
    if kind in ("softmax", "logits"):
        logits = torch.randn((M, E), generator=g, device=device, dtype=torch.float32)
        if kind == "logits":
            out["logits"] = logits
            out["bias"] = torch.randn((E,), generator=g, device=device, dtype=torch.float32) * 0.1
            return out
        vals, idx = torch.topk(logits, k, dim=1)
        out["topk_idx"] = idx.to(torch.int64)
        out["topk_weights"] = torch.softmax(vals, dim=1).to(torch.float32)
        return out
    if kind == "uniform":
        keys = torch.rand((M, E), generator=g, device=device)
    elif kind == "zipf":
        logp = -1.2 * torch.log(torch.arange(1, E + 1, device=device, dtype=torch.float32))
        u = torch.rand((M, E), generator=g, device=device).clamp_(1e-12, 1.0 - 1e-7)
        keys = logp[None, :] - torch.log(-torch.log(u))          # Gumbel-top-k
    else:
        raise ValueError(kind)
    out["topk_idx"] = torch.topk(keys, k, dim=1).indices.to(torch.int64)
    ex = -torch.log(torch.rand((M, k), generator=g, device=device).clamp_(1e-12, 1.0))
    out["topk_weights"] = (ex / ex.sum(dim=1, keepdim=True)).to(torch.float32)  # Dirichlet(1)
    return out


def make_inputs(p, seed=0, device="cpu"):
    """Draw every input of problem ``p`` (a dict from ``problem``) with ``seed``.

    Returns a dict of torch tensors on ``device``:
      x, x_scale, w13, w13_scale, w2, w2_scale,
      gate_up_expert_scales, down_expert_scales, c_input_scales  (NVFP4),
      topk_idx, topk_weights          (precomputed routing), or
      logits, bias                    (routing from logits).
    Layouts: x [M, H] (BF16 / E4M3) or [M, H/2] packed e2m1; x_scale
    FP32 [M, H/128], E4M3 [M, H/16] or UE8M0 [M, H/32]; w13 [E, 2I, H(/2)]
    with gate rows first; w2 [E, H, I(/2)]; weight scales FP32
    [E, N/128, K/128], E4M3 [E, N, K/16] or UE8M0 [E, N, K/32].
    """
    device = torch.device(device)
    g = _gen(device, seed)
    fmt = p["format"]
    M, H, I, E = p["num_tokens"], p["hidden"], p["intermediate_hidden"], p["num_experts"]
    # experts whose weights are drawn: the routed ones, then a shared expert
    # (EPConfig fused_shared_expert) if the problem has one
    Ew = E + int(p.get("shared_expert", 0))
    d = {}
    if fmt == "bf16":
        d["x"] = _bf16_codes((M, H), BF16_X_STD, g, device)
        d["w13"] = _bf16_codes((Ew, 2 * I, H), W_STD, g, device)
        d["w2"] = _bf16_codes((Ew, H, I), W_STD, g, device)
        d["x_scale"] = d["w13_scale"] = d["w2_scale"] = None
    elif fmt == "fp8":
        d["x"] = _e4m3_codes((M, H), g, device)
        d["x_scale"] = _uniform((M, H // 128), 0.5, 1.5, g, device) * (X_STD / FP8_CODE_STD)
        d["w13"] = torch.empty((Ew, 2 * I, H), dtype=torch.uint8, device=device)
        d["w2"] = torch.empty((Ew, H, I), dtype=torch.uint8, device=device)
        for e in range(Ew):                       # per expert: bounded host memory
            d["w13"][e] = _e4m3_codes((2 * I, H), g, device)
            d["w2"][e] = _e4m3_codes((H, I), g, device)
        d["w13_scale"] = _uniform((Ew, 2 * I // 128, H // 128), 0.5, 1.5, g, device) * (W_STD / FP8_CODE_STD)
        d["w2_scale"] = _uniform((Ew, H // 128, I // 128), 0.5, 1.5, g, device) * (W_STD / FP8_CODE_STD)
    elif fmt == "nvfp4":
        d["x"] = _fp4_bytes((M, H // 2), g, device)
        d["x_scale"] = _e4m3_positive((M, H // 16), 0.5, 1.5, g, device)
        d["w13"] = _fp4_bytes((Ew, 2 * I, H // 2), g, device)
        d["w13_scale"] = _e4m3_positive((Ew, 2 * I, H // 16), 0.5, 1.5, g, device)
        d["w2"] = _fp4_bytes((Ew, H, I // 2), g, device)
        d["w2_scale"] = _e4m3_positive((Ew, H, I // 16), 0.5, 1.5, g, device)
        # Per-tensor activation global and per-expert weight globals, as
        # dequant multipliers; the layer takes their products per expert.
        x_global = X_STD / FP4_CODE_RMS
        w13_global = _uniform((Ew,), 0.8, 1.2, g, device) * (W_STD / FP4_CODE_RMS)
        w2_global = _uniform((Ew,), 0.8, 1.2, g, device) * (W_STD / FP4_CODE_RMS)
        # Static per-expert re-quant scale (a checkpoint-style calibration):
        # with the clamp c, |h| < c*c, so 2688 * G >= c*c never saturates the
        # E4M3 block scale.  Without a clamp a fixed bound of 1000 stands in.
        c = float(p.get("activation_clamp", 10.0))
        # |h| < c*c for the clamped SwiGLU, < c*(c+1) for swigluoai
        bound = (c * (c + 1.0) if p.get("activation") == "swigluoai" else c * c) if math.isfinite(c) else 1000.0
        c_in = _uniform((Ew,), 1.0, 1.2, g, device) * (bound / 2688.0)
        d["gate_up_expert_scales"] = (w13_global * x_global).to(torch.float32)
        d["down_expert_scales"] = (w2_global * c_in).to(torch.float32)
        d["c_input_scales"] = c_in.to(torch.float32)
    elif fmt == "fp8_tensor":
        # one FP32 scale for the activations and one per expert matrix; the
        # intermediate's static re-quant scale G with 448 * G above |h|
        d["x"] = _e4m3_codes((M, H), g, device)
        d["x_scale"] = _uniform((1,), 0.5, 1.5, g, device) * (X_STD / FP8_CODE_STD)
        d["w13"] = torch.empty((Ew, 2 * I, H), dtype=torch.uint8, device=device)
        d["w2"] = torch.empty((Ew, H, I), dtype=torch.uint8, device=device)
        for e in range(Ew):
            d["w13"][e] = _e4m3_codes((2 * I, H), g, device)
            d["w2"][e] = _e4m3_codes((H, I), g, device)
        d["w13_scale"] = _uniform((Ew,), 0.5, 1.5, g, device) * (W_STD / FP8_CODE_STD)
        d["w2_scale"] = _uniform((Ew,), 0.5, 1.5, g, device) * (W_STD / FP8_CODE_STD)
        c = float(p.get("activation_clamp", 10.0))
        bound = (c * (c + 1.0) if p.get("activation") == "swigluoai" else c * c) if math.isfinite(c) else 1000.0
        d["c_input_scales"] = (_uniform((Ew,), 1.0, 1.2, g, device) * (bound / 448.0)).to(torch.float32)
    elif fmt == "mxfp8":
        # power-of-two scales around X_STD / FP8_CODE_STD = 2^-6 (codes
        # 120..122) and W_STD / FP8_CODE_STD ~ 2^-11.6 (codes 115..117)
        d["x"] = _e4m3_codes((M, H), g, device)
        d["x_scale"] = _ue8m0_codes((M, H // 32), 120, 122, g, device)
        d["w13"] = torch.empty((Ew, 2 * I, H), dtype=torch.uint8, device=device)
        d["w2"] = torch.empty((Ew, H, I), dtype=torch.uint8, device=device)
        for e in range(Ew):
            d["w13"][e] = _e4m3_codes((2 * I, H), g, device)
            d["w2"][e] = _e4m3_codes((H, I), g, device)
        d["w13_scale"] = _ue8m0_codes((Ew, 2 * I, H // 32), 115, 117, g, device)
        d["w2_scale"] = _ue8m0_codes((Ew, H, I // 32), 115, 117, g, device)
    else:
        raise ValueError(fmt)
    if p.get("act") == "bf16":
        # raw activations for the per-token quantiser
        d["x_bf16"] = _bf16_codes((M, H), X_STD, g, device)
    d.update(_routing(p, g, device))
    return d


def to_numpy(d):
    """Host numpy copies of a ``make_inputs`` dict (None entries kept)."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.int16:
            out[k] = v.cpu().view(torch.int16).numpy().view("uint16")
        else:
            out[k] = v.cpu().numpy()
    return out
