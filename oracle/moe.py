"""Plain float64 oracle of the routed MoE FFN: route, permute, FFN, combine.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Notation: M tokens, H = hidden, I = intermediate_hidden, E = num_experts,
k = num_topk.  A routed *slot* is the pair (token t, position j < k), with the
flat slot index s = t*k + j.

What is computed, per token t (the definition this file restates):

    for every slot j with e = topk_idx[t, j] >= 0:
        x^     = decode(x[t])                             activation decode
        g, u   = gate / up projections of x^ by expert e  (L1, "gate_up")
        h      = min(g, c) * sigmoid(min(g, c)) * clamp(u, -c, c)
        h^     = decode(requant(h))                       L1 epilogue re-quant
        y      = down projection of h^ by expert e        (L2, "down")
    out[t] = bf16( sum_j topk_weights[t, j] * y )         the combine

Sources, by page and section:

* Struct_mega_ffn_ep_combine_send, Args: ``gate_up_weight`` (E, N1, K1//2),
  ``down_weight`` (E, N2, moe_dim//2), ``gate_up_expert_scales`` (L1
  per-expert output scaling), ``down_expert_scales`` (L2 per-expert output
  scaling), ``c_input_scales`` (per-expert input scale of the NVFP4
  re-quant), ``expert_start_indices`` (per-expert prefix-sum offsets),
  ``expert_ids`` (-1 = masked), ``a_scale_offsets`` (per-expert scale-block
  offsets), ``src_info`` (per-row metadata that leads back to the source).
  Parameters: ``clamp_activation`` (the clamped L1 activation).
* flashinfer.megamoe.MegaMoESymmBuffer, Parameters: ``activation_clamp`` (the
  SwiGLU clamp value, 10.0 by default); staging views: E4M3 x with FP32
  [.., hidden // 128] scales, INT64 topk_idx, FP32 topk_weights.
* flashinfer.fused_moe.MoEActivationPack: NVFP4 activations (packed uint8
  [M, H/2] + float8_e4m3fn [M, H/16] block scales); ``FromLogits`` routing
  with a ``routing_bias`` for bias-aware methods.
* DistributedEPCombine, Args: ``router_weights`` scale each expert's
  contribution; the combine reduces the expert rows back to their tokens.

Readings taken where the pages are silent (each one is listed with its
reasoning in the design notes of the repository):

* Routing: select on score = fp32(logit + bias), descending, ties to the lower
  expert index, NaN scores last; the weights are the softmax of the
  *unbiased* logits over the chosen k.
* Permutation: stable in the flat slot index; ``src_info[row] = t*k + j``.
* ``topk_idx == -1`` is a skipped slot (the masked-id convention of
  ``expert_ids``); duplicates within a token are independent slots.
* Activation: h = min(g,c) * sigmoid(min(g,c)) * clamp(u,-c,c); c = +inf is
  the textbook SwiGLU (or the clamped swigluoai, see ``swigluoai``).  Gate
  rows are W13[e, :I], up rows are W13[e, I:].
* Re-quant of h (computed in float64, then held in float32 as the kernel
  holds it): NVFP4 per 16 values along I with an E4M3 block scale and the
  per-expert FP32 ``c_input_scales`` G as the dequant multiplier; FP8 per 128
  values with an FP32 scale amax/448; MXFP8 per 32 values with a power-of-two
  scale; FP8 per-tensor against the per-expert G; BF16 by
  round-to-nearest-even.  The
  FP32 steps of the quantisers are fixed (see ``requant``) so that a code is
  decided in the same precision on both sides.
* NVFP4 GEMMs: the MMA sums products of (e2m1 x e4m3 block scale) operands,
  then the per-expert scale (``gate_up_expert_scales`` or
  ``down_expert_scales``) multiplies the sum.  FP8, FP8 per-tensor and MXFP8
  GEMMs: every operand is its E4M3 code times its scale.
* The output is BF16, rounded once from the float64 sum (via float32).
"""

import numpy as np

from . import formats as F

FORMATS = ("bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor")


# ----------------------------------------------------------------------------
# Routing (flashinfer.fused_moe.MoEActivationPack, routing_input_mode FromLogits)
# ----------------------------------------------------------------------------

def route(logits, bias, k):
    """Top-k expert selection from router logits, bias used for selection only.

    Returns (topk_idx int64 [M, k], topk_weights float64 [M, k]).
    Slots are ordered by selection score, highest first.
    """
    l32 = np.asarray(logits, dtype=np.float32)
    M, E = l32.shape
    if not (1 <= k <= E):
        raise ValueError("num_topk must be in [1, num_experts]")
    b32 = np.zeros(E, np.float32) if bias is None else np.asarray(bias, np.float32)
    score = l32 + b32[None, :]                      # one IEEE float32 add
    nan = np.isnan(score)
    key = np.where(nan, -np.inf, score).astype(np.float64)
    ids = np.broadcast_to(np.arange(E), (M, E))
    # lexsort: the last key is the primary one.
    order = np.lexsort((ids, -key, nan), axis=-1)
    topk_idx = order[:, :k].astype(np.int64)
    chosen = np.take_along_axis(l32, topk_idx, axis=1).astype(np.float64)
    # a token with a non-finite chosen logit has no softmax value: its
    # weights come out NaN here and are unspecified at the boundary
    with np.errstate(invalid="ignore"):
        z = np.exp(chosen - chosen.max(axis=1, keepdims=True))
        topk_weights = z / z.sum(axis=1, keepdims=True)
    return topk_idx, topk_weights


# ----------------------------------------------------------------------------
# Permutation (Struct_mega_ffn_ep_combine_send: expert_start_indices, expert_ids,
# a_scale_offsets, src_info, num_active_experts)
# ----------------------------------------------------------------------------

def check_indices(topk_idx, num_experts):
    idx = np.asarray(topk_idx)
    if idx.size and (idx.min() < -1 or idx.max() >= num_experts):
        raise ValueError("topk_idx out of range [-1, num_experts)")


def permute(topk_idx, num_experts, scale_block_rows=128):
    """Group the routed slots by expert, stably in the flat slot index.

    Returns a dict of int64 arrays:
      expert_counts [E]          valid slots per expert
      expert_start_indices [E+1] exclusive prefix sum of the counts
      src_info [R_valid]         flat slot index s = t*k + j of each row
      slot_to_row [M*k]          row of each slot, -1 for a skipped slot
      expert_ids [E]             active experts ascending, -1 padded
      num_active                 number of experts with at least one slot
      a_scale_offsets [E+1]      prefix sum of counts rounded up to 128 rows
    """
    check_indices(topk_idx, num_experts)
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    E = num_experts
    counts = np.zeros(E, np.int64)
    for e in range(E):
        counts[e] = np.count_nonzero(flat == e)
    starts = np.zeros(E + 1, np.int64)
    starts[1:] = np.cumsum(counts)
    src_info = np.zeros(int(starts[-1]), np.int64)
    slot_to_row = np.full(flat.shape[0], -1, np.int64)
    for e in range(E):
        slots = np.nonzero(flat == e)[0]            # ascending slot index
        rows = starts[e] + np.arange(slots.shape[0])
        src_info[rows] = slots
        slot_to_row[slots] = rows
    active = np.nonzero(counts > 0)[0]
    expert_ids = np.full(E, -1, np.int64)
    expert_ids[: active.shape[0]] = active
    padded = -(-counts // scale_block_rows) * scale_block_rows
    a_scale_offsets = np.zeros(E + 1, np.int64)
    a_scale_offsets[1:] = np.cumsum(padded)
    return dict(expert_counts=counts, expert_start_indices=starts,
                src_info=src_info, slot_to_row=slot_to_row,
                expert_ids=expert_ids, num_active=int(active.shape[0]),
                a_scale_offsets=a_scale_offsets)


# ----------------------------------------------------------------------------
# Decoding of activations and expert weights
# ----------------------------------------------------------------------------

def decode_x(fmt, x, x_scale, H, rows=None, row_scale=None):
    """Activations [M, H] -> float64.

    fp8: E4M3 codes times the FP32 per-128 block scale of the token.
    fp8_tensor: E4M3 codes times the one FP32 dequantisation scale of the
    whole activation tensor (x_scale of shape [1]).
    mxfp8: E4M3 codes times the UE8M0 per-32 block scale of the token.
    nvfp4: e2m1 codes times the E4M3 per-16 block scale, times the token's
    BF16 rowwise scale when the activations were quantised per token
    (``row_scale``, see quantize_nvfp4_rowwise); the static global scale is
    carried by the per-expert L1 output scaling instead.
    """
    x = np.asarray(x)
    if fmt == "fp8_tensor":
        x = x if rows is None else x[rows]
        return F.e4m3_decode(x) * float(np.asarray(x_scale, np.float32).reshape(-1)[0])
    if rows is not None:
        x = x[rows]
        x_scale = None if x_scale is None else np.asarray(x_scale)[rows]
        row_scale = None if row_scale is None else np.asarray(row_scale)[rows]
    if fmt == "bf16":
        return F.bf16_decode(x)
    if fmt == "fp8":
        s = np.asarray(x_scale, np.float32).astype(np.float64)
        return F.e4m3_decode(x) * np.repeat(s, 128, axis=1)
    if fmt == "mxfp8":
        return F.e4m3_decode(x) * np.repeat(F.ue8m0_decode(x_scale), 32, axis=1)
    if fmt == "nvfp4":
        codes = F.fp4_unpack(x, H)
        s = F.e4m3_decode(x_scale)
        v = F.e2m1_decode(codes) * np.repeat(s, 16, axis=1)
        if row_scale is not None:
            v = v * F.bf16_decode(np.asarray(row_scale, np.uint16))[:, None]
        return v
    raise ValueError(fmt)


# The largest E4M3 block scale times the largest E2M1 code: a token whose
# largest magnitude is rowmax is quantised against 2688 / rowmax.
NVFP4_ROW_RANGE = 448.0 * 6.0


def quantize_nvfp4_rowwise(x):
    """Per-token dynamic NVFP4 quantisation of activations (EPConfig,
    ``nvfp4_dyn_global_scales``): each token is quantised against its own
    global scale 2688 / rowmax instead of a static one, and the scale's BF16
    inverse travels with the token as its rowwise scale, so a row dequantises
    as e2m1 * block_scale * rowwise_scale.

    x: float activations [M, H] (FP32 values, e.g. decoded BF16).  Per token:
      rowmax = max |x[t]|;  G = fp32(rowmax / 2688), the dequant multiplier;
      blocks of 16 then follow the same steps as the intermediate's re-quant
      (``requant`` with G): sf = e4m3(amax_b / (6 G)), q = e2m1(x / (sf G));
      rowwise scale = bf16_rn(G).  An all-zero token gives zero codes, scales
      and rowwise scale.
    Returns dict(codes uint8 [M, H/2], scales uint8 E4M3 [M, H/16],
    rowwise uint16 BF16 [M]).
    """
    x32 = np.asarray(x, np.float32)
    M, H = x32.shape
    codes = np.zeros((M, H // 2), np.uint8)
    scales = np.zeros((M, H // 16), np.uint8)
    rowwise = np.zeros(M, np.uint16)
    for t in range(M):
        rowmax = np.float32(np.max(np.abs(x32[t]))) if H else np.float32(0)
        if rowmax == 0:
            continue
        G = np.float32(rowmax / np.float32(NVFP4_ROW_RANGE))
        rq = requant("nvfp4", x32[t:t + 1], G)
        codes[t] = rq["codes"][0]
        scales[t] = rq["scales"][0]
        rowwise[t] = F.bf16_encode(np.array([G], np.float32))[0]
    return dict(codes=codes, scales=scales, rowwise=rowwise)


def decode_weight(fmt, w, w_scale, e, n_rows, k_cols):
    """Expert e's weight [n_rows, k_cols] (K-major, as stored) -> float64.

    fp8 scales are per 128 x 128 block; fp8_tensor has one FP32 scale per
    expert's matrix (w_scale [E]); mxfp8 (UE8M0) scales per 1 x 32 block;
    nvfp4 scales per 1 x 16 block.
    """
    if fmt == "bf16":
        return F.bf16_decode(np.asarray(w)[e])
    if fmt == "fp8":
        s = np.asarray(w_scale, np.float32)[e].astype(np.float64)
        full = np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)
        return F.e4m3_decode(np.asarray(w)[e]) * full
    if fmt == "fp8_tensor":
        return F.e4m3_decode(np.asarray(w)[e]) * float(np.asarray(w_scale, np.float32)[e])
    if fmt == "mxfp8":
        return F.e4m3_decode(np.asarray(w)[e]) * np.repeat(F.ue8m0_decode(np.asarray(w_scale)[e]), 32, axis=1)
    if fmt == "nvfp4":
        codes = F.fp4_unpack(np.asarray(w)[e], k_cols)
        s = F.e4m3_decode(np.asarray(w_scale)[e])
        return F.e2m1_decode(codes) * np.repeat(s, 16, axis=1)
    raise ValueError(fmt)


# ----------------------------------------------------------------------------
# The expert FFN
# ----------------------------------------------------------------------------

def clamped_swiglu(g, u, clamp):
    """h = min(g, c) * sigmoid(min(g, c)) * clamp(u, -c, c), in float64.

    flashinfer.megamoe.MegaMoESymmBuffer, ``activation_clamp``: the SwiGLU
    clamp value; Struct_mega_ffn_ep_combine_send, ``clamp_activation``.
    The gate is clamped from above only, the up branch on both sides.
    """
    c = float(clamp)
    g = np.minimum(g, c)
    u = np.clip(u, -c, c)
    return g / (1.0 + np.exp(-g)) * u


def swigluoai(g, u, clamp, alpha):
    """h = min(g, c) * sigmoid(alpha * min(g, c)) * (clamp(u, -c, c) + 1), in
    float64.

    Struct_mega_ffn_ep_combine_send, ``clamp_activation``: the clamped
    ("swigluoai") L1 activation; its constants come from the dispatch code.  Read
    as the SwiGLU variant with a sigmoid slope alpha on the gate and a bias of
    1 on the up branch (the pages print neither; alpha is an input), with the
    same clamps as clamped_swiglu: the gate from above, the up branch on both
    sides.
    """
    c = float(clamp)
    a = float(alpha)
    g = np.minimum(g, c)
    u = np.clip(u, -c, c)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-a * g)) * (u + 1.0)


def activation(problem, g, u):
    """The L1 activation the problem selects: "swiglu" (the default, the
    clamped SwiGLU) or "swigluoai" with slope problem["activation_alpha"]."""
    clamp = problem.get("activation_clamp", 10.0)
    if problem.get("activation", "swiglu") == "swigluoai":
        return swigluoai(g, u, clamp, problem["activation_alpha"])
    return clamped_swiglu(g, u, clamp)


def gate_up(fmt, xhat, w13hat, alpha1, I):
    """L1: g = x^ W1^T, u = x^ W3^T with W1 = W13[:I], W3 = W13[I:]; NVFP4 scaled by alpha1."""
    acc = xhat @ w13hat.T
    if fmt == "nvfp4":
        acc = acc * float(np.float32(alpha1))
    return acc[:, :I], acc[:, I:]


def requant(fmt, h32, G=None):
    """Re-quantise the FP32 intermediate h [rows, I] to the L2 input format.

    Returns dict(codes, scales, hhat, pre, pre_scale): hhat float64 = the
    dequantised value the down GEMM sees (for NVFP4 without the global G,
    which the L2 output scaling carries); pre = the FP32 value each element
    code is rounded from (h itself for BF16, h * inv for FP8 and NVFP4);
    pre_scale = the FP32 value each NVFP4 block-scale code is rounded from
    (amax / (6 G)), None otherwise.

    nvfp4, per block of 16 along I (all steps FP32, round to nearest):
        sf   = e4m3_satfinite(amax / (6 * G))
        q    = e2m1_satfinite(h * (1 / (sf * G)))      (q = 0 where sf == 0)
    fp8, per block of 128 along I:
        s    = amax / 448
        q    = e4m3_satfinite(h * (1 / s))             (q = 0, s = 0 where amax == 0)
    bf16:  q = bf16_rn(h)
    mxfp8, per block of 32 along I (the OCP microscaling rule; E8M0 scales
    carry no per-expert input scale):
        X    = floor(log2(amax)) - 8, clamped to [-127, 127]  (8: the largest
               E4M3 exponent; X = -127 where amax == 0)
        q    = e4m3_satfinite(h * 2**-X)      (exact power-of-two scaling)
        scale code = X + 127
    fp8_tensor, one static scale per expert (the per-tensor FP8 encoding of
    MoEActivationPack read with the static re-quant scale of
    Struct_mega_ffn_ep_combine_send, c_input_scales = G, a dequant
    multiplier):
        q    = e4m3_satfinite(h * (1 / G))     (FP32 steps)
        hhat = q * G                           (scales = G per row)
    """
    h32 = np.asarray(h32, np.float32)
    rows, I = h32.shape
    if fmt == "bf16":
        codes = F.bf16_encode(h32)
        return dict(codes=codes, scales=None, hhat=F.bf16_decode(codes), pre=h32, pre_scale=None)
    if fmt == "fp8":
        blk = h32.reshape(rows, I // 128, 128)
        amax = np.max(np.abs(blk), axis=2)                          # float32
        s = (amax / np.float32(448.0)).astype(np.float32)
        with np.errstate(divide="ignore"):
            inv = (np.float32(1.0) / s).astype(np.float32)
        v = (blk * inv[:, :, None]).astype(np.float32)
        codes = F.e4m3_encode(v)
        codes = np.where((s == 0)[:, :, None], np.uint8(0), codes).reshape(rows, I)
        hhat = F.e4m3_decode(codes).reshape(rows, I // 128, 128) * s[:, :, None].astype(np.float64)
        return dict(codes=codes, scales=s, hhat=hhat.reshape(rows, I), pre=v.reshape(rows, I), pre_scale=None)
    if fmt == "fp8_tensor":
        G32 = np.float32(G)
        inv = np.float32(np.float32(1.0) / G32)
        v = (h32 * inv).astype(np.float32)
        codes = F.e4m3_encode(v)
        hhat = F.e4m3_decode(codes) * float(G32)
        return dict(codes=codes, scales=np.full(rows, G32, np.float32), hhat=hhat, pre=v, pre_scale=None)
    if fmt == "mxfp8":
        blk = h32.reshape(rows, I // 32, 32)
        amax = np.max(np.abs(blk), axis=2).astype(np.float64)
        with np.errstate(divide="ignore"):
            X = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
        X = np.clip(X, -127, 127).astype(np.int64)
        v = blk.astype(np.float64) * np.ldexp(1.0, -X)[:, :, None]   # exact
        codes = F.e4m3_encode(v).reshape(rows, I)
        sc = (X + 127).astype(np.uint8)
        hhat = F.e4m3_decode(codes).reshape(rows, I // 32, 32) * F.ue8m0_decode(sc)[:, :, None]
        return dict(codes=codes, scales=sc, hhat=hhat.reshape(rows, I), pre=v.reshape(rows, I).astype(np.float32),
                    pre_scale=None)
    if fmt == "nvfp4":
        G32 = np.float32(G)
        blk = h32.reshape(rows, I // 16, 16)
        amax = np.max(np.abs(blk), axis=2)
        denom = np.float32(np.float32(6.0) * G32)
        sf_pre = (amax / denom).astype(np.float32)
        sf_code = F.e4m3_encode(sf_pre)
        sf = F.e4m3_decode(sf_code).astype(np.float32)
        sg = (sf * G32).astype(np.float32)
        with np.errstate(divide="ignore"):
            inv = (np.float32(1.0) / sg).astype(np.float32)
        v = (blk * inv[:, :, None]).astype(np.float32)
        q = F.e2m1_encode(v)
        q = np.where((sf == 0)[:, :, None], np.uint8(0), q).reshape(rows, I)
        hhat = (F.e2m1_decode(q).reshape(rows, I // 16, 16)
                * sf[:, :, None].astype(np.float64)).reshape(rows, I)
        return dict(codes=F.fp4_pack(q), scales=sf_code, hhat=hhat, pre=v.reshape(rows, I), pre_scale=sf_pre)
    raise ValueError(fmt)


def dequant_intermediate(fmt, codes, scales, I):
    """Decode re-quantised intermediate rows (as ``requant`` returns them) to float64."""
    if fmt == "bf16":
        return F.bf16_decode(codes)
    if fmt == "fp8":
        s = np.asarray(scales, np.float32).astype(np.float64)
        return F.e4m3_decode(codes) * np.repeat(s, 128, axis=1)
    if fmt == "fp8_tensor":
        return F.e4m3_decode(codes) * np.asarray(scales, np.float32).astype(np.float64).reshape(-1, 1)
    if fmt == "mxfp8":
        return F.e4m3_decode(codes) * np.repeat(F.ue8m0_decode(scales), 32, axis=1)
    if fmt == "nvfp4":
        q = F.fp4_unpack(codes, I)
        return F.e2m1_decode(q) * np.repeat(F.e4m3_decode(scales), 16, axis=1)
    raise ValueError(fmt)


def down(fmt, hhat, w2hat, alpha2):
    """L2: y = h^ W2^T; NVFP4 scaled by alpha2 (``down_expert_scales``)."""
    y = hhat @ w2hat.T
    if fmt == "nvfp4":
        y = y * float(np.float32(alpha2))
    return y


def _expert_scale(inputs, name, e):
    arr = inputs.get(name)
    return None if arr is None else np.asarray(arr, np.float32)[e]


def shared_expert_slots(topk_idx, topk_weights, num_experts):
    """EPConfig fused_shared_expert / DistributedEPCombine fused_shared_expert:
    the shared expert's computation is fused with the routed experts'.  Read
    as one more expert, index num_experts (after the routed ones, same shapes),
    that every token goes through with router weight 1: each token's slot list
    gains a last column (num_experts, 1.0) after its k routed slots."""
    idx = np.asarray(topk_idx, np.int64)
    w = np.asarray(topk_weights, np.float32)
    M = idx.shape[0]
    return (np.concatenate([idx, np.full((M, 1), num_experts, np.int64)], axis=1),
            np.concatenate([w, np.ones((M, 1), np.float32)], axis=1))


def moe_forward(problem, inputs, topk_idx, topk_weights, tokens=None,
                keep_intermediate=False, hhat_override=None):
    """The routed MoE FFN by its per-token definition.

    problem: dict(hidden, intermediate_hidden, num_experts, num_topk,
                  activation_clamp, format, optional shared_expert,
                  optional activation ("swiglu" | "swigluoai") and
                  activation_alpha)
             With shared_expert = 1 the weights hold num_experts + 1 experts
             (the last one shared) and topk_idx / topk_weights carry the
             shared slot (shared_expert_slots).
    inputs:  dict(x, x_scale, w13, w13_scale, w2, w2_scale,
                  gate_up_expert_scales, down_expert_scales, c_input_scales,
                  and for NVFP4 quantised per token, x_row_scale: BF16 [M])
    tokens:  optional subset of token indices (every quantity here is per
             token, so a subset is computed exactly as in the full problem).
    hhat_override: optional callable (e, t_array, j_array) -> float64 rows
             that replaces the oracle's own re-quantised intermediate (used to
             recompute L2 and the combine from another implementation's codes).

    Returns dict(out_f64 [T, H], out_bf16 uint16 [T, H], and, when
    keep_intermediate, per-slot h32 / codes / scales keyed by (t, j)).
    """
    fmt = problem["format"]
    H = problem["hidden"]
    I = problem["intermediate_hidden"]
    E = problem["num_experts"] + int(problem.get("shared_expert", 0))
    idx = np.asarray(topk_idx, np.int64)
    w = np.asarray(topk_weights, np.float32).astype(np.float64)
    check_indices(idx, E)
    tok = np.arange(idx.shape[0]) if tokens is None else np.asarray(tokens, np.int64)
    idx_t = idx[tok]
    w_t = w[tok]
    xhat = decode_x(fmt, inputs["x"], inputs.get("x_scale"), H, rows=tok, row_scale=inputs.get("x_row_scale"))
    out = np.zeros((tok.shape[0], H), np.float64)
    inter = {} if keep_intermediate else None
    for e in range(E):
        ti, sj = np.nonzero(idx_t == e)             # ascending (token, slot)
        if ti.shape[0] == 0:
            continue
        w13hat = decode_weight(fmt, inputs["w13"], inputs.get("w13_scale"), e, 2 * I, H)
        w2hat = decode_weight(fmt, inputs["w2"], inputs.get("w2_scale"), e, H, I)
        g, u = gate_up(fmt, xhat[ti], w13hat, _expert_scale(inputs, "gate_up_expert_scales", e), I)
        h32 = activation(problem, g, u).astype(np.float32)
        rq = requant(fmt, h32, _expert_scale(inputs, "c_input_scales", e))
        hhat = rq["hhat"] if hhat_override is None else hhat_override(e, tok[ti], sj)
        y = down(fmt, hhat, w2hat, _expert_scale(inputs, "down_expert_scales", e))
        np.add.at(out, ti, w_t[ti, sj][:, None] * y)
        if keep_intermediate:
            for n in range(ti.shape[0]):
                key = (int(tok[ti[n]]), int(sj[n]))
                inter[key] = dict(expert=e, h32=h32[n],
                                  codes=rq["codes"][n],
                                  scales=None if rq["scales"] is None else rq["scales"][n],
                                  pre=rq["pre"][n],
                                  pre_scale=None if rq["pre_scale"] is None else rq["pre_scale"][n])
    res = dict(out_f64=out, out_bf16=F.bf16_encode(out.astype(np.float32)))
    if keep_intermediate:
        res["intermediate"] = inter
    return res
