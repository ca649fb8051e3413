"""A routed-MoE layer object over the C ABI: owns the device workspace and the
prepared weight blobs (the tensor-core tile layout ``moe_prepare_weights``
writes once, NVFP4 scale tiles included), and forwards calls to ``api``.

torch supplies device memory and streams only; every step runs in the
library's kernels.
"""

import torch

from . import api


def _i32(n, device):
    return torch.empty(max(int(n), 1), dtype=torch.int32, device=device)


class LayoutBuffers:
    """Caller-owned device arrays of ``moe_layout_t`` for one problem size."""

    def __init__(self, M, k, E, device):
        R = M * k
        self.expert_counts = _i32(E, device)
        self.expert_start_indices = _i32(E + 1, device)
        self.src_info = _i32(R, device)
        self.slot_to_row = _i32(R, device)
        self.expert_ids = _i32(E, device)
        self.num_active = _i32(1, device)
        self.a_scale_offsets = _i32(E + 1, device)
        self.tile_offsets = _i32(E + 1, device)
        self.struct = api.layout(self.expert_counts, self.expert_start_indices, self.src_info,
                                 self.slot_to_row, self.expert_ids, self.num_active,
                                 self.a_scale_offsets, self.tile_offsets)

    def host(self):
        return {k: getattr(self, k).cpu().numpy() for k in (
            "expert_counts", "expert_start_indices", "src_info", "slot_to_row", "expert_ids",
            "num_active", "a_scale_offsets", "tile_offsets")}


class MoELayer:
    """One routed-MoE FFN layer on one GPU.

    p:       problem dict (hidden, intermediate_hidden, num_experts, num_topk,
             activation_clamp, format, num_tokens = the largest batch served)
    weights: dict of device tensors w13, w13_scale, w2, w2_scale and, for
             NVFP4, gate_up_expert_scales, down_expert_scales, c_input_scales
             (FP8 per-tensor: c_input_scales) in the logical layouts of
             include/moe.h; the weights are prepared here
    p may also carry "shared_expert" (0/1), "activation" ("swiglu" |
    "swigluoai") and "activation_alpha"
    p may also carry "tile_regime" ("auto", "large_m", "small_m")
    """

    def __init__(self, p, weights, device=None, fast_math=1):
        self.p = dict(p)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.fast_math = fast_math
        api.init(self.device.index if self.device.index is not None else 0)
        self.max_tokens = int(p["num_tokens"])
        # a fused shared expert (p["shared_expert"] = 1) is one more expert
        # and one more slot per token after the routing
        self.shared = int(p.get("shared_expert", 0))
        self.k_all = int(p["num_topk"]) + self.shared
        self.E_all = int(p["num_experts"]) + self.shared
        self.prob = api.problem_from_dict(self.p, fast_math=fast_math)
        w = weights
        self.alpha1 = w.get("gate_up_expert_scales")
        self.alpha2 = w.get("down_expert_scales")
        self.c_in = w.get("c_input_scales")
        # FP8 block and per-tensor scales stay logical; NVFP4 and MXFP8 scales
        # go into the prepared blobs
        keep = self.p["format"] in ("fp8", "fp8_tensor")
        self.w13_scale = w.get("w13_scale") if keep else None
        self.w2_scale = w.get("w2_scale") if keep else None
        n13, n2 = api.prepared_weights_size(self.prob)
        self.w13 = torch.empty(n13, dtype=torch.uint8, device=self.device)
        self.w2 = torch.empty(n2, dtype=torch.uint8, device=self.device)
        logical = api.weights(w["w13"], w.get("w13_scale"), w["w2"], w.get("w2_scale"))
        api.prepare_weights(self.prob, logical, self.w13, self.w2)
        self.weights = api.weights(self.w13, self.w13_scale, self.w2, self.w2_scale,
                                   self.alpha1, self.alpha2, self.c_in)
        self.ws_bytes = api.workspace_size(self.prob)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        api.workspace_init(self.ws, self.ws_bytes)

    def problem(self, M):
        if M > self.max_tokens:
            raise ValueError(f"{M} tokens > the {self.max_tokens} this layer was sized for")
        return api.problem_from_dict(self.p, num_tokens=M, fast_math=self.fast_math)

    def forward(self, x, x_scale=None, topk_idx=None, topk_weights=None, logits=None, bias=None,
                out=None, stream=None, x_rowwise_scale=None):
        """moe_fused: the whole layer, BF16 out [M, H]."""
        M = x.shape[0]
        if out is None:
            out = torch.empty((M, self.p["hidden"]), dtype=torch.bfloat16, device=self.device)
        api.fused(self.problem(M), api.act(x, x_scale, x_rowwise_scale), self.weights, out, self.ws,
                  self.ws_bytes, topk_idx=topk_idx, topk_weights=topk_weights, logits=logits, bias=bias,
                  stream=stream)
        return out

    def quantize_rowwise(self, x_bf16, stream=None):
        """Per-token dynamic NVFP4 quantisation of BF16 activations [M, H]:
        (codes uint8 [M, H/2], block scales E4M3 [M, H/16], rowwise BF16 [M])."""
        M, H = x_bf16.shape
        codes = torch.empty((M, H // 2), dtype=torch.uint8, device=self.device)
        scales = torch.empty((M, H // 16), dtype=torch.uint8, device=self.device)
        rowwise = torch.empty((M,), dtype=torch.int16, device=self.device)
        api.quantize_nvfp4_rowwise(self.problem(M), x_bf16, codes, scales, rowwise, stream=stream)
        return codes, scales, rowwise

    def shared_slots(self, topk_idx, topk_weights):
        """Precomputed routing [M, k] -> [M, k + 1]: the shared expert's slot
        (index num_experts, weight 1) appended, as every call after the
        routing expects when the layer has a shared expert."""
        if not self.shared:
            return topk_idx, topk_weights
        M = topk_idx.shape[0]
        idx = torch.cat([topk_idx, torch.full((M, 1), self.p["num_experts"], dtype=topk_idx.dtype,
                                              device=topk_idx.device)], dim=1)
        w = torch.cat([topk_weights, torch.ones((M, 1), dtype=topk_weights.dtype, device=topk_weights.device)],
                      dim=1)
        return idx.contiguous(), w.contiguous()

    def route(self, logits, bias=None, stream=None):
        M = logits.shape[0]
        k = self.k_all
        idx = torch.empty((M, k), dtype=torch.int64, device=self.device)
        w = torch.empty((M, k), dtype=torch.float32, device=self.device)
        api.route(self.problem(M), logits, bias, idx, w, stream=stream)
        return idx, w

    def permute(self, topk_idx, stream=None):
        M = topk_idx.shape[0]
        lay = LayoutBuffers(M, self.k_all, self.E_all, self.device)
        api.permute(self.problem(M), topk_idx, lay.struct, self.ws, self.ws_bytes, stream=stream)
        return lay

    def ffn(self, x, x_scale, lay, topk_weights, out_mode=api.MOE_OUT_ACCUMULATE, keep_intermediate=False,
            stream=None, x_rowwise_scale=None):
        """moe_ffn; returns (out fp32, intermediate bytes or None)."""
        M = x.shape[0]
        prob = self.problem(M)
        H = self.p["hidden"]
        rows = M if out_mode == api.MOE_OUT_ACCUMULATE else M * self.k_all
        out = torch.empty((rows, H), dtype=torch.float32, device=self.device)
        inter = None
        if keep_intermediate:
            n, _ = api.intermediate_size(prob)
            inter = torch.empty(n, dtype=torch.uint8, device=self.device)
        api.ffn(prob, api.act(x, x_scale, x_rowwise_scale), self.weights, lay.struct, topk_weights, out_mode, out,
                self.ws, self.ws_bytes, intermediate=inter, stream=stream)
        return out, inter

    def combine(self, lay, topk_weights, inp, in_mode, M, stream=None):
        out = torch.empty((M, self.p["hidden"]), dtype=torch.bfloat16, device=self.device)
        api.combine(self.problem(M), lay.struct if lay is not None else None, topk_weights, inp, in_mode,
                    out, stream=stream)
        return out

    def workspace_views(self, M):
        """Device views of what the last moe_fused call with M tokens left in
        the workspace (layout arrays, in-kernel routing, the re-quantised
        intermediate and its scales, the FP32 accumulator), for inspection.
        Read them only after that call has completed."""
        prob = self.problem(M)
        off = api.workspace_offsets(prob)
        k, E, H = self.k_all, self.E_all, self.p["hidden"]
        R = M * k
        n_int, so = api.intermediate_size(prob)
        ws = self.ws

        def i32(name, n):
            return ws[off[name]: off[name] + 4 * n].view(torch.int32)

        v = {name: i32(name, n) for name, n in (
            ("expert_counts", E), ("expert_start_indices", E + 1), ("src_info", R), ("slot_to_row", R),
            ("expert_ids", E), ("num_active", 1), ("a_scale_offsets", E + 1), ("tile_offsets", E + 1))}
        v["topk_idx"] = ws[off["topk_idx"]: off["topk_idx"] + 8 * R].view(torch.int64).view(M, k)
        v["topk_weights"] = ws[off["topk_weights"]: off["topk_weights"] + 4 * R].view(torch.float32).view(M, k)
        v["intermediate"] = ws[off["intermediate"]: off["intermediate"] + so]
        v["intermediate_scales"] = ws[off["intermediate_scales"]: off["intermediate_scales"] + (n_int - so)]
        v["scale_rows"] = off["scale_rows"]
        v["accumulator"] = ws[off["accumulator"]: off["accumulator"] + 4 * M * H].view(torch.float32).view(M, H)
        return v

    def status(self, stream=None):
        return api.read_status(self.ws, stream=stream)

    def check_status(self, stream=None):
        code = self.status(stream)
        if code != api.MOE_OK:
            raise api.MoEError("device status", code)

    def clear_status(self, stream=None):
        api.workspace_init(self.ws, self.ws_bytes, stream=stream)
