"""ctypes binding of ``include/moe.h`` (``libmoe_b200.so``).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensor arguments may be torch tensors (their ``data_ptr()``
is passed), plain integers (raw device addresses) or ``None`` (NULL).
Streams are torch streams, raw ``cudaStream_t`` integers, or ``None`` for
torch's current stream.

The library is loaded on first use from this package directory; a missing
library raises ``RuntimeError`` -- there is no fallback of any kind.
"""

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(_HERE, LIB_NAME)

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_BAD_INDEX = 5
MOE_ERR_TIMEOUT = 6

FORMATS = {"bf16": 0, "fp8": 1, "nvfp4": 2, "mxfp8": 3, "fp8_tensor": 4}

MOE_OUT_ACCUMULATE = 0
MOE_OUT_STAGED = 1
MOE_IN_ACCUMULATED = 0
MOE_IN_STAGED = 1

# Every entry point declared in include/moe.h.
EXPORTS = (
    "moe_init", "moe_get_workspace_size", "moe_workspace_init", "moe_prepare_weights",
    "moe_get_prepared_weights_size",
    "moe_route", "moe_permute", "moe_ffn", "moe_get_intermediate_size", "moe_combine",
    "moe_fused", "moe_read_status", "moe_status_string", "moe_timing_enable", "moe_timing_read",
    "moe_permute_noalloc", "moe_get_tile_regime", "moe_get_workspace_offsets",
    "moe_workspace_test_hooks", "moe_quantize_nvfp4_rowwise",
)

SLOTS = ("route", "permute", "gather", "gemm1", "zero", "gemm2", "finalize", "combine", "fused")


class MoEError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} returned {status_string(code)} ({code})")


class Problem(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("hidden", ctypes.c_int32),
        ("intermediate_hidden", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("num_topk", ctypes.c_int32),
        ("activation_clamp", ctypes.c_float),
        ("format", ctypes.c_int32),
        ("fast_math", ctypes.c_int32),
        ("tile_regime", ctypes.c_int32),
        ("shared_expert", ctypes.c_int32),
        ("activation", ctypes.c_int32),
        ("activation_alpha", ctypes.c_float),
    ]


class Act(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_scale", ctypes.c_void_p), ("x_rowwise_scale", ctypes.c_void_p)]


class Weights(ctypes.Structure):
    _fields_ = [
        ("w13", ctypes.c_void_p), ("w13_scale", ctypes.c_void_p),
        ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p),
        ("gate_up_expert_scales", ctypes.c_void_p),
        ("down_expert_scales", ctypes.c_void_p),
        ("c_input_scales", ctypes.c_void_p),
    ]


class Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "expert_counts", "expert_start_indices", "src_info", "slot_to_row",
        "expert_ids", "num_active", "a_scale_offsets", "tile_offsets")]


WS_OFFSET_FIELDS = ("status", "topk_idx", "topk_weights", "expert_counts", "expert_start_indices",
                    "src_info", "slot_to_row", "expert_ids", "num_active", "a_scale_offsets",
                    "tile_offsets", "intermediate", "intermediate_scales", "scale_rows", "accumulator")


class WorkspaceOffsets(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64 if n == "scale_rows" else ctypes.c_size_t) for n in WS_OFFSET_FIELDS]


_lib = None


def lib():
    """The loaded library (loads it on first call; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run __graft_entry__.build() "
                               "(or python -m mixture_experts_routed_03_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        P = ctypes.POINTER(Problem)
        sig = {
            "moe_init": [ctypes.c_int],
            "moe_get_workspace_size": [P, ctypes.POINTER(sz)],
            "moe_workspace_init": [vp, sz, vp],
            "moe_workspace_test_hooks": [vp, sz, i32, i32, vp],
            "moe_quantize_nvfp4_rowwise": [P, vp, vp, vp, vp, vp],
            "moe_prepare_weights": [P, ctypes.POINTER(Weights), vp, vp, vp],
            "moe_get_prepared_weights_size": [P, ctypes.POINTER(sz), ctypes.POINTER(sz)],
            "moe_route": [P, vp, vp, vp, vp, vp],
            "moe_permute": [P, vp, ctypes.POINTER(Layout), vp, sz, vp],
            "moe_ffn": [P, ctypes.POINTER(Act), ctypes.POINTER(Weights), ctypes.POINTER(Layout),
                        vp, i32, vp, vp, vp, sz, vp],
            "moe_get_intermediate_size": [P, ctypes.POINTER(sz), ctypes.POINTER(sz)],
            "moe_get_tile_regime": [P, ctypes.POINTER(i32)],
            "moe_get_workspace_offsets": [P, ctypes.POINTER(WorkspaceOffsets)],
            "moe_combine": [P, ctypes.POINTER(Layout), vp, vp, i32, vp, vp],
            "moe_fused": [P, ctypes.POINTER(Act), ctypes.POINTER(Weights), vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_read_status": [vp, vp],
            "moe_timing_enable": [ctypes.c_int, ctypes.c_int],
            "moe_permute_noalloc": [P, vp, ctypes.POINTER(Layout), vp, vp],
            "moe_timing_read": [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code):
    try:
        return lib().moe_status_string(int(code)).decode()
    except RuntimeError:
        return str(code)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, code):
    if code != MOE_OK:
        raise MoEError(fn, code)


TILE_REGIMES = {"auto": 0, "large_m": 1, "small_m": 2}
ACTIVATIONS = {"swiglu": 0, "swigluoai": 1}


def problem(num_tokens, hidden, intermediate_hidden, num_experts, num_topk,
            activation_clamp=10.0, format="bf16", fast_math=1, tile_regime="auto", shared_expert=0,
            activation="swiglu", activation_alpha=1.702):
    """A moe_problem_t.  format: a FORMATS name or code; tile_regime: a
    TILE_REGIMES name or code; shared_expert: 0 or 1 (a fused shared expert,
    one more expert and slot after the routing); activation: "swiglu" or
    "swigluoai", whose gate slope is activation_alpha (1.702 by default, one
    public model's value; the pages leave it to the caller)."""
    fmt = FORMATS[format] if isinstance(format, str) else int(format)
    clamp = float(activation_clamp)
    regime = TILE_REGIMES[tile_regime] if isinstance(tile_regime, str) else int(tile_regime)
    act = ACTIVATIONS[activation] if isinstance(activation, str) else int(activation)
    return Problem(int(num_tokens), int(hidden), int(intermediate_hidden), int(num_experts),
                   int(num_topk), math.inf if math.isinf(clamp) else clamp, fmt, int(fast_math), regime,
                   int(shared_expert), act, float(activation_alpha))


def problem_from_dict(d, num_tokens=None, fast_math=1):
    return problem(d["num_tokens"] if num_tokens is None else num_tokens, d["hidden"],
                   d["intermediate_hidden"], d["num_experts"], d["num_topk"],
                   d.get("activation_clamp", 10.0), d["format"], fast_math, d.get("tile_regime", "auto"),
                   d.get("shared_expert", 0), d.get("activation", "swiglu"), d.get("activation_alpha", 1.702))


def act(x, x_scale=None, x_rowwise_scale=None):
    return Act(_ptr(x), _ptr(x_scale), _ptr(x_rowwise_scale))


def weights(w13, w13_scale, w2, w2_scale, gate_up_expert_scales=None, down_expert_scales=None,
            c_input_scales=None):
    return Weights(_ptr(w13), _ptr(w13_scale), _ptr(w2), _ptr(w2_scale),
                   _ptr(gate_up_expert_scales), _ptr(down_expert_scales), _ptr(c_input_scales))


def layout(expert_counts, expert_start_indices, src_info, slot_to_row, expert_ids, num_active,
           a_scale_offsets, tile_offsets):
    return Layout(*(_ptr(t) for t in (expert_counts, expert_start_indices, src_info, slot_to_row,
                                      expert_ids, num_active, a_scale_offsets, tile_offsets)))


# ---------------------------------------------------------------- entry points

def init(device=0):
    _check("moe_init", lib().moe_init(int(device)))


def workspace_size(prob):
    n = ctypes.c_size_t(0)
    _check("moe_get_workspace_size", lib().moe_get_workspace_size(ctypes.byref(prob), ctypes.byref(n)))
    return n.value


def tile_regime(prob):
    """'large_m' or 'small_m': the grouped GEMMs' tile shape for this problem."""
    r = ctypes.c_int32(0)
    _check("moe_get_tile_regime", lib().moe_get_tile_regime(ctypes.byref(prob), ctypes.byref(r)))
    return {v: k for k, v in TILE_REGIMES.items()}[r.value]


def workspace_offsets(prob):
    """{region: byte offset} of moe_fused's working data in the workspace
    (plus 'scale_rows', the padded scale rows P)."""
    o = WorkspaceOffsets()
    _check("moe_get_workspace_offsets", lib().moe_get_workspace_offsets(ctypes.byref(prob), ctypes.byref(o)))
    return {n: int(getattr(o, n)) for n in WS_OFFSET_FIELDS}


def intermediate_size(prob):
    n, off = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("moe_get_intermediate_size",
           lib().moe_get_intermediate_size(ctypes.byref(prob), ctypes.byref(n), ctypes.byref(off)))
    return n.value, off.value


def workspace_init(ws, nbytes, stream=None):
    _check("moe_workspace_init", lib().moe_workspace_init(_ptr(ws), int(nbytes), _stream(stream)))


def workspace_test_hooks(ws, nbytes, wait_limit_us=0, skip_arrival=0, stream=None):
    """Failure-detection test hooks in the workspace header (see include/moe.h)."""
    _check("moe_workspace_test_hooks", lib().moe_workspace_test_hooks(_ptr(ws), int(nbytes), int(wait_limit_us),
                                                                      int(skip_arrival), _stream(stream)))


def prepared_weights_size(prob):
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("moe_get_prepared_weights_size",
           lib().moe_get_prepared_weights_size(ctypes.byref(prob), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def prepare_weights(prob, logical, out_w13, out_w2, stream=None):
    _check("moe_prepare_weights", lib().moe_prepare_weights(
        ctypes.byref(prob), ctypes.byref(logical), _ptr(out_w13), _ptr(out_w2), _stream(stream)))


def route(prob, logits, bias, topk_idx, topk_weights, stream=None):
    _check("moe_route", lib().moe_route(ctypes.byref(prob), _ptr(logits), _ptr(bias), _ptr(topk_idx),
                                        _ptr(topk_weights), _stream(stream)))


def quantize_nvfp4_rowwise(prob, x_bf16, codes, block_scales, rowwise_scales, stream=None):
    """Per-token dynamic NVFP4 quantisation of BF16 activations (see include/moe.h)."""
    _check("moe_quantize_nvfp4_rowwise", lib().moe_quantize_nvfp4_rowwise(
        ctypes.byref(prob), _ptr(x_bf16), _ptr(codes), _ptr(block_scales), _ptr(rowwise_scales), _stream(stream)))


def permute(prob, topk_idx, lay, ws, ws_bytes, stream=None):
    _check("moe_permute", lib().moe_permute(ctypes.byref(prob), _ptr(topk_idx), ctypes.byref(lay),
                                            _ptr(ws), int(ws_bytes), _stream(stream)))


def ffn(prob, a, w, lay, topk_weights, out_mode, out, ws, ws_bytes, intermediate=None, stream=None):
    _check("moe_ffn", lib().moe_ffn(ctypes.byref(prob), ctypes.byref(a), ctypes.byref(w),
                                    ctypes.byref(lay), _ptr(topk_weights), int(out_mode), _ptr(out),
                                    _ptr(intermediate), _ptr(ws), int(ws_bytes), _stream(stream)))


def combine(prob, lay, topk_weights, inp, in_mode, out_bf16, stream=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(prob), None if lay is None else ctypes.byref(lay),
                                            _ptr(topk_weights), _ptr(inp), int(in_mode),
                                            _ptr(out_bf16), _stream(stream)))


def permute_noalloc(prob, topk_idx, lay, device_status, stream=None):
    """moe_permute without a workspace (see include/moe.h)."""
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(ctypes.byref(prob), _ptr(topk_idx),
                                                            ctypes.byref(lay), _ptr(device_status),
                                                            _stream(stream)))


def fused(prob, a, w, out_bf16, ws, ws_bytes, topk_idx=None, topk_weights=None, logits=None,
          bias=None, stream=None):
    _check("moe_fused", lib().moe_fused(ctypes.byref(prob), ctypes.byref(a), ctypes.byref(w),
                                        _ptr(topk_idx), _ptr(topk_weights), _ptr(logits), _ptr(bias),
                                        _ptr(out_bf16), _ptr(ws), int(ws_bytes), _stream(stream)))


def read_status(ws, stream=None):
    """Synchronise the stream and return the sticky device status code."""
    return lib().moe_read_status(_ptr(ws), _stream(stream))


def timing_enable(enable=True, max_calls=1024):
    _check("moe_timing_enable", lib().moe_timing_enable(int(bool(enable)), int(max_calls)))


def timing_read():
    """{slot: (summed ms, launches)} since the last read (waits for the events)."""
    ms = (ctypes.c_float * len(SLOTS))()
    n = (ctypes.c_int * len(SLOTS))()
    _check("moe_timing_read", lib().moe_timing_read(ms, n))
    return {name: (float(ms[i]), int(n[i])) for i, name in enumerate(SLOTS)}


def raw(fn_name, *args):
    """Call an entry point with raw ctypes arguments and return its status code."""
    return getattr(lib(), fn_name)(*args)
