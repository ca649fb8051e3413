"""The C ABI library builds, loads without a GPU, exports every entry point
include/moe.h declares, and validates arguments on the host (no launch)."""

import ctypes
import os
import re

import pytest

from mixture_experts_routed_03_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^\s*(?:moe_status_t|const char\*)\s+(moe_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("moe_route", "moe_permute", "moe_ffn", "moe_combine", "moe_fused"):
        assert n in names
    assert set(names) == set(api.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def _prob(**kw):
    d = dict(num_tokens=16, hidden=256, intermediate_hidden=128, num_experts=8, num_topk=2,
             activation_clamp=10.0, format="bf16")
    d.update(kw)
    return api.problem(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(hidden=100), api.MOE_ERR_INVALID_ARG),
    (dict(hidden=384), api.MOE_ERR_INVALID_ARG),
    (dict(intermediate_hidden=96), api.MOE_ERR_INVALID_ARG),
    (dict(num_topk=0), api.MOE_ERR_INVALID_ARG),
    (dict(num_topk=9), api.MOE_ERR_INVALID_ARG),
    (dict(num_experts=0), api.MOE_ERR_INVALID_ARG),
    (dict(num_experts=2048, num_topk=2), api.MOE_ERR_UNSUPPORTED),
    (dict(num_tokens=-1), api.MOE_ERR_INVALID_ARG),
    (dict(activation_clamp=float("nan")), api.MOE_ERR_INVALID_ARG),
    (dict(activation_clamp=0.0), api.MOE_ERR_INVALID_ARG),
    (dict(format=7), api.MOE_ERR_INVALID_ARG),
    (dict(format="nvfp4", intermediate_hidden=384), api.MOE_ERR_UNSUPPORTED),
    (dict(tile_regime=3), api.MOE_ERR_INVALID_ARG),
    (dict(shared_expert=2), api.MOE_ERR_INVALID_ARG),
    (dict(activation=2), api.MOE_ERR_INVALID_ARG),
    (dict(activation="swigluoai", activation_alpha=0.0), api.MOE_ERR_INVALID_ARG),
    (dict(activation="swigluoai", activation_alpha=float("nan")), api.MOE_ERR_INVALID_ARG),
    (dict(activation="swigluoai", activation_alpha=float("inf")), api.MOE_ERR_INVALID_ARG),
    (dict(shared_expert=-1), api.MOE_ERR_INVALID_ARG),
    (dict(num_experts=1024, num_topk=2, shared_expert=1), api.MOE_ERR_UNSUPPORTED),
    (dict(format=5), api.MOE_ERR_INVALID_ARG),
])
def test_geometry_validation(lib, kw, code):
    n = ctypes.c_size_t(0)
    got = lib.moe_get_workspace_size(ctypes.byref(_prob(**kw)), ctypes.byref(n))
    assert got == code


def test_valid_geometry_and_sizes(lib):
    for fmt, eb in (("bf16", 2.0), ("fp8", 1.0), ("nvfp4", 0.5), ("mxfp8", 1.0), ("fp8_tensor", 1.0)):
        p = _prob(format=fmt, hidden=512, intermediate_hidden=256)
        assert api.workspace_size(p) > 0
        a, b = api.prepared_weights_size(p)
        # the prepared blobs hold exactly the weights plus their block scales:
        # one byte per 16 elements (NVFP4) or per 32 (MXFP8)
        extra = {"nvfp4": 1.0 / 16, "mxfp8": 1.0 / 32}.get(fmt, 0.0)
        assert a == int(8 * 2 * 256 * 512 * (eb + extra))
        assert b == int(8 * 512 * 256 * (eb + extra))
        n, off = api.intermediate_size(p)
        assert off % 256 == 0 and n > off
    assert api.workspace_size(_prob(activation_clamp=float("inf"))) > 0


def test_null_pointer_arguments_rejected_before_launch(lib):
    p = _prob()
    a, w = api.act(None), api.weights(None, None, None, None)
    lay = api.layout(*([None] * 8))
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), None, None, None, None,
                         None, None, 0, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(p), None, ctypes.byref(lay), None, 0, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(p), None, None, None, None, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(p), None, None, None, 0, None, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_ffn(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), ctypes.byref(lay), None, 5,
                       None, None, None, 0, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_read_status(None, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_prepare_weights(ctypes.byref(p), None, None, None, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_prepare_weights(ctypes.byref(p), ctypes.byref(w), None, None, None) == api.MOE_ERR_INVALID_ARG


def test_fused_needs_exactly_one_routing_source(lib):
    p = _prob()
    fake = 1 << 20  # never dereferenced: validation fails first
    a = api.act(fake)
    w = api.weights(fake, None, fake, None)
    # both routing sources
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), fake, fake, fake, None,
                         fake, fake, 1 << 30, None) == api.MOE_ERR_INVALID_ARG
    # only one half of the precomputed routing
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), fake, None, None, None,
                         fake, fake, 1 << 30, None) == api.MOE_ERR_INVALID_ARG
    # workspace too small
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), fake, fake, None, None,
                         fake, fake, 16, None) == api.MOE_ERR_WORKSPACE


def test_zero_tokens_is_ok_without_touching_memory(lib):
    p = _prob(num_tokens=0)
    a, w = api.act(None), api.weights(None, None, None, None)
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), None, None, None, None,
                         None, None, 0, None) == api.MOE_OK


def test_status_strings(lib):
    for code in range(7):
        assert api.status_string(code).startswith("MOE_")


def test_tile_regime_resolution(lib):
    # AUTO: swapped-operand tiles while routed rows average <= 64 per expert (every format)
    assert api.tile_regime(_prob(num_tokens=256, num_experts=8, num_topk=2)) == "small_m"     # 512 <= 512
    assert api.tile_regime(_prob(num_tokens=257, num_experts=8, num_topk=2)) == "large_m"
    assert api.tile_regime(_prob(num_tokens=256, format="fp8", num_experts=8, num_topk=2)) == "small_m"
    assert api.tile_regime(_prob(num_tokens=16, format="nvfp4", intermediate_hidden=256, num_experts=8,
                                 num_topk=2)) == "small_m"
    assert api.tile_regime(_prob(num_tokens=16, format="mxfp8", num_experts=8, num_topk=2)) == "small_m"
    assert api.tile_regime(_prob(num_tokens=257, format="mxfp8", num_experts=8, num_topk=2)) == "large_m"
    assert api.tile_regime(_prob(num_tokens=16, tile_regime="large_m")) == "large_m"
    # every format has both regimes when forced
    for fmt in ("bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor"):
        kw = dict(num_tokens=16, format=fmt, intermediate_hidden=256)
        assert api.tile_regime(_prob(tile_regime="small_m", **kw)) == "small_m"
        assert api.tile_regime(_prob(tile_regime="large_m", **kw)) == "large_m"
    assert api.tile_regime(_prob(num_tokens=100000, tile_regime="small_m")) == "small_m"


def test_shared_expert_sizes_are_those_of_one_more_expert_and_slot(lib):
    """A fused shared expert is one more expert and one more slot per token
    after the routing: every size equals the plain problem's with E + 1 and
    k + 1."""
    for fmt in ("bf16", "fp8", "nvfp4", "mxfp8"):
        kw = dict(format=fmt, hidden=512, intermediate_hidden=256, num_tokens=300)
        shared = _prob(num_experts=8, num_topk=2, shared_expert=1, **kw)
        plain = _prob(num_experts=9, num_topk=3, **kw)
        assert api.workspace_size(shared) == api.workspace_size(plain)
        assert api.prepared_weights_size(shared) == api.prepared_weights_size(plain)
        assert api.intermediate_size(shared) == api.intermediate_size(plain)
        assert api.workspace_offsets(shared) == api.workspace_offsets(plain)
        assert api.tile_regime(shared) == api.tile_regime(plain)


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4", "mxfp8", "fp8_tensor"])
def test_workspace_size_does_not_depend_on_the_tile_regime(lib, fmt):
    """One workspace serves both tile regimes: a layer sized for its largest
    batch (large-M tiles) also runs its small batches, which auto sends to the
    small-M tiles."""
    for M in (16, 5000):
        sizes = set()
        for regime in ("auto", "large_m", "small_m"):
            n = ctypes.c_size_t(0)
            p = _prob(num_tokens=M, hidden=512, intermediate_hidden=256, format=fmt, tile_regime=regime)
            assert lib.moe_get_workspace_size(ctypes.byref(p), ctypes.byref(n)) == api.MOE_OK
            sizes.add(n.value)
        assert len(sizes) == 1, (fmt, M, sizes)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "mxfp8"])
def test_misaligned_activations_rejected_before_launch(lib, fmt):
    """x must be 16-byte aligned and x_scale 4-byte aligned; both are checked
    before anything touches the device (the pointers are never dereferenced)."""
    p = _prob(format=fmt, intermediate_hidden=256)
    base = 1 << 20
    w = api.weights(base, base, base, base, base, base, base)
    for x, xs in ((base + 8, base), (base, base + 2), (base, base + 1)):
        a = api.act(x, xs)
        assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), base, base, None, None,
                             base, base, 1 << 40, None) == api.MOE_ERR_INVALID_ARG, (x - base, xs - base)
    # aligned pointers get past the checks to the workspace-size test
    a = api.act(base, base + 4)
    assert lib.moe_fused(ctypes.byref(p), ctypes.byref(a), ctypes.byref(w), base, base, None, None,
                         base, base, 16, None) == api.MOE_ERR_WORKSPACE
