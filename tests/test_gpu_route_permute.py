"""GPU parity of moe_route and moe_permute against the oracle: bit-exact
indices and layout arrays, routing weights to 1e-6 relative."""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer, workloads
from oracle import moe as O
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


def _layer_for(M, E, k, fmt="bf16", H=256, I=128):
    p = dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k,
             format=fmt, activation_clamp=10.0)
    dev = S.device()
    E_ = E
    w = dict(w13=torch.zeros((E_, 2 * I, H), dtype=torch.bfloat16, device=dev),
             w2=torch.zeros((E_, H, I), dtype=torch.bfloat16, device=dev))
    return p, layer.MoELayer(p, w, device=dev)


@pytest.mark.parametrize("M,E,k", [(1, 8, 1), (37, 8, 2), (256, 64, 6), (1000, 128, 8),
                                   (64, 256, 8), (300, 1024, 4), (16384, 128, 8), (33, 40, 32)])
def test_route_matches_oracle(M, E, k):
    g = torch.Generator().manual_seed(M * 7 + E)
    logits = torch.randn((M, E), generator=g, dtype=torch.float32)
    # coarse values create exact ties; add a few NaN, inf and signed zeros
    logits[: M // 2] = torch.round(logits[: M // 2] * 2) / 2
    if M > 4:
        logits[0, 0] = float("nan")
        logits[1, :] = 0.0
        logits[1, ::2] = -0.0
        logits[2, E - 1] = float("inf")
        logits[3, 0] = float("-inf")
    bias = torch.round(torch.randn((E,), generator=g) * 4) / 8
    p, L = _layer_for(M, E, k)
    for b in (None, bias):
        idx, w = L.route(logits.cuda(), None if b is None else b.cuda())
        torch.cuda.synchronize()
        ridx, rw = O.route(logits.numpy(), None if b is None else b.numpy(), k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        wg = w.cpu().numpy().astype(np.float64)
        # weights are specified for tokens whose chosen logits are all finite
        chosen = np.take_along_axis(logits.numpy(), ridx, axis=1)
        ok = np.repeat(np.all(np.isfinite(chosen), axis=1, keepdims=True), k, axis=1)
        assert ok.sum() >= 0.9 * ok.size
        assert np.all(np.abs(wg[ok] - rw[ok]) <= 1e-6 * np.abs(rw[ok]) + 1e-7)


def test_route_topk_above_32_is_unsupported():
    p, L = _layer_for(4, 40, 33)
    with pytest.raises(api.MoEError) as ei:
        L.route(torch.zeros((4, 40), device="cuda"))
    assert ei.value.code == api.MOE_ERR_UNSUPPORTED


def _perm_case(M, E, k, seed, frac_skip=0.0, skew=None):
    rng = np.random.default_rng(seed)
    if skew is None:
        idx = np.stack([rng.choice(E, size=k, replace=k > E) for _ in range(M)]) if M else np.zeros((0, k), np.int64)
    else:
        idx = rng.integers(0, max(1, E // skew), (M, k))
    if frac_skip:
        idx[rng.random(idx.shape) < frac_skip] = -1
    return idx.astype(np.int64)


@pytest.mark.parametrize("M,E,k,seed,skip,skew", [
    (1, 1, 1, 0, 0.0, None), (3, 2, 2, 1, 0.0, None), (17, 8, 2, 2, 0.2, None),
    (129, 8, 8, 3, 0.0, None), (256, 64, 6, 4, 0.1, None), (1000, 256, 8, 5, 0.0, 64),
    (4096, 32, 8, 6, 0.0, None), (16384, 128, 8, 7, 0.05, None), (5000, 1024, 3, 8, 0.3, None),
    (64, 256, 8, 9, 0.0, None)])
def test_permute_matches_oracle(M, E, k, seed, skip, skew):
    idx = _perm_case(M, E, k, seed, skip, skew)
    p, L = _layer_for(M, E, k)
    lay = L.permute(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    assert L.status() == api.MOE_OK
    S.check_layout_exact(lay.host(), O.permute(idx, E), M, k)


def test_permute_all_skipped_and_repeated_calls_deterministic():
    M, E, k = 50, 16, 4
    idx = np.full((M, k), -1, np.int64)
    p, L = _layer_for(M, E, k)
    lay = L.permute(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    S.check_layout_exact(lay.host(), O.permute(idx, E), M, k)
    idx2 = _perm_case(M, E, k, 3, 0.2)
    a = L.permute(torch.from_numpy(idx2).cuda()).host()
    b = L.permute(torch.from_numpy(idx2).cuda()).host()
    for key in a:
        assert np.array_equal(a[key], b[key])


def test_permute_bad_index_sets_status():
    M, E, k = 20, 8, 2
    idx = _perm_case(M, E, k, 1)
    idx[5, 1] = 8          # == num_experts: out of range
    idx[7, 0] = -3         # below the skip marker
    p, L = _layer_for(M, E, k)
    L.permute(torch.from_numpy(idx).cuda())
    assert L.status() == api.MOE_ERR_BAD_INDEX
    L.clear_status()
    assert L.status() == api.MOE_OK
    # the bad slots are skipped; the valid ones are laid out as without them
    ok = idx.copy()
    ok[5, 1] = -1
    ok[7, 0] = -1
    lay = L.permute(torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    ref = O.permute(ok, E)
    h = lay.host()
    assert np.array_equal(h["expert_start_indices"], ref["expert_start_indices"])
    assert np.array_equal(h["src_info"][: ref["expert_start_indices"][-1]], ref["src_info"])
    L.clear_status()


def test_zero_tokens_is_a_noop():
    p, L = _layer_for(4, 8, 2)
    prob = api.problem_from_dict(p, num_tokens=0)
    api.permute(prob, None, L.permute(torch.zeros((1, 2), dtype=torch.int64, device="cuda")).struct,
                L.ws, L.ws_bytes)
    torch.cuda.synchronize()
