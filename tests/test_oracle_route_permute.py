"""Pins of the oracle's routing and permutation against brute force and worked examples."""

import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import moe as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _brute_route(logits, bias, k):
    """Full Python sort of (score, index) per token: NaN last, score desc, index asc."""
    logits = np.asarray(logits, np.float32)
    bias = np.zeros(logits.shape[1], np.float32) if bias is None else np.asarray(bias, np.float32)
    idx_out, w_out = [], []
    for row in logits:
        scores = [np.float32(row[e]) + np.float32(bias[e]) for e in range(len(row))]

        def key(e):
            s = scores[e]
            return (1, 0.0, e) if math.isnan(s) else (0, -float(s), e)
        order = sorted(range(len(row)), key=key)[:k]
        idx_out.append(order)
        ls = [float(row[e]) for e in order]
        m = max(ls)
        z = [math.exp(v - m) for v in ls]
        w_out.append([v / sum(z) for v in z])
    return np.array(idx_out), np.array(w_out)


def _brute_permute(topk_idx, E):
    flat = [int(v) for v in np.asarray(topk_idx).reshape(-1)]
    rows = []
    for e in range(E):
        for s, v in enumerate(flat):
            if v == e:
                rows.append(s)
    return rows


def test_route_worked_example():
    ex = GOLDEN["route"]
    idx, w = O.route(np.array(ex["logits"]), np.array(ex["bias"]), ex["k"])
    assert idx.tolist() == ex["topk_idx"]
    assert np.allclose(w, ex["topk_weights"], rtol=1e-15, atol=0)


@pytest.mark.parametrize("seed", range(5))
def test_route_vs_brute_force(seed):
    rng = np.random.default_rng(seed)
    M, E = 40, 12
    # coarse values force many exact ties; a few NaN / inf / signed zeros
    logits = rng.integers(-3, 4, (M, E)).astype(np.float32) * 0.5
    logits[0, 3] = np.nan
    logits[1, :] = 0.0
    logits[1, ::2] = -0.0
    logits[2, 5] = np.inf
    logits[3, 7] = -np.inf
    bias = rng.integers(-2, 3, E).astype(np.float32) * 0.25
    for k in (1, 3, E):
        for b in (None, bias):
            idx, w = O.route(logits, b, k)
            bidx, bw = _brute_route(logits, b, k)
            assert np.array_equal(idx, bidx)
            ok = ~np.isnan(bw)
            assert np.allclose(w[ok], bw[ok], rtol=1e-12, atol=0)


def test_route_weights_are_softmax_over_chosen_unbiased():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((64, 16)).astype(np.float32)
    bias = (rng.standard_normal(16) * 3).astype(np.float32)
    idx, w = O.route(logits, bias, 4)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14)
    # full softmax renormalised over the chosen set gives the same weights
    full = np.exp(logits.astype(np.float64))
    full /= full.sum(axis=1, keepdims=True)
    pick = np.take_along_axis(full, idx, 1)
    assert np.allclose(w, pick / pick.sum(axis=1, keepdims=True), rtol=1e-12)
    # with bias the selection may differ from the unbiased top-k
    idx0, _ = O.route(logits, None, 4)
    assert not np.array_equal(np.sort(idx, 1), np.sort(idx0, 1))


def test_permute_worked_example():
    ex = GOLDEN["permute"]
    pm = O.permute(np.array(ex["topk_idx"]), ex["num_experts"])
    for key in ("expert_counts", "expert_start_indices", "src_info", "slot_to_row",
                "expert_ids", "a_scale_offsets"):
        assert pm[key].tolist() == ex[key], key
    assert pm["num_active"] == ex["num_active"]


@pytest.mark.parametrize("seed", range(6))
def test_permute_vs_brute_force_and_invariants(seed):
    rng = np.random.default_rng(seed)
    M, k, E = int(rng.integers(1, 60)), int(rng.integers(1, 5)), int(rng.integers(1, 9))
    idx = rng.integers(-1, E, (M, k))
    pm = O.permute(idx, E)
    assert pm["src_info"].tolist() == _brute_permute(idx, E)
    valid = idx.reshape(-1) >= 0
    counts = np.bincount(idx.reshape(-1)[valid], minlength=E)
    assert np.array_equal(pm["expert_counts"], counts)
    assert np.array_equal(pm["expert_start_indices"], np.concatenate([[0], np.cumsum(counts)]))
    # each token appears exactly (its number of valid slots) times in src_info
    tok = pm["src_info"] // k
    assert np.array_equal(np.bincount(tok, minlength=M), (idx >= 0).sum(axis=1))
    # slot_to_row inverts src_info; skipped slots map to -1
    assert np.array_equal(pm["slot_to_row"][pm["src_info"]], np.arange(pm["src_info"].shape[0]))
    assert np.all(pm["slot_to_row"][~valid] == -1)
    # rows of one expert ascend in slot index, and carry that expert
    for e in range(E):
        seg = pm["src_info"][pm["expert_start_indices"][e]:pm["expert_start_indices"][e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(idx.reshape(-1)[seg] == e)
    act = [e for e in range(E) if counts[e] > 0]
    assert pm["expert_ids"].tolist() == act + [-1] * (E - len(act))
    assert pm["num_active"] == len(act)
    assert np.array_equal(np.diff(pm["a_scale_offsets"]), -(-counts // 128) * 128)


def test_permute_rejects_out_of_range():
    with pytest.raises(ValueError):
        O.permute(np.array([[0, 3]]), 3)
    with pytest.raises(ValueError):
        O.permute(np.array([[-2, 0]]), 3)


def test_permute_empty_and_all_skipped():
    pm = O.permute(np.zeros((0, 2), np.int64), 4)
    assert pm["src_info"].shape == (0,) and pm["num_active"] == 0
    pm = O.permute(np.full((3, 2), -1), 4)
    assert pm["expert_start_indices"].tolist() == [0] * 5
    assert pm["slot_to_row"].tolist() == [-1] * 6


def test_permute_small_exhaustive():
    """Every topk_idx of a 2-token, k=2, E=2 problem (values in {-1, 0, 1})."""
    for vals in itertools.product([-1, 0, 1], repeat=4):
        idx = np.array(vals).reshape(2, 2)
        pm = O.permute(idx, 2)
        assert pm["src_info"].tolist() == _brute_permute(idx, 2)
