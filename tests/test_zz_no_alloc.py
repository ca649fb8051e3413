"""The allocation-free permutation (moe_permute_noalloc) against moe_permute.

Some callers cannot allocate device memory -- a host runtime with no device
allocator of its own, a serving loop that must not allocate per request --
so the library offers one entry point whose scratch lives in a fixed device
array instead of a caller-sized workspace.  This checks, through the C ABI, that it writes
exactly the layout moe_permute writes, on two calls in a row (the second one
reuses the array the first one left behind), and that it refuses sizes
beyond its array.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer

pytestmark = pytest.mark.gpu

FIELDS = ("expert_counts", "expert_start_indices", "src_info", "slot_to_row", "expert_ids",
          "num_active", "a_scale_offsets", "tile_offsets")


def _layer(M, E, k):
    p = dict(num_tokens=M, hidden=256, intermediate_hidden=128, num_experts=E, num_topk=k,
             format="bf16", activation_clamp=10.0)
    dev = torch.device("cuda", 0)
    w = dict(w13=torch.zeros((E, 256, 256), dtype=torch.bfloat16, device=dev),
             w2=torch.zeros((E, 256, 128), dtype=torch.bfloat16, device=dev))
    return p, layer.MoELayer(p, w, device=dev)


def _routing(M, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(M)]).astype(np.int64)
    idx[rng.random(idx.shape) < 0.05] = -1
    return torch.from_numpy(idx).cuda()


@pytest.mark.parametrize("M,E,k", [(4096, 64, 8),    # 32768 slots: uses the static scratch
                                   (64, 512, 8),     # more than 256 experts, few slots: one chunk, scratch
                                   (8192, 512, 8),   # 64 chunks x 512 experts: the array's full 32768 entries
                                   (300, 16, 4)])    # one-block path: no scratch needed
def test_noalloc_permute_matches_permute_twice(M, E, k):
    p, L = _layer(M, E, k)
    prob = L.problem(M)
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    for call in range(2):
        idx = _routing(M, E, k, seed=call)
        ref = L.permute(idx)
        got = layer.LayoutBuffers(M, k, E, torch.device("cuda", 0))
        api.permute_noalloc(prob, idx, got.struct, status)
        torch.cuda.synchronize()
        assert int(status.item()) == api.MOE_OK
        h_ref, h_got = ref.host(), got.host()
        R = int(h_ref["expert_start_indices"][E])
        na = int(h_ref["num_active"][0])
        for f in FIELDS:
            n = {"src_info": R, "slot_to_row": M * k, "tile_offsets": na + 1}.get(f, len(h_ref[f]))
            assert np.array_equal(h_got[f][:n], h_ref[f][:n]), (call, f)


def test_noalloc_permute_reports_bad_index_and_rejects_oversize():
    M, E, k = 4096, 64, 8
    p, L = _layer(M, E, k)
    idx = _routing(M, E, k, seed=5)
    idx[3, 2] = E
    got = layer.LayoutBuffers(M, k, E, torch.device("cuda", 0))
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    api.permute_noalloc(L.problem(M), idx, got.struct, status)
    torch.cuda.synchronize()
    assert int(status.item()) == api.MOE_ERR_BAD_INDEX
    # more chunk x expert counts than the static array holds: 65 chunks x 512
    # experts, one chunk past the limit (refused before any launch)
    big = api.problem(num_tokens=8320, hidden=256, intermediate_hidden=128, num_experts=512,
                      num_topk=8, format="bf16")
    with pytest.raises(api.MoEError) as ei:
        api.permute_noalloc(big, idx, got.struct, status)
    assert ei.value.code == api.MOE_ERR_UNSUPPORTED
