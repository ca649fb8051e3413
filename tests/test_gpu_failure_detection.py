"""Failure detection of the single launch (EPConfig, fuse_ffn_combine_send:
raise rather than degrade silently): a CTA that never arrives at a grid
barrier makes the other CTAs' bounded waits run out; the call returns, the
status word reads MOE_ERR_TIMEOUT, and after moe_workspace_init the next call
is correct against the oracle.  The stall is made by a test hook (CTA 0
withholds one arrival); nothing faults or hangs the GPU."""

import time

import numpy as np
import pytest
import torch

from mixture_experts_routed_03_b200 import api, layer
from tests import gpu_support as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,M,H,I,E,k", [("bf16", 64, 512, 256, 4, 2), ("fp8", 300, 1024, 384, 8, 4)])
def test_withheld_barrier_arrival_times_out_then_recovers(fmt, M, H, I, E, k):
    p = dict(num_tokens=M, hidden=H, intermediate_hidden=I, num_experts=E, num_topk=k, format=fmt,
             routing="softmax", activation_clamp=10.0)
    d, host = S.make(p, seed=7)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    # a clean call first
    out0 = L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"])
    assert L.status() == api.MOE_OK
    # 5 ms bounded waits, and CTA 0 skips its first grid-barrier arrival
    api.workspace_test_hooks(L.ws, L.ws_bytes, wait_limit_us=5000, skip_arrival=1)
    t0 = time.perf_counter()
    L.forward(d["x"], d.get("x_scale"), topk_idx=d["topk_idx"], topk_weights=d["topk_weights"])
    code = L.status()
    elapsed = time.perf_counter() - t0
    assert code == api.MOE_ERR_TIMEOUT
    assert elapsed < 1.0          # gave up after the short limit, not the 2 s default
    # the hook was one-shot, but the barrier state is stale until re-initialised
    L.clear_status()
    assert L.status() == api.MOE_OK
    res = S.run_fused(L, d)
    assert L.status() == api.MOE_OK
    S.check_against_oracle(p, host, res, np.arange(M), label=f"after-timeout/{fmt}")
    # and agrees with the clean call made before the time-out
    a = S.bf16_to_np(out0)
    assert np.all(S.close_bf16(a, res.out, S.TOL[fmt] * S.rms(a)))


def test_test_hooks_validate_arguments():
    p = dict(num_tokens=16, hidden=256, intermediate_hidden=128, num_experts=4, num_topk=2, format="bf16",
             routing="softmax", activation_clamp=10.0)
    d, _ = S.make(p, seed=1)
    L = layer.MoELayer(p, S.weights_of(d), device=S.device())
    for bad in (dict(wait_limit_us=-1), dict(skip_arrival=2)):
        with pytest.raises(api.MoEError) as ei:
            api.workspace_test_hooks(L.ws, L.ws_bytes, **bad)
        assert ei.value.code == api.MOE_ERR_INVALID_ARG
