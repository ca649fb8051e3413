"""CPU oracle for the routed Mixture-of-Experts FFN.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.

The oracle is a plain, slow, float64 restatement of what the routed MoE FFN
computes, written from the public API pages it cites:

* flashinfer.megamoe.MegaMoESymmBuffer -- geometry (hidden a multiple of 256,
  intermediate_hidden a multiple of 128), the SwiGLU clamp (default 10.0) and
  the staging views (E4M3 activations with FP32 per-128 block scales, INT64
  ``topk_idx``, FP32 ``topk_weights``).
* Struct_mega_ffn_ep_combine_send (MAX mega_ffn) -- the operand list of the
  fused FFN: pre-permuted W13 / W2, per-expert L1 / L2 output scaling, the
  per-expert NVFP4 re-quant input scale, ``expert_start_indices``,
  ``expert_ids`` (-1 = masked), ``a_scale_offsets`` and ``src_info``.
* flashinfer.fused_moe.MoEActivationPack -- the NVFP4 activation encoding
  (packed uint8 [M, H/2] + float8_e4m3fn [M, H/16]) and the ``FromLogits``
  routing mode with a selection-only bias.
* DistributedEPCombine -- the combine: router weights scale each expert's
  contribution and the rows are reduced back to token order.

It shares no code with the CUDA path (``mixture_experts_routed_03_b200``) and
imports nothing from it.  Every function is pinned by ``tests/test_oracle_*``
against something other than itself (ml_dtypes / torch casts, brute force,
closed forms, special cases that reduce to library routines).
"""

from . import formats  # noqa: F401
from . import moe  # noqa: F401
