#!/usr/bin/env python
"""Throughput of the routed MoE FFN layer (moe_fused) on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--chain] [--hot-l2] [--set KEY=VALUE ...]

A step is one moe_fused call -- routing (when the workload routes from
logits), permutation, the two grouped GEMMs with their fused epilogues and the
BF16 finalise -- over one batch of synthetic inputs resident in HBM.  The L2
is flushed (a 512 MiB write, then a 512 MiB read of another buffer that
evicts the write's dirty lines) before every timed step, outside the step's
CUDA-event interval.  With N > 1 (one process per GPU, launched by torchrun)
every rank runs its own batch with its own copy of the experts (data
parallel, no collective on the data path; weak scaling); the time is the
maximum over ranks.

Rank 0 prints one JSON line.  `value` is routed tokens (token, expert slot
pairs) per second summed over ranks; `e2e` is the same through the public API
with the inputs copied from pinned host memory and the output read back every
step; `roofline` is the dominant kernel's algorithmic throughput against the
measured peak; `cpu_baseline` times the float64 CPU oracle on a bounded sample.
`--impl reference` times that oracle alone (the reference arm).
"""

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "fp8_prefill_routed"
METRIC = "routed tokens/sec and achieved TFLOPS (% of roofline) per MoE layer, 1 B200"
FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FMT_TENSOR_RATIO = {"bf16": 1.0, "fp8": 2.0, "nvfp4": 4.0, "mxfp8": 2.0, "fp8_tensor": 2.0}   # nominal dense ratio to bf16
# B200 datasheet dense peaks (the sparse figures halved) and the ~8 TB/s of
# HBM the layer's roofline is stated against: time = max(FLOPs / tensor peak,
# bytes / HBM bandwidth)
SPEC_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0, "nvfp4": 9000.0, "mxfp8": 4500.0, "fp8_tensor": 4500.0}
SPEC_HBM_GBS = 8000.0
ELEM_BYTES = {"bf16": 2.0, "fp8": 1.0, "nvfp4": 0.5, "mxfp8": 1.0, "fp8_tensor": 1.0}
BOUND = {"tiny_bf16": "hbm", "fp8_block": "hbm", "nvfp4_decode": "hbm",
         "nvfp4_prefill": "tensor", "fp8_prefill_routed": "tensor", "nvfp4_prefill_rowwise": "tensor",
         "mxfp8_prefill_routed": "tensor", "fp8_tensor_prefill_routed": "tensor"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-mma-peak", action="store_true",
                    help="skip the tensor-core peak probe (run after the timed steps)")
    ap.add_argument("--side-workloads",
                    default="fp8_block,nvfp4_prefill,nvfp4_decode,nvfp4_prefill_rowwise,mxfp8_prefill_routed,"
                            "fp8_tensor_prefill_routed",
                    help="other configurations timed after the main one (one GPU, rank 0), reported "
                         "under 'workloads'; empty for none")
    ap.add_argument("--chain", action="store_true",
                    help="time the multi-launch chain moe_route/moe_permute/moe_ffn/moe_combine "
                         "instead of the single moe_fused launch (per-kernel breakdown)")
    ap.add_argument("--hot-l2", action="store_true",
                    help="no L2 flush between steps (a hot-L2 number, reported separately)")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (a smaller case for profiling)")
    return ap.parse_args()


def workload(args):
    from mixture_experts_routed_03_b200 import workloads
    over = {}
    for kv in args.set:
        k, v = kv.split("=", 1)
        if k in workloads.WORKLOADS[args.workload]:
            over[k] = type(workloads.WORKLOADS[args.workload][k])(v)
        else:
            try:
                over[k] = float(v)
            except ValueError:       # a named option, e.g. tile_regime=pair
                over[k] = v
    return workloads.problem(args.workload, **over)


def _code_only(text):
    """C/C++/CUDA source without its comments and blank lines (a comment edit
    leaves the compiled kernels, and so a measured traffic figure, unchanged)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_sources_sha():
    """SHA-256 over the code (comments removed) of the CUDA sources and the C
    header: identifies the kernels a stored ncu traffic figure was measured
    on; any code change drops the figure."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_routed_03_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            h.update(_code_only(open(os.path.join(csrc, name)).read()).encode())
    h.update(_code_only(open(os.path.join(ROOT, "include", "moe.h")).read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/traffic.json,
    or None when absent or measured on other kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[workload]
    except Exception:
        return None
    # sources_sha: the kernel sources the counters were taken on; any later
    # change to them drops the figure
    if rec.get("kernel") != kernel or kernel_sources_sha() != rec.get("sources_sha"):
        return None
    return float(rec["dram_bytes_per_launch"])


def dist_env():
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(seed, rank):
    """Each rank draws its own batch (and its own copy of the experts)."""
    return seed + rank


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank floats; every rank calls it at the same
    point (a no-op on one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(units_per_rank, world, steps, t_ms):
    """Units all ranks processed per second, over the slowest rank's time."""
    return units_per_rank * world * steps / (t_ms / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons of one GPU, sampled through NVML while
    the timed steps execute (the host polls until the last step's event has
    completed)."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("sw_power_cap", 0x4))

    def __init__(self, torch_device):
        self.samples = []
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None

    def sample(self):
        if self.handle is None:
            return
        nv = self.nv
        try:
            sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            try:
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            except Exception:
                rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
            pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
            self.samples.append((sm, rs, pw))
        except Exception:
            pass

    def poll_until(self, event, min_samples=3):
        """Sample while `event` (the last timed step) has not completed."""
        import time as _t
        while not event.query() or len(self.samples) < min_samples:
            self.sample()
            if event.query() and len(self.samples) >= min_samples:
                break
            _t.sleep(0.0005)

    def summary(self):
        if self.handle is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        reasons = set()
        for _, rs, _ in self.samples:
            for name, bit in self.REASONS:
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples),
                "sm_max_mhz": self.max_mhz,
                "power_w_max": max(p for _, _, p in self.samples),
                "samples": len(self.samples), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- work model

def work_model(p, num_active):
    """Algorithmic FLOPs and bytes of the layer and of its two GEMM kernels."""
    M, H, I, E, k = (p["num_tokens"], p["hidden"], p["intermediate_hidden"], p["num_experts"],
                     p["num_topk"])
    fmt = p["format"]
    R = M * k
    eb = ELEM_BYTES[fmt]
    if fmt == "fp8":
        w13_sc = (2 * I // 128) * (H // 128) * 4
        w2_sc = (H // 128) * (I // 128) * 4
        x_sc, h_sc = H // 128 * 4, I // 128 * 4
    elif fmt == "nvfp4":
        w13_sc, w2_sc = 2 * I * H // 16, H * I // 16
        x_sc, h_sc = H // 16, I // 16
    elif fmt == "mxfp8":
        w13_sc, w2_sc = 2 * I * H // 32, H * I // 32
        x_sc, h_sc = H // 32, I // 32
    elif fmt == "fp8_tensor":
        w13_sc = w2_sc = 4
        x_sc = h_sc = 0
    else:
        w13_sc = w2_sc = x_sc = h_sc = 0
    w13 = num_active * (2 * I * H * eb + w13_sc)
    w2 = num_active * (H * I * eb + w2_sc)
    x = M * (H * eb + x_sc)
    out = M * H * 2
    gemm1 = dict(flops=4.0 * R * H * I, bytes=w13 + R * (H * eb + x_sc) + R * (I * eb + h_sc))
    gemm2 = dict(flops=2.0 * R * H * I, bytes=w2 + R * (I * eb + h_sc) + M * H * 4)
    layer = dict(flops=6.0 * R * H * I, bytes=w13 + w2 + x + out + (M * E * 4 if p["routing"] == "logits" else 0))
    return dict(gemm1=gemm1, gemm2=gemm2, layer=layer)


def side_workload(name, args, dev, peaks):
    """One more configuration, timed the same way as the main one (moe_fused,
    L2 flushed before every step, CUDA events on the launching stream), with
    fewer steps; its line under 'workloads'."""
    import torch
    from mixture_experts_routed_03_b200 import api, layer, workloads
    p = workloads.problem(name)
    d = workloads.make_inputs(p, seed=args.seed, device=dev)
    L = layer.MoELayer(p, {k: d.get(k) for k in ("w13", "w13_scale", "w2", "w2_scale", "gate_up_expert_scales",
                                                 "down_expert_scales", "c_input_scales")}, device=dev)
    M, k = p["num_tokens"], p["num_topk"]
    out = torch.empty((M, p["hidden"]), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    if p.get("act") == "bf16":
        # BF16 activations: the per-token NVFP4 quantiser, then the layer
        xb = d["x_bf16"].view(torch.bfloat16)

        def step():
            codes, scales, rowwise = L.quantize_rowwise(xb)
            L.forward(codes, scales, topk_idx=d["topk_idx"], topk_weights=d["topk_weights"], out=out,
                      x_rowwise_scale=rowwise)
    elif p["routing"] == "logits":
        # routing from logits inside the single launch, as the main line
        def step():
            L.forward(d["x"], d["x_scale"], logits=d["logits"], bias=d["bias"], out=out)
    else:
        def step():
            L.forward(d["x"], d["x_scale"], topk_idx=d["topk_idx"], topk_weights=d["topk_weights"], out=out)

    steps = max(5, min(args.steps, 20))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    L.check_status()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, out=sink)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    L.check_status()
    med = statistics.median(a.elapsed_time(b) for a, b in ev)
    idx = L.route(d["logits"], d["bias"])[0] if p["routing"] == "logits" else d["topk_idx"]
    num_active = int(torch.unique(idx[idx >= 0]).numel())
    wm = work_model(p, num_active)["layer"]
    if p.get("act") == "bf16":   # the step reads BF16 activations instead of NVFP4 ones
        wm = dict(wm, bytes=wm["bytes"] + M * p["hidden"] * (2.0 - 0.5 - 1.0 / 16))
    bound = BOUND.get(name, "tensor" if p["format"] == "nvfp4" and M * k > 8 * p["num_experts"] * 64 else "hbm")
    if bound == "tensor":
        achieved, peak, unit = wm["flops"] / (med / 1e3) / 1e12, peaks["bf16_tflops"] * FMT_TENSOR_RATIO[p["format"]], "TFLOP/s"
    else:
        achieved, peak, unit = wm["bytes"] / (med / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
    spec_t = max(wm["flops"] / (SPEC_TFLOPS[p["format"]] * 1e12), wm["bytes"] / (SPEC_HBM_GBS * 1e9))
    res = {"value": M * k / (med / 1e3), "unit": "routed_tokens/s", "ms_per_step_median": med, "steps": steps,
           "config": {"num_tokens": M, "hidden": p["hidden"], "intermediate_hidden": p["intermediate_hidden"],
                      "num_experts": p["num_experts"], "num_topk": k, "format": p["format"],
                      "routing": p["routing"], "active_experts": num_active,
                      "gemm_tiles": api.tile_regime(L.problem(M))},
           "roofline": {"kernel": "moe_fused_kernel", "bound": bound, "achieved": achieved, "peak": peak,
                        "unit": unit, "frac": achieved / peak},
           "roofline_spec": {"time_us": spec_t * 1e6, "frac": spec_t / (med / 1e3)}}
    del L, d, out, flush, flush_rd
    torch.cuda.empty_cache()
    return res


def mma_probe(fmt, achieved_tflops):
    """The dense tcgen05 rate of this GPU for the format, measured with the
    peak probe (operands resident in shared memory, back-to-back MMAs on
    every SM), after the timed steps; context for the roofline fraction."""
    try:
        from mixture_experts_routed_03_b200 import peak
        out = {}
        kind = "fp8" if fmt == "fp8_tensor" else fmt   # the same E4M3 MMAs
        for pair in (False, True) if kind in ("bf16", "fp8") else (False,):
            tf, cyc = peak.mma_peak(kind, 256, pair, iters=20000)
            out["cta_pair" if pair else "one_cta"] = {"tflops": tf, "cycles_per_mma": cyc}
        best = max(v["tflops"] for v in out.values())
        out["frac_of_best"] = achieved_tflops / best
        out["shape"] = "M128 (one CTA) / M256 (CTA pair) x N256, K 32 bytes per instruction"
        return out
    except Exception as e:  # the probe is context only; the line stands without it
        return {"error": str(e)}


# --------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_routed_03_b200 import api, layer, workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    p = workload(args)
    d = workloads.make_inputs(p, seed=rank_seed(args.seed, rank), device=dev)
    wts = {k: d.get(k) for k in ("w13", "w13_scale", "w2", "w2_scale", "gate_up_expert_scales",
                                 "down_expert_scales", "c_input_scales")}
    L = layer.MoELayer(p, wts, device=dev)
    routed = p["routing"] == "logits"
    M, k = p["num_tokens"], p["num_topk"]
    R = M * k
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i):
        # write 512 MiB, then read another 512 MiB: the read evicts the
        # write's dirty lines, so their write-back lands before the timed
        # interval instead of inside the step
        if args.hot_l2:
            return
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, out=flush_sink)

    out = torch.empty((M, p["hidden"]), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    lay = layer.LayoutBuffers(M, k, p["num_experts"], dev) if args.chain else None
    acc = torch.empty((M, p["hidden"]), dtype=torch.float32, device=dev) if args.chain else None
    ridx = torch.empty((M, k), dtype=torch.int64, device=dev) if args.chain and routed else None
    rw = torch.empty((M, k), dtype=torch.float32, device=dev) if args.chain and routed else None

    def chain():
        prob = L.problem(M)
        idx, w = d.get("topk_idx"), d.get("topk_weights")
        if routed:
            api.route(prob, d["logits"], d["bias"], ridx, rw)
            idx, w = ridx, rw
        api.permute(prob, idx, lay.struct, L.ws, L.ws_bytes)
        api.ffn(prob, api.act(d["x"], d["x_scale"]), L.weights, lay.struct, w, api.MOE_OUT_ACCUMULATE, acc,
                L.ws, L.ws_bytes)
        api.combine(prob, lay.struct, w, acc, api.MOE_IN_ACCUMULATED, out)

    def step():
        if args.chain:
            chain()
        elif routed:
            L.forward(d["x"], d["x_scale"], logits=d["logits"], bias=d["bias"], out=out)
        else:
            L.forward(d["x"], d["x_scale"], topk_idx=d["topk_idx"], topk_weights=d["topk_weights"], out=out)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        flush_l2(1)
        step()
    torch.cuda.synchronize()
    L.check_status()

    # ---- device-resident timed region
    api.timing_enable(True, max(args.steps, 1))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2(i)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        clocks.sample()
    clocks.poll_until(ends[-1])
    torch.cuda.synchronize()
    barrier()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kern = api.timing_read()
    # the single launch's phase boundaries of the last step (workspace header)
    ts = L.ws[64:128].view(torch.int64).cpu().tolist()
    names = ("route", "permute", "gather+zero", "gemm1", "gemm2", "finalize")
    phases = ({n: (ts[i + 1] - ts[i]) / 1e3 for i, n in enumerate(names)}
              if not args.chain and ts[6] > ts[0] else None)
    api.timing_enable(False, 0)
    L.check_status()
    t_ms = sum(per_step)
    med_ms = statistics.median(per_step)
    launches = sum(n for _, n in kern.values())

    # ---- end to end through the public API, inputs from pinned host memory
    names = ["x"] + (["x_scale"] if d["x_scale"] is not None else []) + \
            (["logits", "bias"] if routed else ["topk_idx", "topk_weights"])
    host_in = {n: d[n].cpu().pin_memory() for n in names}
    dev_in = {n: torch.empty_like(d[n]) for n in names}
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = host_out.numel() * host_out.element_size()
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def e2e_step(i):
        for n in names:
            dev_in[n].copy_(host_in[n], non_blocking=True)
        if routed:
            L.forward(dev_in["x"], dev_in.get("x_scale"), logits=dev_in["logits"], bias=dev_in["bias"], out=out)
        else:
            L.forward(dev_in["x"], dev_in.get("x_scale"), topk_idx=dev_in["topk_idx"],
                      topk_weights=dev_in["topk_weights"], out=out)
        host_out.copy_(out, non_blocking=True)

    for i in range(min(args.warmup, 3)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    for i in range(args.steps):
        flush_l2(i)
        e_starts[i].record(stream)
        e2e_step(i)
        e_ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends))
    L.check_status()

    # ---- active experts of this batch (for the algorithmic byte counts)
    if routed:
        idx, _ = L.route(d["logits"], d["bias"])
    else:
        idx = d["topk_idx"]
    num_active = int(torch.unique(idx[idx >= 0]).numel())

    # ---- max over ranks
    t_ms, e2e_ms = max_over_ranks([t_ms, e2e_ms], world, dev)
    regime = api.tile_regime(L.problem(M))
    return dict(p=p, t_ms=t_ms, med_ms=med_ms, per_step=per_step, kern=kern, launches=launches, e2e_ms=e2e_ms, phases=phases,
                regime=regime,
                h2d=h2d, d2h=d2h, num_active=num_active, clocks=clocks.summary(), R=R, M=M,
                host_inputs=(d, L) if rank == 0 else None)


def _oracle_sample(p, host, seconds):
    """Runs the oracle on growing token samples until `seconds` of CPU work;
    returns (tokens done, seconds spent)."""
    import numpy as np
    from oracle import moe as O

    M, k = p["num_tokens"], p["num_topk"]
    order = np.random.default_rng(0).permutation(M)
    n, done, t_total = 1, 0, 0.0
    while True:
        toks = np.sort(order[done: done + n])
        if toks.size == 0:
            break
        t0 = time.perf_counter()
        if p["routing"] == "logits":
            O.route(host["logits"][toks], host["bias"], k)
        O.moe_forward(p, host, host["topk_idx"], host["topk_weights"], tokens=toks)
        t_total += time.perf_counter() - t0
        done += toks.size
        if t_total >= seconds or done >= M:
            break
        n = min(M - done, max(1, int(n * 2)))
    return done, t_total


def cpu_baseline(p, d, seconds):
    """The oracle, as it stands, on a bounded sample of this workload's tokens,
    with all host threads and with one thread."""
    import numpy as np
    from mixture_experts_routed_03_b200 import workloads
    from oracle import moe as O

    host = workloads.to_numpy({k: v for k, v in d.items()})
    if p["routing"] == "logits":
        host["topk_idx"], host["topk_weights"] = O.route(host["logits"], host["bias"], p["num_topk"])
        host["topk_weights"] = host["topk_weights"].astype(np.float32)
    M, k = p["num_tokens"], p["num_topk"]
    done, t_total = _oracle_sample(p, host, seconds)
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
        with threadpool_limits(limits=1):
            done1, t1 = _oracle_sample(p, host, seconds / 3)
        one = dict(value=done1 * k / t1, cores=1,
                   sample=f"{done1} of {M} tokens ({done1 * k} routed slots), {t1:.1f} s")
    except Exception:
        cores = os.cpu_count()
        one = None
    return dict(value=done * k / t_total, unit="routed_tokens/s", cores=cores, kind="oracle",
                sample=f"{done} of {M} tokens ({done * k} routed slots), float64 numpy oracle incl. "
                       f"per-expert weight decode, {t_total:.1f} s",
                one_thread=one)


def main_ours(args):
    import torch
    import torch.distributed as dist
    import datetime
    world, rank, local_rank = dist_env()
    if world > 1:
        # a short timeout ends a collective whose peer has gone with an error
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                timeout=datetime.timedelta(seconds=120))
    r = run_ours(args, rank, world, local_rank)
    p = r["p"]
    peaks, peak_src = load_peaks()
    value = job_throughput(r["R"], world, args.steps, r["t_ms"])
    e2e_value = job_throughput(r["R"], world, args.steps, r["e2e_ms"])
    wm = work_model(p, r["num_active"])
    kern = r["kern"]
    step_ms = r["t_ms"] / args.steps
    # dominant kernel of the step: the single moe_fused launch (whose
    # algorithmic work is the whole layer's), or the larger GEMM of a chain
    if kern.get("fused", (0.0, 0))[1]:
        slot, work = "fused", wm["layer"]
    else:
        slot = max(("gemm1", "gemm2"), key=lambda s: kern[s][0])
        work = wm[slot]
    k_ms = kern[slot][0] / max(kern[slot][1], 1)
    gemm_name = "moe_gemm_swap_kernel" if r["regime"] == "small_m" else "moe_gemm_kernel"
    bound = BOUND.get(args.workload, "hbm")
    if bound == "tensor":
        peak = peaks["bf16_tflops"] * FMT_TENSOR_RATIO[p["format"]]
        achieved = work["flops"] / (k_ms / 1e3) / 1e12
        unit = "TFLOP/s"
    else:
        peak = peaks["hbm_gbs"]
        achieved = work["bytes"] / (k_ms / 1e3) / 1e9
        unit = "GB/s"
    total_k = sum(v[0] for v in kern.values()) or 1.0
    # the layer's roofline as the pages' problem states it: the slower of its
    # FLOPs at the datasheet dense tensor peak of its format and its bytes at
    # ~8 TB/s, against the median step
    lw = wm["layer"]
    spec_t = max(lw["flops"] / (SPEC_TFLOPS[p["format"]] * 1e12), lw["bytes"] / (SPEC_HBM_GBS * 1e9))
    med_ms = r["med_ms"]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "routed_tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"bf16": "bf16", "fp8": "e4m3+f32 scales (f32 accumulate)",
                  "nvfp4": "e2m1+e4m3 scales (f32 accumulate)",
                  "mxfp8": "e4m3+ue8m0 scales per 32 (f32 accumulate)",
                  "fp8_tensor": "e4m3+f32 per-tensor scales (f32 accumulate)"}[p["format"]],
        "data": "synthetic (seeded torch generators; random-init experts of the workload's shapes)",
        "config": {"workload": args.workload + ("" if not args.set else " (" + ",".join(args.set) + ")"),
                   "path": "multi-launch chain" if args.chain else "moe_fused (one launch)",
                   "num_tokens": p["num_tokens"], "hidden": p["hidden"],
                   "intermediate_hidden": p["intermediate_hidden"], "num_experts": p["num_experts"],
                   "num_topk": p["num_topk"], "format": p["format"], "routing": p["routing"],
                   "active_experts": r["num_active"], "gemm_tiles": r["regime"],
                   "parallelism": f"dp{world} (replicas)",
                   "l2": ("hot: no flush between steps" if args.hot_l2 else
                          "flushed before every timed step, outside the step interval: 512 MiB write, "
                          "then a 512 MiB read of another buffer")},
        "tokens_per_s": job_throughput(p["num_tokens"], world, args.steps, r["t_ms"]),
        "layer_tflops": wm["layer"]["flops"] / (step_ms / 1e3) / 1e12,
        "layer_gbs": wm["layer"]["bytes"] / (step_ms / 1e3) / 1e9,
        "roofline": {"kernel": {"fused": "moe_fused_kernel",
                                "gemm1": gemm_name + " (gate_up)", "gemm2": gemm_name + " (down)"}[slot], "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "traffic": stored_traffic(args.workload, {"fused": "moe_fused_kernel", "gemm1": "gemm1",
                                                              "gemm2": "gemm2"}[slot]) if not args.set else None,
                     "peak_source": f"{peak_src} ({'bf16 burst x nominal ' + p['format'] + ' ratio' if bound == 'tensor' else 'hbm copy'})",
                     "kernel_ms": k_ms},
        "ms_per_step_median": med_ms,
        "value_median": job_throughput(r["R"], world, 1, med_ms),
        "roofline_spec": {"time_us": spec_t * 1e6,
                          "bound": "tensor" if lw["flops"] / (SPEC_TFLOPS[p["format"]] * 1e12) >=
                                   lw["bytes"] / (SPEC_HBM_GBS * 1e9) else "hbm",
                          "tensor_peak_tflops": SPEC_TFLOPS[p["format"]], "hbm_gbs": SPEC_HBM_GBS,
                          "frac": spec_t / (med_ms / 1e3),
                          "note": "B200 datasheet dense peak of the format and ~8 TB/s; median step"},
        "kernels_ms": {s: v[0] / max(v[1], 1) for s, v in kern.items() if v[1]},
        "fused_phases_us": r["phases"],
        "kernel_share": {s: v[0] / total_k for s, v in kern.items() if v[1]},
        "gpu_launches": r["launches"],
        "e2e": {"value": e2e_value, "unit": "routed_tokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"] / args.steps},
        "clocks": r["clocks"],
    }
    if rank == 0 and bound == "tensor" and not args.no_mma_peak:
        line["roofline"]["mma_probe"] = mma_probe(p["format"], achieved)
    if rank == 0 and world == 1 and not args.chain and not args.set and args.side_workloads:
        dev = torch.device("cuda", local_rank)
        line["workloads"] = {}
        for name in [n for n in args.side_workloads.split(",") if n and n != args.workload]:
            try:
                line["workloads"][name] = side_workload(name, args, dev, peaks)
            except Exception as e:  # a side line never takes the main one down
                line["workloads"][name] = {"error": str(e)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        d, _ = r["host_inputs"]
        line["cpu_baseline"] = cpu_baseline(p, d, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- reference arm

def main_reference(args):
    """The CPU oracle timed on the host cores, on this workload (rank 0 only;
    the other ranks return without work)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import numpy as np
    import torch

    from mixture_experts_routed_03_b200 import workloads
    from oracle import moe as O

    p = workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    host = workloads.to_numpy(workloads.make_inputs(p, seed=args.seed, device=dev))
    M, k = p["num_tokens"], p["num_topk"]
    if p["routing"] == "logits":
        idx_all, w_all = O.route(host["logits"], host["bias"], k)
    else:
        idx_all, w_all = host["topk_idx"], host["topk_weights"]
    rng = np.random.default_rng(0)
    # size one step to about 4 s of oracle work
    n = 1
    while True:
        toks = np.sort(rng.choice(M, size=n, replace=False))
        t0 = time.perf_counter()
        O.moe_forward(p, host, idx_all, w_all.astype(np.float32), tokens=toks)
        dt = time.perf_counter() - t0
        if dt >= 1.0 or n >= M:
            break
        n = min(M, n * 4)
    n = int(min(M, max(1, n * 4.0 / max(dt, 1e-3))))
    times = []
    for i in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(M, size=n, replace=False))
        t0 = time.perf_counter()
        if p["routing"] == "logits":
            O.route(host["logits"][toks], host["bias"], k)
        O.moe_forward(p, host, idx_all, w_all.astype(np.float32), tokens=toks)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    t = sum(times)
    value = n * k * args.steps / t
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    sample = f"{n} of {M} tokens per step ({n * k} routed slots), float64 numpy oracle"
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "routed_tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded torch generators)",
        "config": {"workload": args.workload, "num_tokens": M, "hidden": p["hidden"],
                   "intermediate_hidden": p["intermediate_hidden"], "num_experts": p["num_experts"],
                   "num_topk": k, "format": p["format"], "routing": p["routing"]},
        "cpu_baseline": {"value": value, "unit": "routed_tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "routed_tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        main_reference(args)
    else:
        main_ours(args)


if __name__ == "__main__":
    main()
