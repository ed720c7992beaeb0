#!/usr/bin/env python
"""Benchmark of the Gemma-4-26B-A4B MoE feed-forward block on B200.

One "step" is one pass of the block (router, top-k, permutation, gate|up and
down grouped GEMMs, shared MLP, combine) over one batch of T tokens, through
the library's C ABI. Default workload: the decode-sized block, T = 64 tokens;
on one GPU its line also carries the prefill-sized block (T = 4096, key
"prefill", timed first) and the NVFP4 30-layer stack (T = 2048, key
"nvfp4_stack", timed last), each measured the same way.

  python bench.py [--gpus N --steps K --warmup W] [--workload decode|tiny|prefill|skewed]
  python bench.py --impl reference ...   # the CPU oracle on the same workload

N > 1 (torchrun) runs N independent replicas, one per GPU: tokens are
independent in the block, so each rank processes its own batch with no
data-path collective (weak scaling). Timing is on the device with CUDA events,
bracketed by a barrier and a synchronize, max over ranks.

Prints ONE JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

D, E, F, S, K_TOP = 2816, 128, 704, 2112, 8
BYTES_PER_EXPERT = 3 * D * F * 2  # gate, up, down bf16
SHARED_BYTES = 3 * D * S * 2
ROUTER_BYTES = D * E * 2
FLOP_PER_TOKEN_GEMM = 2 * K_TOP * 3 * D * F + 2 * 3 * D * S  # tensor-core work
FLOP_PER_TOKEN = FLOP_PER_TOKEN_GEMM + 2 * D * E

WORKLOADS = {
    "tiny": dict(T=8, bias=False, bound="hbm", desc="Gemma-4-26B-A4B MoE block, T=8 tokens, bf16"),
    "decode": dict(T=64, bias=False, bound="hbm", desc="Gemma-4-26B-A4B MoE block, decode-sized T=64 tokens, bf16"),
    "prefill": dict(T=4096, bias=False, bound="tensor", desc="Gemma-4-26B-A4B MoE block, prefill-sized T=4096, bf16"),
    "skewed": dict(
        T=16384, bias=True, bound="tensor", desc="Gemma-4-26B-A4B MoE block, T=16384, Zipf(1.1) router bias, bf16"
    ),
    "nvfp4_stack": dict(
        T=2048,
        bias=False,
        bound="hbm",
        layers=30,
        desc="30 Gemma-4-26B-A4B MoE blocks in NVFP4 (group 16, e4m3 scales), RMSNorm between blocks, T=2048",
    ),
    "decode_sfp8": dict(
        T=64, bias=False, bound="hbm", wq="sfp8",
        desc="Gemma-4-26B-A4B MoE block, T=64 tokens, SFP8 weight-only expert and shared Linears, bf16 activations",
    ),
    "decode_q4_0": dict(
        T=64, bias=False, bound="hbm", wq="q4_0",
        desc="Gemma-4-26B-A4B MoE block, T=64 tokens, Q4_0 weight-only expert and shared Linears, bf16 activations",
    ),
    "e4b_dense_decode": dict(
        T=64, bias=False, bound="hbm", dense=True,
        desc="Gemma-4-E4B dense GeGLU FFN (embed 2560, hidden 10240), T=64 tokens, bf16",
    ),
    "e4b_dense": dict(
        T=4096, bias=False, bound="tensor", dense=True,
        desc="Gemma-4-E4B dense GeGLU FFN (embed 2560, hidden 10240), T=4096 tokens, bf16",
    ),
}
FP4_TFLOPS_NOMINAL_RATIO = 4.0  # dense fp4 : bf16 tensor throughput, nominal (9 : 2.25 PFLOP/s)
METRIC = "MoE-block tokens/s"

NVML_REASONS = {
    0x1: "gpu_idle",
    0x2: "applications_clocks_setting",
    0x4: "sw_power_cap",
    0x8: "hw_slowdown",
    0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode workload: skip the T=4096 prefill run that the default line carries")
    ap.add_argument("--no-stack", action="store_true",
                    help="decode workload: skip the NVFP4 30-layer stack run that the default line carries (one GPU)")
    ap.add_argument("--sandwich", action="store_true",
                    help="bf16 workloads: time the block with the pre/post-FFN RMSNorm sandwich and the residual add")
    ap.add_argument("--layers", type=int, default=None, help="nvfp4_stack depth (default 30)")
    return ap.parse_args()


# ------------------------------------------------------------ distributed


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return world, rank, local


def reduce_max(value: float, world: int) -> float:
    """Max over ranks (a barrier + one all-reduce); identity at world 1."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def aggregate(tokens_per_rank: int, steps: int, ms_max: float, world: int) -> dict:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    total_tokens = tokens_per_rank * steps * world
    return {"value": total_tokens / (ms_max / 1e3), "ms_per_step": ms_max / steps}


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no clocks
            self._nvml = None

    def _reasons_now(self):
        n = self._nvml
        fn = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or n.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self._h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons_now())
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def report(self):
        if not self._nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"], "samples": 0}
        names = [v for k, v in NVML_REASONS.items() if self.reasons & k and v != "gpu_idle"]
        return {
            "sm_mhz": statistics.median(self.samples) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": names,
            "samples": len(self.samples),
        }


# ----------------------------------------------------------------- peaks


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_digest(files) -> str:
    """Hash of the kernel source files an ncu capture was taken on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_transformer_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(f"{kernel}@{workload}")
    if not ent or ent.get("digest") != source_digest(ent.get("files", [])):
        return None
    return ent.get("bytes_per_launch")


# ----------------------------------------------------------- algorithmics


def algorithmic(kernel: str, T: int, touched: int, cnt: np.ndarray):
    """Algorithmic bytes and FLOPs of one launch of a kernel (each operand and
    result once)."""
    R = T * K_TOP
    if kernel == "grouped_gemm_gateup":
        byts = touched * 2 * D * F * 2 + 2 * D * S * 2 + R * D * 2 + T * D * 2 + R * F * 2 + T * S * 2
        flops = 2 * 2 * D * (R * F + T * S)
    elif kernel == "grouped_gemm_down":
        byts = touched * F * D * 2 + S * D * 2 + R * F * 2 + T * S * 2 + R * D * 2 + T * D * 4
        flops = 2 * D * (R * F + T * S)
    elif kernel == "route_scatter":
        byts = T * D * 2 + R * D * 2
        flops = 0
    elif kernel == "combine":
        byts = R * D * 2 + T * D * 4 + T * D * 2
        flops = 2 * R * D
    elif kernel == "router_logits":
        byts = T * D * 2 + D * E * 2
        flops = 2 * T * D * E
    else:
        byts, flops = 0, 0
    return byts, flops


# --------------------------------------------------------------- our arm


def gen_weights_gpu(seed: int = 0, std: float = 0.02):
    """Random-init weights of the published shapes, drawn on the GPU (seeded)."""
    import torch

    g = torch.Generator(device="cuda").manual_seed(seed)

    def rnd(*shape, s=std):
        return torch.empty(shape, dtype=torch.float32, device="cuda").normal_(0.0, s, generator=g).to(torch.bfloat16)

    from mixture_experts_transformer_b200 import block, inputs

    return block.DeviceWeights(
        inputs.GEMMA4_26B_A4B,
        rnd(D, E),
        rnd(E, D, F),
        rnd(E, D, F),
        rnd(E, F, D),
        rnd(D, S),
        rnd(D, S),
        rnd(S, D),
    )


def _bf16_config(wl, T, world, sandwich: bool) -> dict:
    """The config dict of a bf16 block workload (shared by our arm and the reference arm)."""
    return {
        "workload": wl["desc"] + (", with the pre/post-FFN RMSNorm sandwich and residual" if sandwich else ""),
        "tokens_per_gpu": T,
        "global_batch": T * world,
        "parallelism": f"replicas{world}" if world > 1 else "single",
        "l2": "inputs larger than L2 (1.5 GB of expert weights per step)",
        "router_bias": "zipf(1.1)" if wl["bias"] else None,
        "sandwich": bool(sandwich),
    }


def time_block(B, dw, T, bias, steps, warmup, world, local, sandwich, rank=0):
    """Time one bf16 block workload through the C ABI. Returns a dict with the
    aggregate, the per-kernel breakdown, the dominant kernel's own timing and
    the routing statistics.

    Three device-timed passes of `steps` steps each, after `warmup` untimed
    steps: (1) the headline region, events only at its ends, so every kernel
    keeps its programmatic-dependent-launch overlap; (2) events around the
    dominant kernel only (its achieved bandwidth / throughput); the breakdown
    of every kernel comes from a separate pass with events around each."""
    import torch

    from mixture_experts_transformer_b200 import block, inputs

    gx = torch.Generator(device="cuda").manual_seed(1 + rank)
    x = torch.empty((T, D), dtype=torch.float32, device="cuda").normal_(0.0, 1.0, generator=gx).to(torch.bfloat16)
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    ws, _ = block.workspace_for(inputs.GEMMA4_26B_A4B, T)
    stream = torch.cuda.current_stream()
    p = B.make_params(T, x, *dw.args(), out, router_bias=bias, workspace=ws, **sandwich)

    # routing statistics of this batch (outside the timed regions)
    dbg = block.forward(dw, x, router_bias=bias, debug=True, workspace=ws, **sandwich)
    torch.cuda.synchronize()
    cnt = dbg.cnt.cpu().numpy()
    del dbg
    st = B.moe_get_device_status()
    if st != B.MOE_OK:
        raise RuntimeError(B.moe_status_string(st))

    for _ in range(warmup):
        B.check(B.moe_block_forward_ex(p, stream), "forward")
    torch.cuda.synchronize()
    launches_per_step = B.moe_last_launch_count()

    # per-kernel breakdown: events around every kernel (a pass of its own)
    B.moe_profile_begin()
    for _ in range(min(steps, 50)):
        B.check(B.moe_block_forward_ex(p, stream), "forward")
    torch.cuda.synchronize()
    breakdown = B.moe_profile_end()
    dominant = max(breakdown, key=lambda k: breakdown[k][0])

    # (1) headline: device events around the K steps only
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(steps):
            B.check(B.moe_block_forward_ex(p, stream), "forward")
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(e0.elapsed_time(e1), world)

    # (2) the dominant kernel's own duration, events around it alone
    torch.cuda.synchronize()
    B.moe_profile_begin([dominant])
    for _ in range(steps):
        B.check(B.moe_block_forward_ex(p, stream), "forward")
    torch.cuda.synchronize()
    per_kernel = B.moe_profile_end()
    st = B.moe_get_device_status()
    if st != B.MOE_OK:
        raise RuntimeError(B.moe_status_string(st))
    return {
        "x": x, "out": out, "p": p, "ws": ws, "agg": aggregate(T, steps, ms, world), "breakdown": breakdown,
        "dominant": dominant, "dom_ms": per_kernel[dominant][0] / per_kernel[dominant][1],
        "clocks": clocks.report(), "cnt": cnt, "touched": int((cnt > 0).sum()),
        "launches_per_step": launches_per_step,
    }


def roofline_of(res, T, bound, peaks, ms_total) -> tuple[dict, dict]:
    """(roofline of the dominant kernel, whole-block roofline) for a bf16 block run."""
    dominant, dom_ms, touched, cnt = res["dominant"], res["dom_ms"], res["touched"], res["cnt"]
    byts, flops = algorithmic(dominant, T, touched, cnt)
    long_region = ms_total / 1e3 > 2.0
    if bound == "hbm":
        achieved = byts / (dom_ms / 1e3) / 1e9
        peak, unit, peak_name = peaks["hbm_gbs"], "GB/s", "hbm_gbs"
    else:
        achieved = flops / (dom_ms / 1e3) / 1e12
        peak_name = "bf16_tflops_sustained" if long_region else "bf16_tflops"
        peak, unit = peaks[peak_name], "TFLOP/s"
    step_ms = res["agg"]["ms_per_step"]
    weight_bytes = touched * BYTES_PER_EXPERT + SHARED_BYTES + ROUTER_BYTES
    roof = {
        "bound": bound,
        "kernel": dominant,
        "achieved": achieved,
        "peak": peak,
        "peak_source": f"{peaks['source']} {peak_name}",
        "unit": unit,
        "frac": achieved / peak,
        "traffic": None,
        "algorithmic_bytes": byts,
        "algorithmic_flops": flops,
        "kernel_ms": dom_ms,
        "kernel_timing": "a pass of its own of the same steps, events around this kernel only",
    }
    block_roof = {
        "hbm_touched_weights_gbs": weight_bytes / (step_ms / 1e3) / 1e9,
        "hbm_frac": weight_bytes / (step_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "tensor_tflops": T * FLOP_PER_TOKEN_GEMM / (step_ms / 1e3) / 1e12,
        "tensor_frac": T * FLOP_PER_TOKEN_GEMM / (step_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "touched_experts": touched,
    }
    return roof, block_roof


def run_ours(args, world, rank, local):
    import torch

    from mixture_experts_transformer_b200 import binding as B
    from mixture_experts_transformer_b200 import build, inputs

    if rank == 0:
        build.build()
    barrier(world)
    B.lib()
    torch.cuda.set_device(local)
    wl = WORKLOADS[args.workload]
    T = wl["T"]
    dw = gen_weights_gpu(seed=0)
    bias = torch.from_numpy(inputs.zipf_router_bias()).cuda() if wl["bias"] else None
    sandwich = {}
    if args.sandwich:
        # learned scales of the pre- and post-FFN RMSNorm, seeded U(0.5, 1.5)
        gs = torch.Generator(device="cuda").manual_seed(9)
        sandwich = {
            "norm_pre": torch.empty(D, device="cuda").uniform_(0.5, 1.5, generator=gs).to(torch.bfloat16),
            "norm_post": torch.empty(D, device="cuda").uniform_(0.5, 1.5, generator=gs).to(torch.bfloat16),
            "residual": True,
        }
    # ---- the metric's prefill half: the T = 4096 block, timed the same way,
    # first: the tensor-bound half draws the most power, and timed after the
    # decode half's passes it ran at a lower power-capped clock
    prefill = None
    if args.workload == "decode" and not args.no_prefill:
        wp = WORKLOADS["prefill"]
        res_p = time_block(B, dw, wp["T"], None, args.steps, args.warmup, world, local, sandwich, rank)
        del res_p["ws"], res_p["x"], res_p["out"], res_p["p"]
        prefill = res_p
        torch.cuda.empty_cache()
        # let the power limiter's average settle before the decode half, as
        # between two separate runs (timing is on the device in both halves)
        time.sleep(3.0)

    res_t = time_block(B, dw, T, bias, args.steps, args.warmup, world, local, sandwich, rank)
    x, out, p = res_t["x"], res_t["out"], res_t["p"]
    agg = res_t["agg"]
    stream = torch.cuda.current_stream()

    # ---- end to end: host buffers through the C ABI, copies inside the timed
    # region. Two streams, each with its own device buffers and workspace,
    # take alternate batches, as a serving loop would: one batch's copies
    # overlap the other's kernels, and every batch's host-to-device and
    # device-to-host copies stay inside the timed region.
    from mixture_experts_transformer_b200 import block as blk
    from mixture_experts_transformer_b200 import inputs as inp

    x_host = x.cpu().pin_memory()
    lanes = []
    for _ in range(2):
        xk, ok_ = torch.empty_like(x), torch.empty_like(out)
        wsk, _ = blk.workspace_for(inp.GEMMA4_26B_A4B, T)
        pk = B.make_params(T, xk, *dw.args(), ok_, router_bias=bias, workspace=wsk, **sandwich)
        lanes.append((torch.cuda.Stream(), pk, torch.empty((T, D), dtype=torch.bfloat16).pin_memory(), xk, ok_, wsk))

    def e2e_batch(i):
        st, pk, oh = lanes[i % 2][:3]
        B.check(B.moe_block_forward_hostio(pk, x_host, oh, st), "hostio")

    for i in range(4):
        e2e_batch(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for ln in lanes:
        ln[0].wait_stream(stream)
    for i in range(args.steps):
        e2e_batch(i)
    for ln in lanes:
        stream.wait_stream(ln[0])
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t0.elapsed_time(t1), world)
    barrier(world)
    if not all(torch.equal(ln[2], out.cpu()) for ln in lanes):
        raise RuntimeError("host-buffer path disagrees with the device path")
    del lanes
    ws_bytes = res_t["ws"].numel()
    del res_t["ws"], res_t["x"], res_t["out"], res_t["p"]

    if rank != 0:
        return None

    peaks = measured_peaks()
    step_ms = agg["ms_per_step"]
    roof, block_roof = roofline_of(res_t, T, wl["bound"], peaks, agg["ms_per_step"] * args.steps)
    roof["traffic"] = ncu_traffic(res_t["dominant"], args.workload)
    res = {
        "metric": METRIC,
        "value": agg["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,0.02) random-init weights of the published shapes, x ~ N(0,1)",
        "config": _bf16_config(wl, T, world, args.sandwich),
        "roofline": roof,
        "block_roofline": block_roof,
        "kernels_ms_per_launch": {k: v[0] / v[1] for k, v in res_t["breakdown"].items()},
        "gpu_launches": res_t["launches_per_step"] * args.steps,
        "e2e": {
            "value": T * args.steps * world / (e2e_ms / 1e3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": T * D * 2,
            "d2h_bytes_per_step": T * D * 2,
            "overlap": "two streams take alternate batches through moe_block_forward_hostio",
        },
        "clocks": res_t["clocks"],
        "workspace_bytes": ws_bytes,
    }
    if prefill is not None:
        wp = WORKLOADS["prefill"]
        proof, pblock = roofline_of(prefill, wp["T"], wp["bound"], peaks, prefill["agg"]["ms_per_step"] * args.steps)
        proof["traffic"] = ncu_traffic(prefill["dominant"], "prefill")
        res["prefill"] = {
            "metric": METRIC,
            "value": prefill["agg"]["value"],
            "unit": "tokens/s",
            "ms_per_step": prefill["agg"]["ms_per_step"],
            "steps": args.steps,
            "config": _bf16_config(wp, wp["T"], world, args.sandwich),
            "roofline": proof,
            "block_roofline": pblock,
            "tensor_frac": pblock["tensor_frac"],
            "kernels_ms_per_launch": {k: v[0] / v[1] for k, v in prefill["breakdown"].items()},
            "gpu_launches": prefill["launches_per_step"] * args.steps,
            "clocks": prefill["clocks"],
        }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(dw, x, bias, T, budget_s=12.0, sandwich=sandwich)
    return res


# ------------------------------------------------------------ NVFP4 stack


def run_stack(args, world, rank, local):
    """One step = the 30-layer NVFP4 stack over T=2048 tokens."""
    import torch

    from mixture_experts_transformer_b200 import binding as B
    from mixture_experts_transformer_b200 import block, build
    from mixture_experts_transformer_b200 import stack as stk

    if rank == 0:
        build.build()
    barrier(world)
    B.lib()
    torch.cuda.set_device(local)
    wl = WORKLOADS["nvfp4_stack"]
    T, L = wl["T"], (args.layers or wl["layers"])
    gcal = torch.Generator(device="cuda").manual_seed(2)
    x_calib = torch.empty((256, D), device="cuda").normal_(0.0, 1.0, generator=gcal).to(torch.bfloat16)
    st, kept = stk.build_stack(
        lambda l: gen_weights_gpu(seed=l), L, x_calib, keep_bf16=set(range(min(L, 2))) if world == 1 else None
    )
    gx = torch.Generator(device="cuda").manual_seed(1 + rank)
    x = torch.empty((T, D), device="cuda").normal_(0.0, 1.0, generator=gx).to(torch.bfloat16)
    ws = stk.stack_workspace(st, T)
    bufs = [torch.empty((T, D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    stream = torch.cuda.current_stream()

    # touched experts per layer (routing statistics, outside the timed region)
    touched = []
    cur = x
    for l in range(L):
        r = block.forward_nvfp4(st.layers[l], cur, st.scales[l], rms_norm_out=True, debug=True, workspace=ws)
        touched.append(int((r.cnt > 0).sum().item()))
        cur = r.out.clone()
    if B.moe_get_device_status() != B.MOE_OK:
        raise RuntimeError("device status after the debug pass")

    for _ in range(args.warmup):
        stk.stack_forward(st, x, bufs, ws, stream)
    torch.cuda.synchronize()
    launches_per_step = 0
    B.moe_profile_begin()
    stk.stack_forward(st, x, bufs, ws, stream)
    torch.cuda.synchronize()
    breakdown = B.moe_profile_end()
    launches_per_step = sum(v[1] for v in breakdown.values())
    dominant = max(breakdown, key=lambda k: breakdown[k][0])

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            stk.stack_forward(st, x, bufs, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(e0.elapsed_time(e1), world)
    agg = aggregate(T, args.steps, ms, world)
    # the dominant kernel's own duration, in a pass of its own: an event
    # between two kernels ends their programmatic-launch overlap
    B.moe_profile_begin([dominant])
    for _ in range(args.steps):
        stk.stack_forward(st, x, bufs, ws, stream)
    torch.cuda.synchronize()
    per_kernel = B.moe_profile_end()
    if B.moe_get_device_status() != B.MOE_OK:
        raise RuntimeError("device status after the timed region")

    # end to end: host tokens in, host tokens out, through the library per layer
    x_host = x.cpu().pin_memory()
    out_host = torch.empty((T, D), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        r = stk.stack_forward(st, x_dev, bufs, ws, stream)
        out_host.copy_(r.out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t0.elapsed_time(t1), world)
    barrier(world)
    if rank != 0:
        return None

    peaks = measured_peaks()
    step_ms = agg["ms_per_step"]
    dom_ms = per_kernel[dominant][0] / per_kernel[dominant][1]
    mean_touched = float(np.mean(touched))
    dims = st.dims
    lin = lambda K, N: N * K // 2 + ((N + 127) // 128) * (K // 64) * 512  # noqa: E731
    R = T * K_TOP
    if dominant == "fp4_gemm_gateup":
        byts = mean_touched * 2 * lin(D, F) + 2 * lin(D, S) + (R + T) * (D // 2 + D // 16) + (R * F + T * S) * 9 // 16
    elif dominant == "fp4_gemm_down":
        byts = mean_touched * lin(F, D) + lin(S, D) + (R * F + T * S) * 9 // 16 + R * D * 2 + T * D * 4
    else:
        byts, _ = algorithmic(dominant, T, int(mean_touched), None)
    weight_bytes = sum(stk.fp4_weight_bytes(dims, t) for t in touched) + L * ROUTER_BYTES
    fp4_peak = peaks["bf16_tflops"] * FP4_TFLOPS_NOMINAL_RATIO
    gemm_flops = L * T * FLOP_PER_TOKEN_GEMM
    res = {
        "metric": METRIC,
        "value": agg["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 group scales, fp32 accumulate; router bf16)",
        "data": "synthetic: seeded N(0,0.02) random-init weights per layer (seed = layer), x ~ N(0,1)",
        "config": {
            "workload": wl["desc"] if L == 30 else wl["desc"].replace("30 ", f"{L} "),
            "tokens_per_gpu": T,
            "layers": L,
            "global_batch": T * world,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (13 GB of NVFP4 weights per step)",
            "calibration": "static activation scales from a 256-token batch (seed 2) through the stack",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": dominant,
            "achieved": byts / (dom_ms / 1e3) / 1e9,
            "peak": peaks["hbm_gbs"],
            "peak_source": f"{peaks['source']} hbm_gbs",
            "unit": "GB/s",
            "frac": byts / (dom_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "traffic": ncu_traffic(dominant, "nvfp4_stack"),
            "algorithmic_bytes": byts,
            "kernel_ms": dom_ms,
        },
        "block_roofline": {
            "hbm_weights_gbs": weight_bytes / (step_ms / 1e3) / 1e9,
            "hbm_frac": weight_bytes / (step_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "fp4_tensor_tflops": gemm_flops / (step_ms / 1e3) / 1e12,
            "fp4_tensor_frac": gemm_flops / (step_ms / 1e3) / 1e12 / fp4_peak,
            "fp4_peak_tflops": fp4_peak,
            "fp4_peak_source": "measured bf16 burst x nominal fp4:bf16 ratio 4",
            "touched_experts_mean": mean_touched,
        },
        "kernels_ms_per_launch": {k: v[0] / v[1] for k, v in breakdown.items()},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {
            "value": T * args.steps * world / (e2e_ms / 1e3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": T * D * 2,
            "d2h_bytes_per_step": T * D * 2,
        },
        "clocks": clocks.report(),
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_stack(kept, x, L)
    return res


def cpu_baseline_stack(kept, x, n_layers, budget_s=12.0):
    """The oracle's NVFP4 block on one token through the first kept layers,
    scaled to the whole stack (per-token, per-layer time x layers)."""
    from oracle import moe_oracle as mo
    from oracle import nvfp4 as nv

    xb = x[:1].cpu().view(__import__("torch").int16).numpy().view(np.uint16)
    hosts = [_host_weights(kept[l]) for l in sorted(kept)]
    scales = [nv.act_scales_from_calibration(xb, *(h.w_router, h.wg, h.wu, h.wd, h.sg, h.su, h.sd)) for h in hosts]
    t0 = time.perf_counter()
    n = 0
    while True:
        cur = xb
        for h, sc in zip(hosts, scales):
            out = nv.moe_block_nvfp4(cur, h.w_router, h.wg, h.wu, h.wd, h.sg, h.su, h.sd, *sc)["out"]
            from mixture_experts_transformer_b200 import inputs

            cur = inputs.f32_to_bf16_bits(mo.rms_normalize(out).astype(np.float32))
            n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    per_token_layer = el / n
    return {
        "value": 1.0 / (per_token_layer * n_layers),
        "unit": "tokens/s",
        "cores": _oracle_cores(),
        "kind": "oracle",
        "sample": f"1 token through layers {sorted(kept)} of the stack {n} times in {el:.1f} s, scaled to {n_layers} layers",
    }


# ----------------------------------------------------------- CPU oracle


def _host_weights(dw):
    from mixture_experts_transformer_b200 import inputs

    def u16(t):
        return t.cpu().view(__import__("torch").int16).numpy().view(np.uint16)

    return inputs.BlockWeights(*(u16(t) for t in dw.args()))


def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info

        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) if threadpool_info() else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(dw, x, bias, T, budget_s=12.0, sample_tokens=None, sandwich=None):
    """The oracle as it stands, on a bounded sample of the same workload."""
    from oracle import moe_oracle as mo
    from oracle import sandwich as sw

    wh = _host_weights(dw)
    xb = x.cpu().view(__import__("torch").int16).numpy().view(np.uint16)
    b = None if bias is None else bias.cpu().numpy()
    n = min(T, sample_tokens or 64)
    xs = xb[:n]
    done, t0 = 0, time.perf_counter()
    args_w = (wh.w_router, wh.wg, wh.wu, wh.wd, wh.sg, wh.su, wh.sd)
    if sandwich:
        g_pre, g_post = (sandwich[k].float().cpu().numpy() for k in ("norm_pre", "norm_post"))
    while True:
        if sandwich:
            sw.sandwich_block(xs, *args_w, g_pre, g_post, top_k=K_TOP, bias=b)
        else:
            mo.moe_block(xs, *args_w, top_k=K_TOP, bias=b)
        done += n
        if time.perf_counter() - t0 > budget_s or done >= 64 * n:
            break
    el = time.perf_counter() - t0
    return {
        "value": done / el,
        "unit": "tokens/s",
        "cores": _oracle_cores(),
        "kind": "oracle",
        "sample": f"{done} tokens ({done // n} passes over the first {n} tokens of the batch), {el:.1f} s",
    }


def run_reference(args, world, rank):
    """The CPU oracle on our arm's workload, metric and unit (rank 0 only)."""
    if rank != 0:
        return None
    import torch

    from mixture_experts_transformer_b200 import inputs
    from oracle import moe_oracle as mo

    wl = WORKLOADS[args.workload]
    T = wl["T"]
    if wl.get("wq"):
        return {"impl": "reference", "unavailable": "the oracle's weight-only block quantises every touched expert's "
                "weights per call (minutes of host time per step), beyond a bounded step"}
    if args.workload == "nvfp4_stack":
        # one oracle step re-quantises the weights of every touched expert
        # (~126 x 3 matrices per layer, minutes per layer on the host)
        return {"impl": "reference", "unavailable": "the oracle's NVFP4 block needs minutes of host time per layer "
                "(it re-quantises every touched expert's weights per call), beyond a bounded step; this workload's "
                "own line carries its cpu_baseline (one token through the first layers, scaled)"}
    # the same bounded sample as our arm's cpu_baseline leg: the first 64
    # tokens of the batch (the whole batch at the decode workload)
    n = min(T, 64)
    metric = METRIC
    if wl.get("dense"):
        dw = inputs.make_dense_weights()
        x = inputs.make_x(n, inputs.E4B_EMBED_DIM)
        metric = "dense FFN tokens/s"
        step = lambda: mo.dense_ffn(x, dw.wg, dw.wu, dw.wd)  # noqa: E731
    else:
        w = inputs.make_weights()
        x = inputs.make_x(n)
        bias = inputs.zipf_router_bias() if wl["bias"] else None
        args_w = (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    if wl.get("dense"):
        pass
    elif args.sandwich:
        from oracle import sandwich as sw

        rng = np.random.default_rng(9)
        g_pre, g_post = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
        step = lambda: sw.sandwich_block(x, *args_w, g_pre, g_post, bias=bias)  # noqa: E731
    else:
        step = lambda: mo.moe_block(x, *args_w, bias=bias)  # noqa: E731
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = n * args.steps / el
    cores = _oracle_cores()
    return {
        "impl": "reference",
        "metric": metric,
        "value": v,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded N(0,0.02) random-init weights of the published shapes, x ~ N(0,1)",
        "config": _dense_config(wl, T, world) if wl.get("dense") else _bf16_config(wl, T, world, args.sandwich),
        "cpu_baseline": {
            "value": v,
            "unit": "tokens/s",
            "cores": cores,
            "kind": "oracle",
            "sample": f"each step: the first {n} of the workload's {T} tokens through the fp64 oracle"
            + ("" if n == T else f", scaled to tokens/s per token (tokens are independent in the block)"),
        },
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _dense_config(wl, T, world) -> dict:
    return {
        "workload": wl["desc"],
        "tokens_per_gpu": T,
        "global_batch": T * world,
        "parallelism": f"replicas{world}" if world > 1 else "single",
        "l2": "weights 157 MB, larger than L2",
    }


def run_dense(args, world, rank, local):
    """One step = the dense GeGLU FFN of the E4B sibling over T tokens."""
    import torch

    from mixture_experts_transformer_b200 import binding as B
    from mixture_experts_transformer_b200 import block, build, inputs

    if rank == 0:
        build.build()
    barrier(world)
    B.lib()
    torch.cuda.set_device(local)
    wl = WORKLOADS[args.workload]
    T, Dd, Sd = wl["T"], inputs.E4B_EMBED_DIM, inputs.E4B_HIDDEN_DIM
    g = torch.Generator(device="cuda").manual_seed(0)

    def rnd(*shape, s=0.02):
        return torch.empty(shape, device="cuda").normal_(0.0, s, generator=g).to(torch.bfloat16)

    wg, wu, wd = rnd(Dd, Sd), rnd(Dd, Sd), rnd(Sd, Dd)
    gx = torch.Generator(device="cuda").manual_seed(1 + rank)
    x = torch.empty((T, Dd), device="cuda").normal_(0.0, 1.0, generator=gx).to(torch.bfloat16)
    out = torch.empty((T, Dd), dtype=torch.bfloat16, device="cuda")
    p0 = B.make_dense_params(T, embed_dim=Dd, hidden_dim=Sd)
    ws = torch.empty(B.moe_dense_workspace_bytes(p0), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    p = B.make_dense_params(T, x, wg, wu, wd, out, embed_dim=Dd, hidden_dim=Sd, workspace=ws)
    block.dense_forward(x, wg, wu, wd, debug=True, workspace=ws)
    for _ in range(max(args.warmup, 3)):
        B.check(B.moe_dense_ffn_forward(p, stream), "dense")
    torch.cuda.synchronize()
    launches = B.moe_last_launch_count()
    # per-kernel breakdown (a separate pass)
    B.moe_profile_begin()
    for _ in range(min(args.steps, 50)):
        B.check(B.moe_dense_ffn_forward(p, stream), "dense")
    torch.cuda.synchronize()
    breakdown = B.moe_profile_end()
    dominant = max(breakdown, key=lambda k: breakdown[k][0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            B.check(B.moe_dense_ffn_forward(p, stream), "dense")
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(e0.elapsed_time(e1), world)
    agg = aggregate(T, args.steps, ms, world)
    B.moe_profile_begin([dominant])  # the dominant kernel alone, outside the timed region
    for _ in range(args.steps):
        B.check(B.moe_dense_ffn_forward(p, stream), "dense")
    torch.cuda.synchronize()
    per_kernel = B.moe_profile_end()
    if B.moe_get_device_status() != B.MOE_OK:
        raise RuntimeError("device status after the timed region")
    # end to end through the public call: pinned host x in, host out back
    x_host = x.cpu().pin_memory()
    out_host = torch.empty((T, Dd), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    pe = B.make_dense_params(T, x_dev, wg, wu, wd, out, embed_dim=Dd, hidden_dim=Sd, workspace=ws)

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        B.check(B.moe_dense_ffn_forward(pe, stream), "dense")
        out_host.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t0.elapsed_time(t1), world)
    barrier(world)
    if rank != 0:
        return None
    peaks = measured_peaks()
    step_ms = agg["ms_per_step"]
    flops = 2.0 * 3 * Dd * Sd * T
    wbytes = 3 * Dd * Sd * 2
    dom_ms = per_kernel[dominant][0] / per_kernel[dominant][1]
    if dominant == "grouped_gemm_gateup":
        dom_bytes, dom_flops = 2 * Dd * Sd * 2 + T * Dd * 2 + T * Sd * 2, 2.0 * 2 * Dd * Sd * T
    else:
        dom_bytes, dom_flops = Sd * Dd * 2 + T * Sd * 2 + T * Dd * 2, 2.0 * Dd * Sd * T
    if wl["bound"] == "hbm":
        ach, peak, unit, byts = dom_bytes / (dom_ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s", dom_bytes
    else:
        ach, peak, unit, byts = dom_flops / (dom_ms / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s", dom_bytes
    res = {
        "metric": "dense FFN tokens/s",
        "value": agg["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,0.02) random-init weights of the published E4B FFN shapes, x ~ N(0,1)",
        "config": _dense_config(wl, T, world),
        "roofline": {
            "bound": wl["bound"],
            "kernel": dominant,
            "achieved": ach,
            "peak": peak,
            "peak_source": f"{peaks['source']} " + ("hbm_gbs" if wl["bound"] == "hbm" else "bf16_tflops"),
            "unit": unit,
            "frac": ach / peak,
            "traffic": None,
            "algorithmic_bytes": byts,
            "kernel_ms": dom_ms,
        },
        "block_roofline": {
            "hbm_weights_gbs": wbytes / (step_ms / 1e3) / 1e9,
            "hbm_frac": wbytes / (step_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "tensor_tflops": flops / (step_ms / 1e3) / 1e12,
            "tensor_frac": flops / (step_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        },
        "kernels_ms_per_launch": {k: v[0] / v[1] for k, v in breakdown.items()},
        "gpu_launches": launches * args.steps,
        "e2e": {
            "value": T * args.steps * world / (e2e_ms / 1e3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": T * Dd * 2,
            "d2h_bytes_per_step": T * Dd * 2,
        },
        "clocks": clocks.report(),
    }
    if world == 1 and not args.no_cpu_baseline:
        from oracle import moe_oracle as mo

        wh = [a.float().cpu().numpy() for a in (wg, wu, wd)]
        xs = x[: min(T, 64)].float().cpu().numpy()
        done, t0s = 0, time.perf_counter()
        while True:
            mo.dense_ffn(xs, *wh)
            done += xs.shape[0]
            if time.perf_counter() - t0s > 12.0 or done >= 64 * xs.shape[0]:
                break
        el = time.perf_counter() - t0s
        res["cpu_baseline"] = {
            "value": done / el,
            "unit": "tokens/s",
            "cores": _oracle_cores(),
            "kind": "oracle",
            "sample": f"{done} tokens ({done // xs.shape[0]} passes over the first {xs.shape[0]} tokens), {el:.1f} s",
        }
    return res


def wq_weight_bytes(fmt: str, K: int, N: int) -> int:
    """Bytes of one [K, N] Linear in the library's weight-only layout (rows padded to 128)."""
    blk = 8192 if fmt == "sfp8" else 4608
    return ((N + 127) // 128) * (K // 64) * blk


def run_wq(args, world, rank, local):
    """One step = the block with weight-only SFP8 / Q4_0 weights over T tokens."""
    import torch

    from mixture_experts_transformer_b200 import binding as B
    from mixture_experts_transformer_b200 import block, build, inputs

    if rank == 0:
        build.build()
    barrier(world)
    B.lib()
    torch.cuda.set_device(local)
    wl = WORKLOADS[args.workload]
    T, fmt = wl["T"], wl["wq"]
    ww = block.quantize_wq(gen_weights_gpu(seed=0), fmt)
    torch.cuda.synchronize()
    gx = torch.Generator(device="cuda").manual_seed(1 + rank)
    x = torch.empty((T, D), dtype=torch.float32, device="cuda").normal_(0.0, 1.0, generator=gx).to(torch.bfloat16)
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    p0 = block.wq_params(ww, T, None, None)
    ws = torch.empty(B.moe_wq_workspace_bytes(p0), dtype=torch.uint8, device="cuda")
    p = block.wq_params(ww, T, x, out, workspace=ws)
    stream = torch.cuda.current_stream()
    dbg = block.forward_wq(ww, x, debug=True, workspace=ws)
    torch.cuda.synchronize()
    cnt = dbg.cnt.cpu().numpy()
    touched = int((cnt > 0).sum())
    if B.moe_get_device_status() != B.MOE_OK:
        raise RuntimeError("device status after the debug pass")
    for _ in range(max(args.warmup, 3)):
        B.check(B.moe_block_forward_wq(p, stream), "wq")
    torch.cuda.synchronize()
    launches = B.moe_last_launch_count()
    B.moe_profile_begin()
    for _ in range(min(args.steps, 50)):
        B.check(B.moe_block_forward_wq(p, stream), "wq")
    torch.cuda.synchronize()
    breakdown = B.moe_profile_end()
    dominant = max(breakdown, key=lambda k: breakdown[k][0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            B.check(B.moe_block_forward_wq(p, stream), "wq")
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(e0.elapsed_time(e1), world)
    agg = aggregate(T, args.steps, ms, world)
    B.moe_profile_begin([dominant])
    for _ in range(args.steps):
        B.check(B.moe_block_forward_wq(p, stream), "wq")
    torch.cuda.synchronize()
    per_kernel = B.moe_profile_end()
    if B.moe_get_device_status() != B.MOE_OK:
        raise RuntimeError("device status after the timed region")
    # end to end: pinned host x in, host out back, through the public call
    x_host = x.cpu().pin_memory()
    out_host = torch.empty((T, D), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    pe = block.wq_params(ww, T, x_dev, out, workspace=ws)

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        B.check(B.moe_block_forward_wq(pe, stream), "wq")
        out_host.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(t0.elapsed_time(t1), world)
    barrier(world)
    if rank != 0:
        return None
    peaks = measured_peaks()
    step_ms = agg["ms_per_step"]
    R = T * K_TOP
    e_gu = 2 * wq_weight_bytes(fmt, D, F)
    e_dn = wq_weight_bytes(fmt, F, D)
    sh_gu, sh_dn = 2 * wq_weight_bytes(fmt, D, S), wq_weight_bytes(fmt, S, D)
    if dominant == "grouped_gemm_gateup":
        byts = touched * e_gu + sh_gu + (R + T) * D * 2 + (R * F + T * S) * 2
    elif dominant == "grouped_gemm_down":
        byts = touched * e_dn + sh_dn + (R * F + T * S) * 2 + R * D * 2 + T * D * 4
    else:
        byts, _ = algorithmic(dominant, T, touched, cnt)
    dom_ms = per_kernel[dominant][0] / per_kernel[dominant][1]
    weight_bytes = touched * (e_gu + e_dn) + sh_gu + sh_dn + ROUTER_BYTES
    return {
        "metric": METRIC,
        "value": agg["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"{fmt} weights (weight-only), bf16 activations, fp32 accumulate",
        "data": "synthetic: seeded N(0,0.02) random-init weights of the published shapes, quantised by the library",
        "config": {
            "workload": wl["desc"],
            "tokens_per_gpu": T,
            "global_batch": T * world,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": dominant,
            "achieved": byts / (dom_ms / 1e3) / 1e9,
            "peak": peaks["hbm_gbs"],
            "peak_source": f"{peaks['source']} hbm_gbs",
            "unit": "GB/s",
            "frac": byts / (dom_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "traffic": ncu_traffic(dominant, args.workload),
            "algorithmic_bytes": byts,
            "kernel_ms": dom_ms,
        },
        "block_roofline": {
            "hbm_touched_weights_gbs": weight_bytes / (step_ms / 1e3) / 1e9,
            "hbm_frac": weight_bytes / (step_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "touched_experts": touched,
            "weight_bytes": weight_bytes,
        },
        "kernels_ms_per_launch": {k: v[0] / v[1] for k, v in breakdown.items()},
        "gpu_launches": launches * args.steps,
        "e2e": {
            "value": T * args.steps * world / (e2e_ms / 1e3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": T * D * 2,
            "d2h_bytes_per_step": T * D * 2,
        },
        "clocks": clocks.report(),
    }


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        elif args.workload == "nvfp4_stack":
            res = run_stack(args, world, rank, local)
        elif WORKLOADS[args.workload].get("dense"):
            res = run_dense(args, world, rank, local)
        elif WORKLOADS[args.workload].get("wq"):
            res = run_wq(args, world, rank, local)
        else:
            res = run_ours(args, world, rank, local)
            if args.workload == "decode" and world == 1 and not args.no_stack and not args.sandwich:
                # the NVFP4 30-layer stack (T=2048), timed the same way, as a key of the default line
                import copy

                import torch

                torch.cuda.empty_cache()
                time.sleep(3.0)
                sargs = copy.copy(args)
                sargs.workload, sargs.no_cpu_baseline, sargs.layers = "nvfp4_stack", True, None
                res["nvfp4_stack"] = run_stack(sargs, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
