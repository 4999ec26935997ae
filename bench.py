"""Benchmark: MoE FFN layer forward + backward on B200, tokens/s.

One step = the whole hot path over one batch: route (logits, softmax/top-k,
counts, offsets, slot rows) -> dispatch -> grouped SwiGLU FFN forward ->
combine -> combine backward -> grouped FFN backward (dgrad + wgrad) ->
unpermute-grad + router grad (the MXFP8 workload also quantises its FP32
master weights inside every step).  Inputs are seeded synthetic tensors
already resident in HBM; L2 is flushed (256 MiB write) between timed steps,
outside the timed events.  The timed step is a CUDA-graph replay of the C-ABI
calls.  A profiled pass of eager steps then times every kernel launch of the
library with CUDA events (moe_profile_begin / moe_profile_end): the roofline
of the grouped GEMM is taken from the GEMM launches alone.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--capacity-factor] [--recompute] [--accum G] [--no-sweep]
                    [--impl {ours,reference}]

Default workload: mxfp8_e128 (T=32768, d_model=4096, E=128, top_k=4,
d_ff=1536, MXFP8), the largest configuration that fits one GPU.  With the
default workload on one GPU the line also carries a ``sweep`` measured in the
same process: bf16_e8 and bf16_e128 (the expert-pool sweep at fixed
activation), bf16_skew_e128 dropless and padded (device-scheduled against
uniform capacity), and the MXFP8 workload's shapes in bf16 (MXFP8 vs bf16).

Multi-GPU: ``--gpus N`` starts N ranks itself (torch.distributed.run, one
process per GPU, NCCL) unless it already runs under a launcher.  Data
parallel with weak scaling: each rank runs its own token batch (seed = rank)
through its own replica of the layer.  One step is then one optimizer step of
the pages' DDP (kongchang, 容量税: gradients synchronised once per optimizer
step): G micro-batches (``--accum``, default 8 when N > 1) whose weight
gradients accumulate in place, then one all-reduce of dW1, dW2 and dW_router
over NCCL.  The timed region is bracketed by a barrier and a device
synchronisation; the time is the max over ranks.

``--impl reference`` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_offsets_b200 import dist as mdist  # noqa: E402
from mixture_experts_layer_offsets_b200 import inputs  # noqa: E402

METRIC = "MoE FFN fwd+bwd tokens/s on 1 B200; grouped-GEMM % of tensor-core peak"
DEFAULT_WORKLOAD = "mxfp8_e128"
FLUSH_BYTES = 256 << 20
FP8_OVER_BF16 = 2.0   # nominal dense tensor-core ratio (4.5 / 2.25 PFLOP/s)
PHASES = ["quantize_w", "route", "dispatch", "ffn_fwd", "combine", "combine_bwd", "ffn_bwd",
          "route_bwd"]
SWEEP = [("bf16_e8", False, None), ("bf16_e128", False, None), ("bf16_skew_e128", False, None),
         ("bf16_skew_e128", True, None), ("mxfp8_e128", False, "bf16")]

# DRAM bytes (read + write) of the grouped-GEMM launches of one step, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) per workload, with the SHA-256 of the
# GEMM source it was taken on: reported only while that source is unchanged.
GEMM_TRAFFIC = {
    # the six grouped-GEMM launches of a step of mxfp8_e128 at E=16, T=4096 (the same 1024
    # tokens per expert, so every operand and result is 1/8 of the full step's), mean of
    # two steps (2.7199e9 and 2.7174e9 bytes), times 8
    "mxfp8_e128": (21749104640,
                   "378c5362fcf5a9c14aff1d513afeccb423d593e6630c61d4407135140546b152",
                   "scaled x8 from a capture at E=16, T=4096 (1024 tokens per expert as here); "
                   "ncu flushes L2 before each launch and counts the writes that reach DRAM "
                   "while it runs"),
}
GEMM_SOURCES = ("mixture_experts_layer_offsets_b200/csrc/gemm_sm100.cu",
                "mixture_experts_layer_offsets_b200/csrc/common.cuh",
                "mixture_experts_layer_offsets_b200/csrc/mx_common.cuh")


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def resolve(args) -> inputs.MoEConfig:
    cfg = inputs.CONFIGS[args.workload]
    if args.tokens:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@T{args.tokens}", T=args.tokens)
    if args.experts:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@E{args.experts}", E=args.experts)
    if args.dtype and args.dtype != cfg.dtype:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@{args.dtype}", dtype=args.dtype)
    return cfg


def _workload_desc(cfg, capacity, recompute=False, accum=1, world=1):
    d = {"workload": f"{cfg.name}: T={cfg.T} d_model={cfg.d_model} E={cfg.E} top_k={cfg.top_k} "
                     f"d_ff={cfg.d_ff} {cfg.dtype}",
         "T": cfg.T, "d_model": cfg.d_model, "E": cfg.E, "top_k": cfg.top_k, "d_ff": cfg.d_ff,
         "routing": "skewed (logit bias std 2)" if cfg.bias_std else "near-uniform random",
         "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
         "weight_grad_dtype": "fp32"}
    if cfg.dtype == "mxfp8":
        d["operands"] = ("MXFP8 (E4M3 + E8M0 per 32 along K) for all six expert GEMMs; bf16 "
                         "activations; FP32 master weights quantised to four MXFP8 copies "
                         "once per optimizer step, by its first micro-batch (inside the timed "
                         "step)")
    if recompute:
        d["recompute"] = "gate/up GEMM re-run in the backward (a | u | h not kept from the forward)"
    d["layout"] = (f"padded capacity C={capacity} (overflow dropped)" if capacity else
                   "dropless, device-scheduled grouped GEMM")
    d["parallelism"] = f"dp{world}"
    if world > 1 or accum > 1:
        d["step"] = (f"one optimizer step: {accum} micro-batches of T tokens per rank, weight "
                     "gradients accumulated in place" +
                     (", then one NCCL all-reduce of dW1, dW2, dW_router" if world > 1 else ""))
    return d


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------- algorithmic work
def gemm_flop(cfg) -> float:
    """Algorithmic FLOPs of the six expert GEMMs of one step: 18 R d f (dropless rows)."""
    return 18.0 * cfg.R * cfg.d_model * cfg.d_ff


def gemm_bytes(cfg) -> float:
    """Algorithmic DRAM bytes of the six expert GEMMs of one dropless step without recompute:
    each operand read once (a weight once per GEMM), each result written once.  MXFP8
    operands are 1 byte per element plus one scale byte per 32; the MXFP8 epilogues write
    h and [da | du] as their two MXFP8 copies, the bf16 ones write them in bf16."""
    R, d, f, E = cfg.R, cfg.d_model, cfg.d_ff, cfg.E
    if cfg.dtype == "mxfp8":
        s = 1 + 1 / 32
        fwd = (R * d * s + E * 2 * f * d * s + R * 3 * f * 2 + 2 * R * f * s +   # gate/up
               R * f * s + E * d * f * s + R * d * 2)                            # down
        bwd = (R * d * s + E * d * f * s + R * 2 * f * 2 + 2 * R * 2 * f * s +   # dh, da|du
               R * 2 * f * s + E * 2 * f * d * s + R * d * 2 +                   # dx_perm
               R * d * s + R * f * s + E * d * f * 4 +                           # dW2
               R * 2 * f * s + R * d * s + E * 2 * f * d * 4)                    # dW1
        return fwd + bwd
    b = 4 if cfg.dtype == "f32" else 2
    fwd = (R * d * b + E * 2 * f * d * b + R * 3 * f * b +
           R * f * b + E * d * f * b + R * d * b)
    bwd = (R * d * b + E * d * f * b + R * 2 * f * b + R * 2 * f * b +
           R * 2 * f * b + E * 2 * f * d * b + R * d * b +
           R * d * b + R * f * b + E * d * f * 4 +
           R * 2 * f * b + R * d * b + E * 2 * f * d * 4)
    return fwd + bwd


def kernel_bytes(cfg, capacity=None, recompute=False) -> dict:
    """Algorithmic HBM bytes per step of the row-moving and quantising kernels (each
    operand read once, each result written once), by launch name.  The MXFP8 layer
    (without recompute) runs the combine backward fused with dy's quantisation: that
    launch writes no dy_perm rows, and the quantiser reads dout's rows instead."""
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff
    R = E * capacity if capacity else cfg.R
    s = 4 if cfg.dtype == "f32" else 2
    router = T * d * s + E * d * s + T * E * 4 + T * k * 12
    out = {
        "router_gemm": router,   # tensor-core tile router (up to 256 experts)
        "router_mma": router,    # warp-level router (up to 32 experts)
        "permute": T * d * s + R * d * s + T * k * 8,
        "combine": R * d * s + T * d * s + T * k * 8,
        "combine_bwd": T * d * s + (1 if cfg.dtype == "mxfp8" and not recompute else 2) * R * d * s
        + T * k * 12,
    }
    if cfg.dtype == "mxfp8":
        mx = 2 * (1 + 1 / 32)  # two E4M3 copies with their E8M0 scales, per element
        out["mx_weights"] = 4 * E * 3 * f * d + mx * E * 3 * f * d
        # x (gathered rows) and dy (gate x dout rows, without recompute): bf16 in, both
        # MXFP8 copies out; h and [da | du] leave the GEMM epilogues already quantised
        # unless MOE_B200_HMX / MOE_B200_DADU = 0 route them through this kernel too
        # (the recompute quantises x, and h if it goes through here, a second time)
        passes = 2 if recompute else 1
        widths = [d] * passes + [d]
        if os.environ.get("MOE_B200_HMX", "") == "0":
            widths += [f] * passes
        if os.environ.get("MOE_B200_DADU", "") == "0":
            widths.append(2 * f)
        out["mx_act"] = R * sum(widths) * (2 + mx)
    return out


# ------------------------------------------------------------ one layer
class LayerStep:
    """Device buffers, inputs and the call sequence of one layer step through the C ABI."""

    def __init__(self, cfg, dev, seed, capacity=None, recompute=False):
        from mixture_experts_layer_offsets_b200.layer import MoELayer
        self.cfg, self.dev, self.capacity, self.recompute = cfg, dev, capacity, recompute
        self.inp = inputs.make_inputs(cfg, device=dev, seed=seed)
        self.L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, dev,
                          dw_dtype="f32", capacity=capacity, recompute=recompute)

    def grads(self):
        return [self.L.dw1, self.L.dw2, self.L.dw_router]

    def run(self, ev=None, accumulate=False, stream=None):
        from mixture_experts_layer_offsets_b200 import capi
        L, cfg = self.L, self.cfg
        st = stream or torch.cuda.current_stream()
        x, wr, b, w1, w2, dout = (self.inp[k] for k in ("x", "w_router", "bias", "w1", "w2",
                                                         "dout"))

        def mark(i):
            if ev is not None:
                ev[i].record(st)
        s, dt, fdt = L.shape, L.cdtype, L.ffn_dtype
        acc = capi.MOE_DW_ACCUMULATE if accumulate else 0
        mark(0)
        # the MXFP8 weight copies are made once per optimizer step, by its first
        # micro-batch (the later ones, which accumulate, run on the same weights)
        if cfg.dtype == "mxfp8" and not accumulate:
            L.quantize_weights(w1, w2)
        mark(1)
        capi.moe_route(s, dt, x, wr, b, L.logits, L.topk_idx, L.topk_gate, L.counts, L.offsets,
                       L.slot_row, L.ws)
        mark(2)
        if self.capacity:
            capi.moe_padded_dispatch(s, dt, self.capacity, x, L.topk_idx, L.slot_row, L.offsets,
                                     L.x_perm, L.pad_row, L.offsets_pad)
        elif L.fused_dispatch:
            capi.moe_permute_mx(s, x, L.slot_row, L.offsets, L.perm_src, L.ws)
        else:
            capi.moe_permute(s, dt, x, L.slot_row, L.x_perm, L.perm_src)
        mark(3)
        capi.moe_grouped_ffn_fwd(s, fdt, L.rows, L.x_perm, L.ffn_offsets, w1, w2, L.act, L.y_perm,
                                 L.ws, mx=L.mx)
        mark(4)
        capi.moe_combine(s, dt, L.y_perm, L.row_map, L.topk_gate, L.out)
        mark(5)
        if L.fused_dispatch:
            capi.moe_combine_bwd_mx(s, dout, L.y_perm, L.row_map, L.topk_gate, L.perm_src,
                                    L.dgate, L.ws)
        else:
            capi.moe_combine_bwd(s, dt, dout, L.y_perm, L.row_map, L.topk_gate, L.dy_perm,
                                 L.dgate)
        mark(6)
        bwd = capi.moe_grouped_ffn_bwd_recompute if self.recompute else capi.moe_grouped_ffn_bwd
        bwd(s, fdt, L.rows, L.dy_perm, L.x_perm, L.act, L.ffn_offsets, w1, w2, L.dx_perm, L.dw1,
            L.dw2, capi.MOE_F32 | acc, L.ws, mx=L.mx)
        mark(7)
        capi.moe_route_bwd(s, dt | acc, x, wr, L.logits, L.topk_idx, L.dgate, L.dx_perm,
                           L.row_map, L.dx, L.dw_router, L.ws)
        mark(8)


def capture(fn):
    """A CUDA graph of fn() (warmed once on a side stream, as graph capture requires)."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def dp_timed(step_fn, steps, warmup, world, device, flush=None, sampler=None, timer="cuda"):
    """Time `steps` calls of step_fn after `warmup` untimed ones: barrier and device
    synchronisation on both sides, one event pair (or host clock on CPU) per step, L2
    flushed between steps outside the events; returns (max over ranks of the total ms,
    per-step ms of this rank)."""
    cuda = timer == "cuda"
    for _ in range(warmup):
        step_fn()
    if cuda:
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    if cuda:
        torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    per = []
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        if cuda:
            evs[i][0].record()
            step_fn()
            evs[i][1].record()
        else:
            t0 = time.perf_counter()
            step_fn()
            per.append((time.perf_counter() - t0) * 1e3)
    if cuda:
        torch.cuda.synchronize()
        per = [a.elapsed_time(b) for a, b in evs]
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    total = mdist.max_over_ranks(sum(per), device=device)
    return total, per, clocks


def measure(cfg, dev, rank, world, steps, warmup, capacity=None, recompute=False, accum=1,
            clocks=True, profile_steps=5):
    """Timed CUDA-graph steps of one workload, then a profiled pass of eager steps.
    Returns (LayerStep, result dict)."""
    from mixture_experts_layer_offsets_b200 import capi
    ls = LayerStep(cfg, dev, mdist.rank_seed(0, rank), capacity, recompute)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        ls.run()
    torch.cuda.synchronize()
    if ls.L.device_status() != 0:
        raise SystemExit("device status reported a timeout during warm-up")
    # The timed step replays CUDA graphs of the whole path (the library makes no host
    # synchronisation and no allocation, so the calls capture as they are).
    g_over = capture(lambda: ls.run())
    g_acc = capture(lambda: ls.run(accumulate=True)) if accum > 1 else None

    def step():
        for m in range(accum):
            (g_acc if m else g_over).replay()
        if world > 1:
            mdist.allreduce_grads(ls.grads())

    sampler = ClockSampler(torch.cuda.current_device()) if (clocks and rank == 0) else None
    total_ms, per, clk = dp_timed(step, steps, warmup, world, dev, flush, sampler)
    ms_per_step = total_ms / steps
    del g_over, g_acc

    # Profiled pass: eager steps, a GPU-side delay first so that the host enqueues the
    # whole step before the GPU reaches it (the events then see device time only).
    nph = max(1, profile_steps)
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(nph)]
    kernels = {}
    n_launch = 0
    for i in range(nph):
        flush.zero_()
        torch.cuda._sleep(3_000_000)
        with capi.Profile(256) as prof:
            ls.run(pev[i])
        for name, ms in prof.launches():
            e = kernels.setdefault(name, [0, 0.0])
            e[0] += 1
            e[1] += ms
        n_launch = prof.count
    torch.cuda.synchronize()
    ph = {p: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in pev)
          for i, p in enumerate(PHASES)}
    kern = {k: {"launches_per_step": v[0] // nph, "ms_per_step": round(v[1] / nph, 4)}
            for k, v in sorted(kernels.items(), key=lambda kv: -kv[1][1])}
    gemm_ms = sum(v[1] for k, v in kernels.items() if k.startswith("gemm_")) / nph
    gemm_launches = sum(v[0] for k, v in kernels.items() if k.startswith("gemm_")) // nph
    status = ls.L.device_status()
    res = {"ms_per_step": ms_per_step, "per_step_ms": per, "clocks": clk, "phases_ms": ph,
           "kernels": kern, "gemm_ms": gemm_ms, "gemm_launches": gemm_launches,
           "launches_per_micro_batch": n_launch, "device_status": status}
    return ls, res


def dp_line(cfg, total_ms, steps, warmup, accum, world) -> dict:
    """The head of the JSON line: whole-job tokens/s over all ranks from the max-over-ranks
    time of `steps` timed steps of `accum` micro-batches of T tokens per rank."""
    ms = total_ms / steps
    return {"metric": METRIC, "value": round(cfg.T * accum * world / (ms / 1e3), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic (seeded; random-init weights)"}


def roofline(cfg, res, capacity=None, recompute=False):
    pk, pk_kind = _peaks()
    flop = gemm_flop(cfg)
    gemm_ms = res["gemm_ms"]
    achieved = flop / (gemm_ms / 1e3) / 1e12
    if cfg.dtype == "bf16":
        peak, kind = pk["bf16_tflops"], f"bf16_tflops burst, {pk_kind}"
    elif cfg.dtype == "mxfp8":
        peak = pk["bf16_tflops"] * FP8_OVER_BF16
        kind = f"bf16_tflops burst ({pk_kind}) x {FP8_OVER_BF16} nominal fp8/bf16 ratio"
    else:
        peak, kind = None, "fp32 CUDA-core path: no tensor-core peak"
    tr = GEMM_TRAFFIC.get(cfg.name) if not capacity else None
    traffic = tr[0] if tr and tr[1] == gemm_source_sha() else None
    alg = None if capacity or recompute else round(gemm_bytes(cfg))
    out = {"bound": "tensor",
           "kernel": f"grouped GEMM (tcgen05): the {res['gemm_launches']} expert-FFN GEMM "
                     "launches of a step (gemm_* in kernels_ms)",
           "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
           "frac": round(achieved / peak, 4) if peak else None, "peak_kind": kind,
           "traffic": traffic,
           "traffic_unit": "DRAM bytes per step over the six grouped-GEMM launches (ncu "
                           "dram__bytes_read.sum + dram__bytes_write.sum); null unless "
                           "captured on this GEMM source",
           "traffic_note": tr[2] if traffic else None,
           "algorithmic_bytes_per_step": alg,
           "algorithmic_flop_per_step": flop, "gemm_ms_per_step": round(gemm_ms, 4),
           "timing": "CUDA events around each GEMM launch (moe_profile_begin), eager steps"}
    return out


def hbm_kernels(cfg, res, capacity=None, recompute=False):
    """Achieved bandwidth of the memory-bound kernels from their algorithmic bytes."""
    pk, pk_kind = _peaks()
    out = {}
    for name, nbytes in kernel_bytes(cfg, capacity, recompute).items():
        k = res["kernels"].get(name)
        if not k or k["ms_per_step"] <= 0:
            continue
        gbs = nbytes / (k["ms_per_step"] / 1e3) / 1e9
        out[name] = {"bytes_per_step": int(nbytes), "ms_per_step": k["ms_per_step"],
                     "gb_s": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4)}
    return out


def run_ours(args, rank, world):
    cfg = resolve(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    from mixture_experts_layer_offsets_b200 import capi
    shape = capi.shape_of(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff)
    capacity = (capi.moe_capacity(shape, *cfg.padded_cf)
                if args.capacity_factor and cfg.padded_cf else None)
    accum = args.accum if args.accum else (8 if world > 1 else 1)
    ls, res = measure(cfg, dev, rank, world, args.steps, args.warmup, capacity, args.recompute,
                      accum)
    e2e = None if args.no_e2e else run_e2e(args, ls, dev, capacity, world, accum)
    del ls
    torch.cuda.empty_cache()

    sweep = None
    if (not args.no_sweep and world == 1 and args.workload == DEFAULT_WORKLOAD and
            not (args.tokens or args.experts or args.dtype or args.capacity_factor or
                 args.recompute)):
        sweep = run_sweep(args, dev)

    if rank != 0:
        return None
    line = dp_line(cfg, res["ms_per_step"] * args.steps, args.steps, args.warmup, accum, world)
    line.update({
        "config": _workload_desc(cfg, capacity, args.recompute, accum, world),
        "roofline": roofline(cfg, res, capacity, args.recompute),
        "hbm_kernels": hbm_kernels(cfg, res, capacity, args.recompute),
        "phases_ms": {k: round(v, 4) for k, v in res["phases_ms"].items()},
        "kernels_ms": res["kernels"],
        "timing": "value: CUDA-graph replay of the step, CUDA events per step, max over ranks; "
                  "phases_ms, kernels_ms and roofline: eager steps with CUDA events between "
                  "calls and around every launch (host kept ahead of the GPU)",
        "gpu_launches": res["launches_per_micro_batch"] * accum * args.steps,
        "device_status": res["device_status"],
        "e2e": e2e,
        "clocks": res["clocks"],
    })
    if sweep:
        line["sweep"] = sweep
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_seconds, single_core=True)
    return line


def run_sweep(args, dev):
    """The comparison workloads, measured in this process with the same timing."""
    out = {}
    steps = min(args.steps, 10)
    from mixture_experts_layer_offsets_b200 import capi
    for name, padded, dtype in SWEEP:
        cfg = inputs.CONFIGS[name]
        if dtype:
            cfg = inputs.shrink(cfg, name=f"{name}@{dtype}", dtype=dtype)
        shape = capi.shape_of(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff)
        capacity = capi.moe_capacity(shape, *cfg.padded_cf) if padded else None
        ls, res = measure(cfg, dev, 0, 1, steps, 3, capacity, profile_steps=3)
        del ls
        torch.cuda.empty_cache()
        rf = roofline(cfg, res, capacity)
        key = cfg.name + ("_padded" if padded else "")
        out[key] = {"value": round(cfg.T / (res["ms_per_step"] / 1e3), 1), "unit": "tokens/s",
                    "ms_per_step": round(res["ms_per_step"], 4), "steps": steps,
                    "gemm_tflops": rf["achieved"], "gemm_frac": rf["frac"],
                    "gemm_ms_per_step": rf["gemm_ms_per_step"],
                    "layout": "padded capacity C=%d" % capacity if capacity else "dropless",
                    "clocks": res["clocks"], "device_status": res["device_status"]}
    if "bf16_e8" in out and "bf16_e128" in out:
        out["e_sweep_drop"] = round(1 - out["bf16_e128"]["value"] / out["bf16_e8"]["value"], 4)
    if "bf16_skew_e128" in out and "bf16_skew_e128_padded" in out:
        out["padded_over_dropless"] = round(out["bf16_skew_e128_padded"]["value"] /
                                            out["bf16_skew_e128"]["value"], 4)
    return out


def run_e2e(args, ls, dev, capacity, world, accum):
    """Same metric through the public API with pinned host buffers: every micro-batch copies
    its inputs x and dout host->device and its outputs out and dx device->host, inside the
    timed region.  Micro-batches are pipelined the way an input pipeline would run them: two
    layer instances take turns (sharing one set of weight-gradient buffers), and while one
    computes on the compute stream, the next one's inputs come in on a copy stream and the
    previous one's outputs go out on another; events order every copy against the compute
    that produces or reuses its buffers.  With N > 1 every `accum` micro-batches end with
    the all-reduce of the gradients.  The working set is several times L2, so no flush."""
    from mixture_experts_layer_offsets_b200.layer import MoELayer
    L = ls.L
    L2 = MoELayer(L.T, L.d, L.E, L.k, L.f, L.dtype, dev, dw_dtype=L.dw_dtype, capacity=capacity,
                  recompute=L.recompute)
    L2.dw1, L2.dw2, L2.dw_router = L.dw1, L.dw2, L.dw_router
    if L.mx is not None:
        L2.share_weight_copies(L)
    layers = [L, L2]
    inp = ls.inp
    hx = inp["x"].cpu().pin_memory()
    hd = inp["dout"].cpu().pin_memory()
    hout = [torch.empty_like(hx).pin_memory() for _ in range(2)]
    hdx = [torch.empty_like(hx).pin_memory() for _ in range(2)]
    xin = [torch.empty_like(inp["x"]) for _ in range(2)]
    din = [torch.empty_like(inp["dout"]) for _ in range(2)]
    wr, b, w1, w2 = inp["w_router"], inp["bias"], inp["w1"], inp["w2"]
    cs = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def issue(i):
        k = i % 2
        h2d.wait_event(ev_comp[k])            # micro-batch i-2 has finished reading buffer k
        with torch.cuda.stream(h2d):
            xin[k].copy_(hx, non_blocking=True)
            din[k].copy_(hd, non_blocking=True)
            ev_in[k].record(h2d)
        cs.wait_event(ev_in[k])
        cs.wait_event(ev_out[k])              # micro-batch i-2's outputs have left layer k
        first = i % accum == 0  # first micro-batch of an optimizer step
        layers[k].step(xin[k], wr, b, w1, w2, din[k], accumulate=not first, requantize=first)
        if world > 1 and (i % accum) == accum - 1:
            mdist.allreduce_grads([L.dw1, L.dw2, L.dw_router])
        ev_comp[k].record(cs)
        d2h.wait_event(ev_comp[k])
        with torch.cuda.stream(d2h):
            hout[k].copy_(layers[k].out, non_blocking=True)
            hdx[k].copy_(layers[k].dx, non_blocking=True)
            ev_out[k].record(d2h)

    n_warm = max(2, args.warmup) * accum
    for i in range(n_warm):
        issue(i)
    torch.cuda.synchronize()
    n = max(2, args.steps) * accum
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    st.record(cs)
    h2d.wait_event(st)
    d2h.wait_event(st)
    for i in range(n):
        issue(i)
    cs.wait_event(ev_out[0])
    cs.wait_event(ev_out[1])
    en.record(cs)
    torch.cuda.synchronize()
    ms = mdist.max_over_ranks(st.elapsed_time(en) / n, device=dev)
    status = max(layers[0].device_status(), layers[1].device_status())
    T = inp["x"].shape[0]
    nbytes = hx.numel() * hx.element_size()
    del L2
    return {"value": round(T * world / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": 2 * nbytes * accum, "d2h_bytes_per_step": 2 * nbytes * accum,
            "ms_per_micro_batch": round(ms, 4), "micro_batches": n, "device_status": status,
            "api": "MoELayer.step (C ABI) with pinned host buffers; copies of micro-batch i+1 in "
                   "and i-1 out overlap micro-batch i's compute (two layer instances, three "
                   "streams)"}


# ------------------------------------------------- CPU oracle (baseline)
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    return os.cpu_count()


def _draw_weights(cfg, g, E):
    T, d, f = cfg.T, cfg.d_model, cfg.d_ff
    wr = (torch.randn(E, d, generator=g) * cfg.router_std).to(cfg.act_dtype).double().numpy()
    w1 = (torch.randn(E, 2 * f, d, generator=g) * cfg.w_std).to(cfg.weight_dtype).double().numpy()
    w2 = (torch.randn(E, d, f, generator=g) * cfg.w_std).to(cfg.weight_dtype).double().numpy()
    bias = (torch.randn(E, generator=g) * cfg.bias_std).double().numpy() if cfg.bias_std else None
    return wr, w1, w2, bias


def cpu_baseline(cfg, budget_s=12.0, chunk=64, single_core=False):
    """The float64 oracle on a bounded sample of the workload, tokens/s.

    bf16 / fp32 workloads: whole oracle fwd+bwd calls on micro-batches of `chunk` tokens
    (the full expert weights) until `budget_s` seconds have run.

    MXFP8: the oracle quantises every expert weight on each call (four MXFP8 copies of the
    FP32 masters), which at E = 128 alone is minutes of float64 work.  The step is
    therefore extrapolated from two samples with the workload's d_model, d_ff and top_k:
    (a) the oracle's four weight quantisations of whole experts, one expert after another
    until `budget_s` has run (at least one), scaled to E experts (once per step, as the layer
    does); (b) the cost per token: one oracle call on 256 tokens with E_s = max(top_k, 4)
    experts minus the quantisation of those E_s experts timed alone (the call re-quantises
    them), timed once per process and reused by later samples.

    With ``single_core`` the line also carries the rate with one BLAS thread, so that the
    all-core and the one-core figure are both reported."""
    if cfg.dtype == "mxfp8":
        cb = _cpu_baseline_mx(cfg, budget_s)
        if single_core:
            cb["single_core"] = ("not run: the MXFP8 oracle's time is its element-wise "
                                 "quantisation, which NumPy runs on one core either way")
        return cb
    from oracle import moe_ref as ref
    g = torch.Generator().manual_seed(0)
    T, d, k = cfg.T, cfg.d_model, cfg.top_k
    wr, w1, w2, bias = _draw_weights(cfg, g, cfg.E)

    def run(budget):
        done = 0
        t0 = time.perf_counter()
        while True:
            x = torch.randn(chunk, d, generator=g).to(cfg.act_dtype).double().numpy()
            dout = torch.randn(chunk, d, generator=g).to(cfg.act_dtype).double().numpy()
            ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, bias)
            done += chunk
            el = time.perf_counter() - t0
            if el >= budget or done >= T:
                return done, el
    run(0.0)   # one untimed call: thread-pool start, first touch of the weights
    done, el = run(budget_s)
    cb = {"value": round(done / el, 2), "unit": "tokens/s", "cores": _blas_threads(),
          "kind": "oracle", "extrapolated": False, "sample_s": round(el, 2),
          "sample": f"{done} of {T} tokens of {cfg.name} in micro-batches of {chunk} "
                    f"(full expert weights; float64 NumPy), {el:.1f} s"}
    if single_core:
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                d1, e1 = run(max(2.0, budget_s / 4))
            cb["single_core"] = {"value": round(d1 / e1, 2), "cores": 1,
                                 "sample": f"{d1} tokens with one BLAS thread, {e1:.1f} s"}
        except ImportError:
            cb["single_core"] = "not run: threadpoolctl is missing"
    return cb


def _mx_quantise_experts(mxr, w1, w2):
    """The oracle's four MXFP8 copies of these experts' weights (what a step makes)."""
    Es, f2, d = w1.shape
    f = f2 // 2
    mxr.mx_qdq(w1.reshape(Es * 2 * f, d), 0)
    mxr.mx_qdq(w2.reshape(Es * d, f), 0)
    mxr.mx_qdq(w2.reshape(Es * d, f), 1)
    mxr.mx_qdq(w1.reshape(Es * 2 * f, d), 1)


_MX_TOKEN_COST = {}


def _mx_token_cost(cfg, mxr, tokens=256):
    """Seconds per token of the oracle MXFP8 layer call with the workload's d_model, d_ff,
    top_k and E_s = max(top_k, 4) experts: one call on `tokens` tokens minus the oracle's
    quantisation of those E_s experts timed alone (the call re-quantises them).  Measured
    once per process."""
    key = (cfg.d_model, cfg.d_ff, cfg.top_k, cfg.act_dtype, cfg.weight_dtype)
    if key not in _MX_TOKEN_COST:
        g = torch.Generator().manual_seed(0)
        Es = max(cfg.top_k, 4)
        wr, w1, w2, bias = _draw_weights(cfg, g, Es)
        t0 = time.perf_counter()
        _mx_quantise_experts(mxr, w1, w2)
        t_w = time.perf_counter() - t0
        x = torch.randn(tokens, cfg.d_model, generator=g).to(cfg.act_dtype).double().numpy()
        dout = torch.randn(tokens, cfg.d_model, generator=g).to(cfg.act_dtype).double().numpy()
        t0 = time.perf_counter()
        mxr.layer_fwd_bwd_mx(x, wr, w1, w2, dout, cfg.top_k, bias, act_round=mxr.round_bf16)
        t_call = time.perf_counter() - t0
        _MX_TOKEN_COST[key] = (max(t_call - t_w, 1e-9) / tokens, tokens, Es, t_w, t_call)
    return _MX_TOKEN_COST[key]


def _cpu_baseline_mx(cfg, budget_s=12.0):
    from oracle import moe_mx_ref as mxr
    per_token, tokens, Es, t_w_es, t_call = _mx_token_cost(cfg, mxr)
    g = torch.Generator().manual_seed(1)
    d, f, k = cfg.d_model, cfg.d_ff, cfg.top_k
    _, w1, w2, _ = _draw_weights(cfg, g, 1)
    n, t_w = 0, 0.0
    while n == 0 or (t_w < budget_s and n < cfg.E):
        t0 = time.perf_counter()
        _mx_quantise_experts(mxr, w1, w2)
        t_w += time.perf_counter() - t0
        n += 1
    step_s = t_w / n * cfg.E + per_token * cfg.T
    return {"value": round(cfg.T / step_s, 3), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle", "extrapolated": True, "sample_s": round(t_w, 2),
            "extrapolated_step_s": round(step_s, 1),
            "sample": (f"{cfg.name} extrapolated: oracle weight quantisation (four MXFP8 "
                       f"copies) of {n} of {cfg.E} experts {t_w:.1f} s (x {cfg.E / n:g}, once "
                       f"per step) + {per_token * 1e3:.2f} ms per token (x {cfg.T}): one oracle "
                       f"MXFP8 layer call on {tokens} tokens with {Es} experts, d_model={d}, "
                       f"d_ff={f}, top_k={k}, {t_call:.1f} s, minus the quantisation of those "
                       f"{Es} experts alone, {t_w_es:.1f} s (timed once per process)")}


def run_reference(args, rank, world):
    """The float64 oracle as the reference arm: each step is one bounded sample of the
    workload (see cpu_baseline); ms_per_step is the time that sample took, value the rate
    it gives for the workload (extrapolated for MXFP8)."""
    if rank != 0:
        return None
    cfg = resolve(args)
    budget = max(2.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(min(args.warmup, 1)):
        cpu_baseline(cfg, budget_s=min(1.0, budget))
    steps = [cpu_baseline(cfg, budget_s=budget) for _ in range(args.steps)]
    v = statistics.mean(s["value"] for s in steps)
    cb = dict(steps[-1])
    cb["value"] = round(v, 3)
    ms = statistics.mean(s["sample_s"] for s in steps) * 1e3
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 1),
            "ms_per_step_kind": "measured time of one sampled step (see cpu_baseline.sample)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _workload_desc(cfg, None), "cpu_baseline": cb,
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------- launching
def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launcher_argv(n: int, argv: list[str], port: int) -> list[str]:
    """The command that runs this script as n ranks of one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.CONFIGS))
    ap.add_argument("--capacity-factor", action="store_true",
                    help="padded-capacity layout (workloads that define a capacity factor)")
    ap.add_argument("--recompute", action="store_true",
                    help="backward recomputes a | u | h (moe_grouped_ffn_bwd_recompute)")
    ap.add_argument("--accum", type=int, default=0,
                    help="micro-batches per optimizer step (default 1 on one GPU, 8 on more)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--dtype", default=None, choices=["f32", "bf16", "mxfp8"],
                    help="run the workload's shapes at another compute dtype")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller cases for profiling); not a bench line")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiling); not a bench line")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    return args


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        if args.impl == "ours" and torch.cuda.device_count() < args.gpus:
            raise SystemExit(f"--gpus {args.gpus}: only {torch.cuda.device_count()} GPUs visible")
        return subprocess.call(launcher_argv(args.gpus, argv, _free_port()))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
        return 0
    torch.cuda.set_device(local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
