"""Benchmark: MoE FFN layer forward + backward on B200, tokens/s.

One step = the whole hot path over one batch: route (logits, softmax/top-k,
counts, offsets, slot rows) -> permute -> grouped SwiGLU FFN forward ->
combine -> combine backward -> grouped FFN backward (dgrad + wgrad) ->
unpermute-grad + router grad.  Inputs are seeded synthetic tensors already
resident in HBM; L2 is flushed (256 MiB write) between timed steps, outside
the timed events.  The timed step is a CUDA-graph replay of the C-ABI calls;
the per-phase breakdown comes from eager steps with events between calls.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--capacity-factor] [--impl {ours,reference}]

Multi-GPU (torchrun, one process per GPU): data parallel with weak scaling,
each rank runs its own token batch (seed = rank) through its own copy of the
layer; there is no collective inside a step.  The timed region is bracketed
by a barrier and a device synchronisation; the time is the max over ranks.

``--impl reference`` times the float64 CPU oracle on the host cores on a
bounded token sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
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
FLUSH_BYTES = 256 << 20
def launches_per_step(cfg, capacity, recompute, fused_dispatch) -> int:
    """Kernel launches of this library in one step, counted per C-ABI call from the
    launch sequences in csrc (and checked against ncu launch lists)."""
    mx, f32 = cfg.dtype == "mxfp8", cfg.dtype == "f32"
    tc_router_bwd = not f32 and cfg.E % 128 == 0 and cfg.top_k <= 8 and cfg.d_model % 256 == 0
    n = 2 if mx else 0                                   # the two weight quantisers
    n += 3                                               # router, block scan, slot rows
    n += 2 if capacity else (4 if fused_dispatch else 1)  # dispatch
    n += (3 if fused_dispatch else 6) if mx else (3 if f32 else 2)   # forward FFN
    n += 1 + 1                                           # combine, combine backward
    n += 8 if mx else (5 if f32 else 6)                  # backward FFN
    n += 5 if tc_router_bwd else 4                       # router backward
    if recompute:                                        # the gate/up half again
        n += 5 if mx else (2 if f32 else 1)
    return n


FP8_OVER_BF16 = 2.0   # nominal dense tensor-core ratio (4.5 / 2.25 PFLOP/s)
# DRAM bytes (read + write) of the six grouped-GEMM launches of one step, from one ncu capture
# of the current kernels per workload (profiles/launches_bf16_e8.md,
# profiles/launches_mxfp8_e128.md); None for workloads without such a capture.
GEMM_TRAFFIC_BYTES = {"bf16_e8": 3.820e+09, "mxfp8_e128": 2.4088e+10}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _workload_desc(cfg, capacity, recompute=False):
    d = {"workload": f"{cfg.name}: T={cfg.T} d_model={cfg.d_model} E={cfg.E} top_k={cfg.top_k} "
                     f"d_ff={cfg.d_ff} {cfg.dtype}",
         "T": cfg.T, "d_model": cfg.d_model, "E": cfg.E, "top_k": cfg.top_k, "d_ff": cfg.d_ff,
         "routing": "skewed (logit bias std 2)" if cfg.bias_std else "near-uniform random",
         "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
         "weight_grad_dtype": "fp32"}
    if cfg.dtype == "mxfp8":
        d["operands"] = ("MXFP8 (E4M3 + E8M0 per 32 along K) for all six expert GEMMs; bf16 "
                         "activations; FP32 master weights quantised to four MXFP8 copies "
                         "every step (inside the timed step)")
    if recompute:
        d["recompute"] = "gate/up GEMM re-run in the backward (a | u | h not kept from the forward)"
    if capacity:
        d["layout"] = f"padded capacity C={capacity} (overflow dropped)"
    else:
        d["layout"] = "dropless, device-scheduled grouped GEMM"
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


# ------------------------------------------------------------- our arm
def run_ours(args, rank, world):
    from mixture_experts_layer_offsets_b200.layer import MoELayer, capacity_for

    cfg = inputs.CONFIGS[args.workload]
    if args.tokens:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@T{args.tokens}", T=args.tokens)
    if args.experts:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@E{args.experts}", E=args.experts)
    if args.dtype and args.dtype != cfg.dtype:
        cfg = inputs.shrink(cfg, name=f"{cfg.name}@{args.dtype}", dtype=args.dtype)
    mxfp8 = cfg.dtype == "mxfp8"
    dev = torch.device("cuda", torch.cuda.current_device())
    capacity = capacity_for(cfg.R, cfg.E, *cfg.padded_cf) if args.capacity_factor and cfg.padded_cf else None
    inp = inputs.make_inputs(cfg, device=dev, seed=mdist.rank_seed(0, rank))
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, dev,
                 dw_dtype="f32", capacity=capacity, recompute=args.recompute)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    x, wr, b, w1, w2, dout = (inp[k] for k in ("x", "w_router", "bias", "w1", "w2", "dout"))
    phases = ["quantize_w", "route", "dispatch", "ffn_fwd", "combine", "combine_bwd", "ffn_bwd",
              "route_bwd"]
    fdt = L.ffn_dtype

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        s, dt = L.shape, L.cdtype
        from mixture_experts_layer_offsets_b200 import capi
        mark(0)
        if mxfp8:
            L.quantize_weights(w1, w2)
        mark(1)
        capi.moe_route(s, dt, x, wr, b, L.logits, L.topk_idx, L.topk_gate, L.counts, L.offsets,
                       L.slot_row, L.ws)
        mark(2)
        if capacity:
            capi.moe_padded_dispatch(s, dt, capacity, x, L.topk_idx, L.slot_row, L.offsets,
                                     L.x_perm, L.pad_row, L.offsets_pad)
        else:
            if L.fused_dispatch:
                capi.moe_permute_mx(s, x, L.slot_row, L.offsets, L.perm_src, L.ws)
            else:
                capi.moe_permute(s, dt, x, L.slot_row, L.x_perm, L.perm_src)
        mark(3)
        capi.moe_grouped_ffn_fwd(s, fdt, L.rows, L.x_perm, L.ffn_offsets, w1, w2, L.act, L.y_perm,
                                 L.ws, mx=L.mx)
        mark(4)
        capi.moe_combine(s, dt, L.y_perm, L.row_map, L.topk_gate, L.out)
        mark(5)
        capi.moe_combine_bwd(s, dt, dout, L.y_perm, L.row_map, L.topk_gate, L.dy_perm, L.dgate)
        mark(6)
        bwd = capi.moe_grouped_ffn_bwd_recompute if args.recompute else capi.moe_grouped_ffn_bwd
        bwd(s, fdt, L.rows, L.dy_perm, L.x_perm, L.act, L.ffn_offsets, w1, w2, L.dx_perm, L.dw1,
            L.dw2, capi.MOE_F32, L.ws, mx=L.mx)
        mark(7)
        capi.moe_route_bwd(s, dt, x, wr, L.logits, L.topk_idx, L.dgate, L.dx_perm, L.row_map,
                           L.dx, L.dw_router, L.ws)
        mark(8)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if L.device_status() != 0:
        raise SystemExit("device status reported a timeout during warm-up")

    # The timed step is one CUDA-graph replay of the whole path (the library makes
    # no host synchronisation and no allocation, so the step captures as is).
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        graph.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    per_step = [a.elapsed_time(b) for a, b in evs]
    total_ms = mdist.max_over_ranks(sum(per_step), device=dev)
    ms_per_step = total_ms / args.steps

    # Phase breakdown: eager steps with CUDA events between the calls; a GPU-side
    # delay before each step lets the host enqueue the whole step first, so the
    # events see device time only.
    nph = min(args.steps, 10)
    pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(nph)]
    for i in range(nph):
        flush.zero_()
        torch.cuda._sleep(3_000_000)
        step(pevs[i])
    torch.cuda.synchronize()
    ph = {p: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in pevs) for i, p in enumerate(phases)}
    status = L.device_status()
    del graph

    # e2e: through the public API with host buffers, copies inside the timed region
    e2e = None if args.no_e2e else run_e2e(args, L, inp, dev, flush, capacity, world)

    if rank != 0:
        return None
    tokens_per_s = cfg.T * world / (ms_per_step / 1e3)
    pk, pk_kind = _peaks()
    gemm_ms = ph["ffn_fwd"] + ph["ffn_bwd"]
    rows = L.rows
    gemm_flop = 18.0 * cfg.R * cfg.d_model * cfg.d_ff   # algorithmic (dropless) FLOPs per step
    achieved = gemm_flop / (gemm_ms / 1e3) / 1e12
    if cfg.dtype == "bf16":
        peak, peak_kind = pk["bf16_tflops"], f"bf16_tflops burst, {pk_kind}"
    elif mxfp8:
        peak = pk["bf16_tflops"] * FP8_OVER_BF16
        peak_kind = (f"bf16_tflops burst ({pk_kind}) x {FP8_OVER_BF16} nominal fp8/bf16 ratio; "
                     "the ffn phases include the activation quantisations")
    else:
        peak, peak_kind = None, "fp32 CUDA-core path: no tensor-core peak"
    n_launch = launches_per_step(cfg, capacity, args.recompute, L.fused_dispatch)
    line = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic (seeded; random-init weights)",
        "config": _workload_desc(cfg, capacity, args.recompute),
        "roofline": {
            "bound": "tensor", "kernel": "grouped GEMM (tcgen05), all 6 launches of a step",
            "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4) if peak else None,
            "peak_kind": peak_kind,
            "traffic": (GEMM_TRAFFIC_BYTES.get(cfg.name) if not capacity else None),
            "traffic_unit": "DRAM bytes per step (6 launches), ncu dram__bytes_read.sum + dram__bytes_write.sum",
            "algorithmic_flop_per_step": gemm_flop, "gemm_ms_per_step": round(gemm_ms, 4),
            "rows_computed": rows,
        },
        "phases_ms": {k: round(v, 4) for k, v in ph.items()},
        "timing": "value: CUDA-graph replay of the step, CUDA events per step; phases_ms and "
                  "roofline: eager steps with events between calls (host kept ahead of the GPU)",
        "gpu_launches": n_launch * args.steps,
        "device_status": status,
        "e2e": e2e,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = (cpu_baseline(cfg, budget_s=args.cpu_seconds) if not mxfp8 else
                                {"value": None, "unit": "tokens/s", "kind": "oracle", "cores": None,
                                 "sample": "not run: the MXFP8 oracle quantises the full FP32 "
                                           "expert weights (2.4e9 values) on every call, which "
                                           "alone exceeds the CPU time budget"})
    return line


def run_e2e(args, L, inp, dev, flush, capacity, world):
    """Same metric through the public API with pinned host buffers: every step copies its
    inputs x and dout host->device and its outputs out and dx device->host, inside the
    timed region.  Steps are pipelined the way an input pipeline would run them: two layer
    instances take turns, and while one step computes on the compute stream, the next
    step's inputs come in on a copy stream and the previous step's outputs go out on
    another; events order every copy against the compute that produces or reuses its
    buffers.  Working set per step is several times L2, so no flush is needed."""
    from mixture_experts_layer_offsets_b200.layer import MoELayer
    L2 = MoELayer(L.T, L.d, L.E, L.k, L.f, L.dtype, dev, dw_dtype=L.dw_dtype, capacity=capacity,
                  recompute=L.recompute)
    layers = [L, L2]
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
        h2d.wait_event(ev_comp[k])            # step i-2 has finished reading buffer k
        with torch.cuda.stream(h2d):
            xin[k].copy_(hx, non_blocking=True)
            din[k].copy_(hd, non_blocking=True)
            ev_in[k].record(h2d)
        cs.wait_event(ev_in[k])
        cs.wait_event(ev_out[k])              # step i-2's outputs have left layer k
        layers[k].step(xin[k], wr, b, w1, w2, din[k])
        ev_comp[k].record(cs)
        d2h.wait_event(ev_comp[k])
        with torch.cuda.stream(d2h):
            hout[k].copy_(layers[k].out, non_blocking=True)
            hdx[k].copy_(layers[k].dx, non_blocking=True)
            ev_out[k].record(d2h)

    for i in range(max(2, args.warmup)):
        issue(i)
    torch.cuda.synchronize()
    n = max(2, args.steps)
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
            "h2d_bytes_per_step": 2 * nbytes, "d2h_bytes_per_step": 2 * nbytes,
            "ms_per_step": round(ms, 4), "steps": n, "device_status": status,
            "api": "MoELayer.step (C ABI) with pinned host buffers; copies of step i+1 in and "
                   "i-1 out overlap step i's compute (two layer instances, three streams)"}


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


def cpu_baseline(cfg, budget_s=12.0, chunk=64):
    """Float64 oracle fwd+bwd on micro-batches of `chunk` tokens of the workload's
    shapes until `budget_s` seconds of CPU work have run; tokens/s."""
    from oracle import moe_ref as ref
    g = torch.Generator().manual_seed(0)
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff
    wr = (torch.randn(E, d, generator=g) * cfg.router_std).to(cfg.act_dtype).double().numpy()
    w1 = (torch.randn(E, 2 * f, d, generator=g) * cfg.w_std).to(cfg.weight_dtype).double().numpy()
    w2 = (torch.randn(E, d, f, generator=g) * cfg.w_std).to(cfg.weight_dtype).double().numpy()
    bias = (torch.randn(E, generator=g) * cfg.bias_std).double().numpy() if cfg.bias_std else None
    done = 0
    t0 = time.perf_counter()
    while True:
        x = torch.randn(chunk, d, generator=g).to(cfg.act_dtype).double().numpy()
        dout = torch.randn(chunk, d, generator=g).to(cfg.act_dtype).double().numpy()
        ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, bias)
        done += chunk
        el = time.perf_counter() - t0
        if el >= budget_s or done >= T:
            break
    return {"value": round(done / el, 2), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{done} of {T} tokens of {cfg.name} in micro-batches of {chunk} "
                      f"(full expert weights; float64 NumPy), {el:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg = inputs.CONFIGS[args.workload]
    steps = []
    budget = max(2.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        cpu_baseline(cfg, budget_s=min(1.0, budget))
    for _ in range(args.steps):
        steps.append(cpu_baseline(cfg, budget_s=budget))
    v = statistics.mean(s["value"] for s in steps)
    cb = dict(steps[-1])
    cb["value"] = round(v, 2)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(cfg.T / v * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _workload_desc(cfg, None), "cpu_baseline": cb,
            "e2e": {"value": round(v, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="bf16_e8", choices=sorted(inputs.CONFIGS))
    ap.add_argument("--capacity-factor", action="store_true",
                    help="padded-capacity layout (workloads that define a capacity factor)")
    ap.add_argument("--recompute", action="store_true",
                    help="backward recomputes a | u | h (moe_grouped_ffn_bwd_recompute)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dtype", default=None, choices=["f32", "bf16", "mxfp8"],
                    help="run the workload's shapes at another compute dtype")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller cases for profiling); not a bench line")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiling); not a bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
        return
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
