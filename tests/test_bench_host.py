"""Host-side pieces of bench.py that need no GPU: its defaults, the command that
starts N ranks, the algorithmic work it divides by, and the data-parallel timing
path run as two gloo ranks on CPU with a stand-in step (each step ends with the
gradient all-reduce, the reported time is the slowest rank's, the line counts the
tokens of both ranks)."""

import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from mixture_experts_layer_offsets_b200 import dist as mdist
from mixture_experts_layer_offsets_b200 import inputs
from oracle import moe_ref as ref


def test_defaults_measure_the_largest_workload():
    a = bench.parse_args([])
    assert a.workload == "mxfp8_e128" and a.gpus == 1 and a.warmup >= 3
    cfgs = inputs.CONFIGS.values()
    big = max(cfgs, key=lambda c: bench.gemm_flop(c))
    assert big.name == a.workload
    assert bench.parse_args(["--warmup", "1"]).warmup == 3


def test_weight_copies_are_made_once_per_optimizer_step():
    # the config names when the MXFP8 weight copies are made, and an accumulation window
    # is described at one rank too; two layer instances of one shape share their copies
    from mixture_experts_layer_offsets_b200.layer import MoELayer
    cfg = inputs.CONFIGS["mxfp8_e128"]
    d = bench._workload_desc(cfg, None, accum=4, world=1)
    assert "once per optimizer step" in d["operands"] and "4 micro-batches" in d["step"]
    assert "all-reduce" not in d["step"]
    assert "all-reduce" in bench._workload_desc(cfg, None, accum=8, world=2)["step"]
    assert "step" not in bench._workload_desc(cfg, None)
    a = MoELayer(64, 128, 8, 2, 128, "mxfp8", "cpu")
    b = MoELayer(64, 128, 8, 2, 128, "mxfp8", "cpu")
    b.share_weight_copies(a)
    assert b.mx is a.mx and b.mxq["w1_q"] is a.mxq["w1_q"]
    with pytest.raises(ValueError):
        MoELayer(64, 128, 8, 2, 256, "mxfp8", "cpu").share_weight_copies(a)
    with pytest.raises(ValueError):
        MoELayer(64, 128, 8, 2, 128, "bf16", "cpu").share_weight_copies(a)


def test_cpu_baseline_samples_are_bounded_and_labelled():
    # the oracle's rate on a bounded sample: bf16 whole calls within the budget; MXFP8 per
    # sample the weight quantisation of whole experts (at least one), with the cost per
    # token measured once per process and reused
    small = inputs.shrink(inputs.CONFIGS["bf16_e8"], name="cb_bf16", T=64, d_model=128, E=4,
                          top_k=2, d_ff=128)
    cb = bench.cpu_baseline(small, budget_s=0.2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    mx = inputs.shrink(inputs.CONFIGS["mxfp8_e128"], name="cb_mx", T=64, d_model=128, E=8,
                       top_k=2, d_ff=128)
    bench._MX_TOKEN_COST.clear()
    a = bench.cpu_baseline(mx, budget_s=0.0)
    assert len(bench._MX_TOKEN_COST) == 1
    cost = dict(bench._MX_TOKEN_COST)
    b = bench.cpu_baseline(mx, budget_s=0.0)
    assert bench._MX_TOKEN_COST == cost          # measured once, reused
    for r in (a, b):
        assert r["extrapolated"] and r["value"] > 0 and "of 8 experts" in r["sample"]
        assert "1 of 8 experts" in r["sample"]    # a zero budget still times one expert


def test_launcher_starts_n_ranks_of_this_script_on_one_node():
    cmd = bench.launcher_argv(8, ["--gpus", "8", "--steps", "4"], 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=8" in cmd and "--nnodes=1" in cmd
    assert "--master-addr=127.0.0.1" in cmd and "--master-port=29555" in cmd
    assert cmd[-4:] == ["--gpus", "8", "--steps", "4"]
    assert os.path.samefile(cmd[-5], bench.__file__)


def test_algorithmic_work():
    c = inputs.CONFIGS
    assert bench.gemm_flop(c["bf16_e8"]) == 18 * 16384 * 4 * 2048 * 1024
    kb = bench.kernel_bytes(c["bf16_e8"])
    R, T, d = 65536, 16384, 2048
    assert kb["permute"] == T * d * 2 + R * d * 2 + T * 4 * 8
    mx = bench.kernel_bytes(c["mxfp8_e128"])
    assert "mx_weights" in mx and "mx_act" in mx
    # padded layout: the row count is E * C
    assert bench.kernel_bytes(c["bf16_skew_e128"], 1280)["combine"] > \
        bench.kernel_bytes(c["bf16_skew_e128"])["combine"]
    # the six expert GEMMs at bf16_e8, summed by hand from the operand and result sizes
    # (R = 65536, d = 2048, f = 1024, E = 8; fp32 weight gradients): 1174405120 forward
    # + 2583691264 backward
    assert bench.gemm_bytes(c["bf16_e8"]) == 3758096384
    # MXFP8 moves fewer operand bytes than the same shapes in bf16, and the captured
    # traffic of the default workload is reported with its algorithmic bytes
    big = c["mxfp8_e128"]
    assert bench.gemm_bytes(big) < bench.gemm_bytes(inputs.shrink(big, name="x", dtype="bf16"))
    rf = bench.roofline(big, {"gemm_ms": 9.0, "gemm_launches": 8})
    assert rf["algorithmic_bytes_per_step"] == round(bench.gemm_bytes(big))
    assert rf["traffic"] is None or 0.8 < rf["traffic"] / rf["algorithmic_bytes_per_step"] < 1.2


CFG = inputs.shrink(inputs.CONFIGS["tiny_f32"], name="gloo_bench", T=24, d_model=16, E=4,
                    top_k=2, d_ff=8, router_std=0.25)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = inputs.make_inputs(CFG, seed=0)
        mine = inputs.make_inputs(CFG, seed=mdist.rank_seed(0, rank))
        f64 = lambda t: t.double().numpy()  # noqa: E731
        grads = []

        def step():
            # stand-in for the layer step: the oracle's gradients of this rank's batch,
            # then the one all-reduce of the optimizer step; rank 1 is the slower one
            r = ref.layer_fwd_bwd(f64(mine["x"]), f64(w["w_router"]), f64(w["w1"]), f64(w["w2"]),
                                  f64(mine["dout"]), CFG.top_k)
            g = [torch.from_numpy(r[k].copy()) for k in ("dw1", "dw2", "dw_router")]
            mdist.allreduce_grads(g)
            grads[:] = g
            time.sleep(0.02 * (1 + 4 * rank))

        total, per, _ = bench.dp_timed(step, 3, 1, world, None, timer="cpu")
        line = bench.dp_line(CFG, total, 3, 1, 1, world)
        out[rank] = (total, sum(per), line, [g.numpy() for g in grads])
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_through_the_bench_timing_path():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    t0, own0, line, g0 = out[0]
    t1, own1, _, g1 = out[1]
    assert t0 == t1 == max(own0, own1) == own1          # the slowest rank's time
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["value"] == pytest.approx(2 * CFG.T / (t0 / 3 / 1e3), rel=1e-3)
    # the all-reduce inside the step: both ranks hold the gradient of the joint batch
    w = inputs.make_inputs(CFG, seed=0)
    shards = [inputs.make_inputs(CFG, seed=mdist.rank_seed(0, r)) for r in range(world)]
    x = np.concatenate([s["x"].double().numpy() for s in shards])
    dout = np.concatenate([s["dout"].double().numpy() for s in shards])
    full = ref.layer_fwd_bwd(x, w["w_router"].double().numpy(), w["w1"].double().numpy(),
                             w["w2"].double().numpy(), dout, CFG.top_k)
    for g in (g0, g1):
        for a, key in zip(g, ("dw1", "dw2", "dw_router")):
            np.testing.assert_allclose(a, full[key], rtol=1e-12, atol=1e-14, err_msg=key)
