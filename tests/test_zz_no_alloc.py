"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers have no way to allocate device memory: a plugin inside a host
framework that owns every byte of device memory and gives plugins no
allocation hook, code on a latency-critical path where cudaMalloc could
synchronise the device, or a deployment whose footprint is fixed at start-up.
For them the library offers moe_route_noalloc, which keeps its scratch in a
fixed array inside the library instead of a caller workspace.

This file is collected last on purpose (a run that stops at the first failure
has run every other test first).  It must pass both on its own in a fresh
process and after the rest of the suite.
"""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from mixture_experts_layer_offsets_b200 import capi, inputs
from oracle import moe_ref as ref

HERE = os.path.dirname(os.path.abspath(__file__))

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}


def _buffers(cfg):
    dev = "cuda"
    return dict(
        logits=torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev),
        topk_idx=torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev),
        topk_gate=torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=dev),
        counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
        offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
        slot_row=torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev),
    )


def _dtype(cfg):
    return capi.MOE_F32 if cfg.dtype == "f32" else capi.MOE_BF16


def _with_workspace(cfg, inp):
    shape = capi.shape_of(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff)
    b = _buffers(cfg)
    ws = torch.zeros(capi.moe_workspace_size(shape, _dtype(cfg), 0), dtype=torch.uint8,
                     device="cuda")
    capi.moe_route(shape, _dtype(cfg), inp["x"], inp["w_router"], inp["bias"], b["logits"],
                   b["topk_idx"], b["topk_gate"], b["counts"], b["offsets"], b["slot_row"], ws)
    return b


def _no_alloc(cfg, inp):
    shape = capi.shape_of(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff)
    b = _buffers(cfg)
    capi.moe_route_noalloc(shape, _dtype(cfg), inp["x"], inp["w_router"], inp["bias"],
                           b["logits"], b["topk_idx"], b["topk_gate"], b["counts"], b["offsets"],
                           b["slot_row"])
    return b


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / max(b.norm().item(), 1e-300))


def test_no_alloc_route_matches_workspace_route_on_two_calls_in_a_row():
    # two different problems back to back: the second call finds the first
    # call's leftovers in the shared scratch array
    first = inputs.shrink(inputs.CONFIGS["bf16_skew_e128"], name="first", T=3000, d_model=512,
                          E=64, top_k=4, d_ff=256, router_std=512 ** -0.5)
    second = inputs.shrink(inputs.CONFIGS["tiny_f32"], name="second", T=777)
    cases = []
    for cfg, seed in ((first, 1), (second, 2)):
        inp = inputs.make_inputs(cfg, device="cuda", seed=seed)
        cases.append((cfg, inp, _no_alloc(cfg, inp)))   # the two calls, in a row
    for cfg, inp, got in cases:
        want = _with_workspace(cfg, inp)
        torch.cuda.synchronize()
        for key in ("topk_idx", "counts", "offsets", "slot_row"):
            assert torch.equal(got[key], want[key]), (cfg.name, key)
        for key in ("logits", "topk_gate"):
            assert _rel(got[key], want[key]) <= TOL[cfg.dtype], (cfg.name, key)
        assert int(got["offsets"][-1]) == cfg.T * cfg.top_k


def test_no_alloc_route_rejects_shapes_beyond_its_scratch():
    big = capi.shape_of(1 << 18, 256, 1024, 8, 256)  # needs far more than the fixed array
    lib = capi.lib()
    status = lib.moe_route_noalloc(big, capi.MOE_BF16, 1 << 20, 1 << 20, None, 1 << 20, 1 << 20,
                                   1 << 20, 1 << 20, 1 << 20, 1 << 20, None)
    assert status == capi.MOE_ERR_UNSUPPORTED


def test_no_alloc_route_reproduces_the_hand_derived_golden_routing():
    """tests/golden/routing_tiny.json gives logits, with ties, and the routing derived
    from them by hand.  x holds each token's logits in its first E columns and the
    router weight is the identity there, so the device logits are exactly the fixture's
    (small integers are exact in bf16 and in fp32 sums)."""
    fx = json.load(open(os.path.join(HERE, "golden", "routing_tiny.json")))
    lg = np.array(fx["logits"], dtype=np.float64)
    T, E = lg.shape
    k, d = fx["top_k"], 64
    x = torch.zeros(T, d, dtype=torch.bfloat16)
    x[:, :E] = torch.tensor(lg, dtype=torch.bfloat16)
    w = torch.zeros(E, d, dtype=torch.bfloat16)
    w[:, :E] = torch.eye(E, dtype=torch.bfloat16)
    cfg = inputs.shrink(inputs.CONFIGS["bf16_e8"], name="golden", T=T, d_model=d, E=E, top_k=k,
                        d_ff=64)
    got = _no_alloc(cfg, {"x": x.cuda(), "w_router": w.cuda(), "bias": None})
    torch.cuda.synchronize()
    assert capi.moe_route_noalloc_status() == capi.MOE_OK
    assert np.array_equal(got["logits"].cpu().numpy(), lg)
    for key in ("idx", "counts", "offsets", "slot_row"):
        dev = got["topk_idx" if key == "idx" else key].cpu().numpy()
        assert np.array_equal(dev, np.array(fx[key])), key
    np.testing.assert_allclose(got["topk_gate"].cpu().numpy(), np.array(fx["gate"]), rtol=1e-6)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_no_alloc_route_matches_the_oracle(dtype):
    """Ragged token blocks, 64 experts: the discrete routing taken by the oracle on the
    device's own fp32 logits is reproduced bit for bit; logits and gates are within the
    dtype's tolerance of the oracle's float64 values."""
    cfg = inputs.shrink(inputs.CONFIGS["bf16_skew_e128"], name="noalloc_oracle", T=1500,
                        d_model=256, E=64, top_k=4, d_ff=256, router_std=256 ** -0.5,
                        dtype=dtype)
    cpu = inputs.make_inputs(cfg, device="cpu", seed=3)
    got = _no_alloc(cfg, {k: (v.cuda() if v is not None else None) for k, v in cpu.items()})
    torch.cuda.synchronize()
    assert capi.moe_route_noalloc_status() == capi.MOE_OK

    def f64(t):
        return t.to(torch.float64).cpu().numpy()

    o = ref.route(f64(cpu["x"]), f64(cpu["w_router"]), cfg.top_k, f64(cpu["bias"]),
                  select_logits=f64(got["logits"]))
    for key, dev in (("idx", "topk_idx"), ("counts", "counts"), ("offsets", "offsets"),
                     ("slot_row", "slot_row")):
        assert np.array_equal(got[dev].cpu().numpy().astype(np.int64), o[key]), key
    for key, dev in (("logits", "logits"), ("gate", "topk_gate")):
        assert _rel(got[dev].cpu(), torch.from_numpy(o[key])) <= TOL[dtype], key


@pytest.mark.timeout(120)
def test_no_alloc_route_reports_a_timeout_in_its_status_word():
    """A child process sets the library's test hooks (20 ms wait limit, CTA 0 of the
    tensor-core tile router, used for 64 experts, skips its second pipeline stage): the
    router gives up its wait,
    the status word of the fixed array reads MOE_ERR_TIMEOUT, a second read finds it
    cleared, and the context still works.  Nothing traps, faults or hangs."""
    env = dict(os.environ, MOE_B200_WAIT_NS="20000000", MOE_B200_TEST_DROP_STAGE="2")
    out = subprocess.run([sys.executable, os.path.join(HERE, "failure_child.py"), "route_noalloc"],
                         env=env, capture_output=True, text=True, timeout=100)
    assert out.returncode == 0, out.stderr[-2000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    assert res["before"] == capi.MOE_OK
    assert res["launches"][0] == "router_gemm", res["launches"]
    assert res["status"] == capi.MOE_ERR_TIMEOUT
    assert res["cleared"] == capi.MOE_OK
    assert res["usable_after"]
    assert res["elapsed_s"] < 10.0
