"""Helpers shared by the GPU parity tests (run the CUDA path; compare to the oracle)."""

from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_offsets_b200 import inputs
from mixture_experts_layer_offsets_b200.layer import MoELayer
from oracle import moe_ref as ref

# Tolerances on relative Frobenius error, by compute dtype.
TOL = {"f32": 1e-5, "bf16": 1e-2, "mxfp8": 5e-2}


def f64(t) -> np.ndarray:
    if t is None:
        return None
    return t.detach().to(torch.float64).cpu().numpy()


def i64(t) -> np.ndarray:
    return t.detach().to(torch.int64).cpu().numpy()


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def run_layer(cfg, seed=0, capacity=None, dw_dtype="f32", renorm=False, **kw):
    """Seeded inputs drawn on the CPU, copied to the GPU, one fwd+bwd step."""
    cpu = inputs.make_inputs(cfg, device="cpu", seed=seed)
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                 dw_dtype=dw_dtype, capacity=capacity, renorm=renorm, **kw)
    L.step(dev["x"], dev["w_router"], dev["bias"], dev["w1"], dev["w2"], dev["dout"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return cpu, L


def oracle_for(cpu, L, capacity=None):
    """Oracle pass on the same inputs; discrete routing taken on the device's logits."""
    args = (f64(cpu["x"]), f64(cpu["w_router"]), f64(cpu["w1"]), f64(cpu["w2"]), f64(cpu["dout"]),
            L.k)
    bias = f64(cpu["bias"]) if cpu["bias"] is not None else None
    if capacity:
        return ref.padded_layer_fwd_bwd(*args, capacity, bias, select_logits=f64(L.logits),
                                        renorm=L.renorm)
    return ref.layer_fwd_bwd(*args, bias, select_logits=f64(L.logits), renorm=L.renorm)


def check_recompute_bit_exact(cfg):
    """Two layers share one activation buffer and one workspace; layer A's backward
    runs after layer B's forward has overwritten both, recomputing what it needs.  Its
    results equal, bit for bit, those of a layer that kept its own activations."""
    _, L0 = run_layer(cfg, seed=0)
    dev = lambda d: {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    a_in = dev(inputs.make_inputs(cfg, device="cpu", seed=0))
    b_in = dev(inputs.make_inputs(cfg, device="cpu", seed=1))
    tdt = L0.act.dtype
    act = torch.empty(L0.act.numel(), dtype=tdt, device="cuda")
    ws = torch.zeros_like(L0.ws)
    mk = lambda: MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                          recompute=True, act_scratch=act, ws=ws)
    A, B = mk(), mk()
    A.forward(a_in["x"], a_in["w_router"], a_in["bias"], a_in["w1"], a_in["w2"])
    a_act = act.clone()
    B.forward(b_in["x"], b_in["w_router"], b_in["bias"], b_in["w1"], b_in["w2"])
    torch.cuda.synchronize()
    assert cfg.T == 0 or not torch.equal(act, a_act), "layer B did not overwrite the shared buffer"
    A.backward(a_in["dout"], a_in["x"], a_in["w_router"], a_in["w1"], a_in["w2"])
    torch.cuda.synchronize()
    assert A.device_status() == 0
    assert torch.equal(act, a_act), "the recompute did not restore a | u | h"
    for key in ("out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
        assert torch.equal(getattr(A, key), getattr(L0, key)), key


def check_accumulate(cfg, dw_dtype="f32"):
    """A layer that steps on batch A, then on batch B with MOE_DW_ACCUMULATE, holds the sum of
    the weight gradients of two layers that each stepped on one batch.  fp32 weight gradients
    get one fp32 addition per element, so the sum is exact against torch's fp32 addition
    (subnormal results aside); bf16 ones are rounded once, within the bf16 tolerance."""
    _, A = run_layer(cfg, seed=0, dw_dtype=dw_dtype)
    _, B = run_layer(cfg, seed=1, dw_dtype=dw_dtype)
    dev = lambda d: {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    a_in = dev(inputs.make_inputs(cfg, device="cpu", seed=0))
    b_in = dev(inputs.make_inputs(cfg, device="cpu", seed=1))
    C = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda", dw_dtype=dw_dtype)
    args = lambda i: (i["x"], i["w_router"], i["bias"], i["w1"], i["w2"], i["dout"])
    C.step(*args(a_in))
    C.step(*args(b_in), accumulate=True)
    torch.cuda.synchronize()
    assert C.device_status() == 0
    keys = ("dw1", "dw2", "dw_router")
    for key in keys:
        got, a, b = getattr(C, key), getattr(A, key), getattr(B, key)
        if got.dtype == torch.float32:
            want = a + b
            diff = got != want
            # only a subnormal sum may differ (flushed to zero by the reducing store)
            assert not diff.any() or bool((want[diff].abs() < 1.2e-38).all()), key
        else:
            want = a.double() + b.double()
            assert rel(f64(got), want.cpu().numpy()) <= TOL["bf16"], key
    # the step that accumulated still computed its own non-gradient outputs normally
    assert torch.equal(C.out, B.out) and torch.equal(C.dx, B.dx)
