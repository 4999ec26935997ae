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

import numpy as np
import pytest
import torch

from mixture_experts_layer_offsets_b200 import capi, inputs

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
