"""GPU parity of the routing step for a few experts (bf16, E <= 32, d % 128 == 0), the
warp-level tensor-core router whose last block also scans the per-block expert counts.

kongchang, section 路由不只是模型问题，更是系统问题: routing metadata is made on the
device.  Against the oracle: top-k, counts, offsets and slot rows bit for bit (the oracle
taking its discrete steps on the device's own fp32 logits), logits and gates within the
bf16 tolerance of the float64 values.  Token counts that leave a ragged last block of 32,
expert counts that are not multiples of 8, a bias, one token, and calls repeated on one
workspace (the block counter that finds the last block must be back at zero after each
call)."""

import numpy as np
import pytest
import torch

from gpu_helpers import f64, i64, rel
from mixture_experts_layer_offsets_b200 import capi, inputs
from oracle import moe_ref as ref

pytestmark = pytest.mark.gpu

BASE = inputs.CONFIGS["bf16_e8"]
CASES = {
    "e8_ragged": dict(T=1000, d_model=256, E=8, top_k=4),
    "e1": dict(T=77, d_model=128, E=1, top_k=1),
    "e5_k2_bias": dict(T=333, d_model=384, E=5, top_k=2, bias_std=1.0, router_std=384 ** -0.5),
    "e13_k3": dict(T=513, d_model=640, E=13, top_k=3, router_std=640 ** -0.5),
    "e16": dict(T=64, d_model=2048, E=16, top_k=4),
    "e32_k8": dict(T=2049, d_model=512, E=32, top_k=8, router_std=512 ** -0.5),
    "one_token": dict(T=1, d_model=128, E=8, top_k=2),
    # more 16-token groups than 8 per SM: CTAs loop over several token tiles
    "e8_many_tiles": dict(T=20000, d_model=256, E=8, top_k=2),
}


def _route(cfg, inp, ws=None):
    shape = capi.shape_of(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff)
    dev = "cuda"
    b = dict(
        logits=torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev),
        idx=torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev),
        gate=torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=dev),
        counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
        offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
        slot_row=torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev),
    )
    if ws is None:
        ws = torch.zeros(capi.moe_workspace_size(shape, capi.MOE_BF16, 0), dtype=torch.uint8,
                         device=dev)
    with capi.Profile(16) as prof:
        capi.moe_route(shape, capi.MOE_BF16, inp["x"], inp["w_router"], inp["bias"], b["logits"],
                       b["idx"], b["gate"], b["counts"], b["offsets"], b["slot_row"], ws)
    names = [n for n, _ in prof.launches()]
    assert capi.moe_get_device_status(ws) == capi.MOE_OK
    return b, ws, names


def _check(cfg, cpu, b):
    bias = f64(cpu["bias"]) if cpu["bias"] is not None else None
    o = ref.route(f64(cpu["x"]), f64(cpu["w_router"]), cfg.top_k, bias,
                  select_logits=f64(b["logits"]))
    for key in ("idx", "counts", "offsets", "slot_row"):
        assert np.array_equal(i64(b[key]), o[key]), key
    assert rel(f64(b["logits"]), o["logits"]) <= 1e-2
    assert rel(f64(b["gate"]), o["gate"]) <= 1e-2


@pytest.mark.parametrize("name", list(CASES))
def test_warp_router_matches_oracle(name):
    cfg = inputs.shrink(BASE, name=name, d_ff=128, **CASES[name])
    cpu = inputs.make_inputs(cfg, device="cpu", seed=11)
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    b, ws, names = _route(cfg, dev)
    assert names == ["router_mma", "route_slot_rows"], names   # this path, and no scan launch
    _check(cfg, cpu, b)
    # the same workspace again, then another batch: the block counter was reset
    b2, _, _ = _route(cfg, dev, ws)
    for key in b:
        assert torch.equal(b[key], b2[key]), key
    cpu3 = inputs.make_inputs(cfg, device="cpu", seed=12)
    dev3 = {k: (v.cuda() if v is not None else None) for k, v in cpu3.items()}
    b3, _, _ = _route(cfg, dev3, ws)
    _check(cfg, cpu3, b3)


def test_router_paths_agree_on_their_own_logits():
    """E = 64 takes the tensor-core tile router, E = 32 the warp router: both route their
    own logits by the same rule (covered above), and both give near-uniform counts."""
    for E in (32, 64):
        cfg = inputs.shrink(BASE, name=f"e{E}", T=4096, d_model=256, E=E, top_k=4, d_ff=128)
        cpu = inputs.make_inputs(cfg, device="cpu", seed=1)
        dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
        b, _, names = _route(cfg, dev)
        assert names[0] == ("router_mma" if E <= 32 else "router_gemm")
        _check(cfg, cpu, b)


def test_tile_router_on_the_same_shapes(monkeypatch):
    """The tensor-core tile router (forced) on shapes the warp router takes by default:
    its own logits routed by the same rule."""
    monkeypatch.setenv("MOE_B200_ROUTER", "tile")
    cfg = inputs.shrink(BASE, name="tile_e8", T=1000, d_model=256, E=8, top_k=4, d_ff=128)
    cpu = inputs.make_inputs(cfg, device="cpu", seed=4)
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    b, _, names = _route(cfg, dev)
    assert names[0] == "router_gemm", names
    _check(cfg, cpu, b)

