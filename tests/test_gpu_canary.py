"""Out-of-bounds writes (a stand-in for a memory sanitizer, which is not available here):
every output buffer of one forward + backward step sits between two 64 KiB guard bands
filled with a canary byte; after the step every guard byte must be unchanged.  Shapes are
ragged (expert segments that are not multiples of the 128-row tile, empty experts) so that
the tile edges and the row-wise store fallbacks are exercised."""

import pytest
import torch

from mixture_experts_layer_offsets_b200 import capi
from mixture_experts_layer_offsets_b200.inputs import CONFIGS, make_inputs, shrink

pytestmark = pytest.mark.gpu

GUARD = 64 << 10
CANARY = 0xA5


class Guarded:
    """Tensors carved out of one byte buffer, each between guard bands."""

    def __init__(self):
        self.parts = []

    def alloc(self, shape, dtype):
        n = 1
        for s_ in shape:
            n *= s_
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD + ((nbytes + 255) // 256) * 256 + GUARD,), CANARY,
                         dtype=torch.uint8, device="cuda")
        t = raw[GUARD:GUARD + nbytes].view(dtype).view(*shape)
        self.parts.append((raw, nbytes))
        return t

    def check(self):
        for raw, nbytes in self.parts:
            head = raw[:GUARD]
            tail = raw[GUARD + nbytes:]
            assert bool((head == CANARY).all()) and bool((tail == CANARY).all())


CASES = {
    "bf16": shrink(CONFIGS["bf16_skew_e128"], name="c_bf16", T=700, d_model=256, E=32, top_k=2,
                   d_ff=256, router_std=1 / 16.0),
    "mxfp8": shrink(CONFIGS["mxfp8_e128"], name="c_mx", T=700, d_model=384, E=16, top_k=2,
                    d_ff=384, router_std=1 / 16.0, bias_std=2.0),
}


@pytest.mark.parametrize("name,fused", [("bf16", False), ("mxfp8", False), ("mxfp8", True)])
def test_no_write_outside_outputs(name, fused):
    """fused: the MXFP8 layer's own path (moe_permute_mx and moe_combine_bwd_mx write the
    quantised copies of x and dy into the workspace; no x_perm, no dy_perm)."""
    cfg = CASES[name]
    T, d, E, k, f = cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff
    R = T * k
    inp = {kk: (v.cuda() if v is not None else None) for kk, v in make_inputs(cfg).items()}
    g = Guarded()
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    shape = capi.shape_of(T, d, E, k, f)
    mx = None
    fdt = capi.MOE_MXFP8 if cfg.dtype == "mxfp8" else capi.MOE_BF16
    if cfg.dtype == "mxfp8":
        qs = {n: g.alloc((sz,), torch.uint8) for n, sz in (
            ("w1_q", E * 2 * f * d), ("w1_s", E * 2 * f * d // 32), ("w1t_q", E * 2 * f * d),
            ("w1t_s", E * 2 * f * d // 32), ("w2_q", E * d * f), ("w2_s", E * d * f // 32),
            ("w2t_q", E * d * f), ("w2t_s", E * d * f // 32))}
        mx = capi.moe_mx_weights(**{n: t.data_ptr() for n, t in qs.items()})
        capi.moe_mx_quantize_weights(shape, inp["w1"], inp["w2"], mx)
    o = dict(
        logits=g.alloc((T, E), f32), idx=g.alloc((T, k), i32), gate=g.alloc((T, k), f32),
        counts=g.alloc((E,), i32), offsets=g.alloc((E + 1,), i32), slot=g.alloc((T, k), i32),
        x_perm=g.alloc((R, d), bf), perm_src=g.alloc((R,), i32), act=g.alloc((R, 3 * f), bf),
        y=g.alloc((R, d), bf), out=g.alloc((T, d), bf), dy=g.alloc((R, d), bf),
        dgate=g.alloc((T, k), f32), dx_perm=g.alloc((R, d), bf), dw1=g.alloc((E, 2 * f, d), f32),
        dw2=g.alloc((E, d, f), f32), dx=g.alloc((T, d), bf), dwr=g.alloc((E, d), f32))
    nws = capi.moe_workspace_size(shape, fdt, R)
    ws = g.alloc((nws,), torch.uint8)
    ws.zero_()
    x, wr, b = inp["x"], inp["w_router"], inp["bias"]
    w1 = inp["w1"] if mx is None else None
    w2 = inp["w2"] if mx is None else None
    capi.moe_route(shape, capi.MOE_BF16, x, wr, b, o["logits"], o["idx"], o["gate"], o["counts"],
                   o["offsets"], o["slot"], ws)
    if fused:
        capi.moe_permute_mx(shape, x, o["slot"], o["offsets"], o["perm_src"], ws)
    else:
        capi.moe_permute(shape, capi.MOE_BF16, x, o["slot"], o["x_perm"], o["perm_src"])
    xp = None if fused else o["x_perm"]
    capi.moe_grouped_ffn_fwd(shape, fdt, R, xp, o["offsets"], w1, w2, o["act"], o["y"], ws,
                             mx=mx)
    capi.moe_combine(shape, capi.MOE_BF16, o["y"], o["slot"], o["gate"], o["out"])
    if fused:
        capi.moe_combine_bwd_mx(shape, inp["dout"], o["y"], o["slot"], o["gate"], o["perm_src"],
                                o["dgate"], ws)
    else:
        capi.moe_combine_bwd(shape, capi.MOE_BF16, inp["dout"], o["y"], o["slot"], o["gate"],
                             o["dy"], o["dgate"])
    capi.moe_grouped_ffn_bwd(shape, fdt, R, None if fused else o["dy"], xp, o["act"],
                             o["offsets"], w1, w2, o["dx_perm"], o["dw1"], o["dw2"], capi.MOE_F32,
                             ws, mx=mx)
    capi.moe_route_bwd(shape, capi.MOE_BF16, x, wr, o["logits"], o["idx"], o["dgate"],
                       o["dx_perm"], o["slot"], o["dx"], o["dwr"], ws)
    torch.cuda.synchronize()
    assert capi.moe_get_device_status(ws) == 0
    g.check()
    assert torch.isfinite(o["dw1"]).all() and torch.isfinite(o["dx"].float()).all()
