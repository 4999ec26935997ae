"""Device buffers for one MoE FFN layer and the call sequence of its forward
and backward pass through the C ABI.

PyTorch only allocates device memory here; every step runs in the CUDA
library (``capi``).  Forward: moe_route -> moe_permute -> moe_grouped_ffn_fwd
-> moe_combine.  Backward: moe_combine_bwd -> moe_grouped_ffn_bwd ->
moe_route_bwd.  With ``capacity`` set, the padded-capacity comparison layout
is used instead (moe_padded_dispatch after the route, uniform E x capacity
rows in the grouped FFN, dropped pairs marked -1).

dtype "mxfp8": bf16 activations and router, FP32 master expert weights whose
MXFP8 copies (two orientations per weight, see ``moe_mx_weights``) are made
by moe_mx_quantize_weights at the start of a forward; the later micro-batches of an
optimizer step pass ``requantize=False`` and reuse them, so they are made once per
optimizer step.  The grouped FFN calls run with MOE_MXFP8 and write
FP32 weight gradients.  Unless it recomputes, the MXFP8 layer dispatches with
moe_permute_mx and runs the combine backward as moe_combine_bwd_mx: both write the
MXFP8 operand copies of x and dy straight into the workspace, and no bf16 x_perm or
dy_perm exists (those attributes are None).
"""

from __future__ import annotations

import torch

from . import capi

_DT = {"f32": capi.MOE_F32, "bf16": capi.MOE_BF16, "mxfp8": capi.MOE_MXFP8}


class MoELayer:
    def __init__(self, T: int, d_model: int, E: int, top_k: int, d_ff: int, dtype: str = "bf16",
                 device="cuda", dw_dtype: str | None = None, capacity: int | None = None,
                 renorm: bool = False, recompute: bool = False, act_scratch=None, ws=None,
                 fused_dispatch: bool | None = None):
        if dtype not in _DT:
            raise ValueError(f"dtype {dtype!r} is not supported by the layer path")
        self.T, self.d, self.E, self.k, self.f = T, d_model, E, top_k, d_ff
        self.dtype = dtype
        self.ffn_dtype = _DT[dtype]
        # routing, permute and combine of the MXFP8 layer run on bf16 activations
        self.cdtype = capi.MOE_BF16 if dtype == "mxfp8" else _DT[dtype]
        self.dw_dtype = dw_dtype or "f32"
        if dtype == "mxfp8" and self.dw_dtype != "f32":
            raise ValueError("the MXFP8 layer writes FP32 weight gradients")
        if dtype == "mxfp8" and capacity:
            raise ValueError("the padded layout is not offered with MXFP8")
        self.capacity = capacity
        self.renorm = renorm
        # recompute: the backward refills a | u | h (and the MXFP8 token-block copies)
        # from x_perm, so act_scratch and ws may be shared by several layers
        self.recompute = recompute
        # MXFP8: the dispatch writes the quantised copies of x directly (moe_permute_mx);
        # the recompute needs the bf16 x_perm, so it keeps the plain permute
        if fused_dispatch is None:
            fused_dispatch = dtype == "mxfp8" and not recompute
        if fused_dispatch and (dtype != "mxfp8" or recompute):
            raise ValueError("the fused dispatch is the MXFP8 layer's, without recompute")
        self.fused_dispatch = fused_dispatch
        # with it, the combine backward writes dy's MXFP8 copies directly
        # (moe_combine_bwd_mx) and no bf16 dy_perm
        self.shape = capi.shape_of(T, d_model, E, top_k, d_ff)
        self.R = T * top_k
        self.rows = E * capacity if capacity else self.R
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        wdt = torch.float32 if self.dw_dtype == "f32" else torch.bfloat16
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        act = dict(dtype=tdt, device=dev)
        rows = max(self.rows, 1)
        self.logits = torch.empty(T, E, **f32)
        self.topk_idx = torch.empty(T, top_k, **i32)
        self.topk_gate = torch.empty(T, top_k, **f32)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.slot_row = torch.empty(T, top_k, **i32)
        self.perm_src = torch.empty(max(self.R, 1), **i32)
        # (the fused MXFP8 dispatch writes no bf16 copy of the routed rows)
        self.x_perm = None if fused_dispatch else torch.empty(rows, d_model, **act)
        if act_scratch is not None:
            if not recompute:
                raise ValueError("a shared activation buffer needs recompute=True")
            if act_scratch.numel() < rows * 3 * d_ff or act_scratch.dtype != tdt:
                raise ValueError("act_scratch is too small or of the wrong type")
            self.act = act_scratch.view(-1)[:rows * 3 * d_ff].view(rows, 3 * d_ff)
        else:
            self.act = torch.empty(rows, 3 * d_ff, **act)
        self.y_perm = torch.empty(rows, d_model, **act)
        self.out = torch.empty(T, d_model, **act)
        self.dgate = torch.empty(T, top_k, **f32)
        self.dy_perm = None if fused_dispatch else torch.zeros(rows, d_model, **act)
        self.dx_perm = torch.empty(rows, d_model, **act)
        self.dw1 = torch.empty(E, 2 * d_ff, d_model, dtype=wdt, device=dev)
        self.dw2 = torch.empty(E, d_model, d_ff, dtype=wdt, device=dev)
        self.dx = torch.empty(T, d_model, **act)
        self.dw_router = torch.empty(E, d_model, **f32)
        self.stats = torch.zeros(8, **f32)
        if renorm:  # the combine's gates and their gradient under the renormalised rule
            self.gate_rn = torch.empty(T, top_k, **f32)
            self.dgate_rn = torch.empty(T, top_k, **f32)
        if capacity:
            self.pad_row = torch.empty(T, top_k, **i32)
            self.offsets_pad = torch.empty(E + 1, **i32)
        if dtype == "mxfp8":
            u8 = dict(dtype=torch.uint8, device=dev)
            self.mxq = dict(
                w1_q=torch.empty(E * 2 * d_ff, d_model, **u8),
                w1_s=torch.empty(E * 2 * d_ff * d_model // 32, **u8),
                w1t_q=torch.empty(E * 2 * d_ff, d_model, **u8),
                w1t_s=torch.empty(E * 2 * d_ff * d_model // 32, **u8),
                w2_q=torch.empty(E * d_model, d_ff, **u8),
                w2_s=torch.empty(E * d_model * d_ff // 32, **u8),
                w2t_q=torch.empty(E * d_model, d_ff, **u8),
                w2t_s=torch.empty(E * d_model * d_ff // 32, **u8),
            )
            self.mx = capi.moe_mx_weights(**{k: v.data_ptr() for k, v in self.mxq.items()})
        else:
            self.mx = None
        nbytes = capi.moe_workspace_size(self.shape, self.ffn_dtype, self.rows)
        if nbytes == 0:
            raise ValueError("invalid MoE shape")
        if ws is not None:
            if ws.numel() * ws.element_size() < nbytes:
                raise ValueError("the shared workspace is too small")
            self.ws = ws
        else:
            self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)

    # the row map and offsets that the grouped FFN and combine steps use
    @property
    def row_map(self):
        return self.pad_row if self.capacity else self.slot_row

    @property
    def combine_gate(self):
        return self.gate_rn if self.renorm else self.topk_gate

    @property
    def ffn_offsets(self):
        return self.offsets_pad if self.capacity else self.offsets

    def quantize_weights(self, w1, w2, stream=None):
        """MXFP8 copies of the FP32 master weights w1 [E, 2f, d], w2 [E, d, f]:
        blocks along each GEMM's contraction axis (d and 2f for W1, f and d for W2)."""
        capi.moe_mx_quantize_weights(self.shape, w1, w2, self.mx, stream)

    def share_weight_copies(self, other: "MoELayer") -> None:
        """Use ``other``'s MXFP8 weight copies (layers of one shape that run the same
        weights, e.g. instances that take turns over micro-batches): a quantisation by
        either serves both.  Both must run on one stream, or be ordered by the caller."""
        dims = lambda L: (L.T, L.d, L.E, L.k, L.f)
        if self.mx is None or other.mx is None or dims(self) != dims(other):
            raise ValueError("weight copies are shared between MXFP8 layers of one shape")
        self.mxq, self.mx = other.mxq, other.mx

    def forward(self, x, w_router, bias, w1, w2, stream=None, requantize: bool = True):
        """With ``requantize=False`` an MXFP8 layer reuses the weight copies of an earlier
        forward instead of quantising w1 and w2 again: valid while the master weights have
        not changed since, as within the micro-batches of one optimizer step."""
        s, dt = self.shape, self.cdtype
        if self.mx is not None and requantize:
            self.quantize_weights(w1, w2, stream)
        capi.moe_route(s, dt, x, w_router, bias, self.logits, self.topk_idx, self.topk_gate,
                       self.counts, self.offsets, self.slot_row, self.ws, stream)
        if self.capacity:
            capi.moe_padded_dispatch(s, dt, self.capacity, x, self.topk_idx, self.slot_row,
                                     self.offsets, self.x_perm, self.pad_row, self.offsets_pad,
                                     stream)
        elif self.fused_dispatch:
            capi.moe_permute_mx(s, x, self.slot_row, self.offsets, self.perm_src, self.ws, stream)
        else:
            capi.moe_permute(s, dt, x, self.slot_row, self.x_perm, self.perm_src, stream)
        xp = None if self.fused_dispatch else self.x_perm
        capi.moe_grouped_ffn_fwd(s, self.ffn_dtype, self.rows, xp, self.ffn_offsets, w1,
                                 w2, self.act, self.y_perm, self.ws, mx=self.mx, stream=stream)
        if self.renorm:
            capi.moe_renorm_gates(s, self.topk_gate, self.gate_rn, stream)
        capi.moe_combine(s, dt, self.y_perm, self.row_map, self.combine_gate, self.out, stream)
        return self.out

    def backward(self, dout, x, w_router, w1, w2, stream=None, accumulate: bool = False):
        """With ``accumulate`` the weight gradients are added to dw1, dw2 and dw_router
        (gradient accumulation over micro-batches) instead of overwriting them."""
        s, dt = self.shape, self.cdtype
        acc = capi.MOE_DW_ACCUMULATE if accumulate else 0
        dg = self.dgate_rn if self.renorm else self.dgate
        if self.fused_dispatch:
            capi.moe_combine_bwd_mx(s, dout, self.y_perm, self.row_map, self.combine_gate,
                                    self.perm_src, dg, self.ws, stream)
        else:
            capi.moe_combine_bwd(s, dt, dout, self.y_perm, self.row_map, self.combine_gate,
                                 self.dy_perm, dg, stream)
        if self.renorm:
            capi.moe_renorm_gates_bwd(s, self.topk_gate, self.dgate_rn, self.dgate, stream)
        bwd = capi.moe_grouped_ffn_bwd_recompute if self.recompute else capi.moe_grouped_ffn_bwd
        xp = None if self.fused_dispatch else self.x_perm
        bwd(s, self.ffn_dtype, self.rows, self.dy_perm, xp, self.act, self.ffn_offsets,
            w1, w2, self.dx_perm, self.dw1, self.dw2, _DT[self.dw_dtype] | acc, self.ws, mx=self.mx,
            stream=stream)
        capi.moe_route_bwd(s, dt | acc, x, w_router, self.logits, self.topk_idx, self.dgate,
                           self.dx_perm, self.row_map, self.dx, self.dw_router, self.ws, stream)
        return self.dx

    def step(self, x, w_router, bias, w1, w2, dout, stream=None, accumulate: bool = False,
             requantize: bool = True):
        self.forward(x, w_router, bias, w1, w2, stream, requantize)
        return self.backward(dout, x, w_router, w1, w2, stream, accumulate)

    def routing_stats(self, capacity: int | None = None, stream=None):
        """Load statistics of the last forward's routing, on the device (fp32 [8]):
        rows, mean, max/mean, min/mean, coefficient of variation, empty experts,
        and for a capacity (the layer's own by default) the dropped and used fractions."""
        cap = self.capacity if capacity is None else capacity
        capi.moe_routing_stats(self.shape, self.counts, cap or 0, self.stats, stream)
        return self.stats

    def device_status(self, stream=None) -> int:
        return capi.moe_get_device_status(self.ws, stream)
