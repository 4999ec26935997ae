"""One rank of an expert-parallel MoE layer: buffers, the library's calls, and the
collectives between them.

kongchang, section 容量税 (capacity tax): the routed experts are spread over the ranks
and only the selected token rows are written into the target rank's buffer;
bytechap, "Cách thức hoạt động": each GPU holds a fraction of the experts.  Rank o owns
experts [o E_loc, (o + 1) E_loc).  Every step of the method runs in the CUDA library
(moe_route, moe_ep_layout, moe_ep_dispatch, the grouped FFN on the owner's rows,
moe_ep_combine, moe_ep_combine_bwd, moe_route_bwd); this module allocates buffers and
orders the ranks:

  phase 1  route (local), gather every rank's expert counts, layout, dispatch (rows
           written into the owners' receive buffers)
  -- ranks in step --
  phase 2  owner: grouped FFN forward on its received rows
  -- ranks in step --
  phase 3  source: combine (reads the owners' output rows), combine backward (writes
           the output-gradient rows into the owners' buffers)
  -- ranks in step --
  phase 4  owner: grouped FFN backward (input-gradient rows, its experts' weight
           gradients, which stay local)
  -- ranks in step --
  phase 5  source: gather of the input-gradient rows, router backward; the router is
           replicated, so its gradient is summed over the ranks.

"In step" is a collective on the compute stream (an all-reduce of one word): it orders
one rank's writes into peer memory before the other ranks' reads.  The receive buffers
must be mapped on every rank (symmetric memory); ``exchange`` provides the allocation,
the all-gather of the counts, the step barrier and the gradient all-reduce.
"""

from __future__ import annotations

import torch

from . import capi

_DT = {"f32": capi.MOE_F32, "bf16": capi.MOE_BF16}


class NcclExchange:
    """Collectives and peer-mapped buffers of a torch.distributed process group (NCCL):
    symmetric-memory buffers give every rank's device pointers on every rank."""

    def __init__(self, device, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.device = torch.device(device)
        self.group = group
        self.n = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self._flag = None
        self._handles = []

    def shared(self, shape, dtype):
        """A buffer of this rank and the device pointers of every rank's buffer."""
        from torch.distributed import _symmetric_memory as symm
        t = symm.empty(*shape, dtype=dtype, device=self.device)
        hdl = symm.rendezvous(t, self.group if self.group is not None else
                              self.dist.group.WORLD)
        self._handles.append(hdl)
        return t, list(hdl.buffer_ptrs)

    def all_gather_counts(self, counts, out):
        self.dist.all_gather_into_tensor(out.view(-1), counts, group=self.group)

    def step_barrier(self, device):
        if self._flag is None:
            self._flag = torch.zeros(1, dtype=torch.int32, device=device)
        self.dist.all_reduce(self._flag, group=self.group)

    def sum_(self, t):
        self.dist.all_reduce(t, group=self.group)


class EPLayer:
    """Buffers and calls of rank `rank` of `n_ranks` (see the module docstring).

    T tokens per rank, d_model, E experts in total, top_k, d_ff; dtype "bf16" or "f32".
    ``shared`` allocates the receive buffers: a callable (shape, dtype) -> (local tensor,
    list of every rank's device pointer) -- symmetric memory across processes, or, for
    several ranks emulated on one device, plain tensors shared between the instances."""

    def __init__(self, T, d_model, E, top_k, d_ff, dtype, device, n_ranks, rank, shared):
        if E % n_ranks:
            raise ValueError("E must be a multiple of the number of ranks")
        if dtype not in _DT:
            raise ValueError(f"dtype {dtype!r}: the expert-parallel layer takes bf16 or f32")
        self.T, self.d, self.E, self.k, self.f = T, d_model, E, top_k, d_ff
        self.n, self.rank = n_ranks, rank
        self.El = E // n_ranks
        self.dtype, self.cdt = dtype, _DT[dtype]
        self.cap = n_ranks * T * top_k          # rows an owner can receive
        dev = torch.device(device)
        adt = torch.float32 if dtype == "f32" else torch.bfloat16
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.shape = capi.shape_of(T, d_model, E, top_k, d_ff)
        # the owner's grouped FFN sees its E_loc experts and up to `cap` rows
        self.shape_loc = capi.shape_of(self.cap, d_model, self.El, 1, d_ff)
        self.logits = torch.empty(T, E, **f32)
        self.topk_idx = torch.empty(T, top_k, **i32)
        self.topk_gate = torch.empty(T, top_k, **f32)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.slot_row = torch.empty(T, top_k, **i32)
        self.counts_all = torch.empty(n_ranks, E, **i32)
        self.recv_offsets = torch.empty(self.El + 1, **i32)
        self.send_base = torch.empty(E, **i32)
        self.ep_row = torch.empty(T, top_k, **i32)
        # receive buffers, mapped on every rank
        self.x_recv, self.peer_x = shared((self.cap, d_model), adt)
        self.y_recv, self.peer_y = shared((self.cap, d_model), adt)
        self.dy_recv, self.peer_dy = shared((self.cap, d_model), adt)
        self.dx_recv, self.peer_dx = shared((self.cap, d_model), adt)
        self.act = torch.empty(self.cap, 3 * d_ff, dtype=adt, device=dev)
        self.out = torch.empty(T, d_model, dtype=adt, device=dev)
        self.dgate = torch.empty(T, top_k, **f32)
        self.dx_sum = torch.empty(T, d_model, dtype=adt, device=dev)
        self.dx = torch.empty(T, d_model, dtype=adt, device=dev)
        self.dw1 = torch.empty(self.El, 2 * d_ff, d_model, **f32)
        self.dw2 = torch.empty(self.El, d_model, d_ff, **f32)
        self.dw_router = torch.empty(E, d_model, **f32)
        nbytes = max(capi.moe_workspace_size(self.shape, self.cdt, 0),
                     capi.moe_workspace_size(self.shape_loc, self.cdt, self.cap))
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)

    # ---- phases (each rank runs phase p only after every rank finished phase p - 1)
    def route(self, x, w_router, bias):
        s, dt = self.shape, self.cdt
        capi.moe_route(s, dt, x, w_router, bias, self.logits, self.topk_idx, self.topk_gate,
                       self.counts, self.offsets, self.slot_row, self.ws)

    def dispatch(self, x):
        """After counts_all holds every rank's counts."""
        s, dt = self.shape, self.cdt
        capi.moe_ep_layout(s, self.n, self.rank, self.counts_all, self.recv_offsets,
                           self.send_base)
        capi.moe_ep_dispatch(s, dt, self.n, x, self.topk_idx, self.slot_row, self.offsets,
                             self.send_base, self.peer_x, self.ep_row)

    def expert_fwd(self, w1_local, w2_local):
        capi.moe_grouped_ffn_fwd(self.shape_loc, self.cdt, self.cap, self.x_recv,
                                 self.recv_offsets, w1_local, w2_local, self.act, self.y_recv,
                                 self.ws)

    def combine_and_grad(self, dout):
        s, dt = self.shape, self.cdt
        capi.moe_ep_combine(s, dt, self.n, self.peer_y, self.topk_idx, self.ep_row,
                            self.topk_gate, self.out)
        capi.moe_ep_combine_bwd(s, dt, self.n, dout, self.peer_y, self.topk_idx, self.ep_row,
                                self.topk_gate, self.peer_dy, self.dgate)

    def expert_bwd(self, w1_local, w2_local):
        capi.moe_grouped_ffn_bwd(self.shape_loc, self.cdt, self.cap, self.dy_recv, self.x_recv,
                                 self.act, self.recv_offsets, w1_local, w2_local, self.dx_recv,
                                 self.dw1, self.dw2, capi.MOE_F32, self.ws)

    def router_bwd(self, x, w_router):
        s, dt = self.shape, self.cdt
        capi.moe_ep_combine(s, dt, self.n, self.peer_dx, self.topk_idx, self.ep_row, None,
                            self.dx_sum)
        capi.moe_route_bwd(s, dt, x, w_router, self.logits, self.topk_idx, self.dgate,
                           self.dx_sum, None, self.dx, self.dw_router, self.ws)

    def step(self, exchange, x, w_router, bias, w1_local, w2_local, dout):
        """The whole forward + backward of this rank, with the collectives between the
        phases; returns dx.  dw_router is summed over the ranks."""
        dev = x.device
        self.route(x, w_router, bias)
        exchange.all_gather_counts(self.counts, self.counts_all)
        self.dispatch(x)
        exchange.step_barrier(dev)
        self.expert_fwd(w1_local, w2_local)
        exchange.step_barrier(dev)
        self.combine_and_grad(dout)
        exchange.step_barrier(dev)
        self.expert_bwd(w1_local, w2_local)
        exchange.step_barrier(dev)
        self.router_bwd(x, w_router)
        exchange.sum_(self.dw_router)
        return self.dx
