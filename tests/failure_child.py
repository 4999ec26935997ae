"""Child process of the failure tests (run with the GEMM test hooks set in its
environment): one call in which CTA 0 of every tensor-core launch loses a pipeline stage,
so that its bounded wait runs out.  Modes: "bf16" / "mxfp8" (a grouped-FFN forward with a
workspace status word) and "route_noalloc" (the tensor-core router of moe_route_noalloc,
whose status word sits in the library's fixed array).  Prints one line of JSON."""

import json
import os
import sys
import time

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from mixture_experts_layer_offsets_b200 import capi  # noqa: E402


def _usable_after(dev) -> bool:
    """The context still works: a row permute with a valid map, checked by torch."""
    T, d, k = 600, 256, 2
    R = T * k
    shape = capi.shape_of(T, d, 8, k, 256)
    slot = torch.randperm(R, device=dev).to(torch.int32).view(T, k)
    x = torch.randn(T, d, device=dev).to(torch.bfloat16)
    xp = torch.empty(R, d, dtype=torch.bfloat16, device=dev)
    src = torch.empty(R, dtype=torch.int32, device=dev)
    capi.moe_permute(shape, capi.MOE_BF16, x, slot, xp, src)
    torch.cuda.synchronize()
    return bool(torch.equal(xp[slot.view(-1).long()], x.repeat_interleave(k, 0)))


def route_noalloc() -> None:
    torch.manual_seed(0)
    # 64 experts: the tensor-core tile router, whose pipeline waits are bounded (the
    # warp-level router of up to 32 experts has no waits)
    T, d, E, k = 600, 256, 64, 2
    dev = torch.device("cuda")
    shape = capi.shape_of(T, d, E, k, 256)
    x = torch.randn(T, d, device=dev).to(torch.bfloat16)
    w = (torch.randn(E, d, device=dev) * 0.05).to(torch.bfloat16)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    # indices start as a valid expert: the tile whose kernel gives up leaves them unwritten,
    # and the slot-row pass that follows reads them
    idx = torch.zeros(T, k, dtype=torch.int32, device=dev)
    gate = torch.empty(T, k, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    slot = torch.empty(T, k, dtype=torch.int32, device=dev)
    before = capi.moe_route_noalloc_status()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with capi.Profile(16) as prof:
        capi.moe_route_noalloc(shape, capi.MOE_BF16, x, w, None, logits, idx, gate, counts,
                               offsets, slot)
    torch.cuda.synchronize()
    names = [n for n, _ in prof.launches()]
    elapsed = time.perf_counter() - t0
    status = capi.moe_route_noalloc_status()
    cleared = capi.moe_route_noalloc_status()
    print(json.dumps({"before": before, "status": status, "cleared": cleared,
                      "elapsed_s": elapsed, "usable_after": _usable_after(dev),
                      "launches": names}))


def main(dtype: str) -> None:
    if dtype == "route_noalloc":
        return route_noalloc()
    torch.manual_seed(0)
    T, d, E, k, f = 600, 256, 8, 2, 256
    R = T * k
    dev = torch.device("cuda")
    shape = capi.shape_of(T, d, E, k, f)
    # routing metadata made on the host: 150 rows per expert (no GEMM feeds any index)
    offsets = torch.arange(0, R + 1, R // E, dtype=torch.int32, device=dev)
    x_perm = torch.randn(R, d, device=dev).to(torch.bfloat16)
    act = torch.empty(R, 3 * f, dtype=torch.bfloat16, device=dev)
    y = torch.empty(R, d, dtype=torch.bfloat16, device=dev)
    w1 = (torch.randn(E, 2 * f, d, device=dev) * 0.02)
    w2 = (torch.randn(E, d, f, device=dev) * 0.02)
    mx = None
    cdt = capi.MOE_MXFP8 if dtype == "mxfp8" else capi.MOE_BF16
    if dtype == "mxfp8":
        u8 = dict(dtype=torch.uint8, device=dev)
        bufs = [torch.empty(E * 2 * f * d, **u8) for _ in range(4)] + \
               [torch.empty(E * d * f, **u8) for _ in range(4)]
        mx = capi.moe_mx_weights(*[b.data_ptr() for b in (bufs[0], bufs[1], bufs[2], bufs[3],
                                                          bufs[4], bufs[5], bufs[6], bufs[7])])
        capi.moe_mx_quantize_weights(shape, w1, w2, mx)
        w1 = w2 = None
    else:
        w1, w2 = w1.to(torch.bfloat16), w2.to(torch.bfloat16)
    ws = torch.zeros(capi.moe_workspace_size(shape, cdt, R), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    capi.moe_grouped_ffn_fwd(shape, cdt, R, x_perm, offsets, w1, w2, act, y, ws, mx=mx)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    status = capi.moe_get_device_status(ws)
    ok_after = _usable_after(dev)
    print(json.dumps({"status": status, "elapsed_s": elapsed, "usable_after": ok_after}))


if __name__ == "__main__":
    main(sys.argv[1])
