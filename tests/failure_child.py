"""Child process of test_gpu_failure.py (run with the GEMM test hooks set in its
environment): one grouped-FFN forward in which CTA 0 of every GEMM launch loses a pipeline
stage, so that its bounded wait runs out.  Prints one line of JSON."""

import json
import os
import sys
import time

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from mixture_experts_layer_offsets_b200 import capi  # noqa: E402


def main(dtype: str) -> None:
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
    # the context is still usable: a row permute with a valid map, then a torch op
    slot = torch.randperm(R, device=dev).to(torch.int32).view(T, k)
    x = torch.randn(T, d, device=dev).to(torch.bfloat16)
    xp = torch.empty(R, d, dtype=torch.bfloat16, device=dev)
    src = torch.empty(R, dtype=torch.int32, device=dev)
    capi.moe_permute(shape, capi.MOE_BF16, x, slot, xp, src)
    torch.cuda.synchronize()
    ok_after = bool(torch.equal(xp[slot.view(-1).long()], x.repeat_interleave(k, 0)))
    print(json.dumps({"status": status, "elapsed_s": elapsed, "usable_after": ok_after}))


if __name__ == "__main__":
    main(sys.argv[1])
