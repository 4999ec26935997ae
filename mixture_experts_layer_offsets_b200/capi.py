"""Thin ctypes binding of ``include/moe.h`` (argument marshalling only).

Every function here has the name of its C entry point and forwards torch
tensors as raw device pointers plus the current CUDA stream.  No step of the
method runs in Python; if the CUDA library is missing the import of a
function fails loudly (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(5)
MOE_F32, MOE_BF16, MOE_MXFP8 = 0, 1, 2
MOE_DW_ACCUMULATE = 0x100   # OR into dw_dtype / the router backward's dtype: dW += ...
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_CUDA", 4: "MOE_ERR_TIMEOUT"}


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("E", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32)]


class moe_mx_weights(ctypes.Structure):
    """MXFP8 copies of the expert weights (device pointers), see include/moe.h."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w1_q", "w1_s", "w1t_q", "w1t_s", "w2_q", "w2_s", "w2t_q", "w2t_s")]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_SIGS = {
    "moe_version": (ctypes.c_char_p, []),
    "moe_workspace_size": (_SZ, [moe_shape, _I, _I64]),
    "moe_get_device_status": (_I, [_P, _P, _P]),
    "moe_route": (_I, [moe_shape, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_route_noalloc": (_I, [moe_shape, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_noalloc_status": (_I, [_P, _P]),
    "moe_mx_workspace_layout": (_I, [moe_shape, _I64, _P, _I]),
    "moe_profile_begin": (_I, [_P, _P, _I]),
    "moe_capacity": (ctypes.c_int32, [moe_shape, ctypes.c_int32, ctypes.c_int32]),
    "moe_ep_layout": (_I, [moe_shape, _I, _I, _P, _P, _P, _P]),
    "moe_ep_dispatch": (_I, [moe_shape, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_ep_combine": (_I, [moe_shape, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_ep_combine_bwd": (_I, [moe_shape, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_profile_end": (_I, [_P]),
    "moe_permute": (_I, [moe_shape, _I, _P, _P, _P, _P, _P]),
    "moe_grouped_ffn_fwd": (_I, [moe_shape, _I, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_combine": (_I, [moe_shape, _I, _P, _P, _P, _P, _P]),
    "moe_combine_bwd": (_I, [moe_shape, _I, _P, _P, _P, _P, _P, _P, _P]),
    "moe_grouped_ffn_bwd": (_I, [moe_shape, _I, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                 _I, _P, _SZ, _P]),
    "moe_grouped_ffn_bwd_recompute": (_I, [moe_shape, _I, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                 _I, _P, _SZ, _P]),
    "moe_route_bwd": (_I, [moe_shape, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "mxfp8_quantize": (_I, [_I64, _I64, _I, _P, _I, _P, _I, _P, _P, _P]),
    "moe_mx_quantize_weights": (_I, [moe_shape, _P, _P, _P, _P]),
    "moe_padded_dispatch": (_I, [moe_shape, _I, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_routing_stats": (_I, [moe_shape, _P, ctypes.c_int32, _P, _P]),
    "moe_permute_mx": (_I, [moe_shape, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine_bwd_mx": (_I, [moe_shape, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_renorm_gates": (_I, [moe_shape, _P, _P, _P]),
    "moe_renorm_gates_bwd": (_I, [moe_shape, _P, _P, _P, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_layer_offsets_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def header_symbols() -> list[str]:
    """Entry points declared in include/moe.h."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:moe_status|size_t|int32_t|const char\*)\s+(\w+)\s*\(",
                                 txt, re.M)))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, ctypes.Structure):     # host struct passed by address
        return ctypes.addressof(t)
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(name: str, status: int) -> None:
    if status != MOE_OK:
        raise MoEError(name, status)


def shape_of(T: int, d_model: int, E: int, top_k: int, d_ff: int) -> moe_shape:
    return moe_shape(T, d_model, E, top_k, d_ff)


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_workspace_size(shape: moe_shape, dtype: int, rows: int = 0) -> int:
    return lib().moe_workspace_size(shape, dtype, rows)


def moe_get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("moe_get_device_status",
           lib().moe_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(out)))
    return out.value


class Profile:
    """Per-launch device times of the library's kernels (moe_profile_begin /
    moe_profile_end): ``with Profile() as p: <calls>`` then ``p.launches()`` gives
    (kernel name, milliseconds) per launch, in launch order."""

    def __init__(self, capacity: int = 256):
        import torch
        self.cap = capacity
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.ev:          # CUDA events are created on their first record
            e.record()
        self._events = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.ev])
        self._names = (ctypes.c_char_p * capacity)()
        self.count = 0

    def __enter__(self):
        _check("moe_profile_begin", lib().moe_profile_begin(self._events, self._names, self.cap))
        return self

    def __exit__(self, *exc):
        n = ctypes.c_int32(0)
        _check("moe_profile_end", lib().moe_profile_end(ctypes.byref(n)))
        self.count = n.value
        return False

    def launches(self) -> list[tuple[str, float]]:
        import torch
        torch.cuda.synchronize()
        n = min(self.count, self.cap)
        return [(self._names[i].decode(), self.ev[2 * i].elapsed_time(self.ev[2 * i + 1]))
                for i in range(n)]


def moe_route(shape, dtype, x, w_router, bias, logits, topk_idx, topk_gate, counts, offsets,
              slot_row, ws, stream=None) -> None:
    _check("moe_route", lib().moe_route(
        shape, dtype, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits), _ptr(topk_idx),
        _ptr(topk_gate), _ptr(counts), _ptr(offsets), _ptr(slot_row), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_route_noalloc(shape, dtype, x, w_router, bias, logits, topk_idx, topk_gate, counts,
                      offsets, slot_row, stream=None) -> None:
    """moe_route without a workspace: for callers that cannot allocate device
    memory; its scratch is a fixed array inside the library (see include/moe.h)."""
    _check("moe_route_noalloc", lib().moe_route_noalloc(
        shape, dtype, _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits), _ptr(topk_idx),
        _ptr(topk_gate), _ptr(counts), _ptr(offsets), _ptr(slot_row), _stream(stream)))


def moe_route_noalloc_status(stream=None) -> int:
    """Read and clear the status word of moe_route_noalloc's fixed array (synchronises)."""
    out = ctypes.c_int32(0)
    _check("moe_route_noalloc_status",
           lib().moe_route_noalloc_status(_stream(stream), ctypes.byref(out)))
    return out.value


def moe_permute(shape, dtype, x, slot_row, x_perm, perm_src, stream=None) -> None:
    _check("moe_permute", lib().moe_permute(shape, dtype, _ptr(x), _ptr(slot_row), _ptr(x_perm),
                                            _ptr(perm_src), _stream(stream)))


def moe_grouped_ffn_fwd(shape, dtype, rows, x_perm, offsets, w1, w2, act_saved, y_perm, ws,
                        mx=None, stream=None) -> None:
    _check("moe_grouped_ffn_fwd", lib().moe_grouped_ffn_fwd(
        shape, dtype, rows, _ptr(x_perm), _ptr(offsets), _ptr(w1), _ptr(w2), _ptr(mx),
        _ptr(act_saved), _ptr(y_perm), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_combine(shape, dtype, y_perm, slot_row, topk_gate, out, stream=None) -> None:
    _check("moe_combine", lib().moe_combine(shape, dtype, _ptr(y_perm), _ptr(slot_row),
                                            _ptr(topk_gate), _ptr(out), _stream(stream)))


def moe_combine_bwd(shape, dtype, dout, y_perm, slot_row, topk_gate, dy_perm, dgate,
                    stream=None) -> None:
    _check("moe_combine_bwd", lib().moe_combine_bwd(
        shape, dtype, _ptr(dout), _ptr(y_perm), _ptr(slot_row), _ptr(topk_gate), _ptr(dy_perm),
        _ptr(dgate), _stream(stream)))


def moe_combine_bwd_mx(shape, dout, y_perm, slot_row, topk_gate, perm_src, dgate, ws,
                       stream=None) -> None:
    _check("moe_combine_bwd_mx", lib().moe_combine_bwd_mx(
        shape, _ptr(dout), _ptr(y_perm), _ptr(slot_row), _ptr(topk_gate), _ptr(perm_src),
        _ptr(dgate), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_grouped_ffn_bwd(shape, dtype, rows, dy_perm, x_perm, act_saved, offsets, w1, w2,
                        dx_perm, dw1, dw2, dw_dtype, ws, mx=None, stream=None) -> None:
    _check("moe_grouped_ffn_bwd", lib().moe_grouped_ffn_bwd(
        shape, dtype, rows, _ptr(dy_perm), _ptr(x_perm), _ptr(act_saved), _ptr(offsets),
        _ptr(w1), _ptr(w2), _ptr(mx), _ptr(dx_perm), _ptr(dw1), _ptr(dw2), dw_dtype, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_grouped_ffn_bwd_recompute(shape, dtype, rows, dy_perm, x_perm, act_scratch, offsets, w1,
                                  w2, dx_perm, dw1, dw2, dw_dtype, ws, mx=None,
                                  stream=None) -> None:
    _check("moe_grouped_ffn_bwd_recompute", lib().moe_grouped_ffn_bwd_recompute(
        shape, dtype, rows, _ptr(dy_perm), _ptr(x_perm), _ptr(act_scratch), _ptr(offsets),
        _ptr(w1), _ptr(w2), _ptr(mx), _ptr(dx_perm), _ptr(dw1), _ptr(dw2), dw_dtype, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_route_bwd(shape, dtype, x, w_router, logits, topk_idx, dgate, dx_perm, slot_row, dx,
                  dw_router, ws, stream=None) -> None:
    _check("moe_route_bwd", lib().moe_route_bwd(
        shape, dtype, _ptr(x), _ptr(w_router), _ptr(logits), _ptr(topk_idx), _ptr(dgate),
        _ptr(dx_perm), _ptr(slot_row), _ptr(dx), _ptr(dw_router), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def mxfp8_quantize(rows, K, src_dtype, src, axis, seg_offsets, nseg, q, scale,
                   stream=None) -> None:
    _check("mxfp8_quantize", lib().mxfp8_quantize(
        rows, K, src_dtype, _ptr(src), axis, _ptr(seg_offsets), nseg, _ptr(q), _ptr(scale),
        _stream(stream)))


def moe_mx_quantize_weights(shape, w1, w2, out, stream=None) -> None:
    _check("moe_mx_quantize_weights", lib().moe_mx_quantize_weights(
        shape, _ptr(w1), _ptr(w2), _ptr(out), _stream(stream)))


def moe_capacity(shape, cf_num: int = 5, cf_den: int = 4) -> int:
    """Uniform per-expert capacity of the padded layout (computed by the library)."""
    c = lib().moe_capacity(shape, cf_num, cf_den)
    if c < 0:
        raise MoEError("moe_capacity", MOE_ERR_INVALID_ARG)
    return c


def moe_padded_dispatch(shape, dtype, capacity, x, topk_idx, slot_row, offsets, x_pad, pad_row,
                        offsets_pad, stream=None) -> None:
    _check("moe_padded_dispatch", lib().moe_padded_dispatch(
        shape, dtype, capacity, _ptr(x), _ptr(topk_idx), _ptr(slot_row), _ptr(offsets),
        _ptr(x_pad), _ptr(pad_row), _ptr(offsets_pad), _stream(stream)))


def moe_routing_stats(shape, counts, capacity, stats, stream=None) -> None:
    _check("moe_routing_stats", lib().moe_routing_stats(
        shape, _ptr(counts), capacity, _ptr(stats), _stream(stream)))


def moe_renorm_gates(shape, topk_gate, gate_out, stream=None) -> None:
    _check("moe_renorm_gates", lib().moe_renorm_gates(
        shape, _ptr(topk_gate), _ptr(gate_out), _stream(stream)))


def moe_renorm_gates_bwd(shape, topk_gate, dgate_out, dgate, stream=None) -> None:
    _check("moe_renorm_gates_bwd", lib().moe_renorm_gates_bwd(
        shape, _ptr(topk_gate), _ptr(dgate_out), _ptr(dgate), _stream(stream)))


MX_WS_REGIONS = ("qx1", "sx1", "qh1", "sh1", "row_tile", "blocks", "nblocks", "qx0", "sx0",
                 "qh0", "sh0", "dadu", "qdy0", "sdy0", "qda0", "sda0", "qdy1", "sdy1", "qda1",
                 "sda1")


def moe_mx_workspace_layout(shape, rows: int = 0) -> dict:
    """Byte offsets in the workspace of the MXFP8 operand copies (diagnostic)."""
    n = len(MX_WS_REGIONS)
    out = (ctypes.c_int64 * n)()
    _check("moe_mx_workspace_layout", lib().moe_mx_workspace_layout(shape, rows, out, n))
    return dict(zip(MX_WS_REGIONS, list(out)))


def moe_permute_mx(shape, x, slot_row, offsets, perm_src, ws, stream=None) -> None:
    _check("moe_permute_mx", lib().moe_permute_mx(
        shape, _ptr(x), _ptr(slot_row), _ptr(offsets), _ptr(perm_src), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def _ptr_array(ptrs) -> ctypes.Array:
    """Host array of device pointers (tensors or integer addresses)."""
    return (ctypes.c_void_p * len(ptrs))(*[_ptr(p) for p in ptrs])


def moe_ep_layout(shape, n_ranks, rank, counts_all, recv_offsets, send_base, stream=None) -> None:
    _check("moe_ep_layout", lib().moe_ep_layout(shape, n_ranks, rank, _ptr(counts_all),
                                                _ptr(recv_offsets), _ptr(send_base),
                                                _stream(stream)))


def moe_ep_dispatch(shape, dtype, n_ranks, x, topk_idx, slot_row, offsets, send_base, peer_x,
                    ep_row, stream=None) -> None:
    """peer_x: the n_ranks receive buffers (tensors or device addresses)."""
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(
        shape, dtype, n_ranks, _ptr(x), _ptr(topk_idx), _ptr(slot_row), _ptr(offsets),
        _ptr(send_base), _ptr_array(peer_x), _ptr(ep_row), _stream(stream)))


def moe_ep_combine(shape, dtype, n_ranks, peer_y, topk_idx, ep_row, gate, out,
                   stream=None) -> None:
    _check("moe_ep_combine", lib().moe_ep_combine(
        shape, dtype, n_ranks, _ptr_array(peer_y), _ptr(topk_idx), _ptr(ep_row), _ptr(gate),
        _ptr(out), _stream(stream)))


def moe_ep_combine_bwd(shape, dtype, n_ranks, dout, peer_y, topk_idx, ep_row, gate, peer_dy,
                       dgate, stream=None) -> None:
    _check("moe_ep_combine_bwd", lib().moe_ep_combine_bwd(
        shape, dtype, n_ranks, _ptr(dout), _ptr_array(peer_y), _ptr(topk_idx), _ptr(ep_row),
        _ptr(gate), _ptr_array(peer_dy), _ptr(dgate), _stream(stream)))
