"""The C-ABI library loads, exports every entry point that include/moe.h
declares, and rejects bad arguments on the host before touching the GPU.

No compute call runs here (there may be no GPU): every call below is
rejected by host-side validation, which the library performs before any CUDA
call.
"""

import ctypes
import os
import subprocess

import pytest

from mixture_experts_layer_offsets_b200 import capi


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(capi.LIB_PATH):
        from mixture_experts_layer_offsets_b200 import build
        build.build()
    return capi.lib()


def test_exports_every_header_symbol(lib):
    declared = capi.header_symbols()
    assert {"moe_route", "moe_permute", "moe_grouped_ffn_fwd", "moe_grouped_ffn_bwd",
            "moe_combine", "mxfp8_quantize"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", capi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(lib, s)


def test_version_string(lib):
    assert "sm_100a" in capi.moe_version()


def test_library_is_built_for_sm100a(lib):
    out = subprocess.run(["strings", capi.LIB_PATH], capture_output=True, text=True).stdout
    assert "sm_100a" in out


SHAPE = dict(T=64, d_model=256, E=8, top_k=2, d_ff=256)


def _shape(**kw):
    s = dict(SHAPE)
    s.update(kw)
    return capi.moe_shape(**s)


@pytest.mark.parametrize("bad", [dict(top_k=9), dict(top_k=0), dict(E=0), dict(E=2048, top_k=2),
                                 dict(d_model=260), dict(d_ff=12), dict(T=-1), dict(top_k=33, E=64),
                                 dict(T=1 << 30, top_k=4)])
def test_workspace_size_rejects_bad_shapes(lib, bad):
    assert capi.moe_workspace_size(_shape(**bad), capi.MOE_BF16, 0) == 0


def test_workspace_size_grows_with_rows(lib):
    s = _shape()
    a = capi.moe_workspace_size(s, capi.MOE_BF16, 0)
    b = capi.moe_workspace_size(s, capi.MOE_BF16, 64 * 2 * 4)
    assert 256 < a < b


FAKE = 1 << 20  # an aligned non-null address that is never dereferenced


def _route(lib, shape, dtype=capi.MOE_BF16, x=FAKE, w=FAKE, bias=None, ptr=FAKE, ws=FAKE,
           ws_bytes=1 << 30):
    return lib.moe_route(shape, dtype, x, w, bias, ptr, ptr, ptr, ptr, ptr, ptr, ws, ws_bytes, None)


def test_route_validation(lib):
    ok = _shape()
    assert _route(lib, _shape(top_k=9)) == capi.MOE_ERR_INVALID_ARG
    assert _route(lib, ok, x=None) == capi.MOE_ERR_INVALID_ARG
    assert _route(lib, ok, x=FAKE + 4) == capi.MOE_ERR_INVALID_ARG   # misaligned
    assert _route(lib, ok, ws_bytes=16) == capi.MOE_ERR_INVALID_ARG
    assert _route(lib, ok, dtype=7) == capi.MOE_ERR_INVALID_ARG
    assert _route(lib, ok, dtype=capi.MOE_MXFP8) == capi.MOE_ERR_UNSUPPORTED
    assert _route(lib, ok, bias=FAKE + 8) == capi.MOE_ERR_INVALID_ARG


def test_ffn_validation(lib):
    s = _shape()
    f = lib.moe_grouped_ffn_fwd
    assert f(s, capi.MOE_BF16, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) \
        == capi.MOE_ERR_INVALID_ARG  # MXFP8 weights given to a bf16 call
    assert f(s, capi.MOE_MXFP8, 128, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1 << 30, None) \
        == capi.MOE_ERR_INVALID_ARG  # MXFP8 call without its weights
    assert f(s, capi.MOE_BF16, -1, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1 << 30, None) \
        == capi.MOE_ERR_INVALID_ARG
    assert f(_shape(d_model=136), capi.MOE_BF16, 128, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE,
             FAKE, 1 << 30, None) == capi.MOE_ERR_UNSUPPORTED  # tensor-core tiles need d % 256
    b = lib.moe_grouped_ffn_bwd
    args = [FAKE] * 6
    assert b(s, capi.MOE_BF16, 128, *args, None, FAKE, FAKE, FAKE, 9, FAKE, 1 << 30, None) \
        == capi.MOE_ERR_INVALID_ARG  # bad dw dtype
    assert b(s, capi.MOE_F32, 128, *args, None, FAKE, FAKE, FAKE, capi.MOE_BF16, FAKE, 1 << 30,
             None) == capi.MOE_ERR_INVALID_ARG
    assert b(s, capi.MOE_BF16, 128, *args, None, FAKE, FAKE, FAKE, capi.MOE_F32, FAKE, 300, None) \
        == capi.MOE_ERR_INVALID_ARG  # workspace too small
    # the SwiGLU backward reads a and u in 32-byte pieces: act_saved aligned to 16 only
    assert b(s, capi.MOE_BF16, 128, FAKE, FAKE, FAKE + 16, FAKE, FAKE, FAKE, None, FAKE, FAKE,
             FAKE, capi.MOE_F32, FAKE, 1 << 30, None) == capi.MOE_ERR_INVALID_ARG


def test_row_ops_validation(lib):
    s = _shape()
    assert lib.moe_permute(s, capi.MOE_BF16, FAKE, None, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(s, capi.MOE_BF16, FAKE, FAKE, FAKE + 2, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_bwd(_shape(top_k=40, E=64), capi.MOE_BF16, *([FAKE] * 6), None) \
        == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_padded_dispatch(s, capi.MOE_BF16, 0, *([FAKE] * 7), None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_route_bwd(s, capi.MOE_BF16, *([FAKE] * 9), FAKE, 16, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_routing_stats(s, FAKE, -1, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_routing_stats(s, None, 0, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_routing_stats(_shape(E=2048), FAKE, 0, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_renorm_gates(s, FAKE + 4, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_renorm_gates_bwd(s, FAKE, None, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_renorm_gates(_shape(T=0), None, None, None) == capi.MOE_OK
    assert lib.moe_grouped_ffn_bwd_recompute(s, capi.MOE_BF16, 64, *([FAKE] * 3), None,
                                             *([FAKE] * 6), capi.MOE_F32, FAKE, 1 << 30,
                                             None) == capi.MOE_ERR_INVALID_ARG
    # T == 0 is a valid no-op for the row movers
    assert lib.moe_permute(_shape(T=0), capi.MOE_BF16, None, None, None, None, None) == capi.MOE_OK


def test_mxfp8_validation(lib):
    q = lib.mxfp8_quantize
    assert q(4, 48, capi.MOE_BF16, FAKE, 0, None, 0, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert q(4, 64, capi.MOE_BF16, FAKE, 2, None, 0, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert q(4, 64, 5, FAKE, 0, None, 0, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert q(4, 24, capi.MOE_F32, FAKE, 1, None, 0, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert q(4, 64, capi.MOE_F32, FAKE, 1, FAKE, 0, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert q(0, 64, capi.MOE_F32, None, 0, None, 0, None, None, None) == capi.MOE_OK


def test_status_query_validation(lib):
    assert lib.moe_get_device_status(None, None, ctypes.byref(ctypes.c_int32())) == capi.MOE_ERR_INVALID_ARG


def _mxw(**kw):
    fields = {n: FAKE for n, _ in capi.moe_mx_weights._fields_}
    fields.update(kw)
    return capi.moe_mx_weights(**fields)


def test_mxfp8_ffn_validation(lib):
    f, b = lib.moe_grouped_ffn_fwd, lib.moe_grouped_ffn_bwd
    s = _shape()
    mx = _mxw()
    big = capi.moe_workspace_size(s, capi.MOE_MXFP8, 128)
    assert big > capi.moe_workspace_size(s, capi.MOE_BF16, 128)   # room for the MXFP8 operands

    def fwd(shape=s, mxw=mx, ws_bytes=big):
        return f(shape, capi.MOE_MXFP8, 128, FAKE, FAKE, None, None, ctypes.addressof(mxw), FAKE,
                 FAKE, FAKE, ws_bytes, None)

    def bwd(dw_dtype=capi.MOE_F32, mxw=mx, ws_bytes=big, act=FAKE):
        return b(s, capi.MOE_MXFP8, 128, FAKE, FAKE, act, FAKE, None, None, ctypes.addressof(mxw),
                 FAKE, FAKE, FAKE, dw_dtype, FAKE, ws_bytes, None)

    assert fwd(shape=_shape(d_model=192)) == capi.MOE_ERR_UNSUPPORTED     # d % 128
    assert fwd(shape=_shape(d_ff=200)) == capi.MOE_ERR_UNSUPPORTED        # f % 128
    assert fwd(mxw=_mxw(w2t_s=None)) == capi.MOE_ERR_INVALID_ARG
    assert fwd(mxw=_mxw(w1_q=FAKE + 8)) == capi.MOE_ERR_INVALID_ARG      # misaligned
    assert fwd(ws_bytes=big // 2) == capi.MOE_ERR_INVALID_ARG
    assert bwd(dw_dtype=capi.MOE_BF16) == capi.MOE_ERR_INVALID_ARG       # dW is fp32
    assert bwd(ws_bytes=1024) == capi.MOE_ERR_INVALID_ARG
    assert bwd(act=FAKE + 16) == capi.MOE_ERR_INVALID_ARG               # act_saved 32-byte aligned
    # the MXFP8 epilogues write their operand copies into ws with 32-byte stores
    assert f(s, capi.MOE_MXFP8, 128, FAKE, FAKE, None, None, ctypes.addressof(mx), FAKE, FAKE,
             FAKE + 16, big, None) == capi.MOE_ERR_INVALID_ARG
    assert b(s, capi.MOE_MXFP8, 128, FAKE, FAKE, FAKE, FAKE, None, None, ctypes.addressof(mx),
             FAKE, FAKE, FAKE, capi.MOE_F32, FAKE + 16, big, None) == capi.MOE_ERR_INVALID_ARG


def test_mxfp8_combine_bwd_validation(lib):
    """moe_combine_bwd_mx (dgate plus dy's MXFP8 copies into the workspace) and the
    backward's dy_perm = NULL form, which the recompute backward refuses."""
    s = _shape()
    big = capi.moe_workspace_size(s, capi.MOE_MXFP8, 0)

    def cb(shape=s, dout=FAKE, perm_src=FAKE, ws=FAKE, ws_bytes=big):
        return lib.moe_combine_bwd_mx(shape, dout, FAKE, FAKE, FAKE, perm_src, FAKE, ws, ws_bytes,
                                      None)

    assert cb(shape=_shape(d_model=192)) == capi.MOE_ERR_UNSUPPORTED      # d % 128
    assert cb(dout=None) == capi.MOE_ERR_INVALID_ARG
    assert cb(perm_src=None) == capi.MOE_ERR_INVALID_ARG
    assert cb(perm_src=FAKE + 4) == capi.MOE_ERR_INVALID_ARG               # misaligned
    assert cb(ws=None) == capi.MOE_ERR_INVALID_ARG
    assert cb(ws_bytes=big // 2) == capi.MOE_ERR_INVALID_ARG
    assert cb(shape=_shape(top_k=9)) == capi.MOE_ERR_INVALID_ARG
    mx = _mxw()
    rows = s.T * s.top_k
    wsb = capi.moe_workspace_size(s, capi.MOE_MXFP8, rows)
    rc = lib.moe_grouped_ffn_bwd_recompute(s, capi.MOE_MXFP8, rows, None, FAKE, FAKE, FAKE, None,
                                           None, ctypes.addressof(mx), FAKE, FAKE, FAKE,
                                           capi.MOE_F32, FAKE, wsb, None)
    assert rc == capi.MOE_ERR_INVALID_ARG   # the recompute needs dy_perm


def test_mx_quantize_weights_validation(lib):
    g = lib.moe_mx_quantize_weights
    mx = _mxw()
    assert g(_shape(d_model=192), FAKE, FAKE, ctypes.addressof(mx), None) == capi.MOE_ERR_UNSUPPORTED
    assert g(_shape(), None, FAKE, ctypes.addressof(mx), None) == capi.MOE_ERR_INVALID_ARG
    assert g(_shape(), FAKE, FAKE, None, None) == capi.MOE_ERR_INVALID_ARG
    assert g(_shape(), FAKE, FAKE, ctypes.addressof(_mxw(w1t_q=FAKE + 1)), None) == capi.MOE_ERR_INVALID_ARG


def test_capacity_is_the_exact_integer_ceiling(lib):
    # ceil(cf * T*k / E); the skewed workload: ceil(1.25 * 131072 / 128) = 1280
    assert capi.moe_capacity(capi.shape_of(32768, 2048, 128, 4, 1024), 5, 4) == 1280
    for T, E, k, num, den in [(3, 4, 2, 5, 4), (1, 7, 1, 5, 4), (1000, 3, 3, 1, 1), (0, 8, 2, 5, 4),
                              (999, 64, 4, 3, 2)]:
        want = -(-num * T * k // (den * E))
        assert capi.moe_capacity(capi.shape_of(T, 256, E, k, 256), num, den) == want
    assert lib.moe_capacity(_shape(), 0, 4) == -1
    assert lib.moe_capacity(_shape(), 5, 0) == -1
    assert lib.moe_capacity(_shape(top_k=9), 5, 4) == -1
    assert lib.moe_capacity(capi.shape_of(1 << 28, 256, 1, 1, 256), 1 << 30, 1) == -1  # > INT32_MAX


def test_mx_workspace_layout(lib):
    s = capi.shape_of(500, 384, 16, 4, 384)
    lay = capi.moe_mx_workspace_layout(s)
    assert list(lay) == list(capi.MX_WS_REGIONS)
    size = capi.moe_workspace_size(s, capi.MOE_MXFP8, 0)
    R, d, f = 2000, 384, 384
    # regions are 256-byte aligned, past the status word, and inside the workspace
    for name, off in lay.items():
        assert off % 256 == 0 and 256 <= off < size, name
    assert lay["qx0"] == lay["dadu"]                    # forward row copies share with backward
    assert lay["sx1"] - lay["qx1"] >= R * d and lay["sh1"] - lay["qh1"] >= R * f
    assert lay["qdy0"] - lay["dadu"] >= R * 2 * f * 2
    out = (ctypes.c_int64 * 20)()
    assert lib.moe_mx_workspace_layout(s, 0, out, 19) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_mx_workspace_layout(_shape(d_model=192), 0, out, 20) == capi.MOE_ERR_UNSUPPORTED
    assert lib.moe_mx_workspace_layout(_shape(top_k=9), 0, out, 20) == capi.MOE_ERR_INVALID_ARG


def test_profile_begin_end_bookkeeping(lib):
    # no launch happens between begin and end here, so no event is touched
    ev = (ctypes.c_void_p * 4)()
    names = (ctypes.c_char_p * 2)()
    n = ctypes.c_int32(-1)
    assert lib.moe_profile_end(ctypes.byref(n)) == capi.MOE_ERR_INVALID_ARG      # not open
    assert lib.moe_profile_begin(None, names, 2) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_profile_begin(ev, names, 0) == capi.MOE_ERR_INVALID_ARG
    assert lib.moe_profile_begin(ev, names, 2) == capi.MOE_OK
    assert lib.moe_profile_begin(ev, names, 2) == capi.MOE_ERR_INVALID_ARG      # already open
    # a call rejected on the host launches nothing and records nothing
    assert lib.moe_permute(_shape(), capi.MOE_BF16, FAKE, None, FAKE, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG
    assert lib.moe_profile_end(ctypes.byref(n)) == capi.MOE_OK and n.value == 0


def test_noalloc_status_validation(lib):
    assert lib.moe_route_noalloc_status(None, None) == capi.MOE_ERR_INVALID_ARG


def test_expert_parallel_validation(lib):
    s = _shape()   # E = 8
    peers2 = (ctypes.c_void_p * 2)(FAKE, FAKE)
    bad_peers = (ctypes.c_void_p * 2)(FAKE, FAKE + 8)
    lay = lib.moe_ep_layout
    assert lay(s, 3, 0, FAKE, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG     # E % N
    assert lay(s, 2, 2, FAKE, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG     # rank >= N
    assert lay(s, 0, 0, FAKE, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lay(s, 2, 0, None, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert lay(_shape(E=128, top_k=2), 65, 0, FAKE, FAKE, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    dis = lib.moe_ep_dispatch
    args = [FAKE] * 5
    assert dis(s, capi.MOE_BF16, 2, *args, bad_peers, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert dis(s, capi.MOE_BF16, 2, *args, None, FAKE, None) == capi.MOE_ERR_INVALID_ARG
    assert dis(s, capi.MOE_MXFP8, 2, *args, peers2, FAKE, None) == capi.MOE_ERR_UNSUPPORTED
    assert dis(s, capi.MOE_BF16, 2, FAKE, None, FAKE, FAKE, FAKE, peers2, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG
    assert dis(_shape(T=0), capi.MOE_BF16, 2, None, None, None, None, None, None, None,
               None) == capi.MOE_OK
    com = lib.moe_ep_combine
    assert com(s, capi.MOE_BF16, 2, bad_peers, FAKE, FAKE, None, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG
    assert com(s, capi.MOE_BF16, 2, peers2, FAKE, FAKE, FAKE + 4, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG
    cb = lib.moe_ep_combine_bwd
    assert cb(s, capi.MOE_BF16, 2, FAKE, peers2, FAKE, FAKE, FAKE, bad_peers, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG
    assert cb(s, capi.MOE_BF16, 2, FAKE, peers2, FAKE, FAKE, None, peers2, FAKE, None) == \
        capi.MOE_ERR_INVALID_ARG   # gates required
