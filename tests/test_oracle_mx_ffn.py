"""Pins of the MXFP8 expert-FFN oracle (``oracle.moe_mx_ref``).

Exactness: MXFP8 quantise-dequantise is the identity on a block whose values
all have a 3-bit mantissa (at most 1.75 x a power of two) and lie within a
small power-of-two range of the block maximum.  Each test below builds
operands that are exact in the blocks the reading prescribes for one GEMM
(along its contraction axis; token blocks restarting at every expert) and
strongly inexact in any other blocking (neighbouring rows, columns or
segments scaled 2^16 .. 2^42 apart, so that small values flush to zero).  On
such inputs the MXFP8 oracle must reproduce the unquantised oracle exactly,
and a wrong operand, axis, segment rule or dropped term shows up as a
mismatch.  The preconditions (exact along the right axis, inexact along the
wrong one) are asserted, so the tests keep their power to discriminate.

A last test checks on Gaussian data that quantisation really happens and that
the layer stays near the unquantised one: one MXFP8 quantisation of Gaussian
data costs about 3 % relative error (E4M3 keeps 3 mantissa bits), and an
output of the expert FFN sits behind up to four quantised operands, hence the
bound of 15 %; a wrong operand or a dropped term costs O(100 %).
"""

import numpy as np
import pytest

from oracle import moe_mx_ref as mxr
from oracle import moe_ref as ref

MANT = np.array([1.0, 1.25, 1.5, 1.75])
COUNTS = [37, 0, 70, 33]                      # ragged segments, one empty expert
OFFS = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int64)
E, R, D, F = len(COUNTS), int(OFFS[-1]), 64, 64


def exact(rng, shape, lo=-2, hi=1, zero_frac=0.1):
    """Values +-m * 2^j, m in {1, 1.25, 1.5, 1.75}, j in [lo, hi]; some zeros."""
    v = rng.choice([-1.0, 1.0], size=shape) * rng.choice(MANT, size=shape)
    v = v * 2.0 ** rng.integers(lo, hi + 1, size=shape)
    v[rng.random(shape) < zero_frac] = 0.0
    return v


def pow2(rng, shape, lo, hi, signed=True):
    v = 2.0 ** rng.integers(lo, hi + 1, size=shape)
    return v * rng.choice([-1.0, 1.0], size=shape) if signed else v


def alt(n, a, b):
    """Exponents a, b, a, b, ... of length n."""
    return np.where(np.arange(n) % 2 == 0, a, b)


def block_exps(offs, a=-8, b=8):
    """Per-row exponent that is constant in each 32-row block of each segment
    and alternates between neighbouring blocks (a global block counter)."""
    out = np.zeros(int(offs[-1]), dtype=np.int64)
    n = 0
    for g in range(len(offs) - 1):
        for b0 in range(int(offs[g]), int(offs[g + 1]), 32):
            out[b0:min(b0 + 32, int(offs[g + 1]))] = a if n % 2 == 0 else b
            n += 1
    return out


def same(a, b):
    return np.array_equal(a, b)


def assert_exact_only(v, axis, seg=None):
    """v is exact in the given blocking and not exact in the other ones."""
    assert same(mxr.mx_qdq(v, axis, seg), v)
    if axis == 0:
        assert not same(mxr.mx_qdq(v, 1), v)
    else:
        assert not same(mxr.mx_qdq(v, 0), v)
        if seg is not None:
            assert not same(mxr.mx_qdq(v, 1), v)     # blocks that ignore segments


def test_forward_exact_on_representable_operands():
    rng = np.random.default_rng(1)
    # one-hot rows of x; row exponents 3 / 24 alternate (exact along d only)
    s = alt(R, 3, 24)
    x = np.zeros((R, D))
    x[np.arange(R), rng.integers(0, D, R)] = 2.0 ** s
    # gate rows >= 8 (so a >= 64, silu(a) == a in float64), scaled 2^g per row;
    # up rows +-2^{0,1} scaled 2^-g, so that h = a * u does not depend on g
    g = alt(F, 0, 20)
    w1 = np.zeros((E, 2 * F, D))
    w1[:, :F] = rng.choice(MANT, (E, F, D)) * 2.0 ** rng.integers(3, 5, (E, F, D)) * 2.0 ** g[:, None]
    w1[:, F:] = pow2(rng, (E, F, D), 0, 1) * 2.0 ** -g[:, None]
    # W2 rows scaled 2^0 / 2^20 (exact along f only)
    w2 = exact(rng, (E, D, F)) * 2.0 ** alt(D, 0, 20)[None, :, None]
    a0, u0, h0, y0 = ref.expert_ffn_fwd(x, OFFS, w1, w2)
    assert np.all(a0 >= 64)
    assert_exact_only(x, 0)
    assert_exact_only(w1.reshape(-1, D), 0)
    assert_exact_only(h0, 0)
    assert_exact_only(w2.reshape(-1, F), 0)
    a, u, h, y = mxr.expert_ffn_fwd_mx(x, OFFS, w1, w2)
    for got, want in ((a, a0), (u, u0), (h, h0), (y, y0)):
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_backward_dh_exact_on_representable_operands():
    rng = np.random.default_rng(2)
    dy = exact(rng, (R, D)) * 2.0 ** alt(R, -12, 12)[:, None]          # exact along d
    w2 = exact(rng, (E, D, F)) * 2.0 ** alt(F, -12, 12)[None, None, :]  # exact along d
    a, u, h = rng.normal(size=(3, R, F))
    x = rng.normal(size=(R, D))
    w1 = rng.normal(size=(E, 2 * F, D))
    assert_exact_only(dy, 0)
    assert_exact_only(w2.reshape(-1, F), 1)
    *_, parts = mxr.expert_ffn_bwd_mx(dy, x, a, u, h, OFFS, w1, w2, parts=True)
    for e in range(E):
        r0, r1 = OFFS[e], OFFS[e + 1]
        np.testing.assert_allclose(parts["dh"][r0:r1], dy[r0:r1] @ w2[e], rtol=1e-13, atol=0)


def test_backward_dx_exact_on_representable_operands():
    rng = np.random.default_rng(3)
    s = alt(R, -10, 10)
    dy = np.zeros((R, D))
    dy[np.arange(R), rng.integers(0, D, R)] = 2.0 ** s                  # one-hot rows
    w2 = exact(rng, (E, D, F))
    a = pow2(rng, (R, F), 6, 7, signed=False)                           # silu'(a) == 1
    u = pow2(rng, (R, F), 0, 1)
    h = rng.normal(size=(R, F))
    x = rng.normal(size=(R, D))
    w1 = exact(rng, (E, 2 * F, D)) * 2.0 ** alt(D, -12, 12)[None, None, :]  # exact along 2f
    dx0, _, _ = ref.expert_ffn_bwd(dy, x, a, u, h, OFFS, w1, w2)
    dx, _, _, parts = mxr.expert_ffn_bwd_mx(dy, x, a, u, h, OFFS, w1, w2, parts=True)
    dadu = np.concatenate([parts["da"], parts["du"]], axis=1)
    assert_exact_only(dy, 0)
    assert_exact_only(dadu, 0)
    assert_exact_only(w1.reshape(-1, D), 1)
    np.testing.assert_allclose(dx, dx0, rtol=1e-12, atol=0)


def test_backward_dw2_exact_on_representable_operands():
    rng = np.random.default_rng(4)
    S = block_exps(OFFS)[:, None]
    dy = exact(rng, (R, D)) * 2.0 ** S * 2.0 ** alt(D, -8, 8)[None, :]
    h = exact(rng, (R, F)) * 2.0 ** -S * 2.0 ** alt(F, 8, -8)[None, :]
    a, u = rng.normal(size=(2, R, F))
    x = rng.normal(size=(R, D))
    w1 = rng.normal(size=(E, 2 * F, D))
    w2 = rng.normal(size=(E, D, F))
    assert_exact_only(dy, 1, OFFS)
    assert_exact_only(h, 1, OFFS)
    _, _, dw2_0 = ref.expert_ffn_bwd(dy, x, a, u, h, OFFS, w1, w2)
    _, _, dw2 = mxr.expert_ffn_bwd_mx(dy, x, a, u, h, OFFS, w1, w2)
    np.testing.assert_allclose(dw2, dw2_0, rtol=1e-12, atol=0)
    assert not dw2[1].any()                                             # the empty expert


def test_backward_dw1_exact_on_representable_operands():
    rng = np.random.default_rng(5)
    S = block_exps(OFFS)
    dy = np.zeros((R, D))
    dy[np.arange(R), rng.integers(0, D, R)] = 2.0 ** S                  # one-hot rows
    w2 = exact(rng, (E, D, F)) * 2.0 ** alt(F, -8, 8)[None, None, :]
    a = pow2(rng, (R, F), 6, 7, signed=False)
    u = pow2(rng, (R, F), 0, 1)
    h = rng.normal(size=(R, F))
    x = exact(rng, (R, D)) * 2.0 ** -S[:, None] * 2.0 ** alt(D, 8, -8)[None, :]
    w1 = rng.normal(size=(E, 2 * F, D))
    _, dw1_0, _ = ref.expert_ffn_bwd(dy, x, a, u, h, OFFS, w1, w2)
    _, dw1, _, parts = mxr.expert_ffn_bwd_mx(dy, x, a, u, h, OFFS, w1, w2, parts=True)
    dadu = np.concatenate([parts["da"], parts["du"]], axis=1)
    assert_exact_only(dadu, 1, OFFS)
    assert_exact_only(x, 1, OFFS)
    np.testing.assert_allclose(dw1, dw1_0, rtol=1e-12, atol=0)


def test_layer_close_to_unquantised_layer_on_gaussian_data():
    rng = np.random.default_rng(6)
    T, d, Ex, k, f = 96, 64, 4, 2, 64
    x = rng.normal(size=(T, d))
    wr = rng.normal(size=(Ex, d)) * 0.1
    w1 = rng.normal(size=(Ex, 2 * f, d)) * 0.05
    w2 = rng.normal(size=(Ex, d, f)) * 0.05
    dout = rng.normal(size=(T, d))
    o = ref.layer_fwd_bwd(x, wr, w1, w2, dout, k)
    m = mxr.layer_fwd_bwd_mx(x, wr, w1, w2, dout, k)
    assert same(m["idx"], o["idx"]) and same(m["offsets"], o["offsets"])
    for key in ("y_perm", "out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
        err = np.linalg.norm(m[key] - o[key]) / np.linalg.norm(o[key])
        assert 1e-3 < err < 0.15, (key, err)
    assert same(m["logits"], o["logits"])      # the router is not quantised


@pytest.mark.parametrize("axis", [0, 1])
def test_qdq_is_idempotent(axis):
    rng = np.random.default_rng(7)
    v = rng.normal(size=(70, 64)) * np.exp(rng.normal(size=(70, 1)) * 3)
    seg = [0, 33, 33, 70] if axis == 1 else None
    once = mxr.mx_qdq(v, axis, seg)
    assert same(mxr.mx_qdq(once, axis, seg), once)


def test_round_bf16_matches_torch_on_fp32_values():
    """torch rounds fp32 to bf16 to nearest, ties to even; on fp32 inputs the
    float64 -> bf16 rounding must agree bit for bit (ties included)."""
    import torch
    g = torch.Generator().manual_seed(8)
    v = (torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 8)).float()
    ties = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7), 0.0, -0.0,
                         3.0 * 2.0 ** -100], dtype=torch.float32)
    v = torch.cat([v, ties])
    want = v.to(torch.bfloat16).double().numpy()
    got = mxr.round_bf16(v.double().numpy())
    assert np.array_equal(got, want)


def test_act_round_only_touches_the_stored_values():
    rng = np.random.default_rng(9)
    T, d, Ex, k, f = 64, 64, 4, 2, 64
    args = (rng.normal(size=(T, d)), rng.normal(size=(Ex, d)) * 0.1,
            rng.normal(size=(Ex, 2 * f, d)) * 0.05, rng.normal(size=(Ex, d, f)) * 0.05,
            rng.normal(size=(T, d)), k)
    plain = mxr.layer_fwd_bwd_mx(*args)
    ident = mxr.layer_fwd_bwd_mx(*args, act_round=lambda a: a)
    rounded = mxr.layer_fwd_bwd_mx(*args, act_round=mxr.round_bf16)
    for key in ("out", "dx", "dw1", "dw2", "dw_router"):
        assert same(plain[key], ident[key]), key
        err = np.linalg.norm(rounded[key] - plain[key]) / np.linalg.norm(plain[key])
        assert 0 < err < 0.05, (key, err)
    # the stored activations are bf16 values
    for key in ("a", "u", "h"):
        assert same(mxr.round_bf16(rounded[key]), rounded[key]), key
