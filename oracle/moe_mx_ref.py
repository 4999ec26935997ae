"""Float64 oracle of the grouped SwiGLU expert FFN with MXFP8 GEMM operands.

TEST INFRASTRUCTURE ONLY (see the package docstring).

kongchang, section 吞吐量数字的边界条件 (boundary conditions): MXFP8 is the
OCP 8-bit microscaling format (32 elements share one scale); it shortens the
GEMMs and shrinks saved activations while an FP32 master weight is kept.
aikraft, section "Технические оптимизации": MXFP8 is one of the optimisations
behind the throughput.  Neither page says which operands are quantised or
along which axis.  Reading taken here (the plain one for a block-scaled GEMM,
whose scale blocks must run along the contraction axis):

* every operand of every expert GEMM is quantised to MXFP8 right before that
  GEMM, in blocks of 32 along that GEMM's contraction (K) axis, and the GEMM
  is exact on the dequantised values (fp32 accumulation on the device);
* forward: ``x`` (K = d) with ``W1[e]`` (K = d) for gate/up; ``h`` (K = f)
  with ``W2[e]`` (K = f) for down;
* input gradient: ``dy`` (K = d) with ``W2[e]`` blocked along d;
  ``[da | du]`` (K = 2f) with ``W1[e]`` blocked along 2f;
* weight gradient: ``dy``, ``h``, ``[da | du]`` and ``x`` blocked along the
  token axis, with blocks restarting at every expert's first row (an expert's
  last block is zero-padded);
* the SwiGLU nonlinearity and its derivative use the unquantised ``a``, ``u``
  of the forward GEMM; master weights stay full precision.

The quantisation rule is ``mxfp8_ref.mxfp8_quantize`` (OCP floor rule).

Storage precision of quantised activations.  An MXFP8 code is an integer
decision taken by floating point, so it has to be taken on the same value on
both sides.  A layer that keeps its activations in bf16 quantises the bf16
copies of ``h``, ``dy`` and ``[da | du]`` and feeds the bf16 copies of ``a``
and ``u`` to the SwiGLU backward.  ``act_round`` (default: none, pure
float64) names the rounding applied to exactly those stored values before
they are used; ``round_bf16`` is the bf16 one.
"""

from __future__ import annotations

import numpy as np

from .moe_ref import (_f64, combine, combine_bwd, permute, route, route_bwd,
                      sigmoid, silu)
from .mxfp8_ref import mxfp8_dequantize, mxfp8_quantize

__all__ = ["round_bf16", "mx_qdq", "expert_ffn_fwd_mx", "expert_ffn_bwd_mx", "layer_fwd_bwd_mx"]


def round_bf16(a) -> np.ndarray:
    """Round to the nearest bfloat16 value (8 significant bits), ties to even.

    Written for the normal range (|a| >= 2^-126, the magnitudes of this layer);
    it keeps 8 significant bits below it as well instead of bf16's subnormals.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                    # a = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def _keep(a):
    return a


def mx_qdq(a, axis: int = 0, seg_offsets=None) -> np.ndarray:
    """The value an MXFP8 operand stands for: quantise, then dequantise.

    axis 0: blocks of 32 along each row; axis 1: blocks of 32 rows within each
    column, restarting at every ``seg_offsets`` boundary.
    """
    q, s = mxfp8_quantize(a, axis=axis, seg_offsets=seg_offsets)
    return mxfp8_dequantize(q, s, axis=axis, seg_offsets=seg_offsets)


def expert_ffn_fwd_mx(x_perm, offsets, w1, w2, act_round=None):
    """MXFP8 forward of the grouped SwiGLU FFN: returns (a, u, h, y).

    ``a | u = Q_d(x) Q_d(W1[e])^T``, ``h = silu(a) * u``,
    ``y = Q_f(h) Q_f(W2[e])^T`` where ``Q_k`` quantises in blocks along k.
    ``h`` is computed from the unrounded ``a``, ``u``; the returned (stored)
    a, u, h and the h that is quantised pass through ``act_round``.
    """
    rnd = act_round or _keep
    x_perm, w1, w2 = _f64(x_perm), _f64(w1), _f64(w2)
    offsets = np.asarray(offsets, dtype=np.int64)
    E, f2, d = w1.shape
    f = f2 // 2
    xq = mx_qdq(x_perm, 0)
    w1q = mx_qdq(w1.reshape(E * f2, d), 0).reshape(E, f2, d)
    w2q = mx_qdq(w2.reshape(E * d, f), 0).reshape(E, d, f)
    R = x_perm.shape[0]
    a = np.zeros((R, f))
    u = np.zeros((R, f))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            a[r0:r1] = xq[r0:r1] @ w1q[e, :f].T
            u[r0:r1] = xq[r0:r1] @ w1q[e, f:].T
    h = rnd(silu(a) * u)
    a, u = rnd(a), rnd(u)
    hq = mx_qdq(h, 0)
    y = np.zeros((R, d))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            y[r0:r1] = hq[r0:r1] @ w2q[e].T
    return a, u, h, y


def expert_ffn_bwd_mx(dy_perm, x_perm, a, u, h, offsets, w1, w2, parts: bool = False,
                      act_round=None):
    """MXFP8 backward of the grouped SwiGLU FFN: returns (dx_perm, dw1, dw2).

    ``dh = Q_d(dy) Q_d(W2[e])``; ``da = dh * u * silu'(a)``,
    ``du = dh * silu(a)``; ``dx = Q_2f([da|du]) Q_2f(W1[e])``;
    ``dW2[e] = Q_t(dy)^T Q_t(h)``, ``dW1[e] = Q_t([da|du])^T Q_t(x)`` with
    ``Q_t`` blocked along the expert's own rows.  With ``parts`` the dict
    {dh, da, du} is returned as a fourth item.  ``dy`` and ``[da | du]`` pass
    through ``act_round`` before they are quantised (a, u, h arrive stored).
    """
    rnd = act_round or _keep
    dy_perm, x_perm = rnd(_f64(dy_perm)), _f64(x_perm)
    a, u, h, w1, w2 = _f64(a), _f64(u), _f64(h), _f64(w1), _f64(w2)
    offsets = np.asarray(offsets, dtype=np.int64)
    E, f2, d = w1.shape
    f = f2 // 2
    R = dy_perm.shape[0]
    # dgrad operands, blocked along the contraction axis
    dyq = mx_qdq(dy_perm, 0)
    w2t = mx_qdq(w2.reshape(E * d, f), 1).reshape(E, d, f)      # blocks along d
    w1t = mx_qdq(w1.reshape(E * f2, d), 1).reshape(E, f2, d)    # blocks along 2f
    dh = np.zeros((R, f))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            dh[r0:r1] = dyq[r0:r1] @ w2t[e]
    s = sigmoid(a)
    da = dh * u * s * (1.0 + a * (1.0 - s))
    du = dh * silu(a)
    dadu = rnd(np.concatenate([da, du], axis=1))
    daq = mx_qdq(dadu, 0)
    dx_perm = np.zeros((R, d))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            dx_perm[r0:r1] = daq[r0:r1] @ w1t[e]
    # wgrad operands, blocked along each expert's rows
    dyt = mx_qdq(dy_perm, 1, offsets)
    ht = mx_qdq(h, 1, offsets)
    dat = mx_qdq(dadu, 1, offsets)
    xt = mx_qdq(x_perm, 1, offsets)
    dw1 = np.zeros((E, f2, d))
    dw2 = np.zeros((E, d, f))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            dw2[e] = dyt[r0:r1].T @ ht[r0:r1]
            dw1[e] = dat[r0:r1].T @ xt[r0:r1]
    if parts:
        return dx_perm, dw1, dw2, dict(dh=dh, da=da, du=du)
    return dx_perm, dw1, dw2


def layer_fwd_bwd_mx(x, w_router, w1, w2, dout, k: int, bias=None, select_logits=None,
                     act_round=None) -> dict:
    """Forward + backward of the layer with MXFP8 expert GEMMs.

    Routing, permute, combine and their backward are those of the unquantised
    layer (the router is not an expert GEMM); only the expert FFN changes.
    ``act_round``: see the module docstring.
    """
    r = route(x, w_router, k, bias, select_logits)
    x_perm = permute(x, r["slot_row"])
    a, u, h, y_perm = expert_ffn_fwd_mx(x_perm, r["offsets"], w1, w2, act_round)
    out = combine(y_perm, r["slot_row"], r["gate"])
    dgate, dy_perm = combine_bwd(dout, y_perm, r["slot_row"], r["gate"])
    dx_perm, dw1, dw2 = expert_ffn_bwd_mx(dy_perm, x_perm, a, u, h, r["offsets"], w1, w2,
                                          act_round=act_round)
    dx, dw_router, dl = route_bwd(x, w_router, r["logits"], r["idx"], dgate, dx_perm,
                                  r["slot_row"])
    r.update(x_perm=x_perm, a=a, u=u, h=h, y_perm=y_perm, out=out, dgate=dgate,
             dy_perm=dy_perm, dx_perm=dx_perm, dw1=dw1, dw2=dw2, dx=dx,
             dw_router=dw_router, dl=dl)
    return r
