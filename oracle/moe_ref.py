"""Float64 oracle of the token-routed MoE SwiGLU FFN layer: forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it and
for the page names used in the citations below).

Notation follows the pages' statement of the problem: T tokens of width
d_model, E experts, each token routed to top_k of them, expert hidden width
d_ff (written f), R = T * top_k permuted rows.

Everything here is the plain definition written out with NumPy float64
matrix products as the only library primitive: no blocking, no fusion, no
reordering beyond what each definition states.  Inputs arrive as NumPy arrays
holding the exact values of the (fp32 or bf16) tensors the device uses;
they are promoted to float64 exactly.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "router_logits", "softmax", "topk_select", "expert_counts_offsets",
    "slot_rows", "perm_src_from_slots", "route", "route_from_logits",
    "permute", "sigmoid", "silu", "expert_ffn_fwd", "combine", "combine_bwd",
    "expert_ffn_bwd", "route_bwd", "layer_fwd_bwd", "capacity",
    "padded_layout", "padded_layer_fwd_bwd", "routing_stats", "renorm_gates",
    "renorm_gates_bwd",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# Routing
# --------------------------------------------------------------------------

def router_logits(x, w_router, bias=None) -> np.ndarray:
    """Router logits ``l[t, e] = sum_c x[t, c] * w_router[e, c] (+ bias[e])``.

    kongchang, section 容量税 (capacity tax): every token goes through a route
    function that activates only a few of the experts ("e.g. 4 of 128").  The
    pages give no formula; the reading taken is a linear router on the token's
    hidden state, with an optional per-expert additive bias (the skewed-routing
    workload adds one).
    """
    l = _f64(x) @ _f64(w_router).T
    if bias is not None:
        l = l + _f64(bias)[None, :]
    return l


def softmax(l) -> np.ndarray:
    """Row softmax over the E experts, max-subtracted.

    Reading: the router probability is a softmax over all E experts, taken
    before the top-k selection, and the selected probabilities are used as
    gates without renormalisation (the pages name no activation; this makes
    "top_k = E equals a dense softmax mixture" exactly true).
    """
    l = _f64(l)
    m = l.max(axis=1, keepdims=True)
    z = np.exp(l - m)
    return z / z.sum(axis=1, keepdims=True)


def topk_select(l, k: int) -> np.ndarray:
    """Indices ``idx[t, 0..k-1]`` of the k largest logits of each token.

    Experts are ordered by (-l[t, e], e): descending logit, and on equal
    logits the lowest expert index first.  Selection is made on the logits
    (softmax is monotone, and selecting on logits avoids ties created by
    rounding in exp).  A stable sort of -l gives exactly this order.
    """
    l = _f64(l)
    E = l.shape[1]
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    return np.argsort(-l, axis=1, kind="stable")[:, :k].astype(np.int64)


def expert_counts_offsets(idx, E: int):
    """Per-expert row counts and their exclusive prefix sum.

    kongchang, section 路由不只是模型问题，更是系统问题 (routing is a systems
    problem): the routing metadata (all-to-all split sizes and the expert
    GEMM group sizes) stays on the GPU.  ``counts[e]`` is the number of
    (token, slot) pairs routed to expert e; ``offsets`` has E + 1 entries,
    ``offsets[0] = 0`` and ``offsets[E] = T * k``.
    """
    idx = np.asarray(idx, dtype=np.int64)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return counts, offsets


def slot_rows(idx, offsets) -> np.ndarray:
    """Row of the expert input buffer that (token t, slot j) is written to.

    bytechap, section "Cách thức hoạt động" (how it works): rowwise dispatch
    places routed data directly into the experts' input buffers.  Within an
    expert's segment ``[offsets[e], offsets[e+1])`` rows are ordered by
    ascending token id (a stable counting sort); each token picks an expert
    at most once, so this order is total.
    """
    idx = np.asarray(idx, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    slot = np.empty(idx.shape, dtype=np.int64)
    for e in range(len(offsets) - 1):
        t_sel, j_sel = np.nonzero(idx == e)  # row-major: ascending token id
        slot[t_sel, j_sel] = offsets[e] + np.arange(len(t_sel))
    return slot


def perm_src_from_slots(slot) -> np.ndarray:
    """Inverse map: ``perm_src[r]`` is the token whose row sits at row r."""
    slot = np.asarray(slot, dtype=np.int64)
    T, k = slot.shape
    src = np.full(T * k, -1, dtype=np.int64)
    src[slot.ravel()] = np.repeat(np.arange(T), k)
    return src


def route_from_logits(l, k: int, select_logits=None) -> dict:
    """All routing outputs from logits ``l`` (float64 values).

    ``select_logits`` (optional) are the logits the discrete decision is taken
    on; when the device computed the logits, the oracle takes the top-k on the
    device's own values (promoted exactly to float64) so that the indices,
    counts, offsets and rows can be compared bit for bit, while gate values
    still come from ``l``.
    """
    l = _f64(l)
    E = l.shape[1]
    sel = l if select_logits is None else _f64(select_logits)
    idx = topk_select(sel, k)
    p = softmax(l)
    gate = np.take_along_axis(p, idx, axis=1)
    counts, offsets = expert_counts_offsets(idx, E)
    slot = slot_rows(idx, offsets)
    return dict(logits=l, p=p, idx=idx, gate=gate, counts=counts,
                offsets=offsets, slot_row=slot, perm_src=perm_src_from_slots(slot))


def route(x, w_router, k: int, bias=None, select_logits=None) -> dict:
    """Router logits, softmax, top-k, counts, offsets, slot rows (see above)."""
    return route_from_logits(router_logits(x, w_router, bias), k, select_logits)


def permute(x, slot) -> np.ndarray:
    """``x_perm[slot[t, j]] = x[t]`` for every token t and slot j."""
    x = _f64(x)
    slot = np.asarray(slot, dtype=np.int64)
    T, k = slot.shape
    x_perm = np.zeros((T * k, x.shape[1]))
    for j in range(k):
        x_perm[slot[:, j]] = x
    return x_perm


# --------------------------------------------------------------------------
# Experts (SwiGLU) on the permuted rows
# --------------------------------------------------------------------------

def sigmoid(a) -> np.ndarray:
    a = _f64(a)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-a[pos]))
    ea = np.exp(a[~pos])
    out[~pos] = ea / (1.0 + ea)
    return out


def silu(a) -> np.ndarray:
    a = _f64(a)
    return a * sigmoid(a)


def expert_ffn_fwd(x_perm, offsets, w1, w2):
    """Grouped SwiGLU expert FFN over the per-expert row segments.

    kongchang, section 路由不只是模型问题，更是系统问题: a device-scheduled
    grouped GEMM handles the uneven per-expert shapes that routing produces.
    For expert e and rows ``r in [offsets[e], offsets[e+1])``:
    ``a = X W1[e, :f]^T`` (gate), ``u = X W1[e, f:]^T`` (up),
    ``h = silu(a) * u``, ``y = h W2[e]^T``.  ``w1`` is [E, 2f, d] (gate rows
    first, then up rows), ``w2`` is [E, d, f].  Experts have no bias terms.
    Returns (a, u, h, y) over all R rows.
    """
    x_perm, w1, w2 = _f64(x_perm), _f64(w1), _f64(w2)
    offsets = np.asarray(offsets, dtype=np.int64)
    R, d = x_perm.shape
    E, f2, _ = w1.shape
    f = f2 // 2
    a = np.zeros((R, f))
    u = np.zeros((R, f))
    y = np.zeros((R, d))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        X = x_perm[r0:r1]
        a[r0:r1] = X @ w1[e, :f].T
        u[r0:r1] = X @ w1[e, f:].T
    h = silu(a) * u
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        y[r0:r1] = h[r0:r1] @ w2[e].T
    return a, u, h, y


def combine(y_perm, slot, gate) -> np.ndarray:
    """Gate-weighted combine: ``out[t] = sum_j gate[t, j] * y_perm[slot[t, j]]``.

    kongchang, section 容量税: the token's output is the mix of the few experts
    it activated.  The sum runs over ascending j.
    """
    y_perm, gate = _f64(y_perm), _f64(gate)
    slot = np.asarray(slot, dtype=np.int64)
    T, k = slot.shape
    out = np.zeros((T, y_perm.shape[1]))
    for j in range(k):
        out += gate[:, j:j + 1] * y_perm[slot[:, j]]
    return out


def combine_bwd(dout, y_perm, slot, gate):
    """Gradient of ``combine`` with respect to its gates and expert rows.

    ``dgate[t, j] = <dout[t], y_perm[slot[t, j]]>`` and
    ``dy_perm[slot[t, j]] = gate[t, j] * dout[t]``.
    """
    dout, y_perm, gate = _f64(dout), _f64(y_perm), _f64(gate)
    slot = np.asarray(slot, dtype=np.int64)
    T, k = slot.shape
    dgate = np.zeros((T, k))
    dy_perm = np.zeros_like(y_perm)
    for j in range(k):
        dgate[:, j] = np.sum(dout * y_perm[slot[:, j]], axis=1)
        dy_perm[slot[:, j]] = gate[:, j:j + 1] * dout
    return dgate, dy_perm


def renorm_gates(gate) -> np.ndarray:
    """Optional gate rule: the k selected probabilities rescaled to sum to one,
    ``g'[t, j] = g[t, j] / S[t]`` with ``S[t] = sum_j g[t, j]``.

    Reading: the pages fix no gate rule (the default keeps the softmax values as
    they are); renormalising over the selected experts is offered as an option
    beside the routing-balance statistics (kongchang, routing section).
    """
    g = _f64(gate)
    return g / g.sum(axis=1, keepdims=True)


def renorm_gates_bwd(gate, dgate_rn) -> np.ndarray:
    """Gradient of ``renorm_gates`` with respect to the selected probabilities:
    ``dg[t, j] = (dg'[t, j] - sum_i g'[t, i] dg'[t, i]) / S[t]``, from
    ``d g'_i / d g_j = (delta_ij - g'_i) / S``."""
    g = _f64(gate)
    S = g.sum(axis=1, keepdims=True)
    gr = g / S
    dgr = _f64(dgate_rn)
    return (dgr - np.sum(gr * dgr, axis=1, keepdims=True)) / S


def expert_ffn_bwd(dy_perm, x_perm, a, u, h, offsets, w1, w2):
    """Backward of ``expert_ffn_fwd``: grouped dgrad and wgrad.

    Per expert e (rows of its segment): ``dh = dy W2[e]``;
    ``silu'(a) = s (1 + a (1 - s))`` with ``s = sigmoid(a)``;
    ``da = dh * u * silu'(a)``; ``du = dh * silu(a)``;
    ``dx = da W1[e, :f] + du W1[e, f:]``; ``dW2[e] = dy^T h``;
    ``dW1[e, :f] = da^T x``; ``dW1[e, f:] = du^T x``.  An expert with no rows
    gets zero weight gradients.  Returns (dx_perm, dw1, dw2).
    """
    dy_perm, x_perm = _f64(dy_perm), _f64(x_perm)
    a, u, h, w1, w2 = _f64(a), _f64(u), _f64(h), _f64(w1), _f64(w2)
    offsets = np.asarray(offsets, dtype=np.int64)
    E, f2, d = w1.shape
    f = f2 // 2
    dx_perm = np.zeros_like(x_perm)
    dw1 = np.zeros_like(w1)
    dw2 = np.zeros_like(w2)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        dY, A, U, H, X = dy_perm[r0:r1], a[r0:r1], u[r0:r1], h[r0:r1], x_perm[r0:r1]
        dH = dY @ w2[e]
        s = sigmoid(A)
        dA = dH * U * s * (1.0 + A * (1.0 - s))
        dU = dH * A * s
        dx_perm[r0:r1] = dA @ w1[e, :f] + dU @ w1[e, f:]
        dw2[e] = dY.T @ H
        dw1[e, :f] = dA.T @ X
        dw1[e, f:] = dU.T @ X
    return dx_perm, dw1, dw2


def route_bwd(x, w_router, logits, idx, dgate, dx_perm, slot):
    """Unpermute-grad plus router grad.

    ``dx[t] = sum_j dx_perm[slot[t, j]]`` (expert path) plus the router path:
    ``dp[t, e] = dgate[t, j]`` where ``e = idx[t, j]`` (0 at unselected
    experts), ``dl = p * (dp - <p, dp>)`` (softmax Jacobian),
    ``dw_router = dl^T x``, ``dx += dl w_router``.  The optional logit bias is
    an input, not a parameter, so it gets no gradient.  Returns (dx, dw_router, dl).
    """
    x, w_router, dgate, dx_perm = _f64(x), _f64(w_router), _f64(dgate), _f64(dx_perm)
    idx = np.asarray(idx, dtype=np.int64)
    slot = np.asarray(slot, dtype=np.int64)
    T, k = idx.shape
    p = softmax(logits)
    dp = np.zeros_like(p)
    for j in range(k):
        dp[np.arange(T), idx[:, j]] = dgate[:, j]
    dl = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    dx = np.zeros_like(x)
    for j in range(k):
        dx += dx_perm[slot[:, j]]
    dx = dx + dl @ w_router
    dw_router = dl.T @ x
    return dx, dw_router, dl


def layer_fwd_bwd(x, w_router, w1, w2, dout, k: int, bias=None,
                  select_logits=None, renorm: bool = False) -> dict:
    """One forward + backward pass of the whole layer, all intermediates.

    route -> permute -> grouped SwiGLU FFN -> combine; then combine-grad ->
    grouped dgrad/wgrad -> unpermute-grad + router grad.  ``select_logits``
    is passed to ``route`` (see ``route_from_logits``).  With ``renorm`` the
    combine takes ``renorm_gates`` of the gates; ``dgate_rn`` is then the
    combine's gate gradient and ``dgate`` its image under ``renorm_gates_bwd``.
    """
    r = route(x, w_router, k, bias, select_logits)
    x_perm = permute(x, r["slot_row"])
    a, u, h, y_perm = expert_ffn_fwd(x_perm, r["offsets"], w1, w2)
    gate = renorm_gates(r["gate"]) if renorm else r["gate"]
    out = combine(y_perm, r["slot_row"], gate)
    dgate_c, dy_perm = combine_bwd(dout, y_perm, r["slot_row"], gate)
    dgate = renorm_gates_bwd(r["gate"], dgate_c) if renorm else dgate_c
    dx_perm, dw1, dw2 = expert_ffn_bwd(dy_perm, x_perm, a, u, h, r["offsets"], w1, w2)
    dx, dw_router, dl = route_bwd(x, w_router, r["logits"], r["idx"], dgate, dx_perm,
                                  r["slot_row"])
    r.update(x_perm=x_perm, a=a, u=u, h=h, y_perm=y_perm, out=out, dgate=dgate,
             gate_rn=gate, dgate_rn=dgate_c,
             dy_perm=dy_perm, dx_perm=dx_perm, dw1=dw1, dw2=dw2, dx=dx,
             dw_router=dw_router, dl=dl)
    return r


# --------------------------------------------------------------------------
# Padded-capacity comparison (uniform per-expert capacity, overflow dropped)
# --------------------------------------------------------------------------

def capacity(R: int, E: int, cf_num: int = 5, cf_den: int = 4) -> int:
    """``C = ceil(cf * R / E)`` with cf = cf_num / cf_den (default 1.25), exactly.

    kongchang, section 路由不只是模型问题，更是系统问题: the report measured the
    device-scheduled grouped GEMM against padding every expert's batch to one
    uniform capacity.  Reading: capacity factor times the mean load, rounded up.
    """
    return -((-cf_num * R) // (cf_den * E))


def padded_layout(idx, slot, offsets, C: int):
    """Row of the padded buffer [E * C, d] for each (t, j), or -1 if dropped.

    A pair is kept iff its rank inside its expert's segment (token order) is
    below C; kept pairs go to row ``e * C + rank``.
    """
    idx = np.asarray(idx, dtype=np.int64)
    slot = np.asarray(slot, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    rank = slot - offsets[idx]
    return np.where(rank < C, idx * C + rank, -1)


def padded_layer_fwd_bwd(x, w_router, w1, w2, dout, k: int, C: int, bias=None,
                         select_logits=None, renorm: bool = False) -> dict:
    """Forward + backward of the layer on the padded-capacity layout.

    Dropped pairs contribute nothing to ``out`` and get zero gradient; the gates
    are not renormalised after the drop (with ``renorm`` they are renormalised
    over all k selected experts before it).  Unused padded rows are zero, so
    they produce zero expert outputs and zero weight gradients.
    """
    x = _f64(x)
    r = route(x, w_router, k, bias, select_logits)
    E = w1.shape[0]
    T, d = x.shape
    prow = padded_layout(r["idx"], r["slot_row"], r["offsets"], C)
    keep = prow >= 0
    x_pad = np.zeros((E * C, d))
    for j in range(k):
        x_pad[prow[keep[:, j], j]] = x[keep[:, j]]
    offs_pad = np.arange(E + 1, dtype=np.int64) * C
    a, u, h, y_pad = expert_ffn_fwd(x_pad, offs_pad, w1, w2)
    out = np.zeros((T, d))
    dgate = np.zeros((T, k))
    dy_pad = np.zeros_like(y_pad)
    gate = renorm_gates(r["gate"]) if renorm else r["gate"]
    dout = _f64(dout)
    for j in range(k):
        kj = keep[:, j]
        rows = prow[kj, j]
        out[kj] += gate[kj, j:j + 1] * y_pad[rows]
        dgate[kj, j] = np.sum(dout[kj] * y_pad[rows], axis=1)
        dy_pad[rows] = gate[kj, j:j + 1] * dout[kj]
    dx_pad, dw1, dw2 = expert_ffn_bwd(dy_pad, x_pad, a, u, h, offs_pad, w1, w2)
    dx_perm_like = np.zeros((T * k, d))
    # Route the padded row gradients back through the dropless slots so that
    # route_bwd can sum them; dropped pairs keep a zero row.
    for j in range(k):
        kj = keep[:, j]
        dx_perm_like[r["slot_row"][kj, j]] = dx_pad[prow[kj, j]]
    dgate_c = dgate
    if renorm:
        dgate = renorm_gates_bwd(r["gate"], dgate_c)
    dx, dw_router, dl = route_bwd(x, w_router, r["logits"], r["idx"], dgate,
                                  dx_perm_like, r["slot_row"])
    r.update(C=C, pad_row=prow, x_pad=x_pad, a=a, u=u, h=h, y_pad=y_pad, out=out,
             dgate=dgate, gate_rn=gate, dgate_rn=dgate_c, dy_pad=dy_pad, dx_pad=dx_pad, dw1=dw1, dw2=dw2, dx=dx,
             dw_router=dw_router, dl=dl)
    return r


# --------------------------------------------------------------------------
# Load balance of a routing (kongchang, routing section: balancing the load, not the loss
# value, is what matters for throughput)
# --------------------------------------------------------------------------

ROUTING_STATS = ("rows", "mean", "max_over_mean", "min_over_mean", "cv", "empty",
                 "dropped_frac", "capacity_use")


def routing_stats(counts, C: int = 0) -> np.ndarray:
    """Load statistics of the per-expert row counts ``c`` (R = sum c, E experts):

    rows R; mean R / E; max(c) / mean; min(c) / mean; coefficient of variation
    std(c) / mean (population std); number of empty experts; and for a capacity C > 0
    the fraction of the R rows a capacity-C layout drops, sum max(0, c - C) / R, and the
    fraction of its E * C slots that hold a row, (R - dropped) / (E C).  Ratios are 0
    when R = 0; the capacity entries are 0 when C = 0.
    """
    c = np.asarray(counts, dtype=np.float64)
    E = c.size
    R = c.sum()
    mean = R / E
    out = np.zeros(8)
    out[0], out[1] = R, mean
    if R > 0:
        out[2] = c.max() / mean
        out[3] = c.min() / mean
        out[4] = np.sqrt(np.mean((c - mean) ** 2)) / mean
    out[5] = float(np.sum(c == 0))
    if C > 0 and R > 0:
        dropped = np.maximum(c - C, 0).sum()
        out[6] = dropped / R
        out[7] = (R - dropped) / (E * C)
    return out
