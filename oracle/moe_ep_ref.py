"""Float64 oracle of the layer under expert parallelism across N ranks.

TEST INFRASTRUCTURE ONLY (see the package docstring).

kongchang, section 容量税 (capacity tax): expert parallelism spreads the routed
experts over the ranks and writes only the selected token rows directly into the
target rank's buffer (over NVSHMEM on the pages' system); section
路由不只是模型问题，更是系统问题: the split sizes of that exchange stay on the
device.  aizyradar (glossary on NVSHMEM): the kernels read and write the remote
GPU's memory directly, with no host round trip and no explicit all-to-all.
bytechap, "Cách thức hoạt động": each device stores only a fraction of the
experts, and rowwise expert parallelism places the routed rows directly in the
experts' input buffers.

The pages fix no layout.  Readings taken here (the plainest that these passages
support):

* ranks hold equal contiguous blocks of experts: with E_loc = E / N, rank o owns
  experts [o * E_loc, (o + 1) * E_loc);
* every rank routes its own T tokens with the replicated router over all E
  experts; the global token order is (rank, token), i.e. the ranks' batches
  concatenated;
* an owner's receive buffer holds its experts' rows expert by expert, within an
  expert by source rank, within a source in token order: exactly the rows that a
  single device would permute for those experts from the concatenated batch,
  in the same order;
* the owner runs its experts on its rows; the source rank reads the expert
  outputs of its pairs back from the owners (the combine), writes the gate-
  weighted output gradient into the owners' buffers, and after the owners' expert
  backward reads the input-gradient rows back; expert-weight gradients stay with
  their owner; the router is replicated, so its gradient is summed over ranks.

Under these readings expert parallelism changes where rows live, never what is
computed: ``ep_layer_fwd_bwd`` equals ``moe_ref.layer_fwd_bwd`` of the
concatenated batch, which is its pin.
"""

from __future__ import annotations

import numpy as np

from .moe_ref import (_f64, combine, combine_bwd, expert_ffn_bwd, expert_ffn_fwd, route,
                      route_bwd)

__all__ = ["ep_owner", "ep_recv_offsets", "ep_send_base", "ep_rows", "ep_dispatch",
           "ep_layer_fwd_bwd"]


def ep_owner(e, E: int, N: int):
    """Rank that owns expert e (equal contiguous blocks of E / N experts)."""
    if E % N:
        raise ValueError("E must be a multiple of the number of ranks")
    return np.asarray(e) // (E // N)


def ep_recv_offsets(counts_all, o: int) -> np.ndarray:
    """Segment starts of owner o's receive buffer, one segment per local expert:
    segment size = the rows that all ranks send to that expert (counts_all[s, e] summed
    over the source ranks s); length E_loc + 1, the last entry = rows received."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    N, E = counts_all.shape
    El = E // N
    sizes = counts_all[:, o * El:(o + 1) * El].sum(axis=0)
    return np.concatenate([[0], np.cumsum(sizes)])


def ep_send_base(counts_all, s: int) -> np.ndarray:
    """For every expert e: the first row, in the receive buffer of e's owner, of the rows
    that source rank s sends to e (after the rows of the ranks before s)."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    N, E = counts_all.shape
    El = E // N
    base = np.zeros(E, dtype=np.int64)
    for e in range(E):
        o = e // El
        base[e] = ep_recv_offsets(counts_all, o)[e - o * El] + counts_all[:s, e].sum()
    return base


def ep_rows(idx, counts_all, s: int) -> np.ndarray:
    """Row of every pair (t, j) of source rank s in its expert owner's receive buffer:
    send base of the expert plus the number of earlier tokens of s that chose it."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    base = ep_send_base(counts_all, s)
    seen = np.zeros(np.asarray(counts_all).shape[1], dtype=np.int64)
    row = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            row[t, j] = base[e] + seen[e]
        for j in range(k):
            seen[idx[t, j]] += 1
    return row


def ep_dispatch(xs, idxs, counts_all):
    """Receive buffers of all owners: rows written by every source rank at ep_rows.
    Returns (list of [rows_o, d] buffers, list of per-source ep_rows)."""
    N = len(xs)
    E = np.asarray(counts_all).shape[1]
    d = _f64(xs[0]).shape[1]
    recv = [np.zeros((int(ep_recv_offsets(counts_all, o)[-1]), d)) for o in range(N)]
    rows = []
    for s in range(N):
        r = ep_rows(idxs[s], counts_all, s)
        own = ep_owner(np.asarray(idxs[s]), E, N)
        x = _f64(xs[s])
        for t in range(x.shape[0]):
            for j in range(r.shape[1]):
                recv[own[t, j]][r[t, j]] = x[t]
        rows.append(r)
    return recv, rows


def ep_layer_fwd_bwd(xs, w_router, w1, w2, douts, k: int, bias=None, select_logits=None) -> dict:
    """Forward + backward of the layer with the experts spread over N = len(xs) ranks.

    xs[s], douts[s]: rank s's tokens and output gradient.  w1 [E, 2f, d], w2 [E, d, f]:
    all experts (owner o uses w1[o E_loc:(o + 1) E_loc]).  select_logits: optional list of
    per-rank logits on which the discrete routing is taken (see route_from_logits).
    Returns per-rank lists (idx, counts, out, dgate, dx, ep_row), per-owner lists
    (recv_offsets, x_recv, y_recv, dy_recv, dx_recv, dw1, dw2) and dw_router (summed)."""
    N = len(xs)
    w1, w2 = _f64(w1), _f64(w2)
    E = w1.shape[0]
    El = E // N
    rs = [route(xs[s], w_router, k, bias, None if select_logits is None else select_logits[s])
          for s in range(N)]
    counts_all = np.stack([r["counts"] for r in rs])
    recv, rows = ep_dispatch(xs, [r["idx"] for r in rs], counts_all)
    own = [ep_owner(r["idx"], E, N) for r in rs]
    # owners: their experts on their rows
    roff, acts, ys = [], [], []
    for o in range(N):
        off = ep_recv_offsets(counts_all, o)
        a, u, h, y = expert_ffn_fwd(recv[o], off, w1[o * El:(o + 1) * El], w2[o * El:(o + 1) * El])
        roff.append(off)
        acts.append((a, u, h))
        ys.append(y)
    # sources: combine from the owners' rows, then its gradient into the owners' buffers
    dys = [np.zeros_like(ys[o]) for o in range(N)]
    outs, dgates = [], []
    for s in range(N):
        T = _f64(xs[s]).shape[0]
        # the k expert rows of each token, gathered from their owners
        yk = np.stack([np.stack([ys[own[s][t, j]][rows[s][t, j]] for j in range(k)])
                       for t in range(T)]) if T else np.zeros((0, k, w2.shape[1]))
        slot = np.arange(T * k).reshape(T, k)
        ylocal = yk.reshape(T * k, -1)
        outs.append(combine(ylocal, slot, rs[s]["gate"]))
        dg, dyl = combine_bwd(douts[s], ylocal, slot, rs[s]["gate"])
        dgates.append(dg)
        for t in range(T):
            for j in range(k):
                dys[own[s][t, j]][rows[s][t, j]] = dyl[slot[t, j]]
    dxr, dw1, dw2 = [], [], []
    for o in range(N):
        a, u, h = acts[o]
        dx_o, dw1_o, dw2_o = expert_ffn_bwd(dys[o], recv[o], a, u, h, roff[o],
                                            w1[o * El:(o + 1) * El], w2[o * El:(o + 1) * El])
        dxr.append(dx_o)
        dw1.append(dw1_o)
        dw2.append(dw2_o)
    # sources: input-gradient rows back from the owners, then the router backward
    dxs, dwr = [], None
    for s in range(N):
        T = _f64(xs[s]).shape[0]
        dxk = np.stack([np.stack([dxr[own[s][t, j]][rows[s][t, j]] for j in range(k)])
                        for t in range(T)]).reshape(T * k, -1) if T else np.zeros((0, w1.shape[2]))
        slot = np.arange(T * k).reshape(T, k)
        dx, dw_r, _ = route_bwd(xs[s], w_router, rs[s]["logits"], rs[s]["idx"], dgates[s], dxk,
                                slot)
        dxs.append(dx)
        dwr = dw_r if dwr is None else dwr + dw_r
    return dict(idx=[r["idx"] for r in rs], counts=[r["counts"] for r in rs],
                counts_all=counts_all, ep_row=rows, recv_offsets=roff, x_recv=recv, y_recv=ys,
                dy_recv=dys, dx_recv=dxr, out=outs, dgate=dgates, dx=dxs, dw1=dw1, dw2=dw2,
                dw_router=dwr)
