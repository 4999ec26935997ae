"""Pins of the expert-parallel oracle (oracle/moe_ep_ref.py).

Expert parallelism moves rows between ranks but must not change what is computed:
with the global token order (rank, token), every owner's receive buffer must hold
exactly the rows that one device permutes for the owner's experts from the
concatenated batch, and every output and gradient must equal the single-device
oracle's (moe_ref.layer_fwd_bwd, itself pinned by brute force, closed forms and
finite differences).  Also checked: the row map is a bijection onto each owner's
buffer, rows come in (source rank, token) order inside each expert, and ranks that
send nothing or experts that receive nothing are handled.
"""

import numpy as np
import pytest
import torch

from mixture_experts_layer_offsets_b200.inputs import CONFIGS, make_inputs, shrink
from oracle import moe_ep_ref as ep
from oracle import moe_ref as ref


def _f64(t):
    return None if t is None else t.double().numpy()


def _ranks(cfg, N):
    w = make_inputs(cfg, seed=100)
    shards = [make_inputs(cfg, seed=s) for s in range(N)]
    return w, [_f64(s["x"]) for s in shards], [_f64(s["dout"]) for s in shards]


CASES = [
    (shrink(CONFIGS["tiny_f32"], name="ep2", T=20, d_model=16, E=4, top_k=2, d_ff=8,
            router_std=0.3), 2),
    (shrink(CONFIGS["tiny_f32"], name="ep3", T=13, d_model=16, E=6, top_k=3, d_ff=8,
            router_std=0.3), 3),
    (shrink(CONFIGS["tiny_f32"], name="ep4", T=9, d_model=16, E=8, top_k=2, d_ff=8,
            router_std=0.3), 4),
    # skewed: a logit bias sends nearly everything to a few experts, leaving owners and
    # (source, owner) pairs with no rows
    (shrink(CONFIGS["tiny_f32"], name="ep_skew", T=7, d_model=16, E=8, top_k=2, d_ff=8,
            router_std=0.05, bias_std=4.0), 4),
    # one rank: the single-device layer itself
    (shrink(CONFIGS["tiny_f32"], name="ep1", T=11, d_model=16, E=4, top_k=2, d_ff=8,
            router_std=0.3), 1),
]


@pytest.mark.parametrize("cfg,N", CASES, ids=[c[0].name for c in CASES])
def test_expert_parallel_layer_equals_the_single_device_layer(cfg, N):
    w, xs, douts = _ranks(cfg, N)
    bias = _f64(w["bias"])
    wr, w1, w2 = _f64(w["w_router"]), _f64(w["w1"]), _f64(w["w2"])
    got = ep.ep_layer_fwd_bwd(xs, wr, w1, w2, douts, cfg.top_k, bias)
    full = ref.layer_fwd_bwd(np.concatenate(xs), wr, w1, w2, np.concatenate(douts), cfg.top_k,
                             bias)
    T, E, El = cfg.T, cfg.E, cfg.E // N
    for s in range(N):
        sl = slice(s * T, (s + 1) * T)
        assert np.array_equal(got["idx"][s], full["idx"][sl])
        for key in ("out", "dgate", "dx"):
            np.testing.assert_allclose(got[key][s], full[key][sl], rtol=1e-12, atol=1e-14,
                                       err_msg=key)
    for o in range(N):
        e0, e1 = o * El, (o + 1) * El
        r0, r1 = full["offsets"][e0], full["offsets"][e1]
        # the owner's buffer is the single-device permutation of its experts' rows
        assert np.array_equal(got["recv_offsets"][o], full["offsets"][e0:e1 + 1] - r0)
        assert np.array_equal(got["x_recv"][o], full["x_perm"][r0:r1])
        np.testing.assert_allclose(got["y_recv"][o], full["y_perm"][r0:r1], rtol=1e-12,
                                   atol=1e-14)
        np.testing.assert_allclose(got["dx_recv"][o], full["dx_perm"][r0:r1], rtol=1e-12,
                                   atol=1e-14)
        np.testing.assert_allclose(got["dw1"][o], full["dw1"][e0:e1], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(got["dw2"][o], full["dw2"][e0:e1], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(got["dw_router"], full["dw_router"], rtol=1e-12, atol=1e-14)
    if cfg.name == "ep_skew":
        ca = got["counts_all"]
        sent = np.stack([ca[:, o * El:(o + 1) * El].sum(axis=1) for o in range(N)], axis=1)
        assert (sent == 0).any(), "the skewed case must leave some (source, owner) pair empty"


@pytest.mark.parametrize("seed", range(5))
def test_row_map_is_a_bijection_in_source_then_token_order(seed):
    rng = np.random.default_rng(seed)
    N, E, k, T = 4, 8, 3, 17
    idxs = [np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) for _ in range(N)]
    counts_all = np.stack([np.bincount(i.ravel(), minlength=E) for i in idxs])
    El = E // N
    for o in range(N):
        off = ep.ep_recv_offsets(counts_all, o)
        seen = []
        for s in range(N):
            rows = ep.ep_rows(idxs[s], counts_all, s)
            own = ep.ep_owner(idxs[s], E, N)
            for t in range(T):
                for j in range(k):
                    if own[t, j] != o:
                        continue
                    e = idxs[s][t, j] - o * El
                    r = rows[t, j]
                    assert off[e] <= r < off[e + 1]      # inside its expert's segment
                    seen.append((r, e, s, t))
        seen.sort()
        assert [r for r, *_ in seen] == list(range(off[-1]))   # a bijection onto the buffer
        # inside each expert: source rank, then token order
        for e in range(El):
            order = [(s, t) for r, ee, s, t in seen if ee == e]
            assert order == sorted(order)


def test_layout_of_hand_counts():
    # 2 ranks, 4 experts (rank 0 owns 0-1, rank 1 owns 2-3)
    counts_all = np.array([[1, 0, 2, 3],
                           [4, 5, 0, 1]])
    assert ep.ep_recv_offsets(counts_all, 0).tolist() == [0, 5, 10]
    assert ep.ep_recv_offsets(counts_all, 1).tolist() == [0, 2, 6]
    assert ep.ep_send_base(counts_all, 0).tolist() == [0, 5, 0, 2]
    assert ep.ep_send_base(counts_all, 1).tolist() == [1, 5, 2, 5]
    with pytest.raises(ValueError):
        ep.ep_owner(3, 6, 4)
