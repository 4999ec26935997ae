"""Pins of the oracle's expert FFN, combine and backward pass.

Checks: identity experts give the closed form (sum of selected gates) * x;
top_k = E gives the dense softmax mixture computed with torch float64 ops;
SwiGLU matches torch's silu; every gradient matches central finite
differences in float64 and torch.autograd; the padded layout equals the
dropless layer when nothing is dropped.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_ref as ref


def _tiny(seed=0, T=6, d=8, E=4, k=2, f=4, bias=False):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, d))
    wr = rng.normal(size=(E, d)) * 0.7
    b = rng.normal(size=E) if bias else None
    w1 = rng.normal(size=(E, 2 * f, d)) * 0.5
    w2 = rng.normal(size=(E, d, f)) * 0.5
    dout = rng.normal(size=(T, d))
    return x, wr, b, w1, w2, dout


def _min_gap(x, wr, b, k):
    l = ref.router_logits(x, wr, b)
    s = np.sort(l, axis=1)[:, ::-1]
    return np.min(s[:, k - 1] - s[:, k]) if k < l.shape[1] else np.inf


def test_identity_experts_give_selected_gate_sum_times_x():
    rng = np.random.default_rng(1)
    T, d, E, k = 40, 5, 7, 3
    x = rng.normal(size=(T, d))
    r = ref.route(x, rng.normal(size=(E, d)), k)
    out = ref.combine(ref.permute(x, r["slot_row"]), r["slot_row"], r["gate"])
    p_sorted = np.sort(ref.softmax(r["logits"]), axis=1)[:, ::-1]
    np.testing.assert_allclose(out, p_sorted[:, :k].sum(1, keepdims=True) * x, rtol=1e-13)


def test_top_k_equal_E_is_dense_softmax_mixture():
    x, wr, _, w1, w2, _ = _tiny(seed=2, T=9, E=3, k=3)
    E, f = w1.shape[0], w1.shape[1] // 2
    r = ref.route(x, wr, E)
    a, u, h, y = ref.expert_ffn_fwd(ref.permute(x, r["slot_row"]), r["offsets"], w1, w2)
    out = ref.combine(y, r["slot_row"], r["gate"])
    X, W1, W2 = (torch.tensor(v, dtype=torch.float64) for v in (x, w1, w2))
    P = torch.softmax(X @ torch.tensor(wr).T, dim=1)
    A = torch.einsum("td,efd->etf", X, W1[:, :f])
    U = torch.einsum("td,efd->etf", X, W1[:, f:])
    Y = torch.einsum("etf,edf->etd", F.silu(A) * U, W2)
    dense = torch.einsum("te,etd->td", P, Y)
    np.testing.assert_allclose(out, dense.numpy(), rtol=1e-12, atol=1e-13)


def test_swiglu_matches_torch_silu():
    rng = np.random.default_rng(4)
    a = rng.normal(size=(64, 16)) * 6
    np.testing.assert_allclose(ref.silu(a), F.silu(torch.tensor(a)).numpy(), rtol=1e-14, atol=1e-300)
    big = np.array([-800.0, -40.0, 0.0, 40.0, 800.0])
    assert np.all(np.isfinite(ref.silu(big)))


def _loss(params, k, bias):
    x, wr, w1, w2, dout = params
    r = ref.route(x, wr, k, bias)
    _, _, _, y = ref.expert_ffn_fwd(ref.permute(x, r["slot_row"]), r["offsets"], w1, w2)
    return float(np.sum(ref.combine(y, r["slot_row"], r["gate"]) * dout))


@pytest.mark.parametrize("bias", [False, True])
def test_gradients_match_finite_differences(bias):
    x, wr, b, w1, w2, dout = _tiny(seed=11, bias=bias)
    k = 2
    assert _min_gap(x, wr, b, k) > 1e-3, "pick a seed away from routing ties"
    res = ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, b)
    params = [x, wr, w1, w2, dout]
    grads = {0: res["dx"], 1: res["dw_router"], 2: res["dw1"], 3: res["dw2"]}
    eps = 1e-6
    for pi, g in grads.items():
        fd = np.zeros_like(params[pi])
        it = np.nditer(params[pi], flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            orig = params[pi][ix]
            params[pi][ix] = orig + eps
            lp = _loss(params, k, b)
            params[pi][ix] = orig - eps
            lm = _loss(params, k, b)
            params[pi][ix] = orig
            fd[ix] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert err < 1e-6, (pi, err)


def test_gradients_match_torch_autograd():
    """Second opinion on the backward formulas: autograd of a gather form of
    the forward with the oracle's (constant) routing decisions."""
    x, wr, b, w1, w2, dout = _tiny(seed=5, T=10, d=6, E=5, k=3, f=3, bias=True)
    k, f = 3, 3
    res = ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, b)
    X, WR, W1, W2 = (torch.tensor(v, dtype=torch.float64, requires_grad=True) for v in (x, wr, w1, w2))
    idx = torch.tensor(res["idx"])
    P = torch.softmax(X @ WR.T + torch.tensor(b), dim=1)
    out = torch.zeros_like(X)
    for j in range(k):
        e = idx[:, j]
        A = torch.einsum("td,tfd->tf", X, W1[e, :f])
        U = torch.einsum("td,tfd->tf", X, W1[e, f:])
        Y = torch.einsum("tf,tdf->td", F.silu(A) * U, W2[e])
        out = out + P.gather(1, e[:, None]) * Y
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(res["out"], out.detach().numpy(), rtol=1e-12, atol=1e-13)
    for mine, t in ((res["dx"], X), (res["dw_router"], WR), (res["dw1"], W1), (res["dw2"], W2)):
        np.testing.assert_allclose(mine, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_empty_expert_has_zero_weight_grads():
    x, wr, _, w1, w2, dout = _tiny(seed=3, T=12, E=5)
    b = np.array([0, 0, 0, 0, -1e3])  # expert 4 never wins
    res = ref.layer_fwd_bwd(x, wr, w1, w2, dout, 2, b)
    assert res["counts"][4] == 0
    assert np.all(res["dw1"][4] == 0) and np.all(res["dw2"][4] == 0)


def test_capacity_rounds_up_exactly():
    assert ref.capacity(10, 4) == 4            # 12.5 / 4 = 3.125
    assert ref.capacity(16, 4) == 5            # exactly 5
    assert ref.capacity(131072, 128) == 1280   # 32768 tokens x top-4 over 128 experts
    assert ref.capacity(7, 7, 1, 1) == 1


def test_padded_equals_dropless_when_nothing_drops():
    x, wr, b, w1, w2, dout = _tiny(seed=7, T=10, E=4, k=2, bias=True)
    full = ref.layer_fwd_bwd(x, wr, w1, w2, dout, 2, b)
    C = int(full["counts"].max())
    pad = ref.padded_layer_fwd_bwd(x, wr, w1, w2, dout, 2, C, b)
    for key in ("out", "dgate", "dx", "dw1", "dw2", "dw_router"):
        np.testing.assert_allclose(pad[key], full[key], rtol=1e-12, atol=1e-14, err_msg=key)


def test_padded_drops_overflow_in_token_order():
    x, wr, b, w1, w2, dout = _tiny(seed=8, T=14, E=4, k=2)
    b = np.array([3.0, 0, 0, 0])  # expert 0 overflows
    pad = ref.padded_layer_fwd_bwd(x, wr, w1, w2, dout, 2, 3, b)
    f = w1.shape[1] // 2
    idx, gate = pad["idx"], pad["gate"]
    seen = np.zeros(4, dtype=int)
    for t in range(x.shape[0]):
        expect = np.zeros(x.shape[1])
        for j in range(2):
            e = idx[t, j]
            if seen[e] < 3:
                a = w1[e, :f] @ x[t]
                u = w1[e, f:] @ x[t]
                expect += gate[t, j] * (w2[e] @ (ref.silu(a) * u))
                assert pad["pad_row"][t, j] == e * 3 + seen[e]
            else:
                assert pad["pad_row"][t, j] == -1 and pad["dgate"][t, j] == 0
            seen[e] += 1
        np.testing.assert_allclose(pad["out"][t], expect, rtol=1e-12, atol=1e-14)
    assert seen[0] > 3


def test_padded_gradients_match_finite_differences():
    x, wr, _, w1, w2, dout = _tiny(seed=12, T=8, E=4, k=2)
    b = np.array([2.0, 0, 0, 0])
    C = 3
    assert _min_gap(x, wr, b, 2) > 1e-3
    res = ref.padded_layer_fwd_bwd(x, wr, w1, w2, dout, 2, C, b)
    assert np.any(res["pad_row"] < 0)

    def loss(xx, ww1):
        return float(np.sum(ref.padded_layer_fwd_bwd(xx, wr, ww1, w2, dout, 2, C, b)["out"] * dout))

    eps = 1e-6
    for arr, g in ((x, res["dx"]), (w1, res["dw1"])):
        fd = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            o = arr[ix]
            arr[ix] = o + eps
            lp = loss(x, w1)
            arr[ix] = o - eps
            lm = loss(x, w1)
            arr[ix] = o
            fd[ix] = (lp - lm) / (2 * eps)
        assert np.linalg.norm(fd - g) / np.linalg.norm(g) < 1e-6


# ---- renormalised gates (optional gate rule) --------------------------------

def _softmax_of_selected(l, idx):
    """Gates as a softmax over the k selected logits only, written out directly."""
    sel = np.take_along_axis(l, idx, axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def test_renorm_gates_are_a_softmax_over_the_selected_logits():
    x, wr, b, *_ = _tiny(seed=4, T=20, E=6, bias=True)
    r = ref.route(x, wr, 3, b)
    got = ref.renorm_gates(r["gate"])
    assert np.allclose(got, _softmax_of_selected(r["logits"], r["idx"]), rtol=1e-14, atol=0)
    assert np.allclose(got.sum(axis=1), 1.0, rtol=1e-15)


def _loss_renorm(params, k, bias):
    x, wr, w1, w2, dout = params
    r = ref.route(x, wr, k, bias)
    _, _, _, y = ref.expert_ffn_fwd(ref.permute(x, r["slot_row"]), r["offsets"], w1, w2)
    g = _softmax_of_selected(r["logits"], r["idx"])
    return float(np.sum(ref.combine(y, r["slot_row"], g) * dout))


def test_renorm_gradients_match_finite_differences():
    x, wr, b, w1, w2, dout = _tiny(seed=11, bias=True)
    k = 2
    assert _min_gap(x, wr, b, k) > 1e-3
    res = ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, b, renorm=True)
    assert np.allclose(res["out"].sum(), _loss_renorm([x, wr, w1, w2, np.ones_like(dout)], k, b))
    params = [x, wr, w1, w2, dout]
    eps = 1e-6
    for pi, g in {0: res["dx"], 1: res["dw_router"]}.items():
        fd = np.zeros_like(params[pi])
        it = np.nditer(params[pi], flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            orig = params[pi][ix]
            params[pi][ix] = orig + eps
            lp = _loss_renorm(params, k, b)
            params[pi][ix] = orig - eps
            lm = _loss_renorm(params, k, b)
            params[pi][ix] = orig
            fd[ix] = (lp - lm) / (2 * eps)
        err = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert err < 1e-6, (pi, err)
    # the renormalised gates change the router gradient (the option is not a no-op)
    plain = ref.layer_fwd_bwd(x, wr, w1, w2, dout, k, b)
    assert np.linalg.norm(plain["dw_router"] - res["dw_router"]) > 1e-3 * np.linalg.norm(plain["dw_router"])


def test_renorm_changes_nothing_when_top_k_equals_E():
    # all experts selected: the softmax values already sum to one
    x, wr, b, w1, w2, dout = _tiny(seed=5, E=4)
    a = ref.layer_fwd_bwd(x, wr, w1, w2, dout, 4, b)
    r = ref.layer_fwd_bwd(x, wr, w1, w2, dout, 4, b, renorm=True)
    for key in ("out", "dx", "dw_router", "dw1", "dw2"):
        assert np.allclose(a[key], r[key], rtol=1e-12, atol=1e-13), key


def test_padded_renorm_equals_dropless_renorm_when_nothing_drops():
    x, wr, b, w1, w2, dout = _tiny(seed=6, T=10, E=4, bias=True)
    full = ref.layer_fwd_bwd(x, wr, w1, w2, dout, 2, b, renorm=True)
    pad = ref.padded_layer_fwd_bwd(x, wr, w1, w2, dout, 2, 20, b, renorm=True)
    for key in ("out", "dgate", "dx", "dw_router", "dw1", "dw2"):
        assert np.allclose(full[key], pad[key], rtol=1e-12, atol=1e-13), key
