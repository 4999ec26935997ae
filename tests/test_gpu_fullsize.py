"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (one MoELayer fwd+bwd step).

The oracle cannot redo a whole 16k-32k-token layer in float64 within
seconds, so these tests check (a) every discrete output for all tokens
(top-k on the device's logits, counts, offsets, slot rows, the permutation,
the padded layout), (b) sampled tokens, whose outputs and input gradients
depend on that token alone, recomputed by the oracle one by one, and (c) the
weight gradients of sampled experts, recomputed by the oracle from that
expert's own rows.
"""

import warnings

import numpy as np
import pytest
import torch

from gpu_helpers import TOL, f64, i64, rel, routing_divergence
from mixture_experts_layer_offsets_b200 import inputs
from mixture_experts_layer_offsets_b200.layer import MoELayer
from oracle import moe_ref as ref

pytestmark = pytest.mark.gpu

N_TOKENS = 24


class RoutingDivergence(UserWarning):
    """Report (shown in pytest's warnings summary): tokens whose routing on the oracle's
    own float64 logits differs from the device routing (allowed only at near ties)."""
N_EXPERTS = 2


def _run(cfg, capacity=None):
    inp = inputs.make_inputs(cfg, device="cuda", seed=0)
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                 capacity=capacity)
    L.step(inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w2"], inp["dout"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return inp, L


def _token_oracle(t, inp, L, wr, bias):
    """Oracle forward/backward of token t alone (its routing taken on the device logits)."""
    k, f = L.k, L.f
    x = f64(inp["x"][t:t + 1])
    dout = f64(inp["dout"][t:t + 1])
    logits = ref.router_logits(x, wr, bias)
    r = ref.route_from_logits(logits, k, select_logits=f64(L.logits[t:t + 1]))
    y = np.zeros((k, x.shape[1]))
    dxp = np.zeros_like(y)
    for j in range(k):
        e = int(r["idx"][0, j])
        w1 = f64(inp["w1"][e:e + 1])
        w2 = f64(inp["w2"][e:e + 1])
        a, u, h, yj = ref.expert_ffn_fwd(x, [0, 1], w1, w2)
        y[j] = yj[0]
        dy = r["gate"][0, j] * dout
        dxj, _, _ = ref.expert_ffn_bwd(dy, x, a, u, h, [0, 1], w1, w2)
        dxp[j] = dxj[0]
    slot = np.arange(k)[None, :]
    out = ref.combine(y, slot, r["gate"])
    dgate, _ = ref.combine_bwd(dout, y, slot, r["gate"])
    dx, _, _ = ref.route_bwd(x, wr, logits, r["idx"], dgate, dxp, slot)
    return out[0], dgate[0], dx[0]


def _check_discrete(L, inp):
    o = ref.route_from_logits(f64(L.logits), L.k)
    assert np.array_equal(i64(L.topk_idx), o["idx"])
    assert np.array_equal(i64(L.counts), o["counts"])
    assert np.array_equal(i64(L.offsets), o["offsets"])
    assert np.array_equal(i64(L.slot_row), o["slot_row"])
    n, worst = routing_divergence(L, inp)
    warnings.warn(RoutingDivergence(
        f"{L.T} tokens, E={L.E}, k={L.k}: {n} route differently on the oracle's own float64 "
        f"logits (largest near-tie gap among them: {worst:.3g} of max|l|)"))
    return o


def _check_tokens(cfg, inp, L, rows_out):
    rng = np.random.default_rng(1)
    toks = rng.choice(cfg.T, size=N_TOKENS, replace=False)
    wr = f64(inp["w_router"])
    bias = f64(inp["bias"]) if inp["bias"] is not None else None
    got, want = {"out": [], "dgate": [], "dx": []}, {"out": [], "dgate": [], "dx": []}
    for t in toks:
        o, dg, dx = _token_oracle(int(t), inp, L, wr, bias)
        want["out"].append(o), want["dgate"].append(dg), want["dx"].append(dx)
        got["out"].append(f64(rows_out["out"][t])), got["dgate"].append(f64(L.dgate[t]))
        got["dx"].append(f64(L.dx[t]))
    # logits of the sampled tokens against the oracle's float64 logits
    lg = ref.router_logits(f64(inp["x"][torch.from_numpy(toks).cuda()]), wr, bias)
    assert rel(f64(L.logits[torch.from_numpy(toks).cuda()]), lg) <= TOL[cfg.dtype]
    for key in got:
        assert rel(np.stack(got[key]), np.stack(want[key])) <= TOL[cfg.dtype], key


@pytest.mark.parametrize("name", ["bf16_e8", "bf16_e128", "bf16_skew_e128"])
def test_fullsize_dropless(name):
    cfg = inputs.CONFIGS[name]
    inp, L = _run(cfg)
    o = _check_discrete(L, inp)
    R = cfg.R
    assert np.array_equal(i64(L.perm_src[:R]), o["perm_src"])
    assert torch.equal(L.x_perm[:R], inp["x"][L.perm_src[:R].long()])
    _check_tokens(cfg, inp, L, {"out": L.out})
    # weight gradients of sampled non-empty experts, each recomputed in float64 from all
    # of its rows (about 8k rows per expert at E = 8: the K accumulation the bench runs)
    rng = np.random.default_rng(2)
    nonempty = np.nonzero(o["counts"] > 0)[0]
    n_experts = N_EXPERTS if cfg.E >= 64 else 1
    wr = f64(inp["w_router"])
    bias = f64(inp["bias"]) if inp["bias"] is not None else None
    f = cfg.d_ff
    for e in rng.choice(nonempty, size=min(n_experts, len(nonempty)), replace=False):
        r0, r1 = int(o["offsets"][e]), int(o["offsets"][e + 1])
        toks = torch.from_numpy(o["perm_src"][r0:r1]).cuda()
        x = f64(inp["x"][toks])
        p = ref.softmax(ref.router_logits(x, wr, bias))
        dy = p[:, e:e + 1] * f64(inp["dout"][toks])
        w1 = f64(inp["w1"][e:e + 1])
        w2 = f64(inp["w2"][e:e + 1])
        off = [0, r1 - r0]
        a, u, h, _ = ref.expert_ffn_fwd(x, off, w1, w2)
        _, dw1, dw2 = ref.expert_ffn_bwd(dy, x, a, u, h, off, w1, w2)
        assert rel(f64(L.dw1[e]), dw1[0]) <= TOL[cfg.dtype]
        assert rel(f64(L.dw2[e]), dw2[0]) <= TOL[cfg.dtype]
    for e in np.nonzero(o["counts"] == 0)[0]:
        assert not L.dw1[e].any() and not L.dw2[e].any()


def test_fullsize_skewed_padded():
    cfg = inputs.CONFIGS["bf16_skew_e128"]
    C = ref.capacity(cfg.R, cfg.E, *cfg.padded_cf)
    inp, L = _run(cfg, capacity=C)
    o = _check_discrete(L, inp)
    prow = ref.padded_layout(o["idx"], o["slot_row"], o["offsets"], C)
    assert np.array_equal(i64(L.pad_row), prow)
    assert (prow < 0).sum() > 0, "the skewed workload must overflow some experts"
    # sampled tokens: the kept pairs only
    rng = np.random.default_rng(3)
    toks = rng.choice(cfg.T, size=N_TOKENS, replace=False)
    wr = f64(inp["w_router"])
    bias = f64(inp["bias"])
    k, f = cfg.top_k, cfg.d_ff
    for t in (int(v) for v in toks):
        x = f64(inp["x"][t:t + 1])
        p = ref.softmax(ref.router_logits(x, wr, bias))[0]
        want = np.zeros(cfg.d_model)
        for j in range(k):
            if prow[t, j] < 0:
                assert L.dgate[t, j].item() == 0.0
                continue
            e = int(o["idx"][t, j])
            _, _, _, y = ref.expert_ffn_fwd(x, [0, 1], f64(inp["w1"][e:e + 1]), f64(inp["w2"][e:e + 1]))
            want += p[e] * y[0]
        assert rel(f64(L.out[t]), want) <= TOL[cfg.dtype]


def test_fullsize_mxfp8_sampled_expert():
    """mxfp8_e128 at full size (fused dispatch, CTA pairs): every discrete output for all
    tokens, then one sampled expert end to end from its own rows (its row-wise operand
    blocks and its token blocks depend on nothing else): a, u, h, y_perm, dx_perm and its
    weight gradients against the MXFP8 oracle."""
    from oracle import moe_mx_ref as mxr
    cfg = inputs.CONFIGS["mxfp8_e128"]
    inp, L = _run(cfg)
    o = _check_discrete(L, inp)
    rng = np.random.default_rng(3)
    e = int(rng.choice(np.nonzero(o["counts"] > 0)[0]))
    r0, r1 = int(o["offsets"][e]), int(o["offsets"][e + 1])
    toks = torch.from_numpy(o["perm_src"][r0:r1]).cuda()
    wr = f64(inp["w_router"])
    bias = f64(inp["bias"]) if inp["bias"] is not None else None
    x = f64(inp["x"][toks])
    p = ref.softmax(ref.router_logits(x, wr, bias))
    dy = p[:, e:e + 1] * f64(inp["dout"][toks])
    w1 = f64(inp["w1"][e:e + 1])
    w2 = f64(inp["w2"][e:e + 1])
    off = [0, r1 - r0]
    a, u, h, y = mxr.expert_ffn_fwd_mx(x, off, w1, w2, act_round=mxr.round_bf16)
    dxp, dw1, dw2 = mxr.expert_ffn_bwd_mx(dy, x, a, u, h, off, w1, w2, act_round=mxr.round_bf16)
    f = cfg.d_ff
    act = f64(L.act[r0:r1])
    tol = TOL["mxfp8"]
    checks = {"a": (act[:, :f], a), "u": (act[:, f:2 * f], u), "h": (act[:, 2 * f:], h),
              "y_perm": (f64(L.y_perm[r0:r1]), y), "dx_perm": (f64(L.dx_perm[r0:r1]), dxp),
              "dw1": (f64(L.dw1[e]), dw1[0]), "dw2": (f64(L.dw2[e]), dw2[0])}
    errs = {k: rel(g, w) for k, (g, w) in checks.items()}
    assert all(v <= tol for v in errs.values()), (e, r1 - r0, errs)
