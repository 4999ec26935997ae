"""GPU parity of the whole layer (route -> permute -> grouped SwiGLU FFN ->
combine, and the backward of each) against the float64 oracle.

Sizes are small enough for the oracle to finish in seconds but span several
128-row tiles per expert with ragged tails, empty experts, top_k = E, a
single token, and the padded-capacity layout.  Integer outputs (indices,
counts, offsets, rows, permutation, permuted rows) must be bit-exact; values
must meet the relative Frobenius tolerance of their dtype.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (TOL, check_accumulate, check_recompute_bit_exact, f64, i64, oracle_for,
                         rel, run_layer)
from mixture_experts_layer_offsets_b200.inputs import CONFIGS, shrink
from oracle import moe_ref as ref

pytestmark = pytest.mark.gpu

CASES = {
    # the fp32 workload exactly as specified
    "tiny_f32": CONFIGS["tiny_f32"],
    # bf16, random routing; ~350 rows per expert -> 3 M tiles, ragged tail
    "bf16_e8_small": shrink(CONFIGS["bf16_e8"], name="bf16_e8_small", T=700, d_model=512, d_ff=256),
    # bf16, skewed routing with a logit bias: heavy-tailed counts, empty experts
    "bf16_skew_small": shrink(CONFIGS["bf16_skew_e128"], name="bf16_skew_small", T=600,
                              d_model=256, E=32, top_k=2, d_ff=256, router_std=1 / 16.0),
    # top_k = E: every expert sees every token (dense mixture)
    "bf16_dense": shrink(CONFIGS["bf16_e8"], name="bf16_dense", T=300, d_model=256, E=4, top_k=4,
                         d_ff=256, router_std=0.05),
    # bf16, E = 128 (tensor-core router forward and backward), two dW_r token splits
    # with ragged tails, ~80 rows per expert
    "bf16_e128_small": shrink(CONFIGS["bf16_e128"], name="bf16_e128_small", T=2600, d_model=256,
                              d_ff=256, router_std=1 / 16.0),
    # skewed routing with experts of 2300 .. 5441 rows: their weight gradients are cut
    # into 2 or 3 K ranges whose fp32 partial sums are added in order; 4 empty experts
    "bf16_skew_split": shrink(CONFIGS["bf16_skew_e128"], name="bf16_skew_split", T=8000,
                              d_model=256, E=16, top_k=2, d_ff=256, router_std=1 / 16.0,
                              bias_std=3.0),
    # a single token; fp32
    "f32_one_token": shrink(CONFIGS["tiny_f32"], name="f32_one_token", T=1, d_model=16, E=4,
                            top_k=3, d_ff=8),
    # fp32 with E = 128 (mostly empty experts)
    "f32_e128": shrink(CONFIGS["tiny_f32"], name="f32_e128", T=40, d_model=64, E=128, top_k=4,
                       d_ff=32, router_std=0.125),
}


def _check_routing(L, o):
    assert np.array_equal(i64(L.topk_idx), o["idx"])
    assert np.array_equal(i64(L.counts), o["counts"])
    assert np.array_equal(i64(L.offsets), o["offsets"])
    assert np.array_equal(i64(L.slot_row), o["slot_row"])


@pytest.mark.parametrize("name", list(CASES))
def test_layer_matches_oracle(name):
    cfg = CASES[name]
    tol = TOL[cfg.dtype]
    cpu, L = run_layer(cfg)
    o = oracle_for(cpu, L)
    _check_routing(L, o)
    R = cfg.R
    assert np.array_equal(i64(L.perm_src[:R]), o["perm_src"])
    # the permuted rows are exact copies
    assert torch.equal(L.x_perm[:R].cpu(), cpu["x"][L.perm_src[:R].long().cpu()])
    assert rel(f64(L.logits), o["logits"]) <= tol
    assert rel(f64(L.topk_gate), o["gate"]) <= tol
    f = cfg.d_ff
    act = f64(L.act[:R])
    checks = {
        "a": (act[:, :f], o["a"]), "u": (act[:, f:2 * f], o["u"]), "h": (act[:, 2 * f:], o["h"]),
        "y_perm": (f64(L.y_perm[:R]), o["y_perm"]), "out": (f64(L.out), o["out"]),
        "dgate": (f64(L.dgate), o["dgate"]), "dy_perm": (f64(L.dy_perm[:R]), o["dy_perm"]),
        "dx_perm": (f64(L.dx_perm[:R]), o["dx_perm"]), "dw1": (f64(L.dw1), o["dw1"]),
        "dw2": (f64(L.dw2), o["dw2"]), "dx": (f64(L.dx), o["dx"]),
        "dw_router": (f64(L.dw_router), o["dw_router"]),
    }
    errs = {k: rel(a, b) for k, (a, b) in checks.items()}
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (name, errs)
    # empty experts get exactly zero weight gradients
    for e in np.nonzero(o["counts"] == 0)[0]:
        assert not L.dw1[e].any() and not L.dw2[e].any()


@pytest.mark.parametrize("name", ["bf16_e8_small", "bf16_skew_split"])
def test_bf16_weight_grads_in_bf16(name):
    cfg = CASES[name]
    cpu, L = run_layer(cfg, dw_dtype="bf16")
    o = oracle_for(cpu, L)
    assert L.dw1.dtype == torch.bfloat16
    assert rel(f64(L.dw1), o["dw1"]) <= TOL["bf16"]
    assert rel(f64(L.dw2), o["dw2"]) <= TOL["bf16"]


@pytest.mark.parametrize("name,cap", [("bf16_skew_small", 40), ("tiny_f32", 80), ("bf16_e8_small", 400)])
def test_padded_capacity_matches_oracle(name, cap):
    cfg = CASES[name]
    tol = TOL[cfg.dtype]
    cpu, L = run_layer(cfg, capacity=cap)
    o = oracle_for(cpu, L, capacity=cap)
    _check_routing(L, o)
    assert np.array_equal(i64(L.pad_row), o["pad_row"])
    assert np.array_equal(i64(L.offsets_pad), np.arange(cfg.E + 1) * cap)
    # kept rows are exact copies, unused rows are zero
    xp = L.x_perm.cpu()
    pr = o["pad_row"]
    for j in range(cfg.top_k):
        keep = pr[:, j] >= 0
        assert torch.equal(xp[torch.from_numpy(pr[keep, j])], cpu["x"][torch.from_numpy(np.nonzero(keep)[0])])
    used = np.zeros(cfg.E * cap, dtype=bool)
    used[pr[pr >= 0]] = True
    assert not xp[torch.from_numpy(~used)].any()
    for key, dev in (("out", L.out), ("dgate", L.dgate), ("dx", L.dx), ("dw1", L.dw1),
                     ("dw2", L.dw2), ("dw_router", L.dw_router)):
        assert rel(f64(dev), o[key]) <= tol, key


@pytest.mark.parametrize("name", ["bf16_skew_small", "bf16_skew_split"])
def test_routing_is_deterministic_across_runs(name):
    cfg = CASES[name]
    _, a = run_layer(cfg)
    _, b = run_layer(cfg)
    for key in ("logits", "topk_idx", "topk_gate", "slot_row", "out", "dx", "dw1", "dw2",
                "dw_router"):
        assert torch.equal(getattr(a, key), getattr(b, key)), key


def _stats_close(dev, want):
    """fp32 entries rounded once from exact integers / double sums."""
    want = np.asarray(want, dtype=np.float64)
    got = dev.double().cpu().numpy()
    assert np.allclose(got, want, rtol=2e-7, atol=0), (got, want)


@pytest.mark.parametrize("name,cap", [("bf16_skew_small", 40), ("bf16_skew_small", None),
                                      ("bf16_e128_small", 25), ("f32_e128", None),
                                      ("f32_one_token", 1)])
def test_routing_stats_of_the_layer(name, cap):
    cfg = CASES[name]
    cpu, L = run_layer(cfg)
    o = oracle_for(cpu, L)
    st = L.routing_stats(capacity=cap)
    torch.cuda.synchronize()
    _stats_close(st, ref.routing_stats(o["counts"], cap or 0))


def test_routing_stats_edge_counts():
    from mixture_experts_layer_offsets_b200 import capi
    out = torch.full((8,), -1.0, device="cuda")
    cases = [
        (np.zeros(7, np.int64), 3),                             # no rows at all
        (np.array([5]), 2),                                     # one expert
        (np.r_[np.full(1023, 0), [1 << 30]], 1 << 20),          # E = 1024, one huge expert
        (np.random.default_rng(1).integers(0, 5000, 1024), 0),  # no capacity
        (np.arange(1, 301), 150),
    ]
    for c, cap in cases:
        s = capi.shape_of(64, 64, len(c), 1, 64)
        dev = torch.tensor(c, dtype=torch.int32, device="cuda")
        capi.moe_routing_stats(s, dev, cap, out)
        torch.cuda.synchronize()
        _stats_close(out, ref.routing_stats(c, cap))


@pytest.mark.parametrize("name,cap", [("bf16_skew_small", None), ("tiny_f32", None),
                                      ("bf16_e128_small", None), ("bf16_skew_small", 40),
                                      ("f32_one_token", None)])
def test_renormalised_gates_match_oracle(name, cap):
    cfg = CASES[name]
    tol = TOL[cfg.dtype]
    cpu, L = run_layer(cfg, capacity=cap, renorm=True)
    o = oracle_for(cpu, L, capacity=cap)
    _check_routing(L, o)
    # the renormalisation itself runs in fp32 on fp32 gates
    assert rel(f64(L.gate_rn), o["gate_rn"]) <= TOL["f32"]
    assert np.allclose(f64(L.gate_rn).sum(axis=1), 1.0, rtol=1e-6)
    checks = {"out": (L.out, o["out"]), "dgate_rn": (L.dgate_rn, o["dgate_rn"]),
              "dgate": (L.dgate, o["dgate"]), "dx": (L.dx, o["dx"]),
              "dw_router": (L.dw_router, o["dw_router"]), "dw1": (L.dw1, o["dw1"]),
              "dw2": (L.dw2, o["dw2"])}
    errs = {k: rel(f64(a), b) for k, (a, b) in checks.items()}
    assert all(v <= tol for v in errs.values()), (name, errs)


def test_renorm_kernels_match_oracle_directly():
    from mixture_experts_layer_offsets_b200 import capi
    rng = np.random.default_rng(7)
    for T, k in [(1, 1), (333, 3), (1000, 8), (77, 32)]:
        g = rng.uniform(1e-4, 1.0, size=(T, k)).astype(np.float32)
        dg = rng.normal(size=(T, k)).astype(np.float32)
        s = capi.shape_of(T, 64, max(k, 2), k, 64)
        gd = torch.from_numpy(g).cuda()
        dgd = torch.from_numpy(dg).cuda()
        out = torch.empty_like(gd)
        dout = torch.empty_like(gd)
        capi.moe_renorm_gates(s, gd, out)
        capi.moe_renorm_gates_bwd(s, gd, dgd, dout)
        torch.cuda.synchronize()
        want = ref.renorm_gates(g.astype(np.float64))
        assert np.allclose(f64(out), want, rtol=1e-6, atol=0)
        wb = ref.renorm_gates_bwd(g.astype(np.float64), dg.astype(np.float64))
        assert rel(f64(dout), wb) <= 1e-6


@pytest.mark.parametrize("name", ["bf16_e8_small", "bf16_skew_split", "tiny_f32", "f32_one_token"])
def test_recompute_with_shared_buffers_is_bit_exact(name):
    check_recompute_bit_exact(CASES[name])


@pytest.mark.parametrize("name,dw", [("bf16_e8_small", "f32"), ("bf16_skew_split", "f32"),
                                     ("bf16_e128_small", "f32"), ("tiny_f32", "f32"),
                                     ("bf16_e8_small", "bf16"), ("bf16_skew_split", "bf16")])
def test_accumulated_weight_grads_are_the_sum_of_two_steps(name, dw):
    check_accumulate(CASES[name], dw_dtype=dw)


@pytest.mark.parametrize("dtype,d,f", [("f32", 64, 32), ("bf16", 256, 256), ("mxfp8", 256, 256)])
def test_empty_batch_is_a_clean_no_op(dtype, d, f):
    # T = 0: nothing is routed; every count and offset is 0 and every weight gradient,
    # written or accumulated, is exactly 0 (each expert's tile sums over no rows)
    base = CONFIGS["tiny_f32"] if dtype == "f32" else CONFIGS["bf16_e8"]
    cfg = shrink(base, name=f"empty_{dtype}", T=0, d_model=d, d_ff=f, E=8, top_k=2, dtype=dtype)
    cpu, L = run_layer(cfg)
    assert not L.counts.any() and not L.offsets.any()
    for key in ("dw1", "dw2", "dw_router"):
        assert not getattr(L, key).any(), key
    assert L.out.numel() == 0 and L.dx.numel() == 0
