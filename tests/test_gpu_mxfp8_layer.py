"""GPU parity of the layer with MXFP8 expert GEMMs against the float64 oracle
that quantises every GEMM operand along its contraction axis.

Routing is bit-exact (bf16 router); the quantised weight copies are byte-exact
with the oracle's MXFP8 rule; every value meets the MXFP8 relative Frobenius
tolerance.  The layer keeps its activations in bf16, so the oracle takes its
MXFP8 codes on the bf16-rounded activations, as the device does (an integer
decision taken in the kernel's precision).  Sizes span several 128-row tiles per expert with ragged tails,
empty experts (skewed routing), d and f that are odd multiples of 128, and a
single token.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import TOL, check_accumulate, check_recompute_bit_exact, f64, i64, rel, run_layer
from mixture_experts_layer_offsets_b200.inputs import CONFIGS, shrink
from oracle import moe_mx_ref as mxr
from oracle import mxfp8_ref as mx

pytestmark = pytest.mark.gpu

BASE = CONFIGS["mxfp8_e128"]
CASES = {
    # ~150 rows per expert: two M tiles, ragged tail
    "mx_e8": shrink(BASE, name="mx_e8", T=600, d_model=256, E=8, top_k=2, d_ff=256),
    # d and f odd multiples of 128; top_k 4 of 16
    "mx_e16_odd": shrink(BASE, name="mx_e16_odd", T=500, d_model=384, E=16, top_k=4, d_ff=384),
    # skewed routing with a logit bias: heavy-tailed counts and empty experts
    "mx_skew": shrink(BASE, name="mx_skew", T=700, d_model=128, E=32, top_k=2, d_ff=128,
                      router_std=1 / 16.0, bias_std=2.0),
    # experts of 3459 and 5998 rows: weight gradients cut into K ranges, partial sums added
    "mx_skew_split": shrink(BASE, name="mx_skew_split", T=6000, d_model=128, E=16, top_k=2,
                            d_ff=128, router_std=1 / 16.0, bias_std=3.0),
    # d and f multiples of 256, ~512 rows per expert: the row-grouped GEMMs run on CTA pairs
    "mx_pairs": shrink(BASE, name="mx_pairs", T=2048, d_model=512, E=8, top_k=2, d_ff=256),
    # skewed, d and f multiples of 256: weight gradients on CTA pairs (256 x 256 tiles)
    # with their K cut into ranges and partial sums added
    "mx_skew_split_pairs": shrink(BASE, name="mx_skew_split_pairs", T=6000, d_model=256, E=16,
                                  top_k=2, d_ff=256, router_std=1 / 16.0, bias_std=3.0),
    # one token
    "mx_one_token": shrink(BASE, name="mx_one_token", T=1, d_model=128, E=4, top_k=2, d_ff=128),
}


def _oracle(cpu, L):
    bias = f64(cpu["bias"]) if cpu["bias"] is not None else None
    return mxr.layer_fwd_bwd_mx(f64(cpu["x"]), f64(cpu["w_router"]), f64(cpu["w1"]),
                                f64(cpu["w2"]), f64(cpu["dout"]), L.k, bias,
                                select_logits=f64(L.logits), act_round=mxr.round_bf16)


@pytest.mark.parametrize("name", list(CASES))
def test_mxfp8_layer_matches_oracle(name):
    cfg = CASES[name]
    tol = TOL["mxfp8"]
    cpu, L = run_layer(cfg)
    o = _oracle(cpu, L)
    for key, dev in (("idx", L.topk_idx), ("counts", L.counts), ("offsets", L.offsets),
                     ("slot_row", L.slot_row)):
        assert np.array_equal(i64(dev), o[key]), key
    R, f = cfg.R, cfg.d_ff
    act = f64(L.act[:R])
    checks = {
        "logits": (f64(L.logits), o["logits"]), "gate": (f64(L.topk_gate), o["gate"]),
        "a": (act[:, :f], o["a"]), "u": (act[:, f:2 * f], o["u"]), "h": (act[:, 2 * f:], o["h"]),
        "y_perm": (f64(L.y_perm[:R]), o["y_perm"]), "out": (f64(L.out), o["out"]),
        "dgate": (f64(L.dgate), o["dgate"]),
        "dx_perm": (f64(L.dx_perm[:R]), o["dx_perm"]), "dw1": (f64(L.dw1), o["dw1"]),
        "dw2": (f64(L.dw2), o["dw2"]), "dx": (f64(L.dx), o["dx"]),
        "dw_router": (f64(L.dw_router), o["dw_router"]),
    }
    if L.dy_perm is not None:  # (the fused combine backward writes only dy's MXFP8 copies)
        checks["dy_perm"] = (f64(L.dy_perm[:R]), o["dy_perm"])
    errs = {k: rel(a, b) for k, (a, b) in checks.items()}
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (name, errs)
    for e in np.nonzero(o["counts"] == 0)[0]:
        assert not L.dw1[e].any() and not L.dw2[e].any()


def _atom_rows_blocks():
    """Row and 32-block index of each byte of a 512-byte scale atom (the layout
    documented with moe_mx_weights: byte (r % 32) * 16 + (r / 32) * 4 + kb)."""
    b = np.arange(512)
    return (b // 16) + 32 * ((b % 16) // 4), b % 4


def _k_major_plain(atoms, E, rows, K):
    """Atoms of a K-major weight copy -> plain scales [E * rows, K / 32]."""
    r, kb = _atom_rows_blocks()
    a = atoms.reshape(E, rows // 128, K // 128, 512)
    e, t, j, b = np.indices(a.shape)
    rr = t * 128 + r[b]
    out = np.full((E * rows, K // 32), -1, dtype=np.int64)
    out[e * rows + rr, 4 * j + kb[b]] = a
    return out


def _mn_major_plain(atoms, E, rows, K):
    """Atoms of a column-block weight copy -> plain scales [E * rows / 32, K]."""
    r, kb = _atom_rows_blocks()
    a = atoms.reshape(E, rows // 128, K // 128, 512)
    e, j, nt, b = np.indices(a.shape)
    out = np.full((E * rows // 32, K), -1, dtype=np.int64)
    out[e * (rows // 32) + 4 * j + kb[b], nt * 128 + r[b]] = a
    return out


def test_mxfp8_weight_copies_are_byte_exact():
    cfg = CASES["mx_e16_odd"]
    cpu, L = run_layer(cfg)
    E, d, f = cfg.E, cfg.d_model, cfg.d_ff
    w1 = f64(cpu["w1"]).reshape(E * 2 * f, d)
    w2 = f64(cpu["w2"]).reshape(E * d, f)
    got = {k: v.cpu().numpy() for k, v in L.mxq.items()}
    plain = {
        "w1": _k_major_plain(got["w1_s"], E, 2 * f, d),
        "w1t": _mn_major_plain(got["w1t_s"], E, 2 * f, d),
        "w2": _k_major_plain(got["w2_s"], E, d, f),
        "w2t": _mn_major_plain(got["w2t_s"], E, d, f),
    }
    for name, src, axis in (("w1", w1, 0), ("w1t", w1, 1), ("w2", w2, 0), ("w2t", w2, 1)):
        q, sc = mx.mxfp8_quantize(src, axis=axis)
        assert np.array_equal(got[name + "_q"], q), name
        assert np.array_equal(plain[name], sc), name


def test_mxfp8_is_closer_to_its_oracle_than_to_the_unquantised_layer():
    """The device really computes with MXFP8 operands: its error against the
    quantising oracle is well below its distance from the unquantised layer."""
    from oracle import moe_ref as ref
    cfg = CASES["mx_e8"]
    cpu, L = run_layer(cfg)
    o = _oracle(cpu, L)
    bias = f64(cpu["bias"]) if cpu["bias"] is not None else None
    u = ref.layer_fwd_bwd(f64(cpu["x"]), f64(cpu["w_router"]), f64(cpu["w1"]), f64(cpu["w2"]),
                          f64(cpu["dout"]), L.k, bias, select_logits=f64(L.logits))
    for key, dev in (("out", L.out), ("dw1", L.dw1), ("dx", L.dx)):
        assert rel(f64(dev), o[key]) < 0.5 * rel(f64(dev), u[key]), key



@pytest.mark.parametrize("name", ["mx_e8", "mx_skew_split", "mx_one_token"])
def test_mxfp8_recompute_with_shared_buffers_is_bit_exact(name):
    # the shared workspace loses the forward's token-block copies to layer B: the
    # recompute rebuilds them along with a | u | h
    check_recompute_bit_exact(CASES[name])


@pytest.mark.parametrize("flag", ["MOE_B200_DADU", "MOE_B200_HMX"])
@pytest.mark.parametrize("name", ["mx_e8", "mx_e16_odd", "mx_skew", "mx_one_token",
                                  "mx_skew_split_pairs", "mx_pairs"])
def test_fused_epilogue_quantisation_is_bit_identical_to_a_separate_pass(name, flag,
                                                                          monkeypatch):
    # [da | du] quantised in the SwiGLU-backward epilogue (MOE_B200_DADU), h in the gate/up
    # epilogue (MOE_B200_HMX), against the bf16 values followed by the activation
    # quantiser: every result of the step bit for bit
    cfg = CASES[name]
    _, A = run_layer(cfg)
    monkeypatch.setenv(flag, "0")
    _, B = run_layer(cfg)
    for key in ("act", "y_perm", "out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
        a, b = getattr(A, key), getattr(B, key)
        if key in ("act", "y_perm", "dx_perm"):
            a, b = a[:cfg.R], b[:cfg.R]
        assert torch.equal(a, b), key


@pytest.mark.parametrize("name", ["mx_e8", "mx_skew"])
def test_fused_paths_with_renormalised_gates_are_bit_identical(name):
    # the fused combine backward takes the renormalised gates the combine used and writes
    # their gradient, which the renormalisation backward then maps back
    cfg = CASES[name]
    _, A = run_layer(cfg, renorm=True, fused_dispatch=True)
    _, B = run_layer(cfg, renorm=True, fused_dispatch=False)
    for key in ("out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
        a, b = getattr(A, key), getattr(B, key)
        if key == "dx_perm":
            a, b = a[:cfg.R], b[:cfg.R]
        assert torch.equal(a, b), key


@pytest.mark.parametrize("name", ["mx_e8", "mx_e16_odd", "mx_skew", "mx_one_token",
                                  "mx_skew_split_pairs"])
def test_fused_dispatch_is_bit_identical_to_permute_then_quantise(name):
    # the fused dispatch (x's copies from x through perm_src) and the fused combine
    # backward (dy's copies from gate x dout, no dy_perm) against the bf16 rows followed
    # by the layer's own quantisation: every result bit for bit
    cfg = CASES[name]
    _, A = run_layer(cfg, fused_dispatch=True)
    _, B = run_layer(cfg, fused_dispatch=False)
    assert A.x_perm is None and A.dy_perm is None
    for key in ("perm_src", "act", "y_perm", "out", "dgate", "dx_perm", "dw1", "dw2", "dx",
                "dw_router"):
        a, b = getattr(A, key), getattr(B, key)
        if key in ("perm_src", "act", "y_perm", "dx_perm"):
            a, b = a[:cfg.R], b[:cfg.R]
        assert torch.equal(a, b), key


@pytest.mark.parametrize("name", ["mx_e8", "mx_skew_split", "mx_skew_split_pairs"])
def test_mxfp8_accumulated_weight_grads_are_the_sum_of_two_steps(name):
    check_accumulate(CASES[name])


@pytest.mark.parametrize("name", ["mx_e8", "mx_pairs"])
def test_reused_weight_copies_give_the_bits_of_a_fresh_quantisation(name):
    # the micro-batches of one optimizer step after the first run on the weight copies the
    # first one made (requantize=False), also when two layer instances share them: the
    # second micro-batch (other tokens, same weights) must match a layer that quantised
    from mixture_experts_layer_offsets_b200.inputs import make_inputs
    from mixture_experts_layer_offsets_b200.layer import MoELayer
    cfg = CASES[name]
    dev = lambda d: {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    a_in = dev(make_inputs(cfg, device="cpu", seed=0))
    b_in = dev(make_inputs(cfg, device="cpu", seed=1))
    for k in ("w_router", "bias", "w1", "w2"):  # batch B: new tokens, A's weights
        b_in[k] = a_in[k]
    args = lambda i: (i["x"], i["w_router"], i["bias"], i["w1"], i["w2"], i["dout"])
    new = lambda: MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda")
    ref = new()
    ref.step(*args(b_in))
    first, second = new(), new()
    second.share_weight_copies(first)
    first.step(*args(a_in))
    first.step(*args(b_in), accumulate=False, requantize=False)
    second.step(*args(b_in), requantize=False)
    torch.cuda.synchronize()
    for L in (first, second):
        assert L.device_status() == 0
        for key in ("out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
            assert torch.equal(getattr(L, key), getattr(ref, key)), key
    with pytest.raises(ValueError):
        MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, "bf16", "cuda").share_weight_copies(first)



@pytest.mark.parametrize("name", ["mx_pairs", "mx_skew_split", "mx_skew_split_pairs"])
def test_mxfp8_cta_pairs_give_the_bits_of_single_ctas(name, monkeypatch):
    # the same dot products in the same K order: 256-row tiles on CTA pairs (row-grouped
    # GEMMs and weight gradients) must reproduce the single-CTA results exactly
    cfg = CASES[name]
    monkeypatch.setenv("MOE_B200_PAIR", "0")
    _, A = run_layer(cfg)
    monkeypatch.setenv("MOE_B200_PAIR", "1")
    _, B = run_layer(cfg)
    for key in ("act", "y_perm", "out", "dx_perm", "dx", "dw1", "dw2", "dw_router"):
        a, b = getattr(A, key), getattr(B, key)
        if key in ("act", "y_perm", "dx_perm"):
            a, b = a[:cfg.R], b[:cfg.R]
        assert torch.equal(a, b), key
