"""Helpers shared by the GPU parity tests (run the CUDA path; compare to the oracle)."""

from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_offsets_b200 import inputs
from mixture_experts_layer_offsets_b200.layer import MoELayer
from oracle import moe_ref as ref

# Tolerances on relative Frobenius error, by compute dtype.
TOL = {"f32": 1e-5, "bf16": 1e-2, "mxfp8": 5e-2}


def f64(t) -> np.ndarray:
    if t is None:
        return None
    return t.detach().to(torch.float64).cpu().numpy()


def i64(t) -> np.ndarray:
    return t.detach().to(torch.int64).cpu().numpy()


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def run_layer(cfg, seed=0, capacity=None, dw_dtype="f32", renorm=False, **kw):
    """Seeded inputs drawn on the CPU, copied to the GPU, one fwd+bwd step."""
    cpu = inputs.make_inputs(cfg, device="cpu", seed=seed)
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                 dw_dtype=dw_dtype, capacity=capacity, renorm=renorm, **kw)
    L.step(dev["x"], dev["w_router"], dev["bias"], dev["w1"], dev["w2"], dev["dout"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return cpu, L


def oracle_for(cpu, L, capacity=None):
    """Oracle pass on the same inputs; discrete routing taken on the device's logits."""
    args = (f64(cpu["x"]), f64(cpu["w_router"]), f64(cpu["w1"]), f64(cpu["w2"]), f64(cpu["dout"]),
            L.k)
    bias = f64(cpu["bias"]) if cpu["bias"] is not None else None
    if capacity:
        return ref.padded_layer_fwd_bwd(*args, capacity, bias, select_logits=f64(L.logits),
                                        renorm=L.renorm)
    return ref.layer_fwd_bwd(*args, bias, select_logits=f64(L.logits), renorm=L.renorm)


def check_recompute_bit_exact(cfg):
    """Two layers share one activation buffer and one workspace; layer A's backward
    runs after layer B's forward has overwritten both, recomputing what it needs.  Its
    results equal, bit for bit, those of a layer that kept its own activations."""
    _, L0 = run_layer(cfg, seed=0)
    dev = lambda d: {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    a_in = dev(inputs.make_inputs(cfg, device="cpu", seed=0))
    b_in = dev(inputs.make_inputs(cfg, device="cpu", seed=1))
    tdt = L0.act.dtype
    act = torch.empty(L0.act.numel(), dtype=tdt, device="cuda")
    ws = torch.zeros_like(L0.ws)
    mk = lambda: MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                          recompute=True, act_scratch=act, ws=ws)
    A, B = mk(), mk()
    A.forward(a_in["x"], a_in["w_router"], a_in["bias"], a_in["w1"], a_in["w2"])
    a_act = act.clone()
    B.forward(b_in["x"], b_in["w_router"], b_in["bias"], b_in["w1"], b_in["w2"])
    torch.cuda.synchronize()
    assert cfg.T == 0 or not torch.equal(act, a_act), "layer B did not overwrite the shared buffer"
    A.backward(a_in["dout"], a_in["x"], a_in["w_router"], a_in["w1"], a_in["w2"])
    torch.cuda.synchronize()
    assert A.device_status() == 0
    assert torch.equal(act, a_act), "the recompute did not restore a | u | h"
    for key in ("out", "dgate", "dx_perm", "dw1", "dw2", "dx", "dw_router"):
        assert torch.equal(getattr(A, key), getattr(L0, key)), key


def check_accumulate(cfg, dw_dtype="f32"):
    """A layer that steps on batch A, then on batch B with MOE_DW_ACCUMULATE, holds the sum of
    the weight gradients of two layers that each stepped on one batch.  fp32 weight gradients
    get one fp32 addition per element, so the sum is exact against torch's fp32 addition
    (subnormal results aside); bf16 ones are rounded once, within the bf16 tolerance."""
    _, A = run_layer(cfg, seed=0, dw_dtype=dw_dtype)
    _, B = run_layer(cfg, seed=1, dw_dtype=dw_dtype)
    dev = lambda d: {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    a_in = dev(inputs.make_inputs(cfg, device="cpu", seed=0))
    b_in = dev(inputs.make_inputs(cfg, device="cpu", seed=1))
    C = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda", dw_dtype=dw_dtype)
    args = lambda i: (i["x"], i["w_router"], i["bias"], i["w1"], i["w2"], i["dout"])
    C.step(*args(a_in))
    C.step(*args(b_in), accumulate=True)
    torch.cuda.synchronize()
    assert C.device_status() == 0
    keys = ("dw1", "dw2", "dw_router")
    for key in keys:
        got, a, b = getattr(C, key), getattr(A, key), getattr(B, key)
        if got.dtype == torch.float32:
            want = a + b
            diff = got != want
            # only a subnormal sum may differ (flushed to zero by the reducing store)
            assert not diff.any() or bool((want[diff].abs() < 1.2e-38).all()), key
        else:
            want = a.double() + b.double()
            assert rel(f64(got), want.cpu().numpy()) <= TOL["bf16"], key
    # the step that accumulated still computed its own non-gradient outputs normally
    assert torch.equal(C.out, B.out) and torch.equal(C.dx, B.dx)


# ---------------------------------------------------------------- MXFP8 operand bytes
def _atom_byte(r, kb):
    """Byte of (row r, 32-block kb) in a 512-byte scale atom of 128 rows x 4 blocks."""
    return (r % 32) * 16 + (r // 32) * 4 + kb


def expected_row_tiles(offsets) -> np.ndarray:
    """Row -> 128 * tile + row within the tile, tiles numbered expert by expert
    (each expert's rows start a new 128-row tile)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    c = np.diff(offsets)
    pre = np.concatenate([[0], np.cumsum(-(-c // 128))])
    out = np.full(int(offsets[-1]), -1, dtype=np.int64)
    for e in range(len(c)):
        out[offsets[e]:offsets[e + 1]] = pre[e] * 128 + np.arange(c[e])
    return out


def expected_token_blocks(offsets) -> np.ndarray:
    """The 32-row token blocks of every expert, in order: {first row, rows, 128-row
    stage (stages numbered expert by expert), block in stage | 4 if last}."""
    offsets = np.asarray(offsets, dtype=np.int64)
    c = np.diff(offsets)
    st = np.concatenate([[0], np.cumsum(-(-c // 128))])
    rows = []
    for e in range(len(c)):
        nb = -(-int(c[e]) // 32)
        for lb in range(nb):
            rows.append((offsets[e] + 32 * lb, min(32, c[e] - 32 * lb), st[e] + lb // 4,
                         (lb & 3) | (4 if lb == nb - 1 else 0)))
    return np.array(rows, dtype=np.int64).reshape(-1, 4)


def check_mx_operand(values, K, offsets, e0, e1, q_row, atoms_row, q_blk, atoms_blk, row_tile,
                     blocks):
    """Byte-exact check of one MXFP8 activation as the layer stores it, on the rows of
    experts e0..e1-1 against oracle mxfp8_quantize of the same bf16 values.

    values: float64 [r1 - r0, K] (the bf16 operand rows r0..r1); q_row / q_blk: u8 codes of
    those rows (row copy, token-block copy); atoms_row / atoms_blk: the whole atom regions
    (u8); row_tile: int [rows] (the layer's map); blocks: int [nblocks, 4] (the layer's)."""
    from oracle import mxfp8_ref as mx
    offsets = np.asarray(offsets, dtype=np.int64)
    r0, r1 = int(offsets[e0]), int(offsets[e1])
    n = r1 - r0
    assert values.shape == (n, K)
    kq = K // 128
    # the maps themselves
    assert np.array_equal(row_tile[r0:r1], expected_row_tiles(offsets)[r0:r1]), "row_tile"
    want_blocks = expected_token_blocks(offsets)
    sel = (want_blocks[:, 0] >= r0) & (want_blocks[:, 0] < r1)
    assert np.array_equal(blocks[sel], want_blocks[sel]), "token blocks"
    # row copy: codes and row-tile scale atoms
    q0, s0 = mx.mxfp8_quantize(values, axis=0)
    assert np.array_equal(q_row, q0), "row codes"
    rt = row_tile[r0:r1]
    kbg = np.arange(K // 32)
    idx = ((rt[:, None] >> 7) * kq + kbg[None, :] // 4) * 512 + \
        _atom_byte(rt[:, None] & 127, kbg[None, :] % 4)
    assert np.array_equal(atoms_row[idx], s0), "row scales"
    # token-block copy: codes (blocks restart at every expert), stage scale atoms, 2^0 pads
    q1, s1 = mx.mxfp8_quantize(values, axis=1, seg_offsets=offsets[e0:e1 + 1] - r0)
    assert np.array_equal(q_blk, q1), "token-block codes"
    bl = want_blocks[sel]
    cols = np.arange(K)
    base = (bl[:, 2:3] * kq + cols[None, :] // 128) * 512
    cc = cols[None, :] % 128
    idx = base + _atom_byte(cc, bl[:, 3:4] & 3)
    assert np.array_equal(atoms_blk[idx], s1), "token-block scales"
    last = bl[bl[:, 3] & 4 > 0]
    for kb in range(1, 4):
        pad = last[(last[:, 3] & 3) < kb]
        if len(pad):
            pidx = (pad[:, 2:3] * kq + cols[None, :] // 128) * 512 + _atom_byte(cc, kb)
            assert np.all(atoms_blk[pidx] == 0x7F), "pad scales"


def routing_divergence(L, inp, gap_frac=1e-3):
    """Tokens whose routing on the oracle's own float64 logits differs from the device's
    (the device routes on its fp32 logits; both use the same tie rule).  Such a token is
    allowed only where its k-th and (k+1)-th largest oracle logits lie within
    gap_frac * max|l| of each other (a near tie that the fp32 sum may order either way).
    Returns (number of such tokens, their largest gap as a fraction of max|l|)."""
    x = f64(inp["x"])
    bias = f64(inp["bias"]) if inp["bias"] is not None else None
    lg = ref.router_logits(x, f64(inp["w_router"]), bias)
    own = ref.route_from_logits(lg, L.k)["idx"]
    dev = i64(L.topk_idx)
    diff = np.nonzero((own != dev).any(axis=1))[0]
    if len(diff) == 0:
        return 0, 0.0
    scale = np.abs(lg).max()
    srt = -np.sort(-lg[diff], axis=1)
    k = L.k
    gap = (srt[:, k - 1] - srt[:, k]) if k < lg.shape[1] else np.zeros(len(diff))
    # a reordering inside the selected set needs a near tie among the selected values
    inside = np.array([np.min(np.diff(-srt[i, :k])) if k > 1 else 0.0 for i in range(len(diff))])
    same_set = np.array([set(own[t]) == set(dev[t]) for t in diff])
    g = np.where(same_set, inside, gap)
    assert np.all(g <= gap_frac * scale), (diff[g > gap_frac * scale][:5], g.max() / scale)
    return len(diff), float(g.max() / scale)
