"""Byte-exact parity of the MXFP8 operands that the layer itself quantises.

kongchang, section 吞吐量数字的边界条件 (boundary conditions): MXFP8 blocks of 32
elements share one E8M0 scale.  Every MXFP8 step quantises four activations with the
same kernel, each into two copies: x (by the fused dispatch moe_permute_mx, or by the
forward from x_perm), h (forward), dy and [da | du] (backward).  The row copy (blocks
of 32 along each row) feeds the row-grouped GEMMs, the token-block copy (blocks of 32
rows within each column, restarting at every expert) the weight-gradient GEMMs.  Here
the codes and scales the layer left in its workspace (located with
moe_mx_workspace_layout) are decoded and compared byte for byte with the oracle's
mxfp8_quantize on the same bf16 values (the token-block copy is column-major over a token
axis padded to whole 128-row stages per expert; its pad codes must be zero) (the layer stores its activations in bf16, so
both sides take their codes on those values), including the 2^0 scales that pad an
expert's last stage and the maps that place every block.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import check_mx_operand, f64, i64
from mixture_experts_layer_offsets_b200 import capi, inputs
from mixture_experts_layer_offsets_b200.layer import MoELayer
from oracle import moe_ref as ref

pytestmark = pytest.mark.gpu

BASE = inputs.CONFIGS["mxfp8_e128"]
CASES = {
    # d and f odd multiples of 128, ~125 rows per expert: ragged 32-row blocks and stages
    "mx_e16_odd": inputs.shrink(BASE, name="mx_e16_odd", T=500, d_model=384, E=16, top_k=4,
                                d_ff=384),
    # skewed routing: heavy-tailed counts, empty experts
    "mx_skew": inputs.shrink(BASE, name="mx_skew", T=700, d_model=128, E=32, top_k=2, d_ff=128,
                             router_std=1 / 16.0, bias_std=2.0),
    # experts of thousands of rows (weight gradients cut into K ranges)
    "mx_skew_split": inputs.shrink(BASE, name="mx_skew_split", T=6000, d_model=128, E=16,
                                   top_k=2, d_ff=128, router_std=1 / 16.0, bias_std=3.0),
    # ~512 rows per expert: the row-grouped GEMMs run on CTA pairs
    "mx_pairs": inputs.shrink(BASE, name="mx_pairs", T=2048, d_model=512, E=8, top_k=2,
                              d_ff=256),
    # one token: two rows, most experts empty
    "mx_one_token": inputs.shrink(BASE, name="mx_one_token", T=1, d_model=128, E=4, top_k=2,
                                  d_ff=128),
}


class _Ws:
    """Reads the MXFP8 regions of a layer's workspace."""

    def __init__(self, L):
        self.L = L
        self.lay = capi.moe_mx_workspace_layout(L.shape, L.rows)

    def _bytes(self, name, start, n):
        off = self.lay[name] + start
        return self.L.ws[off:off + n]

    def codes(self, name, r0, r1, K):
        return self._bytes(name, r0 * K, (r1 - r0) * K).view(r1 - r0, K).cpu().numpy()

    def atoms(self, name, K):
        tiles = self.L.rows // 128 + self.L.E
        return self._bytes(name, 0, tiles * (K // 128) * 512).cpu().numpy()

    def maps(self):
        R = self.L.rows
        rt = self._bytes("row_tile", 0, 4 * R).view(torch.int32).cpu().numpy().astype(np.int64)
        nb, ns = self._bytes("nblocks", 0, 8).view(torch.int32).tolist()
        bl = self._bytes("blocks", 0, 16 * nb).view(torch.int32).view(nb, 4).cpu().numpy()
        # the stage table after the block map: first block of every stage, then nb
        sm = self._bytes("blocks", 16 * (R // 32 + self.L.E), 4 * (ns + 1))
        sm = sm.view(torch.int32).cpu().numpy().astype(np.int64)
        bl = bl.astype(np.int64)
        assert sm[-1] == nb and np.all(np.diff(sm) >= 1) and np.all(np.diff(sm) <= 4)
        assert np.array_equal(bl[sm[:-1], 2], np.arange(ns)), "stage table"
        assert np.all(bl[sm[:-1], 3] & 3 == 0), "a stage starts at its first block"
        return rt, bl

    def blk_codes(self, name, K, blocks, r0, r1):
        """Token-block codes of operand rows r0..r1 as [r1 - r0, K], read from the copy's
        column-major layout over the stage-padded token axis ([K][Rp]), and the padded
        positions of those rows' stages that hold no row (they must be zero)."""
        Rp = (self.L.rows // 128 + self.L.E) * 128
        qT = self._bytes(name, 0, K * Rp).view(K, Rp)
        sel = blocks[(blocks[:, 0] >= r0) & (blocks[:, 0] < r1)]
        pos = np.zeros(r1 - r0, dtype=np.int64)
        for rb, n, z, w in sel:
            pos[rb - r0:rb - r0 + n] = 128 * z + 32 * (w & 3) + np.arange(n)
        codes = qT[:, torch.from_numpy(pos).cuda()].t().cpu().numpy() if r1 > r0 else \
            np.zeros((0, K), dtype=np.uint8)
        stages = np.unique(sel[:, 2]) if len(sel) else np.zeros(0, dtype=np.int64)
        allpos = (128 * stages[:, None] + np.arange(128)[None, :]).ravel()
        pads = np.setdiff1d(allpos, pos)
        padv = qT[:, torch.from_numpy(pads).cuda()].cpu().numpy() if len(pads) else np.zeros(0)
        return codes, padv

    def dadu(self, r0, r1):
        f2 = 2 * self.L.f
        b = self._bytes("dadu", r0 * f2 * 2, (r1 - r0) * f2 * 2)
        return f64(b.view(torch.bfloat16).view(r1 - r0, f2))


def _check(ws, name, values, K, offsets, e0, e1, q_row, s_row, q_blk, s_blk):
    r0, r1 = int(offsets[e0]), int(offsets[e1])
    rt, bl = ws.maps()
    blk, pads = ws.blk_codes(q_blk, K, bl, r0, r1)
    try:
        check_mx_operand(values, K, offsets, e0, e1, ws.codes(q_row, r0, r1, K),
                         ws.atoms(s_row, K), blk, ws.atoms(s_blk, K), rt, bl)
        assert not np.any(pads), "token-block pad codes"
    except AssertionError as err:
        raise AssertionError(f"{name}: {err}") from None


def run_and_check_bytes(cfg, fused, expert=None):
    """One MXFP8 step; after the forward and after the backward, every quantised
    activation is checked on the rows of all experts (or of one sampled expert)."""
    cpu = inputs.make_inputs(cfg, device="cpu", seed=0)
    dev = {k: (v.cuda() if v is not None else None) for k, v in cpu.items()}
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                 fused_dispatch=fused)
    ws = _Ws(L)
    L.forward(dev["x"], dev["w_router"], dev["bias"], dev["w1"], dev["w2"])
    torch.cuda.synchronize()
    o = ref.route_from_logits(f64(L.logits), L.k)
    offsets = i64(L.offsets)
    assert np.array_equal(offsets, o["offsets"])
    e0, e1 = (0, cfg.E) if expert is None else (expert, expert + 1)
    r0, r1 = int(offsets[e0]), int(offsets[e1])
    d, f = cfg.d_model, cfg.d_ff
    src = L.perm_src[r0:r1].long()
    x_rows = f64(dev["x"][src])
    h_rows = f64(L.act[r0:r1, 2 * f:3 * f])
    _check(ws, "x", x_rows, d, offsets, e0, e1, "qx0", "sx0", "qx1", "sx1")
    _check(ws, "h", h_rows, f, offsets, e0, e1, "qh0", "sh0", "qh1", "sh1")
    L.backward(dev["dout"], dev["x"], dev["w_router"], dev["w1"], dev["w2"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    if L.dy_perm is not None:
        dy_rows = f64(L.dy_perm[r0:r1])
    else:
        # the fused combine backward quantises gate x dout rows, rounded to bf16 first, as
        # the combine backward rounds dy_perm
        gp = torch.zeros(max(L.R, 1), dtype=torch.float32, device="cuda")
        gp[L.slot_row.reshape(-1).long()] = L.topk_gate.reshape(-1)
        dy = dev["dout"][src].float() * gp[r0:r1, None]
        dy_rows = f64(dy.to(torch.bfloat16))
    _check(ws, "dy", dy_rows, d, offsets, e0, e1, "qdy0", "sdy0", "qdy1", "sdy1")
    _check(ws, "[da|du]", ws.dadu(r0, r1), 2 * f, offsets, e0, e1, "qda0", "sda0", "qda1",
           "sda1")
    return L, offsets


@pytest.mark.parametrize("name,fused", [("mx_e16_odd", True), ("mx_e16_odd", False),
                                        ("mx_skew", True), ("mx_skew_split", True),
                                        ("mx_pairs", False), ("mx_one_token", True)])
def test_mxfp8_activation_bytes_are_exact(name, fused, monkeypatch):
    # [da | du] leaves the SwiGLU-backward epilogue as its MXFP8 copies; "keep" also writes
    # its bf16 rows, against which those copies are checked
    monkeypatch.setenv("MOE_B200_DADU", "keep")
    cfg = CASES[name]
    L, offsets = run_and_check_bytes(cfg, fused)
    if name == "mx_skew":
        assert (np.diff(offsets) == 0).any(), "the skewed case must leave experts empty"


def test_fullsize_mxfp8_activation_bytes_of_a_sampled_expert(monkeypatch):
    """mxfp8_e128 at full size (T = 32768, d = 4096, E = 128, f = 1536), fused dispatch as
    the benchmark runs it: the four activations' codes and scales on one sampled expert's
    rows (a row's codes and an expert's token blocks depend on nothing else)."""
    monkeypatch.setenv("MOE_B200_DADU", "keep")
    cfg = BASE
    rng = np.random.default_rng(5)
    expert = int(rng.integers(0, cfg.E))
    L, offsets = run_and_check_bytes(cfg, True, expert=expert)
    assert offsets[expert + 1] - offsets[expert] > 128  # several stages, ragged tail
