"""GPU parity of mxfp8_quantize: element and scale bytes bit-exact with the
oracle's MXFP8 rule, along rows (axis 0) and along segmented columns (axis 1)."""

import json
import os

import numpy as np
import pytest
import torch

from mixture_experts_layer_offsets_b200 import capi
from oracle import mxfp8_ref as mx

pytestmark = pytest.mark.gpu


def _src(rows, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(rows, K, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 4)
    v[0, :] = 0.0                       # an all-zero block
    v[1, 3] = 1e30 if dtype == torch.float32 else 3e38
    v[2, :5] = torch.tensor([2.0 ** -140, -(2.0 ** -133), 0.0, -0.0, 1e-41])  # fp32 subnormals
    return v.to(dtype)


def _dev_quant(src, axis, segs=None):
    rows, K = src.shape
    d = src.cuda()
    q = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
    nseg = len(segs) - 1 if segs is not None else 1
    srows = rows // 32 + nseg + 1
    scale = torch.full((srows if axis == 1 else rows, K // 32 if axis == 0 else K), 0xAB,
                       dtype=torch.uint8, device="cuda")
    seg_t = torch.tensor(segs, dtype=torch.int32, device="cuda") if segs is not None else None
    dt = capi.MOE_BF16 if src.dtype == torch.bfloat16 else capi.MOE_F32
    capi.mxfp8_quantize(rows, K, dt, d, axis, seg_t, nseg if segs is not None else 0, q, scale)
    torch.cuda.synchronize()
    return q.cpu().numpy(), scale.cpu().numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_axis0_bytes_exact(dtype):
    src = _src(300, 1024, dtype, 1)
    q, s = _dev_quant(src, 0)
    rq, rs = mx.mxfp8_quantize(src.to(torch.float64).numpy(), axis=0)
    assert np.array_equal(s, rs)
    assert np.array_equal(q, rq)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_axis1_segments_bytes_exact(dtype):
    segs = [0, 0, 37, 100, 100, 164, 300]  # empty segments, ragged tails
    src = _src(300, 256, dtype, 2)
    q, s = _dev_quant(src, 1, segs)
    rq, rs = mx.mxfp8_quantize(src.to(torch.float64).numpy(), axis=1, seg_offsets=segs)
    assert np.array_equal(q, rq)
    assert np.array_equal(s[: rs.shape[0]], rs)
    assert np.all(s[rs.shape[0]:] == 0xAB)   # rows past the last block are untouched


def test_axis1_without_segments_bytes_exact():
    src = _src(97, 64, torch.bfloat16, 3)
    q, s = _dev_quant(src, 1, None)
    rq, rs = mx.mxfp8_quantize(src.to(torch.float64).numpy(), axis=1)
    assert np.array_equal(q, rq)
    assert np.array_equal(s[: rs.shape[0]], rs)


def test_golden_blocks_on_device(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "mxfp8_blocks.json")))
    blocks = np.zeros((len(fx["blocks"]), 32), dtype=np.float32)
    for i, b in enumerate(fx["blocks"]):
        blocks[i, : len(b["values"])] = b["values"]
    q, s = _dev_quant(torch.from_numpy(blocks), 0)
    for i, b in enumerate(fx["blocks"]):
        assert s[i, 0] == b["scale_byte"], b["note"]
        assert q[i, : len(b["codes"])].tolist() == b["codes"], b["note"]


def test_every_finite_bf16_pattern_bytes_exact():
    """All 65024 finite bf16 bit patterns (signed zeros and subnormals included), in a
    fixed shuffled order, blocked along rows and along columns: the device's element codes
    (sign of every value, ties, saturation) and scales equal the oracle's rule."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = bits[((bits >> 7) & 0xFF) != 0xFF]
    rng = np.random.default_rng(7)
    pat = rng.permutation(finite)
    n = -(-len(pat) // 1024) * 1024
    pat = np.concatenate([pat, np.zeros(n - len(pat), dtype=np.uint32)])
    vals = (pat << 16).view(np.float32).reshape(-1, 64)
    src = torch.from_numpy(vals.copy()).to(torch.bfloat16)   # exact: every value is a bf16
    for axis in (0, 1):
        q, s = _dev_quant(src, axis, [0, 333, vals.shape[0]] if axis else None)
        segs = [0, 333, vals.shape[0]] if axis else None
        rq, rs = mx.mxfp8_quantize(vals.astype(np.float64), axis=axis, seg_offsets=segs)
        assert np.array_equal(q, rq), axis
        assert np.array_equal(s[: rs.shape[0]], rs), axis
