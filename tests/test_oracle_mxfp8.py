"""Pins of the oracle's MXFP8 rule (E4M3 elements, E8M0 scales per 32 values).

Checks: the E4M3 decode table equals torch.float8_e4m3fn's; element rounding
equals torch's round-to-nearest-even cast; brute-force nearest-grid-point
search over all finite bf16 bit patterns; the scale invariant
2**(e+8) <= amax < 2**(e+9); exact round trips of powers of two; saturation;
the segmented axis-1 layout against zero-padded axis-0 blocks; and the
hand-derived fixture under tests/golden/.
"""

import json
import os

import numpy as np
import torch

from oracle import mxfp8_ref as mx


def test_decode_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    tv = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = mx.e4m3_decode(np.arange(256))
    nan = np.isnan(tv)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(tv[~nan], mine[~nan])
    assert np.nanmax(mine) == 448.0


def test_rne_matches_torch_cast():
    rng = np.random.default_rng(0)
    grid = mx.e4m3_decode(np.arange(0x7F))
    mids = (grid[1:] + grid[:-1]) / 2
    vals = np.concatenate([
        rng.normal(size=20000) * 40, rng.uniform(-464, 464, 20000),
        rng.normal(size=5000) * 2.0 ** -8, mids, -mids, grid, -grid,
        np.nextafter(mids, 0), np.nextafter(mids, 1000),
    ]).astype(np.float32).astype(np.float64)
    vals = vals[np.abs(vals) <= 464]
    t = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mx.e4m3_rne(vals), t)


def test_saturation_and_signed_zero():
    assert mx.e4m3_rne(np.array([449.0, 1e30, -1e30, 480.0])).tolist() == [0x7E, 0x7E, 0xFE, 0x7E]
    assert mx.e4m3_rne(np.array([-0.0, 0.0, -1e-9])).tolist() == [0x80, 0x00, 0x80]


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[np.isfinite(v)].astype(np.float64)


def test_exhaustive_bf16_blocks_round_to_nearest_grid_point():
    v = _all_finite_bf16()
    rng = np.random.default_rng(1)
    v = rng.permutation(v)
    n = (len(v) // 32) * 32
    v = v[:n].reshape(-1, 32)
    # group magnitudes so that blocks span realistic dynamic ranges
    v = v[np.argsort(np.max(np.abs(v), axis=1))]
    q, s = mx.mxfp8_quantize(v, axis=0)
    e = s.astype(np.int64).ravel() - 127
    amax = np.max(np.abs(v), axis=1)
    nz = amax > 0
    e_unclamped = np.floor(np.log2(amax[nz])) - 8
    ok = (e_unclamped >= -127) & (e_unclamped <= 127)
    assert np.array_equal(e[nz][ok], e_unclamped[ok].astype(np.int64))
    assert np.all(2.0 ** (e[nz][ok] + 8) <= amax[nz][ok])
    assert np.all(amax[nz][ok] < 2.0 ** (e[nz][ok] + 9))
    # brute force: each code is a nearest finite grid point of v / 2**e
    grid = mx.e4m3_decode(np.arange(256))
    fin = np.isfinite(grid)
    g = grid[fin]
    scaled = np.ldexp(v, -e[:, None]).ravel()
    sat = np.clip(scaled, -448, 448)
    dist = np.abs(g[None, :] - sat[:, None]).min(axis=1)
    got = mx.e4m3_decode(q.ravel())
    assert np.array_equal(np.abs(got - sat), dist)


def test_powers_of_two_round_trip_exactly():
    for top in (-120, -3, 0, 7, 100):
        blk = np.array([2.0 ** (top - i) for i in range(17)] + [0.0] * 15)[None, :]
        q, s = mx.mxfp8_quantize(blk, axis=0)
        assert np.array_equal(mx.mxfp8_dequantize(q, s, axis=0), blk)


def test_block_in_saturation_window_clamps_to_448():
    amax = 1.9 * 2 ** 5               # amax * 2**-e = 486.4 lands in (448, 512)
    blk = np.zeros((1, 32))
    blk[0, 0] = amax
    blk[0, 1] = -amax
    q, s = mx.mxfp8_quantize(blk, axis=0)
    assert s[0, 0] == 5 - 8 + 127
    assert q[0, 0] == 0x7E and q[0, 1] == 0xFE


def test_axis1_segments_equal_padded_axis0_blocks():
    rng = np.random.default_rng(2)
    K = 64
    segs = [0, 5, 5, 70, 101, 101]  # includes empty segments and ragged tails
    src = rng.normal(size=(segs[-1], K)) * np.exp(rng.normal(size=(segs[-1], 1)) * 3)
    q, s = mx.mxfp8_quantize(src, axis=1, seg_offsets=segs)
    assert s.shape[0] == mx.mxfp8_scale_rows(segs[-1], segs)
    sb = 0
    for g in range(len(segs) - 1):
        r0, r1 = segs[g], segs[g + 1]
        for b0 in range(r0, r1, 32):
            b1 = min(b0 + 32, r1)
            blk = np.zeros((32, K))
            blk[: b1 - b0] = src[b0:b1]
            qq, ss = mx.mxfp8_quantize(blk.T, axis=0)
            assert np.array_equal(q[b0:b1], qq.T[: b1 - b0])
            assert np.array_equal(s[sb], ss[:, 0])
            sb += 1
    deq = mx.mxfp8_dequantize(q, s, axis=1, seg_offsets=segs)
    assert np.linalg.norm(deq - src) / np.linalg.norm(src) < 0.05


def test_golden_blocks(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "mxfp8_blocks.json")))
    for b in fx["blocks"]:
        blk = np.zeros((1, 32))
        blk[0, : len(b["values"])] = b["values"]
        q, s = mx.mxfp8_quantize(blk, axis=0)
        assert int(s[0, 0]) == b["scale_byte"], b["note"]
        assert q[0, : len(b["codes"])].tolist() == b["codes"], b["note"]
        assert np.all(q[0, len(b["codes"]):] == 0)
