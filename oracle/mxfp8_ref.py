"""Float64 oracle of MXFP8 block quantisation (E4M3 elements, E8M0 block scales).

TEST INFRASTRUCTURE ONLY (see the package docstring).

kongchang, section 吞吐量数字的边界条件 (boundary conditions of the throughput
numbers): MXFP8 is the Open Compute Project 8-bit microscaling format in which
every 32 elements share one scale factor; it cuts GEMM time, saved activations
and dispatch payload while an authoritative FP32 master weight is kept.  The
pages give no more than that.  The scale and rounding rule is the reading of
the OCP MX v1.0 conversion taken here:

* element format E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
  exponent 0 encodes subnormals ``m / 8 * 2**-6``; code 0x7F / 0xFF is NaN;
  there is no infinity; the largest finite magnitude is 448 = 1.75 * 2**8;
* per block V of 32 values: ``amax = max |V_i|``;
  ``e = floor(log2(amax)) - 8`` (8 is the exponent of E4M3's largest normal),
  clamped to [-127, 127]; ``amax == 0`` gives e = -127;
  scale byte (E8M0) ``= e + 127``;
* element code ``q_i = RNE_E4M3(V_i / 2**e)``: round to the nearest finite
  E4M3 value, ties to an even mantissa, magnitudes above 448 saturate to 448;
  the sign bit is the sign of V_i (so a negative value that rounds to zero
  gives 0x80);
* dequantised value ``= E4M3(q_i) * 2**e``.
"""

from __future__ import annotations

import numpy as np

__all__ = ["e4m3_decode", "e4m3_rne", "mx_block_exponent", "mxfp8_quantize",
           "mxfp8_dequantize", "mxfp8_scale_rows", "E4M3_MAX"]

E4M3_MAX = 448.0


def _decode_one(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    ex = (code >> 3) & 0xF
    m = code & 0x7
    if ex == 0xF and m == 0x7:
        return float("nan")
    if ex == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (ex - 7)


_TABLE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)
# finite non-negative magnitudes, codes 0x00 .. 0x7E, strictly increasing
_POS = _TABLE[:0x7F].copy()


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (NaN for 0x7F and 0xFF)."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_rne(v) -> np.ndarray:
    """Round float64 values to E4M3 codes: nearest, ties to even, saturating."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")          # _POS[hi] >= a
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(a == _POS[hi], hi, np.where(pick_hi, hi, lo))
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def mx_block_exponent(amax) -> np.ndarray:
    """Shared block exponent ``e = floor(log2(amax)) - 8`` clamped to [-127, 127]."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(amax)                 # amax = m * 2**ex, 0.5 <= m < 1
    e = (ex.astype(np.int64) - 1) - 8
    e = np.where(amax == 0, -127, e)
    return np.clip(e, -127, 127)


def _quantize_blocks(blocks):
    """blocks: [..., 32] float64 -> (codes [..., 32] u8, scale bytes [...] u8)."""
    amax = np.max(np.abs(blocks), axis=-1)
    e = mx_block_exponent(amax)
    scaled = np.ldexp(blocks, -e[..., None])
    return e4m3_rne(scaled), (e + 127).astype(np.uint8)


def mxfp8_scale_rows(rows: int, seg_offsets=None) -> int:
    """Number of scale rows that axis-1 quantisation produces."""
    if seg_offsets is None:
        return -(-rows // 32)
    seg = np.diff(np.asarray(seg_offsets, dtype=np.int64))
    return int(np.sum(-(-seg // 32)))


def mxfp8_quantize(src, axis: int = 0, seg_offsets=None):
    """MXFP8-quantise a [rows, K] matrix.

    axis 0: blocks of 32 consecutive elements along each row (K % 32 == 0);
    returns q [rows, K] u8 and scale [rows, K // 32] u8.

    axis 1: blocks of 32 consecutive rows within each column (the GEMM's K
    runs along the rows, as in a weight gradient whose K is the token axis).
    With ``seg_offsets`` (length nseg + 1) blocks restart at every segment
    start, and a segment's last partial block is padded with zeros (which
    leave amax unchanged); without it the whole matrix is one segment.
    Returns q [rows, K] u8 and scale [S, K] u8 where S is the total block
    count, segment by segment.
    """
    src = np.asarray(src, dtype=np.float64)
    rows, K = src.shape
    if axis == 0:
        if K % 32:
            raise ValueError("K must be a multiple of 32")
        q, s = _quantize_blocks(src.reshape(rows, K // 32, 32))
        return q.reshape(rows, K), s
    if axis != 1:
        raise ValueError("axis must be 0 or 1")
    if seg_offsets is None:
        seg_offsets = [0, rows]
    seg_offsets = np.asarray(seg_offsets, dtype=np.int64)
    q = np.zeros((rows, K), dtype=np.uint8)
    scales = []
    for g in range(len(seg_offsets) - 1):
        r0, r1 = int(seg_offsets[g]), int(seg_offsets[g + 1])
        for b0 in range(r0, r1, 32):
            b1 = min(b0 + 32, r1)
            blk = np.zeros((32, K))
            blk[: b1 - b0] = src[b0:b1]
            qb, sb = _quantize_blocks(blk.T)        # [K, 32], [K]
            q[b0:b1] = qb.T[: b1 - b0]
            scales.append(sb)
    scale = np.stack(scales) if scales else np.zeros((0, K), dtype=np.uint8)
    return q, scale.astype(np.uint8)


def mxfp8_dequantize(q, scale, axis: int = 0, seg_offsets=None) -> np.ndarray:
    """Inverse of ``mxfp8_quantize``: ``E4M3(q) * 2**(scale - 127)``."""
    q = np.asarray(q, dtype=np.uint8)
    scale = np.asarray(scale, dtype=np.int64)
    rows, K = q.shape
    vals = e4m3_decode(q)
    if axis == 0:
        e = np.repeat(scale - 127, 32, axis=1)
        return np.ldexp(vals, e)
    if seg_offsets is None:
        seg_offsets = [0, rows]
    seg_offsets = np.asarray(seg_offsets, dtype=np.int64)
    out = np.zeros((rows, K))
    sb = 0
    for g in range(len(seg_offsets) - 1):
        r0, r1 = int(seg_offsets[g]), int(seg_offsets[g + 1])
        for b0 in range(r0, r1, 32):
            b1 = min(b0 + 32, r1)
            out[b0:b1] = np.ldexp(vals[b0:b1], (scale[sb] - 127)[None, :])
            sb += 1
    return out
