"""NF4 storage format: code book, dequantisation, quantisation (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Format, as the pages fix it and as read where they are silent:

* 4-bit packed fused expert stacks, two codes per byte, one float32 absmax
  per block of 64 consecutive elements of a row (package METADATA,
  §"The package family": the experts are packed 4-bit stacks, decoded in
  registers and summed in fp32; block size 64 and float32 absmax are the
  standard bitsandbytes NF4 defaults).
* Reading (pages silent): element ``2m`` of a row is the HIGH nibble of byte
  ``m`` and element ``2m+1`` the LOW nibble.
* Reading (pages silent): a block is 64 consecutive elements of one row of an
  expert's row-major matrix; rows are multiples of 64 long, so blocks never
  straddle rows, and absmax is laid out ``[E, rows, K/64]``.
* Reading (pages: "fp32 accumulation"): a weight dequantises to
  ``bf16_rn(float32(T[code]) * float32(absmax))`` -- one IEEE float32
  multiply, then round-to-nearest-even to bfloat16, the model dtype.  This
  bfloat16 value is the bit-exact quantity both sides must agree on.

Pins (tests/test_oracle_nf4.py): the table against the values printed in the
QLoRA paper's NF4 appendix and against its invariants; bf16 rounding against
torch's float32->bfloat16 conversion; nibble order on hand-built bytes;
quantise/dequantise round trip, brute-force argmin and error bound; the
storage's bytes per weight against the size of a frozen stack the pages print
(16.31 GB for a real model's expert stacks).
"""

from __future__ import annotations

import numpy as np
from scipy.special import ndtri

BLOCK = 64


def nf4_table() -> np.ndarray:
    """The 16 NormalFloat-4 levels as float32, ascending.

    Construction (QLoRA, NF4 data type): 8 positive levels at the standard
    normal quantiles of 8 probabilities spaced evenly from ``delta`` down to
    1/2 (the 1/2 end excluded), 7 negative levels mirrored from 7 quantiles
    spaced evenly over the same range, plus an exact zero; all divided by the
    largest so that the ends are -1 and +1.  ``delta = 1 - (1/30 + 1/32)/2``
    (the average of the outermost quantile positions of a 15- and a 16-level
    half) is 0.9677083 in float32.  The probability grid is evaluated in
    float32 from both ends (first half from ``delta``, second half from 1/2),
    the quantiles in float64 and rounded to float32, and the normalisation is
    a float32 division -- this reproduces the published float32 levels.
    """
    delta = np.float32(0.9677083)
    half = np.float32(0.5)

    def grid(n: int) -> np.ndarray:
        step = (half - delta) / np.float32(n - 1)
        pts = []
        for i in range(n):
            if i < n // 2:
                pts.append(delta + np.float32(i) * step)
            else:
                pts.append(half - np.float32(n - 1 - i) * step)
        return np.array(pts, dtype=np.float32)

    positive = ndtri(grid(9)[:-1].astype(np.float64))   # 8 levels
    negative = -ndtri(grid(8)[:-1].astype(np.float64))  # 7 levels
    levels = np.concatenate([positive, [0.0], negative]).astype(np.float32)
    levels = np.sort(levels)
    levels = (levels / levels.max()).astype(np.float32)
    return levels


def bf16_round_bits(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    if nan.any():
        r = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), r)
    return r


def bf16_bits_to_f32(b) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> the exactly equal float32 values."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def _unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes; element 2m = high nibble of byte m."""
    packed = np.asarray(packed, dtype=np.uint8)
    hi = packed >> 4
    lo = packed & 0x0F
    codes = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    codes[..., 0::2] = hi
    codes[..., 1::2] = lo
    return codes


def dequantize_nf4(packed: np.ndarray, absmax: np.ndarray):
    """Dequantise rows of packed NF4 codes.

    ``packed``: uint8 ``[..., K/2]``; ``absmax``: float32 ``[..., K/64]``.
    Returns ``(bf16_bits uint16 [..., K], product float32 [..., K])`` where
    ``product = float32(T[code]) * float32(absmax[block])`` (one float32
    multiply) and ``bf16_bits`` is its round-to-nearest-even bfloat16.
    """
    table = nf4_table()
    codes = _unpack_codes(packed)
    K = codes.shape[-1]
    absmax = np.asarray(absmax, dtype=np.float32)
    if absmax.shape[-1] * BLOCK != K:
        raise ValueError("absmax has %d blocks for K=%d" % (absmax.shape[-1], K))
    scale = np.repeat(absmax, BLOCK, axis=-1)
    product = (table[codes] * scale).astype(np.float32)
    return bf16_round_bits(product), product


def dequantize_nf4_matrix(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """The dequantised bfloat16 weights widened exactly to float64."""
    bits, _ = dequantize_nf4(packed, absmax)
    return bf16_bits_to_f32(bits).astype(np.float64)


def quantize_nf4(w: np.ndarray):
    """Blockwise NF4 quantisation of float32 rows ``[..., K]`` (K % 64 == 0).

    Per block of 64: ``absmax = max |w|``; each element's code is the level
    nearest to ``w / absmax`` (float32 division, float32 distance, an exact
    tie goes to the lower code).  A block of zeros gets absmax 0 and the code
    of the level 0.0.  Returns ``(packed uint8 [..., K/2], absmax float32
    [..., K/64])``.  Used only to prepare test data.
    """
    table = nf4_table()
    w = np.asarray(w, dtype=np.float32)
    K = w.shape[-1]
    if K % BLOCK:
        raise ValueError("K must be a multiple of 64")
    blocks = w.reshape(w.shape[:-1] + (K // BLOCK, BLOCK))
    absmax = np.abs(blocks).max(axis=-1).astype(np.float32)
    safe = np.where(absmax > 0, absmax, np.float32(1.0)).astype(np.float32)
    normed = (blocks / safe[..., None]).astype(np.float32)
    dist = np.abs(normed[..., None] - table).astype(np.float32)
    codes = np.argmin(dist, axis=-1).astype(np.uint8)  # first minimum = lower code
    zero_code = np.uint8(int(np.flatnonzero(table == 0.0)[0]))
    codes = np.where((absmax > 0)[..., None], codes, zero_code).astype(np.uint8)
    codes = codes.reshape(w.shape)
    packed = ((codes[..., 0::2] << 4) | codes[..., 1::2]).astype(np.uint8)
    return packed, absmax
