"""Pins of the oracle's NF4 format functions (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden_floats


def test_table_matches_published_levels():
    # The construction must reproduce the printed float32 code book bit for bit.
    pub = np.array(read_golden_floats("nf4_levels_qlora.txt"), dtype=np.float32)
    t = oracle.nf4_table()
    assert t.dtype == np.float32 and t.shape == (16,)
    assert np.array_equal(t.view(np.uint32), pub.view(np.uint32))


def test_table_invariants():
    t = oracle.nf4_table()
    assert t[0] == -1.0 and t[15] == 1.0 and t[7] == 0.0
    assert np.all(np.diff(t) > 0)
    assert (t < 0).sum() == 7 and (t > 0).sum() == 8


def test_table_levels_are_normal_quantiles_by_sampling():
    # Independent of the quantile function: the positive levels, rescaled by
    # the outermost quantile, sit at the empirical normal quantiles of
    # probabilities evenly spaced from 0.9677083 to 1/2.
    rng = np.random.default_rng(0)
    z = np.sort(rng.standard_normal(4_000_000))
    t = oracle.nf4_table().astype(np.float64)
    probs = np.linspace(0.9677083, 0.5, 9)[:-1]
    emp = np.quantile(z, probs)
    scale = emp[0]
    got = np.sort(t[8:])[::-1] * scale
    assert np.max(np.abs(got - emp)) < 4e-3


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * 10 ** rng.uniform(-30, 30, 200_000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, np.inf, -np.inf], dtype=np.float32),
        # exact ties: the dropped half is 0x8000
        (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ]).astype(np.float32)
    ours = oracle.bf16_round_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = oracle.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(vals).to(torch.bfloat16).float().numpy())


def test_nibble_order_and_block_index():
    t = oracle.nf4_table()
    packed = np.zeros((2, 64), dtype=np.uint8)  # 2 rows, K = 128 -> 2 blocks per row
    packed[0, 0] = 0x1F          # element 0 <- code 1 (high nibble), element 1 <- code 15
    packed[1, 40] = 0x70 | 0x3   # row 1: element 80 <- code 7, element 81 <- code 3
    absmax = np.array([[0.5, 2.0], [4.0, 0.25]], dtype=np.float32)
    bits, prod = oracle.dequantize_nf4(packed, absmax)
    assert prod.shape == (2, 128)
    assert prod[0, 0] == np.float32(t[1] * np.float32(0.5))
    assert prod[0, 1] == np.float32(t[15] * np.float32(0.5))
    assert prod[0, 2] == np.float32(t[0] * np.float32(0.5))   # zero byte -> code 0
    assert prod[0, 64] == np.float32(t[0] * np.float32(2.0))  # second block of row 0
    assert prod[1, 80] == 0.0
    assert prod[1, 81] == np.float32(t[3] * np.float32(0.25))  # element 81 is in block 1
    assert np.array_equal(bits, oracle.bf16_round_bits(prod))


def test_dequant_product_is_one_float32_multiply():
    rng = np.random.default_rng(2)
    packed = rng.integers(0, 256, (8, 32), dtype=np.uint8)
    absmax = rng.uniform(1e-3, 1.0, (8, 1)).astype(np.float32)
    _, prod = oracle.dequantize_nf4(packed, absmax)
    t = oracle.nf4_table()
    codes = np.stack([packed >> 4, packed & 15], axis=-1).reshape(8, 64)
    expect = np.float32(t[codes].astype(np.float64) * absmax.astype(np.float64)).astype(np.float32)
    # float64 product of two float32s is exact; rounding it once to float32 is
    # the correctly rounded float32 product.
    assert np.array_equal(prod, expect)


def test_quantise_round_trip_every_code():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (16, 128), dtype=np.uint8)
    codes[:, 0] = 15  # make the block maximum attain |T| = 1 so absmax is recovered
    codes[:, 64] = 0
    packed = ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)
    absmax = rng.uniform(1e-3, 10.0, (16, 2)).astype(np.float32)
    _, prod = oracle.dequantize_nf4(packed, absmax)
    p2, a2 = oracle.quantize_nf4(prod)
    assert np.array_equal(a2, absmax)
    assert np.array_equal(p2, packed)


def test_quantise_brute_force_and_error_bound():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((6, 192)) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize_nf4(w)
    t = oracle.nf4_table()
    codes = np.stack([packed >> 4, packed & 15], axis=-1).reshape(6, 192)
    for i in range(6):
        for kk in range(192):
            a = absmax[i, kk // 64]
            assert a == np.max(np.abs(w[i, (kk // 64) * 64:(kk // 64 + 1) * 64]))
            n = np.float32(w[i, kk] / a)
            d = [abs(np.float32(n - t[c])) for c in range(16)]
            assert codes[i, kk] == int(np.argmin(d))
    _, prod = oracle.dequantize_nf4(packed, absmax)
    max_gap = np.max(np.diff(t.astype(np.float64)))
    err = np.abs(prod.astype(np.float64) - w) / np.repeat(absmax, 64, axis=1)
    assert err.max() <= 0.5 * max_gap + 1e-6


def test_quantise_zero_block_and_tie():
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, 64] = 2.0
    t = oracle.nf4_table()
    # exact midpoint between levels 8 and 9 (after division by absmax 2.0)
    mid = np.float32((np.float64(t[8]) + np.float64(t[9])) / 2)
    w[0, 65] = np.float32(mid * 2.0)
    packed, absmax = oracle.quantize_nf4(w)
    assert absmax[0, 0] == 0.0 and absmax[0, 1] == 2.0
    codes = np.stack([packed >> 4, packed & 15], axis=-1).reshape(1, 128)
    assert np.all(codes[0, :64] == 7)
    assert codes[0, 64] == 15
    n = np.float32(w[0, 65] / np.float32(2.0))
    d8, d9 = abs(np.float32(n - t[8])), abs(np.float32(n - t[9]))
    assert codes[0, 65] == (8 if d8 <= d9 else 9)


@pytest.mark.parametrize("K", [64, 256])
def test_dequant_rejects_bad_absmax_shape(K):
    with pytest.raises(ValueError):
        oracle.dequantize_nf4(np.zeros((1, K // 2), np.uint8), np.zeros((1, K // 64 + 1), np.float32))


def _golden_ints(name):
    from conftest import golden_path
    out = {}
    for line in open(golden_path(name)):
        line = line.strip()
        if line and not line.startswith("#"):
            key, val = line.split()
            out[key] = int(val)
    return out


def test_storage_layout_matches_the_printed_stack_size():
    # The oracle's storage -- two codes per byte, one float32 absmax per 64 weights of a row -- applied to
    # a real model's expert stacks gives the byte count the pages print (16.31 GB). Double-quantised
    # scales or another block size would not.
    g = _golden_ints("qwen3_nf4_stack_bytes.txt")
    rng = np.random.default_rng(0)
    K = 256
    packed, absmax = oracle.quantize_nf4(rng.standard_normal((3, K)).astype(np.float32))
    bytes_per_weight = (packed.nbytes + absmax.nbytes) / (3 * K)
    weights = g["layers"] * g["experts"] * (2 * g["intermediate"] * g["hidden"] + g["hidden"] * g["intermediate"])
    assert round(weights * bytes_per_weight / 1e7) == g["hashed_gb_x100"]
    for alt in (0.5 + 4 / 32, 0.5 + 4 / 128, 0.5 + 1 / 64 + 4 / (64 * 256)):  # block 32, block 128, 8-bit scales
        assert round(weights * alt / 1e7) != g["hashed_gb_x100"]
