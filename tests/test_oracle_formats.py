"""Pins for the oracle's storage formats (bf16, FP8 e4m3, FP4 e2m1).

The formats are fixed outside the pages: bf16 is the upper half of an IEEE
binary32, e4m3 is the OCP 8-bit floating-point "E4M3" encoding and e2m1 the
OCP microscaling FP4 element. The compressed cache is stored in FP8 and the
indexer path in FP4 (10100.com DeepSeek-V4 article, section 5; DeepSeek-V4
report digest, section 7), so the oracle decodes those bytes itself, from the
bit definitions; these tests check that decoding against torch's own
conversions and the specifications' value tables.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_decode_all_patterns_match_torch(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decode_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_named_points(orc):
    # OCP 8-bit FP spec, E4M3: max normal 448 (S.1111.110), min normal 2^-6,
    # min subnormal 2^-9, S.1111.111 is NaN, no infinities.
    assert orc.e4m3_to_f64(np.array([0x7E]))[0] == 448.0
    assert orc.e4m3_to_f64(np.array([0xFE]))[0] == -448.0
    assert orc.e4m3_to_f64(np.array([0x08]))[0] == 2.0 ** -6
    assert orc.e4m3_to_f64(np.array([0x01]))[0] == 2.0 ** -9
    assert np.isnan(orc.e4m3_to_f64(np.array([0x7F]))[0])
    assert orc.e4m3_to_f64(np.array([0x78]))[0] == 256.0


def _golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                code, v = line.split()
                vals[int(code, 2)] = float(v)
    return vals


def test_e2m1_decode_matches_spec_table(orc):
    table = _golden_e2m1()
    assert len(table) == 16
    for code, v in table.items():
        got = orc.e2m1_to_f64(np.array([code], np.uint8))[0]
        assert got == v and np.signbit(got) == np.signbit(v), (code, got, v)


def test_bf16_encode_matches_torch_rne(orc):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-39).astype(np.float32),  # subnormal range
        (rng.standard_normal(1000) * 1e30).astype(np.float32),
    ])
    # exact ties: low 16 bits 0x8000, upper bits odd and even
    hi = rng.integers(0x3000, 0x4F00, 1000).astype(np.uint32)
    ties = ((hi << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    got = orc.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_e4m3_encode_matches_torch_rne_in_range(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        (rng.standard_normal(3000) * 50).astype(np.float32),
        (rng.standard_normal(1000) * 1e-2).astype(np.float32),  # subnormals of e4m3
        rng.uniform(-448, 448, 1000).astype(np.float32),
    ])
    # every exact midpoint between consecutive finite e4m3 values (ties to even)
    vals = np.unique(torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy())
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    got = orc.f32_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates(orc):
    x = np.array([449.0, 464.0, 1e6, -500.0, np.float32(3e38)], np.float32)
    got = orc.e4m3_to_f64(orc.f32_to_e4m3(x))
    assert np.array_equal(got, [448.0, 448.0, 448.0, -448.0, 448.0])


def test_e2m1_encode_brute_force(orc):
    # nearest table value, ties to the even code (mantissa bit 0), saturating at 6
    table = _golden_e2m1()
    pos = sorted((v, c) for c, v in table.items() if c < 8)
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(-8, 8, 4000), np.arange(-7, 7.01, 0.25)]).astype(np.float32)
    got = orc.f32_to_e2m1(x)
    for xi, gi in zip(x, got):
        a = min(abs(float(xi)), 6.0)
        best = None
        for v, c in pos:
            d = abs(a - v)
            key = (d, c & 1)  # closer first, then even mantissa
            if best is None or key < best[0]:
                best = (key, c)
        want = best[1] | (8 if (xi < 0 or (xi == 0 and np.signbit(xi))) else 0)
        if best[1] == 0 and xi < 0:
            want = 8
        assert gi == want, (xi, gi, want)


def test_store_e4m3_rows_scale_rule(orc):
    rng = np.random.default_rng(3)
    v = rng.standard_normal((50, 96))
    v[7] = 0.0
    s = orc.store(v, orc.E4M3)
    amax = np.abs(v.astype(np.float32)).max(axis=1)
    want = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(s.scale, want)
    dec = orc.decode(s)
    # the element of largest magnitude maps to +-448 * scale
    r = np.arange(50)
    c = np.abs(v).argmax(axis=1)
    nz = amax > 0
    assert np.allclose(np.abs(dec[r, c])[nz], (448.0 * s.scale.astype(np.float64))[nz], rtol=0, atol=0)
    # round-to-nearest: error at most half a quantum (2^-4 relative) of the element
    err = np.abs(dec - v)
    assert np.all(err <= np.maximum(np.abs(v) * 2.0 ** -4, s.scale[:, None] * 2.0 ** -10) * 1.0000001)
    assert np.all(dec[7] == 0.0) and s.scale[7] == 1.0


def test_store_e2m1_blocks(orc):
    rng = np.random.default_rng(4)
    v = rng.standard_normal((20, 64))
    s = orc.store(v, orc.E2M1)
    assert s.data.shape == (20, 32) and s.scale.shape == (20, 4)
    dec = orc.decode(s)
    sc = orc.e4m3_to_f64(s.scale)  # [20, 4]
    for b in range(4):
        blk = slice(16 * b, 16 * b + 16)
        amax = np.abs(v[:, blk].astype(np.float32)).max(axis=1)
        want = orc.f32_to_e4m3((amax / np.float32(6.0)).astype(np.float32))
        assert np.array_equal(s.scale[:, b], want)
        q = dec[:, blk] / sc[:, b:b + 1]
        # every decoded element is scale x (an e2m1 value)
        table = np.array(sorted(set(abs(x) for x in _golden_e2m1().values())))
        assert np.all(np.isin(np.abs(np.round(q, 12)), table))
        # nearest e2m1 value of v/scale (ties aside): error at most the local half quantum
        r = np.clip(np.abs(v[:, blk]) / sc[:, b:b + 1], 0, 6)
        half_q = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
        assert np.all(np.abs(np.abs(q) - r) <= half_q + 1e-6)


def test_store_bf16_roundtrip(orc):
    rng = np.random.default_rng(5)
    v = rng.standard_normal((10, 33))
    s = orc.store(v, orc.BF16)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.decode(s), ref)
