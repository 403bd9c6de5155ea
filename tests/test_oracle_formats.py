"""Pins of the oracle's element formats and block quantizers.

E4M3 and E8M0 are cross-checked against torch's own float8 types; E2M1 against
a brute-force nearest search; all three against hand values in
tests/golden/formats_hand_values.txt.  The MXFP8 scale rule and the NVFP4 scale
steps are pinned by closed forms, round trips and error bounds.
"""

import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "formats_hand_values.txt")


def _golden():
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                out.append(line.split())
    return out


def _num(s):
    return int(s, 16) if s.startswith("0x") else float(s)


def test_hand_values():
    for row in _golden():
        kind = row[0]
        if kind == "e4m3_decode":
            assert O.decode_e4m3(np.array([_num(row[1])]))[0] == _num(row[2])
        elif kind == "e4m3_encode":
            assert O.encode_e4m3(np.array([_num(row[1])]))[0] == _num(row[2])
        elif kind == "e2m1_encode":
            assert O.encode_e2m1(np.array([_num(row[1])]))[0] == _num(row[2])
        elif kind == "e8m0_decode":
            assert O.decode_e8m0(np.array([int(row[1])]))[0] == _num(row[2])
        elif kind == "mx_block":
            amax = float(row[1])
            blk = np.zeros((1, 32))
            blk[0, 5] = amax
            blk[0, 9] = amax / 4
            c, s = O.mxfp8_quantize(blk)
            assert int(s[0, 0]) == int(row[2]) and int(c[0, 5]) == _num(row[3])
        else:
            raise AssertionError(kind)


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.decode_e4m3(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_encode_matches_torch_in_range():
    # every bf16 value in [-448, 448], the midpoints of adjacent e4m3 values
    # (exact ties) and random fp32 values
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v)].astype(np.float64)
    mags = O.E4M3_MAG
    mids = (mags[1:] + mags[:-1]) / 2
    rnd = np.random.default_rng(3).uniform(-448, 448, 200000).astype(np.float32).astype(np.float64)
    v = np.concatenate([v, mids, -mids, rnd])
    v = v[np.isfinite(v) & (np.abs(v) <= 448)]
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.encode_e4m3(v)
    assert np.array_equal(ref, got)


def test_e4m3_saturates():
    v = np.array([448.0, 449.0, 463.9, 464.0, 1e6, -1e6])
    assert O.encode_e4m3(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_e8m0_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    got = O.decode_e8m0(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def _e2m1_from_definition(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_table_from_definition():
    for c in range(16):
        assert O.decode_e2m1(np.array([c]))[0] == _e2m1_from_definition(c)


def test_e2m1_encode_brute_force():
    vals = [_e2m1_from_definition(c) for c in range(8)]
    xs = np.concatenate([np.linspace(-8, 8, 4097), np.array(vals) + 0.0,
                         (np.array(vals[1:]) + np.array(vals[:-1])) / 2])
    for x in xs:
        a = min(abs(x), 6.0)
        d = [abs(a - vals[c]) for c in range(8)]
        best = min(d)
        cands = [c for c in range(8) if d[c] == best]
        c = [q for q in cands if q % 2 == 0][0] if len(cands) > 1 else cands[0]
        if np.signbit(x):
            c |= 8
        assert O.encode_e2m1(np.array([x]))[0] == c, x


def _rand_bf16(rng, shape, scale=1.0):
    return O.round_bf16(rng.normal(0, scale, shape))


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    v = rng.normal(0, 10, 100000).astype(np.float32)
    # exact ties: low 16 bits 0x8000
    ties = ((rng.integers(0, 2**31, 20000, dtype=np.uint32) & 0xFFFF0000) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    v = np.concatenate([v, ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().double().numpy()
    got = O.round_bf16(v.astype(np.float64))
    assert np.array_equal(ref, got)


def test_mxfp8_round_trip_and_bound():
    rng = np.random.default_rng(1)
    v = _rand_bf16(rng, (64, 256), 3.0)
    c, s = O.mxfp8_quantize(v)
    d = O.mxfp8_dequantize(c, s)
    X = O.decode_e8m0(s).repeat(32, axis=1)
    q = v / X
    # half an e4m3 spacing at |q| (spacing 2^(floor(log2|q|)-3), 2^-9 below 2^-6)
    _, e = np.frexp(np.maximum(np.abs(q), 2.0 ** -6))
    half = np.ldexp(1.0, e - 1 - 3 - 1)
    err = np.abs(d - v) / X
    sat = np.maximum(np.abs(q) - 448.0, 0)
    assert np.all(err <= np.maximum(half, sat) + 1e-12)
    # values exactly representable as code * scale round-trip exactly
    c2, s2 = O.mxfp8_quantize(d)
    assert np.array_equal(O.mxfp8_dequantize(c2, s2), d)


def test_mxfp8_constructed_round_trip():
    rng = np.random.default_rng(2)
    R, K = 16, 128
    scode = rng.integers(100, 140, (R, K // 32)).astype(np.uint8)
    codes = rng.integers(0, 0x7E, (R, K)).astype(np.uint8)
    codes |= (rng.integers(0, 2, (R, K)) << 7).astype(np.uint8)
    # force one element of each block into [256, 448] so the scale is the amax's
    codes.reshape(R, K // 32, 32)[:, :, 0] = rng.integers(0x78, 0x7F, (R, K // 32))
    v = O.mxfp8_dequantize(codes, scode)
    c2, s2 = O.mxfp8_quantize(v)
    assert np.array_equal(s2, scode)
    # +0 and -0 both decode to 0; compare values
    assert np.array_equal(O.decode_e4m3(c2), O.decode_e4m3(codes))


def test_mxfp8_zero_block():
    c, s = O.mxfp8_quantize(np.zeros((2, 64)))
    assert np.all(s == 127) and np.all(c == 0)


def test_nvfp4_global_scale():
    assert O.nvfp4_global_scale(2688.0) == np.float32(1.0)
    assert O.nvfp4_global_scale(448.0) == np.float32(6.0)
    assert O.nvfp4_global_scale(0.0) == np.float32(1.0)


def test_nvfp4_constructed_round_trip():
    rng = np.random.default_rng(4)
    R, K = 8, 64
    g = np.float32(4.0)
    sb = rng.integers(0x20, 0x60, (R, K // 16)).astype(np.uint8)
    codes = rng.integers(0, 16, (R, K)).astype(np.uint8)
    codes.reshape(R, K // 16, 16)[:, :, 3] = 7  # amax element +6 in every block
    v = O.nvfp4_dequantize(codes, sb, g)
    c2, s2 = O.nvfp4_quantize(v, g)
    assert np.array_equal(s2, sb)
    assert np.array_equal(O.decode_e2m1(c2), O.decode_e2m1(codes))


def test_nvfp4_hand_block():
    blk = np.zeros((1, 16))
    blk[0, :4] = [6.0, 2.5, -0.75, 1.25]
    c, s = O.nvfp4_quantize(blk, np.float32(1.0))
    assert s[0, 0] == 0x38
    assert c[0, :4].tolist() == [7, 4, 0xA, 2]


def test_nvfp4_error_bound():
    rng = np.random.default_rng(6)
    v = _rand_bf16(rng, (32, 512), 1.0)
    g = O.nvfp4_global_scale(np.abs(v).max())
    c, s = O.nvfp4_quantize(v, g)
    d = O.nvfp4_dequantize(c, s, g)
    dec_sb = O.decode_e4m3(s).repeat(16, axis=1)
    r = np.float64(g) / dec_sb
    q = np.abs(v) * r
    half = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0))
    sat = np.maximum(q - 6.0, 0)
    err = np.abs(d - v) * r
    assert np.all(err <= np.maximum(half, sat) * (1 + 1e-6) + 1e-9)


def test_quantize_commutes_with_permute():
    # Block scales run along K, so quantizing rows then gathering them equals
    # gathering rows then quantizing (MXFP8 codes; NVFP4 with a fixed global).
    rng = np.random.default_rng(8)
    x = _rand_bf16(rng, (40, 128), 1.0)
    row_token = np.array([3, 3, -1, 0, 39, 17, -1, 5])
    c, s = O.mxfp8_quantize(x)
    c1, s1 = O.mxfp8_quantize(O.gather_rows(x, row_token))
    assert np.array_equal(O.gather_rows(c, row_token), c1)
    assert np.array_equal(O.gather_rows(s, row_token)[row_token >= 0], s1[row_token >= 0])
    g = O.nvfp4_global_scale(np.abs(x).max())
    c, s = O.nvfp4_quantize(x, g)
    c1, s1 = O.nvfp4_quantize(O.gather_rows(x, row_token), g)
    assert np.array_equal(O.gather_rows(c, row_token), c1)
