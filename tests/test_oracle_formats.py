"""Pins of the oracle's E4M3 / E2M1 decode and encode (no GPU).

Decode: all 256 E4M3 codes against PyTorch's float8_e4m3fn conversion (an
independent library routine) and hand-decoded points; all 16 E2M1 codes
against the MX-spec table.  Encode: every finite bf16 bit pattern times
2^k (k = -8..8) against a brute-force nearest-value search over the decoded
table with the even-code tie rule, plus hand-derived ties.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from synth.tensors import bf16_bits_to_f32


def test_e4m3_decode_exhaustive_vs_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # only S.1111.111
    assert np.array_equal(ref[~nan], got[~nan])
    # sign of zero
    assert math.copysign(1.0, got[0x80]) == -1.0


def test_e4m3_decode_golden_points(orc):
    for code, val in read_golden("e4m3_points.txt"):
        c = int(code, 16)
        v = orc.e4m3_decode(c)
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val), (code, v, val)
            assert math.copysign(1, v) == math.copysign(1, float(val))


def test_e2m1_decode_exhaustive_table(orc):
    rows = list(read_golden("e2m1_table.txt"))
    assert len(rows) == 16
    for code, val in rows:
        v = orc.e2m1_decode(int(code, 16))
        assert v == float(val)
        assert math.copysign(1, v) == math.copysign(1, float(val))


def _brute_force_encode(a: np.ndarray, table: np.ndarray, maxcode: int) -> np.ndarray:
    """Nearest non-negative table entry to |a|, ties to the even code,
    saturating above the largest entry; sign bit added separately."""
    mag = np.abs(a.astype(np.float64))
    d = np.abs(mag[:, None] - table[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    idx = np.argmax(cand, axis=1)  # lowest candidate code
    two = cand.sum(axis=1) == 2
    # when two codes are equally near, they are adjacent; keep the even one
    odd_low = (idx % 2) == 1
    idx = np.where(two & odd_low, idx + 1, idx)
    idx = np.where(mag > table[maxcode], maxcode, idx)
    return idx.astype(np.uint8)


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_f32(bits)
    return f[np.isfinite(f)]


@pytest.mark.parametrize("k", list(range(-8, 9)))
def test_e4m3_encode_bruteforce_all_bf16(orc, k):
    table = np.array([orc.e4m3_decode(c) for c in range(127)])  # 0 .. 448
    assert table[126] == 448.0 and np.all(np.diff(table) > 0)
    with np.errstate(over="ignore"):
        vals = (_all_finite_bf16().astype(np.float64) * 2.0 ** k).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    got = orc.e4m3_encode_array(vals)
    sign = (np.signbit(vals)).astype(np.uint8) << 7
    # chunk the brute force to bound memory
    exp = np.empty_like(got)
    for s in range(0, len(vals), 8192):
        exp[s:s + 8192] = _brute_force_encode(vals[s:s + 8192], table, 126)
    exp = exp | sign
    assert np.array_equal(got, exp)


@pytest.mark.parametrize("k", list(range(-8, 9)))
def test_e2m1_encode_bruteforce_all_bf16(orc, k):
    table = np.array([orc.e2m1_decode(c) for c in range(8)])
    with np.errstate(over="ignore"):
        vals = (_all_finite_bf16().astype(np.float64) * 2.0 ** k).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    got = orc.e2m1_encode_array(vals)
    sign = (np.signbit(vals)).astype(np.uint8) << 3
    exp = _brute_force_encode(vals, table, 7) | sign
    assert np.array_equal(got, exp)


def test_encode_golden_ties(orc):
    n = 0
    for fmt, val, code in read_golden("rounding_ties.txt"):
        enc = orc.e2m1_encode if fmt == "e2m1" else orc.e4m3_encode
        assert enc(float(val)) == int(code, 16), (fmt, val, code)
        n += 1
    assert n >= 20


def test_encode_decode_roundtrip(orc):
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert orc.e4m3_encode(orc.e4m3_decode(c)) == c
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_decode(c)) == c


def test_e4m3_encode_matches_torch_in_range(orc):
    # torch's float -> float8_e4m3fn is round-to-nearest-even and agrees with
    # the saturating encoder for |v| <= 448
    g = np.random.default_rng(7)
    v = (g.standard_normal(200000) * g.choice([1e-3, 0.1, 10, 100], 200000)).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.e4m3_encode_array(v), ref)
