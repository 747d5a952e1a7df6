"""Pins of the oracle's per-token FP8 and two-level NVFP4 quantizers (no GPU).

Hand-derived worked rows (golden), closed-form special cases (all-zero rows,
the element that holds the amax), exact power-of-two scaling invariance, and
reconstruction-error bounds that follow from the formats' precision.
"""
import numpy as np
import pytest

from conftest import read_golden
from synth.tensors import bf16_bits_from_f64, bf16_bits_to_f32, draw


def _golden(name):
    d = {}
    for row in read_golden(name):
        d[row[0]] = row[1:]
    return d


def test_fp8_worked_row(orc):
    g = _golden("fp8_row_example.txt")
    x = bf16_bits_from_f64(np.array([float(v) for v in g["x"]]))[None, :]
    # the fixture's inputs are exact bf16 values
    assert np.array_equal(bf16_bits_to_f32(x)[0], np.array([float(v) for v in g["x"]], np.float32))
    codes, scales = orc.quant_fp8_rows(x)
    assert scales[0] == np.float32(float(g["scale"][0]))
    assert [int(c, 16) for c in g["codes"]] == codes[0].tolist()


def test_nvfp4_worked_row(orc):
    g = _golden("nvfp4_row_example.txt")
    vals = np.array([float(v) for v in g["x"]])
    x = bf16_bits_from_f64(vals)[None, :]
    x[0, 15] = 0x8000  # the fixture's -0
    codes, sf, G = orc.quant_nvfp4(x)
    assert np.float32(G).view(np.uint32) == int(g["G"][0], 16)
    assert sf[0].tolist() == [int(c, 16) for c in g["sf"]]
    assert codes[0].tolist() == [int(c, 16) for c in g["codes"]]


def test_fp8_zero_row_and_signed_zero(orc):
    x = np.zeros((2, 32), np.uint16)
    x[1, 3] = 0x8000
    codes, scales = orc.quant_fp8_rows(x)
    assert np.all(scales == 0)
    assert np.all(codes[0] == 0)
    assert codes[1, 3] == 0x80 and np.count_nonzero(codes[1]) == 1


@pytest.mark.parametrize("a", [1.0, 3.140625, 0.0009765625, 250.0, -7.5])
def test_fp8_one_hot_row_gives_max_code(orc, a):
    x = np.zeros((1, 48), np.uint16)
    x[0, 17] = bf16_bits_from_f64(np.array([a]))[0]
    codes, scales = orc.quant_fp8_rows(x)
    af = float(bf16_bits_to_f32(x[0, 17:18])[0])
    assert scales[0] == np.float32(abs(af)) / np.float32(448.0)
    assert codes[0, 17] == (0x7E | (0x80 if a < 0 else 0))
    assert np.count_nonzero(codes[0]) == 1


@pytest.mark.parametrize("k", [-20, -5, -1, 1, 3, 12])
def test_fp8_power_of_two_invariance(orc, k):
    x = draw("normal", (16, 256), 3, "x")
    xf = bf16_bits_to_f32(x).astype(np.float64)
    x2 = bf16_bits_from_f64(xf * 2.0 ** k)
    assert np.array_equal(bf16_bits_to_f32(x2).astype(np.float64), xf * 2.0 ** k)  # exact
    c1, s1 = orc.quant_fp8_rows(x)
    c2, s2 = orc.quant_fp8_rows(x2)
    assert np.array_equal(c1, c2)
    assert np.array_equal(s2.astype(np.float64), s1.astype(np.float64) * 2.0 ** k)


def test_fp8_reconstruction_bound(orc):
    x = draw("student_t", (64, 1024), 5, "x", nu=3, outlier_frac=0.01, outlier_factor=20)
    codes, s = orc.quant_fp8_rows(x)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    lut = np.array([orc.e4m3_decode(c) for c in range(256)])
    xr = lut[codes] * s[:, None].astype(np.float64)
    # E4M3 keeps 4 significant bits: relative rounding error <= 2^-4 in the
    # normal range, absolute <= 2^-10 (half the subnormal step) below it
    err = np.abs(xr - xf)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) * (1 + 1e-6) + 1e-30
    assert np.all(err <= bound)
    # the amax element of every row decodes to exactly 448 * s
    i = np.argmax(np.abs(xf), axis=1)
    assert np.all(np.abs(lut[codes[np.arange(64), i]]) == 448.0)


def test_nvfp4_zero_tensor(orc):
    x = np.zeros((3, 64), np.uint16)
    codes, sf, G = orc.quant_nvfp4(x)
    assert G == 0 and np.all(sf == 0) and np.all(codes == 0)


def test_nvfp4_amax_block_closed_form(orc):
    x = draw("normal", (8, 128), 11, "x")
    codes, sf, G = orc.quant_nvfp4(x)
    xf = bf16_bits_to_f32(x)
    A = np.abs(xf).max()
    assert G == np.float32(A) / np.float32(2688.0)
    r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    # the block holding the tensor amax gets scale code 448 and the amax
    # element gets E2M1 code 6 (magnitude)
    assert sf[r, c // 16] == 0x7E
    byte = codes[r, c // 2]
    nib = (byte >> 4) if (c % 2) else (byte & 15)
    assert (nib & 7) == 0x7


@pytest.mark.parametrize("k", [-12, -3, 2, 9])
def test_nvfp4_power_of_two_invariance(orc, k):
    x = draw("student_t", (8, 256), 13, "x", nu=4)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    x2 = bf16_bits_from_f64(xf * 2.0 ** k)
    c1, f1, g1 = orc.quant_nvfp4(x)
    c2, f2, g2 = orc.quant_nvfp4(x2)
    assert np.array_equal(c1, c2) and np.array_equal(f1, f2)
    assert float(g2) == float(g1) * 2.0 ** k


def test_nvfp4_reconstruction_bound(orc):
    x = draw("student_t", (32, 512), 17, "x", nu=4)
    codes, sf, G = orc.quant_nvfp4(x)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    l4 = np.array([orc.e2m1_decode(c) for c in range(16)])
    l8 = np.array([orc.e4m3_decode(c) for c in range(256)])
    q = np.empty(xf.shape, np.int64)
    q[:, 0::2] = codes & 15
    q[:, 1::2] = codes >> 4
    scale = l8[np.repeat(sf, 16, axis=1)] * float(G)
    xr = l4[q] * scale
    # one E2M1 step is at most 2 (between 4 and 6) in code units; RNE halves it,
    # and a block scale rounded down can push the top element past 6 by <= 2^-4
    # (block scales in the E4M3 subnormal range round coarser; excluded)
    err = np.abs(xr - xf)
    normal = np.repeat(sf, 16, axis=1) >= 0x08
    assert normal.mean() > 0.99
    assert np.all((err <= scale * (1.0 + 6 * 2.0 ** -4) + 1e-30)[normal])
    # blocks are scaled so that their amax lands near the top of the E2M1 range
    bmax = np.abs(xf).reshape(32, -1, 16).max(axis=2)
    top = np.abs(l4[q]).reshape(32, -1, 16).max(axis=2)
    assert np.all(top[(bmax > 0) & (sf >= 0x08)] >= 4.0)


def test_nvfp4_nibble_order(orc):
    # a row where every element is a distinct exactly representable value
    # under inv = 1 (A = 6 gives dec(448) * G = 1 for the amax block)
    row = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 0.0] * 2, np.float64)
    row[-1] = -6.0
    x = bf16_bits_from_f64(row)[None, :]
    codes, sf, G = orc.quant_nvfp4(x)
    assert sf[0, 0] == 0x7E
    assert codes[0].tolist() == [0x21, 0x43, 0x65, 0x07, 0x21, 0x43, 0x65, 0xF7]
