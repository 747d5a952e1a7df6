"""Pins of the oracle's GEMM over decoded codes and its epilogues (no GPU).

Matmul: an exact rational (fractions.Fraction) triple loop on tiny shapes,
including one-hot operands; exactness of the binary64 FP8 accumulation
(``math.fsum`` -- the correctly rounded sum -- must agree bit for bit).
Epilogues: PyTorch's float64 GELU(tanh) and SiLU (independent library
routines), closed forms at 0, the gate = 0 residual identity and the split
boundary column.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from synth.tensors import bf16_bits_from_f64, bf16_bits_to_f32, draw


def _dec_tables(orc):
    l8 = [Fraction(orc.e4m3_decode(c)) if c not in (0x7F, 0xFF) else None for c in range(256)]
    l4 = [Fraction(orc.e2m1_decode(c)) for c in range(16)]
    return l8, l4


@pytest.mark.parametrize("M,N,K", [(3, 5, 16), (7, 4, 48), (1, 9, 32)])
def test_fp8_gemm_exact_triple_loop(orc, M, N, K):
    g = np.random.default_rng(M * 100 + N)
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qw = g.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x11  # no NaN codes
    qw[(qw & 0x7F) == 0x7F] = 0x22
    sa = np.array([2.0 ** -i * 1.5 for i in range(M)], np.float32)
    sw = np.array([2.0 ** -(i % 5) * 0.75 for i in range(N)], np.float32)
    y = orc.gemm_fp8(qa, sa, qw, sw)
    l8, _ = _dec_tables(orc)
    for i in range(M):
        for n in range(N):
            acc = sum((l8[qa[i, k]] * l8[qw[n, k]] for k in range(K)), Fraction(0))
            ref = acc * Fraction(float(sa[i])) * Fraction(float(sw[n]))
            assert y[i, n] == float(ref), (i, n)  # the scale products are exact here


def test_fp8_gemm_one_hot(orc):
    K, N = 64, 8
    qa = np.zeros((2, K), np.uint8)
    qa[0, 5] = 0x38   # 1.0
    qa[1, 63] = 0xB8  # -1.0
    qw = np.arange(N * K, dtype=np.int64).reshape(N, K).astype(np.uint8) & 0x77
    y = orc.gemm_fp8(qa, np.ones(2, np.float32), qw, np.ones(N, np.float32))
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(y[0], dec[qw[:, 5]])
    assert np.array_equal(y[1], -dec[qw[:, 63]])


def test_fp8_gemm_sum_is_exact(orc):
    # products of E4M3 values are multiples of 2^-18 below 448^2; with K = 12288
    # the binary64 sum stays exact, so it equals the correctly rounded fsum
    K, N = 12288, 6
    x = draw("student_t", (3, K), 1, "x", nu=3)
    w = draw("normal", (N, K), 1, "w", std=0.02)
    qa, sa = orc.quant_fp8_rows(x)
    qw, sw = orc.quant_fp8_rows(w)
    one = np.ones(3, np.float32)
    y = orc.gemm_fp8(qa, one, qw, np.ones(N, np.float32))
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    for i in range(3):
        for n in range(N):
            assert y[i, n] == math.fsum(dec[qa[i]] * dec[qw[n]])


def test_w8a16_gemm_one_hot(orc):
    # a bf16 one-hot row (value 1.0 at k) picks dec(qw[n, k]) * sw[n] exactly
    K, N = 64, 8
    x = np.zeros((2, K), np.uint16)
    x[0, 7] = 0x3F80   # 1.0
    x[1, 40] = 0xC000  # -2.0
    qw = (np.arange(N * K, dtype=np.int64).reshape(N, K) * 7 % 256).astype(np.uint8) & 0x77
    sw = np.array([2.0 ** -i for i in range(N)], np.float32)
    y = orc.gemm_w8a16(x, qw, sw)
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(y[0], dec[qw[:, 7]] * sw)
    assert np.array_equal(y[1], -2.0 * dec[qw[:, 40]] * sw)


@pytest.mark.parametrize("K", [48, 3072])
def test_w8a16_gemm_equals_fp8_gemm_on_fp8_valued_activations(orc, K):
    # bf16 activations that are E4M3 values times a power of two per row: the
    # weight-only GEMM must give exactly what the FP8 GEMM gives on the codes
    # (every product and both sums are exact in binary64)
    g = np.random.default_rng(K)
    M, N = 4, 5
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x31
    qw = g.integers(0, 256, (N, K), dtype=np.uint8)
    qw[(qw & 0x7F) == 0x7F] = 0x42
    sa = np.array([2.0 ** (-3 + i) for i in range(M)], np.float32)
    sw = g.uniform(0.5, 2.0, N).astype(np.float32)
    dec = np.array([orc.e4m3_decode(c) for c in range(256)])
    x = bf16_bits_from_f64(dec[qa] * sa[:, None].astype(np.float64))
    assert np.array_equal(bf16_bits_to_f32(x).astype(np.float64), dec[qa] * sa[:, None])
    assert np.array_equal(orc.gemm_w8a16(x, qw, sw), orc.gemm_fp8(qa, sa, qw, sw))


@pytest.mark.parametrize("M,N,K", [(2, 3, 32), (4, 2, 64)])
def test_nvfp4_gemm_exact_triple_loop(orc, M, N, K):
    g = np.random.default_rng(K + N)
    qa = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = g.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfa = g.integers(0, 0x7F, (M, K // 16), dtype=np.uint8)
    sfw = g.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
    Ga, Gw = np.float32(0.375), np.float32(2.0 ** -7)
    y = orc.gemm_nvfp4(qa, sfa, Ga, qw, sfw, Gw)
    l8, l4 = _dec_tables(orc)

    def elem(q, row, k):
        b = q[row, k // 2]
        return l4[(b >> 4) if k % 2 else (b & 15)]

    for i in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += (l8[sfa[i, k // 16]] * l8[sfw[n, k // 16]] * elem(qa, i, k) * elem(qw, n, k))
            ref = acc * Fraction(float(Ga)) * Fraction(float(Gw))
            assert y[i, n] == float(ref), (i, n)


def test_gemm_row_subset_matches_full(orc):
    x = draw("normal", (40, 128), 2, "x")
    w = draw("normal", (24, 128), 2, "w", std=0.02)
    qa, sa = orc.quant_fp8_rows(x)
    qw, sw = orc.quant_fp8_rows(w)
    full = orc.gemm_fp8(qa, sa, qw, sw)
    rows = np.array([39, 0, 17, 17])
    assert np.array_equal(orc.gemm_fp8(qa, sa, qw, sw, rows), full[rows])


def test_gelu_silu_vs_torch(orc):
    v = np.concatenate([np.linspace(-12, 12, 4001), [0.0, -0.0, 1e-8, -30, 30]])
    t = torch.from_numpy(v)
    g_ref = torch.nn.functional.gelu(t, approximate="tanh").numpy()
    s_ref = torch.nn.functional.silu(t).numpy()
    g = np.array([orc.gelu_tanh(a) for a in v])
    s = np.array([orc.silu(a) for a in v])
    # tanh saturates to -1 for v < -7 in binary64, so compare absolutely there
    assert np.allclose(g, g_ref, rtol=1e-13, atol=1e-14)
    assert np.allclose(s, s_ref, rtol=1e-13, atol=1e-14)
    assert orc.gelu_tanh(0.0) == 0.0 and orc.silu(0.0) == 0.0


def test_epilogue_kinds_closed_forms(orc):
    g = np.random.default_rng(3)
    y = g.standard_normal((5, 64))
    bias = draw("normal", (64,), 0, "bias", std=0.5)
    b = bf16_bits_to_f32(bias).astype(np.float64)
    out = orc.epilogue("bias", y, bias=bias)
    assert np.array_equal(out, y + b)
    out = orc.epilogue("bias_gelu", y, bias=bias)
    ref = torch.nn.functional.gelu(torch.from_numpy(y + b), approximate="tanh").numpy()
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-15)
    # swiglu: gate half first, up half second
    out = orc.epilogue("swiglu", y, bias=None)
    ref = torch.nn.functional.silu(torch.from_numpy(y[:, :32])).numpy() * y[:, 32:]
    assert out.shape == (5, 32) and np.allclose(out, ref, rtol=1e-13, atol=1e-15)
    # gated residual with gate = 0 returns the residual exactly
    res = draw("normal", (9, 64), 0, "residual")
    rows = np.array([8, 0, 3, 3, 1])
    zero_gate = np.zeros(64, np.uint16)
    out = orc.epilogue("bias_gated_residual", y, bias=bias, residual=res, gate=zero_gate, rows=rows)
    assert np.array_equal(out, bf16_bits_to_f32(res).astype(np.float64)[rows])
    one_gate = bf16_bits_from_f64(np.ones(64))
    out = orc.epilogue("bias_gated_residual", y, bias=bias, residual=res, gate=one_gate, rows=rows)
    assert np.array_equal(out, bf16_bits_to_f32(res).astype(np.float64)[rows] + (y + b))
    # split: columns < split_col bias only, >= split_col GELU
    out = orc.epilogue("split_bias_gelu", y, bias=bias, split_col=40)
    assert np.array_equal(out[:, :40], (y + b)[:, :40])
    ref = torch.nn.functional.gelu(torch.from_numpy(y + b), approximate="tanh").numpy()
    assert np.allclose(out[:, 40:], ref[:, 40:], rtol=1e-13, atol=1e-15)
    assert out[0, 39] == (y + b)[0, 39]
