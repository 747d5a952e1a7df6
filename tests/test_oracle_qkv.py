"""Pins of the oracle's QKV epilogue (per-head RMS normalization of q and k,
rotary embedding of their pairs, bias-only v) against closed forms and
invariants that hold independently of the implementation (no GPU)."""
import numpy as np

import oracle

ONE = 0x3F80  # bf16 1.0


def _ones(d):
    return np.full(d, ONE, np.uint16)


def _bf16(a):
    """float array -> bf16 bit patterns (round to nearest even)."""
    b = np.asarray(a, np.float32).view(np.uint32)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _tables(rng, tokens, half):
    th = rng.uniform(-np.pi, np.pi, (tokens, half))
    return np.cos(th).astype(np.float32), np.sin(th).astype(np.float32), th


def test_hand_worked_example():
    # one head of D = 2: (3, 4) has rms sqrt(12.5); normalized (0.6 sqrt2, 0.8 sqrt2);
    # a quarter turn maps (a, b) to (-b, a); v = (1, 2) only gets its bias (0)
    y = np.array([[3.0, 4.0, 3.0, 4.0, 1.0, 2.0]])
    out = oracle.qkv_norm_rope(y, None, _ones(2), _ones(2), np.zeros((1, 1), np.float32),
                               np.ones((1, 1), np.float32), D=2, eps=0.0)
    s2 = np.sqrt(2.0)
    expect = np.array([[-0.8 * s2, 0.6 * s2, -0.8 * s2, 0.6 * s2, 1.0, 2.0]])
    assert np.allclose(out, expect, rtol=0, atol=1e-15)


def test_weight_applies_before_rotation():
    # (3, 4) normalized to (0.6, 0.8) sqrt2, times w = (2, 3) -> (1.2, 2.4) sqrt2,
    # then a quarter turn -> (-2.4, 1.2) sqrt2 (weighting after the turn would
    # give (-1.6, 1.8) sqrt2)
    y = np.array([[3.0, 4.0, 3.0, 4.0, 0.0, 0.0]])
    w = np.array([0x4000, 0x4040], np.uint16)  # bf16 2.0, 3.0
    out = oracle.qkv_norm_rope(y, None, w, w, np.zeros((1, 1), np.float32),
                               np.ones((1, 1), np.float32), D=2, eps=0.0)
    s2 = np.sqrt(2.0)
    assert np.allclose(out[0, :2], [-2.4 * s2, 1.2 * s2], rtol=0, atol=1e-14)


def test_normalized_heads_have_unit_rms_without_rotation():
    rng = np.random.default_rng(0)
    D, H, M = 128, 2, 5
    y = rng.normal(0, 3, (M, 3 * H * D))
    out = oracle.qkv_norm_rope(y, None, _ones(D), _ones(D), np.ones((M, D // 2), np.float32),
                               np.zeros((M, D // 2), np.float32), D=D, eps=0.0)
    for h in range(2 * H):
        seg = out[:, h * D:(h + 1) * D]
        assert np.allclose(np.sqrt(np.mean(seg ** 2, axis=1)), 1.0, rtol=1e-13)
    assert np.array_equal(out[:, 2 * H * D:], y[:, 2 * H * D:])  # v untouched (no bias)


def test_rotation_preserves_pair_norms_and_inverts():
    rng = np.random.default_rng(1)
    D, H, M = 128, 1, 4
    y = rng.normal(0, 1, (M, 3 * D))
    c, s, th = _tables(rng, M, D // 2)
    rot = oracle.qkv_norm_rope(y, None, _ones(D), _ones(D), c, s, D=D, eps=0.0)
    flat = oracle.qkv_norm_rope(y, None, _ones(D), _ones(D), np.ones_like(c), np.zeros_like(s),
                                D=D, eps=0.0)
    for h in range(2):
        a = rot[:, h * D:(h + 1) * D].reshape(M, D // 2, 2)
        b = flat[:, h * D:(h + 1) * D].reshape(M, D // 2, 2)
        assert np.allclose(np.hypot(a[..., 0], a[..., 1]), np.hypot(b[..., 0], b[..., 1]),
                           rtol=1e-6)
    # rotating the rotated heads back (their rms is already 1, so the second
    # normalization is the identity) returns the unrotated result; the tables
    # are fp32, so agreement is to fp32 precision
    back = oracle.qkv_norm_rope(rot, None, _ones(D), _ones(D), c, (-s).astype(np.float32), D=D,
                                eps=0.0)
    assert np.allclose(back[:, :2 * D], flat[:, :2 * D], rtol=0, atol=1e-6)


def test_scale_invariance_and_weights():
    rng = np.random.default_rng(2)
    D, M = 128, 3
    y = rng.normal(0, 1, (M, 3 * D))
    c, s, _ = _tables(rng, M, D // 2)
    w = _bf16(rng.uniform(0.5, 2.0, D))
    base = oracle.qkv_norm_rope(y, None, w, w, c, s, D=D, eps=0.0)
    for k in (-3, 5):   # a power-of-two scale changes nothing in q and k
        scaled = oracle.qkv_norm_rope(y * 2.0 ** k, None, w, w, c, s, D=D, eps=0.0)
        assert np.allclose(scaled[:, :2 * D], base[:, :2 * D], rtol=1e-14, atol=1e-15)
    # without rotation, the weight multiplies the normalized values
    plain = oracle.qkv_norm_rope(y, None, w, w, np.ones_like(c), np.zeros_like(s), D=D, eps=0.0)
    unit = oracle.qkv_norm_rope(y, None, _ones(D), _ones(D), np.ones_like(c), np.zeros_like(s),
                                D=D, eps=0.0)
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.allclose(plain[:, :D], unit[:, :D] * wf, rtol=1e-15)


def test_bias_is_added_before_normalization_and_to_v():
    rng = np.random.default_rng(3)
    D, M = 128, 2
    y = rng.normal(0, 1, (M, 3 * D))
    bias = _bf16(rng.normal(0, 0.5, 3 * D))
    bf = (bias.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    c1, s0 = np.ones((M, D // 2), np.float32), np.zeros((M, D // 2), np.float32)
    a = oracle.qkv_norm_rope(y, bias, _ones(D), _ones(D), c1, s0, D=D, eps=0.0)
    b = oracle.qkv_norm_rope(y + bf, None, _ones(D), _ones(D), c1, s0, D=D, eps=0.0)
    assert np.allclose(a, b, rtol=1e-15, atol=1e-15)
    assert np.array_equal(a[:, 2 * D:], y[:, 2 * D:] + bf[2 * D:])


def test_eps_enters_inside_the_square_root():
    # a head of constant value v: rms = |v|; out = v / sqrt(v^2 + eps)
    D, v, eps = 128, 0.001, 1e-6
    y = np.full((1, 3 * D), v)
    out = oracle.qkv_norm_rope(y, None, _ones(D), _ones(D), np.ones((1, D // 2), np.float32),
                               np.zeros((1, D // 2), np.float32), D=D, eps=eps)
    assert np.allclose(out[0, :D], v / np.sqrt(v * v + eps), rtol=1e-15)
