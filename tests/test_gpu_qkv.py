"""GPU parity of the QKV epilogue (per-head RMS normalization of q and k with
learned weights, rotary embedding of their pairs, bias-only v) against the
oracle, element by element, within |gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref)."""
import numpy as np
import pytest

import oracle
from qlutil import assert_close, from_dev_bf16, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu

QL_ERR_INVALID_ARG = 1


def _bf16(a):
    b = np.asarray(a, np.float32).view(np.uint32)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _run(fmt, M, N, K, seed, variant, eps=1e-6):
    import torch
    import precision_gemm_qlinear_b200 as ql
    rng = np.random.default_rng(seed)
    x = draw("normal", (M, K), seed, "x", outlier_frac=0.01, outlier_factor=8.0)
    w = draw("normal", (N, K), seed, "w", std=0.02)
    b = draw("normal", (N,), seed, "bias", std=0.05)
    qw, kw = _bf16(rng.uniform(0.5, 1.5, 128)), _bf16(rng.uniform(0.5, 1.5, 128))
    theta = rng.uniform(-np.pi, np.pi, (M, 64))
    cos, sin = np.cos(theta).astype(np.float32), np.sin(theta).astype(np.float32)
    lay = ql.QLinear(fmt, "qkv_norm_rope", to_dev_bf16(w), to_dev_bf16(b), variant=variant)
    lay.set_qk_norm(to_dev_bf16(qw), to_dev_bf16(kw), eps)
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    lay.forward_rope(codes, scales, M, torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda(),
                     out)
    torch.cuda.synchronize()
    assert lay.check() == 0
    y = oracle.qlinear_reference(fmt, "bias", x, w)["y"]     # GEMM result, before any epilogue
    ref = oracle.qkv_norm_rope(y, b, qw, kw, cos, sin, D=128, eps=eps)
    return from_dev_bf16(out), ref


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "w8a16"])
def test_qkv_norm_rope_matches_oracle(fmt, variant):
    # 3 ragged M tiles (one CTA) / 2 pair tiles; q, k, v of two heads each
    got, ref = _run(fmt, 300, 768, 256, 21, variant)
    assert_close(got, ref)
    # the normalized heads really are normalized: rms / weight ~ 1 per head
    assert np.all(np.abs(np.sqrt(np.mean(ref[:, :512] ** 2, axis=1)) - 1.0) < 0.5)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "w8a16"])
def test_qkv_norm_rope_more_heads_and_tiles(fmt):
    got, ref = _run(fmt, 520, 1536, 512, 22, 0, eps=1e-3)
    assert_close(got, ref)


def test_qkv_layer_call_rules():
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    d = dummy.data_ptr()
    w = to_dev_bf16(draw("normal", (768, 256), 23, "w", std=0.02))
    qkv = ql.QLinear("fp8", "qkv_norm_rope", w)
    plain = ql.QLinear("fp8", "bias", w)
    # a QKV layer needs the rotary tables; other layers take none
    assert _abi.qlinear_forward(qkv.h, d, d, 64, None, None, d, 0, check=False) == QL_ERR_INVALID_ARG
    assert _abi.qlinear_forward_rope(plain.h, d, d, 64, d, d, d, 0, check=False) == QL_ERR_INVALID_ARG
    assert _abi.qlinear_set_qk_norm(plain.h, d, d, 1e-6, 0, check=False) == QL_ERR_INVALID_ARG
    assert _abi.qlinear_set_qk_norm(qkv.h, d, d, -1.0, 0, check=False) == QL_ERR_INVALID_ARG
