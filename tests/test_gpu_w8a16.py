"""GPU parity of the weight-only layer (bf16 activations, FP8-E4M3 weights
expanded to bf16 in shared memory, bf16 tensor-core MMAs) against the
oracle, element by element, within |gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref)."""
import numpy as np
import pytest

import oracle
from qlutil import assert_close, from_dev_bf16, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu

EPIS = ["bias", "bias_gelu", "swiglu", "bias_gated_residual", "split_bias_gelu"]


def _run(epi, M, N, K, seed, variant=0):
    import torch
    import precision_gemm_qlinear_b200 as ql
    x = draw("normal", (M, K), seed, "x", outlier_frac=0.01, outlier_factor=8.0)
    w = draw("normal", (N, K), seed, "w", std=0.02)
    b = draw("normal", (N,), seed, "bias", std=0.01)
    Nout = N // 2 if epi == "swiglu" else N
    sc = (N // 2) // 32 * 32 if epi == "split_bias_gelu" else 0
    gate = res = None
    if epi == "bias_gated_residual":
        gate = draw("normal", (Nout,), seed, "gate", mean=1.0, std=0.1)
        res = draw("normal", (M, Nout), seed, "residual")
    lay = ql.QLinear("w8a16", epi, to_dev_bf16(w), to_dev_bf16(b), split_col=sc, variant=variant)
    out = lay(to_dev_bf16(x), residual=None if res is None else to_dev_bf16(res),
              gate=None if gate is None else to_dev_bf16(gate))
    torch.cuda.synchronize()
    assert lay.check() == 0
    ref = oracle.qlinear_reference("w8a16", epi, x, w, bias=b, residual=res, gate=gate,
                                   split_col=sc)
    return from_dev_bf16(out), ref["out"]


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("epi", EPIS)
def test_w8a16_all_epilogues(epi, variant):
    got, ref = _run(epi, 300, 512, 512, 41, variant)
    assert_close(got, ref)


def test_w8a16_ragged_shapes():
    # K not a multiple of the 64-element stage, N not a multiple of the tile
    got, ref = _run("bias", 333, 288, 400, 42)
    assert_close(got, ref)


@pytest.mark.parametrize("epi", ["bias", "bias_gated_residual"])
@pytest.mark.parametrize("variant", [1, 2])
def test_w8a16_many_tiles_ragged_in_m_n_and_k(epi, variant):
    # M = 1100 ends in a partly filled row tile; N = 544 ends in a 32-column
    # ragged tile; K = 1088 is 17 stages, so the 5- (pairs) or 3-stage
    # (single CTAs) ring wraps several times, the converter warp that owns two
    # of the five stages alternates between them, and every converter warp
    # converts stages of several tiles
    got, ref = _run(epi, 1100, 544, 1088, 44, variant)
    assert_close(got, ref)


def test_w8a16_forward_takes_the_activations_directly():
    # the layer's "codes" are the bf16 activations themselves; scales may be NULL
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    M, N, K = 260, 512, 256
    x = to_dev_bf16(draw("normal", (M, K), 43, "x"))
    w = to_dev_bf16(draw("normal", (N, K), 43, "w", std=0.02))
    lay = ql.QLinear("w8a16", "bias", w)
    o1 = lay(x)
    o2 = torch.empty_like(o1)
    _abi.qlinear_forward(lay.h, x.data_ptr(), None, M, None, None, o2.data_ptr(), 0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_w8a16_weight_expansion_is_exact_for_every_code():
    # weight row n holds code (n + k) mod 256 at position k (NaN codes -> 0),
    # unit scales; activation row m is one-hot at k = 4 m, so out[m, n] must be
    # the E4M3 value of code (n + 4 m) mod 256 bit for bit (every E4M3 value,
    # subnormals included, is a bf16 value) -- for every code and for 16
    # positions spread over the 16-byte chunks of a stage
    import torch
    import precision_gemm_qlinear_b200 as ql
    N, K, M = 256, 64, 16
    codes = ((np.arange(N)[:, None] + np.arange(K)[None, :]) % 256).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0
    x = np.zeros((M, K), np.uint16)
    x[np.arange(M), 4 * np.arange(M)] = 0x3F80  # 1.0
    lay = ql.QLinear.from_quantized("w8a16", "bias", torch.from_numpy(codes).cuda(),
                                    torch.ones(N, dtype=torch.float32, device="cuda"))
    out = lay(to_dev_bf16(x))
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    dec = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float32)
    sel = codes[:, 4 * np.arange(M)].T
    want = (dec[sel].view(np.uint32) >> 16).astype(np.uint16)
    # code 0x80 is -0: summed with the +0 products of the other positions it
    # is +0, as IEEE addition gives
    want[sel == 0x80] = 0
    bad = sorted({int(c) for c in sel[got != want]})
    assert not bad, f"E4M3 codes expanded wrongly: {bad}"
