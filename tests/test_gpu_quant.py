"""GPU parity of the activation / weight quantization kernels against the
oracle: codes, per-token scales, block scales and global scales must be
bit-exact (same binary32 operations, same rounding)."""
import numpy as np
import pytest

import oracle
from qlutil import sf_unswizzle, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu


def _layer(fmt, N, K, epi="bias", w=None):
    import precision_gemm_qlinear_b200 as ql
    if w is None:
        w = draw("normal", (N, K), 0, "w", std=0.02)
    return ql.QLinear(fmt, epi, to_dev_bf16(w)), w


@pytest.mark.parametrize("M,K", [(1, 16), (7, 48), (128, 256), (300, 3072), (129, 12288),
                                 (33, 12304), (64, 16)])
def test_fp8_act_quant_bitexact(M, K):
    import torch
    lay, _ = _layer("fp8", 256, K)
    x = draw("normal", (M, K), 1, "x", outlier_frac=0.01, outlier_factor=8.0)
    x[0, 0] = 0x8000  # -0
    if M > 2:
        x[2, :] = 0   # all-zero row
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    torch.cuda.synchronize()
    rc, rs = oracle.quant_fp8_rows(x)
    gc = codes[: M * K].cpu().numpy().reshape(M, K)
    gs = scales[: 4 * M].cpu().numpy().view(np.float32)
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(gc, rc)


# The block pass keeps 8, 6 or 4 steps of 256 elements in flight (the most
# that divide the row's full steps) and runs a remainder one step at a time;
# the shapes cover each depth with and without a remainder: 32 / 256 / 544
# (4, remainder only), 3072 (6), 3168 (6 + a partial step), 12288 (8),
# 8224 (8 + a partial step).
@pytest.mark.parametrize("M,K,dist", [(1, 32, "n"), (128, 256, "t"), (300, 3072, "t"),
                                      (257, 544, "n"), (64, 12288, "t"), (129, 3168, "t"),
                                      (40, 8224, "n")])
def test_nvfp4_act_quant_bitexact(M, K, dist):
    import torch
    lay, _ = _layer("nvfp4", 256, K)
    if dist == "t":
        x = draw("student_t", (M, K), 2, "x", nu=3, outlier_frac=0.005, outlier_factor=20.0)
    else:
        x = draw("normal", (M, K), 2, "x")
    x[0, 1] = 0x8000
    codes, scales = lay.act_buffers(M)
    scales.fill_(0xAB)  # padding scales must be rewritten as 0
    lay.quantize(to_dev_bf16(x), codes, scales)
    torch.cuda.synchronize()
    rc, rsf, rg = oracle.quant_nvfp4(x)
    gc = codes[: M * K // 2].cpu().numpy().reshape(M, K // 2)
    sb = scales.cpu().numpy()
    kch = ((K + 255) // 256) * 4
    nsf = ((M + 127) // 128) * kch * 512
    gsf = sf_unswizzle(sb[:nsf], M, K)
    gg = sb[nsf:nsf + 4].view(np.float32)[0]
    assert np.float32(gg).view(np.uint32) == np.float32(rg).view(np.uint32)
    assert np.array_equal(gsf, rsf)
    assert np.array_equal(gc, rc)
    # every padding scale byte (rows >= M, blocks >= K/16) is zero
    mask = np.ones(nsf, bool)
    r = np.arange(M)[:, None]
    b = np.arange(K // 16)[None, :]
    mask[(((r // 128) * kch + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4).ravel()] = False
    assert np.all(sb[:nsf][mask] == 0)


@pytest.mark.parametrize("fmt,epi,N,K", [("fp8", "bias", 512, 256), ("fp8", "swiglu", 768, 384),
                                         ("nvfp4", "bias", 512, 544), ("nvfp4", "swiglu", 1024, 256)])
def test_weight_quant_export_bitexact(fmt, epi, N, K):
    w = draw("normal", (N, K), 3, "w", std=0.02)
    lay, _ = _layer(fmt, N, K, epi=epi, w=w)
    codes, scales, g = lay.export_weights()
    if fmt == "fp8":
        rc, rs = oracle.quant_fp8_rows(w)
        assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))
    else:
        rc, rsf, rg = oracle.quant_nvfp4(w)
        assert np.array_equal(scales, rsf)
        assert np.float32(g).view(np.uint32) == np.float32(rg).view(np.uint32)
    assert np.array_equal(codes, rc)
