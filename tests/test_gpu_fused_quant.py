"""GPU parity of the NVFP4-output epilogue (the next layer's activation
quantization fused into the producing GEMM).

The epilogue rounds each value to bf16 exactly as the bf16 path stores it and
quantizes that with a supplied tensor amax, so:
  * with the output's true amax its codes and scales are byte-identical to the
    standalone quantize kernel run on the bf16 output, and bit-exact against
    the oracle's NVFP4 quantization of that output (every epilogue);
  * with any other amax (here one that saturates) codes, block scales and G
    are bit-exact against the oracle's NVFP4 quantization of the same bf16
    values with that amax, and the recorded observed amax is max |output|.
"""
import numpy as np
import pytest

import oracle
from qlutil import sf_logical_offsets, sf_unswizzle, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu

QL_ERR_UNSUPPORTED = 3
# (epilogue, N, K): Nout = N (N/2 for SwiGLU) is a multiple of 256
CASES = [("bias", 768, 512), ("bias_gelu", 512, 256), ("swiglu", 1024, 512),
         ("bias_gated_residual", 512, 256), ("split_bias_gelu", 512, 256)]


def _layer_and_output(epi, M, N, K, seed, variant):
    import torch
    import precision_gemm_qlinear_b200 as ql
    x = draw("student_t", (M, K), seed, "x", nu=4)
    w = draw("normal", (N, K), seed, "w", std=0.02)
    b = draw("normal", (N,), seed, "bias", std=0.01)
    Nout = N // 2 if epi == "swiglu" else N
    res = gate = None
    if epi == "bias_gated_residual":
        res = to_dev_bf16(draw("normal", (M, Nout), seed, "residual"))
        gate = to_dev_bf16(draw("normal", (Nout,), seed, "gate", mean=1.0, std=0.1))
    lay = ql.QLinear("nvfp4", epi, to_dev_bf16(w), to_dev_bf16(b),
                     split_col=256 if epi == "split_bias_gelu" else 0, variant=variant)
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    y = torch.empty((M, Nout), dtype=torch.bfloat16, device="cuda")
    lay.forward_codes(codes, scales, M, y, res, gate)
    # a consumer layer with K = Nout sizes (and later reads) the fused output
    nxt = ql.QLinear("nvfp4", "bias", to_dev_bf16(draw("normal", (256, Nout), seed, "w2",
                                                      std=0.02)))
    torch.cuda.synchronize()
    return lay, nxt, codes, scales, y, res, gate


def _fused(lay, nxt, codes, scales, M, res, gate, amax_value):
    import torch
    qc, qs = nxt.act_buffers(M)
    qc.fill_(0xCD)
    qs.fill_(0xCD)
    amax = torch.tensor([amax_value], dtype=torch.float32, device="cuda")
    lay.forward_nvfp4_out(codes, scales, M, amax, qc, qs, res, gate)
    torch.cuda.synchronize()
    assert lay.check() == 0
    return qc, qs


def _bf16_bits(y):
    import torch
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def _amax_of(bits):
    """max |x| of a bf16 bit array, as float32 (exact)."""
    return np.float32(np.max(np.abs((bits.astype(np.uint32) << 16).view(np.float32))))


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("epi,N,K", CASES)
def test_fused_output_equals_quantize_kernel_at_true_amax(epi, N, K, variant):
    M = 300  # ragged: padded rows 300..383 of the last 128-row block
    lay, nxt, codes, scales, y, res, gate = _layer_and_output(epi, M, N, K, 5, variant)
    ybits = _bf16_bits(y)
    qc, qs = _fused(lay, nxt, codes, scales, M, res, gate, float(_amax_of(ybits)))
    rc, rs = nxt.act_buffers(M)
    nxt.quantize(y, rc, rs)
    import torch
    torch.cuda.synchronize()
    Nout = y.shape[1]
    nsf = ((M + 127) // 128) * ((Nout + 255) // 256) * 4 * 512
    assert np.array_equal(qc[: M * Nout // 2].cpu().numpy(), rc[: M * Nout // 2].cpu().numpy())
    # block scales (padding included), then G and the amax word of the tail
    assert np.array_equal(qs[: nsf + 8].cpu().numpy(), rs[: nsf + 8].cpu().numpy())
    # and directly against the oracle's NVFP4 quantization of the bf16 output
    oc, osf, og = oracle.quant_nvfp4(ybits)
    sb = qs.cpu().numpy()
    assert np.array_equal(qc[: M * Nout // 2].cpu().numpy().reshape(M, Nout // 2), oc)
    assert np.array_equal(sf_unswizzle(sb[:nsf], M, Nout), osf)
    assert sb[nsf:nsf + 4].view(np.uint32)[0] == np.float32(og).view(np.uint32)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("epi,N,K", [CASES[1], CASES[2]])
def test_fused_output_saturating_amax_matches_oracle(epi, N, K, variant):
    M = 300
    lay, nxt, codes, scales, y, res, gate = _layer_and_output(epi, M, N, K, 6, variant)
    ybits = _bf16_bits(y)
    true_amax = _amax_of(ybits)
    a_s = np.float32(0.3) * true_amax  # values above a_s saturate
    qc, qs = _fused(lay, nxt, codes, scales, M, res, gate, float(a_s))
    Nout = y.shape[1]
    oc, osf, og = oracle.quant_nvfp4(ybits, amax=float(a_s))
    nsf = ((M + 127) // 128) * ((Nout + 255) // 256) * 4 * 512
    sb = qs.cpu().numpy()
    assert np.array_equal(qc[: M * Nout // 2].cpu().numpy().reshape(M, Nout // 2), oc)
    assert np.array_equal(sf_unswizzle(sb[:nsf], M, Nout), osf)
    assert sb[nsf:nsf + 4].view(np.float32)[0].view(np.uint32) == np.float32(og).view(np.uint32)
    assert sb[nsf + 4:nsf + 8].view(np.uint32)[0] == np.float32(true_amax).view(np.uint32)
    mask = np.ones(nsf, bool)
    mask[sf_logical_offsets(M, Nout).ravel()] = False
    assert np.all(sb[:nsf][mask] == 0)
    assert np.any(osf == 0x7E)  # the case really saturates (E4M3 448)


def test_fused_output_feeds_the_next_layer():
    # the consumer's output from the fused buffers equals its output from the
    # standalone quantization of the bf16 tensor (same bytes in, same math)
    import torch
    M = 520
    lay, nxt, codes, scales, y, res, gate = _layer_and_output("bias_gelu", M, 512, 512, 7, 0)
    qc, qs = _fused(lay, nxt, codes, scales, M, res, gate, float(_amax_of(_bf16_bits(y))))
    rc, rs = nxt.act_buffers(M)
    nxt.quantize(y, rc, rs)
    o1 = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    nxt.forward_codes(qc, qs, M, o1)
    nxt.forward_codes(rc, rs, M, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_fused_output_rejects_unsupported_layers():
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    amax = torch.ones(1, dtype=torch.float32, device="cuda")
    for fmt, N in [("fp8", 512), ("nvfp4", 288)]:  # FP8 input; Nout % 256 != 0
        lay = ql.QLinear(fmt, "bias", to_dev_bf16(draw("normal", (N, 256), 8, "w", std=0.02)))
        s = _abi.qlinear_forward_nvfp4_out(lay.h, dummy.data_ptr(), dummy.data_ptr(), 64, None,
                                           None, amax.data_ptr(), dummy.data_ptr(),
                                           dummy.data_ptr(), 0, check=False)
        assert s == QL_ERR_UNSUPPORTED
        lay.close()
