"""Allocation-free activation quantization, qlinear_quantize_act_noalloc.

Some callers cannot allocate device memory: code running inside another
framework's memory pool, an operator plugin that is handed only its input and
output tensors, or a graph-replay path that must not touch the allocator.  The
allocation-free entry point keeps its working memory (the NVFP4 amax partials)
in an array inside the library.  These tests call it through the C ABI two
times in a row, with different inputs and sizes, and check that it produces
exactly what qlinear_quantize_act produces (codes and scales are integer and
bit patterns, so the tolerance is exact equality), and that the GEMM on its
output stays within the parity tolerance of the oracle-checked path.  This
file is collected last on purpose.
"""
import numpy as np
import pytest

from qlutil import assert_close, from_dev_bf16, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu


def _run_both(lay, x, M):
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    stream = torch.cuda.current_stream().cuda_stream
    ca, sa = lay.act_buffers(M)
    cb, sb = lay.act_buffers(M)
    cb.fill_(0xAB)
    sb.fill_(0xCD)
    ql.qlinear_quantize_act(lay.h, x.data_ptr(), M, ca.data_ptr(), sa.data_ptr(), stream)
    _abi.qlinear_quantize_act_noalloc(lay.h, x.data_ptr(), M, cb.data_ptr(), sb.data_ptr(), stream)
    torch.cuda.synchronize()
    return ca, sa, cb, sb


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
def test_noalloc_matches_quantize_act_twice_in_a_row(fmt):
    import torch
    import precision_gemm_qlinear_b200 as ql
    K, N = 512, 512
    w = draw("normal", (N, K), 21, "w", std=0.02)
    b = draw("normal", (N,), 21, "bias", std=0.01)
    lay = ql.QLinear(fmt, "bias", to_dev_bf16(w), to_dev_bf16(b))
    # second call is smaller and has a larger amax: stale partials from the
    # first call would change the global scale
    for M, seed, scale in ((300, 31, 1.0), (129, 32, 4.0)):
        xh = draw("student_t", (M, K), seed, "x", nu=3)
        x = to_dev_bf16(xh) * scale
        ca, sa, cb, sb = _run_both(lay, x, M)
        ncode = M * K // 2 if fmt == "nvfp4" else M * K
        assert np.array_equal(ca[:ncode].cpu().numpy(), cb[:ncode].cpu().numpy())
        if fmt == "nvfp4":
            kch = ((K + 255) // 256) * 4
            nsf = ((M + 127) // 128) * kch * 512
            # block scales and the fp32 global scale; the amax word after them
            # is working memory of the other entry point only
            nbytes = nsf + 4
        else:
            nbytes = 4 * M
        assert np.array_equal(sa[:nbytes].cpu().numpy(), sb[:nbytes].cpu().numpy())
        # the GEMM on the allocation-free output matches the regular path
        out_a = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        out_b = torch.empty_like(out_a)
        lay.forward_codes(ca, sa, M, out_a)
        lay.forward_codes(cb, sb, M, out_b)
        torch.cuda.synchronize()
        assert lay.check() == 0
        assert_close(from_dev_bf16(out_b), from_dev_bf16(out_a), f"noalloc {fmt} M={M}")
    lay.close()


@pytest.mark.parametrize("M,K", [(4608, 3072), (257, 96)])
def test_noalloc_matches_quantize_act_at_flux_and_ragged_k(M, K):
    # the FLUX hidden size, and a K that is a multiple of 32 but not of 256
    # (the last 256-element stage holds padding blocks with zero scales)
    import precision_gemm_qlinear_b200 as ql
    w = draw("normal", (256, K), 23, "w", std=0.02)
    lay = ql.QLinear("nvfp4", "bias", to_dev_bf16(w))
    x = to_dev_bf16(draw("student_t", (M, K), 33, "x", nu=3, outlier_frac=0.005,
                         outlier_factor=20.0))
    ca, sa, cb, sb = _run_both(lay, x, M)
    kch = ((K + 255) // 256) * 4
    nsf = ((M + 127) // 128) * kch * 512
    assert np.array_equal(ca[: M * K // 2].cpu().numpy(), cb[: M * K // 2].cpu().numpy())
    assert np.array_equal(sa[: nsf + 4].cpu().numpy(), sb[: nsf + 4].cpu().numpy())
    lay.close()


def test_noalloc_at_the_row_maximum():
    # M == QL_NOALLOC_MAX_ROWS with a small K (32 MB of activations): the
    # largest accepted call, bit for bit the regular entry point's output
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    M, K = _abi.QL_NOALLOC_MAX_ROWS, 32
    w = draw("normal", (256, K), 24, "w", std=0.02)
    lay = ql.QLinear("nvfp4", "bias", to_dev_bf16(w))
    x = to_dev_bf16(draw("normal", (M, K), 34, "x"))
    ca, sa, cb, sb = _run_both(lay, x, M)
    nsf = (M // 128) * 4 * 512
    assert np.array_equal(ca[: M * K // 2].cpu().numpy(), cb[: M * K // 2].cpu().numpy())
    assert np.array_equal(sa[: nsf + 4].cpu().numpy(), sb[: nsf + 4].cpu().numpy())
    lay.close()


def test_noalloc_rejects_rows_beyond_the_maximum():
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    w = draw("normal", (256, 256), 22, "w", std=0.02)
    lay = ql.QLinear("nvfp4", "bias", to_dev_bf16(w))
    s = _abi.qlinear_quantize_act_noalloc(lay.h, None, _abi.QL_NOALLOC_MAX_ROWS + 1, None, None, 0,
                                          check=False)
    assert s == _abi.QL_ERR_INVALID_ARG
    assert "invalid" in ql.status_string(s)
    lay.close()
