"""GPU checks of the pre-quantized weight import and of per-batch adaLN gates.

* A layer built from the oracle's quantized weights (a stand-in for a
  pre-quantized checkpoint) computes exactly what the layer that quantized the
  same bf16 weights itself computes (the codes are bit-identical, so the
  outputs are equal element for element), and export -> import round-trips.
* Gated residual with one gate row per group of tokens matches the oracle
  applied group by group, with a group boundary inside a 32-row warp slab.
"""
import numpy as np
import pytest

import oracle
from qlutil import assert_close, from_dev_bf16, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu

QL_ERR_INVALID_ARG = 1


def _dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


@pytest.mark.parametrize("epi", ["bias_gelu", "swiglu"])
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_layer_from_oracle_quantized_weights_equals_self_quantized(fmt, epi):
    import torch
    import precision_gemm_qlinear_b200 as ql
    M, N, K = 300, 512, 512
    w = draw("normal", (N, K), 11, "w", std=0.02)
    b = draw("normal", (N,), 11, "bias", std=0.01)
    x = to_dev_bf16(draw("normal", (M, K), 11, "x"))
    ref_layer = ql.QLinear(fmt, epi, to_dev_bf16(w), to_dev_bf16(b))
    if fmt == "fp8":
        qw, sw = oracle.quant_fp8_rows(w)
        imp = ql.QLinear.from_quantized(fmt, epi, _dev_u8(qw), _dev_f32(sw), bias=to_dev_bf16(b))
    else:
        qw, sfw, gw = oracle.quant_nvfp4(w)
        imp = ql.QLinear.from_quantized(fmt, epi, _dev_u8(qw), _dev_u8(sfw), global_scale=gw,
                                        bias=to_dev_bf16(b))
    o1, o2 = ref_layer(x), imp(x)
    torch.cuda.synchronize()
    assert imp.check() == 0
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_export_then_import_round_trips(fmt):
    import torch
    import precision_gemm_qlinear_b200 as ql
    N, K = 768, 544 if fmt == "nvfp4" else 400
    w = draw("normal", (N, K), 12, "w", std=0.02)
    a = ql.QLinear(fmt, "swiglu", to_dev_bf16(w))
    codes, scales, g = a.export_weights()
    sc = _dev_f32(scales) if fmt == "fp8" else _dev_u8(scales)
    b = ql.QLinear.from_quantized(fmt, "swiglu", _dev_u8(codes), sc, global_scale=g)
    torch.cuda.synchronize()
    c2, s2, g2 = b.export_weights()
    assert np.array_equal(codes, c2)
    assert np.array_equal(np.asarray(scales).view(np.uint8), np.asarray(s2).view(np.uint8))
    assert np.float32(g).view(np.uint32) == np.float32(g2).view(np.uint32)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "w8a16"])
def test_gate_rows_match_oracle_per_group(fmt, variant):
    import torch
    import precision_gemm_qlinear_b200 as ql
    M, N, K, R = 300, 512, 256, 150   # two groups; the boundary splits rows 128..159
    x = draw("normal", (M, K), 13, "x")
    w = draw("normal", (N, K), 13, "w", std=0.02)
    b = draw("normal", (N,), 13, "bias", std=0.01)
    res = draw("normal", (M, N), 13, "residual")
    gates = draw("normal", (2, N), 13, "gate", mean=1.0, std=0.3)
    lay = ql.QLinear(fmt, "bias_gated_residual", to_dev_bf16(w), to_dev_bf16(b), variant=variant)
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    lay.forward_codes_gate_rows(codes, scales, M, out, to_dev_bf16(res), to_dev_bf16(gates), R)
    torch.cuda.synchronize()
    assert lay.check() == 0
    got = from_dev_bf16(out)
    for g in range(2):
        rows = np.arange(g * R, min(M, (g + 1) * R))
        ref = oracle.qlinear_reference(fmt, "bias_gated_residual", x, w, bias=b, residual=res,
                                       gate=gates[g], rows=rows)["out"]
        assert_close(got[rows], ref)


def test_gate_rows_and_import_reject_bad_arguments():
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _abi
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    w = to_dev_bf16(draw("normal", (256, 256), 14, "w", std=0.02))
    for epi, rows in [("bias_gated_residual", 0), ("bias", 64)]:
        lay = ql.QLinear("fp8", epi, w)
        s = _abi.qlinear_forward_gate_rows(lay.h, dummy.data_ptr(), dummy.data_ptr(), 64,
                                           dummy.data_ptr(), dummy.data_ptr(), rows,
                                           dummy.data_ptr(), 0, check=False)
        assert s == QL_ERR_INVALID_ARG
        lay.close()
    desc = _abi.make_desc("nvfp4", "bias", 256, 256, 0, 0)
    nbytes = _abi.qlinear_weight_bytes(desc)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s, _ = _abi.qlinear_create_prequantized(desc, dummy.data_ptr(), dummy.data_ptr(), -1.0, None,
                                            ws.data_ptr(), nbytes, 0, check=False)
    assert s == QL_ERR_INVALID_ARG
