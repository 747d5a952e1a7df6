"""The C-ABI library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import precision_gemm_qlinear_b200 as ql
from precision_gemm_qlinear_b200 import _abi


def _header_functions():
    src = open(os.path.join(ROOT, "include", "qlinear.h")).read()
    return sorted(set(re.findall(r"^QL_API\s+[\w\s\*]+?\b(qlinear_\w+)\s*\(", src, re.M)))


def test_header_declares_the_binding_exports():
    assert _header_functions() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = _abi.load()
    for name in _header_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version():
    assert ql.qlinear_abi_version() == 1
    assert ql.status_string(0) == "ok"
    assert "timed out" in ql.status_string(5)


@pytest.mark.parametrize("fmt,epi,N,K,ok", [
    ("fp8", "bias", 9216, 3072, True),
    ("fp8", "bias", 9216, 3070, False),      # K % 16
    ("fp8", "bias", 9200, 3072, False),      # N % 32
    ("nvfp4", "bias", 9216, 3072, True),
    ("nvfp4", "bias", 9216, 3056, False),    # K % 32
    ("nvfp4", "bias", 9248, 3072, True),     # N % 32 (ragged last tile)
    ("nvfp4", "swiglu", 9248, 3072, False),  # SwiGLU needs N % 256
    ("fp8", "swiglu", 16384, 3072, True),
    ("fp8", "swiglu", 16416, 3072, False),   # SwiGLU needs N % 256
    ("fp8", "bias", 0, 3072, False),
    ("fp8", "qkv_norm_rope", 9216, 3072, True),      # 3 x 24 heads of 128
    ("nvfp4", "qkv_norm_rope", 9216, 3072, True),
    ("fp8", "qkv_norm_rope", 9600, 3072, False),     # N % 768: q|k|v not tile-aligned
])
def test_weight_bytes_shape_rules(fmt, epi, N, K, ok):
    s, n = ql.qlinear_weight_bytes(ql.make_desc(fmt, epi, N, K), check=False)
    assert (s == 0) == ok
    if ok:
        code = N * K if fmt == "fp8" else N * K // 2
        assert n >= code + 2 * N


def test_unknown_epilogue_is_rejected():
    d = ql.make_desc("fp8", "bias", 512, 256)
    d.epi = 6
    s, _ = ql.qlinear_weight_bytes(d, check=False)
    assert s == _abi.QL_ERR_INVALID_ARG


def test_split_col_rules():
    s, _ = ql.qlinear_weight_bytes(ql.make_desc("fp8", "split_bias_gelu", 21504, 3072, 9216),
                                   check=False)
    assert s == 0
    s, _ = ql.qlinear_weight_bytes(ql.make_desc("fp8", "split_bias_gelu", 21504, 3072, 9217),
                                   check=False)
    assert s == _abi.QL_ERR_INVALID_ARG


def test_create_rejects_before_any_cuda_call():
    d = ql.make_desc("fp8", "bias", 512, 256)
    # null weight pointer
    s, h = ql.qlinear_create(d, None, None, 1 << 20, 1 << 30, check=False)
    assert s == _abi.QL_ERR_INVALID_ARG and not h
    # misaligned pointers
    s, h = ql.qlinear_create(d, 0x1008, None, 1 << 20, 1 << 30, check=False)
    assert s == _abi.QL_ERR_ALIGNMENT and not h
    s, h = ql.qlinear_create(d, 0x1000, None, 0x100080, 1 << 30, check=False)
    assert s == _abi.QL_ERR_ALIGNMENT and not h
    # workspace too small
    s, h = ql.qlinear_create(d, 0x1000, None, 0x100000, 16, check=False)
    assert s == _abi.QL_ERR_INVALID_ARG and not h
    # bad descriptor
    bad = ql.make_desc("fp8", "bias", 512, 256, flags=1)
    s, h = ql.qlinear_create(bad, 0x1000, None, 0x100000, 1 << 30, check=False)
    assert s == _abi.QL_ERR_INVALID_ARG
    bad = ql.make_desc("fp8", "bias", 512, 256, variant=3)
    s, h = ql.qlinear_create(bad, 0x1000, None, 0x100000, 1 << 30, check=False)
    assert s == _abi.QL_ERR_INVALID_ARG


def test_null_handle_calls():
    L = _abi.load()
    assert L.qlinear_quantize_act(None, None, 4, None, None, None) == _abi.QL_ERR_INVALID_ARG
    assert L.qlinear_forward(None, None, None, 4, None, None, None, None) == _abi.QL_ERR_INVALID_ARG
    assert L.qlinear_check(None, None) == _abi.QL_ERR_INVALID_ARG
    assert L.qlinear_destroy(None) == _abi.QL_ERR_INVALID_ARG
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.qlinear_act_bytes(None, 4, ctypes.byref(c), ctypes.byref(s)) == _abi.QL_ERR_INVALID_ARG


def test_binding_refuses_tensors_the_kernels_cannot_read():
    # checked in Python before any CUDA call: a host tensor, a wrong dtype or
    # a wrong shape never reaches a kernel as a pointer
    import pytest
    import torch
    import precision_gemm_qlinear_b200 as ql
    from precision_gemm_qlinear_b200 import _need
    with pytest.raises(TypeError, match="CUDA"):
        ql.QLinear("fp8", "bias", torch.zeros(256, 256, dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="CUDA"):
        ql.QLinear.from_quantized("fp8", "bias", torch.zeros(256, 256, dtype=torch.uint8),
                                  torch.ones(256))

    class FakeCuda:  # the checks only look at these attributes
        def __init__(self, dtype, shape, contiguous=True):
            self.is_cuda, self.dtype, self.shape = True, dtype, shape
            self._c = contiguous
            self.device = "cuda:0"

        def is_contiguous(self):
            return self._c

    _need(FakeCuda(torch.bfloat16, (8, 4)), "x", torch.bfloat16, (8, 4))
    with pytest.raises(TypeError, match="float32"):
        _need(FakeCuda(torch.float32, (8, 4)), "x", torch.bfloat16)
    with pytest.raises(ValueError, match="contiguous"):
        _need(FakeCuda(torch.bfloat16, (8, 4), contiguous=False), "x", torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        _need(FakeCuda(torch.bfloat16, (8, 5)), "gate", torch.bfloat16, (8, 4))
