"""CPU oracle for the quantized linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product library never does.

The arithmetic lives in ``qlinear_oracle.c`` (plain C, binary32 steps with
round-to-nearest-even, binary64 matmul and epilogue); this module only
marshals numpy arrays through ctypes.  Each function names the passage it
follows in the C source.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None

EPI = {"bias": 0, "bias_gelu": 1, "swiglu": 2, "bias_gated_residual": 3, "split_bias_gelu": 4}


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.or_e4m3_decode.restype = ctypes.c_double
        L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e2m1_decode.restype = ctypes.c_double
        L.or_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.or_e4m3_encode.restype = ctypes.c_uint8
        L.or_e4m3_encode.argtypes = [ctypes.c_float]
        L.or_e2m1_encode.restype = ctypes.c_uint8
        L.or_e2m1_encode.argtypes = [ctypes.c_float]
        L.or_e4m3_encode_n.argtypes = [P, i64, P]
        L.or_e2m1_encode_n.argtypes = [P, i64, P]
        L.or_quant_fp8_rows.argtypes = [P, i64, i64, P, P]
        L.or_tensor_amax.restype = ctypes.c_float
        L.or_tensor_amax.argtypes = [P, i64]
        L.or_quant_nvfp4.argtypes = [P, i64, i64, ctypes.c_float, P, P, P]
        L.or_gemm_fp8.argtypes = [P, P, P, P, i64, i64, P, i64, P]
        L.or_gemm_nvfp4.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, i64, i64, P,
                                    i64, P]
        L.or_epilogue.argtypes = [ctypes.c_int, P, i64, i64, P, P, P, P, i64, P]
        L.or_gemm_w8a16.argtypes = [P, P, P, i64, i64, P, i64, P]
        L.or_qkv_norm_rope.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, ctypes.c_double, P]
        L.or_gelu_tanh.restype = ctypes.c_double
        L.or_gelu_tanh.argtypes = [ctypes.c_double]
        L.or_silu.restype = ctypes.c_double
        L.or_silu.argtypes = [ctypes.c_double]
        L.or_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().or_num_threads())


def e4m3_decode(code: int) -> float:
    return float(lib().or_e4m3_decode(code & 0xFF))


def e2m1_decode(code: int) -> float:
    return float(lib().or_e2m1_decode(code & 0xF))


def e4m3_encode(v: float) -> int:
    return int(lib().or_e4m3_encode(float(v)))


def e2m1_encode(v: float) -> int:
    return int(lib().or_e2m1_encode(float(v)))


def e4m3_encode_array(v) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.empty(flat.size, np.uint8)
    lib().or_e4m3_encode_n(_p(flat), flat.size, _p(out))
    return out.reshape(np.shape(v))


def e2m1_encode_array(v) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.empty(flat.size, np.uint8)
    lib().or_e2m1_encode_n(_p(flat), flat.size, _p(out))
    return out.reshape(np.shape(v))


def quant_fp8_rows(x_bf16: np.ndarray):
    """Per-token FP8 quantization (C: or_quant_fp8_rows).  x_bf16: uint16 [rows, K]."""
    x = _c(x_bf16, np.uint16)
    rows, K = x.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty(rows, np.float32)
    lib().or_quant_fp8_rows(_p(x), rows, K, _p(codes), _p(scales))
    return codes, scales


def tensor_amax(x_bf16: np.ndarray) -> float:
    x = _c(x_bf16, np.uint16)
    return float(np.float32(lib().or_tensor_amax(_p(x), x.size)))


def quant_nvfp4(x_bf16: np.ndarray, amax: float = None):
    """Two-level NVFP4 quantization (C: or_quant_nvfp4).

    Returns (codes uint8 [rows, K/2], sf uint8 [rows, K/16] logical order, G float32).
    """
    x = _c(x_bf16, np.uint16)
    rows, K = x.shape
    assert K % 16 == 0
    if amax is None:
        amax = tensor_amax(x)
    codes = np.empty((rows, K // 2), np.uint8)
    sf = np.empty((rows, K // 16), np.uint8)
    G = np.zeros(1, np.float32)
    lib().or_quant_nvfp4(_p(x), rows, K, ctypes.c_float(amax), _p(codes), _p(sf), _p(G))
    return codes, sf, np.float32(G[0])


def gemm_fp8(qa, sa, qw, sw, rows=None):
    """y = (sum_k dec(qa) dec(qw)) * sa * sw over the listed rows (C: or_gemm_fp8)."""
    qa = _c(qa, np.uint8)
    qw = _c(qw, np.uint8)
    sa = _c(sa, np.float32)
    sw = _c(sw, np.float32)
    K = qa.shape[1]
    N = qw.shape[0]
    assert qw.shape[1] == K
    rows = np.arange(qa.shape[0], dtype=np.int64) if rows is None else _c(rows, np.int64)
    y = np.empty((len(rows), N), np.float64)
    lib().or_gemm_fp8(_p(qa), _p(sa), _p(qw), _p(sw), K, N, _p(rows), len(rows), _p(y))
    return y


def gemm_w8a16(x_bf16, qw, sw, rows=None):
    """y = (sum_k x dec(qw)) * sw over the listed rows, x left in bf16
    (weight-only quantization; C: or_gemm_w8a16)."""
    x = _c(x_bf16, np.uint16)
    qw = _c(qw, np.uint8)
    sw = _c(sw, np.float32)
    K = x.shape[1]
    N = qw.shape[0]
    assert qw.shape[1] == K
    rows = np.arange(x.shape[0], dtype=np.int64) if rows is None else _c(rows, np.int64)
    y = np.empty((len(rows), N), np.float64)
    lib().or_gemm_w8a16(_p(x), _p(qw), _p(sw), K, N, _p(rows), len(rows), _p(y))
    return y


def gemm_nvfp4(qa, sfa, Ga, qw, sfw, Gw, rows=None):
    """Block-scaled NVFP4 GEMM over the listed rows (C: or_gemm_nvfp4)."""
    qa = _c(qa, np.uint8)
    qw = _c(qw, np.uint8)
    sfa = _c(sfa, np.uint8)
    sfw = _c(sfw, np.uint8)
    K = qa.shape[1] * 2
    N = qw.shape[0]
    rows = np.arange(qa.shape[0], dtype=np.int64) if rows is None else _c(rows, np.int64)
    y = np.empty((len(rows), N), np.float64)
    lib().or_gemm_nvfp4(_p(qa), _p(sfa), ctypes.c_float(Ga), _p(qw), _p(sfw), ctypes.c_float(Gw),
                        K, N, _p(rows), len(rows), _p(y))
    return y


def epilogue(kind: str, y, bias=None, residual=None, gate=None, rows=None, split_col=0):
    """Fused epilogue in binary64 (C: or_epilogue).  Returns the pre-bf16 reference."""
    y = _c(y, np.float64)
    nrows, N = y.shape
    k = EPI[kind]
    Nout = N // 2 if kind == "swiglu" else N
    rows = np.arange(nrows, dtype=np.int64) if rows is None else _c(rows, np.int64)
    bias = None if bias is None else _c(bias, np.uint16)
    residual = None if residual is None else _c(residual, np.uint16)
    gate = None if gate is None else _c(gate, np.uint16)
    out = np.empty((nrows, Nout), np.float64)
    lib().or_epilogue(k, _p(y), nrows, N, _p(bias), _p(residual), _p(rows), _p(gate),
                      int(split_col), _p(out))
    return out


def qkv_norm_rope(y, bias, qw, kw, rope_cos, rope_sin, D=128, eps=1e-6, rows=None):
    """QKV epilogue with per-head RMS normalization of q and k and rotary
    embedding of their pairs (C: or_qkv_norm_rope).  y [nrows, 3*H*D]
    (binary64, e.g. the GEMM result of the listed rows); bias bf16 [N] or None;
    qw, kw bf16 [D]; rope_cos, rope_sin fp32 [tokens, D/2] indexed by rows.
    Returns the pre-bf16 reference [nrows, N]."""
    y = _c(y, np.float64)
    nrows, N = y.shape
    assert N % (3 * D) == 0 and D % 2 == 0
    rows = np.arange(nrows, dtype=np.int64) if rows is None else _c(rows, np.int64)
    bias = None if bias is None else _c(bias, np.uint16)
    qw, kw = _c(qw, np.uint16), _c(kw, np.uint16)
    rc, rs = _c(rope_cos, np.float32), _c(rope_sin, np.float32)
    out = np.empty((nrows, N), np.float64)
    lib().or_qkv_norm_rope(_p(y), nrows, N, int(D), _p(bias), _p(qw), _p(kw), _p(rc), _p(rs),
                           _p(rows), ctypes.c_double(eps), _p(out))
    return out


def gelu_tanh(v: float) -> float:
    return float(lib().or_gelu_tanh(float(v)))


def silu(v: float) -> float:
    return float(lib().or_silu(float(v)))


def qlinear_reference(fmt: str, epi: str, x_bf16, w_bf16, bias=None, residual=None, gate=None,
                      split_col=0, rows=None):
    """The whole path, oracle side: quantize x and W, GEMM the codes, epilogue.

    Returns a dict with the codes/scales of both operands and ``out`` (binary64,
    before bf16 rounding) for the requested activation rows.
    """
    if fmt == "fp8":
        qa, sa = quant_fp8_rows(x_bf16)
        qw, sw = quant_fp8_rows(w_bf16)
        y = gemm_fp8(qa, sa, qw, sw, rows)
        res = dict(qa=qa, sa=sa, qw=qw, sw=sw)
    elif fmt == "w8a16":
        qw, sw = quant_fp8_rows(w_bf16)
        y = gemm_w8a16(x_bf16, qw, sw, rows)
        res = dict(qw=qw, sw=sw)
    elif fmt == "nvfp4":
        qa, sfa, Ga = quant_nvfp4(x_bf16)
        qw, sfw, Gw = quant_nvfp4(w_bf16)
        y = gemm_nvfp4(qa, sfa, Ga, qw, sfw, Gw, rows)
        res = dict(qa=qa, sfa=sfa, Ga=Ga, qw=qw, sfw=sfw, Gw=Gw)
    else:
        raise ValueError(fmt)
    res["y"] = y
    res["out"] = epilogue(epi, y, bias=bias, residual=residual, gate=gate, rows=rows,
                          split_col=split_col)
    return res
