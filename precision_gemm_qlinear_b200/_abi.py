"""ctypes binding of the C ABI in ``include/qlinear.h`` (argument marshalling only).

Every function here has the name of the C entry point it calls.  The library
is the in-tree ``libqlinear_b200.so``; if it is missing the import fails
loudly -- there is no other implementation of the path.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlinear_b200.so")

QL_OK, QL_ERR_INVALID_ARG, QL_ERR_ALIGNMENT, QL_ERR_UNSUPPORTED, QL_ERR_CUDA, QL_ERR_TIMEOUT = range(6)
QL_FP8_E4M3, QL_NVFP4, QL_W8A16 = 0, 1, 2
FORMATS = {"fp8": QL_FP8_E4M3, "nvfp4": QL_NVFP4, "w8a16": QL_W8A16}
EPILOGUES = {"bias": 0, "bias_gelu": 1, "swiglu": 2, "bias_gated_residual": 3,
             "split_bias_gelu": 4, "qkv_norm_rope": 5}

# every entry point declared in include/qlinear.h
EXPORTS = ("qlinear_weight_bytes", "qlinear_create", "qlinear_create_prequantized",
           "qlinear_act_bytes", "qlinear_out_features",
           "qlinear_quantize_act", "qlinear_quantize_act_noalloc", "qlinear_forward",
           "qlinear_forward_gate_rows", "qlinear_forward_nvfp4_out", "qlinear_forward_rope",
           "qlinear_set_qk_norm", "qlinear_export_weights", "qlinear_check", "qlinear_debug_set_fault",
           "qlinear_debug_encode", "qlinear_destroy",
           "qlinear_status_string", "qlinear_abi_version")


class ql_desc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("epi", ctypes.c_int32), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("split_col", ctypes.c_int64),
                ("variant", ctypes.c_int32), ("flags", ctypes.c_int32)]


class QLinearError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run precision_gemm_qlinear_b200/build.py)")
    L = ctypes.CDLL(path)
    P, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    D = ctypes.POINTER(ql_desc)
    L.qlinear_weight_bytes.argtypes = [D, ctypes.POINTER(sz)]
    L.qlinear_create.argtypes = [D, P, P, P, sz, P, ctypes.POINTER(P)]
    L.qlinear_act_bytes.argtypes = [P, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.qlinear_out_features.argtypes = [P, ctypes.POINTER(i64)]
    L.qlinear_quantize_act.argtypes = [P, P, i64, P, P, P]
    L.qlinear_quantize_act_noalloc.argtypes = [P, P, i64, P, P, P]
    L.qlinear_forward.argtypes = [P, P, P, i64, P, P, P, P]
    L.qlinear_forward_nvfp4_out.argtypes = [P, P, P, i64, P, P, P, P, P, P]
    L.qlinear_forward_gate_rows.argtypes = [P, P, P, i64, P, P, i64, P, P]
    L.qlinear_forward_rope.argtypes = [P, P, P, i64, P, P, P, P]
    L.qlinear_set_qk_norm.argtypes = [P, P, P, ctypes.c_float, P]
    L.qlinear_create_prequantized.argtypes = [D, P, P, ctypes.c_float, P, P, sz, P,
                                              ctypes.POINTER(P)]
    L.qlinear_export_weights.argtypes = [P, P, P, ctypes.POINTER(ctypes.c_float), P]
    L.qlinear_check.argtypes = [P, P]
    L.qlinear_debug_set_fault.argtypes = [P, ctypes.c_int32]
    L.qlinear_debug_encode.argtypes = [ctypes.c_int32, P, i64, P, P, P]
    L.qlinear_destroy.argtypes = [P]
    L.qlinear_status_string.argtypes = [st]
    L.qlinear_status_string.restype = ctypes.c_char_p
    L.qlinear_abi_version.argtypes = []
    L.qlinear_abi_version.restype = ctypes.c_int32
    for name in EXPORTS:
        if name not in ("qlinear_status_string", "qlinear_abi_version"):
            getattr(L, name).restype = st
    _lib = L
    return L


def _ck(fn, status):
    if status != QL_OK:
        raise QLinearError(fn, status)


def status_string(status: int) -> str:
    return load().qlinear_status_string(int(status)).decode()


def qlinear_abi_version() -> int:
    return int(load().qlinear_abi_version())


def make_desc(fmt, epi, N, K, split_col=0, variant=0, flags=0) -> ql_desc:
    fmt = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    epi = EPILOGUES[epi] if isinstance(epi, str) else int(epi)
    return ql_desc(fmt, epi, int(N), int(K), int(split_col), int(variant), int(flags))


def qlinear_weight_bytes(desc: ql_desc, check=True):
    n = ctypes.c_size_t(0)
    s = load().qlinear_weight_bytes(ctypes.byref(desc), ctypes.byref(n))
    if check:
        _ck("qlinear_weight_bytes", s)
        return n.value
    return s, n.value


def qlinear_create(desc: ql_desc, w_ptr, bias_ptr, ws_ptr, ws_bytes, stream=0, check=True):
    h = ctypes.c_void_p(0)
    s = load().qlinear_create(ctypes.byref(desc), w_ptr, bias_ptr, ws_ptr, ws_bytes, stream,
                              ctypes.byref(h))
    if check:
        _ck("qlinear_create", s)
        return h.value
    return s, h.value


def qlinear_create_prequantized(desc: ql_desc, codes_ptr, scales_ptr, global_scale, bias_ptr,
                                ws_ptr, ws_bytes, stream=0, check=True):
    h = ctypes.c_void_p(0)
    s = load().qlinear_create_prequantized(ctypes.byref(desc), codes_ptr, scales_ptr,
                                           ctypes.c_float(global_scale), bias_ptr, ws_ptr, ws_bytes,
                                           stream, ctypes.byref(h))
    if check:
        _ck("qlinear_create_prequantized", s)
        return h.value
    return s, h.value


def qlinear_act_bytes(h, M, check=True):
    c, sc = ctypes.c_size_t(0), ctypes.c_size_t(0)
    s = load().qlinear_act_bytes(h, M, ctypes.byref(c), ctypes.byref(sc))
    if check:
        _ck("qlinear_act_bytes", s)
        return c.value, sc.value
    return s, c.value, sc.value


def qlinear_out_features(h):
    n = ctypes.c_int64(0)
    _ck("qlinear_out_features", load().qlinear_out_features(h, ctypes.byref(n)))
    return n.value


def qlinear_quantize_act(h, x_ptr, M, codes_ptr, scales_ptr, stream=0, check=True):
    s = load().qlinear_quantize_act(h, x_ptr, M, codes_ptr, scales_ptr, stream)
    if check:
        _ck("qlinear_quantize_act", s)
    return s


QL_NOALLOC_MAX_ROWS = 524288


def qlinear_quantize_act_noalloc(h, x_ptr, M, codes_ptr, scales_ptr, stream=0, check=True):
    """Allocation-free activation quantization (working memory inside the library)."""
    s = load().qlinear_quantize_act_noalloc(h, x_ptr, M, codes_ptr, scales_ptr, stream)
    if check:
        _ck("qlinear_quantize_act_noalloc", s)
    return s


def qlinear_forward(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr, out_ptr, stream=0,
                    check=True):
    s = load().qlinear_forward(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr, out_ptr, stream)
    if check:
        _ck("qlinear_forward", s)
    return s


def qlinear_forward_gate_rows(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr, rows_per_gate,
                              out_ptr, stream=0, check=True):
    s = load().qlinear_forward_gate_rows(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr,
                                         rows_per_gate, out_ptr, stream)
    if check:
        _ck("qlinear_forward_gate_rows", s)
    return s


def qlinear_forward_rope(h, codes_ptr, scales_ptr, M, cos_ptr, sin_ptr, out_ptr, stream=0,
                         check=True):
    s = load().qlinear_forward_rope(h, codes_ptr, scales_ptr, M, cos_ptr, sin_ptr, out_ptr, stream)
    if check:
        _ck("qlinear_forward_rope", s)
    return s


def qlinear_set_qk_norm(h, q_ptr, k_ptr, eps=1e-6, stream=0, check=True):
    s = load().qlinear_set_qk_norm(h, q_ptr, k_ptr, ctypes.c_float(eps), stream)
    if check:
        _ck("qlinear_set_qk_norm", s)
    return s


def qlinear_forward_nvfp4_out(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr, amax_ptr,
                              out_codes_ptr, out_scales_ptr, stream=0, check=True):
    s = load().qlinear_forward_nvfp4_out(h, codes_ptr, scales_ptr, M, residual_ptr, gate_ptr,
                                         amax_ptr, out_codes_ptr, out_scales_ptr, stream)
    if check:
        _ck("qlinear_forward_nvfp4_out", s)
    return s


def qlinear_export_weights(h, codes_host_ptr, scales_host_ptr, stream=0):
    g = ctypes.c_float(0)
    _ck("qlinear_export_weights",
        load().qlinear_export_weights(h, codes_host_ptr, scales_host_ptr, ctypes.byref(g), stream))
    return g.value


def qlinear_check(h, stream=0):
    return load().qlinear_check(h, stream)


def qlinear_destroy(h):
    _ck("qlinear_destroy", load().qlinear_destroy(h))


def qlinear_debug_set_fault(h, mode):
    _ck("qlinear_debug_set_fault", load().qlinear_debug_set_fault(h, mode))


def qlinear_debug_encode(mode, in_ptr, n, amax_ptr, out_ptr, stream=0, check=True):
    """Device encoders on given values (test hook): mode 0 E4M3, 1 E2M1 of
    fp32 in[n]; mode 2 NVFP4 blocks of bf16 in[n] against the amax scalar."""
    s = load().qlinear_debug_encode(int(mode), in_ptr, int(n), amax_ptr, out_ptr, stream)
    if check:
        _ck("qlinear_debug_encode", s)
    return s
