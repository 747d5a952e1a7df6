"""B200 (sm_100a) dynamically quantized linear layer: FP8-E4M3 / NVFP4.

The compute path is the C ABI in ``include/qlinear.h`` (``libqlinear_b200.so``,
hand-written CUDA for sm_100a).  This package is a thin binding: ``_abi``
marshals arguments to the C calls, and :class:`QLinear` owns the device
buffers (allocated with PyTorch) and passes their pointers through.  No step
of the path runs in Python or PyTorch.
"""
import numpy as np

from . import _abi
from ._abi import (EPILOGUES, FORMATS, QLinearError, make_desc, qlinear_abi_version,  # noqa: F401
                   qlinear_act_bytes, qlinear_check, qlinear_create, qlinear_create_prequantized,
                   qlinear_destroy, qlinear_forward_gate_rows, qlinear_forward_rope,
                   qlinear_set_qk_norm,
                   qlinear_export_weights, qlinear_forward, qlinear_forward_nvfp4_out,
                   qlinear_out_features,
                   qlinear_quantize_act, qlinear_weight_bytes, status_string)

__all__ = ["QLinear", "make_desc", "QLinearError"]


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype, shape=None):
    """Refuse, before any launch, a tensor the kernels cannot read: not on
    the GPU, of another dtype, not contiguous, or of the wrong shape."""
    if t is None:
        return
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (got device {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")


class QLinear:
    """One quantized linear layer: weights quantized once, activations per call.

    ``w`` is a bf16 CUDA tensor [N, K]; ``bias`` bf16 [N] or None.  The
    workspace is a uint8 CUDA tensor owned by this object.
    """

    def __init__(self, fmt, epi, w, bias=None, split_col=0, variant=0, stream=None):
        import torch
        _need(w, "w", torch.bfloat16)
        if w.dim() != 2:
            raise ValueError(f"w must be 2-D [N, K] (got {tuple(w.shape)})")
        N, K = w.shape
        _need(bias, "bias", torch.bfloat16, (N,))
        self.fmt, self.epi, self.N, self.K = fmt, epi, int(N), int(K)
        self.desc = make_desc(fmt, epi, N, K, split_col, variant)
        nbytes = qlinear_weight_bytes(self.desc)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=w.device)
        self.h = qlinear_create(self.desc, w.data_ptr(), _ptr(bias), self.ws.data_ptr(), nbytes,
                                _stream_ptr(stream))
        self.Nout = qlinear_out_features(self.h)

    @classmethod
    def from_quantized(cls, fmt, epi, codes, scales, global_scale=0.0, bias=None, split_col=0,
                       variant=0, stream=None):
        """A layer from pre-quantized weights in the order export_weights
        returns: codes uint8 CUDA [N, K] (FP8) or [N, K/2] (NVFP4); scales
        fp32 [N] (FP8) or uint8 [N, K/16] E4M3 block scales (NVFP4); G."""
        import torch
        _need(codes, "codes", torch.uint8)
        _need(scales, "scales", torch.float32 if fmt != "nvfp4" else torch.uint8)
        self = cls.__new__(cls)
        N = int(codes.shape[0])
        _need(bias, "bias", torch.bfloat16, (N,))
        K = int(codes.shape[1]) * (2 if fmt == "nvfp4" else 1)
        self.fmt, self.epi, self.N, self.K = fmt, epi, N, K
        self.desc = make_desc(fmt, epi, N, K, split_col, variant)
        nbytes = qlinear_weight_bytes(self.desc)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
        self.h = qlinear_create_prequantized(self.desc, codes.data_ptr(), scales.data_ptr(),
                                             float(global_scale), _ptr(bias), self.ws.data_ptr(),
                                             nbytes, _stream_ptr(stream))
        self.Nout = qlinear_out_features(self.h)
        return self

    def act_buffers(self, M, device="cuda"):
        import torch
        cb, sb = qlinear_act_bytes(self.h, M)
        return (torch.empty(max(cb, 16), dtype=torch.uint8, device=device),
                torch.empty(max(sb, 16), dtype=torch.uint8, device=device))

    def quantize(self, x, codes, scales, stream=None):
        M = x.shape[0]
        qlinear_quantize_act(self.h, x.data_ptr(), M, codes.data_ptr(), scales.data_ptr(),
                             _stream_ptr(stream))

    def forward_codes(self, codes, scales, M, out, residual=None, gate=None, stream=None):
        qlinear_forward(self.h, codes.data_ptr(), scales.data_ptr(), M, _ptr(residual), _ptr(gate),
                        out.data_ptr(), _stream_ptr(stream))

    def forward_codes_gate_rows(self, codes, scales, M, out, residual, gate, rows_per_gate,
                                stream=None):
        """Gated-residual forward with gate [ceil(M / rows_per_gate), Nout]."""
        qlinear_forward_gate_rows(self.h, codes.data_ptr(), scales.data_ptr(), M,
                                  residual.data_ptr(), gate.data_ptr(), rows_per_gate,
                                  out.data_ptr(), _stream_ptr(stream))

    def set_qk_norm(self, q_weight, k_weight, eps=1e-6, stream=None):
        """QKV layers: bf16 CUDA norm weights [128] for q and k heads, and eps."""
        qlinear_set_qk_norm(self.h, q_weight.data_ptr(), k_weight.data_ptr(), eps,
                            _stream_ptr(stream))

    def forward_rope(self, codes, scales, M, rope_cos, rope_sin, out, stream=None):
        """QKV layers: forward with fp32 CUDA rotary tables [M, 64] (cos, sin)."""
        qlinear_forward_rope(self.h, codes.data_ptr(), scales.data_ptr(), M, rope_cos.data_ptr(),
                             rope_sin.data_ptr(), out.data_ptr(), _stream_ptr(stream))

    def forward_nvfp4_out(self, codes, scales, M, amax, out_codes, out_scales, residual=None,
                          gate=None, stream=None):
        """GEMM + epilogue written as the next NVFP4 layer's quantized input
        (codes, scales sized by that layer's act_buffers), against the tensor
        amax held in the device fp32 tensor `amax`."""
        qlinear_forward_nvfp4_out(self.h, codes.data_ptr(), scales.data_ptr(), M, _ptr(residual),
                                  _ptr(gate), amax.data_ptr(), out_codes.data_ptr(),
                                  out_scales.data_ptr(), _stream_ptr(stream))

    def __call__(self, x, residual=None, gate=None, out=None, bufs=None, stream=None):
        import torch
        _need(x, "x", torch.bfloat16)
        if x.dim() != 2 or x.shape[1] != self.K:
            raise ValueError(f"x must be [M, {self.K}] (got {tuple(x.shape)})")
        M = x.shape[0]
        _need(residual, "residual", torch.bfloat16, (M, self.Nout))
        _need(gate, "gate", torch.bfloat16, (self.Nout,))
        _need(out, "out", torch.bfloat16, (M, self.Nout))
        codes, scales = bufs if bufs is not None else self.act_buffers(M, x.device)
        if out is None:
            out = torch.empty((M, self.Nout), dtype=torch.bfloat16, device=x.device)
        self.quantize(x, codes, scales, stream)
        self.forward_codes(codes, scales, M, out, residual, gate, stream)
        return out

    def export_weights(self):
        """Quantized weights in logical order: (codes, scales, global_scale)."""
        if self.fmt == "fp8":
            codes = np.empty((self.N, self.K), np.uint8)
            scales = np.empty(self.N, np.float32)
        else:
            codes = np.empty((self.N, self.K // 2), np.uint8)
            scales = np.empty((self.N, self.K // 16), np.uint8)
        g = qlinear_export_weights(self.h, codes.ctypes.data, scales.ctypes.data,
                                   _stream_ptr(None))
        return codes, scales, np.float32(g)

    def check(self, stream=None):
        return qlinear_check(self.h, _stream_ptr(stream))

    def close(self):
        if getattr(self, "h", None):
            qlinear_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
