"""The FLUX-shaped workloads of the quantized DiT linear layer.

Shapes: FLUX.1-dev at 1024x1024 has 4096 image tokens (8x VAE downsampling,
2x2 patches) plus 512 text tokens = 4608 tokens, hidden size 3072, QKV 3*3072,
MLP 4*3072.  At 2048x2048 there are 16384 image tokens + 512 text = 16896;
classifier-free guidance batches the conditional and unconditional passes,
giving 2*16896 tokens.  The pages give none of these dimensions; they are the
public FLUX architecture figures and are stated here as the synthetic stand-in
for real activations and weights (no checkpoint is used).
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

from .tensors import draw


@dataclass(frozen=True)
class Layer:
    fmt: str                 # "fp8" | "nvfp4" | "w8a16" (bf16 activations, FP8 weights)
    M: int
    K: int
    N: int                   # GEMM output columns (SwiGLU: gate|up = 2*Nout)
    epi: str                 # bias | bias_gelu | swiglu | bias_gated_residual | split_bias_gelu
    x_dist: dict             # distribution of the activations (ignored when chained)
    w_std: float = 0.02
    bias_std: Optional[float] = 0.01
    split_col: int = 0
    chained: bool = False    # input is the bf16 output of the previous layer

    @property
    def Nout(self) -> int:
        return self.N // 2 if self.epi == "swiglu" else self.N

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple
    note: str = ""

    @property
    def flops(self) -> int:
        return sum(l.flops for l in self.layers)


_N01 = dict(kind="normal", mean=0.0, std=1.0)
_N01_OUT8 = dict(kind="normal", mean=0.0, std=1.0, outlier_frac=0.01, outlier_factor=8.0)
_T4 = dict(kind="student_t", nu=4)
_T3_OUT20 = dict(kind="student_t", nu=3, outlier_frac=0.005, outlier_factor=20.0)

WORKLOADS = {
    "tiny_fp8": Workload("tiny_fp8", (
        Layer("fp8", 128, 256, 512, "bias_gelu", _N01),
    ), "tiny FP8 qlinear 128x256x512, bias+GELU-tanh"),
    "flux_qkv_fp8": Workload("flux_qkv_fp8", (
        Layer("fp8", 4608, 3072, 9216, "bias", _N01_OUT8),
    ), "FLUX-dev QKV projection, FP8, 4608x3072x9216, bias"),
    "flux_qkv_normrope_fp8": Workload("flux_qkv_normrope_fp8", (
        Layer("fp8", 4608, 3072, 9216, "qkv_norm_rope", _N01_OUT8),
    ), "FLUX-dev QKV projection, FP8, 4608x3072x9216, q/k RMS norm per 128-column head + "
       "rotary embedding, v bias"),
    "flux_qkv_w8a16": Workload("flux_qkv_w8a16", (
        Layer("w8a16", 4608, 3072, 9216, "bias", _N01_OUT8),
    ), "FLUX-dev QKV projection, weight-only: bf16 activations x FP8 weights, 4608x3072x9216, bias"),
    "flux_mlp_fp8": Workload("flux_mlp_fp8", (
        Layer("fp8", 4608, 3072, 12288, "bias_gelu", _N01_OUT8),
        Layer("fp8", 4608, 12288, 3072, "bias_gated_residual", _N01, chained=True),
    ), "FLUX-dev MLP pair, FP8: up 4608x3072x12288 bias+GELU, down 4608x12288x3072 "
       "residual + gate*(xW+b)"),
    "flux2k_swiglu_nvfp4": Workload("flux2k_swiglu_nvfp4", (
        Layer("nvfp4", 16896, 3072, 16384, "swiglu", _T4, bias_std=None),
    ), "NVFP4 2048^2 MLP up-projection with SwiGLU, 16896x3072x(2x8192)"),
    "flux2k_mlp_nvfp4": Workload("flux2k_mlp_nvfp4", (
        Layer("nvfp4", 16896, 3072, 16384, "swiglu", _T4, bias_std=None),
        Layer("nvfp4", 16896, 8192, 3072, "bias_gated_residual", _N01, chained=True),
    ), "NVFP4 2048^2 MLP pair: up 16896x3072x(2x8192) SwiGLU, down 16896x8192x3072 "
       "residual + gate*(xW+b)"),
    "cfg_linear1_fp8": Workload("cfg_linear1_fp8", (
        Layer("fp8", 33792, 3072, 21504, "split_bias_gelu", _T3_OUT20, split_col=9216),
    ), "CFG-batched parallel-block linear1, FP8, 33792x3072x21504, split bias/GELU"),
    "cfg_linear1": Workload("cfg_linear1", (
        Layer("fp8", 33792, 3072, 21504, "split_bias_gelu", _T3_OUT20, split_col=9216),
        Layer("nvfp4", 33792, 3072, 21504, "split_bias_gelu", _T3_OUT20, split_col=9216),
    ), "CFG-batched parallel-block linear1 in its FP8 and NVFP4 variants (two independent "
       "layers on their own inputs), 33792x3072x21504 each, split bias/GELU"),
    "cfg_linear1_nvfp4": Workload("cfg_linear1_nvfp4", (
        Layer("nvfp4", 33792, 3072, 21504, "split_bias_gelu", _T3_OUT20, split_col=9216),
    ), "CFG-batched parallel-block linear1, NVFP4, 33792x3072x21504, split bias/GELU"),
}


def make_inputs(layer: Layer, seed: int = 0, layer_index: int = 0, M: int = None,
                w_seed: int = None):
    """Draw the host-side bf16 tensors of one layer (uint16 bit patterns).

    Returns dict with x [M,K] (absent when chained), w [N,K], bias [N] or None,
    gate [Nout] and residual [M,Nout] for the gated-residual epilogue.  The
    per-token tensors (x, residual) come from `seed`; the layer's parameters
    (w, bias, gate) from `w_seed` (default: `seed`).
    """
    M = layer.M if M is None else M
    ws = seed if w_seed is None else w_seed
    sfx = "" if layer_index == 0 else "2"
    out = {}
    if not layer.chained:
        d = dict(layer.x_dist)
        kind = d.pop("kind")
        out["x"] = draw(kind, (M, layer.K), seed, "x" + sfx, **d)
    out["w"] = draw("normal", (layer.N, layer.K), ws, "w" + sfx, std=layer.w_std)
    out["bias"] = (None if layer.bias_std is None else
                   draw("normal", (layer.N,), ws, "bias" + sfx, std=layer.bias_std))
    if layer.epi == "bias_gated_residual":
        out["gate"] = draw("normal", (layer.Nout,), ws, "gate", mean=1.0, std=0.1)
        out["residual"] = draw("normal", (M, layer.Nout), seed, "residual", std=1.0)
    if layer.epi == "qkv_norm_rope":
        # norm weights near 1; rotary angles of a 1-D position grid with the
        # usual geometric frequency ladder (base 10000) over the 64 pairs
        out["q_norm"] = draw("normal", (128,), ws, "q_norm", mean=1.0, std=0.1)
        out["k_norm"] = draw("normal", (128,), ws, "k_norm", mean=1.0, std=0.1)
        pos = np.arange(M, dtype=np.float64)[:, None]
        freq = 10000.0 ** (-np.arange(64, dtype=np.float64) / 64.0)[None, :]
        out["rope_cos"] = np.cos(pos * freq).astype(np.float32)
        out["rope_sin"] = np.sin(pos * freq).astype(np.float32)
    return out
