"""Host-side arithmetic of bench.py (no GPU): algorithmic bytes of the
quantize kernels and the weak-scaling aggregate."""
import bench
from synth import WORKLOADS


def test_quant_bytes_fp8_is_read_write_and_row_scales():
    layer = WORKLOADS["flux_qkv_fp8"].layers[0]          # 4608 x 3072
    assert bench.quant_bytes(layer) == 4608 * 3072 * 2 + 4608 * 3072 + 4608 * 4


def test_quant_bytes_nvfp4_counts_the_amax_pass():
    layer = WORKLOADS["flux2k_swiglu_nvfp4"].layers[0]   # 16896 x 3072
    mk = 16896 * 3072
    assert bench.quant_bytes(layer) == 2 * mk + 2 * mk + mk // 2 + mk // 16 + 16


def test_weak_scaling_counts_every_rank_over_the_slowest():
    # 2 ranks x 10 steps x 1e12 FLOP in 4 s (the max over ranks) = 5 TFLOP/s
    assert abs(bench.weak_scaling_tflops(1e12, 2, 10, 4000.0) - 5.0) < 1e-12
