"""GPU parity of the whole path (quantize -> tcgen05 GEMM -> fused epilogue)
against the oracle, element by element, within
|gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref)  (ref = binary64, before bf16)."""
import numpy as np
import pytest

import oracle
from qlutil import assert_close, from_dev_bf16, sample_rows, to_dev_bf16
from synth.tensors import draw

pytestmark = pytest.mark.gpu

EPIS = ["bias", "bias_gelu", "swiglu", "bias_gated_residual", "split_bias_gelu"]


def _run(fmt, epi, M, N, K, seed=0, x_kind="normal", bias=True, rows=None, split_col=None,
         variant=0):
    import torch
    import precision_gemm_qlinear_b200 as ql
    if x_kind == "normal":
        x = draw("normal", (M, K), seed, "x", outlier_frac=0.01, outlier_factor=8.0)
    else:
        x = draw("student_t", (M, K), seed, "x", nu=3, outlier_frac=0.005, outlier_factor=20.0)
    w = draw("normal", (N, K), seed, "w", std=0.02)
    b = draw("normal", (N,), seed, "bias", std=0.01) if bias else None
    Nout = N // 2 if epi == "swiglu" else N
    sc = (split_col if split_col is not None else (N // 2) // 32 * 32) if epi == "split_bias_gelu" else 0
    gate = res = None
    if epi == "bias_gated_residual":
        gate = draw("normal", (Nout,), seed, "gate", mean=1.0, std=0.1)
        res = draw("normal", (M, Nout), seed, "residual")
    lay = ql.QLinear(fmt, epi, to_dev_bf16(w), None if b is None else to_dev_bf16(b), split_col=sc,
                     variant=variant)
    out = lay(to_dev_bf16(x), residual=None if res is None else to_dev_bf16(res),
              gate=None if gate is None else to_dev_bf16(gate))
    torch.cuda.synchronize()
    assert lay.check() == 0
    ref = oracle.qlinear_reference(fmt, epi, x, w, bias=b, residual=res, gate=gate, split_col=sc,
                                   rows=rows)
    got = from_dev_bf16(out)
    if rows is not None:
        got = got[rows]
    return got, ref["out"]


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("epi", EPIS)
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_small_all_epilogues(fmt, epi, variant):
    # 3 M tiles (one CTA) / 2 pair tiles with a ragged tail, 2-3 N tiles,
    # several K stages; variant 1 = one CTA per 128-row tile, 2 = CTA pairs
    K = 384 if fmt == "fp8" else 512
    got, ref = _run(fmt, epi, 300, 768 if epi != "swiglu" else 1024, K, variant=variant)
    assert_close(got, ref, f"{fmt}/{epi}/v{variant}")


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_tiny_config(fmt):
    got, ref = _run(fmt, "bias_gelu", 128, 512, 256)
    assert_close(got, ref, f"tiny {fmt}")


@pytest.mark.parametrize("variant", [0, 2])
@pytest.mark.parametrize("M", [1, 5, 127, 129, 255, 257])
def test_ragged_m(M, variant):
    got, ref = _run("fp8", "bias", M, 512, 256, variant=variant)
    assert_close(got, ref, f"M={M}")


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_k_tail_and_no_bias(fmt):
    # K not a multiple of the 128-byte stage: zero-filled by TMA
    K = 208 if fmt == "fp8" else 544
    got, ref = _run(fmt, "bias", 200, 512, K, bias=False)
    assert_close(got, ref, f"K tail {fmt}")


def test_fp8_n_not_multiple_of_tile():
    got, ref = _run("fp8", "bias_gelu", 256, 288, 256)
    assert_close(got, ref, "N=288")


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_many_tiles_per_cta(fmt, variant):
    # more tiles than SMs (or CTA pairs): every CTA runs several tiles and
    # cycles both TMEM accumulator buffers; oracle on a row sample covering
    # every M tile
    M, N, K = 2000, 2560 if variant == 1 else 5120, 256
    rows = sample_rows(M, 48, seed=1)
    got, ref = _run(fmt, "split_bias_gelu", M, N, K, x_kind="t", rows=rows, split_col=1024,
                    variant=variant)
    assert_close(got, ref, f"many tiles {fmt} v{variant}")


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "w8a16"])
def test_zero_activation_rows_give_the_bias(fmt):
    # an all-zero token has amax 0: its scale (FP8) or block scales (NVFP4)
    # are 0, its codes are 0 and its output row is exactly the bias; the
    # other rows are unaffected (whole output against the oracle)
    import torch
    import precision_gemm_qlinear_b200 as ql
    M, N, K = 300, 512, 512
    x = draw("normal", (M, K), 51, "x")
    zero_rows = [0, 5, 130, 255, 256, M - 1]
    x[zero_rows] = 0
    w = draw("normal", (N, K), 51, "w", std=0.02)
    b = draw("normal", (N,), 51, "bias", std=0.01)
    lay = ql.QLinear(fmt, "bias", to_dev_bf16(w), to_dev_bf16(b))
    out = lay(to_dev_bf16(x))
    torch.cuda.synchronize()
    assert lay.check() == 0
    bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for r in zero_rows:
        assert np.array_equal(bits[r], b), f"row {r}"
    ref = oracle.qlinear_reference(fmt, "bias", x, w, bias=b)["out"]
    assert_close(from_dev_bf16(out), ref, f"zero rows {fmt}")


def test_nvfp4_all_zero_tensor():
    # tensor amax 0: the global scale and every block scale are 0, every code
    # is 0, and the output is the bias broadcast over the tokens
    import torch
    import precision_gemm_qlinear_b200 as ql
    M, N, K = 200, 256, 256
    w = draw("normal", (N, K), 52, "w", std=0.02)
    b = draw("normal", (N,), 52, "bias", std=0.01)
    lay = ql.QLinear("nvfp4", "bias_gelu", to_dev_bf16(w), to_dev_bf16(b))
    x = np.zeros((M, K), np.uint16)
    out = lay(to_dev_bf16(x))
    torch.cuda.synchronize()
    assert lay.check() == 0
    ref = oracle.qlinear_reference("nvfp4", "bias_gelu", x, w, bias=b)["out"]
    assert_close(from_dev_bf16(out), ref, "all-zero NVFP4")
    bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(bits == bits[0])  # every token the same row: gelu(bias)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "w8a16"])
def test_empty_batch_is_a_no_op(fmt):
    # M = 0: quantize and forward return success and write nothing
    import torch
    import precision_gemm_qlinear_b200 as ql
    N, K = 256, 256
    lay = ql.QLinear(fmt, "bias_gelu", to_dev_bf16(draw("normal", (N, K), 53, "w", std=0.02)))
    x = to_dev_bf16(draw("normal", (4, K), 53, "x"))
    codes, scales = lay.act_buffers(4)
    codes.fill_(0xA5)
    scales.fill_(0xA5)
    out = torch.full((4, N), 7.0, dtype=torch.bfloat16, device="cuda")
    lay.quantize(x[:0], codes, scales)
    lay.forward_codes(x if fmt == "w8a16" else codes, scales, 0, out)
    torch.cuda.synchronize()
    assert lay.check() == 0
    assert bool((codes == 0xA5).all()) and bool((scales == 0xA5).all())
    assert bool((out == 7.0).all())
