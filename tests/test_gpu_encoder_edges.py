"""GPU parity of the encoders on their edge cases, bit for bit against the
oracle.

Random FLUX-like activations almost never reach the cases where rounding
decides: exact round-to-nearest-even ties, values just above the largest
finite code, E4M3 subnormals, NVFP4 block scales that fall in the E4M3
subnormal range or round so that a block's largest element no longer fits.
These tests build inputs that reach each of them on purpose:

  * the device conversions alone (test hook qlinear_debug_encode), on every
    finite bf16 value times 2^k, k = -8..8, plus +-inf (and NaN for E4M3):
    the inputs of the oracle's own brute-force pin;
  * per-token FP8 quantization (qlinear_quantize_act) of rows whose amax is
    448 * 2^j, so that the inverse scale 448/amax = 2^-j is exact and every
    finite bf16 value below the amax reaches the encoder scaled exactly;
  * NVFP4 quantization of a tensor whose amax A = 448 * 2^4 makes the
    block-scale factor 448/A a power of two, with blocks whose maxima run
    over every positive finite bf16 value up to A (every block-scale code,
    its ties and its subnormals);
  * NVFP4 quantization with G = A/2688 = 1 and blocks whose maxima 6 * 2^e * f
    sweep f over every bf16 mantissa and e over the normal and subnormal
    block-scale range, holding the E2M1 ties (0.25, 0.75, ... 5 times 2^e),
    so that ties are exact when the block scale decodes to 2^e and elements
    saturate when the block scale rounds down;
  * the same NVFP4 blocks through the block encoder of the NVFP4-output GEMM
    epilogue (the test hook's mode 2), and through weight quantization
    (qlinear_create, read back with qlinear_export_weights).

The formats and their rounding are the OCP 8-bit floating-point and MX
definitions (the pages name the formats, FP8 dynamic quantization in
wavespeed.ai's "Cuantizacion Dinamica FP8" and NVFP4 in algoritmulzilei.ro's
FLUX 3 Image Klein page, but give no bit layout).
"""
import numpy as np
import pytest

import oracle
from qlutil import sf_unswizzle, to_dev_bf16
from synth.tensors import bf16_bits_from_f64, bf16_bits_to_f32

pytestmark = pytest.mark.gpu

FINITE_POS = np.arange(0x0000, 0x7F80, dtype=np.uint32)  # every finite bf16 value >= +0


def _bf16_of(v: float) -> np.uint16:
    b = np.float32(v).view(np.uint32)
    assert b & 0xFFFF == 0, f"{v} is not a bf16 value"
    return np.uint16(b >> 16)


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


def _debug_encode(mode, values, amax=None):
    import torch
    from precision_gemm_qlinear_b200 import _abi
    if mode == 2:
        inp = _dev(values.view(np.int16), torch.bfloat16)
        n = values.size
        out = torch.empty(n // 2 + n // 16, dtype=torch.uint8, device="cuda")
        am = torch.tensor([amax], dtype=torch.float32, device="cuda")
        _abi.qlinear_debug_encode(2, inp.data_ptr(), n, am.data_ptr(), out.data_ptr())
    else:
        inp = _dev(np.ascontiguousarray(values, np.float32))
        n = values.size
        out = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        _abi.qlinear_debug_encode(mode, inp.data_ptr(), n, None, out.data_ptr())
    torch.cuda.synchronize()
    return out.cpu().numpy()[: (n // 2 + n // 16) if mode == 2 else n]


def _all_bf16_times_2k(signs=True):
    v = (FINITE_POS << 16).view(np.float32)
    if signs:
        v = np.concatenate([v, -v])
    return np.concatenate([v * np.float32(2.0 ** k) for k in range(-8, 9)])


# ------------------------------------------------------ the conversions alone

def test_device_e4m3_encoder_every_bf16_times_2k():
    edge = np.array([449.0, 463.99, 464.0, 464.01, 480.0, 1e30, np.inf, -464.0, -np.inf, np.nan],
                    np.float32)
    v = np.concatenate([_all_bf16_times_2k(), edge])
    got = _debug_encode(0, v)
    ref = oracle.e4m3_encode_array(v)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"{bad.size} E4M3 codes differ, e.g. {v[bad[:4]]} -> {got[bad[:4]]} vs {ref[bad[:4]]}"
    # values in (448, 464], beyond, and infinities saturate to +-448
    tail = got[-edge.size:]
    assert np.all(tail[:7] == 0x7E) and np.all(tail[7:9] == 0xFE)


def test_device_e2m1_encoder_every_bf16_times_2k():
    v = np.concatenate([_all_bf16_times_2k(),
                        np.array([np.inf, -np.inf, 6.5, 7.0, -7.0, 1e30], np.float32)])
    got = _debug_encode(1, v)
    ref = oracle.e2m1_encode_array(v)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"{bad.size} E2M1 codes differ, e.g. {v[bad[:4]]} -> {got[bad[:4]]} vs {ref[bad[:4]]}"


# ------------------------------------------------------------ crafted inputs

def _fp8_power_of_two_rows(K=2048, seed=0):
    """Rows whose amax is 448 * 2^j (j = -8..8), each holding, with both
    signs, every finite bf16 value not above that amax."""
    g = np.random.default_rng(seed)
    pos_vals = (FINITE_POS << 16).view(np.float32)
    rows = []
    for j in range(-8, 9):
        amax = np.float32(448.0 * 2.0 ** j)
        a = _bf16_of(amax)
        sel = FINITE_POS[pos_vals <= amax].astype(np.uint16)
        vals = np.concatenate([sel, sel | np.uint16(0x8000)])
        g.shuffle(vals)
        for c in range(0, vals.size, K - 1):
            chunk = vals[c:c + K - 1]
            row = np.zeros(K, np.uint16)
            row[: chunk.size] = chunk
            row = np.insert(row[:K - 1], int(g.integers(0, K)), a if c % 2 == 0 else a | 0x8000)
            rows.append(row)
    return np.stack(rows)


def _block(amax_bits, others):
    b = np.empty(16, np.uint16)
    b[0] = amax_bits
    b[1:] = others
    return b


def _nvfp4_scale_sweep_tensor(K=4096, seed=1):
    """A = 7168 = 448 * 2^4, so the block-scale factor 448/A = 2^-4 is exact.
    One 16-element block per positive finite bf16 maximum b <= A: b (with a
    random sign) and 15 values within [-b, b]."""
    g = np.random.default_rng(seed)
    A = np.float32(448.0 * 16)
    pos_vals = (FINITE_POS << 16).view(np.float32)
    maxima = FINITE_POS[(pos_vals <= A)].astype(np.uint16)
    blocks = []
    for b in maxima:
        bv = float(bf16_bits_to_f32(np.array([b]))[0])
        others = bf16_bits_from_f64(g.uniform(-1.0, 1.0, 15) * bv)
        blk = _block(b | (np.uint16(0x8000) if g.integers(0, 2) else 0), others)
        g.shuffle(blk)
        blocks.append(blk)
    return _pack_blocks(blocks, K), float(A)


def _nvfp4_tie_tensor(K=4096, seed=2):
    """A = 2688 (G = 1).  Blocks with maximum 6 * 2^e * f for e = -9..7 and f
    every bf16 mantissa in [1, 2), holding the E2M1 ties t * 2^e,
    t in {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 5.5, 6}, with both signs."""
    g = np.random.default_rng(seed)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 6.0, -0.25, -0.75, -1.25, -2.5,
                     -3.5, -5.0], np.float64)
    blocks = [_block(_bf16_of(2688.0), bf16_bits_from_f64(g.uniform(-2688, 2688, 15)))]
    for e in range(-9, 8):
        for m in range(128):
            f = 1.0 + m / 128.0
            amax = 6.0 * 2.0 ** e * f
            blk = _block(bf16_bits_from_f64(np.array([amax]))[0], bf16_bits_from_f64(ties * 2.0 ** e))
            g.shuffle(blk)
            blocks.append(blk)
    return _pack_blocks(blocks, K), 2688.0


def _pack_blocks(blocks, K):
    flat = np.concatenate(blocks)
    rows = (flat.size + K - 1) // K
    out = np.zeros(rows * K, np.uint16)
    out[: flat.size] = flat
    return out.reshape(rows, K)


# ------------------------------------------------ through the quantize kernels

def _fp8_layer(K):
    import precision_gemm_qlinear_b200 as ql
    from synth.tensors import draw
    return ql.QLinear("fp8", "bias", to_dev_bf16(draw("normal", (256, K), 0, "w", std=0.02)))


def _nvfp4_layer(K):
    import precision_gemm_qlinear_b200 as ql
    from synth.tensors import draw
    return ql.QLinear("nvfp4", "bias", to_dev_bf16(draw("normal", (256, K), 0, "w", std=0.02)))


def test_fp8_quantize_power_of_two_scales_every_bf16():
    import torch
    x = _fp8_power_of_two_rows()
    M, K = x.shape
    lay = _fp8_layer(K)
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    torch.cuda.synchronize()
    rc, rs = oracle.quant_fp8_rows(x)
    gs = scales[: 4 * M].cpu().numpy().view(np.uint32)
    assert np.array_equal(gs, rs.view(np.uint32))
    gc = codes[: M * K].cpu().numpy().reshape(M, K)
    bad = np.argwhere(gc != rc)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:4].tolist()}"
    # every row's scale is 2^j exactly, and both +-448 codes occur
    assert np.all(np.log2(rs.astype(np.float64)) == np.round(np.log2(rs.astype(np.float64))))
    assert np.any(rc == 0x7E) and np.any(rc == 0xFE)


@pytest.mark.parametrize("which", ["scale_sweep", "ties"])
def test_nvfp4_quantize_crafted_blocks(which):
    import torch
    x, A = _nvfp4_scale_sweep_tensor() if which == "scale_sweep" else _nvfp4_tie_tensor()
    M, K = x.shape
    lay = _nvfp4_layer(K)
    codes, scales = lay.act_buffers(M)
    lay.quantize(to_dev_bf16(x), codes, scales)
    torch.cuda.synchronize()
    rc, rsf, rg = oracle.quant_nvfp4(x)
    assert np.float32(oracle.tensor_amax(x)) == np.float32(A)
    sb = scales.cpu().numpy()
    nsf = ((M + 127) // 128) * ((K + 255) // 256) * 4 * 512
    assert sb[nsf:nsf + 4].view(np.uint32)[0] == np.float32(rg).view(np.uint32)
    gsf = sf_unswizzle(sb[:nsf], M, K)
    assert np.array_equal(gsf, rsf), f"{int((gsf != rsf).sum())} block scales differ"
    gc = codes[: M * K // 2].cpu().numpy().reshape(M, K // 2)
    assert np.array_equal(gc, rc), f"{int((gc != rc).sum())} code bytes differ"
    if which == "scale_sweep":
        # E4M3 subnormal block scales (0x01..0x07) and the largest one occur
        assert np.any((rsf >= 1) & (rsf <= 7)) and np.any(rsf == 0x7E)
    else:
        # the case is reached: blocks whose largest element exceeds 6 * dec(sb) * G,
        # i.e. whose block scale rounded down so that the element saturates
        dec = np.array([oracle.e4m3_decode(c) for c in range(256)])[rsf]
        bmax = np.abs(bf16_bits_to_f32(x).astype(np.float64)).reshape(M, K // 16, 16).max(axis=2)
        assert np.any(bmax > 6.0 * dec * float(rg) * (1 + 1e-6))


@pytest.mark.parametrize("which", ["scale_sweep", "ties"])
def test_nvfp4_epilogue_block_encoder_crafted_blocks(which):
    """The block encoder of the NVFP4-output GEMM epilogue on the same blocks,
    against the oracle's NVFP4 quantization with the same tensor amax."""
    x, A = _nvfp4_scale_sweep_tensor() if which == "scale_sweep" else _nvfp4_tie_tensor()
    M, K = x.shape
    out = _debug_encode(2, x.ravel(), A)
    n = x.size
    rc, rsf, _ = oracle.quant_nvfp4(x, amax=A)
    assert np.array_equal(out[: n // 2].reshape(M, K // 2), rc)
    assert np.array_equal(out[n // 2:].reshape(M, K // 16), rsf)


def test_nvfp4_quantize_crafted_blocks_other_amax():
    """The tie blocks against a supplied amax that is not the tensor's own
    (every block scale shifts; the fused epilogue quantizes this way)."""
    x, _ = _nvfp4_tie_tensor()
    for A in (1000.0, 2688.0 * 4, 3.0e-3):
        out = _debug_encode(2, x.ravel(), A)
        n = x.size
        rc, rsf, _ = oracle.quant_nvfp4(x, amax=A)
        M, K = x.shape
        assert np.array_equal(out[: n // 2].reshape(M, K // 2), rc), A
        assert np.array_equal(out[n // 2:].reshape(M, K // 16), rsf), A


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_weight_quantize_crafted_rows(fmt):
    """Weight quantization (qlinear_create) of the crafted rows, exported in
    logical order and compared with the oracle."""
    import precision_gemm_qlinear_b200 as ql
    x = _fp8_power_of_two_rows() if fmt == "fp8" else _nvfp4_scale_sweep_tensor()[0]
    N = (x.shape[0] + 31) // 32 * 32
    w = np.zeros((N, x.shape[1]), np.uint16)
    w[: x.shape[0]] = x
    lay = ql.QLinear(fmt, "bias", to_dev_bf16(w))
    codes, scales, g = lay.export_weights()
    if fmt == "fp8":
        rc, rs = oracle.quant_fp8_rows(w)
        assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))
    else:
        rc, rsf, rg = oracle.quant_nvfp4(w)
        assert np.array_equal(scales, rsf)
        assert np.float32(g).view(np.uint32) == np.float32(rg).view(np.uint32)
    assert np.array_equal(codes, rc)
    lay.close()
