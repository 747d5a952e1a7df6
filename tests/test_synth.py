"""The seeded input generators (`synth/`), on the CPU: determinism, the
binary64 -> binary32 -> bf16 rounding chain against PyTorch's own
conversion, the outlier-channel recipe, the distributions, and the FLUX
workload shapes every parity test and the benchmark draw from."""
import numpy as np
import pytest

from synth import WORKLOADS
from synth.tensors import bf16_bits_from_f64, bf16_bits_to_f32, draw, rng_for


def test_draws_are_deterministic_and_stream_separated():
    a = draw("normal", (64, 96), 0, "x")
    assert np.array_equal(a, draw("normal", (64, 96), 0, "x"))
    assert not np.array_equal(a, draw("normal", (64, 96), 1, "x"))    # another seed
    assert not np.array_equal(a, draw("normal", (64, 96), 0, "w"))    # another tensor
    # one PCG64 stream per (seed, tensor id): the same stream whatever else was drawn
    g = rng_for(0, "x")
    assert np.array_equal(bf16_bits_from_f64(g.normal(0.0, 1.0, size=(64, 96))), a)


def test_bf16_rounding_matches_torch_on_random_and_tie_values():
    import torch
    rng = np.random.default_rng(7)
    f = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact ties at the 16 dropped bits, both parities of the kept LSB
        (np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40490000 | 0x8000,
                   0x00008000, 0x00018000, 0x7F7F8000], dtype=np.uint32)).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.4e38, -3.4e38], dtype=np.float32),
    ]).astype(np.float32)
    ours = bf16_bits_from_f64(f.astype(np.float64))
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # and back: bf16 -> f32 is exact
    assert np.array_equal(bf16_bits_to_f32(ours).astype(np.float32),
                          torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_binary64_values_round_through_binary32_first():
    # 1 + 2^-8 + 2^-30 lies above the bf16 tie at 1 + 2^-8 in binary64, but
    # binary32 rounds it onto the tie, which then rounds to the even bf16 1.0
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert bf16_bits_from_f64(np.array([v]))[0] == 0x3F80


def test_outlier_channels_scale_a_seeded_choice_of_columns():
    K = 3072
    base = draw("normal", (32, K), 0, "x")
    out = draw("normal", (32, K), 0, "x", outlier_frac=0.01, outlier_factor=8.0)
    changed = np.flatnonzero((base != out).any(axis=0))
    assert len(changed) == round(0.01 * K)                        # 31 of 3072
    # the chosen columns carry exactly the base draw times the factor
    g = rng_for(0, "x")
    a = g.normal(0.0, 1.0, size=(32, K))
    cols = g.choice(K, size=31, replace=False)
    assert sorted(cols.tolist()) == changed.tolist()
    a[:, cols] *= 8.0
    assert np.array_equal(out, bf16_bits_from_f64(a))


def test_distributions_have_the_stated_moments():
    x = bf16_bits_to_f32(draw("normal", (512, 1024), 0, "x")).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    w = bf16_bits_to_f32(draw("normal", (512, 1024), 0, "w", std=0.02)).astype(np.float64)
    assert abs(w.std() / 0.02 - 1.0) < 0.01
    g = bf16_bits_to_f32(draw("normal", (4096,), 0, "gate", mean=1.0, std=0.1)).astype(np.float64)
    assert abs(g.mean() - 1.0) < 0.01 and abs(g.std() - 0.1) < 0.01
    # Student-t(4) has excess kurtosis (infinite in theory; heavy in a sample)
    t = bf16_bits_to_f32(draw("student_t", (512, 1024), 0, "x", nu=4)).astype(np.float64)
    kurt = ((t - t.mean()) ** 4).mean() / t.var() ** 2
    assert kurt > 5.0 and abs(t.var() - 2.0) < 0.3                 # var = nu / (nu - 2)


@pytest.mark.parametrize("name,shapes", [
    ("tiny_fp8", [("fp8", 128, 256, 512)]),
    ("flux_qkv_fp8", [("fp8", 4608, 3072, 9216)]),
    ("flux_mlp_fp8", [("fp8", 4608, 3072, 12288), ("fp8", 4608, 12288, 3072)]),
    ("flux2k_swiglu_nvfp4", [("nvfp4", 16896, 3072, 16384)]),
    ("cfg_linear1", [("fp8", 33792, 3072, 21504), ("nvfp4", 33792, 3072, 21504)]),
])
def test_flux_workload_shapes(name, shapes):
    # 4608 = 4096 image + 512 text tokens (1024^2), 16896 = 16384 + 512
    # (2048^2), CFG doubles M; hidden 3072, QKV 3 x 3072, MLP 4 x 3072,
    # linear1 = QKV + MLP = 21504 with the split at 9216
    wl = WORKLOADS[name]
    assert [(l.fmt, l.M, l.K, l.N) for l in wl.layers] == shapes
    for l in wl.layers:
        if l.epi == "split_bias_gelu":
            assert l.split_col == 9216
        if l.epi == "swiglu":
            assert l.Nout == l.N // 2 == 8192
