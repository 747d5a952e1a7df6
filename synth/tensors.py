"""Seeded random tensors, rounded to bf16 on the host.

Recipe (stated once, used everywhere):
  * one numpy PCG64 stream per (seed, tensor id), seeded through
    ``np.random.SeedSequence([seed, tensor_id])``;
  * values are drawn in binary64, rounded to binary32 (round to nearest even)
    and then to bf16 (round to nearest even on the 16 dropped bits);
  * ``N(mu, sigma)``: sigma is the standard deviation;
  * Student-t(nu): numpy's ``standard_t``;
  * outlier channels: a seeded choice (without replacement) of
    ``round(frac * K)`` input channels whose values are multiplied by a factor
    before the rounding.
"""
import numpy as np

TENSOR_IDS = {"x": 1, "w": 2, "bias": 3, "gate": 4, "residual": 5, "x2": 6, "w2": 7, "bias2": 8,
              "q_norm": 9, "k_norm": 10}


def rng_for(seed: int, tensor: str) -> np.random.Generator:
    tid = TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), tid])))


def bf16_bits_from_f64(a) -> np.ndarray:
    """binary64 -> binary32 (RNE) -> bf16 (RNE), returned as uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = r.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32)


def draw(kind: str, shape, seed: int, tensor: str, *, mean=0.0, std=1.0, nu=None,
         outlier_frac=0.0, outlier_factor=1.0) -> np.ndarray:
    """Draw a bf16 tensor (uint16 bit patterns) of the given distribution."""
    g = rng_for(seed, tensor)
    shape = tuple(int(s) for s in shape)
    if kind == "normal":
        a = g.normal(mean, std, size=shape)
    elif kind == "student_t":
        a = g.standard_t(nu, size=shape)
    else:
        raise ValueError(kind)
    if outlier_frac > 0:
        K = shape[-1]
        n_out = int(round(outlier_frac * K))
        if n_out > 0:
            cols = g.choice(K, size=n_out, replace=False)
            a[..., cols] *= outlier_factor
    return bf16_bits_from_f64(a)
