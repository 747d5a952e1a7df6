"""Helpers shared by the GPU parity tests (host side only)."""
import numpy as np

RTOL = 8e-3   # |gpu - ref| <= RTOL*|ref| + ATOL_RMS*rms(ref), ref = binary64 pre-bf16
ATOL_RMS = 1e-3


def to_dev_bf16(h):
    """uint16 bf16 bit patterns (numpy) -> CUDA bf16 tensor."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(h).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t):
    """CUDA bf16 tensor -> float64 numpy."""
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(gpu, ref, what="", rms=None):
    """Per element |gpu - ref| <= RTOL |ref| + ATOL_RMS rms(ref); rms(ref) is
    over the given elements unless the caller passes the whole output's."""
    ref = np.asarray(ref, np.float64)
    gpu = np.asarray(gpu, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if rms is None:
        rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = RTOL * np.abs(ref) + ATOL_RMS * rms
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:8]
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} elements outside tolerance; rms(ref)={rms:.4g}; "
            f"worst at {worst}: gpu={gpu[worst]!r} ref={ref[worst]!r}; first bad {idx.tolist()}")


def sf_unswizzle(sf_bytes: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Undo the GEMM's scale-factor atom layout -> logical [rows, K/16].

    Atom layout: rows in blocks of 128, K in chunks of 64 (4 scales), 512-byte
    atoms stored chunk-fastest with ceil(K/256)*4 chunks per row block; inside
    an atom, row r and K-block j sit at (r%32)*16 + (r//32)*4 + j.
    """
    kch = ((K + 255) // 256) * 4
    nb = K // 16
    r = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    off = ((r // 128) * kch + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    return np.asarray(sf_bytes)[off]


def sf_logical_offsets(rows: int, K: int) -> np.ndarray:
    """Offsets of the real scales (row < rows, block < K/16), shape [rows, K/16]."""
    kch = ((K + 255) // 256) * 4
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    return ((r // 128) * kch + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)


def sf_layout_offsets(rows: int, K: int) -> np.ndarray:
    """Every (row, block) offset of the padded scale layout, for the bijection test."""
    kch = ((K + 255) // 256) * 4
    mpad = ((rows + 127) // 128) * 128
    r = np.arange(mpad)[:, None]
    b = np.arange(kch * 4)[None, :]
    return (((r // 128) * kch + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)).ravel()


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    """Seeded row sample that includes every tile-boundary row and the tail."""
    g = np.random.default_rng(seed)
    edges = set()
    for t in range(0, M, 128):
        edges.update({t, min(t + 127, M - 1)})
    edges.update({M - 1})
    rest = g.choice(M, size=min(n, M), replace=False)
    return np.array(sorted(edges | set(int(r) for r in rest)), dtype=np.int64)



def sfb_word_offsets(N: int, K: int, bn: int = 256):
    """Byte offset of the scale word of every (weight row n, stage ks, MMA step
    j, replica q) in the replicated weight layout: per bn-row tile, stage and
    step a 4096-byte chunk of 128 rows x 32 bytes in core-matrix order; row
    l = 32 q + (n % bn) % 32, word (n % bn) // 32."""
    nks = (K + 255) // 256
    n = np.arange(((N + bn - 1) // bn) * bn)[:, None, None, None]
    ks = np.arange(nks)[None, :, None, None]
    j = np.arange(4)[None, None, :, None]
    q = np.arange(4)[None, None, None, :]
    loc = n % bn
    l = q * 32 + loc % 32
    w = loc // 32
    return (((n // bn) * nks + ks) * 4 + j) * 4096 + (l // 8) * 256 + (w // 4) * 128 + (l % 8) * 16 + (w % 4) * 4
