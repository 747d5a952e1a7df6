"""The scale-factor layouts used by the GEMM are bijections on the padded block
grid, so un-swizzling is exact, and the activation layout is the copy source
the GEMM assumes (no GPU)."""
import numpy as np
import pytest

from qlutil import sf_layout_offsets, sf_unswizzle, sfb_word_offsets


@pytest.mark.parametrize("rows,K", [(1, 32), (128, 256), (300, 3072), (257, 544), (16896, 3072)])
def test_sf_layout_is_a_bijection(rows, K):
    off = sf_layout_offsets(rows, K)
    total = ((rows + 127) // 128) * ((K + 255) // 256) * 4 * 512
    assert off.size == total
    assert np.array_equal(np.sort(off), np.arange(total))


def _atoms_then_pairs(logical, rows, K):
    """Build the activation scale buffer in two explicit steps: 512-byte atoms
    (row r, block j of a chunk at (r%32)*16 + ((r%128)//32)*4 + j), then each
    pair of atoms interleaved in 128-byte pieces."""
    kch = ((K + 255) // 256) * 4
    nrb = (rows + 127) // 128
    atoms = np.zeros((nrb, kch, 512), np.uint8)
    for r in range(rows):
        for b in range(K // 16):
            atoms[r // 128, b // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4] = logical[r, b]
    units = np.zeros((nrb, kch // 2, 1024), np.uint8)
    for piece in range(4):
        units[:, :, piece * 256:piece * 256 + 128] = atoms[:, 0::2, piece * 128:(piece + 1) * 128]
        units[:, :, piece * 256 + 128:piece * 256 + 256] = atoms[:, 1::2, piece * 128:(piece + 1) * 128]
    return atoms, units.ravel()


def test_sf_unswizzle_roundtrip():
    rows, K = 300, 544
    g = np.random.default_rng(0)
    logical = g.integers(0, 256, (rows, K // 16), dtype=np.uint8)
    _, buf = _atoms_then_pairs(logical, rows, K)
    assert np.array_equal(sf_unswizzle(buf, rows, K), logical)


def test_four_copies_of_a_pair_are_the_128x256b_copy_source():
    # The GEMM loads each 1 KB pair four times side by side and copies the
    # 4 KB with one 128 x 256-bit tcgen05.cp (8-row core matrices: row group g
    # at g*256 bytes, second 16-byte column at +128).  TMEM lane L = 32q + l
    # must then receive atom 2i's 16 bytes of lane l (columns 0-3) and atom
    # 2i+1's (columns 4-7), for every sub-partition q.
    rows, K = 128, 512
    g = np.random.default_rng(1)
    logical = g.integers(0, 256, (rows, K // 16), dtype=np.uint8)
    atoms, buf = _atoms_then_pairs(logical, rows, K)
    for unit in range(2):
        src = np.tile(buf[unit * 1024:(unit + 1) * 1024], 4)
        for L in range(128):
            for h in range(2):
                o = (L >> 3) * 256 + h * 128 + (L & 7) * 16
                l = L & 31
                assert np.array_equal(src[o:o + 16], atoms[0, 2 * unit + h, l * 16:l * 16 + 16])


@pytest.mark.parametrize("N,K", [(256, 32), (512, 256), (768, 3072), (256, 544)])
def test_weight_sf_layout_words_tile_the_buffer(N, K):
    # every (row, stage, step, replica) word has its own 4-byte slot and the
    # slots cover the buffer exactly
    off = sfb_word_offsets(N, K).ravel()
    total = ((N + 255) // 256) * ((K + 255) // 256) * 4 * 4096
    assert np.all(off % 4 == 0)
    assert np.array_equal(np.sort(off), np.arange(0, total, 4))


@pytest.mark.parametrize("N,K", [(224, 256), (768, 3072), (21504, 512)])
def test_weight_sf_layout_224_row_tiles(N, K):
    # 224-row tiles use words 0..6 of every row: the slots are distinct and
    # the unused word 7 of each row is exactly what is left over
    off = sfb_word_offsets(N, K, 224).ravel()
    tiles = (N + 223) // 224
    total = tiles * ((K + 255) // 256) * 4 * 4096
    assert len(np.unique(off)) == off.size
    assert off.size * 8 == total // 4 * 7
    assert np.all(((off % 256) % 16 // 4 + 4 * ((off % 256) // 128)) != 7)
