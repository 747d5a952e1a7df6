"""The scale-factor atom layout used by the GEMM is a bijection on the padded
[ceil(M/128)*128, ceil(K/256)*16] block grid, so un-swizzling is exact (no GPU)."""
import numpy as np
import pytest

from qlutil import sf_layout_offsets, sf_unswizzle, sfb_word_offsets


@pytest.mark.parametrize("rows,K", [(1, 32), (128, 256), (300, 3072), (257, 544), (16896, 3072)])
def test_sf_layout_is_a_bijection(rows, K):
    off = sf_layout_offsets(rows, K)
    total = ((rows + 127) // 128) * ((K + 255) // 256) * 4 * 512
    assert off.size == total
    assert np.array_equal(np.sort(off), np.arange(total))


def test_sf_unswizzle_roundtrip():
    rows, K = 300, 544
    g = np.random.default_rng(0)
    logical = g.integers(0, 256, (rows, K // 16), dtype=np.uint8)
    kch = ((K + 255) // 256) * 4
    buf = np.zeros(((rows + 127) // 128) * kch * 512, np.uint8)
    for r in range(rows):
        for b in range(K // 16):
            buf[((r // 128) * kch + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4] = logical[r, b]
    assert np.array_equal(sf_unswizzle(buf, rows, K), logical)



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
    # the layout also serves tiles narrower than 256 rows: 224-row tiles use
    # words 0..6 of every row, the slots are distinct and
    # the unused word 7 of each row is exactly what is left over
    off = sfb_word_offsets(N, K, 224).ravel()
    tiles = (N + 223) // 224
    total = tiles * ((K + 255) // 256) * 4 * 4096
    assert len(np.unique(off)) == off.size
    assert off.size * 8 == total // 4 * 7
    assert np.all(((off % 256) % 16 // 4 + 4 * ((off % 256) // 128)) != 7)
