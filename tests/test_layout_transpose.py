"""Transposed lists (s2_build_layout_transpose, host C++) for the backward pass:
for each head and key block, the ascending query blocks that list it."""
import ctypes

import numpy as np
import pytest

from head_heterogeneous_block_s2_b200 import s2attn


def mask_of(lay):
    m = np.zeros((lay.heads, lay.num_blocks, lay.num_blocks), dtype=np.uint8)
    for h in range(lay.heads):
        for i in range(lay.num_blocks):
            m[h, i, lay.row(h, i)] = 1
    return m


def transposed_mask(lay):
    lay.transposed()
    nb = lay.num_blocks
    m = np.zeros((lay.heads, nb, nb), dtype=np.uint8)
    for h in range(lay.heads):
        for j in range(nb):
            a, b = lay.t_col_ptr[h * (nb + 1) + j], lay.t_col_ptr[h * (nb + 1) + j + 1]
            col = lay.t_row_idx[a:b]
            assert np.all(np.diff(col) > 0) and (len(col) == 0 or col[0] >= j)
            m[h, col, j] = 1
    assert lay.t_col_ptr[0] == 0 and lay.t_col_ptr[-1] == lay.nnz
    return m


@pytest.mark.parametrize("args", [(4, 64, 4, 1, 8, ()), (16, 64, 8, 2, 128, ()),
                                  (32, 128, 16, 4, 256, (0, 1, 2, 3)), (5, 64, 3, 2, 37, (4,))])
def test_transpose_of_hhst_layouts(args):
    lay = s2attn.build_layout(*args)
    assert np.array_equal(transposed_mask(lay), mask_of(lay))


def test_transpose_of_masks_with_empty_rows_and_columns():
    rng = np.random.default_rng(4)
    m = np.tril(rng.random((3, 30, 30)) < 0.2).astype(np.uint8)
    m[1, :, 5] = 0
    m[2, 7] = 0
    lay = s2attn.build_layout_mask(m, 64)
    assert np.array_equal(transposed_mask(lay), m)
    empty = s2attn.build_layout_mask(np.zeros((2, 4, 4), np.uint8), 64)
    assert (transposed_mask(empty) == 0).all()


def _raw(row_ptr, col_idx, H, nb):
    rp = np.asarray(row_ptr, np.int32)
    ci = np.asarray(col_idx, np.int32)
    cp = np.zeros(H * (nb + 1), np.int32)
    ri = np.zeros(max(1, ci.size), np.int32)
    return s2attn.load().s2_build_layout_transpose(H, nb, rp.ctypes.data, ci.ctypes.data, ci.size,
                                                   cp.ctypes.data, ri.ctypes.data)


def test_transpose_rejects_malformed_layouts():
    assert _raw([0, 1, 3], [0, 0, 1], 1, 2) == 0
    assert _raw([0, 1, 3], [0, 1, 0], 1, 2) == 1   # not ascending
    assert _raw([0, 2, 3], [0, 1, 1], 1, 2) == 1   # j > i in row 0
    assert _raw([0, 1, 4], [0, 0, 1, 1], 1, 2) == 1  # duplicate
    assert _raw([1, 1, 2], [0, 0], 1, 2) == 1      # offsets not starting at 0


@pytest.mark.parametrize("args", [(16, 64, 8, 2, 128, ()), (5, 64, 3, 2, 37, (4,)), (3, 64, 4, 1, 1, ())])
def test_key_tiles_cover_every_block_once(args):
    lay = s2attn.build_layout(*args).transposed()
    kt = lay.t_key_tiles
    H, nb = lay.heads, lay.num_blocks
    assert kt.shape == (H, (nb + 1) // 2, 2)
    for h in range(H):
        got = sorted(int(x) for x in kt[h].reshape(-1) if x >= 0)
        assert got == list(range(nb))
        assert (kt[h].reshape(-1) < 0).sum() == (nb % 2)


def test_key_tiles_pair_strided_blocks_under_hhst():
    # B 64, S 8, L 2: strided blocks of head h are j = -h mod 8; they pair with j + 8
    lay = s2attn.build_layout(16, 64, 8, 2, 128).transposed()
    for h in (0, 3, 9):
        j0 = (-h) % 8
        strided = list(range(j0, 126, 8))
        tiles = [tuple(t) for t in lay.t_key_tiles[h]]
        for a, b in zip(strided[0:-1:2], strided[1::2]):
            assert (a, b) in tiles
