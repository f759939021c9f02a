"""Per-context-range and per-head-mask layout builders (host C++) against the
oracle's block rules.

s2_build_layout_ranges and s2_build_layout_mask must produce lists equal, bit
for bit, to the oracle's masks, ascending, with global offsets, and reject
malformed specifications.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
from conftest import GOLDEN, read_block_pattern
from head_heterogeneous_block_s2_b200 import s2attn

FIXTURE_RANGES = [
    [(2, 0, 0, True), (8, 3, 1, False)],
    [(3, 2, 2, False), (5, 0, 3, False), (8, 4, 1, False)],
    [(4, 0, 0, False), (8, 2, 1, False)],
]


def csr_to_mask(lay):
    H, nb = lay.heads, lay.num_blocks
    m = np.zeros((H, nb, nb), dtype=np.uint8)
    for h in range(H):
        for i in range(nb):
            m[h, i, lay.row(h, i)] = 1
    return m


def check_csr(lay):
    H, nb = lay.heads, lay.num_blocks
    assert lay.row_ptr[0] == 0 and lay.row_ptr[-1] == lay.nnz
    for h in range(H):
        base = h * (nb + 1)
        if h + 1 < H:
            assert lay.row_ptr[base + nb] == lay.row_ptr[base + nb + 1]
        for i in range(nb):
            r = lay.row(h, i)
            assert np.all(np.diff(r) > 0) and (len(r) == 0 or (r[0] >= 0 and r[-1] <= i))


def random_ranges(rng, H, nb):
    out = []
    for _ in range(H):
        cuts = sorted(set(rng.integers(1, nb, size=rng.integers(0, 4)).tolist()))
        ends = cuts + [nb]
        head = []
        for e in ends:
            head.append((e, int(rng.integers(0, 9)), int(rng.integers(0, 4)), bool(rng.random() < 0.2)))
        out.append(head)
    return out


def test_fixture_through_the_library():
    want = read_block_pattern(os.path.join(GOLDEN, "range_block_pattern.txt"))
    lay = s2attn.build_layout_ranges(FIXTURE_RANGES, 64, 8)
    got = {(h, i): [int(j) for j in lay.row(h, i)] for h in range(3) for i in range(8)}
    assert got == want and lay.nnz == 54
    check_csr(lay)


@pytest.mark.parametrize("seed", range(6))
def test_random_ranges_equal_oracle_mask(seed):
    rng = np.random.default_rng(seed)
    H, nb = int(rng.integers(1, 9)), int(rng.integers(1, 70))
    ranges = random_ranges(rng, H, nb)
    lay = s2attn.build_layout_ranges(ranges, 128, nb)
    assert np.array_equal(csr_to_mask(lay), oracle.range_block_mask(nb, ranges))
    check_csr(lay)


@pytest.mark.parametrize("H,B,S,L,nb,dense", [(16, 64, 8, 2, 128, ()), (32, 128, 16, 4, 256, (0, 1, 2, 3)),
                                              (5, 64, 3, 2, 37, (4,))])
def test_one_range_equals_hhst_builder(H, B, S, L, nb, dense):
    a = s2attn.build_layout(H, B, S, L, nb, dense)
    b = s2attn.build_layout_ranges([[(nb, S, L, h in dense)] for h in range(H)], B, nb)
    assert np.array_equal(a.row_ptr, b.row_ptr) and np.array_equal(a.col_idx, b.col_idx)


def test_dense_prefix_at_long_context():
    """Every head sees the first 4 blocks, then the long-context HHST rule."""
    nb, H = 1024, 32
    ranges = [[(4, 0, 0, True), (nb, 16, 4, False)] for _ in range(H)]
    lay = s2attn.build_layout_ranges(ranges, 128, nb)
    base = s2attn.build_layout(H, 128, 16, 4, nb)
    # rows gain exactly the prefix blocks HHST did not already list
    for h in (0, 5, 31):
        for i in (0, 3, 4, 7, 500, 1023):
            want = sorted(set(base.row(h, i).tolist()) | set(range(min(4, i + 1))))
            assert lay.row(h, i).tolist() == want


@pytest.mark.parametrize("seed", range(4))
def test_mask_builder_round_trip(seed):
    rng = np.random.default_rng(100 + seed)
    H, nb = int(rng.integers(1, 6)), int(rng.integers(1, 50))
    m = np.tril(rng.random((H, nb, nb)) < 0.3).astype(np.uint8)
    lay = s2attn.build_layout_mask(m, 64)
    assert np.array_equal(csr_to_mask(lay), m)
    check_csr(lay)


def test_empty_layout():
    lay = s2attn.build_layout_mask(np.zeros((2, 5, 5), np.uint8), 64)
    assert lay.nnz == 0 and (lay.row_ptr == 0).all()
    lay = s2attn.build_layout_ranges([[(5, 0, 0, False)]] * 2, 64, 5)
    assert lay.nnz == 0


def _raw_ranges(ptr, ranges, nb, H=None):
    lib = s2attn.load()
    ptr = np.asarray(ptr, dtype=np.int32)
    arr = (s2attn._ContextRange * max(1, len(ranges)))(*[s2attn._ContextRange(*r) for r in ranges])
    nnz = ctypes.c_int64(0)
    return lib.s2_build_layout_ranges(len(ptr) - 1 if H is None else H, nb, ptr.ctypes.data,
                                      ctypes.cast(arr, ctypes.c_void_p), None, None, 0,
                                      ctypes.byref(nnz)), nnz.value


def test_ranges_builder_rejects_malformed_specs():
    bad = 1  # S2_ERR_INVALID_ARG
    assert _raw_ranges([0, 1], [(8, 2, 1, 0)], 8)[0] == 0
    assert _raw_ranges([0, 1], [(7, 2, 1, 0)], 8)[0] == bad          # does not end at nb
    assert _raw_ranges([0, 1], [(9, 2, 1, 0)], 8)[0] == bad          # past nb
    assert _raw_ranges([0, 2], [(5, 2, 1, 0), (5, 2, 1, 0)], 8)[0] == bad  # not ascending
    assert _raw_ranges([0, 1], [(8, -1, 1, 0)], 8)[0] == bad         # negative stride
    assert _raw_ranges([0, 1], [(8, 2, -1, 0)], 8)[0] == bad         # negative window
    assert _raw_ranges([0, 0, 1], [(8, 2, 1, 0)], 8)[0] == bad       # head 0 has no range
    assert _raw_ranges([1, 2], [(8, 2, 1, 0), (8, 2, 1, 0)], 8)[0] == bad  # range_ptr[0] != 0
    with pytest.raises(s2attn.S2Error):
        s2attn.build_layout_ranges([[(4, 1, 1, False)]], 64, 8)


def test_mask_builder_rejects_blocks_above_the_diagonal():
    m = np.zeros((1, 4, 4), np.uint8)
    m[0, 1, 2] = 1
    with pytest.raises(s2attn.S2Error) as e:
        s2attn.build_layout_mask(m, 64)
    assert e.value.status == 1


def test_two_call_protocol_and_capacity():
    lib = s2attn.load()
    m = np.tril(np.ones((2, 6, 6), np.uint8))
    nnz = ctypes.c_int64(0)
    assert lib.s2_build_layout_mask(2, 6, m.ctypes.data, None, None, 0, ctypes.byref(nnz)) == 0
    assert nnz.value == 2 * 21
    rp = np.zeros(2 * 7, np.int32)
    ci = np.zeros(10, np.int32)
    assert lib.s2_build_layout_mask(2, 6, m.ctypes.data, rp.ctypes.data, ci.ctypes.data, 10,
                                    ctypes.byref(nnz)) == 3  # S2_ERR_CAPACITY
    assert lib.s2_build_layout_mask(2, 6, None, None, None, 0, ctypes.byref(nnz)) == 1
