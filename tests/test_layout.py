"""Layout builder (s2_build_layout, host C++) against the oracle's block rule.

The compacted lists must equal the oracle mask bit-exactly for every
(head, query block, key block) of every workload, be ascending with the
diagonal block last, and the C ABI must reject bad arguments.
"""
import ctypes

import numpy as np
import pytest

import oracle
from head_heterogeneous_block_s2_b200 import s2attn, synth

WORKLOADS = [
    ("tiny", 4, 64, 4, 1, 8, ()),
    ("prefill_1p3b", 16, 64, 8, 2, 128, ()),
    ("prefill_7b_hybrid", 32, 128, 16, 4, 256, (0, 1, 2, 3)),
    ("prefill_long_131k", 32, 128, 16, 4, 1024, ()),
    ("decode_paged", 32, 128, 16, 4, 256, ()),
    ("odd", 5, 64, 3, 2, 37, (4,)),
    ("wide_window", 3, 128, 2, 50, 40, ()),
]

# Active-block totals of the four prefill workloads over all (batch, head):
# batch x per-batch nnz, enumerated independently by the oracle's rule.
EXPECTED_TOTAL = {"tiny": 60, "prefill_1p3b": 4 * 20082, "prefill_7b_hybrid": 216062,
                  "prefill_long_131k": 1172300}


def csr_to_mask(lay):
    H, nb = lay.heads, lay.num_blocks
    m = np.zeros((H, nb, nb), dtype=np.uint8)
    for h in range(H):
        for i in range(nb):
            m[h, i, lay.row(h, i)] = 1
    return m


@pytest.mark.parametrize("name,H,B,S,L,nb,dense", WORKLOADS, ids=[w[0] for w in WORKLOADS])
def test_layout_equals_oracle_mask(name, H, B, S, L, nb, dense):
    lay = s2attn.build_layout(H, B, S, L, nb, dense)
    ref = oracle.block_mask(H, nb, S, L, dense)
    assert np.array_equal(csr_to_mask(lay), ref)
    assert lay.nnz == int(ref.sum())
    # global offsets, ascending lists, diagonal last
    assert lay.row_ptr[0] == 0
    for h in range(H):
        base = h * (nb + 1)
        if h + 1 < H:
            assert lay.row_ptr[base + nb] == lay.row_ptr[base + nb + 1]
        for i in range(nb):
            r = lay.row(h, i)
            assert len(r) >= 1 and r[-1] == i
            assert np.all(np.diff(r) > 0)
    if name in EXPECTED_TOTAL:
        batch = {"prefill_1p3b": 4}.get(name, 1)
        assert batch * lay.nnz == EXPECTED_TOTAL[name]


def test_workload_layouts_match_synth_definitions():
    for w in synth.PREFILL_WORKLOADS.values():
        lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, w.dense_heads)
        assert lay.nnz == int(oracle.block_mask(w.heads, w.num_blocks, w.stride, w.local,
                                                w.dense_heads).sum())


def test_layout_two_call_protocol_and_capacity():
    lib = s2attn.load()
    nnz_only = s2attn.layout_nnz(4, 64, 4, 1, 8)
    assert nnz_only == 60
    d, _keep = s2attn._desc(4, 64, 4, 1, 8, ())
    row_ptr = np.zeros(4 * 9, dtype=np.int32)
    small = np.zeros(10, dtype=np.int32)
    nnz = ctypes.c_int64(0)
    rc = lib.s2_build_layout(ctypes.byref(d), row_ptr.ctypes.data, small.ctypes.data, small.size,
                             ctypes.byref(nnz))
    assert rc == 3 and nnz.value == 60  # S2_ERR_CAPACITY, count still reported


@pytest.mark.parametrize("bad", [dict(H=0), dict(B=0), dict(S=0), dict(L=0), dict(nb=0)])
def test_layout_rejects_bad_arguments(bad):
    p = dict(H=4, B=64, S=4, L=1, nb=8)
    p.update(bad)
    with pytest.raises(s2attn.S2Error) as e:
        s2attn.build_layout(p["H"], p["B"], p["S"], p["L"], p["nb"])
    assert e.value.status == 1
