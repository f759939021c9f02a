"""The benchmark's work counts against brute force over the oracle's block
mask (small layouts): prefill FLOPs and chunked-prefill FLOPs."""
import sys
import os

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import oracle  # noqa: E402
from head_heterogeneous_block_s2_b200 import s2attn, synth  # noqa: E402


def visible_pairs(m, B, rows):
    return sum(int(m[:, pos // B, k // B].sum()) for pos in rows for k in range(pos + 1))


def test_prefill_flops_brute_force():
    w = synth.PrefillWorkload("t", 2, 3, 16, 64, 8, 3, 1, seed=0)
    lay = s2attn.build_layout(3, 8, 3, 1, 8)
    m = oracle.block_mask(3, 8, 3, 1)
    assert bench.prefill_flops(lay, w) == 4 * 16 * 2 * visible_pairs(m, 8, range(64))


def test_chunk_flops_brute_force():
    w = synth.CHUNK_PAGED.with_(heads=3, block=8, stride=3, local=1)
    lay = s2attn.build_layout(3, 8, 3, 1, 10)
    m = oracle.block_mask(3, 10, 3, 1)
    ctx, ql = [37, 80, 5, 9], [20, 80, 0, 1]
    want = sum(visible_pairs(m, 8, range(n - q, n)) for n, q in zip(ctx, ql))
    assert bench.chunk_flops(lay, w, ctx, ql) == 4 * w.head_dim * want


def test_prefill_mma_flops_brute_force():
    """The pair kernel's MMA work, against an enumeration from the oracle's
    block mask: a 128-row tile (two 64-row query blocks) computes, for all its
    rows, every key block either of its query blocks lists; with 128-key
    blocks a tile is one query block and the count is the whole-block one."""
    m = oracle.block_mask(4, 9, 3, 2, (1,))  # odd block count: the last tile holds one block
    w = synth.PrefillWorkload("t", 2, 4, 64, 9 * 64, 64, 3, 2, dense_heads=(1,), seed=0)
    lay = s2attn.build_layout(4, 64, 3, 2, 9, (1,))
    visits = sum(int((m[h, t:t + 2].max(axis=0)).sum()) for h in range(4) for t in range(0, 9, 2))
    assert bench.prefill_mma_flops(lay, w) == 4 * 64 * 128 * 64 * visits * 2
    assert bench.prefill_mma_flops(lay, w) >= bench.prefill_issued_flops(lay, w)
    w2 = synth.PrefillWorkload("t", 2, 4, 64, 9 * 128, 128, 3, 2, dense_heads=(1,), seed=0)
    lay2 = s2attn.build_layout(4, 128, 3, 2, 9, (1,))
    assert bench.prefill_mma_flops(lay2, w2) == bench.prefill_issued_flops(lay2, w2)


def test_prefill_mma_flops_of_the_bench_workloads():
    """Host cost and values on the benchmark's own layouts (+15.3 % over the
    algorithmic count on the 1.3B one: 10,994 tile visits per batch element)."""
    import time

    for name in ("prefill_1p3b", "prefill_7b_hybrid", "prefill_long_131k"):
        w = synth.PREFILL_WORKLOADS[name]
        lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, w.dense_heads)
        t0 = time.time()
        mma = bench.prefill_mma_flops(lay, w)
        assert time.time() - t0 < 10.0
        assert mma >= bench.prefill_issued_flops(lay, w) >= bench.prefill_flops(lay, w)
        if name == "prefill_1p3b":
            assert mma == 4 * w.head_dim * 128 * w.block * 10994 * w.batch


def test_planted_positions_from_the_layout_equal_those_from_the_oracle_mask():
    """bench.py plants the 131K workload's keys from the library's layout on
    the GPU arm and from the oracle's block mask on the reference arm: both
    pick the same tokens, each in a strided key block (beyond the local
    window) of the first half that the last query block sees."""
    w = synth.PREFILL_LONG_131K
    nb = w.num_blocks
    lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, nb)
    m = oracle.block_mask(w.heads, nb, w.stride, w.local)
    a = bench.plant_positions(w, [lay.row(h, nb - 1) for h in range(w.heads)])
    b = bench.plant_positions(w, [np.nonzero(m[h, nb - 1])[0] for h in range(w.heads)])
    assert a == b and len(a) == w.heads
    for h, t in a.items():
        j = t // w.block
        assert m[h, nb - 1, j] and j <= nb // 2 and nb - 1 - j >= w.local
