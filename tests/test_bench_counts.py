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
