"""Per-context-range and per-head-mask layouts on the GPU: the prefill and decode
kernels (through the C ABI) against the oracle's mask entry points.

The kernels are driven by the compacted lists alone, so any layout the
builders accept must give masked softmax attention over exactly the listed
blocks, including query blocks whose list is empty (zero output, LSE -inf)
and whole 128-row tiles, or tile pairs, with no key at all.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu

FIXTURE_RANGES = [
    [(2, 0, 0, True), (8, 3, 1, False)],
    [(3, 2, 2, False), (5, 0, 3, False), (8, 4, 1, False)],
    [(4, 0, 0, False), (8, 2, 1, False)],
]


def sink_then_hhst(H, nb, sink, S, L):
    return [[(sink, 0, 0, True), (nb, S, L, False)] for _ in range(H)]


def prefill_vs_oracle(s2, lay, w, bmask, rows=None):
    q, k, v = synth.prefill_inputs(w)
    out, lse = s2.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill_mask(q, k, v, w.block, bmask, w.scale, rows=rows)
    got = out.reshape(-1, w.head_dim).cpu()
    gl = lse.reshape(-1).cpu().double().numpy()
    if rows is not None:
        got, gl = got[torch.as_tensor(rows)], gl[rows]
    parity(got, ref)
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(gl), empty)
    if empty.any():
        assert (got[torch.as_tensor(empty)] == 0).all()
    if (~empty).any():
        parity(gl[~empty], ref_lse[~empty], max_tol=1e-3, mean_tol=1e-4)
    return empty


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("bk", [64, 128])
def test_fixture_ranges_all_rows(s2gpu, hd, bk):
    w = synth.PrefillWorkload("t", 2, 3, hd, 8 * bk, bk, 1, 1, seed=50)
    lay = s2gpu.build_layout_ranges(FIXTURE_RANGES, bk, 8, device="cuda")
    empty = prefill_vs_oracle(s2gpu, lay, w, oracle.range_block_mask(8, FIXTURE_RANGES))
    # head 2 sees nothing in blocks 0..3: whole tile pairs with no key
    e = empty.reshape(2, 3, 8 * bk)
    assert e[:, 2, : 4 * bk].all() and not e[:, :2].any()


@pytest.mark.parametrize("hd,bk,nb", [(128, 64, 9), (128, 128, 5), (64, 64, 12)])
def test_sink_then_hhst_all_rows(s2gpu, hd, bk, nb):
    ranges = sink_then_hhst(4, nb, 2, 3, 1)
    w = synth.PrefillWorkload("t", 2, 4, hd, nb * bk, bk, 1, 1, seed=51)
    lay = s2gpu.build_layout_ranges(ranges, bk, nb, device="cuda")
    prefill_vs_oracle(s2gpu, lay, w, oracle.range_block_mask(nb, ranges))


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("bk", [64, 128])
def test_random_masks_with_empty_rows(s2gpu, seed, bk):
    nb, H = 10, 3
    rng = np.random.default_rng(60 + seed)
    m = np.tril(rng.random((H, nb, nb)) < 0.35).astype(np.uint8)
    m[1, 3] = 0  # one empty query block inside a tile that also has a seen block
    m[2, :4] = 0  # whole tiles with no key
    w = synth.PrefillWorkload("t", 1, H, 128, nb * bk, bk, 1, 1, seed=70 + seed)
    lay = s2gpu.build_layout_mask(m, bk, device="cuda")
    empty = prefill_vs_oracle(s2gpu, lay, w, m)
    assert empty.reshape(H, -1)[1, 3 * bk:4 * bk].all()


def test_layout_with_no_block_at_all(s2gpu):
    w = synth.PrefillWorkload("t", 1, 2, 128, 512, 128, 1, 1, seed=52)
    lay = s2gpu.build_layout_mask(np.zeros((2, 4, 4), np.uint8), 128, device="cuda")
    assert lay.nnz == 0
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    out, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    assert (out == 0).all() and torch.isneginf(lse).all()


def test_long_context_sink_sampled_rows(s2gpu):
    """32 heads x 16K tokens, B = 128: a dense 4-block sink, then S 16, L 4."""
    H, nb, bk = 32, 128, 128
    ranges = sink_then_hhst(H, nb, 4, 16, 4)
    w = synth.PrefillWorkload("t", 1, H, 128, nb * bk, bk, 1, 1, seed=53)
    lay = s2gpu.build_layout_ranges(ranges, bk, nb, device="cuda")
    rng = np.random.default_rng(5)
    seq = nb * bk
    rows = []
    for h in range(H):
        for qpos in [0, 129, 511, 512, seq - 1] + rng.integers(0, seq, 6).tolist():
            rows.append(h * seq + int(qpos))
    prefill_vs_oracle(s2gpu, lay, w, oracle.range_block_mask(nb, ranges), rows=rows)


# ---------------------------------------------------------------- decode

def decode_vs_oracle(s2, lay, w, d, bmask, splits):
    out, lse = s2.decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(),
                         d.ctx_lens.cuda(), lay, scale=w.scale, num_splits=splits, want_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_mask(d.q, d.k_cache, d.v_cache, d.block_table.cpu().numpy(),
                                      d.ctx_lens.cpu().numpy(), w.block, bmask, w.scale)
    got = out.reshape(-1, w.head_dim).cpu()
    gl = lse.reshape(-1).cpu().double().numpy()
    parity(got, ref)
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(gl), empty)
    assert (got[torch.as_tensor(empty)] == 0).all()
    parity(gl[~empty], ref_lse[~empty], max_tol=1e-3, mean_tol=1e-4)
    return empty


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_decode_fixture_ranges(s2gpu, splits):
    # 3 heads, blocks of 128 tokens, contexts ending in every block (and in the
    # empty blocks 0..3 of head 2)
    w = synth.DecodeWorkload("t", 8, 3, 128, 1, 1024, 16, 128, 1, 1, seed=54)
    ctx = [1, 100, 300, 512, 513, 700, 900, 1024]
    d = synth.decode_inputs(w, ctx_lens=ctx)
    lay = s2gpu.build_layout_ranges(FIXTURE_RANGES, 128, 8, device="cuda")
    empty = decode_vs_oracle(s2gpu, lay, w, d, oracle.range_block_mask(8, FIXTURE_RANGES), splits)
    assert empty.reshape(8, 3)[:4, 2].all() and not empty.reshape(8, 3)[4:, 2].any()


@pytest.mark.parametrize("splits", [1, 7])
def test_decode_sink_then_hhst(s2gpu, splits):
    w = synth.DecodeWorkload("t", 6, 8, 128, 1, 6000, 16, 128, 4, 2, seed=55)
    nb = w.num_blocks
    ranges = sink_then_hhst(8, nb, 3, 4, 2)
    d = synth.decode_inputs(w, ctx_lens=[1, 129, 385, 2000, 4097, 6000])
    lay = s2gpu.build_layout_ranges(ranges, 128, nb, device="cuda")
    decode_vs_oracle(s2gpu, lay, w, d, oracle.range_block_mask(nb, ranges), splits)
