"""Pins for the oracle's chunked prefill over a paged cache.

Each sequence appends a chunk of query tokens at the end of its context (the
chunk's own keys and values already in the cache) and every chunk row attends
to the keys up to its position under the same block rule. Pinned against the
oracle prefill on the same tokens laid out densely (itself pinned against SDPA
and hand-enumerated patterns), against the decode oracle for one-token
chunks, and for independence from the physical page order.
"""
import numpy as np
import pytest
import torch

import oracle
from head_heterogeneous_block_s2_b200 import synth


def paged(k_dense, v_dense, ctx, page, seed):
    batch, H, n, D = k_dense.shape
    pages = [-(-c // page) for c in ctx]
    perm = np.random.default_rng(seed).permutation(sum(pages)).astype(np.int32)
    bt = np.full((batch, max(pages)), -1, dtype=np.int32)
    kc = torch.zeros(sum(pages), H, page, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    off = 0
    for s in range(batch):
        for lp in range(pages[s]):
            pp = perm[off + lp]
            bt[s, lp] = pp
            t0, t1 = lp * page, min((lp + 1) * page, ctx[s])
            kc[pp, :, : t1 - t0] = k_dense[s, :, t0:t1]
            vc[pp, :, : t1 - t0] = v_dense[s, :, t0:t1]
        off += pages[s]
    return kc, vc, bt


def make(ctx, qlen, H=3, D=16, B=8, S=3, L=1, dense=(), seed=0):
    batch, n = len(ctx), max(ctx)
    w = synth.PrefillWorkload("t", batch, H, D, n, B, S, L, dense_heads=dense, seed=seed)
    qd, kd, vd = synth.prefill_inputs(w)
    q_start = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    rows = [qd[s, :, ctx[s] - qlen[s]:ctx[s]].transpose(0, 1) for s in range(batch)]
    q = torch.cat(rows, 0).contiguous() if sum(qlen) else torch.zeros(0, H, D, dtype=torch.bfloat16)
    return w, qd, kd, vd, q, q_start


@pytest.mark.parametrize("dense", [(), (1,)])
def test_chunk_rows_equal_prefill_rows(dense):
    ctx, qlen = [5, 40, 64, 33, 17], [5, 13, 1, 0, 9]
    w, qd, kd, vd, q, q_start = make(ctx, qlen, dense=dense, seed=1)
    kc, vc, bt = paged(kd, vd, ctx, 4, 0)
    out, lse = oracle.chunk(q, kc, vc, bt, ctx, q_start, 8, w.scale, S=3, L=1, dense_heads=dense)
    H = 3
    for s in range(len(ctx)):
        c = ctx[s]
        if qlen[s] == 0:
            continue
        rows = [h * c + p for p in range(c - qlen[s], c) for h in range(H)]
        ref, lref = oracle.prefill(qd[s:s + 1, :, :c].contiguous(), kd[s:s + 1, :, :c].contiguous(),
                                   vd[s:s + 1, :, :c].contiguous(), 8, 3, 1, w.scale, dense,
                                   rows=rows)
        got = out[q_start[s]:q_start[s + 1]].reshape(-1, 16)
        assert np.abs(got - ref).max() < 1e-12
        assert np.abs(lse[q_start[s]:q_start[s + 1]].reshape(-1) - lref).max() < 1e-12


def test_one_token_chunks_equal_decode():
    ctx = [7, 30, 64]
    w, qd, kd, vd, q, q_start = make(ctx, [1, 1, 1], seed=2)
    kc, vc, bt = paged(kd, vd, ctx, 4, 1)
    out, lse = oracle.chunk(q, kc, vc, bt, ctx, q_start, 8, w.scale, S=3, L=1)
    dout, dlse = oracle.decode(q, kc, vc, bt, ctx, 8, 3, 1, w.scale)
    assert np.array_equal(out.reshape(-1, 16), dout) and np.array_equal(lse.reshape(-1), dlse)


def test_mask_rule_and_page_order():
    ctx, qlen = [40, 64], [40, 20]
    w, qd, kd, vd, q, q_start = make(ctx, qlen, seed=3)
    kc, vc, bt = paged(kd, vd, ctx, 4, 2)
    a = oracle.chunk(q, kc, vc, bt, ctx, q_start, 8, w.scale, S=3, L=1)
    b = oracle.chunk(q, kc, vc, bt, ctx, q_start, 8, w.scale, bmask=oracle.block_mask(3, 8, 3, 1))
    kc2, vc2, bt2 = paged(kd, vd, ctx, 4, 9)
    c = oracle.chunk(q, kc2, vc2, bt2, ctx, q_start, 8, w.scale, S=3, L=1)
    for x, y in ((a, b), (a, c)):
        assert np.array_equal(x[0], y[0]) and np.array_equal(x[1], y[1])


def test_chunk_longer_than_context_is_rejected():
    ctx = [8]
    w, qd, kd, vd, q, q_start = make(ctx, [8], seed=4)
    kc, vc, bt = paged(kd, vd, ctx, 4, 0)
    with pytest.raises(ValueError):
        oracle.chunk(q, kc, vc, bt, [7], q_start, 8, w.scale, S=3, L=1)
