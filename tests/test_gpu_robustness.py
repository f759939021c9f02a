"""Failure detection without a GPU fault.

* Every device wait is bounded: with the limit forced to 0, any wait that is
  not already satisfied gives up, the kernel sets the device timeout flag,
  drains its own copies and MMAs, frees TMEM and returns. The context must stay
  usable: after clearing the flag, the same call gives correct results.
* Malformed layouts (out-of-range or non-causal key blocks, broken row
  offsets) are skipped and reported as S2_ERR_DEVICE_INDEX, never faulted.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import s2attn, synth

pytestmark = pytest.mark.gpu

S2_ERR_TIMEOUT, S2_ERR_DEVICE_INDEX = 5, 6


def tiny():
    w = synth.TINY
    q, k, v = synth.prefill_inputs(w)
    lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, device="cuda")
    return w, q, k, v, lay


def test_prefill_wait_timeout_is_reported_and_recoverable(s2gpu):
    w, q, k, v, lay = tiny()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    s2gpu.set_wait_timeout_ns(0)
    try:
        s2gpu.prefill(qc, kc, vc, lay, scale=w.scale)
        rc, flags = s2gpu.device_status(reset=True)
    finally:
        s2gpu.set_wait_timeout_ns(500_000_000)
    assert rc == S2_ERR_TIMEOUT and flags & 1
    out = s2gpu.prefill(qc, kc, vc, lay, scale=w.scale)
    torch.cuda.synchronize()
    ref, _ = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale)
    parity(out.reshape(-1, w.head_dim), ref)


def test_decode_wait_timeout_is_reported_and_recoverable(s2gpu):
    # dense heads and one split: each CTA streams ~125 pages through its 8-stage
    # ring, so the producer must wait for stages to be released
    dense = tuple(range(8))
    wd = synth.DecodeWorkload("t", 4, 8, 128, 1, 2000, 16, 128, 4, 2, dense_heads=dense, seed=3)
    d = synth.decode_inputs(wd, ctx_lens=[1900, 1950, 1990, 2000])
    lay = s2gpu.build_layout(wd.heads, wd.block, wd.stride, wd.local, wd.num_blocks, dense, device="cuda")
    args = (d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(), d.ctx_lens.cuda(), lay)
    s2gpu.set_wait_timeout_ns(0)
    try:
        s2gpu.decode(*args, scale=wd.scale, num_splits=1)
        rc, flags = s2gpu.device_status(reset=True)
    finally:
        s2gpu.set_wait_timeout_ns(500_000_000)
    assert rc == S2_ERR_TIMEOUT and flags & 1
    out = s2gpu.decode(*args, scale=wd.scale, num_splits=1)
    ref, _ = oracle.decode(d.q, d.k_cache, d.v_cache, d.block_table.numpy(), d.ctx_lens.numpy(),
                           wd.block, wd.stride, wd.local, wd.scale, dense)
    parity(out.reshape(-1, wd.head_dim), ref)


@pytest.mark.parametrize("corrupt", ["future_block", "huge_block", "negative_block", "bad_row_ptr"])
def test_malformed_prefill_layout_is_flagged_not_faulted(s2gpu, corrupt):
    w, q, k, v, lay = tiny()
    row_ptr, col_idx = lay.row_ptr.copy(), lay.col_idx.copy()
    if corrupt == "future_block":
        col_idx[row_ptr[2]] = 7  # head 0, query block 2 lists key block 7 > 2
    elif corrupt == "huge_block":
        col_idx[5] = 1 << 20
    elif corrupt == "negative_block":
        col_idx[3] = -4
    else:
        row_ptr[4] = row_ptr[5] + 3  # offsets out of order
    bad = s2attn.Layout(lay.heads, lay.block_size, lay.stride, lay.local, lay.num_blocks, (),
                        row_ptr, col_idx).to("cuda")
    out = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), bad, scale=w.scale)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == S2_ERR_DEVICE_INDEX and flags == 2
    assert torch.isfinite(out.float()).all()
    # the library still works with the good layout
    good = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale)
    torch.cuda.synchronize()
    ref, _ = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale)
    parity(good.reshape(-1, w.head_dim), ref)


def test_bad_context_length_is_flagged(s2gpu):
    wd = synth.DecodeWorkload("t", 3, 4, 128, 1, 512, 16, 128, 4, 1, seed=2)
    d = synth.decode_inputs(wd, ctx_lens=[10, 200, 512])
    lay = s2gpu.build_layout(wd.heads, wd.block, wd.stride, wd.local, wd.num_blocks, device="cuda")
    cl = d.ctx_lens.clone()
    cl[1] = 100000  # beyond the block table and the layout
    out = s2gpu.decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(), cl.cuda(),
                       lay, scale=wd.scale, num_splits=1)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == S2_ERR_DEVICE_INDEX and flags == 2
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("bk", [128, 64])
def test_backward_wait_timeout_is_reported_and_recoverable(s2gpu, bk):
    w = synth.PrefillWorkload("t", 1, 4, 128, 2048, bk, 1, 1, seed=31)  # dense: long lists
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    lay = s2gpu.build_layout(4, bk, 1, 1, 2048 // bk, device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    do = torch.randn_like(q, dtype=torch.float32).to(torch.bfloat16)
    s2gpu.set_wait_timeout_ns(0)
    try:
        s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
        rc, flags = s2gpu.device_status(reset=True)
    finally:
        s2gpu.set_wait_timeout_ns(500_000_000)
    assert rc == S2_ERR_TIMEOUT and flags & 1
    a = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    b = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and torch.isfinite(x.float()).all()


def test_chunk_wait_timeout_is_reported_and_recoverable(s2gpu):
    wd = synth.DecodeWorkload("t", 2, 4, 128, 1, 4096, 16, 128, 1, 1, dense_heads=(0, 1, 2, 3), seed=32)
    ctx = [4000, 4096]
    d = synth.decode_inputs(wd, ctx_lens=ctx)
    lay = s2gpu.build_layout(4, 128, 1, 1, wd.num_blocks, (0, 1, 2, 3), device="cuda")
    q = torch.randn(600, 4, 128).to(torch.bfloat16)
    q_start = torch.tensor([0, 300, 600], dtype=torch.int32)
    args = (q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(), d.ctx_lens.cuda(),
            q_start.cuda(), lay, 300)
    s2gpu.set_wait_timeout_ns(0)
    try:
        s2gpu.chunk_prefill(*args, scale=wd.scale)
        rc, flags = s2gpu.device_status(reset=True)
    finally:
        s2gpu.set_wait_timeout_ns(500_000_000)
    assert rc == S2_ERR_TIMEOUT and flags & 1
    out = s2gpu.chunk_prefill(*args, scale=wd.scale)
    ref, _ = oracle.chunk(q, d.k_cache, d.v_cache, d.block_table.cpu().numpy(), ctx, q_start.numpy(),
                          128, wd.scale, S=1, L=1, dense_heads=(0, 1, 2, 3))
    parity(out.reshape(-1, 128), ref.reshape(-1, 128))


@pytest.mark.parametrize("bk", [128, 64])
def test_malformed_transposed_layout_is_flagged_not_faulted(s2gpu, bk):
    w = synth.PrefillWorkload("t", 1, 2, 128, 512, bk, 2, 1, seed=33)
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    lay = s2gpu.build_layout(2, bk, 2, 1, 512 // bk, device="cuda").transposed("cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    lay.d_t_row_idx[1] = 1 << 20  # a query block far outside the layout
    s2gpu.backward(q, k, v, o, lse, torch.ones_like(q), lay, scale=w.scale)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == S2_ERR_DEVICE_INDEX and flags == 2


def tiny128():
    # 128-key blocks: the prefill runs one 128-row tile per item (split kernel)
    w = synth.PrefillWorkload("t128", 1, 4, 128, 640, 128, 2, 1, seed=12)
    q, k, v = synth.prefill_inputs(w)
    lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, device="cuda")
    return w, q, k, v, lay


def test_prefill_128_key_wait_timeout_is_reported_and_recoverable(s2gpu):
    w, q, k, v, lay = tiny128()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    s2gpu.set_wait_timeout_ns(0)
    try:
        s2gpu.prefill(qc, kc, vc, lay, scale=w.scale)
        rc, flags = s2gpu.device_status(reset=True)
    finally:
        s2gpu.set_wait_timeout_ns(500_000_000)
    assert rc == S2_ERR_TIMEOUT and flags & 1
    out, lse = s2gpu.prefill(qc, kc, vc, lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale)
    parity(out.reshape(-1, w.head_dim), ref)
    parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)


@pytest.mark.parametrize("corrupt", ["future_block", "huge_block", "negative_block", "row_past_nnz"])
def test_malformed_128_key_layout_is_flagged_not_faulted(s2gpu, corrupt):
    w, q, k, v, lay = tiny128()
    row_ptr, col_idx = lay.row_ptr.copy(), lay.col_idx.copy()
    nb = w.num_blocks
    if corrupt == "future_block":
        col_idx[row_ptr[2]] = 4  # head 0, query block 2 lists key block 4 > 2
    elif corrupt == "huge_block":
        col_idx[5] = 1 << 20
    elif corrupt == "negative_block":
        col_idx[3] = -4
    else:
        row_ptr[(nb + 1) + 3] = col_idx.size + 7  # head 1, block 3 ends past the lists
    bad = s2attn.Layout(lay.heads, lay.block_size, lay.stride, lay.local, lay.num_blocks, (),
                        row_ptr, col_idx).to("cuda")
    out = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), bad, scale=w.scale)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == S2_ERR_DEVICE_INDEX and flags == 2
    assert torch.isfinite(out.float()).all()
    good = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale)
    torch.cuda.synchronize()
    ref, _ = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale)
    parity(good.reshape(-1, w.head_dim), ref)
