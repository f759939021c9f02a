"""The longest work-item lists: 2046 key blocks per sequence.

The prefill, backward and chunked-prefill kernels stage each work item's
compacted key-block list (the union of its query blocks' rows, or for the
dK/dV kernel the transposed list of a key tile) in shared memory, so a layout
may have at most 2046 blocks. These tests run every kernel at exactly 2046
blocks, with a ragged last block:
  * a dense head, whose last query tiles list every key block (the longest
    prefill, dQ and chunk lists), and
  * a strided head, whose earliest strided key block is listed by every later
    query block (the longest transposed dK/dV list),
and compare sampled rows with the fp64 oracle. 2047 blocks must be refused
before anything runs, with every output buffer left as it was. All buffers
handed to the library are real device allocations of the full size, so a
missing check could not make a kernel touch memory outside them.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import s2attn, synth
from test_gpu_backward import grad_parity
from test_gpu_chunk import case as chunk_case

pytestmark = pytest.mark.gpu

NB_MAX = 2046
UNSUPPORTED = 2  # S2_ERR_UNSUPPORTED
S_CAP, L_CAP = 16, 2


def _cap_workload(bk, nb=NB_MAX, seed=61):
    # head 0 dense, head 1 strided; the last block holds bk - 5 tokens
    return synth.PrefillWorkload("capacity", 1, 2, 128, nb * bk - 5, bk, S_CAP, L_CAP,
                                 dense_heads=(0,), seed=seed)


def _first_strided_block(w, h):
    """The smallest key block that head h lists for every query block past
    its local window (oracle rule)."""
    nb = w.num_blocks
    for j in range(nb):
        if all(oracle.block_active(h, i, j, w.stride, w.local) for i in range(j + w.local, nb)):
            return j
    raise AssertionError("no strided block")


def _rows_in_blocks(rng, w, blocks, per_block):
    rows = set()
    for i in blocks:
        lo, hi = i * w.block, min((i + 1) * w.block, w.seq)
        rows |= {lo, hi - 1} | set(int(x) for x in lo + rng.choice(hi - lo, per_block - 2, replace=False))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("bk", [64, 128])
def test_prefill_at_the_list_capacity(s2gpu, bk):
    w = _cap_workload(bk)
    assert w.num_blocks == NB_MAX
    q, k, v = synth.prefill_inputs(w, device="cuda")
    lay = s2gpu.build_layout(w.heads, bk, w.stride, w.local, NB_MAX, w.dense_heads, device="cuda")
    out, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = []
    for h in range(w.heads):
        blocks = {0, NB_MAX // 2, NB_MAX - 2, NB_MAX - 1} | set(int(x) for x in rng.choice(NB_MAX, 2))
        rows += [h * w.seq + t for t in _rows_in_blocks(rng, w, sorted(blocks), 6)]
    rows = np.array(rows, dtype=np.int64)
    ref, ref_lse = oracle.prefill(q.cpu(), k.cpu(), v.cpu(), bk, w.stride, w.local, w.scale,
                                  w.dense_heads, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    parity(out.reshape(-1, w.head_dim)[idx], ref)
    parity(lse.reshape(-1)[idx], ref_lse, max_tol=1e-3, mean_tol=1e-4)
    assert torch.isfinite(out).all()


def test_backward_at_the_list_capacity(s2gpu):
    # 64-key blocks: the persistent dQ kernel (union lists paired into 128-key
    # elements) and the persistent dK/dV kernel (transposed lists)
    w = _cap_workload(64, seed=62)
    q, k, v = synth.prefill_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(78)
    do = torch.randn(q.shape, generator=gen, device="cuda").to(torch.bfloat16)
    lay = s2gpu.build_layout(w.heads, w.block, w.stride, w.local, NB_MAX, w.dense_heads,
                             device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    dq, dk, dv = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    torch.cuda.synchronize()
    qh, kh, vh, doh = (t.cpu() for t in (q, k, v, do))
    rng = np.random.default_rng(9)
    # dense head 0: dQ rows of the last query blocks (their lists hold every
    # key block); key rows near the end keep the oracle's cost small
    tail = [NB_MAX - 3, NB_MAX - 2, NB_MAX - 1]
    qr = _rows_in_blocks(rng, w, tail, 8)
    kr = _rows_in_blocks(rng, w, tail, 8)
    # strided head 1: key rows of its first strided block (listed by every
    # later query block) and of the last blocks
    j0 = _first_strided_block(w, 1)
    kr1 = _rows_in_blocks(rng, w, [j0] + tail, 6)
    qr1 = _rows_in_blocks(rng, w, [j0 + 1, NB_MAX // 2] + tail, 6)
    for h, qrows, krows in ((0, qr, kr), (1, qr1, kr1)):
        rq, rk, rv = oracle.backward_sampled(qh, kh, vh, doh, w.block, w.scale, [h], qrows, krows,
                                             S=w.stride, L=w.local, dense_heads=w.dense_heads)
        grad_parity(f"capacity dq h{h}", dq[0, h, torch.from_numpy(qrows).cuda()], rq[0])
        grad_parity(f"capacity dk h{h}", dk[0, h, torch.from_numpy(krows).cuda()], rk[0])
        grad_parity(f"capacity dv h{h}", dv[0, h, torch.from_numpy(krows).cuda()], rv[0])


def test_chunk_prefill_at_the_list_capacity(s2gpu):
    # one sequence at 2046 blocks of 64 (its last chunk's tiles list every
    # key block of the dense head) beside a short one; every row checked
    chunk_case(s2gpu, ctx=[NB_MAX * 64 - 3, 700], qlen=[256, 700], H=2, B=64, S=S_CAP, L=L_CAP,
               dense=(0,), seed=63)


def test_2047_blocks_are_refused_before_launch(s2gpu):
    bk = 64
    w = _cap_workload(bk, nb=NB_MAX + 1, seed=64)
    assert w.num_blocks == NB_MAX + 1
    q, k, v = synth.prefill_inputs(w, device="cuda")
    lay = s2gpu.build_layout(w.heads, bk, w.stride, w.local, NB_MAX + 1, w.dense_heads,
                             device="cuda")
    sentinel = float("nan")
    out = torch.full_like(q, sentinel)
    lse = torch.full((1, w.heads, w.seq), sentinel, dtype=torch.float32, device="cuda")
    with pytest.raises(s2attn.S2Error) as e:
        s2gpu.prefill(q, k, v, lay, scale=w.scale, out=out, lse=lse)
    assert e.value.status == UNSUPPORTED
    # backward: real o, lse and dO of the full size (the forward output slots
    # are stand-ins; nothing may be read or written)
    o = q.clone()
    lse_in = torch.zeros((1, w.heads, w.seq), dtype=torch.float32, device="cuda")
    with pytest.raises(s2attn.S2Error) as e:
        s2gpu.backward(q, k, v, o, lse_in, q, lay, scale=w.scale)
    assert e.value.status == UNSUPPORTED
    # chunked prefill over a zero-filled paged cache of the same length
    ctx = [w.seq]
    pages = -(-w.seq // 16)
    kc = torch.zeros((pages, w.heads, 16, w.head_dim), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    bt = torch.arange(pages, dtype=torch.int32, device="cuda").reshape(1, pages)
    cq = q[0, :, -100:].transpose(0, 1).contiguous()
    cout = torch.full_like(cq, sentinel)
    with pytest.raises(s2attn.S2Error) as e:
        s2gpu.chunk_prefill(cq, kc, vc, bt, torch.tensor(ctx, dtype=torch.int32, device="cuda"),
                            torch.tensor([0, 100], dtype=torch.int32, device="cuda"), lay, 100,
                            scale=w.scale, out=cout)
    assert e.value.status == UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all() and torch.isnan(cout).all()
