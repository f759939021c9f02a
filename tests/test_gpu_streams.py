"""Persistent kernels launched concurrently on several streams.

Every prefill, chunked prefill and backward launch takes its work items from a
counter slot it owns from start to end; slots are handed out in turn from a
ring of 1024. These tests overlap launches on four streams, including more
launches than there are slots (so slots come round again while launches on
other streams may still hold theirs), and check every result against the
fp64 oracle and that no wait ran out.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu


def _prefill_case(s2, w):
    q, k, v = synth.prefill_inputs(w)
    lay = s2.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, w.dense_heads,
                          device="cuda")
    ref, _ = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale, w.dense_heads)
    return dict(w=w, q=q.cuda(), k=k.cuda(), v=v.cuda(), lay=lay, ref=ref)


def test_four_streams_of_prefills_past_the_slot_ring(s2gpu):
    cases = [_prefill_case(s2gpu, w) for w in (
        synth.TINY,
        synth.PrefillWorkload("a", 2, 3, 128, 9 * 64, 64, 3, 2, dense_heads=(1,), seed=41),
        synth.PrefillWorkload("b", 1, 4, 128, 5 * 128, 128, 4, 1, seed=42),
        synth.PrefillWorkload("c", 2, 2, 64, 7 * 128, 128, 2, 2, seed=43))]
    streams = [torch.cuda.Stream() for _ in cases]
    outs = [[torch.empty_like(c["q"]) for _ in range(2)] for c in cases]
    torch.cuda.synchronize()
    n = 1100  # per stream (> 1024 slots in all)
    for it in range(n):
        for i, c in enumerate(cases):
            with torch.cuda.stream(streams[i]):
                s2gpu.prefill(c["q"], c["k"], c["v"], c["lay"], scale=c["w"].scale,
                              out=outs[i][it & 1])
    torch.cuda.synchronize()
    for i, c in enumerate(cases):
        for o in outs[i]:
            parity(o.reshape(-1, c["w"].head_dim), c["ref"])


def test_prefill_chunk_and_backward_overlapping_on_three_streams(s2gpu):
    # a 64-key prefill with its backward (persistent dQ and dK/dV kernels) on
    # one stream, a 128-key prefill on a second, a chunked prefill on a third
    w = synth.PrefillWorkload("t", 2, 3, 128, 9 * 64, 64, 3, 2, dense_heads=(1,), seed=44)
    q, k, v = synth.prefill_inputs(w)
    g = torch.Generator().manual_seed(3)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    lay = s2gpu.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, w.dense_heads,
                             device="cuda")
    w2 = synth.PrefillWorkload("u", 1, 4, 128, 6 * 128, 128, 3, 1, seed=45)
    p2 = _prefill_case(s2gpu, w2)
    wd = synth.DecodeWorkload("c", 3, 4, 128, 1, 1500, 16, 128, 4, 2, seed=46)
    d = synth.decode_inputs(wd, ctx_lens=[1500, 700, 129])
    lay_d = s2gpu.build_layout(wd.heads, wd.block, wd.stride, wd.local, wd.num_blocks, device="cuda")
    qlen = [300, 200, 129]
    q_start = torch.tensor(np.concatenate([[0], np.cumsum(qlen)]), dtype=torch.int32)
    cq = torch.randn((sum(qlen), wd.heads, wd.head_dim), generator=g).to(torch.bfloat16)
    ctx = torch.tensor([1500, 700, 129], dtype=torch.int32)

    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    dev = dict(kc=d.k_cache.cuda(), vc=d.v_cache.cuda(), bt=d.block_table.cuda(), ctx=ctx.cuda(),
               qs=q_start.cuda(), cq=cq.cuda())
    s = [torch.cuda.Stream() for _ in range(3)]
    torch.cuda.synchronize()
    for _ in range(40):
        with torch.cuda.stream(s[0]):
            o, lse = s2gpu.prefill(qc, kc, vc, lay, scale=w.scale, want_lse=True)
            grads = s2gpu.backward(qc, kc, vc, o, lse, doc, lay, scale=w.scale)
        with torch.cuda.stream(s[1]):
            o2 = s2gpu.prefill(p2["q"], p2["k"], p2["v"], p2["lay"], scale=w2.scale)
        with torch.cuda.stream(s[2]):
            co = s2gpu.chunk_prefill(dev["cq"], dev["kc"], dev["vc"], dev["bt"], dev["ctx"], dev["qs"],
                                     lay_d, max(qlen), scale=wd.scale)
    torch.cuda.synchronize()
    ref_o, _ = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale, w.dense_heads)
    parity(o.reshape(-1, w.head_dim), ref_o)
    parity(o2.reshape(-1, w2.head_dim), p2["ref"])
    ref_g = oracle.backward(q, k, v, do, w.block, w.scale, S=w.stride, L=w.local,
                            dense_heads=w.dense_heads)
    for got, want in zip(grads, ref_g):
        err = np.abs(got.double().cpu().numpy() - want)
        assert err.max() <= 2e-2 * max(1.0, np.abs(want).max())
        assert err.mean() <= 2e-3 * max(1.0, np.abs(want).mean())
    ref_c, _ = oracle.chunk(cq, d.k_cache, d.v_cache, d.block_table.numpy(), ctx.numpy(),
                            q_start.numpy(), wd.block, wd.scale, S=wd.stride, L=wd.local)
    parity(co.reshape(ref_c.shape), ref_c)
