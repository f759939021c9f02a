"""Partial last blocks (seq not a multiple of the block size) and grouped K/V
heads (GQA/MQA) on the GPU, against the fp64 oracle.

A partial last block is read through a 3-D tensor map whose rows past seq
come back as zeros; its missing keys lie past every valid query, so causality
hides them, and rows past seq are never written. Grouped heads read K/V head
h / (heads / heads_kv) with the layout applied per query head.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu


def guarded_out(shape, dtype=torch.bfloat16):
    """An output tensor followed by a sentinel tail that must stay untouched."""
    n = int(np.prod(shape))
    buf = torch.full((n + 4096,), 7.0, dtype=dtype, device="cuda")
    return buf, buf[:n].view(shape)


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("bk", [64, 128])
@pytest.mark.parametrize("seq", [1, 63, 130, 777])
def test_ragged_sequence_all_rows(s2gpu, hd, bk, seq):
    nb = -(-seq // bk)
    w = synth.PrefillWorkload("t", 2, 3, hd, seq, bk, 2, 1, dense_heads=(1,), seed=80)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout(3, bk, 2, 1, nb, (1,), device="cuda")
    buf, out = guarded_out(q.shape)
    lbuf, lse = guarded_out((2, 3, seq), torch.float32)
    s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale, out=out, lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(q, k, v, bk, 2, 1, w.scale, (1,))
    parity(out.reshape(-1, hd), ref)
    parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)
    assert (buf[out.numel():] == 7.0).all() and (lbuf[lse.numel():] == 7.0).all()


def test_ragged_long_sequence_sampled_rows(s2gpu):
    w = synth.PrefillWorkload("t", 1, 8, 128, 20000, 128, 16, 4, dense_heads=(0,), seed=81)
    q, k, v = synth.prefill_inputs(w)
    nb = -(-w.seq // w.block)
    lay = s2gpu.build_layout(8, 128, 16, 4, nb, (0,), device="cuda")
    out, lse = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = [h * w.seq + int(p) for h in range(8)
            for p in [0, 127, 128, w.seq - 33, w.seq - 1] + rng.integers(0, w.seq, 5).tolist()]
    ref, ref_lse = oracle.prefill(q, k, v, 128, 16, 4, w.scale, (0,), rows=rows)
    parity(out.reshape(-1, 128)[torch.as_tensor(rows)].cpu(), ref)
    parity(lse.reshape(-1)[torch.as_tensor(rows)].cpu(), ref_lse, max_tol=1e-3, mean_tol=1e-4)


@pytest.mark.parametrize("hkv", [1, 2, 4])
@pytest.mark.parametrize("bk,seq", [(64, 9 * 64), (128, 700)])
def test_grouped_kv_heads_prefill(s2gpu, hkv, bk, seq):
    H, hd = 8, 128
    w = synth.PrefillWorkload("t", 2, H, hd, seq, bk, 4, 1, seed=82)
    q, k, v = synth.prefill_inputs(w)
    k, v = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()
    nb = -(-seq // bk)
    lay = s2gpu.build_layout(H, bk, 4, 1, nb, device="cuda")
    out, lse = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill_mask(q, k, v, bk, oracle.block_mask(H, nb, 4, 1), w.scale)
    parity(out.reshape(-1, hd), ref)
    parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)


@pytest.mark.parametrize("hkv", [1, 4])
@pytest.mark.parametrize("splits", [1, 5])
def test_grouped_kv_heads_decode(s2gpu, hkv, splits):
    H = 8
    w = synth.DecodeWorkload("t", 5, H, 128, 1, 3000, 16, 128, 4, 2, seed=83)
    d = synth.decode_inputs(w, ctx_lens=[1, 130, 1000, 2222, 3000])
    kc, vc = d.k_cache[:, :hkv].contiguous(), d.v_cache[:, :hkv].contiguous()
    lay = s2gpu.build_layout(H, 128, 4, 2, w.num_blocks, device="cuda")
    out, lse = s2gpu.decode(d.q.cuda(), kc.cuda(), vc.cuda(), d.block_table.cuda(),
                            d.ctx_lens.cuda(), lay, scale=w.scale, num_splits=splits,
                            want_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_mask(d.q, kc, vc, d.block_table.cpu().numpy(),
                                      d.ctx_lens.cpu().numpy(), 128,
                                      oracle.block_mask(H, w.num_blocks, 4, 2), w.scale)
    parity(out.reshape(-1, 128), ref)
    parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)
