"""Decode parity: the split-KV kernel + combine (through the C ABI) against the
fp64 oracle, on small paged caches (every item, several split counts, ragged
contexts) and on the full-size paged workload (sampled sequences)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu


def layout_for(s2, w, device="cuda"):
    nb = -(-int(w.ctx_max) // w.block)
    return s2.build_layout(w.heads, w.block, w.stride, w.local, nb, w.dense_heads, device=device)


def small(hd=128, dense=(), ctx=None, seed=9):
    w = synth.DecodeWorkload("t", 6, 8, hd, 1, 3000, 16, 128, 4, 2, dense_heads=dense, seed=seed)
    if ctx is None:
        ctx = [1, 16, 17, 128, 129, 3000]
    return w, synth.decode_inputs(w, ctx_lens=ctx)


def run(s2, w, d, splits, lay=None):
    lay = lay or layout_for(s2, w)
    out, lse = s2.decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(),
                         d.ctx_lens.cuda(), lay, scale=w.scale, num_splits=splits, want_lse=True)
    torch.cuda.synchronize()
    return out, lse


def oracle_decode(w, d, items=None):
    return oracle.decode(d.q, d.k_cache, d.v_cache, d.block_table.cpu().numpy(),
                         d.ctx_lens.cpu().numpy(), w.block, w.stride, w.local, w.scale,
                         w.dense_heads, items=items)


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("splits", [1, 2, 3, 7, 0])
def test_small_paged_cache_all_items(s2gpu, hd, splits):
    w, d = small(hd)
    out, lse = run(s2gpu, w, d, splits)
    ref, ref_lse = oracle_decode(w, d)
    parity(out.reshape(-1, hd), ref)
    parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)


def test_dense_head_and_many_splits(s2gpu):
    w, d = small(dense=(0, 5), ctx=[2500, 700, 1, 33, 2048, 1999], seed=13)
    for splits in (1, 16, 64):
        out, _ = run(s2gpu, w, d, splits)
        ref, _ = oracle_decode(w, d)
        parity(out.reshape(-1, 128), ref)


@pytest.mark.parametrize("S,L", [(4, 1000), (1000, 1), (1000, 3)])
def test_degenerate_strides_and_windows(s2gpu, S, L):
    # a window past the block count (dense causal) and a stride past it
    # (the local window plus at most one strided block per head)
    w = synth.DecodeWorkload("t", 6, 8, 128, 1, 3000, 16, 128, S, L, seed=14)
    d = synth.decode_inputs(w, ctx_lens=[1, 16, 17, 128, 129, 3000])
    for splits in (1, 3):
        out, lse = run(s2gpu, w, d, splits)
        ref, ref_lse = oracle_decode(w, d)
        parity(out.reshape(-1, 128), ref)
        parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)


@pytest.mark.parametrize("batch", [40, 300])
def test_equal_contexts_and_batches_past_the_reordering(s2gpu, batch):
    # Up to 256 sequences start in order of decreasing context length (ties by
    # index): groups of equal lengths must still map one CTA slice to each
    # sequence. Past 256 the index order is kept. Every item is checked.
    rng = np.random.default_rng(batch)
    ctx = [int(c) for c in rng.choice([1, 17, 300, 1000], size=batch)]
    w = synth.DecodeWorkload("t", batch, 4, 128, 1, 1000, 16, 128, 4, 2, seed=batch)
    d = synth.decode_inputs(w, ctx_lens=ctx)
    for splits in (1, 3):
        out, lse = run(s2gpu, w, d, splits)
        ref, ref_lse = oracle_decode(w, d)
        parity(out.reshape(-1, 128), ref)
        parity(lse.reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)


def test_decode_equals_last_prefill_row(s2gpu):
    # Dense-packed prefill of n tokens vs paged decode of the same tokens.
    H, D, B, S, L, n = 4, 128, 128, 4, 2, 1024
    wp = synth.PrefillWorkload("t", 1, H, D, n, B, S, L, seed=17)
    q, k, v = synth.prefill_inputs(wp)
    lay = s2gpu.build_layout(H, B, S, L, n // B, device="cuda")
    pre = s2gpu.prefill(q.cuda(), k.cuda(), v.cuda(), lay, scale=wp.scale)
    pages = n // 16
    perm = torch.from_numpy(np.random.default_rng(1).permutation(pages).astype(np.int32))
    kc = torch.empty(pages, H, 16, D, dtype=torch.bfloat16)
    vc = torch.empty_like(kc)
    kc[perm.long()] = k[0].reshape(H, pages, 16, D).transpose(0, 1)
    vc[perm.long()] = v[0].reshape(H, pages, 16, D).transpose(0, 1)
    d = synth.DecodeInputs(q[0, :, n - 1].unsqueeze(0).contiguous(), kc, vc, perm.view(1, -1),
                           torch.tensor([n], dtype=torch.int32))
    w = synth.DecodeWorkload("t", 1, H, D, n, n, 16, B, S, L)
    for splits in (1, 4):
        out, _ = run(s2gpu, w, d, splits, lay)
        assert (out[0].float() - pre[0, :, n - 1].float()).abs().max().item() < 1e-2


def test_full_size_paged_workload_sampled_sequences(s2gpu):
    w = synth.DECODE_PAGED
    d = synth.decode_inputs(w, device="cuda")
    lay = layout_for(s2gpu, w)
    splits = s2gpu.decode_auto_splits(w.batch, w.heads)
    out, lse = s2gpu.decode(d.q, d.k_cache, d.v_cache, d.block_table, d.ctx_lens, lay,
                            scale=w.scale, num_splits=splits, want_lse=True)
    torch.cuda.synchronize()
    # Oracle on 8 sampled sequences: gather their pages into a compact host cache.
    rng = np.random.default_rng(40)
    seqs = sorted(int(s) for s in rng.choice(w.batch, 8, replace=False))
    bt = d.block_table.cpu()
    cl = d.ctx_lens.cpu()
    used = [bt[s, : -(-int(cl[s]) // 16)] for s in seqs]
    flat = torch.cat(used).long()
    kc = d.k_cache[flat.cuda()].cpu()
    vc = d.v_cache[flat.cuda()].cpu()
    new_bt = torch.full((len(seqs), bt.shape[1]), -1, dtype=torch.int32)
    off = 0
    for r, u in enumerate(used):
        new_bt[r, : len(u)] = torch.arange(off, off + len(u), dtype=torch.int32)
        off += len(u)
    sub = synth.DecodeInputs(d.q[seqs].cpu(), kc, vc, new_bt, cl[seqs])
    ref, ref_lse = oracle_decode(w, sub)
    parity(out[seqs].reshape(-1, w.head_dim), ref)
    parity(lse[seqs].reshape(-1), ref_lse, max_tol=1e-3, mean_tol=1e-4)
    assert torch.isfinite(out).all()
    # split count does not change the result beyond rounding
    out1 = s2gpu.decode(d.q, d.k_cache, d.v_cache, d.block_table, d.ctx_lens, lay, scale=w.scale,
                        num_splits=1)
    assert (out1.float() - out.float()).abs().max().item() < 1e-2


def test_bad_page_ids_are_flagged_not_faulted(s2gpu):
    w, d = small()
    bt = d.block_table.clone()
    bt[3, 2] = 10 ** 7  # inside sequence 3's context (129 tokens = 9 pages)
    bt[4, 0] = -5
    lay = layout_for(s2gpu, w)
    s2gpu.decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), bt.cuda(), d.ctx_lens.cuda(), lay,
                 scale=w.scale, num_splits=2)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == 6 and flags == 2  # S2_ERR_DEVICE_INDEX
