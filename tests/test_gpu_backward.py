"""Backward parity: dQ, dK, dV from the sm_100a kernels (through the C ABI)
against the fp64 oracle's gradients of the same masked attention.

Tolerance. The kernels round P and dS to bf16 as MMA operands (relative
error up to 2^-9 each), accumulate in fp32 and round the gradients to bf16
once; gradient entries reach a few units on these unit-normal inputs, so the
bar is relative to the reference's scale: max-abs <= 2e-2 * max(1, max|ref|)
and mean-abs <= 2e-3 * max(1, mean|ref|).
"""
import numpy as np
import pytest
import torch

import oracle
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu


def grad_parity(name, got, ref):
    got = got.detach().double().cpu().numpy().reshape(ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite"
    err = np.abs(got - ref)
    mx_ref, mean_ref = float(np.abs(ref).max()), float(np.abs(ref).mean())
    mx, mean = float(err.max()), float(err.mean())
    print(f"{name}: max-abs {mx:.3e} (ref max {mx_ref:.3f}) mean-abs {mean:.3e} (ref mean {mean_ref:.3f})")
    assert mx <= 2e-2 * max(1.0, mx_ref), f"{name}: max-abs {mx:.3e}"
    assert mean <= 2e-3 * max(1.0, mean_ref), f"{name}: mean-abs {mean:.3e}"


def run_backward(s2, w, lay, q, k, v, do, bmask=None):
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    o, lse = s2.prefill(qc, kc, vc, lay, scale=w.scale, want_lse=True)
    dq, dk, dv = s2.backward(qc, kc, vc, o, lse, doc, lay, scale=w.scale)
    torch.cuda.synchronize()
    if bmask is None:
        ref = oracle.backward(q, k, v, do, w.block, w.scale, S=w.stride, L=w.local,
                              dense_heads=w.dense_heads)
    else:
        ref = oracle.backward(q, k, v, do, w.block, w.scale, bmask=bmask)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        grad_parity(name, g, r)
    return dq, dk, dv


def upstream(w, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((w.batch, w.heads, w.seq, w.head_dim), generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("bk", [64, 128])
@pytest.mark.parametrize("S,L,dense", [(4, 1, ()), (3, 2, (1,))])
def test_small_shapes_all_gradients(s2gpu, hd, bk, S, L, dense):
    seq = 9 * 64 if bk == 64 else 5 * 128
    w = synth.PrefillWorkload("t", 2, 3, hd, seq, bk, S, L, dense_heads=dense, seed=90)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout(3, bk, S, L, w.seq // bk, dense, device="cuda")
    run_backward(s2gpu, w, lay, q, k, v, upstream(w, 1))


@pytest.mark.parametrize("bk", [64, 128])
@pytest.mark.parametrize("seq", [1, 100, 333])
def test_ragged_lengths(s2gpu, bk, seq):
    w = synth.PrefillWorkload("t", 1, 2, 128, seq, bk, 2, 1, seed=91)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout(2, bk, 2, 1, -(-seq // bk), device="cuda")
    run_backward(s2gpu, w, lay, q, k, v, upstream(w, 2))


@pytest.mark.parametrize("bk", [64, 128])
def test_mask_layout_with_empty_rows(s2gpu, bk):
    nb, H = 8, 3
    rng = np.random.default_rng(7)
    m = np.tril(rng.random((H, nb, nb)) < 0.4).astype(np.uint8)
    m[0, 2] = 0      # an empty query block
    m[1, :, 3] = 0   # a key block nobody lists
    m[2, :4] = 0     # whole tiles with no key
    w = synth.PrefillWorkload("t", 1, H, 128, nb * bk, bk, 1, 1, seed=92)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout_mask(m, bk, device="cuda")
    dq, dk, dv = run_backward(s2gpu, w, lay, q, k, v, upstream(w, 3), bmask=m)
    assert (dk[0, 1, 3 * bk:4 * bk] == 0).all() and (dv[0, 1, 3 * bk:4 * bk] == 0).all()


@pytest.mark.parametrize("bk", [64, 128])
def test_gradients_only_16_byte_aligned(s2gpu, bk):
    # The epilogues store whole 32-byte sectors when a gradient array is
    # 32-byte aligned and fall back to 16-byte stores otherwise: both write the
    # same bytes, and nothing outside the arrays.
    w = synth.PrefillWorkload("t", 1, 3, 128, 5 * 128, bk, 3, 1, seed=96)
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    do = upstream(w, 4).cuda()
    lay = s2gpu.build_layout(w.heads, bk, w.stride, w.local, w.num_blocks, device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    ref = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    n = q.numel()
    bufs, outs = [], []
    for _ in range(3):
        buf = torch.full((n + 24,), float("nan"), dtype=torch.bfloat16, device="cuda")
        off = next(e for e in range(0, 24, 8) if (buf.data_ptr() + 2 * e) % 32 == 16)
        bufs.append((buf, off))
        outs.append(buf[off:off + n].view(q.shape))
    s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale, dq=outs[0], dk=outs[1], dv=outs[2])
    torch.cuda.synchronize()
    for got, want, (buf, off) in zip(outs, ref, bufs):
        assert torch.equal(got, want)
        assert torch.isnan(buf[:off].float()).all() and torch.isnan(buf[off + n:].float()).all()


def test_odd_union_lists_and_empty_key_tiles(s2gpu):
    """64-key blocks: query tiles (two query blocks) whose union list has an
    odd length (the dQ kernel pairs entries into 128-key elements, so the last
    pair is a masked pad) and key tiles that no query lists (the persistent
    dK/dV kernel must write zeros for them)."""
    nb, H, bk = 10, 2, 64
    m = np.zeros((H, nb, nb), dtype=np.uint8)
    for t in range(nb // 2):
        m[0, 2 * t, 0] = 1            # head 0: unions {0, 1}, then {0, 2t, 2t+1} (odd)
        m[0, 2 * t, 2 * t] = 1
        m[0, 2 * t + 1, 2 * t + 1] = 1
        m[1, 2 * t + 1, 2 * t + 1] = 1  # head 1: union {2t+1} (one entry); even blocks unlisted
    w = synth.PrefillWorkload("t", 2, H, 128, nb * bk, bk, 1, 1, seed=95)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout_mask(m, bk, device="cuda")
    dq, dk, dv = run_backward(s2gpu, w, lay, q, k, v, upstream(w, 6), bmask=m)
    for j in range(0, nb, 2):  # head 1's even key blocks: no query lists them
        assert (dk[:, 1, j * bk:(j + 1) * bk] == 0).all() and (dv[:, 1, j * bk:(j + 1) * bk] == 0).all()
    # head 1's even query blocks list no key: zero dQ
    for i in range(0, nb, 2):
        assert (dq[:, 1, i * bk:(i + 1) * bk] == 0).all()


def test_stride_one_matches_autograd_of_causal_sdpa(s2gpu):
    w = synth.PrefillWorkload("t", 1, 2, 128, 512, 128, 1, 1, seed=93)
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    do = upstream(w, 4).cuda()
    lay = s2gpu.build_layout(2, 128, 1, 1, 4, device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    dq, dk, dv = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    qf, kf, vf = (t.float().requires_grad_() for t in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qf, kf, vf, is_causal=True, scale=w.scale)
    (ref * do.float()).sum().backward()
    for g, r in ((dq, qf.grad), (dk, kf.grad), (dv, vf.grad)):
        assert (g.float() - r).abs().max().item() <= 2e-2 * max(1.0, r.abs().max().item())


@pytest.mark.parametrize("bk,batch,seq", [(64, 8, 2048), (128, 4, 4096)])
def test_many_items_per_cta(s2gpu, bk, batch, seq):
    # 1024 query tiles for at most 148 persistent dQ CTAs: each CTA runs several
    # items (double-buffered lists, barrier phases carried across items)
    w = synth.PrefillWorkload("t", batch, 8, 64, seq, bk, 4, 1, seed=96)
    q, k, v = synth.prefill_inputs(w)
    lay = s2gpu.build_layout(w.heads, bk, 4, 1, w.num_blocks, device="cuda")
    run_backward(s2gpu, w, lay, q, k, v, upstream(w, 7))


def test_backward_is_deterministic(s2gpu):
    w = synth.PrefillWorkload("t", 1, 4, 128, 1024, 64, 4, 2, seed=94)
    q, k, v = (t.cuda() for t in synth.prefill_inputs(w))
    do = upstream(w, 5).cuda()
    lay = s2gpu.build_layout(4, 64, 4, 2, 16, device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    a = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    b = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("hkv", [1, 2])
@pytest.mark.parametrize("bk", [64, 128])
def test_grouped_kv_heads(s2gpu, hkv, bk):
    H, seq = 4, 9 * 64 if bk == 64 else 5 * 128
    w = synth.PrefillWorkload("t", 2, H, 128, seq, bk, 3, 1, dense_heads=(1,), seed=95)
    q, k, v = synth.prefill_inputs(w)
    k, v = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()
    do = upstream(w, 6)
    lay = s2gpu.build_layout(H, bk, 3, 1, seq // bk, (1,), device="cuda")
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    o, lse = s2gpu.prefill(qc, kc, vc, lay, scale=w.scale, want_lse=True)
    dq, dk, dv = s2gpu.backward(qc, kc, vc, o, lse, doc, lay, scale=w.scale)
    torch.cuda.synchronize()
    assert dk.shape == k.shape and dv.shape == v.shape
    ref = oracle.backward(q, k, v, do, bk, w.scale, S=3, L=1, dense_heads=(1,))
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        grad_parity(name, g, r)


def _rows(rng, lo, hi, n, block):
    """n seeded positions in [lo, hi) plus the block edges at both ends."""
    pos = {lo, hi - 1, lo + block - 1 if hi - lo > block else lo}
    pos |= set(int(x) for x in rng.integers(lo, hi, n))
    return np.array(sorted(pos), dtype=np.int64)


@pytest.mark.parametrize("name,picks", [
    # (batch, head, first sampled position): sparse heads over the whole
    # sequence; a dense head (7B hybrid) over its last blocks only, since every
    # earlier key of a dense head is seen by all later rows
    ("prefill_1p3b", [(0, 3, 0), (3, 12, 0), (2, 7, 0)]),
    ("prefill_7b_hybrid", [(0, 5, 0), (0, 30, 0), (0, 1, 32768 - 4 * 128)]),
])
def test_full_size_workload_sampled_gradients(s2gpu, name, picks):
    """dQ rows and dK/dV key rows of the full-size workloads, sampled per head,
    against the oracle's gradients of the same rows; the kernels run in the
    launch configuration of the benchmark's backward leg."""
    w = synth.PREFILL_WORKLOADS[name]
    q, k, v = synth.prefill_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(77)
    do = torch.randn(q.shape, generator=gen, device="cuda").to(torch.bfloat16)
    lay = s2gpu.build_layout(w.heads, w.block, w.stride, w.local, w.num_blocks, w.dense_heads,
                             device="cuda")
    o, lse = s2gpu.prefill(q, k, v, lay, scale=w.scale, want_lse=True)
    dq, dk, dv = s2gpu.backward(q, k, v, o, lse, do, lay, scale=w.scale)
    torch.cuda.synchronize()
    qh, kh, vh, doh = (t.cpu() for t in (q, k, v, do))
    rng = np.random.default_rng(w.seed + 300)
    for b, h, lo in picks:
        qr = _rows(rng, lo, w.seq, 24, w.block)
        kr = _rows(rng, lo, w.seq, 24, w.block)
        rq, rk, rv = oracle.backward_sampled(qh, kh, vh, doh, w.block, w.scale, [b * w.heads + h],
                                             qr, kr, S=w.stride, L=w.local,
                                             dense_heads=w.dense_heads)
        grad_parity(f"{name} dq b{b} h{h}", dq[b, h, torch.from_numpy(qr).cuda()], rq[0])
        grad_parity(f"{name} dk b{b} h{h}", dk[b, h, torch.from_numpy(kr).cuda()], rk[0])
        grad_parity(f"{name} dv b{b} h{h}", dv[b, h, torch.from_numpy(kr).cuda()], rv[0])
