"""Pins for the oracle's backward (dQ, dK, dV of masked softmax attention).

The arXiv abstract of "S2-Attention: Hardware-aware context sharding among
attention heads" reports training speedups, so the gradients of the same
masked attention are part of the method. Each pin ties the oracle to
something outside its own code: torch autograd of fp64 SDPA with an explicit
mask (a library routine), central finite differences of that fp64 forward,
closed-form sums that hold for any softmax, and the reduction of grouped K/V
heads to repeated heads.
"""
import numpy as np
import pytest
import torch

import oracle
from head_heterogeneous_block_s2_b200 import synth


def token_mask_hhst(H, seq, B, S, L, dense=()):
    nb = -(-seq // B)
    bm = oracle.block_mask(H, nb, S, L, dense).astype(bool)
    tm = np.repeat(np.repeat(bm, B, axis=1), B, axis=2)[:, :seq, :seq]
    return tm & np.tril(np.ones((seq, seq), dtype=bool))[None]


def sdpa_grads(q, k, v, do, mask, scale):
    """torch autograd of fp64 SDPA with a boolean mask (rows must see >= 1 key)."""
    qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=torch.as_tensor(mask),
                                                         scale=scale)
    (o * do.double()).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


def inputs(batch, H, D, seq, B, S, L, dense=(), seed=0):
    w = synth.PrefillWorkload("t", batch, H, D, seq, B, S, L, dense_heads=dense, seed=seed)
    q, k, v = synth.prefill_inputs(w)
    g = torch.Generator().manual_seed(seed + 1000)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return w, q, k, v, do


@pytest.mark.parametrize("B,S,L,dense,seq", [(4, 4, 1, (), 32), (8, 2, 2, (1,), 40), (4, 3, 1, (), 30),
                                             (16, 1, 1, (), 48)])
def test_backward_equals_autograd_of_fp64_sdpa(B, S, L, dense, seq):
    w, q, k, v, do = inputs(2, 3, 16, seq, B, S, L, dense, seed=B + S)
    dq, dk, dv = oracle.backward(q, k, v, do, B, w.scale, S=S, L=L, dense_heads=dense)
    mask = token_mask_hhst(3, seq, B, S, L, dense)
    rq, rk, rv = sdpa_grads(q, k, v, do, mask[None], w.scale)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - b).max() < 1e-11


def test_backward_matches_central_differences():
    """d(sum O * dO)/dX by central differences of the fp64 SDPA forward."""
    w, q, k, v, do = inputs(1, 2, 8, 12, 4, 2, 1, seed=3)
    mask = torch.as_tensor(token_mask_hhst(2, 12, 4, 2, 1))[None]
    dq, dk, dv = oracle.backward(q, k, v, do, 4, w.scale, S=2, L=1)
    base = [t.double() for t in (q, k, v)]

    def loss(ts):
        o = torch.nn.functional.scaled_dot_product_attention(*ts, attn_mask=mask, scale=w.scale)
        return float((o * do.double()).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in base[which].shape)
            plus = [t.clone() for t in base]
            minus = [t.clone() for t in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(plus) - loss(minus)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7, (which, idx, fd, grad[idx])


def test_closed_form_sums():
    """sum_k dV[k] = sum_q dO[q] (rows of P sum to 1); sum_k dK[k] = 0 (rows of dS sum to 0)."""
    w, q, k, v, do = inputs(2, 4, 32, 64, 8, 4, 2, (2,), seed=5)
    dq, dk, dv = oracle.backward(q, k, v, do, 8, w.scale, S=4, L=2, dense_heads=(2,))
    assert np.abs(dv.sum(axis=2) - do.double().numpy().sum(axis=2)).max() < 1e-10
    assert np.abs(dk.sum(axis=2)).max() < 1e-10


def test_zero_upstream_gradient_gives_zero():
    w, q, k, v, do = inputs(1, 2, 16, 24, 8, 2, 1, seed=6)
    dq, dk, dv = oracle.backward(q, k, v, torch.zeros_like(do), 8, w.scale, S=2, L=1)
    assert not dq.any() and not dk.any() and not dv.any()


def test_mask_entry_equals_rule_and_empty_rows_contribute_nothing():
    w, q, k, v, do = inputs(1, 3, 16, 40, 8, 3, 1, seed=7)
    a = oracle.backward(q, k, v, do, 8, w.scale, S=3, L=1)
    b = oracle.backward(q, k, v, do, 8, w.scale, bmask=oracle.block_mask(3, 5, 3, 1))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # empty query block 2 of head 0: its dQ is zero and removing its dO changes nothing
    m = oracle.block_mask(3, 5, 3, 1)
    m[0, 2] = 0
    dq, dk, dv = oracle.backward(q, k, v, do, 8, w.scale, bmask=m)
    assert not dq[0, 0, 16:24].any()
    do2 = do.clone()
    do2[0, 0, 16:24] = 0
    dq2, dk2, dv2 = oracle.backward(q, k, v, do2, 8, w.scale, bmask=m)
    assert np.array_equal(dk, dk2) and np.array_equal(dv, dv2)


@pytest.mark.parametrize("hkv", [1, 2])
def test_grouped_heads_sum_over_the_group(hkv):
    H = 4
    w, q, k, v, do = inputs(2, H, 16, 24, 8, 2, 1, seed=8)
    k, v = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()
    g = H // hkv
    dq, dk, dv = oracle.backward(q, k, v, do, 8, w.scale, S=2, L=1)
    rq, rk, rv = oracle.backward(q, k.repeat_interleave(g, 1), v.repeat_interleave(g, 1), do, 8,
                                 w.scale, S=2, L=1)
    assert np.abs(dq - rq).max() < 1e-12
    assert np.abs(dk - rk.reshape(2, hkv, g, 24, 16).sum(2)).max() < 1e-12
    assert np.abs(dv - rv.reshape(2, hkv, g, 24, 16).sum(2)).max() < 1e-12


def _sample(rng, grp, seq, nq, nk):
    qr = rng.choice(grp * seq, nq, replace=False)
    kr = rng.choice(seq, nk, replace=False)
    return qr, kr


@pytest.mark.parametrize("B,S,L,dense,seq,hkv,use_mask", [
    (4, 4, 1, (), 32, 3, False), (8, 2, 2, (1,), 40, 3, False), (4, 3, 1, (), 30, 1, False),
    (8, 3, 1, (), 48, 3, True)])
def test_sampled_backward_equals_autograd_rows(B, S, L, dense, seq, hkv, use_mask):
    """The sampled entry's rows against torch autograd of fp64 SDPA (grouped
    heads by repeating K/V; a random block mask with an empty row)."""
    H = 3
    w, q, k, v, do = inputs(2, H, 16, seq, B, S, L, dense, seed=B + seq)
    k, v = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()
    grp = H // hkv
    nb = -(-seq // B)
    if use_mask:
        rng = np.random.default_rng(1)
        bm = np.tril(rng.random((H, nb, nb)) < 0.5).astype(np.uint8)
        for h in range(H):
            bm[h, np.arange(nb), np.arange(nb)] = 1
        tm = np.repeat(np.repeat(bm.astype(bool), B, 1), B, 2)[:, :seq, :seq] & np.tril(
            np.ones((seq, seq), dtype=bool))[None]
        kw = dict(bmask=bm)
    else:
        tm = token_mask_hhst(H, seq, B, S, L, dense)
        kw = dict(S=S, L=L, dense_heads=dense)
    rq, rk, rv = sdpa_grads(q, k.repeat_interleave(grp, 1), v.repeat_interleave(grp, 1), do, tm[None],
                            w.scale)
    rk = rk.reshape(2, hkv, grp, seq, 16).sum(2)
    rv = rv.reshape(2, hkv, grp, seq, 16).sum(2)
    rng = np.random.default_rng(seq)
    planes = [0, 2 * hkv - 1] if hkv > 1 else [1]
    qr, kr = _sample(rng, grp, seq, 7, 6)
    kr[0] = 0  # the first key (seen by every later row that lists its block)
    dq, dk, dv = oracle.backward_sampled(q, k, v, do, B, w.scale, planes, qr, kr, **kw)
    for n, e in enumerate(planes):
        b, g = divmod(e, hkv)
        for r, row in enumerate(qr):
            hh, t = divmod(int(row), seq)
            assert np.abs(dq[n, r] - rq[b, g * grp + hh, t]).max() < 1e-11
        assert np.abs(dk[n] - rk[b, g, kr]).max() < 1e-11
        assert np.abs(dv[n] - rv[b, g, kr]).max() < 1e-11


def test_sampled_backward_equals_full_backward_rows():
    """Same numbers as the full backward's rows (one head per group: query rows
    are positions of the plane's own head)."""
    w, q, k, v, do = inputs(2, 4, 32, 64, 8, 4, 2, (2,), seed=9)
    full = oracle.backward(q, k, v, do, 8, w.scale, S=4, L=2, dense_heads=(2,))
    planes = [1, 2, 4, 7]
    qr = np.array([0, 17, 40, 63])
    kr = np.array([5, 31, 63])
    dq, dk, dv = oracle.backward_sampled(q, k, v, do, 8, w.scale, planes, qr, kr, S=4, L=2,
                                         dense_heads=(2,))
    for n, e in enumerate(planes):
        b, h = divmod(e, 4)
        assert np.abs(dq[n] - full[0][b, h, qr]).max() < 1e-12
        assert np.abs(dk[n] - full[1][b, h, kr]).max() < 1e-12
        assert np.abs(dv[n] - full[2][b, h, kr]).max() < 1e-12
    with pytest.raises(ValueError):  # a query row outside the group's heads
        oracle.backward_sampled(q, k, v, do, 8, w.scale, planes, [64], kr, S=4, L=2)
