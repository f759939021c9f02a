"""Pins for the fp64 oracle: checks that do not trust the oracle itself.

Each test ties the oracle to something fixed outside it: a hand-enumerated
pattern, a closed form, a library routine (torch SDPA in fp64), or an invariant
of softmax attention. The method (HHST sparse attention, "S2-Attention:
Hardware-aware context sharding among attention heads", Abstract) computes
exactly masked softmax attention, so these pins cover the whole definition:
the block rule, diagonal causality, the scale, the softmax normalisation, the
weighted sum of V and the log-sum-exp.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN, read_block_pattern
from head_heterogeneous_block_s2_b200 import synth


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def closed_form_row_count(h, i, S, L, dense):
    """Active blocks in row (h, i): min(L, i+1) local blocks plus the strided
    blocks j <= i-L with j = -h (mod S). Counted arithmetically, not by the rule."""
    if dense:
        return i + 1
    local = min(L, i + 1)
    top = i - L  # strided candidates 0..top
    if top < 0:
        return local
    j0 = (-h) % S  # smallest j >= 0 with (j + h) % S == 0
    strided = 0 if top < j0 else (top - j0) // S + 1
    return local + strided


# ---------------------------------------------------------------- block rule

def test_block_pattern_matches_hand_enumeration():
    want = read_block_pattern(os.path.join(GOLDEN, "tiny_block_pattern.txt"))
    m = oracle.block_mask(4, 8, 4, 1)
    got = {(h, i): [int(j) for j in np.nonzero(m[h, i])[0]] for h in range(4) for i in range(8)}
    assert got == want
    assert int(m.sum()) == 60


@pytest.mark.parametrize("H,nb,S,L,dense", [
    (4, 8, 4, 1, ()), (16, 128, 8, 2, ()), (32, 256, 16, 4, (0, 1, 2, 3)),
    (5, 40, 7, 3, (2,)), (3, 33, 1, 1, ()), (6, 20, 25, 2, ()), (8, 64, 3, 70, ()),
])
def test_row_counts_closed_form(H, nb, S, L, dense):
    m = oracle.block_mask(H, nb, S, L, dense)
    for h in range(H):
        for i in range(nb):
            assert int(m[h, i].sum()) == closed_form_row_count(h, i, S, L, h in dense), (h, i)
            assert m[h, i, i + 1:].sum() == 0  # causal at block level
            assert m[h, i, i] == 1  # the diagonal block is always active (L >= 1)


@pytest.mark.parametrize("H,S", [(4, 4), (16, 8), (32, 16), (5, 3)])
def test_heads_cover_every_causal_block_when_H_ge_S(H, S):
    nb, L = 48, 1
    m = oracle.block_mask(H, nb, S, L)
    union = m.max(axis=0)
    assert np.array_equal(union, np.tril(np.ones((nb, nb), dtype=np.uint8)))


def test_heads_leave_residues_uncovered_when_H_lt_S():
    H, S, L, nb = 3, 8, 1, 40
    union = oracle.block_mask(H, nb, S, L).max(axis=0)
    covered_residues = {(-h) % S for h in range(H)}
    for i in range(nb):
        for j in range(i + 1):
            expect = (i - j < L) or (j % S in covered_residues)
            assert bool(union[i, j]) == expect


def test_stride_one_is_dense_causal():
    m = oracle.block_mask(3, 17, 1, 1)
    tri = np.tril(np.ones((17, 17), dtype=np.uint8))
    assert all(np.array_equal(m[h], tri) for h in range(3))


# ---------------------------------------------------------------- attention values

def token_mask(H, seq, B, S, L, dense=()):
    """Explicit [H, seq, seq] boolean mask from the (separately pinned) block mask
    plus causality inside blocks."""
    nb = seq // B
    bm = oracle.block_mask(H, nb, S, L, dense).astype(bool)
    tm = np.repeat(np.repeat(bm, B, axis=1), B, axis=2)
    causal = np.tril(np.ones((seq, seq), dtype=bool))
    return tm & causal[None]


def sdpa_reference(q, k, v, mask, scale):
    """torch SDPA in fp64 with an explicit boolean mask (a library routine)."""
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=torch.as_tensor(mask), scale=scale)


@pytest.mark.parametrize("B", [4, 8, 16])
@pytest.mark.parametrize("S,L,dense", [(4, 1, ()), (2, 2, (1,)), (3, 1, ())])
def test_brute_force_masked_softmax_agrees(B, S, L, dense):
    w = synth.PrefillWorkload("t", 2, 4, 32, 64, B, S, L, dense_heads=dense, seed=11)
    q, k, v = synth.prefill_inputs(w)
    out, lse = oracle.prefill(q, k, v, B, S, L, w.scale, dense)
    mask = token_mask(4, 64, B, S, L, dense)
    ref = sdpa_reference(q, k, v, mask[None], w.scale).reshape(-1, 32).numpy()
    assert np.abs(out - ref).max() < 1e-12
    # log-sum-exp against an fp64 logsumexp of the masked logits
    s = torch.einsum("bhqd,bhkd->bhqk", q.double(), k.double()) * w.scale
    s = s.masked_fill(~torch.as_tensor(mask)[None], -math.inf)
    assert np.abs(lse - torch.logsumexp(s, -1).reshape(-1).numpy()).max() < 1e-12


def test_stride_one_equals_causal_sdpa():
    w = synth.PrefillWorkload("t", 1, 3, 64, 96, 8, 1, 1, seed=5)
    q, k, v = synth.prefill_inputs(w)
    out, _ = oracle.prefill(q, k, v, 8, 1, 1, w.scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), is_causal=True, scale=w.scale)
    assert np.abs(out - ref.reshape(-1, 64).numpy()).max() < 1e-12


def test_probability_rows_sum_to_one_and_vanish_outside_pattern():
    # With V = identity (seq == D), output row q is the probability row p(q, .).
    H, seq, B, S, L = 4, 64, 8, 4, 1
    w = synth.PrefillWorkload("t", 1, H, seq, seq, B, S, L, seed=3)
    q, k, _ = synth.prefill_inputs(w)
    v = torch.eye(seq, dtype=torch.bfloat16).expand(1, H, seq, seq).contiguous()
    out, _ = oracle.prefill(q, k, v, B, S, L, w.scale)
    p = out.reshape(H, seq, seq)
    assert np.abs(p.sum(-1) - 1.0).max() < 1e-12
    mask = token_mask(H, seq, B, S, L)
    assert np.all(p[~mask] == 0.0)
    assert np.all(p[mask] > 0.0)


def test_zero_query_gives_uniform_attention_closed_form():
    # Q = 0 makes every logit 0: O = mean of the visible V rows, LSE = log(count).
    H, seq, B, S, L = 4, 128, 16, 4, 2
    w = synth.PrefillWorkload("t", 1, H, 32, seq, B, S, L, seed=8)
    _, k, v = synth.prefill_inputs(w)
    q = torch.zeros_like(k)
    out, lse = oracle.prefill(q, k, v, B, S, L, w.scale)
    vd = v.double().numpy()[0]
    for h in range(H):
        for t in range(0, seq, 7):
            i = t // B
            keys = [x for x in range(t + 1)
                    if (i - x // B < L) or ((x // B + h) % S == 0)]
            # the count also follows from the closed-form block count
            nfull = closed_form_row_count(h, i, S, L, False) - 1  # blocks before the diagonal
            assert len(keys) == nfull * B + (t % B + 1)
            r = h * seq + t
            assert abs(lse[r] - math.log(len(keys))) < 1e-12
            assert np.abs(out[r] - vd[h, keys].mean(0)).max() < 1e-12


def test_two_visible_keys_closed_form():
    # Query row 1 of block 0 sees exactly keys 0 and 1. With q = (1, 0, ...),
    # k0 = 0 and k1 = (a, 0, ...), p1 = 1 / (1 + exp(-scale * a)).
    D, seq, B = 8, 16, 4
    q = torch.zeros(1, 1, seq, D)
    k = torch.zeros(1, 1, seq, D)
    v = torch.zeros(1, 1, seq, D)
    q[0, 0, 1, 0] = 1.0
    k[0, 0, 1, 0] = 3.0
    v[0, 0, 0, 0] = 2.0
    v[0, 0, 1, 1] = -5.0
    scale = 0.5
    out, lse = oracle.prefill(bf16(q), bf16(k), bf16(v), B, 4, 1, scale, rows=[1])
    p1 = 1.0 / (1.0 + math.exp(-1.5))
    assert abs(out[0, 0] - 2.0 * (1 - p1)) < 1e-15
    assert abs(out[0, 1] - (-5.0) * p1) < 1e-15
    assert abs(lse[0] - math.log(1.0 + math.exp(1.5))) < 1e-15


def test_scale_multiplies_logits():
    w = synth.PrefillWorkload("t", 1, 2, 16, 32, 8, 2, 1, seed=4)
    q, k, v = synth.prefill_inputs(w)
    a, la = oracle.prefill(q, k, v, 8, 2, 1, 0.25)
    b, lb = oracle.prefill(bf16(q.float() * 2), k, v, 8, 2, 1, 0.125)  # 2x is exact in bf16
    assert np.abs(a - b).max() < 1e-12 and np.abs(la - lb).max() < 1e-12


def test_output_in_convex_hull_of_visible_values():
    w = synth.PrefillWorkload("t", 1, 4, 16, 128, 16, 4, 1, seed=9)
    q, k, v = synth.prefill_inputs(w)
    out, _ = oracle.prefill(q, k, v, 16, 4, 1, w.scale)
    mask = token_mask(4, 128, 16, 4, 1)
    vd = v.double().numpy()[0]
    o = out.reshape(4, 128, 16)
    for h in range(4):
        for t in range(128):
            vis = vd[h, mask[h, t]]
            assert np.all(o[h, t] >= vis.min(0) - 1e-12) and np.all(o[h, t] <= vis.max(0) + 1e-12)


def test_planted_key_dominates_only_when_its_block_is_active():
    H, seq, B, S, L, D = 4, 512, 16, 4, 2, 64
    w = synth.PrefillWorkload("t", 1, H, D, seq, B, S, L, seed=6)
    last_block = (seq - 1) // B
    active_at, inactive_at = {}, {}
    for h in range(H):
        j_on = next(j for j in range(2, last_block - L) if (j + h) % S == 0)
        j_off = next(j for j in range(2, last_block - L) if (j + h) % S != 0)
        active_at[h] = j_on * B + 3
        inactive_at[h] = j_off * B + 3
    rows = [h * seq + seq - 1 for h in range(H)]
    q0, k0, v0 = synth.prefill_inputs(w)
    base, _ = oracle.prefill(q0, k0, v0, B, S, L, w.scale, rows=rows)
    q1, k1, v1 = synth.prefill_inputs(w, plant_positions=active_at)
    on, _ = oracle.prefill(q1, k1, v1, B, S, L, w.scale, rows=rows)
    q2, k2, v2 = synth.prefill_inputs(w, plant_positions=inactive_at)
    off, _ = oracle.prefill(q2, k2, v2, B, S, L, w.scale, rows=rows)
    for h in range(H):
        assert np.abs(on[h] - v1[0, h, active_at[h]].double().numpy()).max() < 1e-3
    assert np.array_equal(off, base)


def test_row_subset_equals_full_rows():
    w = synth.TINY.with_(seq=256)
    q, k, v = synth.prefill_inputs(w)
    full, lf = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale)
    rows = [0, 5, 63, 64, 300, 1023]
    sub, ls = oracle.prefill(q, k, v, w.block, w.stride, w.local, w.scale, rows=rows)
    assert np.array_equal(sub, full[rows]) and np.array_equal(ls, lf[rows])


# ---------------------------------------------------------------- decode

def _dense_to_paged(k_dense, v_dense, ctx, page, perm_seed):
    """Pack dense [batch, H, n, D] K/V into a permuted paged cache (test-side layout)."""
    batch, H, n, D = k_dense.shape
    pages = [-(-c // page) for c in ctx]
    total = sum(pages)
    perm = np.random.default_rng(perm_seed).permutation(total).astype(np.int32)
    maxp = max(pages)
    bt = np.full((batch, maxp), -1, dtype=np.int32)
    kc = torch.zeros(total, H, page, D, dtype=torch.bfloat16)
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


@pytest.mark.parametrize("dense", [(), (1,)])
def test_decode_equals_last_prefill_row_and_ignores_page_order(dense):
    H, D, B, S, L, page = 4, 32, 16, 4, 2, 4
    ctx = [1, 37, 64, 90]
    batch, n = len(ctx), max(ctx)
    w = synth.PrefillWorkload("t", batch, H, D, n, B, S, L, dense_heads=dense, seed=12)
    qd, kd, vd = synth.prefill_inputs(w)
    kc, vc, bt = _dense_to_paged(kd, vd, ctx, page, 0)
    qdec = torch.stack([qd[s, :, ctx[s] - 1] for s in range(batch)])
    out, lse = oracle.decode(qdec, kc, vc, bt, ctx, B, S, L, w.scale, dense)
    for s in range(batch):
        # prefill of the first ctx[s] tokens of sequence s, last row
        sub = synth.PrefillWorkload("t", 1, H, D, ctx[s], B, S, L, dense_heads=dense)
        rows = [h * ctx[s] + ctx[s] - 1 for h in range(H)]
        ref, lref = oracle.prefill(qd[s:s + 1, :, : ctx[s]].contiguous(),
                                   kd[s:s + 1, :, : ctx[s]].contiguous(),
                                   vd[s:s + 1, :, : ctx[s]].contiguous(),
                                   B, S, L, sub.scale, dense, rows=rows)
        assert np.abs(out[s * H:(s + 1) * H] - ref).max() < 1e-12
        assert np.abs(lse[s * H:(s + 1) * H] - lref).max() < 1e-12
    kc2, vc2, bt2 = _dense_to_paged(kd, vd, ctx, page, 99)
    out2, _ = oracle.decode(qdec, kc2, vc2, bt2, ctx, B, S, L, w.scale, dense)
    assert np.array_equal(out, out2)


def test_oracle_rejects_bad_arguments():
    w = synth.TINY.with_(seq=64)
    q, k, v = synth.prefill_inputs(w)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, 64, 4, 0, w.scale)  # L < 1
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, 64, 4, 1, w.scale, rows=[10 ** 9])
