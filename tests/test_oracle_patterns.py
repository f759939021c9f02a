"""Pins for the oracle's generalised block rules: per-context-range patterns,
any per-head block mask, grouped key/value heads and rows that see no key.

The arXiv abstract of "S2-Attention: Hardware-aware context sharding among
attention heads" says the sparse patterns can be customised per head and per
context range. Each test ties the oracle to something outside it: a
hand-enumerated pattern, a closed-form count, the base HHST rule (itself pinned
by its own fixture), torch SDPA in fp64 with an explicit mask, or the reduction
of grouped heads to plain multi-head attention by repeating K and V.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN, read_block_pattern
from head_heterogeneous_block_s2_b200 import synth

# head 0: dense prefix then strided; head 1: three ranges; head 2: empty prefix.
FIXTURE_RANGES = [
    [(2, 0, 0, True), (8, 3, 1, False)],
    [(3, 2, 2, False), (5, 0, 3, False), (8, 4, 1, False)],
    [(4, 0, 0, False), (8, 2, 1, False)],
]


def test_range_pattern_matches_hand_enumeration():
    want = read_block_pattern(os.path.join(GOLDEN, "range_block_pattern.txt"))
    m = oracle.range_block_mask(8, FIXTURE_RANGES)
    got = {(h, i): [int(j) for j in np.nonzero(m[h, i])[0]] for h in range(3) for i in range(8)}
    assert got == want
    assert int(m.sum()) == 54


@pytest.mark.parametrize("H,nb,S,L,dense", [
    (4, 8, 4, 1, ()), (16, 64, 8, 2, (3,)), (6, 40, 7, 3, (0, 5)), (3, 17, 1, 1, ()),
])
def test_one_range_is_the_base_rule(H, nb, S, L, dense):
    ranges = [[(nb, S, L, h in dense)] for h in range(H)]
    assert np.array_equal(oracle.range_block_mask(nb, ranges), oracle.block_mask(H, nb, S, L, dense))


def _hhst_count_from(h, i, lo, S, L):
    """Blocks j in [lo, i] with i - j < L or (j + h) % S == 0, counted arithmetically."""
    if i < lo:
        return 0
    local_lo = max(lo, i - L + 1)
    local = i - local_lo + 1
    top = local_lo - 1  # strided candidates lo..top
    if top < lo:
        return local
    j0 = lo + ((-(lo + h)) % S)  # smallest j >= lo with (j + h) % S == 0
    return local + (0 if top < j0 else (top - j0) // S + 1)


@pytest.mark.parametrize("H,nb,r,S,L", [(8, 64, 4, 8, 2), (5, 33, 1, 3, 1), (4, 20, 20, 4, 1),
                                        (16, 128, 16, 16, 4)])
def test_dense_prefix_counts_closed_form(H, nb, r, S, L):
    """Dense first r blocks (a "sink" range), HHST after it."""
    ranges = [[(r, 1, 0, True)] + ([(nb, S, L, False)] if r < nb else []) for _ in range(H)]
    m = oracle.range_block_mask(nb, ranges)
    for h in range(H):
        for i in range(nb):
            want = min(i + 1, r) + _hhst_count_from(h, i, r, S, L)
            assert int(m[h, i].sum()) == want, (h, i)
            assert m[h, i, i + 1:].sum() == 0


def test_blocks_past_the_last_range_are_invisible():
    assert not oracle.range_block_active(0, 9, 6, [(5, 1, 10, True)])
    assert oracle.range_block_active(0, 9, 4, [(5, 1, 10, True)])
    assert not oracle.range_block_active(0, 3, 4, [(8, 1, 10, True)])  # j > i


# ---------------------------------------------------------------- masked values

def _token_mask(bmask, seq, B):
    H, nbm, _ = bmask.shape
    tm = np.repeat(np.repeat(bmask.astype(bool), B, axis=1), B, axis=2)[:, :seq, :seq]
    return tm & np.tril(np.ones((seq, seq), dtype=bool))[None]


def _explicit(q, k, v, tmask, scale):
    """fp64 masked softmax written with explicit tensors; empty rows -> 0, -inf."""
    s = torch.einsum("bhqd,bhkd->bhqk", q.double(), k.double()) * scale
    s = s.masked_fill(~torch.as_tensor(tmask)[None], -math.inf)
    lse = torch.logsumexp(s, -1)
    p = torch.exp(s - lse[..., None]).nan_to_num(0.0)
    return torch.einsum("bhqk,bhkd->bhqd", p, v.double()), lse


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_block_mask_matches_explicit_softmax(seed):
    B, seq, H, D = 8, 60, 3, 16  # ragged: 60 = 7 full blocks + 4 tokens
    nb = -(-seq // B)
    rng = np.random.default_rng(seed)
    bm = (rng.random((H, nb, nb)) < 0.4).astype(np.uint8)
    bm[0, 2, :] = 0  # one query block with no key at all
    w = synth.PrefillWorkload("t", 2, H, D, seq, B, 4, 1, seed=20 + seed)
    q, k, v = synth.prefill_inputs(w)
    out, lse = oracle.prefill_mask(q, k, v, B, bm, w.scale)
    tm = _token_mask(bm, seq, B)
    ref, lref = _explicit(q, k, v, tm, w.scale)
    assert np.abs(out - ref.reshape(-1, D).numpy()).max() < 1e-12
    lref = lref.reshape(-1).numpy()
    finite = np.isfinite(lref)
    assert np.array_equal(finite, np.isfinite(lse))
    assert np.abs(lse[finite] - lref[finite]).max() < 1e-12
    empty = ~tm.any(-1)  # [H, seq]
    assert empty[0, 2 * B:3 * B].all()
    o = out.reshape(2, H, seq, D)
    assert (o[:, empty] == 0).all() and np.isneginf(lse.reshape(2, H, seq)[:, empty]).all()


def test_all_ones_mask_equals_causal_sdpa():
    w = synth.PrefillWorkload("t", 1, 2, 32, 50, 8, 1, 1, seed=7)
    q, k, v = synth.prefill_inputs(w)
    bm = np.ones((2, 7, 7), dtype=np.uint8)  # entries above the diagonal are ignored
    out, _ = oracle.prefill_mask(q, k, v, 8, bm, w.scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), is_causal=True, scale=w.scale)
    assert np.abs(out - ref.reshape(-1, 32).numpy()).max() < 1e-12


def test_range_mask_values_match_explicit_softmax():
    B, seq, D = 8, 64, 16
    w = synth.PrefillWorkload("t", 1, 3, D, seq, B, 4, 1, seed=31)
    q, k, v = synth.prefill_inputs(w)
    bm = oracle.range_block_mask(8, FIXTURE_RANGES)
    out, lse = oracle.prefill_mask(q, k, v, B, bm, w.scale)
    ref, _ = _explicit(q, k, v, _token_mask(bm, seq, B), w.scale)
    assert np.abs(out - ref.reshape(-1, D).numpy()).max() < 1e-12
    assert np.isneginf(lse.reshape(3, seq)[2, :32]).all()  # head 2, blocks 0..3 empty


@pytest.mark.parametrize("Hkv", [1, 2])
def test_grouped_kv_heads_reduce_to_repeated_heads(Hkv):
    H, B, seq, D = 4, 8, 40, 16
    w = synth.PrefillWorkload("t", 2, H, D, seq, B, 2, 1, seed=40)
    q, k, v = synth.prefill_inputs(w)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    bm = oracle.block_mask(H, 5, 2, 1)
    out, lse = oracle.prefill_mask(q, k, v, B, bm, w.scale)
    g = H // Hkv
    out2, lse2 = oracle.prefill_mask(q, k.repeat_interleave(g, 1), v.repeat_interleave(g, 1), B,
                                     bm, w.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # and head h really reads kv head h // g: swapping kv heads changes the output
    if Hkv == 2:
        out3, _ = oracle.prefill_mask(q, k.flip(1).contiguous(), v.flip(1).contiguous(), B, bm,
                                      w.scale)
        assert not np.allclose(out, out3)


def test_hhst_mask_reproduces_base_oracle_exactly():
    w = synth.PrefillWorkload("t", 1, 4, 16, 64, 8, 4, 2, dense_heads=(1,), seed=41)
    q, k, v = synth.prefill_inputs(w)
    a, la = oracle.prefill(q, k, v, 8, 4, 2, w.scale, (1,))
    b, lb = oracle.prefill_mask(q, k, v, 8, oracle.block_mask(4, 8, 4, 2, (1,)), w.scale)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


# ---------------------------------------------------------------- decode

def _paged(k_dense, v_dense, ctx, page, seed):
    batch, Hkv, n, D = k_dense.shape
    pages = [-(-c // page) for c in ctx]
    perm = np.random.default_rng(seed).permutation(sum(pages)).astype(np.int32)
    bt = np.full((batch, max(pages)), -1, dtype=np.int32)
    kc = torch.zeros(sum(pages), Hkv, page, D, dtype=torch.bfloat16)
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


@pytest.mark.parametrize("Hkv", [3, 1])
def test_decode_mask_equals_last_prefill_row(Hkv):
    H, D, B, page = 3, 16, 8, 4
    ctx = [5, 29, 64, 40]
    batch, n = len(ctx), max(ctx)
    w = synth.PrefillWorkload("t", batch, H, D, n, B, 4, 1, seed=42)
    qd, kd, vd = synth.prefill_inputs(w)
    kd, vd = kd[:, :Hkv].contiguous(), vd[:, :Hkv].contiguous()
    bm = oracle.range_block_mask(8, FIXTURE_RANGES)
    kc, vc, bt = _paged(kd, vd, ctx, page, 0)
    qdec = torch.stack([qd[s, :, ctx[s] - 1] for s in range(batch)])
    out, lse = oracle.decode_mask(qdec, kc, vc, bt, ctx, B, bm, w.scale)
    for s in range(batch):
        c = ctx[s]
        rows = [h * c + c - 1 for h in range(H)]
        ref, lref = oracle.prefill_mask(qd[s:s + 1, :, :c].contiguous(), kd[s:s + 1, :, :c].contiguous(),
                                        vd[s:s + 1, :, :c].contiguous(), B, bm, w.scale, rows=rows)
        assert np.abs(out[s * H:(s + 1) * H] - ref).max() < 1e-12
        assert np.array_equal(np.isneginf(lse[s * H:(s + 1) * H]), np.isneginf(lref))
    # ctx 5 ends in block 0: head 2 sees nothing there
    assert np.isneginf(lse[2]) and (out[2] == 0).all()
    kc2, vc2, bt2 = _paged(kd, vd, ctx, page, 5)
    out2, _ = oracle.decode_mask(qdec, kc2, vc2, bt2, ctx, B, bm, w.scale)
    assert np.array_equal(out, out2)


def test_mask_entry_points_reject_bad_arguments():
    w = synth.PrefillWorkload("t", 1, 4, 16, 32, 8, 2, 1, seed=1)
    q, k, v = synth.prefill_inputs(w)
    with pytest.raises(ValueError):  # 4 query heads over 3 kv heads
        oracle.prefill_mask(q, k[:, :3].contiguous(), v[:, :3].contiguous(), 8,
                            np.ones((4, 4, 4), np.uint8), w.scale)
    with pytest.raises(ValueError):  # mask smaller than the block count
        oracle.prefill_mask(q, k, v, 8, np.ones((4, 3, 3), np.uint8), w.scale)
