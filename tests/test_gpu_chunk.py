"""Chunked prefill over a paged cache: the sm_100a kernel (through the C ABI)
against the oracle's chunk rows, every row of every chunk."""
import numpy as np
import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import synth

pytestmark = pytest.mark.gpu


def paged(k_dense, v_dense, ctx, seed, extra_pages=3):
    """Permuted paged cache holding the contexts; unused rows and pages stay NaN."""
    batch, H, n, D = k_dense.shape
    page = 16
    pages = [-(-c // page) for c in ctx]
    total = sum(pages) + extra_pages
    perm = np.random.default_rng(seed).permutation(total).astype(np.int32)
    bt = np.full((batch, max(pages)), -1, dtype=np.int32)
    kc = torch.full((total, H, page, D), float("nan"), dtype=torch.bfloat16)
    vc = torch.full_like(kc, float("nan"))
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


def case(s2, ctx, qlen, H=4, hkv=None, D=128, B=128, S=4, L=2, dense=(), seed=0, layout=None, bmask=None):
    hkv = hkv or H
    batch, n = len(ctx), max(ctx)
    w = synth.PrefillWorkload("t", batch, H, D, n, B, S, L, dense_heads=dense, seed=seed)
    qd, kd, vd = synth.prefill_inputs(w)
    kd, vd = kd[:, :hkv].contiguous(), vd[:, :hkv].contiguous()
    q_start = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    q = torch.cat([qd[s, :, ctx[s] - qlen[s]:ctx[s]].transpose(0, 1) for s in range(batch)], 0).contiguous()
    kc, vc, bt = paged(kd, vd, ctx, seed)
    nb = -(-n // B)
    lay = layout or s2.build_layout(H, B, S, L, nb, dense, device="cuda")
    out, lse = s2.chunk_prefill(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(bt).cuda(),
                                torch.tensor(ctx, dtype=torch.int32).cuda(), torch.from_numpy(q_start).cuda(),
                                lay, max(qlen), scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    if bmask is None:
        ref, lref = oracle.chunk(q, kc, vc, bt, ctx, q_start, B, w.scale, S=S, L=L, dense_heads=dense)
    else:
        ref, lref = oracle.chunk(q, kc, vc, bt, ctx, q_start, B, w.scale, bmask=bmask)
    parity(out.reshape(-1, D), ref.reshape(-1, D))
    fin = np.isfinite(lref.reshape(-1))
    got_lse = lse.reshape(-1).cpu().double().numpy()
    assert np.array_equal(np.isfinite(got_lse), fin)
    parity(got_lse[fin], lref.reshape(-1)[fin], max_tol=1e-3, mean_tol=1e-4)
    return out


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B", [64, 128])
def test_chunks_of_every_shape(s2gpu, D, B):
    # chunk lengths: whole context, one token, crossing 128-row tiles, starting mid-page
    ctx = [300, 1000, 129, 517, 64]
    qlen = [300, 1, 129, 200, 17]
    case(s2gpu, ctx, qlen, D=D, B=B, S=3, L=1, dense=(1,), seed=B + D)


def test_many_sequences_with_empty_chunks(s2gpu):
    # more than 32 sequences (items are mapped by a warp-wide prefix over the
    # sequences, 32 at a time) and some chunks of zero rows
    rng = np.random.default_rng(21)
    ctx = [int(c) for c in rng.integers(1, 400, size=37)]
    qlen = [int(rng.integers(0, c + 1)) for c in ctx]
    qlen[3] = qlen[20] = qlen[36] = 0
    qlen[0] = ctx[0]
    case(s2gpu, ctx, qlen, H=2, D=64, B=64, S=3, L=1, seed=21)


@pytest.mark.parametrize("B", [64, 128])
def test_many_items_per_cta(s2gpu, B):
    # ~400 tile-pair items for at most 148 persistent CTAs
    rng = np.random.default_rng(22)
    ctx = [int(c) for c in rng.integers(600, 2600, size=16)]
    qlen = [min(c, int(rng.integers(300, 700))) for c in ctx]
    case(s2gpu, ctx, qlen, H=8, D=64, B=B, S=4, L=1, seed=22 + B)


def test_grouped_kv_heads(s2gpu):
    case(s2gpu, [700, 260], [300, 260], H=8, hkv=2, seed=5)


def test_range_layout(s2gpu):
    ranges = [[(2, 0, 0, True), (8, 4, 1, False)] for _ in range(4)]
    lay = s2gpu.build_layout_ranges(ranges, 128, 8, device="cuda")
    case(s2gpu, [1000, 333], [400, 333], layout=lay, bmask=oracle.range_block_mask(8, ranges), seed=6)


@pytest.mark.parametrize("B", [64, 128])
def test_mask_layout_with_empty_rows(s2gpu, B):
    # Random per-head block masks with empty query-block rows: some items have
    # a tile that sees no key block (its Q is released at once and its rows
    # get zeros and an LSE of -inf) beside a tile that does.
    H, n = 3, 1100
    nb = -(-n // B)
    rng = np.random.default_rng(40 + B)
    m = np.tril(rng.random((H, nb, nb)) < 0.35).astype(np.uint8)
    for h in range(H):
        m[h, rng.choice(nb, 3, replace=False)] = 0  # empty query-block rows
    lay = s2gpu.build_layout_mask(m, B, device="cuda")
    case(s2gpu, [n, 700], [600, 700], H=H, B=B, layout=lay, bmask=m, seed=41 + B)


def test_one_token_chunks_match_decode(s2gpu):
    ctx = [1, 17, 500, 1024]
    out = case(s2gpu, ctx, [1, 1, 1, 1], seed=7)
    assert torch.isfinite(out).all()


def test_long_chunk_sampled(s2gpu):
    # 2 sequences of 8K context with 4K-token chunks, 16 heads
    ctx, qlen = [8192, 6000], [4096, 3000]
    case(s2gpu, ctx, qlen, H=16, S=16, L=4, seed=8)


@pytest.mark.parametrize("B", [64, 128])
def test_output_only_16_byte_aligned(s2gpu, B):
    # The epilogue stores whole 32-byte sectors when the output is 32-byte
    # aligned and falls back to 16-byte stores otherwise: both write the same
    # bytes, and nothing outside the output.
    ctx, qlen, H, D = [700, 300], [300, 300], 4, 128
    w = synth.PrefillWorkload("t", 2, H, D, max(ctx), B, 3, 1, seed=31)
    qd, kd, vd = synth.prefill_inputs(w)
    q_start = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    q = torch.cat([qd[s, :, ctx[s] - qlen[s]:ctx[s]].transpose(0, 1) for s in range(2)], 0).contiguous()
    kc, vc, bt = paged(kd, vd, ctx, 31)
    lay = s2gpu.build_layout(H, B, 3, 1, -(-max(ctx) // B), device="cuda")
    args = (q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(bt).cuda(),
            torch.tensor(ctx, dtype=torch.int32).cuda(), torch.from_numpy(q_start).cuda(), lay, max(qlen))
    ref = s2gpu.chunk_prefill(*args, scale=w.scale)
    n = ref.numel()
    buf = torch.full((n + 24,), float("nan"), dtype=torch.bfloat16, device="cuda")
    base = buf.data_ptr()
    off = next(e for e in range(0, 24, 8) if (base + 2 * e) % 32 == 16)  # 16- but not 32-byte aligned
    out = buf[off:off + n].view(ref.shape)
    s2gpu.chunk_prefill(*args, scale=w.scale, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.isnan(buf[:off].float()).all() and torch.isnan(buf[off + n:].float()).all()


def test_bad_chunk_length_is_flagged(s2gpu):
    H, D, B = 2, 128, 128
    q = torch.zeros(8, H, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, H, 16, D, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    lay = s2gpu.build_layout(H, B, 4, 1, 1, device="cuda")
    s2gpu.chunk_prefill(q, kc, kc, bt, torch.tensor([4], dtype=torch.int32, device="cuda"),
                        torch.tensor([0, 8], dtype=torch.int32, device="cuda"), lay, 8)
    rc, flags = s2gpu.device_status(reset=True)
    assert rc == 6 and flags == 2
