"""fp64 CPU oracle for HHST sparse attention (ctypes wrapper of s2_oracle.c).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The library package
(``head_heterogeneous_block_s2_b200``) never imports it, and the oracle imports
nothing from the library: the two share no code.

This module does argument marshalling only; every number is computed by the C
code in ``s2_oracle.c``, which states the definition it follows (masked softmax
attention under the per-head strided block rule of S2-Attention / HHST,
"S2-Attention: Hardware-aware context sharding among attention heads",
Abstract).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s2_oracle.c")
_LIB = os.path.join(_HERE, "libs2oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile s2_oracle.c into libs2oracle.so (plain gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    lib.s2o_block_active.restype = i32
    lib.s2o_block_active.argtypes = [i64, i64, i64, i64, i64, i32]
    lib.s2o_block_mask.restype = None
    lib.s2o_block_mask.argtypes = [i64, i64, i64, i64, vp, vp]
    lib.s2o_default_threads.restype = i32
    lib.s2o_default_threads.argtypes = []
    lib.s2o_prefill_rows.restype = i32
    lib.s2o_prefill_rows.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, vp,
                                     dbl, i64, vp, vp, vp, i32]
    lib.s2o_decode_items.restype = i32
    lib.s2o_decode_items.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64,
                                     i64, vp, dbl, i64, vp, vp, vp, i32]
    lib.s2o_chunk_rows.restype = i32
    lib.s2o_chunk_rows.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64,
                                   i64, vp, i64, vp, dbl, vp, vp, i32]
    lib.s2o_backward.restype = i32
    lib.s2o_backward.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, vp, i64,
                                 vp, dbl, vp, vp, vp, i32]
    lib.s2o_backward_sampled.restype = i32
    lib.s2o_backward_sampled.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, vp,
                                         i64, vp, dbl, i64, vp, i64, vp, i64, vp, vp, vp, vp, i32]
    lib.s2o_range_block_active.restype = i32
    lib.s2o_range_block_active.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp]
    lib.s2o_range_block_mask.restype = None
    lib.s2o_range_block_mask.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp]
    lib.s2o_prefill_rows_mask.restype = i32
    lib.s2o_prefill_rows_mask.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, vp,
                                          dbl, i64, vp, vp, vp, i32]
    lib.s2o_decode_items_mask.restype = i32
    lib.s2o_decode_items_mask.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64,
                                          i64, vp, dbl, i64, vp, vp, vp, i32]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(a) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array of bf16 bits; return uint16 C-contiguous."""
    if hasattr(a, "detach"):  # torch tensor (oracle stays importable without torch)
        import torch

        assert a.dtype == torch.bfloat16, a.dtype
        a = a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _dense(H, dense):
    if dense is None:
        return None
    d = np.zeros(H, dtype=np.uint8)
    for h in dense:
        d[int(h)] = 1
    return d


def default_threads() -> int:
    return int(_load().s2o_default_threads())


def block_active(h, i, j, S, L, dense=False) -> bool:
    return bool(_load().s2o_block_active(h, i, j, S, L, int(bool(dense))))


def block_mask(H, nb, S, L, dense_heads=None) -> np.ndarray:
    """uint8 mask [H, nb, nb]: 1 where key block j is visible to query block i of head h."""
    m = np.zeros((H, nb, nb), dtype=np.uint8)
    d = _dense(H, dense_heads)
    _load().s2o_block_mask(H, nb, S, L, _ptr(d), _ptr(m))
    return m


def prefill(q, k, v, B, S, L, scale, dense_heads=None, rows=None, nthreads=0):
    """Oracle prefill. q, k, v: [batch, H, seq, D] bf16 (torch or uint16 bits).

    rows: None for every row, else linear ids (b*H + h)*seq + q.
    Returns (out fp64 [n_rows, D], lse fp64 [n_rows]).
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    batch, H, seq, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    d = _dense(H, dense_heads)
    if rows is None:
        n = batch * H * seq
        r = None
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = r.size
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = _load().s2o_prefill_rows(_ptr(q), _ptr(k), _ptr(v), batch, H, seq, D, B, S, L,
                                  _ptr(d), float(scale), n, _ptr(r), _ptr(out), _ptr(lse),
                                  int(nthreads))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return out, lse


def decode(q, k_cache, v_cache, block_table, ctx_lens, B, S, L, scale,
           dense_heads=None, items=None, nthreads=0):
    """Oracle decode over a paged cache.

    q: [batch, H, D]; k_cache, v_cache: [pages, H, page_size, D] (bf16);
    block_table: int32 [batch, max_pages]; ctx_lens: int32 [batch].
    items: None for all (s, h), else ids s*H + h. Returns (out [n, D], lse [n]).
    """
    q, kc, vc = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(ctx_lens, dtype=np.int32))
    batch, H, D = q.shape
    _, H2, page_size, D2 = kc.shape
    assert H2 == H and D2 == D and vc.shape == kc.shape
    max_pages = bt.shape[1]
    d = _dense(H, dense_heads)
    if items is None:
        n, it = batch * H, None
    else:
        it = np.ascontiguousarray(np.asarray(items, dtype=np.int64))
        n = it.size
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = _load().s2o_decode_items(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cl), batch, H, D,
                                  page_size, max_pages, B, S, L, _ptr(d), float(scale), n,
                                  _ptr(it), _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return out, lse


def _flat_ranges(ranges):
    """Per-head lists of (end_block, S, L, dense) -> CSR arrays for the C code."""
    ptr = [0]
    end, S, L, dense = [], [], [], []
    for head in ranges:
        for (e, s_, l_, d_) in head:
            end.append(int(e)); S.append(int(s_)); L.append(int(l_)); dense.append(int(bool(d_)))
        ptr.append(len(end))
    a = lambda x, t: np.ascontiguousarray(np.asarray(x, dtype=t))
    return a(ptr, np.int64), a(end, np.int64), a(S, np.int64), a(L, np.int64), a(dense, np.uint8)


def range_block_active(h, i, j, head_ranges) -> bool:
    """Per-context-range rule for head h; head_ranges = [(end_block, S, L, dense), ...]."""
    _ptr_, end, S, L, dense = _flat_ranges([head_ranges])
    return bool(_load().s2o_range_block_active(h, i, j, len(head_ranges), _ptr(end), _ptr(S),
                                               _ptr(L), _ptr(dense)))


def range_block_mask(nb, ranges) -> np.ndarray:
    """uint8 mask [H, nb, nb] of per-head context ranges (ranges[h] = [(end, S, L, dense), ...])."""
    H = len(ranges)
    ptr, end, S, L, dense = _flat_ranges(ranges)
    m = np.zeros((H, nb, nb), dtype=np.uint8)
    _load().s2o_range_block_mask(H, nb, _ptr(ptr), _ptr(end), _ptr(S), _ptr(L), _ptr(dense),
                                 _ptr(m))
    return m


def prefill_mask(q, k, v, B, bmask, scale, rows=None, nthreads=0):
    """Oracle prefill under a block mask [H, nbm, nbm] (uint8).

    q: [batch, H, seq, D]; k, v: [batch, Hkv, seq, D] with Hkv dividing H.
    Rows that see no key come back as zeros with LSE -inf.
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    batch, H, seq, D = q.shape
    Hkv = k.shape[1]
    assert k.shape == (batch, Hkv, seq, D) and v.shape == k.shape
    bm = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
    assert bm.ndim == 3 and bm.shape[0] == H and bm.shape[1] == bm.shape[2]
    if rows is None:
        n, r = batch * H * seq, None
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = r.size
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = _load().s2o_prefill_rows_mask(_ptr(q), _ptr(k), _ptr(v), batch, H, Hkv, seq, D, B,
                                       bm.shape[1], _ptr(bm), float(scale), n, _ptr(r),
                                       _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle prefill_mask rejected its arguments")
    return out, lse


def decode_mask(q, k_cache, v_cache, block_table, ctx_lens, B, bmask, scale, items=None,
                nthreads=0):
    """Oracle decode under a block mask [H, nbm, nbm]; caches [pages, Hkv, page_size, D]."""
    q, kc, vc = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(ctx_lens, dtype=np.int32))
    batch, H, D = q.shape
    _, Hkv, page_size, D2 = kc.shape
    assert D2 == D and vc.shape == kc.shape
    bm = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
    assert bm.ndim == 3 and bm.shape[0] == H and bm.shape[1] == bm.shape[2]
    if items is None:
        n, it = batch * H, None
    else:
        it = np.ascontiguousarray(np.asarray(items, dtype=np.int64))
        n = it.size
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = _load().s2o_decode_items_mask(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cl), batch, H,
                                       Hkv, D, page_size, bt.shape[1], B, bm.shape[1], _ptr(bm),
                                       float(scale), n, _ptr(it), _ptr(out), _ptr(lse),
                                       int(nthreads))
    if rc != 0:
        raise ValueError("oracle decode_mask rejected its arguments")
    return out, lse


def backward(q, k, v, dout, B, scale, S=None, L=None, dense_heads=None, bmask=None, nthreads=0):
    """Oracle gradients (dq, dk, dv) in fp64 of the masked softmax attention.

    q, dout: [batch, H, seq, D]; k, v: [batch, Hkv, seq, D] (bf16). The block
    rule is HHST (S, L, dense_heads) unless ``bmask`` [H, nbm, nbm] is given.
    Returns dq [batch, H, seq, D], dk and dv [batch, Hkv, seq, D].
    """
    q, k, v, do = _bits(q), _bits(k), _bits(v), _bits(dout)
    batch, H, seq, D = q.shape
    Hkv = k.shape[1]
    assert k.shape == (batch, Hkv, seq, D) and v.shape == k.shape and do.shape == q.shape
    if bmask is not None:
        bm = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
        assert bm.ndim == 3 and bm.shape[0] == H and bm.shape[1] == bm.shape[2]
        nbm, S_, L_, d = bm.shape[1], 0, 0, None
    else:
        bm, nbm, S_, L_, d = None, 0, int(S), int(L), _dense(H, dense_heads)
    dq = np.empty((batch, H, seq, D), dtype=np.float64)
    dk = np.empty((batch, Hkv, seq, D), dtype=np.float64)
    dv = np.empty_like(dk)
    rc = _load().s2o_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), batch, H, Hkv, seq, D, B, S_,
                              L_, _ptr(d), nbm, _ptr(bm), float(scale), _ptr(dq), _ptr(dk),
                              _ptr(dv), int(nthreads))
    if rc != 0:
        raise ValueError("oracle backward rejected its arguments")
    return dq, dk, dv


def backward_sampled(q, k, v, dout, B, scale, planes, qrows, krows, S=None, L=None,
                     dense_heads=None, bmask=None, nthreads=0):
    """Oracle gradients of ``backward`` for chosen rows only.

    planes: K/V plane ids b * Hkv + g. qrows: query rows hh * seq + t of each
    plane's group (query head g * (H / Hkv) + hh, position t). krows: key
    positions. Returns dq [n_planes, len(qrows), D] and dk, dv
    [n_planes, len(krows), D] (fp64): the same numbers as the full backward's
    rows, at the cost of the sampled planes' rows from the smallest sampled
    position on.
    """
    q, k, v, do = _bits(q), _bits(k), _bits(v), _bits(dout)
    batch, H, seq, D = q.shape
    Hkv = k.shape[1]
    assert k.shape == (batch, Hkv, seq, D) and v.shape == k.shape and do.shape == q.shape
    if bmask is not None:
        bm = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
        assert bm.ndim == 3 and bm.shape[0] == H and bm.shape[1] == bm.shape[2]
        nbm, S_, L_, d = bm.shape[1], 0, 0, None
    else:
        bm, nbm, S_, L_, d = None, 0, int(S), int(L), _dense(H, dense_heads)
    a = lambda x: np.ascontiguousarray(np.asarray(x, dtype=np.int64).reshape(-1))
    pl, qr, kr = a(planes), a(qrows), a(krows)
    dq = np.zeros((pl.size, qr.size, D), dtype=np.float64)
    dk = np.zeros((pl.size, kr.size, D), dtype=np.float64)
    dv = np.zeros_like(dk)
    rc = _load().s2o_backward_sampled(_ptr(q), _ptr(k), _ptr(v), _ptr(do), batch, H, Hkv, seq, D, B,
                                      S_, L_, _ptr(d), nbm, _ptr(bm), float(scale), pl.size,
                                      _ptr(pl), qr.size, _ptr(qr) if qr.size else None, kr.size,
                                      _ptr(kr) if kr.size else None, _ptr(dq), _ptr(dk), _ptr(dv),
                                      int(nthreads))
    if rc != 0:
        raise ValueError("oracle backward_sampled rejected its arguments")
    return dq, dk, dv


def chunk(q, k_cache, v_cache, block_table, ctx_lens, q_start, B, scale, S=None, L=None,
          dense_heads=None, bmask=None, nthreads=0):
    """Oracle chunked prefill over a paged cache.

    q: [total_q, H, D] packed chunk rows (sequence s owns rows
    q_start[s]..q_start[s+1]-1, the last tokens of its ctx_lens[s]-token
    context); caches [pages, Hkv, page_size, D]. Returns (out [total_q, H, D],
    lse [total_q, H]).
    """
    q, kc, vc = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(ctx_lens, dtype=np.int32))
    qs = np.ascontiguousarray(np.asarray(q_start, dtype=np.int32))
    total_q, H, D = q.shape
    _, Hkv, page_size, D2 = kc.shape
    assert D2 == D and vc.shape == kc.shape and qs[-1] == total_q
    batch = cl.size
    if bmask is not None:
        bm = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
        nbm, S_, L_, d = bm.shape[1], 0, 0, None
    else:
        bm, nbm, S_, L_, d = None, 0, int(S), int(L), _dense(H, dense_heads)
    out = np.zeros((total_q, H, D), dtype=np.float64)
    lse = np.empty((total_q, H), dtype=np.float64)
    rc = _load().s2o_chunk_rows(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cl), _ptr(qs), batch, H,
                                Hkv, D, page_size, bt.shape[1], B, S_, L_, _ptr(d), nbm, _ptr(bm),
                                float(scale), _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle chunk rejected its arguments")
    return out, lse
