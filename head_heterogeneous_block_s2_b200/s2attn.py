"""Thin ctypes binding of libs2attn.so (argument marshalling only).

Every step of the attention path runs in the library's CUDA kernels; this
module checks tensor types, passes raw device pointers and the current torch
stream, and turns status codes into exceptions. There is no fallback: if the
library is missing or a call fails, it raises.

Entry points mirror the C ABI in ``include/s2attn.h``:
``build_layout``, ``build_layout_ranges``, ``build_layout_mask`` and
``Layout.transposed`` (host; the last also builds the backward's key tiles),
``prefill`` (grouped K/V heads when k, v have fewer heads), ``backward``,
``chunk_prefill``, ``decode``, ``decode_noalloc``, ``decode_workspace_size``,
``backward_workspace_size``, ``device_status`` and ``set_wait_timeout_ns``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libs2attn.so")

S2_OK = 0
STATUS_NAMES = {0: "S2_OK", 1: "S2_ERR_INVALID_ARG", 2: "S2_ERR_UNSUPPORTED", 3: "S2_ERR_CAPACITY",
                4: "S2_ERR_CUDA", 5: "S2_ERR_TIMEOUT", 6: "S2_ERR_DEVICE_INDEX"}

EXPORTED = ("s2_status_string", "s2_build_layout", "s2_build_layout_ranges",
            "s2_build_layout_mask", "s2_build_layout_transpose", "s2_attn_prefill",
            "s2_attn_prefill_gqa", "s2_attn_decode_gqa", "s2_attn_backward",
            "s2_attn_backward_workspace_size", "s2_build_key_tiles", "s2_attn_chunk_prefill",
            "s2_attn_decode_workspace_size", "s2_attn_decode_auto_splits", "s2_attn_decode",
            "s2_device_status", "s2_set_wait_timeout_ns", "s2_version", "s2_attn_decode_noalloc")


class S2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class _LayoutDesc(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("vertical_stride", ctypes.c_int32), ("local_blocks", ctypes.c_int32),
                ("num_blocks", ctypes.c_int32), ("dense_head_mask", ctypes.c_void_p)]


class _ContextRange(ctypes.Structure):
    _fields_ = [("end_block", ctypes.c_int32), ("vertical_stride", ctypes.c_int32),
                ("local_blocks", ctypes.c_int32), ("dense", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} not found: build it with "
                      "`python -m head_heterogeneous_block_s2_b200.build`")
    lib = ctypes.CDLL(path)
    i32, i64, vp, f32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
    lib.s2_status_string.restype = ctypes.c_char_p
    lib.s2_status_string.argtypes = [ctypes.c_int]
    lib.s2_version.restype = ctypes.c_char_p
    lib.s2_version.argtypes = []
    lib.s2_build_layout.restype = ctypes.c_int
    lib.s2_build_layout.argtypes = [ctypes.POINTER(_LayoutDesc), vp, vp, i64, ctypes.POINTER(i64)]
    lib.s2_build_layout_ranges.restype = ctypes.c_int
    lib.s2_build_layout_ranges.argtypes = [i32, i32, vp, vp, vp, vp, i64, ctypes.POINTER(i64)]
    lib.s2_build_layout_mask.restype = ctypes.c_int
    lib.s2_build_layout_mask.argtypes = [i32, i32, vp, vp, vp, i64, ctypes.POINTER(i64)]
    lib.s2_attn_prefill.restype = ctypes.c_int
    lib.s2_attn_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, i32, vp, vp,
                                    i64, vp]
    lib.s2_build_layout_transpose.restype = ctypes.c_int
    lib.s2_build_layout_transpose.argtypes = [i32, i32, vp, vp, i64, vp, vp]
    lib.s2_build_key_tiles.restype = ctypes.c_int
    lib.s2_build_key_tiles.argtypes = [i32, i32, vp, vp]
    lib.s2_attn_backward_workspace_size.restype = sz
    lib.s2_attn_backward_workspace_size.argtypes = [i32, i32, i32]
    lib.s2_attn_backward.restype = ctypes.c_int
    lib.s2_attn_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                     f32, i32, i32, vp, vp, vp, vp, vp, i64, vp, sz, vp]
    lib.s2_attn_prefill_gqa.restype = ctypes.c_int
    lib.s2_attn_prefill_gqa.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, i32,
                                        vp, vp, i64, vp]
    lib.s2_attn_decode_gqa.restype = ctypes.c_int
    lib.s2_attn_decode_gqa.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i32,
                                       i32, vp, vp, i64, f32, vp, vp, vp, sz, i32, vp]
    lib.s2_attn_chunk_prefill.restype = ctypes.c_int
    lib.s2_attn_chunk_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64,
                                          i32, i64, i32, i32, vp, vp, i64, f32, vp, vp, vp]
    lib.s2_attn_decode_workspace_size.restype = sz
    lib.s2_attn_decode_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.s2_attn_decode_auto_splits.restype = i32
    lib.s2_attn_decode_auto_splits.argtypes = [i32, i32]
    lib.s2_attn_decode.restype = ctypes.c_int
    lib.s2_attn_decode.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64, i32, i32, vp,
                                   vp, i64, f32, vp, vp, vp, sz, i32, vp]
    lib.s2_attn_decode_noalloc.restype = ctypes.c_int
    lib.s2_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64, i32,
                                           i32, vp, vp, i64, f32, vp, vp, i32, vp]
    lib.s2_device_status.restype = ctypes.c_int
    lib.s2_device_status.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]
    lib.s2_set_wait_timeout_ns.restype = ctypes.c_int
    lib.s2_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != S2_OK:
        raise S2Error(rc, what)


# ------------------------------------------------------------------ layout

@dataclasses.dataclass
class Layout:
    """Per-head compacted key-block lists (CSR) of one layout.

    ``pattern`` says which builder made it: "hhst" (stride, local and
    dense_heads are its parameters), "ranges" (``ranges`` holds the per-head
    context ranges) or "mask"."""
    heads: int
    block_size: int
    stride: int
    local: int
    num_blocks: int
    dense_heads: Tuple[int, ...]
    row_ptr: np.ndarray  # int32 [heads * (num_blocks + 1)]
    col_idx: np.ndarray  # int32 [nnz]
    d_row_ptr: Optional[torch.Tensor] = None
    d_col_idx: Optional[torch.Tensor] = None
    pattern: str = "hhst"
    ranges: Optional[Tuple[Tuple[Tuple[int, int, int, bool], ...], ...]] = None
    # transposed lists (query blocks listing each key block), for the backward
    t_col_ptr: Optional[np.ndarray] = None
    t_row_idx: Optional[np.ndarray] = None
    t_key_tiles: Optional[np.ndarray] = None  # [heads, ceil(nb / 2), 2] (s2_build_key_tiles)
    d_t_col_ptr: Optional[torch.Tensor] = None
    d_t_row_idx: Optional[torch.Tensor] = None
    d_t_key_tiles: Optional[torch.Tensor] = None

    def transposed(self, device=None) -> "Layout":
        """Build (once) the transposed lists (s2_build_layout_transpose) and the
        backward's key tiles (s2_build_key_tiles), and copy them to ``device``."""
        if self.t_col_ptr is None:
            lib = load()
            self.t_col_ptr = np.zeros(self.heads * (self.num_blocks + 1), dtype=np.int32)
            self.t_row_idx = np.zeros(max(1, self.nnz), dtype=np.int32)
            _check(lib.s2_build_layout_transpose(
                self.heads, self.num_blocks, self.row_ptr.ctypes.data,
                self.col_idx.ctypes.data if self.nnz else None, self.nnz,
                self.t_col_ptr.ctypes.data, self.t_row_idx.ctypes.data), "s2_build_layout_transpose")
            self.t_key_tiles = np.zeros((self.heads, (self.num_blocks + 1) // 2, 2), dtype=np.int32)
            _check(lib.s2_build_key_tiles(self.heads, self.num_blocks, self.t_col_ptr.ctypes.data,
                                          self.t_key_tiles.ctypes.data), "s2_build_key_tiles")
        if device is not None and (self.d_t_col_ptr is None or self.d_t_col_ptr.device != torch.device(device)):
            self.d_t_col_ptr = torch.from_numpy(self.t_col_ptr).to(device)
            self.d_t_row_idx = torch.from_numpy(self.t_row_idx).to(device)
            self.d_t_key_tiles = torch.from_numpy(self.t_key_tiles).to(device)
        return self

    @property
    def nnz(self) -> int:
        return int(self.col_idx.size)

    def row(self, h: int, i: int) -> np.ndarray:
        base = h * (self.num_blocks + 1)
        return self.col_idx[self.row_ptr[base + i]:self.row_ptr[base + i + 1]]

    def to(self, device) -> "Layout":
        self.d_row_ptr = torch.from_numpy(self.row_ptr).to(device)
        # an empty layout still gets a (never read) one-element buffer
        col = self.col_idx if self.col_idx.size else np.zeros(1, dtype=np.int32)
        self.d_col_idx = torch.from_numpy(col).to(device)
        return self


def _desc(heads, block_size, stride, local, num_blocks, dense_heads):
    mask = None
    keep = None
    if dense_heads:
        keep = (ctypes.c_uint8 * heads)()
        for h in dense_heads:
            keep[int(h)] = 1
        mask = ctypes.cast(keep, ctypes.c_void_p)
    d = _LayoutDesc(heads, block_size, stride, local, num_blocks, mask)
    return d, keep


def layout_nnz(heads, block_size, stride, local, num_blocks, dense_heads=()) -> int:
    d, _keep = _desc(heads, block_size, stride, local, num_blocks, dense_heads)
    nnz = ctypes.c_int64(0)
    _check(load().s2_build_layout(ctypes.byref(d), None, None, 0, ctypes.byref(nnz)),
           "s2_build_layout")
    return nnz.value


def build_layout(heads: int, block_size: int, stride: int, local: int, num_blocks: int,
                 dense_heads: Sequence[int] = (), device=None) -> Layout:
    """Run s2_build_layout (host) and optionally copy the arrays to ``device``."""
    lib = load()
    d, _keep = _desc(heads, block_size, stride, local, num_blocks, dense_heads)
    nnz = ctypes.c_int64(0)
    _check(lib.s2_build_layout(ctypes.byref(d), None, None, 0, ctypes.byref(nnz)), "s2_build_layout")
    row_ptr = np.zeros(heads * (num_blocks + 1), dtype=np.int32)
    col_idx = np.zeros(max(1, nnz.value), dtype=np.int32)
    _check(lib.s2_build_layout(ctypes.byref(d), row_ptr.ctypes.data, col_idx.ctypes.data,
                               col_idx.size, ctypes.byref(nnz)), "s2_build_layout")
    lay = Layout(heads, block_size, stride, local, num_blocks, tuple(int(h) for h in dense_heads),
                 row_ptr, col_idx[:nnz.value].copy())
    if device is not None:
        lay.to(device)
    return lay


def _two_call(fn, heads: int, num_blocks: int, what: str):
    """Run a builder twice (count, then fill) and return (row_ptr, col_idx)."""
    nnz = ctypes.c_int64(0)
    _check(fn(None, None, 0, ctypes.byref(nnz)), what)
    row_ptr = np.zeros(heads * (num_blocks + 1), dtype=np.int32)
    col_idx = np.zeros(max(1, nnz.value), dtype=np.int32)
    _check(fn(row_ptr.ctypes.data, col_idx.ctypes.data, col_idx.size, ctypes.byref(nnz)), what)
    return row_ptr, col_idx[:nnz.value].copy()


def build_layout_ranges(ranges: Sequence[Sequence[Tuple[int, int, int, bool]]], block_size: int,
                        num_blocks: int, device=None) -> Layout:
    """Run s2_build_layout_ranges (host).

    ``ranges[h]`` lists head h's context ranges as (end_block, stride, local,
    dense) tuples, ends ascending, the last equal to ``num_blocks``; key block
    j follows the range that holds it."""
    lib = load()
    heads = len(ranges)
    ptr = np.zeros(heads + 1, dtype=np.int32)
    flat = []
    for h, head in enumerate(ranges):
        for (e, st, lo, dn) in head:
            flat.append((int(e), int(st), int(lo), int(bool(dn))))
        ptr[h + 1] = len(flat)
    arr = (_ContextRange * max(1, len(flat)))(*[_ContextRange(*t) for t in flat])

    def fn(rp, ci, cap, nnz):
        return lib.s2_build_layout_ranges(heads, num_blocks, ptr.ctypes.data,
                                          ctypes.cast(arr, ctypes.c_void_p), rp, ci, cap, nnz)

    row_ptr, col_idx = _two_call(fn, heads, num_blocks, "s2_build_layout_ranges")
    frozen = tuple(tuple((int(e), int(st), int(lo), bool(dn)) for (e, st, lo, dn) in head)
                   for head in ranges)
    lay = Layout(heads, block_size, 0, 0, num_blocks, (), row_ptr, col_idx, pattern="ranges",
                 ranges=frozen)
    if device is not None:
        lay.to(device)
    return lay


def build_layout_mask(block_mask: np.ndarray, block_size: int, device=None) -> Layout:
    """Run s2_build_layout_mask (host) on a [heads, nb, nb] mask (nonzero = active)."""
    lib = load()
    m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    if m.ndim != 3 or m.shape[1] != m.shape[2]:
        raise ValueError("block_mask must be [heads, num_blocks, num_blocks]")
    heads, num_blocks = int(m.shape[0]), int(m.shape[1])

    def fn(rp, ci, cap, nnz):
        return lib.s2_build_layout_mask(heads, num_blocks, m.ctypes.data, rp, ci, cap, nnz)

    row_ptr, col_idx = _two_call(fn, heads, num_blocks, "s2_build_layout_mask")
    lay = Layout(heads, block_size, 0, 0, num_blocks, (), row_ptr, col_idx, pattern="mask")
    if device is not None:
        lay.to(device)
    return lay


# ------------------------------------------------------------------ kernels

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: Layout,
            scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None, want_lse: bool = False):
    """s2_attn_prefill on [batch, heads, seq, head_dim] bf16 CUDA tensors.

    k and v may have fewer heads (grouped K/V heads, s2_attn_prefill_gqa):
    [batch, heads_kv, seq, head_dim] with heads_kv dividing heads.
    Returns out, or (out, lse) when ``want_lse`` or ``lse`` is given."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    batch, heads, seq, hd = q.shape
    hkv = k.shape[1]
    if k.shape != (batch, hkv, seq, hd) or v.shape != k.shape or heads % hkv:
        raise ValueError("k, v must be [batch, heads_kv, seq, head_dim] with heads_kv | heads")
    if layout.heads != heads:
        raise ValueError(f"layout has {layout.heads} heads, q has {heads}")
    if layout.d_row_ptr is None:
        layout.to(q.device)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out")
    if lse is None and want_lse:
        lse = torch.empty((batch, heads, seq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    sc = 0.0 if scale is None else float(scale)  # 0: the library uses 1/sqrt(head_dim)
    if hkv == heads:
        rc = load().s2_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), batch, heads,
                                    seq, hd, sc, layout.block_size, layout.num_blocks,
                                    _ptr(layout.d_row_ptr), _ptr(layout.d_col_idx), layout.nnz,
                                    _stream(q.device))
        _check(rc, "s2_attn_prefill")
    else:
        rc = load().s2_attn_prefill_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), batch,
                                        heads, hkv, seq, hd, sc, layout.block_size,
                                        layout.num_blocks, _ptr(layout.d_row_ptr),
                                        _ptr(layout.d_col_idx), layout.nnz, _stream(q.device))
        _check(rc, "s2_attn_prefill_gqa")
    return (out, lse) if lse is not None else out


def backward_workspace_size(batch: int, heads: int, seq: int) -> int:
    return int(load().s2_attn_backward_workspace_size(batch, heads, seq))


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, layout: Layout,
             scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
             dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None):
    """s2_attn_backward: gradients (dq, dk, dv) of ``prefill`` for the upstream
    gradient ``dout``, given the forward's output ``o`` and ``lse``. k and v
    may have fewer heads (grouped K/V heads): dk and dv then sum over each K/V
    head's query heads."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n)
    _need(lse, "lse", torch.float32)
    batch, heads, seq, hd = q.shape
    hkv = k.shape[1]
    if k.shape != (batch, hkv, seq, hd) or v.shape != k.shape or heads % hkv:
        raise ValueError("k, v must be [batch, heads_kv, seq, head_dim] with heads_kv | heads")
    for t, n in ((o, "o"), (dout, "dout")):
        if t.shape != q.shape:
            raise ValueError(f"{n} shape differs from q")
    if lse.shape != (batch, heads, seq):
        raise ValueError("lse must be [batch, heads, seq]")
    if layout.heads != heads:
        raise ValueError(f"layout has {layout.heads} heads, q has {heads}")
    if layout.d_row_ptr is None:
        layout.to(q.device)
    layout.transposed(q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, n)
    ws_bytes = backward_workspace_size(batch, heads, seq)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_len = workspace.numel() * workspace.element_size()
    sc = 0.0 if scale is None else float(scale)  # 0: the library uses 1/sqrt(head_dim)
    rc = load().s2_attn_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), batch, heads, hkv, seq, hd, sc,
                                 layout.block_size, layout.num_blocks, _ptr(layout.d_row_ptr),
                                 _ptr(layout.d_col_idx), _ptr(layout.d_t_col_ptr),
                                 _ptr(layout.d_t_row_idx), _ptr(layout.d_t_key_tiles), layout.nnz,
                                 _ptr(workspace), ws_len,
                                 _stream(q.device))
    _check(rc, "s2_attn_backward")
    return dq, dk, dv


def chunk_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_table: torch.Tensor, ctx_lens: torch.Tensor, q_start: torch.Tensor,
                  layout: Layout, max_q_len: int, scale: Optional[float] = None,
                  out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  want_lse: bool = False):
    """s2_attn_chunk_prefill: q [total_q, heads, D] packed chunk rows; caches
    [pages, heads_kv, 16, D]; block_table int32 [batch, max_pages]; ctx_lens
    int32 [batch] (contexts including the chunks); q_start int32 [batch + 1]
    (all CUDA). ``max_q_len`` bounds the chunk lengths."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n)
    for t, n in ((block_table, "block_table"), (ctx_lens, "ctx_lens"), (q_start, "q_start")):
        _need(t, n, torch.int32)
    total_q, heads, hd = q.shape
    num_pages, hkv, page_size, hd2 = k_cache.shape
    if heads % hkv or hd2 != hd or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape does not match q")
    batch = ctx_lens.numel()
    if q_start.numel() != batch + 1:
        raise ValueError("q_start must have batch + 1 entries")
    if layout.heads != heads:
        raise ValueError(f"layout has {layout.heads} heads, q has {heads}")
    if layout.d_row_ptr is None:
        layout.to(q.device)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out")
    if lse is None and want_lse:
        lse = torch.empty((total_q, heads), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    sc = 0.0 if scale is None else float(scale)  # 0: the library uses 1/sqrt(head_dim)
    rc = load().s2_attn_chunk_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                      _ptr(ctx_lens), _ptr(q_start), batch, heads, hkv, hd, page_size,
                                      block_table.shape[1], num_pages, int(max_q_len), total_q,
                                      layout.block_size, layout.num_blocks, _ptr(layout.d_row_ptr),
                                      _ptr(layout.d_col_idx), layout.nnz, sc, _ptr(out), _ptr(lse),
                                      _stream(q.device))
    _check(rc, "s2_attn_chunk_prefill")
    return (out, lse) if lse is not None else out


def decode_auto_splits(batch: int, heads: int) -> int:
    return int(load().s2_attn_decode_auto_splits(batch, heads))


def decode_workspace_size(batch: int, heads: int, head_dim: int, num_splits: int = 0) -> int:
    return int(load().s2_attn_decode_workspace_size(batch, heads, head_dim, num_splits))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           block_table: torch.Tensor, ctx_lens: torch.Tensor, layout: Layout,
           scale: Optional[float] = None, num_splits: int = 0,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           want_lse: bool = False, workspace: Optional[torch.Tensor] = None):
    """s2_attn_decode: q [batch, heads, D]; caches [pages, heads_kv, 16, D]
    (heads_kv dividing heads; fewer heads = s2_attn_decode_gqa);
    block_table int32 [batch, max_pages]; ctx_lens int32 [batch] (all CUDA)."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n)
    _need(block_table, "block_table", torch.int32)
    _need(ctx_lens, "ctx_lens", torch.int32)
    batch, heads, hd = q.shape
    num_pages, h2, page_size, hd2 = k_cache.shape
    if heads % h2 or hd2 != hd or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape does not match q")
    if layout.heads != heads:
        raise ValueError(f"layout has {layout.heads} heads, q has {heads}")
    if layout.d_row_ptr is None:
        layout.to(q.device)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out")
    if lse is None and want_lse:
        lse = torch.empty((batch, heads), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    ws_bytes = decode_workspace_size(batch, heads, hd, num_splits)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    sc = 0.0 if scale is None else float(scale)  # 0: the library uses 1/sqrt(head_dim)
    if h2 == heads:
        rc = load().s2_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                   _ptr(ctx_lens), batch, heads, hd, page_size, block_table.shape[1],
                                   num_pages, layout.block_size, layout.num_blocks,
                                   _ptr(layout.d_row_ptr), _ptr(layout.d_col_idx), layout.nnz, sc,
                                   _ptr(out), _ptr(lse), _ptr(workspace), ws_len, num_splits,
                                   _stream(q.device))
        _check(rc, "s2_attn_decode")
    else:
        rc = load().s2_attn_decode_gqa(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                       _ptr(ctx_lens), batch, heads, h2, hd, page_size,
                                       block_table.shape[1], num_pages, layout.block_size,
                                       layout.num_blocks, _ptr(layout.d_row_ptr),
                                       _ptr(layout.d_col_idx), layout.nnz, sc, _ptr(out),
                                       _ptr(lse), _ptr(workspace), ws_len, num_splits,
                                       _stream(q.device))
        _check(rc, "s2_attn_decode_gqa")
    return (out, lse) if lse is not None else out


# Size of the library's built-in decode scratch (S2_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 8 << 20


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_table: torch.Tensor, ctx_lens: torch.Tensor, layout: Layout,
                   scale: Optional[float] = None, num_splits: int = 0,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   want_lse: bool = False):
    """s2_attn_decode_noalloc: decode for callers that cannot allocate device
    memory. The split partials go to the library's own built-in scratch, so no
    workspace is passed; ``out`` (and ``lse``) must be supplied by a caller
    that cannot allocate (they are only created here for convenience). Calls
    share that scratch, so calls that may overlap on the GPU must be ordered
    by the caller."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, n)
    _need(block_table, "block_table", torch.int32)
    _need(ctx_lens, "ctx_lens", torch.int32)
    batch, heads, hd = q.shape
    num_pages, h2, page_size, hd2 = k_cache.shape
    if h2 != heads or hd2 != hd or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape does not match q")
    if layout.heads != heads:
        raise ValueError(f"layout has {layout.heads} heads, q has {heads}")
    if layout.d_row_ptr is None:
        layout.to(q.device)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out")
    if lse is None and want_lse:
        lse = torch.empty((batch, heads), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    sc = 0.0 if scale is None else float(scale)  # 0: the library uses 1/sqrt(head_dim)
    rc = load().s2_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                       _ptr(ctx_lens), batch, heads, hd, page_size,
                                       block_table.shape[1], num_pages, layout.block_size,
                                       layout.num_blocks, _ptr(layout.d_row_ptr),
                                       _ptr(layout.d_col_idx), layout.nnz, sc, _ptr(out), _ptr(lse),
                                       num_splits, _stream(q.device))
    _check(rc, "s2_attn_decode_noalloc")
    return (out, lse) if lse is not None else out


def device_status(reset: bool = True) -> Tuple[int, int]:
    """(status, raw flags) after synchronising the current device."""
    flags = ctypes.c_uint32(0)
    rc = load().s2_device_status(1 if reset else 0, ctypes.byref(flags))
    return rc, flags.value


def set_wait_timeout_ns(ns: int):
    _check(load().s2_set_wait_timeout_ns(int(ns)), "s2_set_wait_timeout_ns")


def version() -> str:
    return load().s2_version().decode()
