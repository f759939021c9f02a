"""The C-ABI library loads without a GPU and exports every declared entry point.

Also checks host-side argument validation: calls with bad arguments return
an error status before touching any device. Those calls pass made-up device
addresses, so they run only on a machine without a GPU: there a call that got
past validation could not launch anything (it fails at the device check with
S2_ERR_CUDA), while on a GPU a validation slip would launch a kernel on a wild
address.
"""
import ctypes
import os
import re

import pytest
import torch

from head_heterogeneous_block_s2_b200 import s2attn

no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="passes made-up device addresses: CPU-only machines")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(s2_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = s2attn.load()
    names = declared_functions()
    assert "s2_attn_prefill" in names and "s2_attn_decode" in names and "s2_build_layout" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(s2attn.EXPORTED) <= set(names)


def test_status_strings_and_version():
    lib = s2attn.load()
    for code, name in s2attn.STATUS_NAMES.items():
        assert lib.s2_status_string(code).decode() == name
    assert lib.s2_status_string(99).decode() == "S2_ERR_UNKNOWN"
    assert "sm_100a" in s2attn.version()


def _prefill(**over):
    a = dict(q=1 << 20, k=1 << 20, v=1 << 20, o=1 << 20, lse=None, batch=1, heads=4, seq=512, hd=64,
             scale=0.125, bs=64, nb=8, row_ptr=1 << 20, col_idx=1 << 20, nnz=60)
    a.update(over)
    vp = ctypes.c_void_p
    return s2attn.load().s2_attn_prefill(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["o"]),
                                         vp(a["lse"]), a["batch"], a["heads"], a["seq"], a["hd"],
                                         a["scale"], a["bs"], a["nb"], vp(a["row_ptr"]),
                                         vp(a["col_idx"]), a["nnz"], None)


@no_gpu_only
@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(row_ptr=None), 1), (dict(batch=0), 1), (dict(seq=600), 1),
    (dict(nb=7), 1), (dict(hd=96), 2), (dict(bs=32), 2), (dict(q=(1 << 20) + 8), 1),
    (dict(scale=float("nan")), 1), (dict(nnz=-1), 1), (dict(col_idx=None), 1),
    (dict(scale=-0.125), 1),
])
def test_prefill_rejects_bad_arguments_before_launch(over, code):
    assert _prefill(**over) == code


@no_gpu_only
def test_zero_scale_selects_the_default_and_passes_validation():
    # 0 means 1/sqrt(head_dim): validation accepts it and the call reaches the
    # device check, which fails here for want of a GPU (S2_ERR_CUDA).
    assert _prefill(scale=0.0) == 4
    assert _decode(scale=0.0) == 4
    assert _decode(scale=-0.1) == 4  # decode takes any finite multiplier
    assert _decode(scale=float("inf")) == 1


def _decode(**over):
    a = dict(q=1 << 20, kc=1 << 20, vc=1 << 20, bt=1 << 20, cl=1 << 20, batch=2, heads=4, hd=128,
             page=16, max_pages=8, num_pages=16, bs=128, nb=1, rp=1 << 20, ci=1 << 20, nnz=4,
             scale=0.1, out=1 << 20, lse=None, ws=None, ws_bytes=0, splits=1)
    a.update(over)
    vp = ctypes.c_void_p
    return s2attn.load().s2_attn_decode(vp(a["q"]), vp(a["kc"]), vp(a["vc"]), vp(a["bt"]),
                                        vp(a["cl"]), a["batch"], a["heads"], a["hd"], a["page"],
                                        a["max_pages"], a["num_pages"], a["bs"], a["nb"],
                                        vp(a["rp"]), vp(a["ci"]), a["nnz"], a["scale"], vp(a["out"]),
                                        vp(a["lse"]), vp(a["ws"]), a["ws_bytes"], a["splits"], None)


@no_gpu_only
@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(bt=None), 1), (dict(page=32), 2), (dict(hd=80), 2),
    (dict(bs=24), 2), (dict(splits=2, ws=None), 1), (dict(splits=2, ws=1 << 20, ws_bytes=16), 3),
    (dict(splits=2, ws=(1 << 20) + 16, ws_bytes=1 << 20), 1), (dict(splits=1000), 1),
    (dict(nnz=-1), 1), (dict(ci=None), 1),
])
def test_decode_rejects_bad_arguments_before_launch(over, code):
    assert _decode(**over) == code


def test_decode_workspace_size():
    assert s2attn.decode_workspace_size(64, 32, 128, 1) == 0
    n = s2attn.decode_workspace_size(4, 8, 128, 4)
    assert n >= 4 * 8 * 4 * (128 + 2) * 4
    auto = s2attn.decode_auto_splits(4, 8)
    assert 1 <= auto <= 16
    assert s2attn.decode_workspace_size(4, 8, 128, 0) == s2attn.decode_workspace_size(4, 8, 128, auto)


def test_decode_auto_splits_is_about_one_resident_wave():
    # ceil(370 / (batch * heads)), clamped to [1, 16]: the measured best split
    # counts on 32 heads were 3, 2, 1, 1, 1 at batches 4, 8, 16, 32, 64
    assert [s2attn.decode_auto_splits(b, 32) for b in (4, 8, 16, 32, 64)] == [3, 2, 1, 1, 1]
    for b, h in ((1, 1), (1, 8), (2, 32), (3, 7), (300, 32), (65535, 64)):
        want = min(16, max(1, -(-370 // (b * h))))
        assert s2attn.decode_auto_splits(b, h) == want, (b, h)
    assert s2attn.decode_auto_splits(0, 32) == 1 and s2attn.decode_auto_splits(4, 0) == 1


@no_gpu_only
def test_grouped_head_entry_points_reject_bad_head_counts():
    lib = s2attn.load()
    vp = ctypes.c_void_p
    m = vp(1 << 20)
    # 4 query heads over 3 K/V heads; 0 K/V heads
    for hkv in (3, 0):
        assert lib.s2_attn_prefill_gqa(m, m, m, m, None, 1, 4, hkv, 512, 64, 0.125, 64, 8, m, m,
                                       60, None) == 1
        assert lib.s2_attn_decode_gqa(m, m, m, m, m, 2, 4, hkv, 128, 16, 8, 16, 128, 1, m, m, 4,
                                      0.1, m, None, None, 0, 1, None) == 1
