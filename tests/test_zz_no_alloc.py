"""s2_attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: plug-ins whose host
framework owns all device memory, C programs without a device allocator of
their own, and latency-critical loops that must not allocate (cudaMalloc and
cudaFree can synchronise the device). For them the library keeps the decode
split partials in its own built-in scratch array. These tests call that entry
point through the C ABI and check it against s2_attn_decode with a caller
workspace, twice in a row on different inputs (the scratch keeps the previous
call's contents), and check that a shape too large for the scratch is refused.

This file is named to be collected last.
"""
import ctypes

import pytest
import torch

from conftest import parity
from head_heterogeneous_block_s2_b200 import s2attn, synth

pytestmark = pytest.mark.gpu


def _case(seed, ctx):
    w = synth.DecodeWorkload("t", len(ctx), 8, 128, 1, 3000, 16, 128, 4, 2, seed=seed)
    d = synth.decode_inputs(w, ctx_lens=ctx)
    lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, -(-w.ctx_max // w.block),
                              device="cuda")
    return w, d, lay


@pytest.mark.parametrize("splits", [7, 3])
def test_noalloc_decode_matches_workspace_decode_twice(s2gpu, splits):
    cases = [_case(31, [1, 16, 17, 128, 129, 3000]), _case(32, [3000, 2999, 640, 5, 1000, 77])]
    for w, d, lay in cases:  # two calls in a row through the shared scratch
        args = (d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(),
                d.ctx_lens.cuda(), lay)
        ref, ref_lse = s2attn.decode(*args, scale=w.scale, num_splits=splits, want_lse=True)
        got, got_lse = s2attn.decode_noalloc(*args, scale=w.scale, num_splits=splits,
                                             want_lse=True)
        torch.cuda.synchronize()
        parity(got.reshape(-1, w.head_dim), ref.double().cpu().numpy().reshape(-1, w.head_dim))
        parity(got_lse.reshape(-1), ref_lse.double().cpu().numpy().reshape(-1),
               max_tol=1e-3, mean_tol=1e-4)


def test_noalloc_decode_rejects_shapes_beyond_the_scratch(s2gpu):
    lib = s2attn.load()
    vp = ctypes.c_void_p
    # 64 sequences x 32 heads x 64 splits of fp32 partials need ~68 MB > 8 MiB
    assert s2attn.decode_workspace_size(64, 32, 128, 64) > s2attn.NOALLOC_SCRATCH_BYTES
    rc = lib.s2_attn_decode_noalloc(vp(1 << 20), vp(1 << 20), vp(1 << 20), vp(1 << 20),
                                    vp(1 << 20), 64, 32, 128, 16, 2048, 100, 128, 256,
                                    vp(1 << 20), vp(1 << 20), 10, 0.1, vp(1 << 20), None, 64, None)
    assert rc == 3  # S2_ERR_CAPACITY, nothing launched
