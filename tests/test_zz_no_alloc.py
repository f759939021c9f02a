"""s2_attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: plug-ins whose host
framework owns all device memory, C programs without a device allocator of
their own, and latency-critical loops that must not allocate (cudaMalloc and
cudaFree can synchronise the device). For them the library keeps the decode
split partials in its own built-in scratch array.

These tests call that entry point through the C ABI and check each result
against the fp64 oracle and against s2_attn_decode with a caller workspace,
over calls in a row on different inputs that share the scratch: a call with
more splits leaves partials at offsets a later call with fewer splits does
not write, and that later call must not read them. A shape too large for the
scratch is refused before anything runs.

This file is named to be collected last.
"""
import ctypes

import pytest
import torch

import oracle
from conftest import parity
from head_heterogeneous_block_s2_b200 import s2attn, synth

pytestmark = pytest.mark.gpu


def _case(seed, ctx):
    w = synth.DecodeWorkload("t", len(ctx), 8, 128, 1, 3000, 16, 128, 4, 2, seed=seed)
    d = synth.decode_inputs(w, ctx_lens=ctx)
    lay = s2attn.build_layout(w.heads, w.block, w.stride, w.local, -(-w.ctx_max // w.block),
                              device="cuda")
    return w, d, lay


def test_noalloc_decode_matches_oracle_and_workspace_decode_over_calls(s2gpu):
    # 7 splits, then 3 on other inputs (the scratch still holds the 7-split
    # partials), then 7 again: every call is checked on its own
    cases = [(_case(31, [1, 16, 17, 128, 129, 3000]), 7),
             (_case(32, [3000, 2999, 640, 5, 1000, 77]), 3),
             (_case(33, [2048, 1, 2900, 300, 129, 1500]), 7)]
    for (w, d, lay), splits in cases:
        args = (d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.block_table.cuda(),
                d.ctx_lens.cuda(), lay)
        got, got_lse = s2attn.decode_noalloc(*args, scale=w.scale, num_splits=splits,
                                             want_lse=True)
        torch.cuda.synchronize()
        want, want_lse = oracle.decode(d.q, d.k_cache, d.v_cache, d.block_table.numpy(),
                                       d.ctx_lens.numpy(), w.block, w.stride, w.local, w.scale)
        parity(got.reshape(-1, w.head_dim), want)
        parity(got_lse.reshape(-1), want_lse, max_tol=1e-3, mean_tol=1e-4)
        ref, ref_lse = s2attn.decode(*args, scale=w.scale, num_splits=splits, want_lse=True)
        torch.cuda.synchronize()
        parity(got.reshape(-1, w.head_dim), ref.double().cpu().numpy().reshape(-1, w.head_dim))
        parity(got_lse.reshape(-1), ref_lse.double().cpu().numpy().reshape(-1),
               max_tol=1e-3, mean_tol=1e-4)


def test_noalloc_decode_rejects_shapes_beyond_the_scratch(s2gpu):
    lib = s2attn.load()
    # 64 sequences x 32 heads x 64 splits of fp32 partials need ~68 MB > 8 MiB.
    # All pointers are NULL: the size check must refuse the call first, and if
    # it did not, the pointer check behind it would (nothing can launch).
    assert s2attn.decode_workspace_size(64, 32, 128, 64) > s2attn.NOALLOC_SCRATCH_BYTES
    rc = lib.s2_attn_decode_noalloc(None, None, None, None, None, 64, 32, 128, 16, 2048, 100, 128,
                                    256, None, None, 10, 0.1, None, None, 64, None)
    assert rc == 3  # S2_ERR_CAPACITY
