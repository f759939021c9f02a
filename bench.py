#!/usr/bin/env python3
"""Benchmark of the HHST sparse-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * prefill (block-sparse attention, tcgen05 kernel) over the 1.3B-shaped
    layer batch: batch 4, 16 heads, head_dim 128, seq 8192, B 64, S 8, L 2,
    per-head K scale U(0.5, 2);
  * decode (split-KV paged kernel + combine) over 64 sequences, 32 heads,
    head_dim 128, contexts U[4096, 32768], 16-token pages, permuted block table,
    B 128, S 16, L 4.
The layouts are built once (host, per layout) before timing. After the W
warm-up steps, untimed steps run for --settle-s seconds: the GPU reaches its
power cap within ~0.1 s of sustained load, and the timed region is divided
by the sustained tensor peak, so it is timed in that same state.

Headline: prefill effective TFLOP/s (4 * head_dim per visible (query, key)
pair; the dense work the pattern skips is not counted), from CUDA events around
the prefill launches inside the timed steps. The decode part reports active
K+V GB/s and tokens/s in "decode". Multi-GPU: one process per GPU, each
processing its own batch (weak scaling, no collective on the data path);
time = max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HHST sparse attn fwd effective TFLOP/s & % bf16 TC peak; decode KV GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------- work counts

def prefill_flops(lay, w) -> int:
    """Algorithmic FLOPs: 4*D per visible (q, k) pair. A non-diagonal active
    block holds B*B pairs, a diagonal block B*(B+1)/2."""
    nnz = int(lay.col_idx.size)
    rows = lay.heads * lay.num_blocks  # every row holds exactly one diagonal block
    B = w.block
    pairs = (nnz - rows) * B * B + rows * B * (B + 1) // 2
    return 4 * w.head_dim * pairs * w.batch


def prefill_issued_flops(lay, w) -> int:
    """FLOPs of the layout's whole blocks (nnz * B * B pairs)."""
    return 4 * w.head_dim * w.block * w.block * int(lay.col_idx.size) * w.batch


def prefill_mma_flops(lay, w) -> int:
    """FLOPs the prefill kernel's MMAs compute. A 128-row tile visits every
    key block that any of its query blocks lists: with B = 128 that is its one
    row's list (= the whole-block count); with B = 64 it is the union of two
    consecutive rows' lists, computed for all 128 rows."""
    if w.block == 128:
        return prefill_issued_flops(lay, w)
    rp, ci, nb = lay.row_ptr, lay.col_idx, lay.num_blocks
    per = 128 // w.block
    visits = 0
    for h in range(lay.heads):
        for i0 in range(0, nb, per):
            u = set()
            for i in range(i0, min(i0 + per, nb)):
                u.update(ci[rp[h * (nb + 1) + i]: rp[h * (nb + 1) + i + 1]].tolist())
            visits += len(u)
    return 4 * w.head_dim * 128 * w.block * visits * w.batch


def decode_counts(lay, w, ctx_lens):
    """(active tokens over all (seq, head), pages touched) for the batch."""
    tokens = pages = 0
    B = w.block
    for n in ctx_lens:
        n = int(n)
        i = (n - 1) // B
        for h in range(w.heads):
            base = h * (lay.num_blocks + 1)
            for j in lay.col_idx[lay.row_ptr[base + i]:lay.row_ptr[base + i + 1]]:
                t0, t1 = int(j) * B, min((int(j) + 1) * B, n)
                tokens += t1 - t0
                pages += -(-(t1 - t0) // 16)
    return tokens, pages


def chunk_flops(lay, w, ctx_lens, qlens) -> int:
    """Algorithmic FLOPs of a chunked prefill: 4*D per visible (chunk row, key)
    pair, a row at position pos seeing B keys of each listed block below its own
    block and pos - i*B + 1 keys of its own block i when listed."""
    H, nb, B = lay.heads, lay.num_blocks, w.block
    nfull = np.zeros((H, nb), dtype=np.int64)
    diag = np.zeros((H, nb), dtype=np.int64)
    for h in range(H):
        for i in range(nb):
            r = lay.row(h, i)
            nfull[h, i] = int((r < i).sum())
            diag[h, i] = int((r == i).any())
    pairs = 0
    for n, ql in zip(ctx_lens, qlens):
        c0 = n - ql
        for i in range(c0 // B, (n - 1) // B + 1 if ql else 0):
            a, b = max(c0, i * B), min(n, (i + 1) * B)
            rows = b - a
            tri = (a - i * B + 1 + b - i * B) * rows // 2  # sum of pos - iB + 1 over the rows
            pairs += int((rows * nfull[:, i] * B + diag[:, i] * tri).sum())
    return 4 * w.head_dim * pairs


# Sources each kernel is compiled from (its ncu traffic figure stays valid while
# these files are unchanged).
KERNEL_SOURCES = {
    "s2_prefill_pair_kernel": ("prefill_pair_sm100.cuh", "lists.cuh", "ptx.cuh", "umma.cuh"),
    "s2_decode_split_kernel": ("decode.cuh", "ptx.cuh"),
    "s2_bwd": ("backward_sm100.cuh", "lists.cuh", "ptx.cuh", "umma.cuh"),
    "s2_chunk_prefill_kernel": ("chunk_sm100.cuh", "lists.cuh", "ptx.cuh", "umma.cuh"),
}


def source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "head_heterogeneous_block_s2_b200", "csrc")
    for fn in sorted(KERNEL_SOURCES[kernel]):
        h.update(fn.encode())
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def settle(fn, seconds, dist, device, sync=None):
    """Run fn (one untimed step) until `seconds` of wall time have passed, in
    batches with a device sync after each, so that the clocks and power state
    seen by the timed region are the sustained ones. Ranks agree on the count
    (max over ranks), so every rank runs the same number of steps. Returns it."""
    import torch

    if sync is None:
        def sync():
            torch.cuda.synchronize(device)
    if seconds <= 0:
        return 0
    n, batch, t0 = 0, 4, time.time()
    while time.time() - t0 < seconds:
        for _ in range(batch):
            fn()
        n += batch
        sync()
        batch = min(batch * 2, 256)
    if dist is not None:
        t = torch.tensor([n], dtype=torch.int64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        for _ in range(int(t.item()) - n):
            fn()
        n = int(t.item())
        sync()
    return n


def max_over_ranks(vals, dist, device):
    """Element-wise maximum of per-rank timings (one all-reduce; identity on
    one process). Every rank must call it, with the same number of values."""
    if dist is None:
        return list(vals)
    import torch

    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha") != source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read-only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            log(f"clock sampling unavailable: {e}")

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((time.time(), mhz, rs, util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t_on=None, t_off=None):
        """Median SM clock and the reasons seen over the samples taken between
        t_on and t_off (the timed region; the sampler also runs through the
        warm-up so that NVML's readings are current when the region starts)."""
        samples = self.samples
        if t_on is not None:
            inside = [s for s in samples if t_on <= s[0] <= t_off]
            # a region shorter than the period: the samples nearest to it
            samples = inside or sorted(samples, key=lambda s: abs(s[0] - t_on))[:2]
        if not self.ok or not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        loaded = [s for s in samples if not (s[2] & 0x1)] or samples
        reasons = set()
        for _, _, rs, _ in loaded:
            for bit, name in self.REASONS.items():
                if rs & bit and bit != 0x1:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(loaded)}


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, dist):
    import torch

    from head_heterogeneous_block_s2_b200 import s2attn, synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    s2attn.load()
    wp = synth.PREFILL_WORKLOADS[args.prefill]
    wd = synth.DECODE_WORKLOADS[args.decode] if args.decode != "none" else None
    if wd is not None and args.decode_batch > 0:
        wd = wd.with_(batch=args.decode_batch)

    # setup (untimed): inputs resident in HBM, layouts built once per layout
    t0 = time.time()
    q, k, v = synth.prefill_inputs(wp, device=dev)
    lay_p = s2attn.build_layout(wp.heads, wp.block, wp.stride, wp.local, wp.num_blocks,
                                wp.dense_heads, device=dev)
    layout_ms = None
    t1 = time.time()
    _ = s2attn.build_layout(wp.heads, wp.block, wp.stride, wp.local, wp.num_blocks, wp.dense_heads)
    layout_ms = (time.time() - t1) * 1e3
    out = torch.empty_like(q)
    flops = prefill_flops(lay_p, wp)
    issued = prefill_issued_flops(lay_p, wp)
    mma = prefill_mma_flops(lay_p, wp)
    if wd is not None:
        d = synth.decode_inputs(wd, device=dev)
        nb_d = -(-wd.ctx_max // wd.block)
        lay_d = s2attn.build_layout(wd.heads, wd.block, wd.stride, wd.local, nb_d, wd.dense_heads,
                                    device=dev)
        splits = args.splits if args.splits > 0 else s2attn.decode_auto_splits(wd.batch, wd.heads)
        ws_n = s2attn.decode_workspace_size(wd.batch, wd.heads, wd.head_dim, splits)
        ws = torch.empty(max(ws_n, 256), dtype=torch.uint8, device=dev)
        dout = torch.empty_like(d.q)
        ctx_host = d.ctx_lens.cpu().numpy()
        tokens, pages = decode_counts(lay_d, wd, ctx_host)
        kv_bytes = tokens * wd.head_dim * 2 * 2
        kv_page_bytes = pages * 16 * wd.head_dim * 2 * 2
    torch.cuda.synchronize()
    log(f"[rank {rank}] setup {time.time() - t0:.1f}s; prefill {flops / 1e9:.1f} GFLOP/step"
        + (f"; decode {kv_bytes / 1e9:.3f} GB active KV, splits {splits}" if wd else ""))

    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        s2attn.prefill(q, k, v, lay_p, scale=wp.scale, out=out)
        if evs:
            evs[1].record(stream)
        if wd is not None:
            s2attn.decode(d.q, d.k_cache, d.v_cache, d.block_table, d.ctx_lens, lay_d,
                          scale=wd.scale, num_splits=splits, out=dout, workspace=ws)
        if evs:
            evs[2].record(stream)

    sampler = ClockSampler(dev.index)
    sampler.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    settle_steps = settle(step, args.settle_s, dist, dev)
    rc, flags = s2attn.device_status(reset=True)
    if rc != 0:
        raise RuntimeError(f"device flags {flags:#x} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t_on = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    t_off = time.time()
    if dist:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs) if wd else 0.0
    rc, flags = s2attn.device_status(reset=True)
    if rc != 0:
        raise RuntimeError(f"device flags {flags:#x} after timing")

    # ---------------- end to end through the public API with host buffers
    # Prefill leg, pipelined like a serving loop: every step copies its Q, K, V
    # from pinned host memory and reads its output back, on two copy streams
    # with double-buffered device tensors, so step i+1's uploads overlap step
    # i's prefill and download. Decode leg: one stream, step after step.
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, args.e2e_steps))
    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    hout = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    gq = [torch.empty_like(q) for _ in range(2)]
    gk = [torch.empty_like(k) for _ in range(2)]
    gv = [torch.empty_like(v) for _ in range(2)]
    gout = [torch.empty_like(out) for _ in range(2)]
    h2d_pre = 3 * q.numel() * q.element_size()
    d2h_pre = out.numel() * out.element_size()
    s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]  # the slot's D2H (so also its prefill) is done
    if wd is not None:
        hdq = d.q.cpu().pin_memory()
        hbt = d.block_table.cpu().pin_memory()
        hcl = d.ctx_lens.cpu().pin_memory()
        hdout = torch.empty(d.q.shape, dtype=d.q.dtype).pin_memory()
        gdq, gbt, gcl = torch.empty_like(d.q), torch.empty_like(d.block_table), torch.empty_like(d.ctx_lens)
        h2d_dec = sum(t.numel() * t.element_size() for t in (hdq, hbt, hcl))
        d2h_dec = hdout.numel() * hdout.element_size()

    def e2e_prefill(i):
        b = i & 1
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(ev_free[b])
            gq[b].copy_(hq, non_blocking=True)
            gk[b].copy_(hk, non_blocking=True)
            gv[b].copy_(hv, non_blocking=True)
            ev_up[b].record(s_up)
        stream.wait_event(ev_up[b])
        s2attn.prefill(gq[b], gk[b], gv[b], lay_p, scale=wp.scale, out=gout[b])
        ev_done[b].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_done[b])
            hout[b].copy_(gout[b], non_blocking=True)
            ev_free[b].record(s_down)

    def e2e_decode(ev):
        ev[0].record(stream)
        gdq.copy_(hdq, non_blocking=True)
        gbt.copy_(hbt, non_blocking=True)
        gcl.copy_(hcl, non_blocking=True)
        s2attn.decode(gdq, d.k_cache, d.v_cache, gbt, gcl, lay_d, scale=wd.scale,
                      num_splits=splits, out=dout, workspace=ws)
        hdout.copy_(dout, non_blocking=True)
        ev[1].record(stream)

    e2e_pre_ms = e2e_dec_ms = 0.0
    if e2e_steps:
        for i in range(2):  # warm-up: both slots once
            e2e_prefill(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        t0.record(s_up)
        for i in range(e2e_steps):
            e2e_prefill(i)
        t1.record(s_down)
        torch.cuda.synchronize()
        e2e_pre_ms = t0.elapsed_time(t1)
        assert torch.equal(hout[(e2e_steps - 1) & 1], out.cpu()), "e2e output differs from the device output"
        if wd is not None:
            e2e_decode([torch.cuda.Event(enable_timing=True) for _ in range(2)])
            torch.cuda.synchronize()
            eevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(e2e_steps)]
            if dist:
                dist.barrier()
            for i in range(e2e_steps):
                e2e_decode(eevs[i])
            torch.cuda.synchronize()
            e2e_dec_ms = sum(e[0].elapsed_time(e[1]) for e in eevs)

    # ---------------- backward (dQ, dK, dV) of a prefill workload, timed on its own
    bwd_ms, bwd_steps, bwd_info = 0.0, 0, None
    if args.backward != "none":
        wb = wp if args.backward == "same" else synth.PREFILL_WORKLOADS[args.backward]
        if wb is wp:
            bq, bk_, bv, lay_b = q, k, v, lay_p
        else:
            bq, bk_, bv = synth.prefill_inputs(wb, device=dev)
            lay_b = s2attn.build_layout(wb.heads, wb.block, wb.stride, wb.local, wb.num_blocks,
                                        wb.dense_heads, device=dev)
        lay_b.transposed(dev)
        bo, blse = s2attn.prefill(bq, bk_, bv, lay_b, scale=wb.scale, want_lse=True)
        gen = torch.Generator(device=dev).manual_seed(77)
        bdo = torch.randn(bq.shape, generator=gen, device=dev).to(torch.bfloat16)
        bdq, bdk, bdv = torch.empty_like(bq), torch.empty_like(bk_), torch.empty_like(bv)
        bws = torch.empty(s2attn.backward_workspace_size(wb.batch, wb.heads, wb.seq),
                          dtype=torch.uint8, device=dev)

        def bwd():
            s2attn.backward(bq, bk_, bv, bo, blse, bdo, lay_b, scale=wb.scale, dq=bdq, dk=bdk,
                            dv=bdv, workspace=bws)

        for _ in range(3):
            bwd()
        torch.cuda.synchronize()
        settle(bwd, args.settle_s / 3, dist, dev)
        bwd_steps = max(3, min(args.steps, args.bwd_steps))
        bev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        if dist:
            dist.barrier()
        bev[0].record(stream)
        for _ in range(bwd_steps):
            bwd()
        bev[1].record(stream)
        torch.cuda.synchronize()
        bwd_ms = bev[0].elapsed_time(bev[1])
        rc, flags = s2attn.device_status(reset=True)
        if rc != 0:
            raise RuntimeError(f"device flags {flags:#x} after the backward")
        bflops = prefill_flops(lay_b, wb)
        bwd_info = (wb, bflops, prefill_issued_flops(lay_b, wb))

    # ---------------- chunked prefill over the paged cache, timed on its own
    chunk_ms, chunk_steps, chunk_info = 0.0, 0, None
    if args.chunk != "none":
        wc = synth.CHUNK_WORKLOADS[args.chunk]
        ci = synth.chunk_inputs(wc, synth.CHUNK_LEN[wc.name], device=dev)
        nb_c = -(-wc.ctx_max // wc.block)
        lay_c = s2attn.build_layout(wc.heads, wc.block, wc.stride, wc.local, nb_c, wc.dense_heads,
                                    device=dev)
        cout = torch.empty_like(ci.q)

        def chunk_call():
            s2attn.chunk_prefill(ci.q, ci.k_cache, ci.v_cache, ci.block_table, ci.ctx_lens,
                                 ci.q_start, lay_c, ci.max_q_len, scale=wc.scale, out=cout)

        for _ in range(3):
            chunk_call()
        torch.cuda.synchronize()
        settle(chunk_call, args.settle_s / 3, dist, dev)
        chunk_steps = max(3, min(args.steps, args.bwd_steps))
        cev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        if dist:
            dist.barrier()
        cev[0].record(stream)
        for _ in range(chunk_steps):
            chunk_call()
        cev[1].record(stream)
        torch.cuda.synchronize()
        chunk_ms = cev[0].elapsed_time(cev[1])
        rc, flags = s2attn.device_status(reset=True)
        if rc != 0:
            raise RuntimeError(f"device flags {flags:#x} after the chunked prefill")
        ctx_h = ci.ctx_lens.cpu().tolist()
        qs = ci.q_start.cpu().tolist()
        qlens = [qs[i + 1] - qs[i] for i in range(len(ctx_h))]
        chunk_info = (wc, chunk_flops(lay_c, wc, ctx_h, qlens), sum(qlens))
        del ci, cout

    # ---------------- max over ranks
    vals = [total_ms, pre_ms, dec_ms, e2e_pre_ms, e2e_dec_ms, bwd_ms, chunk_ms]
    vals = max_over_ranks(vals, dist, dev)
    total_ms, pre_ms, dec_ms, e2e_pre_ms, e2e_dec_ms, bwd_ms, chunk_ms = vals
    sampler.stop()
    clocks = sampler.summary(t_on, t_off)
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    K = args.steps
    tc_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    pre_tflops = world * flops * K / (pre_ms * 1e-3) / 1e12
    per_launch_tflops = flops / (pre_ms / K * 1e-3) / 1e12
    launches = K * (1 + ((1 + (1 if splits > 1 else 0)) if wd else 0))
    splits = splits if wd else 0
    line = {
        "metric": METRIC,
        "value": round(pre_tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "settle": {"steps": settle_steps, "seconds": args.settle_s,
                   "why": "untimed steps after the warm-up until the GPU's power state has "
                          "settled (sw_power_cap engages within ~0.1 s of sustained load), so "
                          "the timed region matches the sustained peak it is divided by"},
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, torch generator on device)",
        "config": {
            "workload": f"{wp.name}+{wd.name}" if wd else wp.name,
            "prefill": {"batch": wp.batch, "heads": wp.heads, "head_dim": wp.head_dim,
                        "seq": wp.seq, "block": wp.block, "stride": wp.stride,
                        "local": wp.local, "dense_heads": list(wp.dense_heads),
                        "algorithmic_gflop_per_step": round(flops / 1e9, 3),
                        "issued_gflop_per_step": round(issued / 1e9, 3),
                        "mma_gflop_per_step": round(mma / 1e9, 3),
                        "ms_per_step": round(pre_ms / K, 4)},
            "layout_build_ms_host": round(layout_ms, 3),
            "l2": "inputs larger than L2 (prefill Q+K+V 403 MB; decode active KV > 1.7 GB)",
            "parallelism": f"replicas x{world} (no data-path collective)",
        },
        "roofline": {
            "kernel": f"s2_prefill_pair_kernel<{wp.head_dim},{wp.block}>",
            "bound": "tensor",
            "achieved": round(per_launch_tflops, 2),
            "peak": tc_peak,
            "unit": "TFLOP/s",
            "frac": round(per_launch_tflops / tc_peak, 4),
            "traffic": load_traffic("s2_prefill_pair_kernel", wp.name),
            "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long loop)",
        },
        "e2e": None if not e2e_steps else {
            "value": round(world * flops * e2e_steps / (e2e_pre_ms * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d_pre,
            "d2h_bytes_per_step": d2h_pre,
            "steps": e2e_steps,
            "what": "s2attn.prefill with Q, K, V copied from pinned host memory and O read back "
                    "every step, pipelined: step i+1's uploads overlap step i's prefill and "
                    "download (two copy streams, double-buffered device tensors); timed from "
                    "the first upload to the last download",
        },
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if wd is not None:
        dec_gbs = world * kv_bytes * K / (dec_ms * 1e-3) / 1e9
        per_launch_gbs = kv_bytes / (dec_ms / K * 1e-3) / 1e9
        hbm = float(peaks["hbm_gbs"])
        line["decode"] = {
            "value": round(dec_gbs, 1), "unit": "GB/s",
            "tokens_per_s": round(world * wd.batch * K / (dec_ms * 1e-3), 1),
            "ms_per_step": round(dec_ms / K, 4),
            "active_kv_bytes_per_step": kv_bytes,
            "page_granular_kv_bytes_per_step": kv_page_bytes,
            "num_splits": splits,
            "config": {"batch": wd.batch, "heads": wd.heads, "head_dim": wd.head_dim,
                       "ctx": [wd.ctx_min, wd.ctx_max], "page": wd.page_size,
                       "block": wd.block, "stride": wd.stride, "local": wd.local},
            "roofline": {"kernel": "s2_decode_split_kernel<128>" + (" + combine" if splits > 1 else ""),
                         "bound": "hbm", "achieved": round(per_launch_gbs, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(per_launch_gbs / hbm, 4),
                         "traffic": load_traffic("s2_decode_split_kernel", wd.name),
                         "peak_source": f"{peak_src} hbm_gbs"},
            "e2e": None if not e2e_steps else {
                "value": round(world * kv_bytes * e2e_steps / (e2e_dec_ms * 1e-3) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": h2d_dec, "d2h_bytes_per_step": d2h_dec},
        }
    if bwd_info is not None:
        wb, bflops, bissued = bwd_info
        # dS needs S (recomputed), dP, and then dV, dK, dQ: 5 products of the
        # forward's 2, so 2.5x its FLOPs; S and dP are computed by both backward
        # kernels here, so 7 products are issued.
        alg = 2.5 * bflops
        per = alg / (bwd_ms / bwd_steps * 1e-3) / 1e12
        line["backward"] = {
            "value": round(world * alg * bwd_steps / (bwd_ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s",
            "workload": wb.name,
            "ms_per_call": round(bwd_ms / bwd_steps, 4),
            "steps": bwd_steps,
            "algorithmic_gflop_per_call": round(alg / 1e9, 3),
            "issued_gflop_per_call": round(3.5 * bissued / 1e9, 3),
            "kernels": "s2_bwd_stats_kernel + s2_bwd_dq_kernel + s2_bwd_dkv_kernel",
            "roofline": {"bound": "tensor", "achieved": round(per, 2), "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": round(per / tc_peak, 4),
                         "traffic": load_traffic("s2_bwd", wb.name),
                         "peak_source": f"{peak_src} bf16_tflops_sustained"},
        }
        line["gpu_launches_backward"] = 3 * bwd_steps
    if chunk_info is not None:
        wc, cflops, total_q = chunk_info
        per = cflops / (chunk_ms / chunk_steps * 1e-3) / 1e12
        line["chunk"] = {
            "value": round(world * cflops * chunk_steps / (chunk_ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s",
            "workload": wc.name,
            "ms_per_call": round(chunk_ms / chunk_steps, 4),
            "steps": chunk_steps,
            "chunk_rows": total_q,
            "algorithmic_gflop_per_call": round(cflops / 1e9, 3),
            "config": {"batch": wc.batch, "heads": wc.heads, "head_dim": wc.head_dim,
                       "ctx": [wc.ctx_min, wc.ctx_max], "chunk": synth.CHUNK_LEN[wc.name],
                       "page": wc.page_size, "block": wc.block, "stride": wc.stride,
                       "local": wc.local},
            "kernels": "s2_chunk_prefill_kernel",
            "roofline": {"bound": "tensor", "achieved": round(per, 2), "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": round(per / tc_peak, 4),
                         "traffic": load_traffic("s2_chunk_prefill_kernel", wc.name),
                         "peak_source": f"{peak_src} bf16_tflops_sustained"},
        }
        line["gpu_launches_chunk"] = chunk_steps
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wp, args.cpu_seconds)
    return line


# ---------------------------------------------------------------- oracle arm

def oracle_sample(wp, n_rows, seed, q=None, k=None, v=None):
    """Time the fp64 oracle on n_rows seeded random rows of the prefill workload.
    Returns (seconds, algorithmic flops of those rows, threads)."""
    import oracle
    from head_heterogeneous_block_s2_b200 import synth

    if q is None:
        q, k, v = synth.prefill_inputs(wp)
    rng = np.random.default_rng(seed)
    total = wp.batch * wp.heads * wp.seq
    rows = np.sort(rng.choice(total, n_rows, replace=False)).astype(np.int64)
    # visible keys of each sampled row (the work the definition does)
    mask = oracle.block_mask(wp.heads, wp.num_blocks, wp.stride, wp.local, wp.dense_heads)
    t = rows % wp.seq
    h = (rows // wp.seq) % wp.heads
    i = t // wp.block
    full = mask[h, i, :].astype(np.int64)  # active blocks of each row
    nfull = full.sum(1) - 1  # blocks before the diagonal
    keys = nfull * wp.block + (t % wp.block) + 1
    flops = int(4 * wp.head_dim * keys.sum())
    t0 = time.perf_counter()
    oracle.prefill(q, k, v, wp.block, wp.stride, wp.local, wp.scale, wp.dense_heads, rows=rows)
    dt = time.perf_counter() - t0
    return dt, flops, oracle.default_threads(), (q, k, v)


def cpu_baseline(wp, seconds):
    """The oracle as it stands, on the host cores, over a bounded row sample
    calibrated to take about `seconds`."""
    dt, fl, th, qkv = oracle_sample(wp, 512, 1)
    n = int(min(wp.batch * wp.heads * wp.seq, max(512, 512 * seconds / max(dt, 1e-3))))
    dt, fl, th, _ = oracle_sample(wp, n, 2, *qkv)
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": th, "kind": "oracle",
            "sample": f"{n} seeded random query rows of {wp.name} "
                      f"({n / (wp.batch * wp.heads * wp.seq):.2%} of the batch), fp64, "
                      f"{dt:.1f} s on {th} threads"}


def run_reference(args, rank):
    if rank != 0:
        return None
    from head_heterogeneous_block_s2_b200 import synth

    wp = synth.PREFILL_WORKLOADS[args.prefill]
    # calibrate rows per step so the whole run takes about args.ref_seconds
    dt, fl, th, qkv = oracle_sample(wp, 256, 1)
    per_step_s = args.ref_seconds / max(1, args.steps + args.warmup)
    n = int(max(16, min(wp.batch * wp.heads * wp.seq, 256 * per_step_s / max(dt, 1e-4))))
    for i in range(args.warmup):
        oracle_sample(wp, n, 100 + i, *qkv)
    tot_t = tot_f = 0.0
    for i in range(args.steps):
        dt, fl, th, _ = oracle_sample(wp, n, 1000 + i, *qkv)
        tot_t += dt
        tot_f += fl
    val = tot_f / tot_t / 1e12
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wp.name, "rows_per_step": n},
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": th, "kind": "oracle",
                         "sample": f"{n} seeded random query rows of {wp.name} per step"},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--settle-s", type=float, default=1.5,
                    help="untimed steps after the warm-up until this many seconds have passed "
                         "(the power state settles; the backward and chunk legs take a third each)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill", default="prefill_1p3b",
                    choices=["tiny", "prefill_1p3b", "prefill_7b_hybrid", "prefill_long_131k"])
    ap.add_argument("--decode", default="decode_paged", choices=["decode_paged", "none"])
    ap.add_argument("--splits", type=int, default=0, help="decode splits (0 = automatic)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode batch (small cases for profiling only)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling only)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", default="same",
                    help="prefill workload whose backward is timed separately ('same' = the "
                         "prefill workload, 'none' = skip)")
    ap.add_argument("--bwd-steps", type=int, default=20)
    ap.add_argument("--chunk", default="chunk_paged", choices=["chunk_paged", "none"],
                    help="chunked prefill over the paged cache, timed separately")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.impl == "reference":
            line = run_reference(args, rank)
        else:
            line = run_ours(args, rank, world, dist)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
