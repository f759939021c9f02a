#!/usr/bin/env python3
"""Benchmark of the HHST sparse-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * prefill (block-sparse attention, tcgen05 kernel) over the long-context
    workload: batch 1, 32 heads, head_dim 128, seq 131072, B 128, S 16, L 4,
    one planted key row per head (the largest single-GPU prefill);
  * decode (split-KV paged kernel, plus the combine when it splits) over 64
    sequences, 32 heads, head_dim 128, contexts U[4096, 32768], 16-token pages,
    permuted block table, B 128, S 16, L 4.
The layouts are built once (host, per layout) before timing.

Headline: prefill effective TFLOP/s (4 * head_dim per visible (query, key)
pair; the dense work the pattern skips is not counted), from CUDA events around
the prefill launches inside the timed steps. The decode part reports active
K+V GB/s and tokens/s in "decode". The other prefill workloads (1.3B-shaped,
7B hybrid), the backward and the chunked prefill are timed as separate legs,
each with its own roofline. Tensor-bound fractions divide by the measured
burst bf16 peak (cuBLAS, MEASURED_PEAKS.json "bf16_tflops"); the sampled SM
clocks of each timed region are reported beside it.

Multi-GPU: one process per GPU, each processing its own batch (weak scaling,
no collective on the data path); time = max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
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
HEADLINE = "prefill_long_131k"


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


def plant_positions(w, last_row_blocks, seed=7):
    """For every head, a token of a key block j <= nb/2 that the last query
    block lists (a strided block: the local window sits at the end), seeded.
    ``last_row_blocks[h]`` is the key-block list of (head h, last query block)."""
    rng = np.random.default_rng(seed)
    nb = w.num_blocks
    pos = {}
    for h in range(w.heads):
        cands = [int(j) for j in last_row_blocks[h] if int(j) <= nb // 2]
        j = int(rng.choice(cands))
        pos[h] = j * w.block + int(rng.integers(w.block))
    return pos


# Sources each kernel is compiled from (its ncu traffic figure stays valid while
# these files are unchanged).
KERNEL_SOURCES = {
    "s2_prefill_pair_kernel": ("prefill_pair_sm100.cuh", "lists.cuh", "ptx.cuh", "umma.cuh"),
    "s2_decode_split_kernel": ("decode.cuh", "ptx.cuh"),
    "s2_bwd": ("backward_sm100.cuh", "lists.cuh", "ptx.cuh", "store.cuh", "umma.cuh"),
    "s2_chunk_prefill_kernel": ("chunk_sm100.cuh", "lists.cuh", "ptx.cuh", "store.cuh", "umma.cuh"),
}


def source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "head_heterogeneous_block_s2_b200", "csrc")
    for fn in sorted(KERNEL_SOURCES[kernel]):
        h.update(fn.encode())
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


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


def roofline(kernel, bound, achieved, peak, unit, traffic, peak_source):
    return {"kernel": kernel, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
            "unit": unit, "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": peak_source}


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

class Timer:
    """CUDA events on the launching stream around a block of calls, between
    a barrier (multi-rank) and device synchronisations; wall-clock bounds for
    the clock samples."""

    def __init__(self, stream, dist):
        self.stream, self.dist = stream, dist

    def run(self, fn, n):
        import torch

        if self.dist:
            self.dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_on = time.time()
        a.record(self.stream)
        for _ in range(n):
            fn()
        b.record(self.stream)
        torch.cuda.synchronize()
        t_off = time.time()
        if self.dist:
            self.dist.barrier()
        return a.elapsed_time(b), (t_on, t_off)


def check_flags(s2attn, what):
    rc, flags = s2attn.device_status(reset=True)
    if rc != 0:
        raise RuntimeError(f"device flags {flags:#x} after {what}")


def make_prefill(wp, dev, s2attn, synth):
    """Inputs (resident), layout and work counts of one prefill workload."""
    lay = s2attn.build_layout(wp.heads, wp.block, wp.stride, wp.local, wp.num_blocks,
                              wp.dense_heads, device=dev)
    plant = None
    if wp.planted:
        plant = plant_positions(wp, [lay.row(h, wp.num_blocks - 1) for h in range(wp.heads)])
    q, k, v = synth.prefill_inputs(wp, device=dev, plant_positions=plant)
    return dict(w=wp, q=q, k=k, v=v, lay=lay, flops=prefill_flops(lay, wp),
                issued=prefill_issued_flops(lay, wp), mma=prefill_mma_flops(lay, wp), plant=plant)


def prefill_config(P, ms_per_call):
    wp = P["w"]
    return {"batch": wp.batch, "heads": wp.heads, "head_dim": wp.head_dim, "seq": wp.seq,
            "block": wp.block, "stride": wp.stride, "local": wp.local,
            "dense_heads": list(wp.dense_heads), "planted_keys": P["plant"] is not None,
            "algorithmic_gflop_per_call": round(P["flops"] / 1e9, 3),
            "issued_gflop_per_call": round(P["issued"] / 1e9, 3),
            "mma_gflop_per_call": round(P["mma"] / 1e9, 3),
            "ms_per_call": round(ms_per_call, 4)}


def run_ours(args, rank, world, dist):
    import torch

    from head_heterogeneous_block_s2_b200 import s2attn, synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    s2attn.load()
    peaks, peak_src = load_peaks()
    tc_peak = float(peaks["bf16_tflops"])
    tc_src = f"{peak_src} bf16_tflops (burst cuBLAS bf16 GEMM)"
    hbm = float(peaks["hbm_gbs"])
    stream = torch.cuda.current_stream(dev)
    timer = Timer(stream, dist)
    sampler = ClockSampler(dev.index)
    sampler.start()

    # setup (untimed): inputs resident in HBM, layouts built once per layout
    t0 = time.time()
    wp = synth.PREFILL_WORKLOADS[args.prefill]
    P = make_prefill(wp, dev, s2attn, synth)
    q, k, v, lay_p = P["q"], P["k"], P["v"], P["lay"]
    t1 = time.time()
    s2attn.build_layout(wp.heads, wp.block, wp.stride, wp.local, wp.num_blocks, wp.dense_heads)
    layout_ms = (time.time() - t1) * 1e3
    out = torch.empty_like(q)
    flops = P["flops"]
    wd = synth.DECODE_WORKLOADS[args.decode] if args.decode != "none" else None
    if wd is not None and args.decode_batch > 0:
        wd = wd.with_(batch=args.decode_batch)
    splits = 0
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

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check_flags(s2attn, "warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    it = iter(evs)
    total_ms, (t_on, t_off) = timer.run(lambda: step(next(it)), K)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs) if wd else 0.0
    check_flags(s2attn, "timing")
    clocks = sampler.summary(t_on, t_off)

    # ---------------- end to end through the public API with host buffers
    # Prefill leg, pipelined like a serving loop: every step copies its Q, K, V
    # from pinned host memory and reads its output back, on two copy streams
    # with double-buffered device tensors, so step i+1's uploads overlap step
    # i's prefill and download. Decode leg: one stream, step after step.
    e2e_steps = 0 if args.no_e2e else max(1, min(K, args.e2e_steps))
    e2e_pre_ms = e2e_dec_ms = 0.0
    h2d_pre = 3 * q.numel() * q.element_size()
    d2h_pre = out.numel() * out.element_size()
    hq = hk = hv = None
    if e2e_steps or (world == 1 and not args.no_cpu_baseline):
        hq, hk, hv = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
    if e2e_steps:
        hout = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
        gq = [q, torch.empty_like(q)]
        gk = [k, torch.empty_like(k)]
        gv = [v, torch.empty_like(v)]
        gout = [torch.empty_like(out) for _ in range(2)]
        s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_free = [torch.cuda.Event() for _ in range(2)]  # the slot's D2H (so also its prefill) is done

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

        for i in range(2):  # warm-up: both slots once
            e2e_prefill(i)
        torch.cuda.synchronize()
        ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        ta.record(s_up)
        for i in range(e2e_steps):
            e2e_prefill(i)
        tb.record(s_down)
        torch.cuda.synchronize()
        e2e_pre_ms = ta.elapsed_time(tb)
        assert torch.equal(hout[(e2e_steps - 1) & 1], out.cpu()), "e2e output differs from the device output"
        del hout, gout, gq[1], gk[1], gv[1]
        if wd is not None:
            hdq = d.q.cpu().pin_memory()
            hbt = d.block_table.cpu().pin_memory()
            hcl = d.ctx_lens.cpu().pin_memory()
            hdout = torch.empty(d.q.shape, dtype=d.q.dtype).pin_memory()
            gdq, gbt, gcl = torch.empty_like(d.q), torch.empty_like(d.block_table), torch.empty_like(d.ctx_lens)
            h2d_dec = sum(t.numel() * t.element_size() for t in (hdq, hbt, hcl))
            d2h_dec = hdout.numel() * hdout.element_size()

            def e2e_decode():
                gdq.copy_(hdq, non_blocking=True)
                gbt.copy_(hbt, non_blocking=True)
                gcl.copy_(hcl, non_blocking=True)
                s2attn.decode(gdq, d.k_cache, d.v_cache, gbt, gcl, lay_d, scale=wd.scale,
                              num_splits=splits, out=dout, workspace=ws)
                hdout.copy_(dout, non_blocking=True)

            e2e_decode()
            e2e_dec_ms, _ = timer.run(e2e_decode, e2e_steps)
    if wd is not None:
        del d, ws  # free the 21 GB cache before the legs
    torch.cuda.empty_cache()

    # ---------------- other prefill workloads, each timed on its own
    legs = []
    for name in [x for x in args.legs.split(",") if x and x != "none" and x != args.prefill]:
        L = make_prefill(synth.PREFILL_WORKLOADS[name], dev, s2attn, synth)
        lout = torch.empty_like(L["q"])

        def call(L=L, lout=lout):
            s2attn.prefill(L["q"], L["k"], L["v"], L["lay"], scale=L["w"].scale, out=lout)

        for _ in range(3):
            call()
        n = max(3, int(args.leg_ms / max(1e-3, L["flops"] / 1e12)))  # ~leg_ms at 1 PFLOP/s
        ms, win = timer.run(call, n)
        check_flags(s2attn, f"the {name} leg")
        legs.append((L, n, ms, sampler.summary(*win)))
        del L, lout
        torch.cuda.empty_cache()

    # ---------------- backward (dQ, dK, dV), each workload timed on its own
    bwds = []
    for name in [x for x in args.backward.split(",") if x and x != "none"]:
        wb = synth.PREFILL_WORKLOADS[name]
        Bk = make_prefill(wb, dev, s2attn, synth) if name != args.prefill else P
        lay_b = Bk["lay"]
        lay_b.transposed(dev)
        bo, blse = s2attn.prefill(Bk["q"], Bk["k"], Bk["v"], lay_b, scale=wb.scale, want_lse=True)
        gen = torch.Generator(device=dev).manual_seed(77)
        bdo = torch.randn(Bk["q"].shape, generator=gen, device=dev).to(torch.bfloat16)
        bdq, bdk, bdv = torch.empty_like(Bk["q"]), torch.empty_like(Bk["k"]), torch.empty_like(Bk["v"])
        bws = torch.empty(s2attn.backward_workspace_size(wb.batch, wb.heads, wb.seq),
                          dtype=torch.uint8, device=dev)

        def bwd(Bk=Bk, bo=bo, blse=blse, bdo=bdo, bdq=bdq, bdk=bdk, bdv=bdv, bws=bws, wb=wb):
            s2attn.backward(Bk["q"], Bk["k"], Bk["v"], bo, blse, bdo, Bk["lay"], scale=wb.scale,
                            dq=bdq, dk=bdk, dv=bdv, workspace=bws)

        for _ in range(3):
            bwd()
        n = max(3, int(args.leg_ms / max(1e-3, 2.5 * Bk["flops"] / 0.5e12)))  # at 0.5 PFLOP/s
        ms, win = timer.run(bwd, n)
        check_flags(s2attn, f"the {name} backward")
        bwds.append((Bk, n, ms, sampler.summary(*win)))
        del bo, blse, bdo, bdq, bdk, bdv, bws, Bk
        torch.cuda.empty_cache()

    # ---------------- chunked prefill over the paged cache, timed on its own
    chunk = None
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
        ctx_h = ci.ctx_lens.cpu().tolist()
        qs = ci.q_start.cpu().tolist()
        qlens = [qs[i + 1] - qs[i] for i in range(len(ctx_h))]
        cflops = chunk_flops(lay_c, wc, ctx_h, qlens)
        n = max(3, int(args.leg_ms / max(1e-3, cflops / 0.7e12)))  # at 0.7 PFLOP/s
        ms, win = timer.run(chunk_call, n)
        check_flags(s2attn, "the chunked prefill")
        chunk = (wc, cflops, sum(qlens), n, ms, sampler.summary(*win))
        del ci, cout

    # ---------------- max over ranks
    vals = [total_ms, pre_ms, dec_ms, e2e_pre_ms, e2e_dec_ms] + [x[2] for x in legs] + \
        [x[2] for x in bwds] + ([chunk[4]] if chunk else [])
    vals = max_over_ranks(vals, dist, dev)
    total_ms, pre_ms, dec_ms, e2e_pre_ms, e2e_dec_ms = vals[:5]
    rest = vals[5:]
    legs = [(L, n, rest.pop(0), c) for (L, n, _, c) in legs]
    bwds = [(B_, n, rest.pop(0), c) for (B_, n, _, c) in bwds]
    if chunk:
        chunk = chunk[:4] + (rest.pop(0), chunk[5])
    sampler.stop()
    if rank != 0:
        return None

    per_launch = flops / (pre_ms / K * 1e-3) / 1e12
    launches = K * (1 + ((1 + (1 if splits > 1 else 0)) if wd else 0))
    line = {
        "metric": METRIC,
        "value": round(world * flops * K / (pre_ms * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, torch generator on device; planted keys chosen "
                "from the layout)",
        "config": {
            "workload": wp.name,
            "step": f"{wp.name} prefill + {wd.name} decode" if wd else f"{wp.name} prefill",
            "prefill": prefill_config(P, pre_ms / K),
            "layout_build_ms_host": round(layout_ms, 3),
            "l2": "inputs larger than L2 (prefill Q+K+V 3.2 GB; decode active KV 1.7 GB of a "
                  "21 GB cache)",
            "parallelism": f"replicas x{world} (no data-path collective)",
        },
        "roofline": roofline(f"s2_prefill_pair_kernel<{wp.head_dim},{wp.block}>", "tensor", per_launch,
                             tc_peak, "TFLOP/s", load_traffic("s2_prefill_pair_kernel", wp.name),
                             tc_src),
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
        per_gbs = kv_bytes / (dec_ms / K * 1e-3) / 1e9
        line["decode"] = {
            "workload": wd.name,
            "value": round(world * kv_bytes * K / (dec_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "tokens_per_s": round(world * wd.batch * K / (dec_ms * 1e-3), 1),
            "ms_per_step": round(dec_ms / K, 4),
            "active_kv_bytes_per_step": kv_bytes,
            "page_granular_kv_bytes_per_step": kv_page_bytes,
            "num_splits": splits,
            "config": {"batch": wd.batch, "heads": wd.heads, "head_dim": wd.head_dim,
                       "ctx": [wd.ctx_min, wd.ctx_max], "page": wd.page_size,
                       "block": wd.block, "stride": wd.stride, "local": wd.local},
            "roofline": roofline("s2_decode_split_kernel<128>" + (" + combine" if splits > 1 else ""),
                                 "hbm", per_gbs, hbm, "GB/s",
                                 load_traffic("s2_decode_split_kernel", wd.name), f"{peak_src} hbm_gbs"),
            "e2e": None if not e2e_steps else {
                "value": round(world * kv_bytes * e2e_steps / (e2e_dec_ms * 1e-3) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": h2d_dec, "d2h_bytes_per_step": d2h_dec},
        }
    line["prefill_legs"] = []
    for L, n, ms, c in legs:
        w_ = L["w"]
        per = L["flops"] / (ms / n * 1e-3) / 1e12
        line["prefill_legs"].append({
            "workload": w_.name, "value": round(world * per, 2), "unit": "TFLOP/s", "calls": n,
            "config": prefill_config(L, ms / n),
            "roofline": roofline(f"s2_prefill_pair_kernel<{w_.head_dim},{w_.block}>", "tensor", per,
                                 tc_peak, "TFLOP/s", load_traffic("s2_prefill_pair_kernel", w_.name),
                                 tc_src),
            "clocks": c})
    line["gpu_launches_legs"] = sum(n for _, n, _, _ in legs)
    line["backward"] = []
    for Bk, n, ms, c in bwds:
        wb = Bk["w"]
        # dS needs S (recomputed), dP, and then dV, dK, dQ: 5 products of the
        # forward's 2, so 2.5x its FLOPs; S and dP are computed by both backward
        # kernels here, so 7 products are issued.
        alg = 2.5 * Bk["flops"]
        per = alg / (ms / n * 1e-3) / 1e12
        line["backward"].append({
            "workload": wb.name, "value": round(world * per, 2), "unit": "TFLOP/s",
            "ms_per_call": round(ms / n, 4), "calls": n,
            "algorithmic_gflop_per_call": round(alg / 1e9, 3),
            "issued_gflop_per_call": round(3.5 * Bk["issued"] / 1e9, 3),
            "kernels": "s2_bwd_stats_kernel + s2_bwd_dq_kernel + s2_bwd_dkv_kernel",
            "roofline": roofline("backward (3 kernels)", "tensor", per, tc_peak, "TFLOP/s",
                                 load_traffic("s2_bwd", wb.name), tc_src),
            "clocks": c})
    line["gpu_launches_backward"] = sum(3 * n for _, n, _, _ in bwds)
    if chunk is not None:
        wc, cflops, total_q, n, ms, c = chunk
        per = cflops / (ms / n * 1e-3) / 1e12
        line["chunk"] = {
            "workload": wc.name, "value": round(world * per, 2), "unit": "TFLOP/s",
            "ms_per_call": round(ms / n, 4), "calls": n, "chunk_rows": total_q,
            "algorithmic_gflop_per_call": round(cflops / 1e9, 3),
            "config": {"batch": wc.batch, "heads": wc.heads, "head_dim": wc.head_dim,
                       "ctx": [wc.ctx_min, wc.ctx_max], "chunk": synth.CHUNK_LEN[wc.name],
                       "page": wc.page_size, "block": wc.block, "stride": wc.stride,
                       "local": wc.local},
            "kernels": "s2_chunk_prefill_kernel",
            "roofline": roofline("s2_chunk_prefill_kernel<128,128>", "tensor", per, tc_peak, "TFLOP/s",
                                 load_traffic("s2_chunk_prefill_kernel", wc.name), tc_src),
            "clocks": c}
        line["gpu_launches_chunk"] = n
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wp, args.cpu_seconds, (hq, hk, hv), P["plant"], flops)
    return line


# ---------------------------------------------------------------- oracle arm

def oracle_sample(wp, n_rows, seed, qkv):
    """Time the fp64 oracle on n_rows seeded random rows of the prefill workload.
    Returns (seconds, algorithmic flops of those rows, threads)."""
    import oracle

    q, k, v = qkv
    rng = np.random.default_rng(seed)
    total = wp.batch * wp.heads * wp.seq
    rows = np.sort(rng.choice(total, n_rows, replace=False)).astype(np.int64)
    # visible keys of each sampled row (the work the definition does)
    cnt = oracle.block_mask(wp.heads, wp.num_blocks, wp.stride, wp.local,
                            wp.dense_heads).sum(axis=2, dtype=np.int64)  # active blocks per row
    t = rows % wp.seq
    h = (rows // wp.seq) % wp.heads
    i = t // wp.block
    nfull = cnt[h, i] - 1  # active blocks before the diagonal
    keys = nfull * wp.block + (t % wp.block) + 1
    flops = int(4 * wp.head_dim * keys.sum())
    t0 = time.perf_counter()
    oracle.prefill(q, k, v, wp.block, wp.stride, wp.local, wp.scale, wp.dense_heads, rows=rows)
    dt = time.perf_counter() - t0
    return dt, flops, oracle.default_threads()


def oracle_inputs(wp):
    """The workload's inputs on the host (planted keys chosen with the oracle's
    own block mask, which equals the layout's lists)."""
    import oracle
    from head_heterogeneous_block_s2_b200 import synth

    plant = None
    if wp.planted:
        m = oracle.block_mask(wp.heads, wp.num_blocks, wp.stride, wp.local, wp.dense_heads)
        plant = plant_positions(wp, [np.nonzero(m[h, wp.num_blocks - 1])[0] for h in range(wp.heads)])
    return synth.prefill_inputs(wp, plant_positions=plant), plant


def cpu_baseline(wp, seconds, qkv, plant, full):
    """The oracle as it stands, on the host cores, over a bounded row sample
    calibrated to take about `seconds`; the full workload's time is
    extrapolated from the sample's rate (labelled as such)."""
    dt, fl, th = oracle_sample(wp, 256, 1, qkv)
    n = int(min(wp.batch * wp.heads * wp.seq, max(256, 256 * seconds / max(dt, 1e-3))))
    dt, fl, th = oracle_sample(wp, n, 2, qkv)
    rate = fl / dt
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": th, "kind": "oracle",
            "sample": f"{n} seeded random query rows of {wp.name} "
                      f"({n / (wp.batch * wp.heads * wp.seq):.2%} of the batch"
                      f"{', planted keys' if plant else ''}), fp64, {dt:.1f} s on {th} threads",
            "full_workload_s_extrapolated": round(full / rate, 1)}


def run_reference(args, rank):
    if rank != 0:
        return None
    from head_heterogeneous_block_s2_b200 import synth

    wp = synth.PREFILL_WORKLOADS[args.prefill]
    qkv, plant = oracle_inputs(wp)
    # calibrate rows per step so the whole run takes about args.ref_seconds
    dt, fl, th = oracle_sample(wp, 128, 1, qkv)
    per_step_s = args.ref_seconds / max(1, args.steps + args.warmup)
    n = int(max(16, min(wp.batch * wp.heads * wp.seq, 128 * per_step_s / max(dt, 1e-4))))
    for i in range(args.warmup):
        oracle_sample(wp, n, 100 + i, qkv)
    tot_t = tot_f = 0.0
    for i in range(args.steps):
        dt, fl, th = oracle_sample(wp, n, 1000 + i, qkv)
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
                         "sample": f"{n} seeded random query rows of {wp.name} per step"
                                   f"{' (planted keys)' if plant else ''}"},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill", default=HEADLINE,
                    choices=["tiny", "prefill_1p3b", "prefill_7b_hybrid", "prefill_long_131k"],
                    help="the step's prefill workload (the headline)")
    ap.add_argument("--decode", default="decode_paged", choices=["decode_paged", "none"])
    ap.add_argument("--splits", type=int, default=0, help="decode splits (0 = automatic)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode batch (small cases for profiling only)")
    ap.add_argument("--legs", default="prefill_1p3b,prefill_7b_hybrid",
                    help="other prefill workloads, each timed on its own ('none' = skip)")
    ap.add_argument("--leg-ms", type=float, default=150.0,
                    help="approximate GPU time of each separately timed leg")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling only)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", default="prefill_1p3b,prefill_7b_hybrid",
                    help="prefill workloads whose backward is timed separately ('none' = skip)")
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
