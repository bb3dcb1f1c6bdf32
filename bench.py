#!/usr/bin/env python
"""Decode-attention benchmark on B200: one step = append this step's token per
sequence into the paged cache (pa_kv_append) + paged decode attention
(pa_decode, with its split-KV merge) over the whole batch.

Workload (default): the Llama-3-70B-shaped single layer — B=32 sequences of
8192 tokens, Hq=64, Hkv=8, D=128, bf16, pages of P=32 tokens randomly permuted
over an 8192-page pool (1.07 GB of K/V, larger than the 126 MB L2, so no L2
flush is needed between steps). Inputs are seeded synthetic data (seed = rank).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch
(weak scaling) — the sequences are independent, so there is no data-path
collective; only the timing uses a barrier and a max over ranks.

Prints one JSON line (rank 0).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention achieved HBM GB/s and % of B200 peak; sequences/sec per layer"
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
NOMINAL_HBM_GBS = 7700.0   # B200 (HGX) specification figure, for context only
# every source file the decode kernel is compiled from: a recorded ncu traffic
# figure is used only for the exact sources it was captured from
KERNEL_SRCS = [os.path.join(ROOT, "paged_kv_cache_466_b200", "csrc", f)
               for f in ("decode.cu", "pa_device.cuh", "pa_quant.cuh", "pa_internal.h")] + \
              [os.path.join(ROOT, "include", "pagedattn.h")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama70b",
                    choices=["llama70b", "llama8b", "int8", "fp8", "int4", "prefix", "tiny"])
    ap.add_argument("--cascade", action="store_true",
                    help="prefix workload: decode with pa_decode_shared_prefix")
    ap.add_argument("--window", type=int, default=0,
                    help="attend only the last W tokens (+ --sinks) via pa_decode_window")
    ap.add_argument("--sinks", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--splits", type=int, default=0, help="split-KV count (0 = automatic)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's number of sequences (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separate-append", action="store_true",
                    help="time pa_kv_append + pa_decode as two calls instead of the fused "
                         "pa_decode_append step")
    ap.add_argument("--alternate-pools", action="store_true",
                    help="keep two independent copies of the pool and alternate between them "
                         "step by step, so no step reads pages the previous step left in L2")
    ap.add_argument("--context-parallel", action="store_true",
                    help="every rank holds 1/N of each sequence's tokens of the same batch "
                         "and decodes its range; one all-gather of (o, lse) and a merge per "
                         "step (strong scaling over the token dimension)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a buffer of twice the L2 size between timed steps; the step "
                         "time is then the sum of per-step CUDA events, flush excluded")
    return ap.parse_args()


# ------------------------------------------------------------------ accounting
def attended_tokens(w, sinks: int = 0, window: int = 0) -> int:
    """Tokens one decode attends: the whole context, or sinks + the last window."""
    ctx = w.context_lens.astype("int64")
    if window <= 0:
        return int(ctx.sum())
    import numpy as np
    return int(np.minimum(ctx, np.minimum(ctx, sinks) + window).sum())


def decode_bytes(w, sinks: int = 0, window: int = 0) -> int:
    """Algorithmic bytes of one decode: every cached K/V element of every
    attended token once, plus q (Eq. 1 reads nothing else)."""
    row = {"bf16": w.D * 2, "u8": w.D + 8, "fp8": w.D + 8, "u4": w.D // 2 + 8}[w.kv]
    return attended_tokens(w, sinks, window) * w.Hkv * 2 * row + w.B * w.Hq * w.D * 2


def unique_bytes(w) -> int:
    """Bytes the decode must bring from HBM at least once when prefix pages
    are shared: the shared prefix once plus every request's own tokens, plus
    q (the shared prefix workload); decode_bytes for every other workload."""
    pre = int(w.notes.get("prefix_tokens", 0)) if "prefix_pages" in w.notes else 0
    if pre == 0:
        return decode_bytes(w)
    row = {"bf16": w.D * 2, "u8": w.D + 8, "fp8": w.D + 8, "u4": w.D // 2 + 8}[w.kv]
    own = int((w.context_lens.astype("int64") - pre).clip(min=0).sum())
    return (pre + own) * w.Hkv * 2 * row + w.B * w.Hq * w.D * 2


def append_bytes(w) -> int:
    n = len(w.step_seq)
    row = {"bf16": w.D * 2, "u8": w.D + 8, "fp8": w.D + 8, "u4": w.D // 2 + 8}[w.kv]
    return n * w.Hkv * 2 * (w.D * 2 + row)


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sources_sha256() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SRCS:
        h.update(os.path.basename(p).encode())
        h.update(open(p, "rb").read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """ncu DRAM bytes per decode launch, if captured from exactly the current
    kernel sources (any change to them voids the record until it is re-captured)."""
    try:
        rec = json.load(open(TRAFFIC_FILE)).get(workload)
        if rec and rec.get("kernel_sources_sha256") == kernel_sources_sha256():
            return int(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (timing only; no data path)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(step_bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Aggregate throughput: every rank's bytes over the slowest rank's time."""
    return step_bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """NVML sampling of SM clock and clock-event reasons (read-only)."""
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
             0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 5e-5):
        self.ok = False
        self.samples, self.reasons = [], 0       # (host time, MHz)
        self.window = None
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(hh)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        h = hh
                        break
            self.h = h if h is not None else pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _read(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((time.perf_counter(), mhz, int(r)))

    def _loop(self):
        # a read every ~0.1 ms at most (each NVML query releases the GIL): a timed
        # region of a few milliseconds still gets tens of samples
        while not self._stop.is_set():
            try:
                self._read()
            except Exception:
                pass
            self._first.set()
            time.sleep(self.period)

    def start(self):
        if not self.ok:
            return
        # hand the interpreter lock over every 50 us instead of every 5 ms, so
        # the sampler runs while the main thread launches the steps
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(5e-5)
        self._stop = threading.Event()
        self._first = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()
        self._first.wait(5.0)   # sampling has begun before the first step

    def mark(self, begin: bool):
        """Host time at the start (before the first launch) and end (after the
        synchronise) of the timed region."""
        t = time.perf_counter()
        self.window = (t, None) if begin else (self.window[0], t)

    def stop(self):
        if not self.ok:
            return None
        self._stop.set()
        self._t.join()
        sys.setswitchinterval(self._switch)
        lo, hi = self.window if self.window and self.window[1] else (float("-inf"), float("inf"))
        timed = [(m, r) for t, m, r in self.samples if lo <= t <= hi]
        every = [(m, r) for _, m, r in self.samples]
        use = timed if timed else every
        reasons = 0
        for _, r in use:
            reasons |= r
        names = [n for b, n in self.NAMES.items() if reasons & b]
        return {"sm_mhz": statistics.median(m for m, _ in use) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(timed),
                "samples_with_warmup": len(every),
                "sampled": "NVML SM clock and clock-event reasons, read every ~0.1 ms from "
                           "the start of the warm-up to the end of the timed region; sm_mhz, "
                           "reasons and samples cover the timed region"}


# ------------------------------------------------------------------ CPU oracle leg
def cpu_oracle_throughput(w, budget_s: float = 12.0, max_reps: int = 40):
    """The fp64 oracle, as it stands, on this host's cores: the whole batch,
    repeated until ~budget_s of work. Returns (GB/s, cores, sample text)."""
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    cores = int(os.environ["OMP_NUM_THREADS"])
    import oracle
    from paged_kv_cache_466_b200.workloads import bits
    hp = oracle.empty_pool(w.kv, w.num_pages, w.Hkv, w.P, w.D, 0)
    seq, pos, k, v = w.all_rows()
    oracle.scatter_rows(hp, w.block_tables, seq, pos, bits(k), bits(v))
    qb = bits(w.q)
    reps, t_total = 0, 0.0
    while reps < max_reps and (t_total < budget_s or reps == 0):
        t0 = time.perf_counter()
        oracle.paged_attention(hp, qb, w.block_tables, w.context_lens, w.scale)
        t_total += time.perf_counter() - t0
        reps += 1
    gbs = decode_bytes(w) * reps / t_total / 1e9
    sample = (f"{reps} full decode(s) of the {w.name} batch ({w.B} seqs x {w.Hq} heads), "
              f"{t_total:.1f} s total; attention only (no cache write)")
    return gbs, cores, sample


# ------------------------------------------------------------------ arms
def make_workload(name: str, seed: int, batch: int = 0):
    from paged_kv_cache_466_b200 import workloads as W
    kw = {"B": batch} if batch else {}
    if name == "prefix":
        return W.prefix(seed=seed, **kw)[0]
    if name == "tiny":
        return W.tiny(seed=seed)
    return getattr(W, name)(seed=seed, **kw)


def workload_label(w, args) -> str:
    extra = ""
    if args.window > 0:
        extra = f", sinks={args.sinks}, window={args.window}"
    if args.cascade:
        extra += f", cascade over the {w.notes.get('prefix_tokens', 0)}-token shared prefix"
    return extra


def config_of(w, args, n, S):
    c = {"workload": f"{w.name}: B={w.B}, ctx={'U' if len(set(w.context_lens.tolist())) > 1 else ''}"
                     f"{int(w.context_lens.min())}..{int(w.context_lens.max())}, Hq={w.Hq}, "
                     f"Hkv={w.Hkv}, D={w.D}, P={w.P}, kv={w.kv}" + workload_label(w, args),
         "global_batch": w.B * n, "seq_len": int(w.context_lens.max()),
         "parallelism": f"dp{n} (independent sequences, no collective)",
         "num_splits": S, "pool_pages": w.num_pages,
         "l2": "flushed between steps (write of 2x the L2 size, outside the step events)"
               if args.flush_l2 else
               "two independent pools alternated step by step (no step finds the previous "
               "step's pages in L2), not flushed" if args.alternate_pools else
               "inputs larger than the 126 MB L2, not flushed"
               if decode_bytes(w, args.sinks, args.window) > 256e6
               else "L2 not flushed (working set may be L2-resident)"}
    return c


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from paged_kv_cache_466_b200 import (KVPool, pa_decode, pa_decode_num_splits,
                                         pa_decode_num_splits_lens,
                                         pa_decode_shared_prefix,
                                         pa_decode_shared_prefix_workspace_bytes,
                                         pa_decode_window, pa_decode_window_workspace_bytes,
                                         pa_decode_workspace_bytes, pa_kv_append,
                                         pa_decode_append, StepPacket, StepGraph,
                                         PA_STEP_NEWEST_PER_SEQ)

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = make_workload(args.workload, seed=rank, batch=args.batch)
    pool = KVPool(w.num_pages, w.Hkv, w.P, w.D, w.kv, dev, fill_byte=0)
    bt = torch.from_numpy(w.block_tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    q = w.q.to(dev)
    chunk = 1 << 18
    for a in range(0, len(w.prefill_seq), chunk):
        b = min(a + chunk, len(w.prefill_seq))
        pa_kv_append(pool, w.prefill_k[a:b].to(dev), w.prefill_v[a:b].to(dev),
                     torch.from_numpy(w.prefill_seq[a:b]).to(dev),
                     torch.from_numpy(w.prefill_pos[a:b]).to(dev), bt)
    sk, sv = w.step_k.to(dev), w.step_v.to(dev)
    sseq = torch.from_numpy(w.step_seq).to(dev)
    spos = torch.from_numpy(w.step_pos).to(dev)
    # the library schedules the fused step from the host's context lengths
    # (pa_decode_append with host_context_lens), as a serving loop that knows
    # them would; S is the split count that then runs
    host_lens = np.ascontiguousarray(w.context_lens, dtype=np.int32)
    fused_step = not (args.cascade or args.window > 0 or args.separate_append)
    S = (pa_decode_num_splits_lens(pool, w.B, w.max_pages, host_lens, args.splits) if fused_step
         else pa_decode_num_splits(pool, w.B, w.max_pages, args.splits))
    if args.cascade:
        pre_len = int(w.notes["prefix_tokens"])
        # the suffix decode's split count, planned over the suffix pages as the
        # library plans it
        S = pa_decode_num_splits(pool, w.B, w.max_pages - pre_len // w.P, args.splits)
        pre_pages = torch.from_numpy(w.notes["prefix_pages"].copy()).to(dev)
        nbytes = pa_decode_shared_prefix_workspace_bytes(pool, w.B, w.Hq, w.max_pages, pre_len,
                                                         args.splits)
    elif args.window > 0:
        nbytes = pa_decode_window_workspace_bytes(pool, w.B, w.Hq, w.max_pages, args.sinks,
                                                  args.window, args.splits)
    else:
        nbytes = pa_decode_workspace_bytes(w.B, w.Hq, w.D, S)
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def decode(pl, qq, tt, cc):
        if args.cascade:
            pa_decode_shared_prefix(pl, qq, pre_pages, pre_len, tt, cc, w.scale, out=out,
                                    workspace=ws, num_splits=args.splits)
        elif args.window > 0:
            pa_decode_window(pl, qq, tt, cc, w.scale, args.sinks, args.window, out=out,
                             workspace=ws, num_splits=args.splits)
        else:
            pa_decode(pl, qq, tt, cc, w.scale, out=out, workspace=ws, num_splits=S)

    # the usual decode step (one new token per sequence, at ctx - 1) runs as one
    # launch, the cache write fused into the decode; other steps as two calls
    per_seq = (w.step_rows_by_sequence()
               if not (args.cascade or args.window > 0 or args.separate_append) else None)
    fused = per_seq is not None
    if fused:
        kn, vn = per_seq[0].to(dev), per_seq[1].to(dev)

    pools = [pool]
    if args.alternate_pools:
        # a second, independent copy of the pool: steps alternate between the
        # two, so no step can find the previous step's pages in the L2
        twin = KVPool(w.num_pages, w.Hkv, w.P, w.D, w.kv, dev)
        for a_t, b_t in zip(twin.tensors(), pool.tensors()):
            a_t.copy_(b_t)
        pools.append(twin)

    def step(i=0, ev0=None, ev1=None):
        pl = pools[i % len(pools)]
        if fused:
            if ev0 is not None:
                ev0.record(stream)
            pa_decode_append(pl, q, kn, vn, bt, ctx, w.scale, out=out, workspace=ws,
                             num_splits=args.splits, host_context_lens=host_lens)
        else:
            pa_kv_append(pl, sk, sv, sseq, spos, bt)
            if ev0 is not None:
                ev0.record(stream)
            decode(pl, q, bt, ctx)
        if ev1 is not None:
            ev1.record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    for i in range(max(args.warmup, 0)):
        step(i)
    torch.cuda.synchronize()

    # ---- device-resident timed region
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    if args.flush_l2:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        flush = torch.empty(2 * max(l2, 1 << 20), dtype=torch.uint8, device=dev)
        sevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(K)]
    clocks.mark(True)
    t0.record(stream)
    for i in range(K):
        if args.flush_l2:
            flush.fill_(i & 0xFF)
            sevs[i][0].record(stream)
        step(i, *evs[i])
        if args.flush_l2:
            sevs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    clk = clocks.stop()
    barrier()
    if args.flush_l2:
        ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in sevs), world, dev)
    else:
        ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    dec_ms = [a.elapsed_time(b) for a, b in evs]
    ms_step = ms / K
    dbytes = decode_bytes(w, args.sinks, args.window)
    step_bytes = dbytes + append_bytes(w)
    value = whole_job_gbs(step_bytes, world, ms_step)

    # ---- end to end through the public API, host buffers in pinned memory
    h_q = w.q.pin_memory()
    h_k, h_v = w.step_k.pin_memory(), w.step_v.pin_memory()
    h_seq = torch.from_numpy(w.step_seq).pin_memory()
    h_pos = torch.from_numpy(w.step_pos).pin_memory()
    h_ctx = torch.from_numpy(w.context_lens).pin_memory()
    h_bt = torch.from_numpy(w.block_tables).pin_memory()
    h_out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32).pin_memory()
    d2h = h_out.numel() * h_out.element_size()
    graph = None
    if not args.cascade and args.window == 0:
        # the library's host-packet step: one H2D copy of the packed inputs,
        # append, decode and one D2H copy of the output, in one C-ABI call
        if fused:   # one row per sequence, the cache write fused into the decode
            packet = StepPacket(pool, w.B, w.Hq, w.max_pages, PA_STEP_NEWEST_PER_SEQ)
            h_k, h_v = per_seq[0].pin_memory(), per_seq[1].pin_memory()
            fills = ((packet.k_new, h_k), (packet.v_new, h_v))
        else:
            packet = StepPacket(pool, w.B, w.Hq, w.max_pages, len(w.step_seq))
            fills = ((packet.k_new, h_k), (packet.v_new, h_v), (packet.seq_idx, h_seq),
                     (packet.pos, h_pos))
        for view, h in ((packet.q, h_q), (packet.context_lens, h_ctx),
                        (packet.block_tables, h_bt)) + fills:
            view.copy_(h)
        h2d = packet.nbytes
        # the step captured once into a CUDA graph: one graph launch per step
        graph = StepGraph(pool, packet, w.scale, h_out, out_dev=out, workspace=ws, num_splits=S)

        def e2e_step():
            graph.launch(stream=stream, synchronize=True)
    else:
        h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_seq, h_pos, h_ctx,
                                                         h_bt))
        d_q, d_k, d_v = torch.empty_like(q), torch.empty_like(sk), torch.empty_like(sv)
        d_seq, d_pos = torch.empty_like(sseq), torch.empty_like(spos)
        d_ctx, d_bt = torch.empty_like(ctx), torch.empty_like(bt)

        def e2e_step():
            for d, h in ((d_q, h_q), (d_k, h_k), (d_v, h_v), (d_seq, h_seq), (d_pos, h_pos),
                         (d_ctx, h_ctx), (d_bt, h_bt)):
                d.copy_(h, non_blocking=True)
            pa_kv_append(pool, d_k, d_v, d_seq, d_pos, d_bt)
            decode(pool, d_q, d_bt, d_ctx)
            h_out.copy_(out, non_blocking=True)
            stream.synchronize()   # the caller reads the result every step

    for _ in range(max(args.warmup, 3)):
        e2e_step()
    Ke = min(K, 500)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_gbs(step_bytes, world, ems / Ke)
    if graph is not None:
        graph.close()

    peak, peak_kind = measured_peak()
    dec_avg_ms = statistics.mean(dec_ms)
    # the timed kernel: the fused step also reads the new rows and writes them
    kbytes = dbytes + (append_bytes(w) if fused else 0)
    # with shared prefix pages the roofline counts each unique byte once (the
    # logical bytes, every request's prefix included, are the metric's value)
    shared_prefix = "prefix_pages" in w.notes and not args.window
    if shared_prefix:
        kbytes = unique_bytes(w) + (append_bytes(w) if fused else 0)
    achieved = kbytes / (dec_avg_ms * 1e-3) / 1e9
    traffic = recorded_traffic(w.name) if not (args.cascade or args.window) else None
    # append, [prefix pass,] decode[, merge]; the fused step is one launch
    launches_per_step = 1 if fused else 4 if args.cascade else 2
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": {"bf16": "bf16", "u8": "u8 codes, fp32 scale/zero; fp32 accumulate",
                   "fp8": "e4m3 codes, fp32 scale; fp32 accumulate",
                   "u4": "u4 codes, fp32 scale/zero; fp32 accumulate"}[w.kv],
        "data": "synthetic (seeded N(0,1) bf16 K/V/q; no weights needed)",
        "config": config_of(w, args, world, S),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "nominal_gbs": NOMINAL_HBM_GBS,
        "pct_of_nominal": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
        "peak_gbs": peak, "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
        if peak_kind == "measured" else "fallback 6.65 TB/s",
        "seq_per_s_per_layer": round(w.B * world / (ms_step * 1e-3), 1),
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke,
                "ms_per_step": round(ems / Ke, 5)},
        "roofline": {"bound": "hbm",
                     "kernel": ("pa_decode_shared_prefix (prefix pass + decode)" if args.cascade
                                else "pa_decode_window" if args.window > 0
                                else "pa_decode_append (cache write + decode, one launch)"
                                if fused else "pa_decode (one launch, split merge fused)"),
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes": kbytes,
                     "bytes_counted": ("unique: the shared prefix once, each request's own "
                                       "tokens, q" if shared_prefix else
                                       "every attended token's K/V once, q"
                                       + (", the new rows" if fused else "")),
                     "avg_launch_ms": round(dec_avg_ms, 5)},
        "gpu_launches": K * launches_per_step,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, cores, sample = cpu_oracle_throughput(w)
        res["cpu_baseline"] = {"value": round(gbs, 3), "unit": "GB/s", "cores": cores,
                               "kind": "oracle", "sample": sample}
    return res


def cp_shard_rows(w, rank: int, world: int):
    """Rank ``rank``'s share of the batch for the context-parallel mode: the
    tokens per rank, its own tables and page count, and the (seq, pos, k, v)
    rows of its token range, taken from the same seeded workload on every
    rank."""
    import numpy as np
    from paged_kv_cache_466_b200.context_parallel import (rank_range, shard_tables,
                                                           tokens_per_rank_for)
    T = tokens_per_rank_for(int(w.context_lens.max()), world, w.P)
    begin, end = rank_range(rank, world, T)
    tables, n_pages = shard_tables(w.max_pages, w.context_lens, rank, world, T, w.P, seed=rank)
    seq, pos, k, v = w.all_rows()
    sel = np.flatnonzero((pos >= begin) & (pos < end))
    idx = __import__("torch").from_numpy(sel)
    return T, (begin, end), tables, max(n_pages, 1), (seq[sel], pos[sel], k[idx], v[idx])


def run_context_parallel(args, rank, world, local_rank):
    """The context-parallel decode of one batch over the ranks: rank r holds
    tokens [r T, (r + 1) T) of every sequence in a pool of its own, decodes them
    (pa_decode_range), all-gathers (o, lse) and merges (pa_merge_partials). A
    step is the whole decode of the batch; value = the batch's bytes over the
    slowest rank's step time."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_466_b200 import KVPool, pa_kv_append
    from paged_kv_cache_466_b200.context_parallel import decode_context_parallel

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = make_workload(args.workload, seed=0, batch=args.batch)   # the same batch everywhere
    T, (begin, end), tables, n_pages, (seq, pos, k, v) = cp_shard_rows(w, rank, world)
    pool = KVPool(n_pages, w.Hkv, w.P, w.D, w.kv, dev, fill_byte=0)
    bt = torch.from_numpy(tables).to(dev)
    ctx = torch.from_numpy(w.context_lens).to(dev)
    q = w.q.to(dev)
    chunk = 1 << 18
    for a in range(0, len(seq), chunk):
        b = min(a + chunk, len(seq))
        pa_kv_append(pool, k[a:b].to(dev), v[a:b].to(dev), torch.from_numpy(seq[a:b]).to(dev),
                     torch.from_numpy(pos[a:b]).to(dev), bt)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(qq=q):
        decode_context_parallel(pool, qq, bt, ctx, w.scale, T, out=out, num_splits=args.splits)

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    for i in range(K):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    clk = clocks.stop()
    barrier()
    per = [a.elapsed_time(b) for a, b in evs]
    ms_step = max_over_ranks(sum(per) / K, world, dev)
    batch_bytes = decode_bytes(w)
    value = batch_bytes / (ms_step * 1e-3) / 1e9
    rank_tok = int(sum(max(0, min(int(c), end) - begin) for c in w.context_lens))
    rank_bytes = rank_tok * w.Hkv * 2 * {"bf16": w.D * 2, "u8": w.D + 8, "fp8": w.D + 8,
                                         "u4": w.D // 2 + 8}[w.kv] + w.B * w.Hq * w.D * 2
    # end to end: q from pinned host memory, the decode, the output back
    h_q = w.q.pin_memory()
    h_out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32).pin_memory()
    d_q = torch.empty_like(q)

    def e2e_step():
        d_q.copy_(h_q, non_blocking=True)
        step(d_q)
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()

    for _ in range(max(args.warmup, 3)):
        e2e_step()
    Ke = min(K, 500)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1) / Ke, world, dev)
    peak, peak_kind = measured_peak()
    achieved = rank_bytes / (statistics.mean(per) * 1e-3) / 1e9
    cfg = config_of(w, args, world, 0)
    cfg["global_batch"] = w.B
    cfg["parallelism"] = (f"cp{world}: each rank holds {T} tokens of every sequence "
                          f"(the last rank the rest); one all-gather of (o, lse) per step")
    cfg["tokens_per_rank"] = T
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if w.kv == "bf16" else w.kv + " codes; fp32 accumulate",
        "data": "synthetic (seeded N(0,1) bf16 K/V/q; no weights needed)",
        "config": cfg,
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "peak_gbs": peak, "peak_kind": peak_kind,
        "seq_per_s_per_layer": round(w.B / (ms_step * 1e-3), 1),
        "e2e": {"value": round(batch_bytes / (ems * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": h_q.numel() * h_q.element_size(),
                "d2h_bytes_per_step": h_out.numel() * h_out.element_size(),
                "steps": Ke, "ms_per_step": round(ems, 5)},
        "roofline": {"bound": "hbm", "kernel": "context-parallel step on rank 0 (range "
                     "decode + all-gather + merge), its own range's bytes",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "algorithmic_bytes": rank_bytes,
                     "avg_launch_ms": round(statistics.mean(per), 5)},
        "gpu_launches": K * 2,
        "clocks": clk,
    }


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: every step a bounded sample of the
    workload (a fixed set of (sequence, head) rows), timed on the host cores."""
    import numpy as np
    if rank != 0:
        return None
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    cores = int(os.environ["OMP_NUM_THREADS"])
    import oracle
    from paged_kv_cache_466_b200.workloads import bits
    w = make_workload(args.workload, seed=0, batch=args.batch)
    hp = oracle.empty_pool(w.kv, w.num_pages, w.Hkv, w.P, w.D, 0)
    seq, pos, k, v = w.all_rows()
    oracle.scatter_rows(hp, w.block_tables, seq, pos, bits(k), bits(v))
    qb = bits(w.q)
    # calibrate: rows per step so the whole run takes about 90 s
    pairs_all = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    t0 = time.perf_counter()
    oracle.paged_attention(hp, qb, w.block_tables, w.context_lens, w.scale, pairs=pairs_all[:w.Hq])
    per_pair = max((time.perf_counter() - t0) / w.Hq, 1e-6)
    budget = 90.0 / max(args.steps + args.warmup, 1)
    n = int(min(len(pairs_all), max(1, budget / per_pair)))
    sample = pairs_all[:n]
    tok = sum(int(w.context_lens[b]) for b, _ in sample)
    per_tok = 2 * {"bf16": w.D * 2, "u8": w.D + 8, "fp8": w.D + 8, "u4": w.D // 2 + 8}[w.kv]
    sample_bytes = tok * per_tok // w.G + n * w.D * 2     # K/V rows are shared by G heads
    for _ in range(args.warmup):
        oracle.paged_attention(hp, qb, w.block_tables, w.context_lens, w.scale, pairs=sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.paged_attention(hp, qb, w.block_tables, w.context_lens, w.scale, pairs=sample)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = sample_bytes / dt / 1e9
    desc = (f"{n} (sequence, query head) rows of the {w.name} batch per step "
            f"({n / len(pairs_all):.1%} of a decode), fp64, OpenMP")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_of(w, args, 1, 1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=180))
    try:
        res = (run_context_parallel if args.context_parallel else run_ours)(
            args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
