#!/usr/bin/env python
"""Benchmark of the paged-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline]

A step is one pass of the hot path over one batch of seeded synthetic input:
reshape_and_cache of the step's new tokens, then paged decode attention
(split-KV kernel and, when a sequence spans several partitions, the
log-sum-exp merge); the mixed workload adds the chunked-prefill kernel. The
default workload is the Llama-2-7B-shaped decode batch (64 sequences,
lengths uniform in [128, 2048], 32/32 heads, head_dim 128, 16-token blocks,
bf16). Its KV read per step (about 1.1 GB) is far larger than the 126 MB L2,
so no L2 flush is needed between steps.

One process per GPU; under torchrun each rank runs its own batch (different
seed, same shape: weak scaling, no collective on the data path). Timing is
CUDA events on the launching stream between barriers; the JSON line reports
the slowest rank's time and the sum of all ranks' work.

Printed (rank 0, one JSON line): metric/value/unit (KV-read GB/s of the
decode attention, counted from the algorithmic bytes), tokens/s, the
roofline of the dominant call against the measured HBM peak, the host
oracle as a CPU baseline, an end-to-end figure through the public API with
host buffers, the kernel launch count and the SM clocks seen while timing.
``--impl reference`` times the fp64 CPU oracle instead, on bounded samples
of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (frac of HBM peak); tokens/s per batch"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# --------------------------------------------------------------------------
# process / rank plumbing
# --------------------------------------------------------------------------
def rank_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, world


def pin_device(local_rank: int, world: int):
    """Under torchrun each rank sees only its own GPU (set before CUDA starts)."""
    if world > 1:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = vis.split(",") if vis else [str(i) for i in range(64)]
        os.environ["CUDA_VISIBLE_DEVICES"] = ids[local_rank]


def init_dist(world: int, backend: str, timeout_s: int = 300):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def aggregate(units: float, ms: float, world: int, device=None):
    """Sum of every rank's work and the slowest rank's time (identical on all
    ranks). Works with any process-group backend."""
    import torch
    if world <= 1:
        return units, ms
    import torch.distributed as dist
    u = torch.tensor([units], dtype=torch.float64, device=device)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(u.item()), float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------
# work accounting
# --------------------------------------------------------------------------
def decode_bytes(batch) -> float:
    """Algorithmic bytes of one decode call: K and V of every valid token per
    kv head, q and out, each CTA's table slice, and the lengths."""
    import torch
    if batch.q is None or batch.num_seqs == 0:
        return 0.0
    e = batch.k_cache.element_size()
    eq = batch.q.element_size()
    ctx = batch.context_lens.to(torch.int64)
    H_kv, D, bs = batch.num_kv_heads, batch.head_dim, batch.block_size
    lo = torch.zeros_like(ctx)
    if batch.sliding_window > 0:  # only the window's tokens and blocks
        lo = (ctx - batch.sliding_window).clamp(min=0)
    kv = int((2 * (ctx - lo) * H_kv * D * e).sum())
    qo = 2 * batch.num_seqs * batch.num_q_heads * D * eq
    nblk = torch.where(ctx > lo, (ctx - 1) // bs - lo // bs + 1, torch.zeros_like(ctx))
    tbl = int((4 * nblk * H_kv).sum())
    return float(kv + qo + tbl + 4 * batch.num_seqs)


def decode_unique_bytes(batch) -> float:
    """K/V bytes of the distinct cached tokens the decode sequences read:
    sequences that share prefix blocks count them once (what HBM must
    deliver at least once; the logical bytes count every reader)."""
    import torch
    if batch.q is None or batch.num_seqs == 0:
        return 0.0
    bs = batch.block_size
    used = {}
    tables = batch.block_tables.tolist()
    for b, ctx in enumerate(batch.context_lens.tolist()):
        for lb in range(-(-ctx // bs)):
            blk = tables[b][lb]
            used[blk] = max(used.get(blk, 0), min(bs, ctx - lb * bs))
    e = batch.k_cache.element_size()
    return float(2 * sum(used.values()) * batch.num_kv_heads * batch.head_dim * e)


def reshape_bytes(batch) -> float:
    """Algorithmic bytes of the cache scatter: read the K and V rows of every
    non-padding token (input element size), write them into the cache (cache
    element size: 1 for the 8-bit pools), plus the slots."""
    T = int((batch.slot_mapping >= 0).sum())
    rows = 2 * T * batch.num_kv_heads * batch.head_dim  # K and V elements
    return float(rows * (batch.key.element_size() + batch.k_cache.element_size()) +
                 8 * batch.slot_mapping.numel())


def prefill_flops(batch) -> float:
    """Algorithmic FLOPs of the chunked prefill: Q.K^T and P.V over each
    query's causal range, or its band under a sliding window (4 D H_q per
    query-key pair)."""
    if batch.prefill_q is None:
        return 0.0
    qsl = batch.query_start_loc.tolist()
    ctx = batch.prefill_context_lens.tolist()
    H_q, D, W = batch.num_q_heads, batch.head_dim, batch.sliding_window
    f = 0
    for c in range(len(ctx)):
        C = qsl[c + 1] - qsl[c]
        cached = ctx[c] - C
        if W > 0:  # query at position p sees min(p + 1, W) keys
            pairs = sum(min(p + 1, W) for p in range(cached, ctx[c]))
        else:
            pairs = C * cached + C * (C + 1) // 2
        f += 4 * D * H_q * pairs
    return float(f)


def tokens_per_step(batch) -> int:
    n = batch.num_seqs
    if batch.prefill_q is not None:
        n += batch.prefill_q.shape[0]
    return n


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(
            p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_digest(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile: str, kernel_files, workload, units_scale: float = 1.0):
    """DRAM bytes per launch recorded in a committed ncu summary, or None when
    the summary is missing, was taken on another workload (its `workload`
    field against the batch name, which carries head_dim, block size and the
    cache's element type), or the kernel source changed since it was taken.
    `workload` None (a partition or pool-size override) gives None."""
    path = os.path.join(ROOT, "profiles", profile)
    try:
        text = open(path).read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        line = line.strip().lstrip("-* ")  # list items: "- key: `value`"
        if ":" in line and line.startswith(("source-sha256", "dram-bytes-per-launch",
                                            "workload")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if workload is None or fields.get("workload") != workload:
        return None
    if fields.get("source-sha256") != source_digest(kernel_files):
        return None
    try:
        return float(fields["dram-bytes-per-launch"]) * units_scale
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------
# clocks while timing (NVML reads only)
# --------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            h = None
            try:
                p = torch.cuda.get_device_properties(0)
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0]
                h = pynvml.nvmlDeviceGetHandleByIndex(int(vis) if vis.isdigit() else 0)
            self.h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, r))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if not self.ok:
            return
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self._stop.set()
        self._t.join()
        try:
            self._sample()
        except Exception:
            pass
        sms = [s for s, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        names = sorted(n for bit, n in REASONS.items() if mask & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(sms)}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def make_batch(name: str, seed: int, num_blocks=None, block_size=None, head_dim=None):
    from pagedattention_paged_kv_02_b200 import workloads as W
    kw = {}
    if num_blocks:
        kw["num_blocks"] = num_blocks
    if block_size:
        kw["block_size"] = block_size
    if head_dim:
        kw["head_dim"] = head_dim
    return W.WORKLOADS[name](seed=seed, **kw)


class Runner:
    """Holds a device batch and issues one step through the public binding."""

    def __init__(self, batch, dev):
        import torch
        from pagedattention_paged_kv_02_b200 import pa
        self.pa = pa
        self.host = batch
        self.d = batch.to(dev)
        d = self.d
        self.part = d.partition_size
        self.max_ctx = batch.max_context_len  # host-side bound, computed once
        self.ws = None
        self.S = 0
        # sequences sharing prefix blocks go through the prefix-aware decode
        self.shared = (d.decode_group_start is not None and not batch.quantized and
                       batch.sliding_window == 0 and batch.dtype == torch.bfloat16)
        if d.q is not None and d.num_seqs:
            B, H_q, D = d.q.shape
            if self.shared:
                n = pa.pa_decode_shared_prefix_workspace_size(
                    B, H_q, d.num_kv_heads, D, d.decode_prefix_lens.numel(),
                    batch.max_group_size, batch.max_prefix_len, d.max_context_len, self.part)
            else:
                n = pa.pa_decode_workspace_size(B, H_q, D, d.max_context_len, self.part)
            self.ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
            P = pa.pa_decode_partition_tokens(d.max_context_len, self.part)
            self.S = -(-d.max_context_len // P)
            self.out = torch.empty_like(d.q)
        if d.prefill_q is not None:
            self.pout = torch.empty_like(d.prefill_q)
            qsl = d.query_start_loc.cpu()
            self.max_q = int((qsl[1:] - qsl[:-1]).max())
        self._calls = self.calls()
        self.side = None  # second stream of a mixed step

    def launches_per_step(self) -> int:
        n = 1  # reshape_and_cache
        if self.d.q is not None and self.d.num_seqs and self.shared:
            n += 3 if self.host.max_prefix_len > 0 else 2  # prefix, tails, merge
        elif self.d.q is not None and self.d.num_seqs:
            n += 1 + (1 if self.S > 1 else 0)
        if self.d.prefill_q is not None:
            n += 1
        return n

    def calls(self, d=None, out=None, pout=None):
        """The step's C-ABI calls with their arguments marshalled once."""
        pa = self.pa
        d = d or self.d
        if d.k_scale is not None:
            c = {"reshape": pa.prepare_reshape_and_cache_fp8(d.key, d.value, d.k_cache, d.v_cache,
                                                             d.slot_mapping, d.k_scale,
                                                             d.v_scale)}
        else:
            c = {"reshape": pa.prepare_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache,
                                                         d.slot_mapping)}
        if d.prefill_q is not None:
            c["prefill"] = pa.prepare_prefill_chunk(
                pout if pout is not None else self.pout, d.prefill_q, d.k_cache, d.v_cache,
                d.prefill_block_tables, d.prefill_context_lens, d.query_start_loc, self.max_q,
                d.scale, self.host.sliding_window)
        if d.q is not None and d.num_seqs and d.k_scale is not None:
            c["decode"] = pa.prepare_decode_fp8(out if out is not None else self.out, d.q,
                                                d.k_cache, d.v_cache, d.k_scale, d.v_scale,
                                                d.block_tables, d.context_lens, self.max_ctx,
                                                d.scale, self.part, self.ws)
        elif d.q is not None and d.num_seqs and self.shared:
            c["decode"] = pa.prepare_decode_shared_prefix(
                out if out is not None else self.out, d.q, d.k_cache, d.v_cache, d.block_tables,
                d.context_lens, d.decode_group_start, d.decode_prefix_lens,
                self.host.max_group_size, self.host.max_prefix_len, self.max_ctx, d.scale,
                self.part, self.ws)
        elif d.q is not None and d.num_seqs:
            c["decode"] = pa.prepare_decode(out if out is not None else self.out, d.q, d.k_cache,
                                            d.v_cache, d.block_tables, d.context_lens,
                                            self.max_ctx, d.scale, self.part, self.ws,
                                            self.host.sliding_window)
        return c

    def step(self, ev=None, calls=None, stream=None):
        """One pass; ``ev`` maps a call's name ("reshape", "prefill",
        "decode") to (start, end) events recorded around it. Untimed per
        call, a mixed step's prefill and decode go on two streams: both read
        the cache the scatter just wrote and nothing of each other, so the
        GPU may run them side by side (each grid's last wave leaves SMs the
        other can use)."""
        import torch
        c = calls or self._calls
        if ev is None and "prefill" in c and "decode" in c:
            main = stream if stream is not None else torch.cuda.current_stream()
            if self.side is None:
                self.side = torch.cuda.Stream()
            c["reshape"](main)
            self.side.wait_stream(main)
            c["prefill"](self.side)
            c["decode"](main)
            main.wait_stream(self.side)
            return
        for name in ("reshape", "prefill", "decode"):
            if name in c:
                if ev is not None and name in ev:
                    ev[name][0].record()
                c[name](stream)
                if ev is not None and name in ev:
                    ev[name][1].record()

    @property
    def dominant(self):
        return "prefill" if self.d.prefill_q is not None else "decode"


def scatter_burst_ms(r, batch, dev, pair, burst=16):
    """Mean duration of one cache scatter of the step's size, over `burst`
    launches replayed from a CUDA graph, each with its own key/value rows
    and its own slots in a scratch pool (the pool is the step's shape, so
    the slots spread over the same bytes)."""
    import torch
    pa = r.pa
    T = batch.slot_mapping.numel()
    NB, H, bs, D = batch.k_cache.shape
    kc = torch.empty_like(r.d.k_cache)
    vc = torch.empty_like(r.d.v_cache)
    g = torch.Generator(device=dev).manual_seed(1234)
    n_slots = NB * bs
    per = min(T, n_slots // burst)
    perm = torch.randperm(n_slots, generator=g, device=dev)
    calls = []
    for i in range(burst):
        key = torch.randn(per, H, D, generator=g, device=dev).to(batch.key.dtype)
        val = torch.randn(per, H, D, generator=g, device=dev).to(batch.key.dtype)
        slots = perm[i * per:(i + 1) * per].to(torch.int64).contiguous()
        if batch.k_scale is not None:
            c = pa.prepare_reshape_and_cache_fp8(key, val, kc, vc, slots, r.d.k_scale, r.d.v_scale)
        else:
            c = pa.prepare_reshape_and_cache(key, val, kc, vc, slots)
        calls.append((c, key, val, slots))
    bg = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(bg, stream=side):
            for c, *_ in calls:
                c(side)
    torch.cuda.current_stream().wait_stream(side)
    bg.replay()
    b0, b1 = pair()
    b0.record()
    bg.replay()
    b1.record()
    torch.cuda.synchronize()
    # scaled to the step's token count when a launch moved fewer
    return b0.elapsed_time(b1) / burst * (T / per)


def run_ours(args, rank, world):
    import torch
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dist = init_dist(world, "nccl")
    batch = make_batch(args.workload, seed=rank, num_blocks=args.num_blocks,
                       block_size=args.block_size, head_dim=args.head_dim)
    if args.partition is not None:
        batch.partition_size = args.partition
    batch.sliding_window = args.window
    r = Runner(batch, dev)
    hbm, bf16, bf16_sus, basis = load_peaks()

    dbytes = decode_bytes(batch)
    rbytes = reshape_bytes(batch)
    pflops = prefill_flops(batch)

    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()

    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    # the step, back to back, timed as a whole (no events between steps):
    # its launches captured once in a CUDA graph and replayed (launch-bound
    # steps such as the tiny batch run 3x faster), or issued one by one with
    # --eager; the calls marshal nothing per step either way
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                r.step(stream=side)
        torch.cuda.current_stream().wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
    t0.record()
    for i in range(K):
        if graph is not None:
            graph.replay()
        else:
            r.step()
    t1.record()
    torch.cuda.synchronize()
    # the same K steps again, events around the dominant call of each, for
    # its roofline
    pair = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    evs = [{n: pair() for n in r._calls} for _ in range(K)]
    for i in range(K):
        r.step(evs[i])
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms_local = t0.elapsed_time(t1) / K
    call_ms = lambda n: [e[n][0].elapsed_time(e[n][1]) for e in evs]
    dom_all = sorted(call_ms(r.dominant))
    dom_ms = statistics.fmean(dom_all)
    dec_ms = statistics.fmean(call_ms("decode")) if "decode" in r._calls else None
    # the scatter is a few microseconds: events around one launch measure
    # mostly the launch itself, so its duration is taken over a burst of
    # back-to-back launches replayed from one CUDA graph. Each launch of the
    # burst moves its own rows (fresh inputs, distinct slots of a scratch
    # pool of the same shape), so that neither the rows read nor the lines
    # written are still in L2 from the launch before.
    rs_ms = scatter_burst_ms(r, batch, dev, pair)
    pct = lambda q: dom_all[min(len(dom_all) - 1, int(q * len(dom_all)))]

    units = dbytes if r.dominant == "decode" else pflops
    total_units, ms = aggregate(units, ms_local, world, dev)
    tok_total, _ = aggregate(float(tokens_per_step(batch)), ms_local, world, dev)
    dbytes_total, _ = aggregate(dbytes, ms_local, world, dev)

    # end to end through the public API: every step copies its inputs from
    # pinned host memory and reads its result back. Two staging buffers and a
    # copy stream let step i+1's upload and step i's download overlap step
    # i's kernels; the compute stream waits for each upload it consumes.
    import copy
    names = ["key", "value", "slot_mapping"]
    if batch.q is not None:
        names += ["q", "block_tables", "context_lens"]
        if r.shared:
            names += ["decode_group_start", "decode_prefix_lens"]
    if batch.prefill_q is not None:
        names += ["prefill_q", "prefill_block_tables", "prefill_context_lens", "query_start_loc"]
    # the step's inputs packed into one pinned buffer (one upload per step)
    offs, total = {}, 0
    for n in names:
        t = getattr(batch, n)
        offs[n] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_flat = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    for n in names:
        t = getattr(batch, n).contiguous()
        nb = t.numel() * t.element_size()
        h_flat[offs[n]:offs[n] + nb].copy_(t.view(-1).view(torch.uint8))
    h2d = sum(getattr(batch, n).numel() * getattr(batch, n).element_size() for n in names)
    res_name = "q" if batch.q is not None else "prefill_q"
    out_shape = getattr(batch, res_name).shape
    out_dtype = batch.dtype
    d_flats, bufs, outs, pouts, out_hs, bcalls = [], [], [], [], [], []
    for _ in range(2):
        flat = torch.empty(total, dtype=torch.uint8, device=dev)
        dd = copy.copy(r.d)
        for n in names:
            t = getattr(batch, n)
            nb = t.numel() * t.element_size()
            setattr(dd, n, flat[offs[n]:offs[n] + nb].view(t.dtype).view(t.shape))
        d_flats.append(flat)
        bufs.append(dd)
        outs.append(torch.empty_like(r.d.q) if batch.q is not None else None)
        pouts.append(torch.empty_like(r.d.prefill_q) if batch.prefill_q is not None else None)
        out_hs.append(torch.empty(out_shape, dtype=out_dtype, pin_memory=True))
        bcalls.append(r.calls(d=dd, out=outs[-1], pout=pouts[-1]))
    d2h = out_hs[0].numel() * out_hs[0].element_size()
    up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()  # uploads never queue behind downloads
    up_done = [torch.cuda.Event() for _ in range(2)]
    used = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, comp):
        """n steps on stream comp, alternating the two staging buffers: step
        i's upload waits for step i-2's compute (same buffer), its compute for
        its upload and for step i-2's download. The first two steps of a run
        fork from comp's position."""
        up_s.wait_stream(comp)
        down_s.wait_stream(comp)
        for i in range(n):
            k = i % 2
            if i >= 2:
                up_s.wait_event(used[k])      # buffer k's previous step is done with it
            with torch.cuda.stream(up_s):
                d_flats[k].copy_(h_flat, non_blocking=True)
            up_done[k].record(up_s)
            comp.wait_event(up_done[k])
            if i >= 2:
                comp.wait_event(down_done[k])  # its previous result has been read back
            r.step(calls=bcalls[k], stream=comp)
            used[k].record(comp)
            down_s.wait_event(used[k])
            with torch.cuda.stream(down_s):
                out_hs[k].copy_(outs[k] if outs[k] is not None else pouts[k], non_blocking=True)
            down_done[k].record(down_s)
        comp.wait_stream(up_s)
        comp.wait_stream(down_s)

    # the steps, uploads and downloads included, captured as CUDA graphs of
    # up to 32 steps (the host issue cost of a step's dozen stream operations
    # would otherwise exceed a short step's device time); replays of one
    # graph serialise on the stream, so the upload/download pipeline drains
    # once per graph: the longer the graph, the less that costs per step
    comp = torch.cuda.current_stream()
    e2e_graphs = {}
    if args.graph:
        side = torch.cuda.Stream()
        G = min(32, K)
        for n in sorted({G, K % G} - {0}):
            g = torch.cuda.CUDAGraph()
            side.wait_stream(comp)
            with torch.cuda.stream(side):
                with torch.cuda.graph(g, stream=side):
                    e2e_steps(n, side)
            comp.wait_stream(side)
            e2e_graphs[n] = g
        torch.cuda.synchronize()

    def e2e_run(n_steps):
        if not e2e_graphs:
            e2e_steps(n_steps, comp)
            return
        g_len = max(e2e_graphs)
        for _ in range(n_steps // g_len):
            e2e_graphs[g_len].replay()
        if n_steps % g_len:
            e2e_graphs[n_steps % g_len].replay()

    if e2e_graphs:  # warm-up: every captured graph once
        for g in e2e_graphs.values():
            g.replay()
    else:
        e2e_run(max(3, args.warmup // 4))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    e2e_run(K)
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms_local = e0.elapsed_time(e1) / K
    _, e2e_ms = aggregate(0.0, e2e_ms_local, world, dev)

    line = None
    wtag = f"_window{args.window}" if args.window else ""
    # the workload a committed profile must have been taken on for its DRAM
    # bytes to stand for this run's launch
    pwl = batch.name if args.partition is None and not args.num_blocks else None
    if rank == 0:
        if r.dominant == "decode":
            value = dbytes_total / (ms * 1e-3) / 1e9
            unit = "GB/s"
            achieved = dbytes / (dom_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                    "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "peak_basis": f"{basis} hbm_gbs",
                    "kernel": ("pa_decode_fp8 (decode_split_q8 + merge)" if batch.fp8 else
                               "pa_decode_int8 (decode_split_q8 + merge)" if batch.int8 else
                               "pa_decode (decode_split + merge)"),
                    "alg_bytes_per_launch": dbytes,
                    "traffic": profiled_traffic(f"decode_{args.workload}{wtag}.md",
                                                DECODE_FP8_SOURCES if batch.quantized
                                                else DECODE_SOURCES, pwl)}
        else:
            value = dbytes_total / (ms * 1e-3) / 1e9
            unit = "GB/s"
            achieved = pflops / (dom_ms * 1e-3) / 1e12
            # the prefill launch is timed alone (events around one ~0.2 ms
            # call), so against the burst GEMM rate, not the sustained one
            roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": bf16,
                    "unit": "TFLOP/s", "frac": round(achieved / bf16, 4),
                    "peak_basis": f"{basis} bf16_tflops (burst)",
                    "frac_of_sustained": round(achieved / bf16_sus, 4),
                    "kernel": "pa_prefill_chunk", "alg_flops_per_launch": pflops,
                    "traffic": profiled_traffic(f"prefill_{args.workload}{wtag}.md",
                                                PREFILL_SOURCES, pwl)}
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("e4m3 KV / bf16 q" if batch.fp8 else "int8 KV / bf16 q" if batch.int8 else
                      "bf16" if batch.dtype.itemsize == 2 else "f32"),
            "data": "synthetic (seeded; one batch per rank)",
            "config": {**workload_config(batch, args.workload, world, r), **_graph_note(args)},
            "tokens_per_s": round(tok_total / (ms * 1e-3), 1),
            "frac_of_hbm_peak": round(value / world / hbm, 4),
            "frac_of_nominal_8tbs": round(value / world / 8000.0, 4),
            "roofline": roof,
            "e2e": {"value": round(dbytes_total / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 5)},
            "gpu_launches": K * r.launches_per_step(),  # in the region `value` is timed on
            "clocks": clk,
            "dominant_call_ms": {"mean": round(dom_ms, 5), "p10": round(pct(0.1), 5),
                                 "p50": round(pct(0.5), 5), "p90": round(pct(0.9), 5)},
        }
        # the cache scatter against HBM: its algorithmic bytes over its own
        # event-timed duration (the same pass as the dominant call's)
        line["roofline_reshape"] = {
            "bound": "hbm", "achieved": round(rbytes / (rs_ms * 1e-3) / 1e9, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(rbytes / (rs_ms * 1e-3) / 1e9 / hbm, 4),
            "peak_basis": f"{basis} hbm_gbs", "kernel": "pa_reshape_and_cache",
            "alg_bytes_per_launch": rbytes, "ms": round(rs_ms, 5),
            "traffic": profiled_traffic(f"reshape_{args.workload}.md", RESHAPE_SOURCES, pwl)}
        if r.dominant != "decode":
            line["prefill_tflops"] = round(pflops * world / (ms * 1e-3) / 1e12, 1)
            # the decode part of the mixed step reads shared prefix blocks
            # through many tables: logical bytes (value) and distinct bytes
            ubytes = decode_unique_bytes(batch)
            line["decode_bytes_per_step"] = {"logical": dbytes, "unique_kv": ubytes}
            if dec_ms:
                # its roofline on the bytes HBM must deliver at least once
                line["roofline_decode"] = {
                    "bound": "hbm", "achieved": round(ubytes / (dec_ms * 1e-3) / 1e9, 1),
                    "peak": hbm, "unit": "GB/s",
                    "frac": round(ubytes / (dec_ms * 1e-3) / 1e9 / hbm, 4),
                    "peak_basis": f"{basis} hbm_gbs", "basis": "distinct K/V bytes",
                    "kernel": ("pa_decode_shared_prefix (prefix + tails + merge)" if r.shared
                               else "pa_decode (decode_split + merge)"),
                    "ms": round(dec_ms, 5), "logical_bytes_GBps": round(
                        dbytes / (dec_ms * 1e-3) / 1e9, 1),
                    "traffic": (profiled_traffic(f"decode_shared_prefix_{args.workload}.md",
                                                 SHARED_DECODE_SOURCES, pwl)
                                if r.shared else None)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(batch, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


DECODE_SOURCES = ["pagedattention_paged_kv_02_b200/csrc/decode.cuh",
                  "pagedattention_paged_kv_02_b200/csrc/pa_device.cuh"]
PREFILL_SOURCES = ["pagedattention_paged_kv_02_b200/csrc/prefill.cuh",
                   "pagedattention_paged_kv_02_b200/csrc/pa_device.cuh"]
DECODE_FP8_SOURCES = DECODE_SOURCES + ["pagedattention_paged_kv_02_b200/csrc/decode_fp8.cuh"]
RESHAPE_SOURCES = ["pagedattention_paged_kv_02_b200/csrc/reshape_and_cache.cuh",
                   "pagedattention_paged_kv_02_b200/csrc/pa_device.cuh"]
SHARED_DECODE_SOURCES = ["pagedattention_paged_kv_02_b200/csrc/decode.cuh",
                         "pagedattention_paged_kv_02_b200/csrc/decode_prefix.cuh",
                         "pagedattention_paged_kv_02_b200/csrc/decode_merge.cuh",
                         "pagedattention_paged_kv_02_b200/csrc/pa_device.cuh"]


def workload_config(batch, name, world, r=None):
    c = {"workload": batch.name, "name": name, "block_size": batch.block_size,
         "num_q_heads": batch.num_q_heads, "num_kv_heads": batch.num_kv_heads,
         "head_dim": batch.head_dim, "num_blocks": batch.num_blocks,
         "parallelism": f"dp{world} (independent batches, no collective)",
         "l2": "no flush: inputs larger than L2 (KV read per step >> 126 MB)"}
    if batch.q is not None and batch.num_seqs:
        lens = batch.context_lens
        c.update({"num_seqs": batch.num_seqs, "context_len_mean": round(float(lens.float().mean()), 1),
                  "context_len_max": int(lens.max()),
                  "partition_tokens": None if r is None else
                  r.pa.pa_decode_partition_tokens(batch.max_context_len, batch.partition_size)})
    if batch.prefill_q is not None:
        c.update({"prefill_chunks": batch.query_start_loc.numel() - 1,
                  "prefill_tokens": batch.prefill_q.shape[0]})
    if batch.sliding_window > 0:
        c["sliding_window"] = batch.sliding_window
    return c


def _graph_note(args):
    return {"launch": "cuda_graph_replay" if getattr(args, "graph", False) else "eager"}


# --------------------------------------------------------------------------
# the fp64 host oracle as a baseline
# --------------------------------------------------------------------------
def _oracle_step(batch, k, v, select=None, pselect=None):
    import oracle
    if batch.fp8:
        oracle.reshape_and_cache_e4m3(batch.key, batch.value, k, v, batch.slot_mapping,
                                      batch.k_scale, batch.v_scale)
        oracle.decode_e4m3(batch.q, k, v, batch.k_scale, batch.v_scale, batch.block_tables,
                           batch.context_lens, batch.scale, select=select)
        return
    if batch.int8:
        oracle.reshape_and_cache_int8(batch.key, batch.value, k, v, batch.slot_mapping,
                                      batch.k_scale, batch.v_scale)
        oracle.decode_int8(batch.q, k, v, batch.k_scale, batch.v_scale, batch.block_tables,
                           batch.context_lens, batch.scale, select=select)
        return
    oracle.reshape_and_cache(batch.key, batch.value, k, v, batch.slot_mapping)
    W = batch.sliding_window
    if batch.prefill_q is not None:
        if W > 0:
            oracle.prefill_window(batch.prefill_q, k, v, batch.prefill_block_tables,
                                  batch.prefill_context_lens, batch.query_start_loc, batch.scale,
                                  W, select=pselect)
        else:
            oracle.prefill(batch.prefill_q, k, v, batch.prefill_block_tables,
                           batch.prefill_context_lens, batch.query_start_loc, batch.scale,
                           select=pselect)
    if batch.q is not None and batch.num_seqs:
        if W > 0:
            oracle.decode_window(batch.q, k, v, batch.block_tables, batch.context_lens,
                                 batch.scale, W, select=select)
        else:
            oracle.decode(batch.q, k, v, batch.block_tables, batch.context_lens, batch.scale,
                          select=select)


def _sample_masks(batch, frac: float, offset: int):
    """Boolean masks selecting about ``frac`` of the (row, head) outputs,
    rotated by ``offset`` so that successive samples cover different rows."""
    import torch
    sel = psel = None
    if batch.q is not None and batch.num_seqs:
        n = batch.num_seqs * batch.num_q_heads
        k = max(1, int(round(frac * n)))
        idx = (torch.arange(k) * max(1, n // k) + offset) % n
        sel = torch.zeros(n, dtype=torch.bool)
        sel[idx] = True
    if batch.prefill_q is not None:
        n = batch.prefill_q.shape[0] * batch.num_q_heads
        k = max(1, int(round(frac * n)))
        idx = (torch.arange(k) * max(1, n // k) + offset) % n
        psel = torch.zeros(n, dtype=torch.bool)
        psel[idx] = True
    return sel, psel


def cpu_baseline(batch, seconds: float):
    """The oracle as it stands on this host's cores: whole-batch steps (or, for
    workloads whose full step is too slow, evenly spaced samples of it)
    repeated for about ``seconds``; value in the metric's unit."""
    import oracle
    k, v = batch.k_cache, batch.v_cache  # host pool; appending in place is idempotent
    t = time.perf_counter()
    sel, psel = _sample_masks(batch, 1.0 / 64, 0)
    _oracle_step(batch, k, v, sel, psel)
    probe = (time.perf_counter() - t) * 64
    frac = 1.0 if probe < seconds / 2 else max(1e-4, seconds / 2 / probe)
    reps, t0 = 0, time.perf_counter()
    while True:
        sel, psel = (None, None) if frac >= 1.0 else _sample_masks(batch, frac, reps * 7919)
        _oracle_step(batch, k, v, sel, psel)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    work = decode_bytes(batch) * frac * reps
    sample = ("whole batch" if frac >= 1.0 else f"{frac:.4%} of the batch's (row, head) outputs"
              ) + f", {reps} step(s) in {dt:.1f} s"
    return {"value": round(work / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": sample}


def run_reference(args, rank, world):
    """The oracle on the host cores, K timed steps of bounded samples."""
    if rank != 0:
        return
    import oracle
    batch = make_batch(args.workload, seed=0, num_blocks=args.num_blocks)
    batch.sliding_window = args.window
    k, v = batch.k_cache, batch.v_cache
    total = args.steps + args.warmup
    t = time.perf_counter()
    sel, psel = _sample_masks(batch, 1.0 / 64, 0)
    _oracle_step(batch, k, v, sel, psel)
    full = (time.perf_counter() - t) * 64
    budget = max(0.02, args.reference_seconds / max(1, total))
    frac = min(1.0, budget / full)
    for i in range(args.warmup):
        s, ps = _sample_masks(batch, frac, i * 104729)
        _oracle_step(batch, k, v, s, ps)
    t0 = time.perf_counter()
    for i in range(args.steps):
        s, ps = _sample_masks(batch, frac, (i + args.warmup) * 104729)
        _oracle_step(batch, k, v, s, ps)
    dt = time.perf_counter() - t0
    ms = dt / args.steps * 1e3
    value = decode_bytes(batch) * frac / (ms * 1e-3) / 1e9
    sample = f"{frac:.4%} of the batch's (row, head) outputs per step"
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": workload_config(batch, args.workload, world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                             "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_block_copies(args, rank, world):
    """Auxiliary workloads for the block-copy row: ``cow_copy`` copies 1024
    whole blocks inside the Llama-7B-shaped pool (copy-on-write), ``swap_out``
    moves 256 blocks to a pinned host pool. Bytes = read + write of K and V."""
    import torch
    from pagedattention_paged_kv_02_b200 import pa
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    H, bs, D, NB = 32, 16, 128, 4096
    g = torch.Generator(device=dev).manual_seed(rank)
    k = torch.randn(NB, H, bs, D, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(NB, H, bs, D, device=dev, generator=g).to(torch.bfloat16)
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(rank))
    if args.workload == "cow_copy":
        n = 1024
        mapping = torch.stack([perm[:n], perm[n:2 * n]], 1).contiguous().to(dev)
        call = lambda: pa.pa_copy_blocks(k, v, mapping)
        where = "device pool -> same pool"
    else:
        n = 256
        hk = torch.empty(n, H, bs, D, dtype=torch.bfloat16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        mapping = torch.stack([perm[:n], torch.arange(n)], 1).contiguous().to(dev)
        call = lambda: pa.pa_swap_blocks(k, v, hk, hv, mapping)
        where = "device pool -> pinned host pool"
    block_bytes = H * bs * D * 2
    nbytes = 2 * 2 * n * block_bytes  # K and V, read and write
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        call()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    hbm, _, _, basis = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"metric": f"whole-block copy GB/s ({where}; read+write bytes)", "value": round(gbs, 1),
            "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": args.workload, "pairs": n,
                                            "block_bytes_per_cache": block_bytes},
            "frac_of_hbm_peak": round(gbs / hbm, 4) if args.workload == "cow_copy" else None,
            "peak_basis": f"{basis} hbm_gbs", "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama7b_decode",
                    choices=["tiny_fp32", "llama7b_decode", "gqa_decode", "long_context_decode",
                             "mixed_prefill_decode", "llama7b_decode_fp8", "gqa_decode_fp8",
                             "llama7b_decode_int8", "gqa_decode_int8",
                             "cow_copy", "swap_out"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--partition", type=int, default=None,
                    help="decode KV partition tokens (0 automatic, <0 no split)")
    ap.add_argument("--block-size", type=int, default=None, choices=[16, 32, 64],
                    help="block size override for the decode workloads (pool bytes kept)")
    ap.add_argument("--head-dim", type=int, default=None, choices=[64, 128],
                    help="head_dim override for llama7b_decode, gqa_decode and "
                         "mixed_prefill_decode")
    ap.add_argument("--num-blocks", type=int, default=None,
                    help="physical pool size override (a smaller pool for profiler captures)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window: each query sees only its last W positions "
                         "(0: the whole context); not for the FP8 workloads")
    ap.add_argument("--eager", dest="graph", action="store_false",
                    help="time the step as individual launches instead of replays of one "
                         "CUDA graph capture of it")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.head_dim and args.workload not in ("llama7b_decode", "gqa_decode",
                                               "mixed_prefill_decode"):
        ap.error("--head-dim applies to llama7b_decode, gqa_decode and mixed_prefill_decode")
    if args.window < 0 or (args.window and args.workload.endswith(("_fp8", "_int8"))):
        ap.error("--window takes W > 0 and a bf16/fp32 workload")
    rank, local, world = rank_env()
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    pin_device(local, world)
    if args.workload in ("cow_copy", "swap_out"):
        run_block_copies(args, rank, world)
        return
    run_ours(args, rank, world)


if __name__ == "__main__":
    main()
