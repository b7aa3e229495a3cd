#!/usr/bin/env python
"""Paged-decode benchmark: KV-read GB/s (and % of HBM peak), attention tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--partition P] [--no-cpu-baseline]

One step is one pass of the hot path over one batch: copy_blocks (when the
batch has copy-on-write pairs), reshape_and_cache of the step's new tokens,
and paged_attn_decode of every sequence.  Inputs are seeded synthetic data
(paged_kv_cache_394_b200.workloads); the default workload is the
LLaMA-7B-shaped decode layer (64 sequences, 32 heads, head_dim 128, block 16,
fp16, context lengths uniform in [128, 2048]).

`value` is the step's algorithmic bytes (K+V read by decode, q read, out
written, plus the bytes the cache write and block copy move) over the
device-timed step, summed over ranks.  Under torchrun each rank runs its own
replica batch (weak scaling, no collective on the data path); the step time is
the max over ranks.  `e2e` times the same step through the host-buffer entry
point, with the step's inputs copied from pinned host memory and the output
read back inside the timed region.

A workload name with the suffix ``_fp8`` (e.g. ``llama7b_fp8``) runs the
same batch with E4M3 caches: the quantising cache write and the E4M3 decode.

`--impl reference` times the CPU oracle on the host cores instead (rank 0
only), each step a bounded sample of the same workload.
"""

import argparse
import hashlib

import numpy as np
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
# per-cache E4M3 scales of the *_fp8 workloads: N(0,1) values reach about 6
FP8_K_SCALE = FP8_V_SCALE = 6.0 / 448.0
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; barrier and max-reduce only)
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend, timeout_s=120):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, device=None):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def replica_seed(base_seed, rank):
    """Each rank draws its own replica batch of the same shape."""
    return base_seed + 7919 * rank


# ---------------------------------------------------------------------------
# bytes
# ---------------------------------------------------------------------------
def decode_bytes(w, kv_elem=2):
    """Algorithmic bytes of one decode call: K and V of every cached token of
    every kv head (``kv_elem`` bytes per element: 2, or 1 for E4M3), q read
    and out written (16-bit)."""
    kv = 2 * int(w.context_lens.astype("int64").sum()) * w.num_kv_heads * w.head_dim * kv_elem
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * 2
    return kv + qo


def unique_decode_bytes(w, kv_elem=2):
    """decode_bytes with every physical block counted once: each distinct
    block contributes the most tokens any sequence reads from it.  Equal to
    decode_bytes when no block is shared (prefix sharing makes it smaller)."""
    import numpy as np
    most = {}
    for i, c in enumerate(w.context_lens.astype(np.int64)):
        nblk = -(-int(c) // w.block_size)
        for j, b in enumerate(w.block_tables[i, :nblk]):
            used = min(w.block_size, int(c) - j * w.block_size)
            if used > most.get(int(b), 0):
                most[int(b)] = used
    kv = 2 * sum(most.values()) * w.num_kv_heads * w.head_dim * kv_elem
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * 2
    return kv + qo


def write_bytes(w, kv_elem=2):
    """reshape_and_cache: read key and value (16-bit), write them
    (``kv_elem`` bytes per element), read the slots."""
    t = len(w.slot_mapping)
    return 2 * t * w.num_kv_heads * w.head_dim * (2 + kv_elem) + 8 * t


def copy_bytes(w, kv_elem=2):
    """copy_blocks: read and write K and V of every copied block, read the pairs."""
    blk = w.num_kv_heads * w.block_size * w.head_dim * kv_elem
    return len(w.cow_pairs) * (2 * 2 * blk + 16)


def step_bytes(w, kv_elem=2):
    return decode_bytes(w, kv_elem) + write_bytes(w, kv_elem) + copy_bytes(w, kv_elem)


def prefill_flops(w):
    """Algorithmic FLOPs of one prefill call: for every query row, q.K and P.V
    over the keys it sees (position + 1 of them), 2 FLOPs per multiply-add."""
    import numpy as np
    q_len = np.diff(w.query_start).astype(np.int64)
    hist = w.context_lens.astype(np.int64) - q_len
    # sum over sequences of sum_{j<q_len} (hist + j + 1)
    keys = int((q_len * hist + q_len * (q_len + 1) // 2).sum())
    return 4 * keys * w.num_heads * w.head_dim


def tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        self.t_start = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.t_stop = time.time()
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
               "reasons": reasons, "samples": len(rows),
               "power_w_max": max(power) if power else None}
        if self.t_stop - self.t_start < 0.6:
            out["note"] = "timed region shorter than the 200 ms sampling period"
        return out


# ---------------------------------------------------------------------------
# peaks and the committed ncu traffic summary
# ---------------------------------------------------------------------------
def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# device code and the host code that picks its launch shapes
DECODE_SOURCES = ("common.cuh", "paged_attn_kernels.cuh", "paged_attn_decode.cu")
PREFILL_SOURCES = ("common.cuh", "paged_prefill_kernels.cuh", "paged_prefill_tc_kernels.cuh",
                   "paged_attn_prefill.cu")
# cascade decode: the shared-prefix pass, the suffix decode and the merge
CASCADE_SOURCES = DECODE_SOURCES + PREFILL_SOURCES[1:] + ("paged_attn_cascade.cu",)


def kernel_source_hash(sources=DECODE_SOURCES):
    """Hash of one kernel family's sources (kernels, helpers, launch shapes)
    with comments and blank lines left out, so that editing a comment does not
    mark counters taken on the same code as stale."""
    csrc = os.path.join(ROOT, "paged_kv_cache_394_b200", "csrc")
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(csrc, f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        code = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
        h.update(f.encode() + b"\0" + "\n".join(ln for ln in code if ln).encode())
    return h.hexdigest()[:16]


def committed_traffic(workload, kind="decode"):
    """DRAM bytes per launch of the workload's dominant kernel (cascade decode:
    of its three launches together) from profiles/, if the counters were taken
    on the current device code."""
    sources = (PREFILL_SOURCES if kind == "prefill" else
               CASCADE_SOURCES if "_cascade" in workload else DECODE_SOURCES)
    path = os.path.join(ROOT, "profiles", "paged_%s_%s_traffic.md" % (kind, workload))
    try:
        text = open(path).read()
    except OSError:
        return None
    m_src = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    if not (m_src and m_b) or m_src.group(1) != kernel_source_hash(sources):
        return None
    return float(m_b.group(1))


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
# Timed beside the headline workload in the default run (one GPU): the other
# decode configurations (long-context split-K, grouped-query chat, parallel
# sampling with and without cascade), E4M3 caches and chunked prefill, each a
# nested object of the headline line with its own value, roofline and clocks.
OTHER_WORKLOADS = ("llama7b_fp8", "long_splitk", "long_splitk_fp8", "gqa_chat", "gqa_chat_fp8",
                   "prefix_share", "prefix_share_cascade", "prefix_share_cascade_fp8",
                   "llama7b_prefill",
                   "llama7b_prefill_fp8", "gqa_prefill", "gqa_prefill_fp8", "skew_prefill")


def split_name(workload):
    """(base workload, E4M3 cache?, cascade decode?) of a bench workload name."""
    from paged_kv_cache_394_b200 import workloads as W
    fp8 = workload.endswith("_fp8")
    cascade = workload.removesuffix("_fp8").endswith("_cascade")
    base = workload.removesuffix("_fp8").removesuffix("_cascade")
    if base not in W.NAMES + W.PREFILL_NAMES:
        raise ValueError("unknown workload %r" % workload)
    if cascade and base != "prefix_share":
        raise ValueError("cascade decode needs the prefix-sharing workload (prefix_share_cascade)")
    return base, fp8, cascade


class Run:
    """Process-wide state of our arm: ranks, device, and the last workload
    drawn (a variant of the same base workload reuses it)."""

    def __init__(self, args):
        import torch
        self.args = args
        self.rank, self.world = init_dist("nccl") if dist_env()[1] > 1 else (0, 1)
        self.local = dist_env()[2]
        torch.cuda.set_device(self.local)
        self.dev = torch.device("cuda", self.local)
        self._cached = (None, None)

    def workload(self, base):
        from paged_kv_cache_394_b200 import pagedkv as pk
        from paged_kv_cache_394_b200 import workloads as W
        if self._cached[0] != base:
            self._cached = (None, None)    # drop the previous pool before drawing the next
            seed = replica_seed(W.SEED_BASE + (W.NAMES + W.PREFILL_NAMES).index(base), self.rank)
            # parallel sampling: the library's C++ allocator lays out the shared
            # prompt blocks and makes the step's copy-on-write pairs
            self._cached = (base, W.make(base, seed=seed, allocator=pk.BlockAllocator))
        return self._cached[1]


def device_caches(pk, w, dev, fp8):
    """q, key, value and the caches on the device; with fp8 the pool is
    quantised once by the device's own E4M3 cache write (set-up, untimed)."""
    import numpy as np
    import torch
    tdt = torch.float16 if w.dtype == "fp16" else torch.bfloat16

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(tdt)
    q, kc, vc, key, val = up(w.q), up(w.k_cache), up(w.v_cache), up(w.key), up(w.value)
    scales = None
    if fp8:
        nb, hkv, bs, d = kc.shape
        ks8 = torch.full((hkv,), FP8_K_SCALE, dtype=torch.float32, device=dev)
        vs8 = torch.full((hkv,), FP8_V_SCALE, dtype=torch.float32, device=dev)
        k8 = torch.empty(kc.shape, dtype=torch.uint8, device=dev)
        v8 = torch.empty_like(k8)
        every = torch.arange(nb * bs, dtype=torch.int64, device=dev)
        tok = lambda c: c.permute(0, 2, 1, 3).reshape(nb * bs, hkv, d).contiguous()
        pk.reshape_and_cache_fp8(tok(kc), tok(vc), k8, v8, every, ks8, vs8)
        torch.cuda.synchronize(dev)
        kc, vc, scales = k8, v8, (ks8, vs8)
    return q, kc, vc, key, val, scales


TIMING_NOTE = {False: "the timed steps captured once in a CUDA graph, replayed between two "
                      "events on the step's stream",
               True: "the timed steps launched directly between two events on the step's stream"}


def time_steps(run, stream, step, n, graph=False):
    """n back-to-back steps between two CUDA events on `stream`, bracketed by
    a barrier and a synchronize on both sides; the max over ranks, per step,
    with the clocks sampled meanwhile.  With `graph` the n steps are captured
    once into a CUDA graph (untimed) and the timed region replays it, so the
    host's launch calls do not gap the device; the device work is the same
    n steps."""
    import torch
    g = None
    if graph:
        torch.cuda.synchronize(run.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step(i)
        with torch.cuda.stream(stream):
            g.replay()                     # untimed: the first launch uploads the graph
        torch.cuda.synchronize(run.dev)
    clocks = ClockSampler(run.local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(run.dev)
    torch.cuda.synchronize(run.dev)
    t0.record(stream)
    if g is not None:
        with torch.cuda.stream(stream):
            g.replay()
    else:
        for i in range(n):
            step(i)
    t1.record(stream)
    torch.cuda.synchronize(run.dev)
    barrier(run.dev)
    clk = clocks.stop()
    return max_over_ranks(t0.elapsed_time(t1), run.dev) / n, clk


def time_kernel(run, stream, launch, est_ms):
    """The dominant kernel alone, in its own loops after the timed steps, each
    after --warmup untimed launches, each launch between two CUDA events on
    `stream`:
      * as many launches as the timed region has steps (the roofline's
        average launch duration);
      * a sustained loop of about --kernel-seconds, with the clocks sampled
        meanwhile (a long HBM- or tensor-bound loop can reach the board's
        power cap, which lowers the SM clock: reported, not hidden).
    Returns (average ms, launches, sustained average ms, sustained launches,
    sustained clocks)."""
    import torch

    def loop(n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for _ in range(run.args.warmup):   # untimed: the clocks come back up after the pause
            launch()
        torch.cuda.synchronize(run.dev)
        for a, b in ev:
            a.record(stream)
            launch()
            b.record(stream)
        torch.cuda.synchronize(run.dev)
        return statistics.mean(a.elapsed_time(b) for a, b in ev)
    n = max(1, run.args.steps)
    avg = loop(n)
    n_long = int(min(20000, max(50, math.ceil(run.args.kernel_seconds * 1e3 / max(est_ms, 1e-3)))))
    clocks = ClockSampler(run.local)
    clocks.start()
    avg_long = loop(n_long)
    clk = clocks.stop()
    return avg, n, avg_long, n_long, clk


def bench_decode(run, workload, headline):
    """One decode step (copy_blocks, the cache write, decode) of `workload`."""
    import numpy as np
    import torch

    from paged_kv_cache_394_b200 import pagedkv as pk
    from paged_kv_cache_394_b200 import workloads as W
    args, dev = run.args, run.dev
    base, fp8, cascade = split_name(workload)
    w = run.workload(base)
    kv_elem = 1 if fp8 else 2
    q, kc, vc, key, val, scales = device_caches(pk, w, dev, fp8)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    pairs = torch.from_numpy(np.ascontiguousarray(w.cow_pairs)).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    part_req = w.partition_size if args.partition is None else args.partition
    part = (pk.partition_size_fp8 if fp8 else pk.partition_size)(
        w.num_seqs, w.num_kv_heads, w.block_size, w.max_context_len, part_req)
    split = part < w.max_context_len
    if cascade:
        gs_np, sb_np = W.cascade_groups(w)
        gstart = torch.from_numpy(gs_np).to(dev)
        gshared = torch.from_numpy(sb_np).to(dev)
        max_group, max_shared = int(np.diff(gs_np).max()), int(sb_np.max())
        ws = torch.empty(max(16, pk.cascade_workspace_bytes(
            w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
            w.max_context_len, part_req)), dtype=torch.uint8, device=dev)
    else:
        ws = pk.alloc_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                w.block_size, w.max_context_len, part_req, device=dev)
    stream = torch.cuda.Stream(device=dev)
    has_pairs = len(w.cow_pairs) > 0
    # cache write (+ block copy) + decode (+ reduce); cascade: prefix pass + suffix + reduce
    launches_per_step = (1 + (1 if has_pairs else 0) +
                         (3 if cascade else 1 + (1 if split else 0)))
    # CTA schedule, computed on the host from the step's lengths so that long
    # sequences do not start last: by default one CTA per partition that
    # exists, longest first (pkv_decode_plan); or the full grid with the
    # sequences longest first (pkv_decode_order).  Cascade keeps its groups.
    planned = args.schedule == "plan" and not cascade
    sched_key = None if cascade else "work" if planned else "order"

    def schedule(h_lens):
        return (pk.decode_plan(h_lens, w.block_size, part) if planned
                else pk.decode_order(h_lens))
    h_sched = None if cascade else schedule(w.context_lens).pin_memory()
    inputs = dict(q=q, key=key, val=val, slots=slots, pairs=pairs, tables=tables, lens=lens,
                  out=out, order=None, work=None)
    if sched_key is not None:
        inputs[sched_key] = h_sched.to(dev)

    def decode(t=inputs):
        if cascade:
            pk.paged_attn_decode_cascade(t["out"], t["q"], kc, vc, t["tables"], t["lens"], gstart,
                                         gshared, w.scale, w.num_kv_heads, w.block_size,
                                         w.max_context_len, max_group, max_shared,
                                         partition_size=part_req, workspace=ws, dev_err=err,
                                         stream=stream,
                                         k_scales=scales[0] if fp8 else None,
                                         v_scales=scales[1] if fp8 else None)
        elif fp8:
            pk.paged_attn_decode_fp8(t["out"], t["q"], kc, vc, t["tables"], t["lens"], w.scale,
                                     scales[0], scales[1], w.num_kv_heads, w.block_size,
                                     w.max_context_len,
                                     partition_size=part if planned else part_req, workspace=ws,
                                     dev_err=err, stream=stream, seq_order=t["order"],
                                     work=t["work"])
        else:
            pk.paged_attn_decode(t["out"], t["q"], kc, vc, t["tables"], t["lens"], w.scale,
                                 w.num_kv_heads, w.block_size, w.max_context_len,
                                 partition_size=part if planned else part_req, workspace=ws,
                                 dev_err=err, stream=stream, seq_order=t["order"],
                                 work=t["work"])

    def step(i=0, t=inputs):
        if has_pairs:
            pk.copy_blocks(kc, vc, t["pairs"], dev_err=err, stream=stream)
        if fp8:
            pk.reshape_and_cache_fp8(t["key"], t["val"], kc, vc, t["slots"], scales[0],
                                     scales[1], dev_err=err, stream=stream)
        else:
            pk.reshape_and_cache(t["key"], t["val"], kc, vc, t["slots"], dev_err=err,
                                 stream=stream)
        decode(t)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError("%s: device error word %d during warm-up" % (workload, int(err.item())))

    # ---- timed region: K whole steps, nothing else on the stream -------------
    ms_per_step, clk = time_steps(run, stream, step, args.steps, graph=not args.no_graph)
    sbytes = step_bytes(w, kv_elem)
    all_bytes = sum_over_ranks(sbytes, dev)
    value = all_bytes / (ms_per_step * 1e-3) / 1e9
    # ---- the decode call alone, for the roofline ------------------------------
    dec_ms, dec_n, sus_ms, sus_n, sus_clk = time_kernel(run, stream, decode, ms_per_step)
    dbytes = decode_bytes(w, kv_elem)
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()

    # ---- shared blocks: unique bytes, and the decode timed with L2 flushed ----
    ubytes = unique_decode_bytes(w, kv_elem)
    sharing = None
    if ubytes < dbytes:
        l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20)
        scrub = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        n_fl = 50
        fl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(n_fl)]
        with torch.cuda.stream(stream):
            for a, b in fl_ev:
                scrub.zero_()             # evict the previous launch's blocks from L2
                a.record(stream)
                decode()
                b.record(stream)
        torch.cuda.synchronize(dev)
        fl_ms = statistics.mean(a.elapsed_time(b) for a, b in fl_ev)
        del scrub
        traffic = committed_traffic(workload)
        sharing = {
            "unique_bytes_per_launch": ubytes,
            "logical_over_unique": round(dbytes / ubytes, 3),
            "unique_gbs": round(ubytes / (dec_ms * 1e-3) / 1e9, 2),
            "unique_pct_of_hbm_peak": round(100.0 * ubytes / (dec_ms * 1e-3) / 1e9 / peak, 2),
            "dram_over_logical": None if traffic is None else round(traffic / dbytes, 4),
            "l2_flushed": {"achieved": round(dbytes / (fl_ms * 1e-3) / 1e9, 2),
                           "unique_gbs": round(ubytes / (fl_ms * 1e-3) / 1e9, 2),
                           "avg_launch_ms": round(fl_ms, 5), "launches": n_fl,
                           "flush": "%d MB written before each launch" % (2 * l2 >> 20)},
        }
    kernel = (("paged_prefill_tc_kernel (prefix pass) + " if cascade else "")
              + ("paged_decode_mma_kernel" if (fp8 and w.head_dim == 128)
                 or (not fp8 and w.num_heads > w.num_kv_heads) else "paged_decode_kernel")
              + (" + reduce" if split or cascade else ""))
    line = {
        "metric": "paged-decode KV-read GB/s (% of B200 HBM peak) and attention tokens/s",
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": round(ms_per_step, 5),
        "dtype": "e4m3 cache, %s q/out, f32 math" % w.dtype if fp8 else w.dtype,
        "config": dict(W.describe(w), workload=workload,
                       kv_cache="e4m3, per-kv-head scales (all %g here)" % FP8_K_SCALE
                       if fp8 else w.dtype,
                       partition_used=part, split_k=split,
                       seq_order="index order (cascade groups)" if cascade else
                       ("work list of the existing partitions, longest first in 256-token "
                        "buckets (pkv_decode_plan on the host)") if planned else
                       "longest first in 256-token buckets (pkv_decode_order on the host)",
                       timing=TIMING_NOTE[bool(args.no_graph)],
                       l2=("no flush: %.2f GB of KV read per step, larger than the 126 MB L2"
                           % (dbytes / 1e9)) if ubytes >= dbytes else
                          ("no flush between steps: %.2f GB of logical KV reads (%.2f GB of "
                           "distinct blocks) per step; the launch is also timed with L2 "
                           "flushed (shared_blocks.l2_flushed)" % (dbytes / 1e9, ubytes / 1e9))),
        "pct_of_hbm_peak": round(100.0 * value / run.world / peak, 2),
        "tokens_per_s": round(w.num_seqs * run.world / (ms_per_step * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": committed_traffic(workload), "kernel": kernel,
                     "algorithmic_bytes_per_launch": dbytes,
                     "avg_launch_ms": round(dec_ms, 5), "launches_timed": dec_n,
                     "sustained": {"achieved": round(dbytes / (sus_ms * 1e-3) / 1e9, 2),
                                   "frac": round(dbytes / (sus_ms * 1e-3) / 1e9 / peak, 4),
                                   "avg_launch_ms": round(sus_ms, 5), "launches": sus_n,
                                   "clocks": sus_clk},
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
                     if peak_kind == "measured" else "fallback 6.65 TB/s"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if sharing is not None:
        line["shared_blocks"] = sharing
    if not headline or args.no_e2e:
        del ws
        return line

    # ---- end to end through host buffers --------------------------------------
    def pinned(a, view=None):
        return torch.from_numpy(np.ascontiguousarray(a if view is None else a.view(view))).pin_memory()
    tdt = q.dtype
    h_q = pinned(w.q, np.int16).view(tdt)
    h_key = pinned(w.key, np.int16).view(tdt)
    h_val = pinned(w.value, np.int16).view(tdt)
    h_slots, h_pairs = pinned(w.slot_mapping), pinned(w.cow_pairs)
    h_tables, h_lens = pinned(w.block_tables), pinned(w.context_lens)
    h_out = torch.empty(w.q.shape, dtype=tdt).pin_memory()
    staging = torch.empty(pk.staging_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                           w.max_blocks_per_seq, len(w.slot_mapping),
                                           len(w.cow_pairs)), dtype=torch.uint8, device=dev)
    # the per-step order or work list (computed on the host from the step's
    # lengths) is uploaded too
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_key, h_val, h_slots, h_pairs,
                                                     h_tables, h_lens)
              + ((h_sched,) if h_sched is not None else ()))
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step(i=0):
        if not fp8 and not cascade:
            pk.decode_step_host(h_out, h_q, h_key, h_val, h_slots, h_pairs, h_tables, h_lens, kc,
                                vc, w.scale, w.max_context_len, staging, workspace=ws,
                                partition_size=part_req, dev_err=err, stream=stream)
            return
        # E4M3 caches or cascade decode: the same copies through the Python binding's tensors
        with torch.cuda.stream(stream):
            srcs = [(q, h_q), (key, h_key), (val, h_val), (slots, h_slots), (tables, h_tables),
                    (lens, h_lens)]
            if not cascade:
                h_sched.copy_(schedule(h_lens))
                srcs.append((inputs[sched_key], h_sched))
            for dst, src in srcs:
                dst.copy_(src, non_blocking=True)
            if has_pairs:
                pairs.copy_(h_pairs, non_blocking=True)
            step()
            h_out.copy_(out, non_blocking=True)
    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_serial_ms, _ = time_steps(run, stream, e2e_step, args.steps)
    e2e_serial = all_bytes / (e2e_serial_ms * 1e-3) / 1e9

    # pipelined: step i+1's inputs cross the host link while step i computes,
    # and step i's output returns while step i+1 computes.  Every step still
    # copies its own inputs in and its output back inside the timed region;
    # the cache work stays in order on one stream.  16-bit caches: the
    # library's pipeline (pkv_decode_pipeline_*), one C call per step; E4M3
    # and cascade: the same overlap built from the binding's calls.
    h_outs = [h_out, torch.empty_like(h_out).pin_memory()]
    if not fp8 and not cascade:
        pstaging = torch.empty(pk.DecodePipeline.staging_bytes(
            w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_blocks_per_seq,
            len(w.slot_mapping), len(w.cow_pairs)), dtype=torch.uint8, device=dev)
        pipe = pk.DecodePipeline(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                 w.block_size, w.max_blocks_per_seq, len(w.slot_mapping),
                                 len(w.cow_pairs), tdt, pstaging, stream=stream)

        def e2e_pipelined(i):
            pipe.step(h_outs[i % 2], h_q, h_key, h_val, h_slots, h_pairs, h_tables, h_lens, kc,
                      vc, w.scale, w.max_context_len, workspace=ws, partition_size=part_req,
                      dev_err=err)
            if i == args.steps - 1:
                pipe.join(stream)          # the timing event waits for the last download
        e2e_api = "pkv_decode_pipeline_step (one C call per step; upload, compute and " \
                  "download on three streams, consecutive steps overlapped)"
    else:
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        bufs = [inputs, {k: None if v is None else v.clone() for k, v in inputs.items()}]
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        h_src = dict(q=h_q, key=h_key, val=h_val, slots=h_slots, pairs=h_pairs, tables=h_tables,
                     lens=h_lens)
        if not cascade:
            h_src[sched_key] = h_sched
        h_scheds = [h_sched, None if cascade else h_sched.clone().pin_memory()]

        def e2e_pipelined(i):
            b, t = i % 2, bufs[i % 2]
            up.wait_event(ev_comp[b])          # step i-2 has finished reading buffer b
            if not cascade:
                ev_up[b].synchronize()         # step i-2's upload has read h_scheds[b]
                h_scheds[b].copy_(schedule(h_lens))
                h_src[sched_key] = h_scheds[b]
            with torch.cuda.stream(up):
                for k, src in h_src.items():
                    if (k != "pairs" or has_pairs) and src is not None:
                        t[k].copy_(src, non_blocking=True)
            ev_up[b].record(up)
            stream.wait_event(ev_up[b])
            stream.wait_event(ev_down[b])      # step i-2's output has left buffer b
            step(t=t)
            ev_comp[b].record(stream)
            down.wait_event(ev_comp[b])
            with torch.cuda.stream(down):
                h_outs[b].copy_(t["out"], non_blocking=True)
            ev_down[b].record(down)
            if i == args.steps - 1:
                for bb in range(2):
                    stream.wait_event(ev_down[bb])
        e2e_api = ("Python binding (reshape_and_cache%s, paged_attn_decode%s) with "
                   "pinned-host copies on side streams, consecutive steps overlapped"
                   % ("_fp8" if fp8 else "", "_cascade" if cascade else "_fp8" if fp8 else ""))
    for i in range(args.warmup):
        e2e_pipelined(i)
    torch.cuda.synchronize(dev)
    e2e_ms, _ = time_steps(run, stream, e2e_pipelined, args.steps)
    e2e_value = all_bytes / (e2e_ms * 1e-3) / 1e9
    if not fp8 and not cascade:
        pipe.close()
    if int(err.item()) != 0:
        raise RuntimeError("%s: device error word %d" % (workload, int(err.item())))
    line["context_tokens_per_s"] = round(run.world * int(w.context_lens.sum())
                                         / (ms_per_step * 1e-3), 1)
    line["pct_of_8tbs_nominal"] = round(100.0 * value / run.world / 8000.0, 2)
    line["step_bytes"] = sbytes
    line["e2e"] = {
        "value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 5),
        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
        "api": e2e_api,
        "serial": {"value": round(e2e_serial, 2), "ms_per_step": round(e2e_serial_ms, 5),
                   "api": "Python binding with torch copies on one stream"
                   if fp8 or cascade else "pkv_decode_step_host (one call per step)"}}
    if run.rank == 0 and run.world == 1 and not args.no_cpu_baseline and not fp8 and not cascade:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    del ws, staging
    return line


def bench_prefill(run, workload, headline):
    """One chunked-prefill step: reshape_and_cache of the new tokens, then
    paged prefill attention.  Metric: attention TFLOP/s (tensor-bound)."""
    import numpy as np
    import torch

    from paged_kv_cache_394_b200 import pagedkv as pk
    from paged_kv_cache_394_b200 import workloads as W
    args, dev = run.args, run.dev
    base, fp8, _ = split_name(workload)
    w = run.workload(base)
    q, kc, vc, key, val, scales = device_caches(pk, w, dev, fp8)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.context_lens).to(dev)
    qstart = torch.from_numpy(w.query_start).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    max_q = int(np.diff(w.query_start).max())
    stream = torch.cuda.Stream(device=dev)
    # the units of the longest histories cut into key pieces, planned on the
    # host from the step's lengths (pkv_prefill_plan; head_dim 128)
    planned = args.schedule == "plan" and w.head_dim == 128
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def make_plan(qs_host, lens_host):
        return pk.prefill_plan(qs_host, lens_host, w.num_heads, w.num_kv_heads, w.head_dim, sms)
    h_plan = make_plan(w.query_start, w.context_lens) if planned else None
    plan = h_plan.to(dev) if planned else None
    plan_ws = (torch.empty(max(16, h_plan.workspace_bytes), dtype=torch.uint8, device=dev)
               if planned else None)

    def write(k, v, s):
        if fp8:
            pk.reshape_and_cache_fp8(k, v, kc, vc, s, scales[0], scales[1], dev_err=err,
                                     stream=stream)
        else:
            pk.reshape_and_cache(k, v, kc, vc, s, dev_err=err, stream=stream)

    def attend(o=out, qq=q, t=tables, l_=lens, qs=qstart, pl=plan):
        if fp8:
            pk.paged_attn_prefill_fp8(o, qq, kc, vc, t, l_, qs, w.scale, scales[0], scales[1],
                                      w.num_kv_heads, w.block_size, w.max_context_len, max_q,
                                      dev_err=err, stream=stream, plan=pl, workspace=plan_ws)
        else:
            pk.paged_attn_prefill(o, qq, kc, vc, t, l_, qs, w.scale, w.num_kv_heads,
                                  w.block_size, w.max_context_len, max_q, dev_err=err,
                                  stream=stream, plan=pl, workspace=plan_ws)

    def step(i=0):
        write(key, val, slots)
        attend()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError("%s: device error word %d during warm-up" % (workload, int(err.item())))
    ms_per_step, clk = time_steps(run, stream, step, args.steps, graph=not args.no_graph)
    kern_ms, kern_n, sus_ms, sus_n, sus_clk = time_kernel(run, stream, attend, ms_per_step)
    flops = prefill_flops(w)
    all_flops = sum_over_ranks(flops, dev)
    value = all_flops / (ms_per_step * 1e-3) / 1e12
    achieved = flops / (kern_ms * 1e-3) / 1e12
    peak, peak_kind = tensor_peak()
    line = {
        "metric": "paged-prefill attention TFLOP/s",
        "value": round(value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms_per_step, 5),
        "dtype": "e4m3 cache, %s q/out, f32 math" % w.dtype if fp8 else w.dtype,
        "config": dict(W.describe(w), workload=workload,
                       kv_cache="e4m3, per-kv-head scales (all %g here)" % FP8_K_SCALE
                       if fp8 else w.dtype,
                       timing=TIMING_NOTE[bool(args.no_graph)],
                       schedule=("planned (pkv_prefill_plan on the host, %d SMs): %d CTAs per kv "
                                 "head, %d units cut into key pieces and merged"
                                 % (sms, len(h_plan.work), len(h_plan.merges))) if planned else
                                "one CTA per (sequence, query tile, kv head), longest first",
                       l2="no flush: each step rewrites the new tokens' K/V"),
        "tokens_per_s": round(run.world * int(w.query_start[-1]) / (ms_per_step * 1e-3), 1),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": committed_traffic(workload, "prefill"),
                     "kernel": "paged_prefill_tc_kernel" if w.head_dim == 128
                               else "paged_prefill_kernel",
                     "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": round(kern_ms, 5), "launches_timed": kern_n,
                     "sustained": {"achieved": round(flops / (sus_ms * 1e-3) / 1e12, 2),
                                   "frac": round(flops / (sus_ms * 1e-3) / 1e12 / peak, 4),
                                   "avg_launch_ms": round(sus_ms, 5), "launches": sus_n,
                                   "clocks": sus_clk},
                     "peak_source": "%s (MEASURED_PEAKS.json bf16_tflops; fp16 has the same "
                                    "dense rate)" % peak_kind},
        "gpu_launches": (2 + (1 if planned and len(h_plan.merges) else 0)) * args.steps,
        "clocks": clk,
    }
    if planned and len(h_plan.merges):
        line["roofline"]["kernel"] += " + paged_prefill_merge_kernel"
    if not headline or args.no_e2e:
        return line

    # end to end through the Python API: pinned host inputs in, output back
    def pinned(a, view=None):
        return torch.from_numpy(np.ascontiguousarray(a if view is None else a.view(view))).pin_memory()
    hq, hk, hv = pinned(w.q, np.int16), pinned(w.key, np.int16), pinned(w.value, np.int16)
    hs, ht, hl, hqs = (pinned(w.slot_mapping), pinned(w.block_tables), pinned(w.context_lens),
                       pinned(w.query_start))
    hout = torch.empty(w.q.shape, dtype=torch.int16).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(key), torch.empty_like(val)
    ds, dt_, dl, dqs = (torch.empty_like(slots), torch.empty_like(tables), torch.empty_like(lens),
                        torch.empty_like(qstart))
    # the plan (made on the host from the batch's lengths, which stay the same
    # from step to step here) is uploaded with each step's inputs
    h_pw = h_pm = None
    if planned:
        h_pw, h_pm = h_plan.work.pin_memory(), h_plan.merges.pin_memory()
    extra_h = (h_pw, h_pm) if planned else ()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs, ht, hl, hqs) + extra_h)
    d2h = hout.numel() * hout.element_size()

    host_in = (hq, hk, hv, hs, ht, hl, hqs) + extra_h
    dev0 = (dq, dk, dv, ds, dt_, dl, dqs) + tuple(t.to(dev) for t in extra_h)
    dev_in = [dev0, tuple(torch.empty_like(t) for t in dev0)]
    douts = [out, torch.empty_like(out)]
    houts = [hout, torch.empty_like(hout).pin_memory()]

    def upload(bufs, copy_stream):
        with torch.cuda.stream(copy_stream):
            for d, h in zip(bufs, host_in):
                (d.view(torch.int16) if d.dtype in (torch.float16, torch.bfloat16) else d).copy_(
                    h, non_blocking=True)

    def compute(bufs, o):
        bq, bk, bv, bs, bt, bl, bqs = bufs[:7]
        pl = pk.PrefillPlan(bufs[7], bufs[8], h_plan.workspace_bytes) if planned else None
        write(bk, bv, bs)
        attend(o, bq, bt, bl, bqs, pl)

    def e2e_step(i=0):  # serial: copies in, compute, copy out, all on one stream
        upload(dev_in[0], stream)
        compute(dev_in[0], out)
        with torch.cuda.stream(stream):
            hout.copy_(out.view(torch.int16), non_blocking=True)

    # pipelined: step i+1's inputs cross the host link while step i computes,
    # and step i's output returns while step i+1 computes; every step still
    # copies its own inputs in and its output back inside the timed region
    up_s, down_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(i):
        b = i % 2
        up_s.wait_event(ev_comp[b])            # step i-2 has finished reading buffer b
        upload(dev_in[b], up_s)
        ev_up[b].record(up_s)
        stream.wait_event(ev_up[b])
        stream.wait_event(ev_down[b])          # step i-2's output has left buffer b
        compute(dev_in[b], douts[b])
        ev_comp[b].record(stream)
        down_s.wait_event(ev_comp[b])
        with torch.cuda.stream(down_s):
            houts[b].copy_(douts[b].view(torch.int16), non_blocking=True)
        ev_down[b].record(down_s)
        if i == args.steps - 1:
            for bb in range(2):
                stream.wait_event(ev_down[bb])

    for i in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_serial_ms, _ = time_steps(run, stream, e2e_step, args.steps)
    for i in range(args.warmup):
        e2e_pipelined(i)
    torch.cuda.synchronize(dev)
    e2e_ms, _ = time_steps(run, stream, e2e_pipelined, args.steps)
    if int(err.item()) != 0:
        raise RuntimeError("%s: device error word %d" % (workload, int(err.item())))
    line["e2e"] = {
        "value": round(all_flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
        "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
        "api": ("pagedkv.reshape_and_cache_fp8 + paged_attn_prefill_fp8" if fp8 else
                "pagedkv.reshape_and_cache + paged_attn_prefill") +
               " with pinned-host copies on side streams, consecutive steps overlapped",
        "serial": {"value": round(all_flops / (e2e_serial_ms * 1e-3) / 1e12, 2),
                   "ms_per_step": round(e2e_serial_ms, 5),
                   "api": "the same calls with the copies on one stream"}}
    return line


def run_ours(args):
    from paged_kv_cache_394_b200 import workloads as W
    base, _, _ = split_name(args.workload)      # unknown names are refused before any device work
    run = Run(args)

    def bench(name, headline):
        return (bench_prefill if split_name(name)[0] in W.PREFILL_NAMES else bench_decode)(
            run, name, headline)

    line = bench(args.workload, True)
    # the other configurations, on one GPU only (each rank would hold its GPUs
    # that much longer under torchrun)
    others = {}
    if args.workload == "llama7b" and not args.no_other and run.world == 1:
        for name in OTHER_WORKLOADS:
            others[name] = bench(name, False)
    if run.rank == 0:
        head = {"metric": line.pop("metric"), "value": line.pop("value"), "unit": line.pop("unit"),
                "n_gpus": run.world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": line.pop("ms_per_step"), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": line.pop("dtype"),
                "data": "synthetic"}
        head["config"] = dict(line.pop("config"), parallelism="replicas%d" % run.world)
        head.update(line)
        if others:
            head["other_workloads"] = others
        print(json.dumps(head), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(w, seconds, threads=None):
    """Times the oracle's step (cache write, then decode of whole sequences in
    order, all heads) until `seconds` have passed or the batch is done, with
    BLAS limited to `threads` (default: every core this process may use)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from oracle import attention as OA
    from oracle import cache_ops as OC
    cores = threads or len(os.sched_getaffinity(0))
    done_seqs = 0
    nbytes = 0
    with threadpool_limits(limits=cores):
        t0 = time.perf_counter()
        kc, vc, _ = OC.copy_blocks(w.k_cache, w.v_cache, w.cow_pairs, inplace=True)
        kc, vc, _ = OC.reshape_and_cache(w.key, w.value, kc, vc, w.slot_mapping, w.block_size,
                                         inplace=True)
        nbytes += write_bytes(w) + copy_bytes(w)
        for s in range(w.num_seqs):
            pairs = [(s, h) for h in range(w.num_heads)]
            OA.paged_attention_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale,
                                      w.num_kv_heads, w.block_size, w.dtype, pairs=pairs)
            done_seqs += 1
            nbytes += (2 * int(w.context_lens[s]) * w.num_kv_heads * w.head_dim * 2
                       + 2 * w.num_heads * w.head_dim * 2)
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
    _ = np
    return nbytes, dt, done_seqs, cores


def cpu_baseline(w, seconds):
    nbytes, dt, n, cores = oracle_sample(w, seconds)
    nb1, dt1, n1, _ = oracle_sample(w, seconds / 3, threads=1)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": "cache write + float64 decode of the first %d of %d sequences (all %d "
                      "heads), %.1f s on the host cores" % (n, w.num_seqs, w.num_heads, dt),
            "value_1_thread": round(nb1 / dt1 / 1e9, 4),
            "sample_1_thread": "the same, BLAS on 1 thread: %d sequences in %.1f s" % (n1, dt1)}


def replay_trace(mgr, trace, cached, max_live=64):
    """Admits the trace's requests in order, up to max_live at a time; every
    iteration appends one generated token to each live request and frees those
    that are done.  Works on the C++ allocator and on the oracle alike."""
    import collections
    live = collections.OrderedDict()
    prompt_tokens = cached_tokens = peak = 0
    ops = 0
    for rid, (toks, out_len) in enumerate(trace):
        while len(live) >= max_live:
            for sid in list(live):
                mgr.append_slot(sid)
                ops += 1
                live[sid] -= 1
                if live[sid] == 0:
                    mgr.free_seq(sid)
                    ops += 1
                    del live[sid]
        if cached:
            cached_tokens += mgr.add_seq_cached(rid, toks)
        else:
            mgr.add_seq(rid, len(toks))
        ops += 1
        prompt_tokens += len(toks)
        live[rid] = out_len
        peak = max(peak, mgr.num_blocks - mgr.num_free() - (mgr.num_evictable() if cached else 0))
    for sid in list(live):
        mgr.free_seq(sid)
        ops += 1
    return prompt_tokens, cached_tokens, peak, ops


def run_prefix_cache_trace(args):
    """Host measurement of prefix caching on a seeded chat trace."""
    from oracle.block_manager import BlockManager
    from paged_kv_cache_394_b200 import pagedkv as pk
    from paged_kv_cache_394_b200 import workloads as W
    trace = W.chat_trace(W.SEED_BASE + 50)
    nb, bs = 16384, 16
    res = {}
    for cached in (True, False):
        mgr = pk.BlockAllocator(nb, bs)
        t0 = time.perf_counter()
        prompt, hit_tokens, peak, ops = replay_trace(mgr, trace, cached)
        dt = time.perf_counter() - t0
        res[cached] = (prompt, hit_tokens, peak, ops, dt, mgr.cache_stats())
    ref = BlockManager(nb, bs)
    t0 = time.perf_counter()
    _, ref_hit, ref_peak, ref_ops, = replay_trace(ref, trace, True)
    ref_dt = time.perf_counter() - t0
    prompt, hit_tokens, peak, ops, dt, stats = res[True]
    q, h, _, ev = stats
    if (ref_hit, ref_peak) != (hit_tokens, peak) or ref.cache_stats()[:2] != (q, h):
        raise RuntimeError("allocator and oracle disagree on the trace")
    line = {
        "metric": "prefix-cache hit rate on a shared-system-prompt chat trace",
        "value": round(h / q, 4), "unit": "fraction", "higher_is_better": True,
        "config": {"workload": "prefix_cache_trace", "requests": len(trace), "system_prompts": 8,
                   "zipf_a": 1.2, "num_blocks": nb, "block_size": bs, "max_live": 64},
        "prefill_tokens_saved": round(hit_tokens / prompt, 4),
        "peak_blocks": {"cached": peak, "uncached": res[False][2],
                        "saved": round(1 - peak / res[False][2], 4)},
        "evicted_blocks": ev,
        "allocator_ops_per_s": round(ops / dt, 1),
        "cpu_baseline": {"value": round(ref_ops / ref_dt, 1), "unit": "ops/s", "cores": 1,
                         "kind": "oracle", "sample": "the same trace through oracle.block_manager"},
        "data": "synthetic",
    }
    print(json.dumps(line), flush=True)


def run_serving_trace(args):
    """The continuous-batching driver over a seeded Poisson trace of chat-shaped
    requests (LLaMA-7B attention-layer shapes).  Reports generated tokens/s of
    device time and the memory utilization of the allocated pages, the figures
    the pages quote (over 90 % of the cache used, under 4 % wasted)."""
    import torch

    from paged_kv_cache_394_b200 import engine as E
    torch.cuda.set_device(0)
    b = E.ContinuousBatcher(12000, 16, 32, 32, 128, dtype=torch.float16, max_num_seqs=256,
                            max_num_batched_tokens=2048, max_model_len=2560, seed=394)
    trace = E.synthetic_trace(394, 400, mean_interarrival=0.2, prompt_median=300,
                              prompt_sigma=0.8, output_range=(32, 256), max_prompt=2048)
    for r in trace:
        b.submit(r)
    kern_ms = dec_tokens = pre_tokens = steps = 0
    utils, live_peak = [], 0
    t0 = time.perf_counter()
    while not b.idle():
        rec = b.step()
        steps += 1
        kern_ms += rec.kernel_ms
        dec_tokens += len(rec.decoded)
        pre_tokens += rec.prefill_tokens
        live_peak = max(live_peak, rec.live)
        if rec.used_blocks:
            utils.append(rec.cached_tokens / (rec.used_blocks * 16))
    wall = time.perf_counter() - t0
    line = {
        "metric": "continuous-batching decode tokens/s per attention layer (device time)",
        "value": round(dec_tokens / (kern_ms * 1e-3), 1), "unit": "tokens/s",
        "higher_is_better": True, "data": "synthetic",
        "config": {"workload": "serving_trace", "requests": len(trace), "num_heads": 32,
                   "head_dim": 128, "block_size": 16, "dtype": "fp16", "num_blocks": 12000,
                   "max_num_seqs": 256, "max_num_batched_tokens": 2048,
                   "arrivals": "Poisson, mean gap 0.2 steps", "prompt": "lognormal median 300",
                   "output": "U[32, 256]"},
        "steps": steps, "decode_tokens": dec_tokens, "prefill_tokens": pre_tokens,
        "prefill_plus_decode_tokens_per_s": round((dec_tokens + pre_tokens) / (kern_ms * 1e-3), 1),
        "memory_utilization": {"mean": round(float(np.mean(utils)), 4),
                               "min": round(float(np.min(utils)), 4),
                               "waste_mean": round(1 - float(np.mean(utils)), 4)},
        "peak_live_sequences": live_peak,
        "host_steps_per_s": round(steps / wall, 1),
    }
    print(json.dumps(line), flush=True)


def oracle_sample_fp8(w, seconds, threads=None):
    """oracle_sample over E4M3 caches: each sequence's blocks are quantised
    (scale FP8_K_SCALE / FP8_V_SCALE, as in the device runs) and the float64
    E4M3 decode oracle runs over them; the quantisation is timed too."""
    from threadpoolctl import threadpool_limits

    from oracle import cache_ops as OC
    from oracle import fp8 as OF
    cores = threads or len(os.sched_getaffinity(0))
    done, nbytes = 0, 0
    with threadpool_limits(limits=cores):
        t0 = time.perf_counter()
        kc, vc, _ = OC.copy_blocks(w.k_cache, w.v_cache, w.cow_pairs, inplace=True)
        kc, vc, _ = OC.reshape_and_cache(w.key, w.value, kc, vc, w.slot_mapping, w.block_size,
                                         inplace=True)
        nbytes += write_bytes(w, 1) + copy_bytes(w, 1)
        for s in range(w.num_seqs):
            nblk = -(-int(w.context_lens[s]) // w.block_size)
            blocks = w.block_tables[s, :nblk]
            k8 = OF.quantize_cache(kc[blocks], w.dtype, FP8_K_SCALE)
            v8 = OF.quantize_cache(vc[blocks], w.dtype, FP8_V_SCALE)
            table = np.arange(nblk, dtype=np.int32)[None, :]
            OF.paged_attention_decode_fp8(w.q[s:s + 1], k8, v8, table, w.context_lens[s:s + 1],
                                          w.scale, FP8_K_SCALE, FP8_V_SCALE, w.num_kv_heads,
                                          w.block_size, w.dtype)
            done += 1
            nbytes += (2 * int(w.context_lens[s]) * w.num_kv_heads * w.head_dim
                       + 2 * w.num_heads * w.head_dim * 2)
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
    return nbytes, dt, done, cores


def oracle_sample_prefill(w, seconds, fp8=False, threads=None):
    """Times the prefill oracle's step (the new tokens' cache write, then the
    new tokens of the sequences in order, eight tokens x all heads at a time;
    over E4M3 codes of each sequence's blocks when ``fp8``) until ``seconds``
    have passed.  Returns the algorithmic FLOPs of the rows done (4 D per
    (row, visible key)) and the number of sequences begun."""
    from threadpoolctl import threadpool_limits

    from oracle import attention as OA
    from oracle import cache_ops as OC
    from oracle import fp8 as OF
    cores = threads or len(os.sched_getaffinity(0))
    begun, flops = 0, 0
    with threadpool_limits(limits=cores):
        t0 = time.perf_counter()
        kc, vc, _ = OC.reshape_and_cache(w.key, w.value, w.k_cache, w.v_cache, w.slot_mapping,
                                         w.block_size, inplace=True)
        for s in range(w.num_seqs):
            c = int(w.context_lens[s])
            nblk = -(-c // w.block_size)
            blocks = w.block_tables[s, :nblk]
            table = np.arange(nblk, dtype=np.int32)[None, :]
            q0, q1 = int(w.query_start[s]), int(w.query_start[s + 1])
            qs = np.array([0, q1 - q0], dtype=np.int32)
            if fp8:
                k8 = OF.quantize_cache(kc[blocks], w.dtype, FP8_K_SCALE)
                v8 = OF.quantize_cache(vc[blocks], w.dtype, FP8_V_SCALE)
            begun += 1
            for j0 in range(0, q1 - q0, 8):
                rows = [(j, h) for j in range(j0, min(j0 + 8, q1 - q0))
                        for h in range(w.num_heads)]
                if fp8:
                    OF.paged_attention_prefill_fp8(w.q[q0:q1], k8, v8, table,
                                                   w.context_lens[s:s + 1], qs, w.scale,
                                                   FP8_K_SCALE, FP8_V_SCALE, w.num_kv_heads,
                                                   w.block_size, w.dtype, rows=rows)
                else:
                    OA.paged_attention_prefill(w.q[q0:q1], kc[blocks], vc[blocks], table,
                                               w.context_lens[s:s + 1], qs, w.scale,
                                               w.num_kv_heads, w.block_size, w.dtype, rows=rows)
                pos0 = c - (q1 - q0)   # position of new token 0
                flops += sum(4 * w.head_dim * (pos0 + j + 1) for j, _ in rows)
                if time.perf_counter() - t0 > seconds:
                    break
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
    return flops, dt, begun, cores


def run_reference(args):
    """The reference arm: the float64 oracle, timed on the host cores over a
    bounded sample of each step, for the same workload, metric and unit as
    our arm (decode GB/s or prefill TFLOP/s; E4M3 over quantised codes;
    cascade computes plain decode, so it times the decode oracle)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from paged_kv_cache_394_b200 import workloads as W
    fp8 = args.workload.endswith("_fp8")
    name = args.workload.removesuffix("_fp8").removesuffix("_cascade")
    prefill = name in W.PREFILL_NAMES
    # parallel sampling: the oracle's block manager lays out the blocks
    from oracle.block_manager import BlockManager
    w0 = W.make(name, allocator=BlockManager)

    def sample(seconds):
        w = W.make(name, allocator=BlockManager)
        if prefill:
            return oracle_sample_prefill(w, seconds, fp8)
        return oracle_sample_fp8(w, seconds) if fp8 else oracle_sample(w, seconds)

    for _ in range(args.warmup):
        sample(0.5)
    times, total, n_last, cores = [], 0, 0, 1
    for _ in range(args.steps):
        amount, dt, n_last, cores = sample(args.cpu_seconds)
        times.append(dt)
        total += amount
    if prefill:
        value, unit = total / sum(times) / 1e12, "TFLOP/s"
        metric = "paged-prefill attention TFLOP/s"
        what = "the new tokens' cache write + float64 prefill of the new tokens (eight at a time) of the first"
    else:
        value, unit = total / sum(times) / 1e9, "GB/s"
        metric = "paged-decode KV-read GB/s (% of B200 HBM peak) and attention tokens/s"
        what = "cache write + float64 decode of the first"
    line = {
        "impl": "reference",
        "metric": metric,
        "value": round(value, 6), "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1000 * statistics.mean(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": dict(W.describe(w0), workload=args.workload, parallelism="host cores"),
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores,
                         "kind": "oracle",
                         "sample": "per step: %s %d of %d sequences (all heads)%s, bounded to "
                                   "%.0f s" % (what, n_last, w0.num_seqs,
                                               ", over E4M3 codes" if fp8 else "",
                                               args.cpu_seconds)},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama7b")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the steps as direct launches instead of one captured CUDA graph")
    ap.add_argument("--schedule", choices=("order", "plan"), default="plan",
                    help="CTA schedule made on the host from the step's lengths: decode "
                         "sequences longest first over the full grid and the prefill's own "
                         "in-kernel ranking (order), or the work lists of pkv_decode_plan "
                         "(one CTA per existing partition) and pkv_prefill_plan (units by "
                         "cost, the longest cut into key pieces) (plan)")
    ap.add_argument("--partition", type=int, default=None,
                    help="partition size in tokens (0 = let the library choose)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other", action="store_true",
                    help="time the named workload only (the default run also times the other "
                         "configurations as nested objects of the headline line)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffer) loops, e.g. under a profiler")
    ap.add_argument("--kernel-seconds", type=float, default=1.0,
                    help="length of the loop that times the dominant kernel alone")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args(argv)


def main(argv=None):
    args = parse_args(argv)
    # at least three untimed warm-up steps, whatever was asked
    args.warmup = max(3, args.warmup)
    if args.workload == "prefix_cache_trace":
        run_prefix_cache_trace(args)
    elif args.workload == "serving_trace":
        run_serving_trace(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
