"""Iteration-level (continuous) batching over the paged KV cache.

The pages describe vLLM's scheduler as follows: requests join a queue on
arrival; after every iteration, sequences that are ready are packed into the
next batch, and new requests are admitted whenever there is capacity, so short
and long requests share the GPU without waiting for each other ([csdn]
"调度革命：连续批处理如何让GPU持续满载？" and its workflow list; [cortexgrid]
static-vs-continuous batching table and FAQ).  Capacity is bounded by the
free pages and by ``max_num_seqs`` / ``max_num_batched_tokens`` ([csdn] API
example; [betteryeah] §4.3).  Parallel samples of one prompt share its pages
and copy them on write ([cortexgrid] FAQ on parallel sampling).

``ContinuousBatcher.step`` runs one iteration for one attention layer:

1. admit waiting requests in arrival order while ``max_num_seqs``,
   ``max_num_batched_tokens`` and the free pages allow (a request that does
   not fit stops admission for this iteration);
2. reserve one slot for every running sequence (the allocator returns the
   copy-on-write pairs for shared partial blocks);
3. on the GPU: ``copy_blocks`` for the pairs, ``reshape_and_cache`` for every
   new token (whole prompts of admitted requests, one token per running
   sequence), ``paged_attn_prefill`` for the admitted prompts and
   ``paged_attn_decode`` for the running sequences (with a work list that
   ``decode_plan`` makes from the host's context lengths);
4. fork the samples of a request whose prompt was just prefilled, retire
   sequences that reached their output length, free their pages.

Queries, keys and values are synthetic (seeded N(0,1)): the driver exercises
the memory manager and the kernels, not a model.  The host work here is
orchestration; allocation is the C++ allocator and every tensor operation is
a CUDA kernel of libpagedkv.
"""

from collections import deque
from dataclasses import dataclass

import numpy as np
import torch

from . import pagedkv as pk


@dataclass
class Request:
    rid: int
    prompt_len: int
    output_len: int
    arrival: int = 0      # iteration at which it joins the queue
    samples: int = 1      # parallel samples sharing the prompt


@dataclass
class StepRecord:
    """What one iteration did (for tests and statistics)."""
    admitted: list          # (sequence id, prompt length) admitted and prefilled this step
    decoded: list           # sequence ids decoded this step, in batch order
    slots: list             # slot of every new token: prompts first, then decoded sequences
    cow_pairs: list
    forked: list            # (parent, child) samples forked after this step's prefill
    new_tokens: int
    prefill_tokens: int
    finished: list
    live: int
    waiting: int
    used_blocks: int
    cached_tokens: int
    kernel_ms: float


class ContinuousBatcher:
    def __init__(self, num_blocks, block_size, num_heads, num_kv_heads, head_dim,
                 dtype=torch.float16, max_num_seqs=256, max_num_batched_tokens=2048,
                 max_model_len=4096, seed=0, device="cuda", free_order=None, values=None):
        self.bs = block_size
        self.h, self.hkv, self.d = num_heads, num_kv_heads, head_dim
        self.dtype = dtype
        self.max_num_seqs = max_num_seqs
        self.max_batched = max_num_batched_tokens
        self.max_model_len = max_model_len
        self.max_blocks = -(-max_model_len // block_size)
        self.device = torch.device(device)
        self.alloc = pk.BlockAllocator(num_blocks, block_size, free_order=free_order)
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = torch.zeros(shape, dtype=dtype, device=self.device)
        self.v_cache = torch.zeros(shape, dtype=dtype, device=self.device)
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(seed)
        # values(kind, shape) -> device tensor of self.dtype, kind in
        # {"key", "value", "q_prefill", "q_decode"}; N(0,1) from the device RNG by default
        self.values = values or (lambda kind, shape: torch.randn(
            *shape, generator=self.gen, device=self.device, dtype=torch.float32).to(self.dtype))
        self.waiting = deque()
        self.running = {}       # seq id -> remaining tokens to generate
        self.next_seq = 0
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.scale = 1.0 / float(np.sqrt(head_dim))
        self.step_index = 0
        self.last_outputs = {}  # "prefill" / "decode" -> output tensors of the last step

    # -- request queue -----------------------------------------------------
    def submit(self, req):
        if req.prompt_len + req.output_len > self.max_model_len:
            raise ValueError("request longer than max_model_len")
        self.waiting.append(req)

    # -- one iteration ---------------------------------------------------------
    def step(self):
        alloc = self.alloc
        # 1. admission, in arrival order
        admitted = []
        budget = self.max_batched - len(self.running)
        while self.waiting:
            req = self.waiting[0]
            if req.arrival > self.step_index:
                break
            if len(self.running) + len(admitted) + req.samples > self.max_num_seqs:
                break
            if req.prompt_len > budget:
                break
            # keep one free block per running sequence for this step's appends
            need = -(-req.prompt_len // self.bs)
            if alloc.num_free() < need + len(self.running) + len(admitted) * req.samples:
                break
            sid = self.next_seq
            try:
                alloc.add_seq(sid, req.prompt_len)
            except pk.PagedKVError as e:
                if e.status == pk.ERR_OUT_OF_BLOCKS:
                    break
                raise
            self.waiting.popleft()
            self.next_seq += 1
            budget -= req.prompt_len
            admitted.append((sid, req))
        # 2. one new slot per running sequence (CoW pairs for shared partial blocks)
        decoded = list(self.running)
        slots_dec, pairs = [], []
        if decoded:
            try:
                slots_dec, pairs = alloc.append_slots(decoded)
            except pk.PagedKVError as e:
                if e.status != pk.ERR_OUT_OF_BLOCKS:
                    raise
                raise RuntimeError("out of KV blocks while decoding; use a larger pool")
        # 3. device work
        slots_pre = []
        for sid, req in admitted:
            row = alloc.block_table([sid], self.max_blocks)[0]
            slots_pre += [row[t // self.bs] * self.bs + t % self.bs for t in range(req.prompt_len)]
        n_pre, n_dec = len(slots_pre), len(slots_dec)
        # this step's synthetic inputs, drawn before the timed kernels
        if n_pre + n_dec:
            slots = torch.tensor(slots_pre + slots_dec, dtype=torch.int64, device=self.device)
            key = self.values("key", (n_pre + n_dec, self.hkv, self.d))
            val = self.values("value", (n_pre + n_dec, self.hkv, self.d))
        if admitted:
            ids = [sid for sid, _ in admitted]
            lens = [req.prompt_len for _, req in admitted]
            p_tables = torch.tensor(alloc.block_table(ids, self.max_blocks), dtype=torch.int32,
                                    device=self.device)
            p_ctx = torch.tensor(lens, dtype=torch.int32, device=self.device)
            p_qs = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32,
                                device=self.device)
            p_q = self.values("q_prefill", (n_pre, self.h, self.d))
            p_out = torch.empty_like(p_q)
        if decoded:
            d_tables = torch.tensor(alloc.block_table(decoded, self.max_blocks),
                                    dtype=torch.int32, device=self.device)
            ctx_list = alloc.context_lens(decoded)
            d_ctx = torch.tensor(ctx_list, dtype=torch.int32, device=self.device)
            # one CTA per partition that exists, planned from the host's lengths
            d_part = pk.partition_size(n_dec, self.hkv, self.bs, max(ctx_list))
            d_work = pk.decode_plan(ctx_list, self.bs, d_part).to(self.device)
            d_q = self.values("q_decode", (n_dec, self.h, self.d))
            d_out = torch.empty_like(d_q)
        pair_t = torch.tensor(pairs, dtype=torch.int64, device=self.device) if pairs else None
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        if pairs:
            pk.copy_blocks(self.k_cache, self.v_cache, pair_t, dev_err=self.err)
        if n_pre + n_dec:
            pk.reshape_and_cache(key, val, self.k_cache, self.v_cache, slots, dev_err=self.err)
        self.last_outputs = {}
        if admitted:
            pk.paged_attn_prefill(p_out, p_q, self.k_cache, self.v_cache, p_tables, p_ctx, p_qs,
                                  self.scale, self.hkv, self.bs, max(lens), max(lens),
                                  dev_err=self.err)
            self.last_outputs["prefill"] = (ids, p_q, p_out, p_tables, p_ctx, p_qs)
        if decoded:
            pk.paged_attn_decode(d_out, d_q, self.k_cache, self.v_cache, d_tables, d_ctx,
                                 self.scale, self.hkv, self.bs, max(ctx_list),
                                 partition_size=d_part, dev_err=self.err, work=d_work)
            self.last_outputs["decode"] = (decoded, d_q, d_out, d_tables, d_ctx)
        if n_pre + n_dec:
            self.last_outputs["write"] = (key, val)
        t1.record()
        torch.cuda.synchronize(self.device)
        if int(self.err.item()) != 0:
            raise RuntimeError("device error word %d" % int(self.err.item()))
        # 4. bookkeeping: samples fork after their prompt, finished sequences free pages
        finished = []
        for sid in decoded:
            self.running[sid] -= 1
            if self.running[sid] == 0:
                del self.running[sid]
                alloc.free_seq(sid)
                finished.append(sid)
        forked = []
        for sid, req in admitted:
            self.running[sid] = req.output_len
            for _ in range(req.samples - 1):
                child = self.next_seq
                self.next_seq += 1
                alloc.fork(sid, child)
                self.running[child] = req.output_len
                forked.append((sid, child))
        cached, used = alloc.usage()
        self.step_index += 1
        return StepRecord(admitted=[(sid, req.prompt_len) for sid, req in admitted],
                          decoded=decoded, slots=slots_pre + slots_dec, cow_pairs=pairs,
                          forked=forked,
                          new_tokens=n_pre + n_dec, prefill_tokens=n_pre, finished=finished,
                          live=len(self.running), waiting=len(self.waiting), used_blocks=used,
                          cached_tokens=cached, kernel_ms=t0.elapsed_time(t1))

    def idle(self):
        return not self.waiting and not self.running


def synthetic_trace(seed, num_requests, mean_interarrival=0.5, prompt_median=300,
                    prompt_sigma=0.8, output_range=(32, 256), max_prompt=2048, samples=1):
    """Poisson arrivals with lognormal prompt lengths, like chat traffic."""
    rng = np.random.default_rng(seed)
    gaps = rng.exponential(mean_interarrival, num_requests)
    arrivals = np.floor(np.cumsum(gaps)).astype(int)
    prompts = np.clip(np.rint(rng.lognormal(np.log(prompt_median), prompt_sigma, num_requests)),
                      8, max_prompt).astype(int)
    outputs = rng.integers(output_range[0], output_range[1] + 1, num_requests)
    return [Request(i, int(p), int(o), int(a), samples) for i, (p, o, a) in
            enumerate(zip(prompts, outputs, arrivals))]
