"""Seeded synthetic workloads for paged decode attention.

This module only draws inputs: sequence lengths, physical block placement,
N(0, 1) query/key/value values and NaN poison.  For parallel sampling the
placement is a free-list order handed to a block manager that the caller
supplies (the library's allocator, or the oracle's), which then lays out the
shared and copied blocks itself.  It holds none of the
attention arithmetic and is the one module that feeds both the CUDA library
and the CPU oracle, so both see byte-identical inputs.

A workload describes one step of the hot path, applied to a pool state:

1. ``copy_blocks(cow_pairs)``          copy-on-write of shared partial blocks
2. ``reshape_and_cache(key, value, slot_mapping)``   write the step's tokens
3. ``paged_attn_decode(q, ...)``        one query token per sequence

Before the step every slot the step writes, every slot past a sequence's
context, and every unused block holds NaN, so a missed write or a stray read
shows up as NaN in the output.

Prefill workloads (``build_prefill_workload``) instead append several tokens
per sequence whose queries attend causally over the whole context.

The five named workloads follow the chat-serving shapes described for vLLM
(LLaMA-7B/13B-sized heads, grouped-query heads, block sizes 16 and 32,
lengths mixed like chat prompts plus generations, parallel sampling that
shares a prompt).  No dataset is read: lengths come from the distributions
named below.  16-bit tensors are uint16 bit patterns (fp16 or bf16).
"""

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

NAN_BITS = {"fp16": np.uint16(0x7E00), "bf16": np.uint16(0x7FC0)}
SEED_BASE = 394
NAMES = ("tiny", "llama7b", "gqa_chat", "long_splitk", "prefix_share")
PREFILL_NAMES = ("llama7b_prefill", "gqa_prefill", "skew_prefill")


@dataclass
class Workload:
    name: str
    dtype: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray          # int32 [S]
    block_tables: np.ndarray          # int32 [S, max_blocks], pad -1
    q: np.ndarray                     # uint16 [S, H, D]
    k_cache: np.ndarray               # uint16 [N, Hkv, bs, D], state before the step
    v_cache: np.ndarray
    key: np.ndarray                   # uint16 [T, Hkv, D], tokens written by the step
    value: np.ndarray
    slot_mapping: np.ndarray          # int64 [T]
    cow_pairs: np.ndarray             # int64 [P, 2]
    partition_size: int = 0           # 0: the library chooses
    notes: dict = field(default_factory=dict)
    query_start: np.ndarray = None    # int32 [S+1] for prefill (q is [T, H, D]); None for decode

    @property
    def num_seqs(self):
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self):
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self):
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def elem_bytes(self):
        return 2


def _to_bits(x32, dtype):
    """float32 -> 16-bit pattern, round to nearest even."""
    if dtype == "fp16":
        return x32.astype(np.float16).view(np.uint16)
    b = x32.view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


_CHUNK = 1 << 22


def _normal_bits(rng, shape, dtype):
    """N(0,1) values of ``shape`` as 16-bit patterns.

    The array is drawn in fixed chunks of 4 Mi elements, chunk ``i`` from its
    own generator seeded by (a draw from ``rng``, i), so the values do not
    depend on how many threads draw them.
    """
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    root = int(rng.integers(0, 2 ** 63))

    def draw(i):
        a = i * _CHUNK
        m = min(_CHUNK, n - a)
        g = np.random.default_rng(np.random.SeedSequence(root, spawn_key=(i,)))
        out[a:a + m] = _to_bits(g.standard_normal(m, dtype=np.float32), dtype)

    chunks = range(-(-n // _CHUNK))
    if n > _CHUNK:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(draw, chunks))
    else:
        for i in chunks:
            draw(i)
    return out.reshape(shape)


def _blocks_for(n, bs):
    return -(-int(n) // bs)


def _fill_pool(rng, num_blocks, hkv, bs, d, dtype, filled):
    """Pool of NaN with random values in the (block, offset) slots of ``filled``.

    ``filled`` maps physical block -> number of leading offsets that hold data.
    """
    nan = NAN_BITS[dtype]
    k = np.full((num_blocks, hkv, bs, d), nan, dtype=np.uint16)
    v = np.full((num_blocks, hkv, bs, d), nan, dtype=np.uint16)
    if filled:
        ids = np.fromiter(filled.keys(), dtype=np.int64)
        k[ids] = _normal_bits(rng, (len(ids), hkv, bs, d), dtype)
        v[ids] = _normal_bits(rng, (len(ids), hkv, bs, d), dtype)
        for b, n in filled.items():
            if n < bs:
                k[b, :, n:, :] = nan
                v[b, :, n:, :] = nan
    return k, v


def build_decode_workload(context_lens, num_heads, num_kv_heads, head_dim, block_size,
                          dtype, seed, num_blocks=None, pool_factor=1.2,
                          max_blocks_per_seq=None, name="custom", partition_size=0):
    """One decode step for independent sequences with random block placement.

    Sequence i holds ``context_lens[i]`` tokens; the last one is the token this
    step writes (so its slot is NaN before the step).  Physical blocks are a
    random permutation of the pool; the pool holds ``pool_factor`` times the
    blocks needed unless ``num_blocks`` is given.
    """
    rng = np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int64)
    s = len(lens)
    need = [_blocks_for(c, block_size) for c in lens]
    total = int(sum(need))
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * total)))
    if total > num_blocks:
        raise ValueError("pool too small: need %d blocks, have %d" % (total, num_blocks))
    mb = max(1, max(need) if need else 1) if max_blocks_per_seq is None else max_blocks_per_seq
    perm = rng.permutation(num_blocks)
    tables = np.full((s, mb), -1, dtype=np.int32)
    filled = {}
    slots = np.full(s, -1, dtype=np.int64)
    pos = 0
    for i, c in enumerate(lens):
        blocks = perm[pos:pos + need[i]]
        pos += need[i]
        tables[i, :need[i]] = blocks
        for k, b in enumerate(blocks):
            filled[int(b)] = int(min(block_size, c - 1 - k * block_size)) if c > 0 else 0
        if c > 0:
            t = c - 1
            slots[i] = int(blocks[t // block_size]) * block_size + t % block_size
    filled = {b: max(0, n) for b, n in filled.items()}
    kc, vc = _fill_pool(rng, num_blocks, num_kv_heads, block_size, head_dim, dtype, filled)
    q = _normal_bits(rng, (s, num_heads, head_dim), dtype)
    key = _normal_bits(rng, (s, num_kv_heads, head_dim), dtype)
    value = _normal_bits(rng, (s, num_kv_heads, head_dim), dtype)
    return Workload(name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
                    context_lens=lens.astype(np.int32), block_tables=tables, q=q,
                    k_cache=kc, v_cache=vc, key=key, value=value, slot_mapping=slots,
                    cow_pairs=np.zeros((0, 2), dtype=np.int64),
                    partition_size=partition_size, notes={"seed": seed})


def build_prefix_share_workload(num_prompts, samples, prompt_len, div_low, div_high,
                                num_heads, num_kv_heads, head_dim, block_size, dtype,
                                seed, allocator, pool_factor=1.2, name="prefix_share"):
    """Parallel sampling: ``samples`` sequences per prompt share the prompt's blocks.

    The block layout is not drawn here: ``allocator(num_blocks, block_size,
    free_order)`` is a block manager (the library's C++ allocator, or the
    oracle's: ``add_seq``, ``fork``, ``append_slots``, ``block_table``) and
    this function only drives it, so that the step's block
    tables, slots and copy pairs are the ones the block manager produces.
    ``free_order``, a random permutation of the pool, scatters the blocks.

    Each prompt is admitted (``add_seq``) and forked into its other samples,
    then every sample appends its ``U[div_low, div_high]`` divergent tokens
    (``append_slots``), prompt by prompt and sample by sample.  When the prompt
    ends inside a block, the first ``samples - 1`` samples to append copy that
    shared partial block on write (the step's copy pairs) and the last writes
    into the original.  Sequence order is prompt-major: the samples of a
    prompt are adjacent (sequence id = prompt * samples + sample).
    """
    rng = np.random.default_rng(seed)
    bs = block_size
    n_prompt_blocks = _blocks_for(prompt_len, bs)
    partial = prompt_len % bs != 0
    div = rng.integers(div_low, div_high + 1, size=num_prompts * samples)
    lens = prompt_len + div
    # blocks needed: prompt blocks, copies, and each sample's fresh blocks
    room_in_partial = (bs - prompt_len % bs) if partial else 0
    fresh = [_blocks_for(max(0, int(d) - room_in_partial), bs) for d in div]
    n_copies = num_prompts * (samples - 1) if partial else 0
    total = num_prompts * n_prompt_blocks + n_copies + int(sum(fresh))
    num_blocks = int(math.ceil(pool_factor * total))
    free_order = rng.permutation(num_blocks).astype(np.int32)
    mgr = allocator(num_blocks, bs, free_order)
    s = num_prompts * samples
    filled = {}
    for p in range(num_prompts):
        parent = p * samples
        mgr.add_seq(parent, prompt_len)
        for k, b in enumerate(mgr.block_table([parent], n_prompt_blocks)[0]):
            filled[int(b)] = min(bs, prompt_len - k * bs)
        for j in range(1, samples):
            mgr.fork(parent, parent + j)
    slots, cow = [], []
    for i in range(s):
        got, pairs = mgr.append_slots([i] * int(div[i]))
        slots += got
        cow += pairs
    mb = max(_blocks_for(c, bs) for c in lens)
    tables = np.asarray(mgr.block_table(list(range(s)), mb), dtype=np.int32).reshape(s, mb)
    kc, vc = _fill_pool(rng, num_blocks, num_kv_heads, bs, head_dim, dtype, filled)
    t_new = len(slots)
    q = _normal_bits(rng, (s, num_heads, head_dim), dtype)
    key = _normal_bits(rng, (t_new, num_kv_heads, head_dim), dtype)
    value = _normal_bits(rng, (t_new, num_kv_heads, head_dim), dtype)
    return Workload(name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, block_size=bs, num_blocks=num_blocks,
                    context_lens=lens.astype(np.int32), block_tables=tables, q=q,
                    k_cache=kc, v_cache=vc, key=key, value=value,
                    slot_mapping=np.asarray(slots, dtype=np.int64),
                    cow_pairs=np.asarray(cow, dtype=np.int64).reshape(-1, 2),
                    notes={"seed": seed, "prompt_len": prompt_len,
                           "prompt_blocks": n_prompt_blocks, "samples": samples,
                           "free_order": free_order})


def cascade_groups(w, shared_blocks=None):
    """Groups of a prefix-sharing workload for cascade decode: the samples of
    each prompt (adjacent sequences) and the whole prompt blocks they share
    (a partly filled last prompt block is private after copy-on-write).
    Returns int32 arrays (group_start [G+1], shared_blocks [G])."""
    samples = w.notes["samples"]
    n = w.num_seqs // samples
    full = w.notes["prompt_len"] // w.block_size if shared_blocks is None else shared_blocks
    group_start = np.arange(0, w.num_seqs + 1, samples, dtype=np.int32)
    return group_start, np.full(n, full, dtype=np.int32)


def build_prefill_workload(hist_lens, new_lens, num_heads, num_kv_heads, head_dim, block_size,
                           dtype, seed, pool_factor=1.2, name="prefill"):
    """One chunked-prefill step: sequence i already caches hist_lens[i] tokens
    and this step appends new_lens[i] more, whose K/V it writes and whose
    queries then attend causally over the whole context.

    q is [T, H, D] with T = sum(new_lens), packed sequence by sequence;
    ``query_start`` holds the offsets.  Slots of the new tokens hold NaN until
    the step writes them.
    """
    rng = np.random.default_rng(seed)
    hist = np.asarray(hist_lens, dtype=np.int64)
    new = np.asarray(new_lens, dtype=np.int64)
    lens = hist + new
    s = len(lens)
    need = [_blocks_for(c, block_size) for c in lens]
    num_blocks = max(1, int(math.ceil(pool_factor * sum(need))))
    perm = rng.permutation(num_blocks)
    mb = max(1, max(need))
    tables = np.full((s, mb), -1, dtype=np.int32)
    filled = {}
    slots = []
    pos = 0
    for i in range(s):
        blocks = perm[pos:pos + need[i]]
        pos += need[i]
        tables[i, :need[i]] = blocks
        for k, b in enumerate(blocks):
            filled[int(b)] = int(max(0, min(block_size, hist[i] - k * block_size)))
        for t in range(int(hist[i]), int(lens[i])):
            slots.append(int(blocks[t // block_size]) * block_size + t % block_size)
    kc, vc = _fill_pool(rng, num_blocks, num_kv_heads, block_size, head_dim, dtype, filled)
    t_new = int(new.sum())
    q = _normal_bits(rng, (t_new, num_heads, head_dim), dtype)
    key = _normal_bits(rng, (t_new, num_kv_heads, head_dim), dtype)
    value = _normal_bits(rng, (t_new, num_kv_heads, head_dim), dtype)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    return Workload(name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
                    context_lens=lens.astype(np.int32), block_tables=tables, q=q,
                    k_cache=kc, v_cache=vc, key=key, value=value,
                    slot_mapping=np.asarray(slots, dtype=np.int64),
                    cow_pairs=np.zeros((0, 2), dtype=np.int64), query_start=qs,
                    notes={"seed": seed})


def chat_trace(seed, num_requests=2000, num_system=8, zipf_a=1.2, system_len=(256, 1024),
               user_len=(32, 512), output_len=(16, 128), vocab=32000):
    """Synthetic chat requests sharing system prompts, for prefix caching.

    Each request = one of ``num_system`` system prompts (chosen with a Zipf
    law, so a few are popular) + a random user turn, and generates a random
    number of tokens.  Returns a list of (prompt token ids, output length).
    """
    rng = np.random.default_rng(seed)
    systems = [rng.integers(0, vocab, int(rng.integers(*system_len))).tolist()
               for _ in range(num_system)]
    ranks = np.minimum(rng.zipf(zipf_a, num_requests), num_system) - 1
    reqs = []
    for r in ranks:
        user = rng.integers(0, vocab, int(rng.integers(*user_len))).tolist()
        reqs.append((systems[int(r)] + user, int(rng.integers(*output_len))))
    return reqs


def chat_lengths(rng, n, median=600.0, sigma=1.0, low=16, high=4096):
    """Lognormal lengths with the given median, clipped and rounded."""
    x = rng.lognormal(mean=math.log(median), sigma=sigma, size=n)
    return np.clip(np.rint(x), low, high).astype(np.int64)


def make(name, seed=None, allocator=None):
    """The named workload.  ``seed`` defaults to 394 + its index in
    ``NAMES + PREFILL_NAMES``.  ``prefix_share`` lays its blocks out with
    ``allocator`` (see build_prefix_share_workload); the others need none."""
    idx = (NAMES + PREFILL_NAMES).index(name)
    seed = SEED_BASE + idx if seed is None else seed
    rng = np.random.default_rng(seed + 1000)   # lengths; values use ``seed``
    if name == "llama7b_prefill":
        # a chunked-prefill batch of 2048 new tokens (the batched-token budget
        # of the vLLM examples), 512 per sequence, on top of 0..3072 cached
        return build_prefill_workload(rng.integers(0, 3072 + 1, size=4), [512] * 4, 32, 32, 128,
                                      16, "fp16", seed, name=name)
    if name == "gqa_prefill":
        return build_prefill_workload(rng.integers(0, 3072 + 1, size=4), [512] * 4, 32, 8, 128,
                                      32, "bf16", seed, name=name)
    if name == "skew_prefill":
        # the same budget with one long cached history among short ones (a
        # chunk of a long prompt, or a long shared prefix, beside new prompts)
        return build_prefill_workload([8192, 100, 50, 0], [512] * 4, 32, 32, 128, 16, "fp16",
                                      seed, name=name)
    if name == "tiny":
        return build_decode_workload([5, 17, 32, 100], 4, 4, 64, 16, "fp16", seed,
                                     num_blocks=64, name=name)
    if name == "llama7b":
        lens = rng.integers(128, 2048 + 1, size=64)
        return build_decode_workload(lens, 32, 32, 128, 16, "fp16", seed, name=name)
    if name == "gqa_chat":
        lens = chat_lengths(rng, 256)
        return build_decode_workload(lens, 32, 8, 128, 32, "bf16", seed, name=name)
    if name == "long_splitk":
        lens = rng.integers(16384, 32768 + 1, size=8)
        return build_decode_workload(lens, 40, 40, 128, 16, "fp16", seed, name=name,
                                     partition_size=512)
    if name == "prefix_share":
        if allocator is None:
            raise ValueError("prefix_share lays out its blocks with a block allocator")
        return build_prefix_share_workload(64, 8, 1020, 64, 256, 64, 8, 128, 16, "bf16",
                                           seed, allocator)
    raise KeyError(name)


def describe(w):
    """Sizes of a workload, for logs and the benchmark's config object."""
    return {
        "workload": w.name, "num_seqs": w.num_seqs, "num_heads": w.num_heads,
        "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
        "block_size": w.block_size, "dtype": w.dtype, "num_blocks": w.num_blocks,
        "sum_context": int(w.context_lens.astype(np.int64).sum()),
        "max_context": w.max_context_len, "new_tokens": int(len(w.slot_mapping)),
        "cow_pairs": int(len(w.cow_pairs)), "partition_size": w.partition_size,
        **({"query_tokens": int(w.query_start[-1]),
            "max_query_len": int(np.diff(w.query_start).max())}
           if w.query_start is not None else {}),
    }
