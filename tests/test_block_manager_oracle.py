"""Pins for the oracle block manager, from what the pages state.

* The worked example (100/300/500 tokens under a contiguous 500-token
  reservation use 60 % of it) is read from tests/golden/, where it is stored
  with its citation.
* Only each sequence's last block can be partly empty, and waste stays below
  4 % (stored in tests/golden/ with its citation).
* Finished sequences return their blocks for reuse.
* Shared blocks are reference-counted; copy-on-write happens only when a
  shared block must be modified.
"""

import json
import os

import numpy as np
import pytest

from oracle.block_manager import (AllocError, BlockManager, blocks_for,
                                  contiguous_utilization, paged_utilization)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_worked_example_contiguous_utilization():
    g = golden("worked_example_utilization.json")
    assert contiguous_utilization(g["lengths"], g["reserved_len"]) == pytest.approx(
        g["utilization"], abs=1e-12)


def test_worked_example_paged_waste_below_bound():
    ex = golden("worked_example_utilization.json")
    bound = golden("waste_bound.json")["max_waste_fraction"]
    # the pages' usual page size is 16 tokens; there the example wastes 3 %
    util = paged_utilization(ex["lengths"], 16)
    assert 1.0 - util < bound, util
    # whatever the page size, each sequence wastes less than one page
    for bs in (16, 32, 64):
        slots = sum(blocks_for(n, bs) * bs for n in ex["lengths"])
        assert slots - sum(ex["lengths"]) < len(ex["lengths"]) * bs
    # the same through the manager: 7 + 19 + 32 = 58 blocks of 16 for 900 tokens
    mgr = BlockManager(64, 16)
    for i, n in enumerate(ex["lengths"]):
        mgr.add_seq(i, n)
    assert mgr.num_free() == 64 - 58
    assert mgr.physical_utilization() == pytest.approx(900 / (58 * 16), abs=1e-15)


def random_trace(mgr, rng, steps, max_seqs=12):
    """Random add / fork / append / free operations; yields after each one."""
    live = []
    next_id = 0
    for _ in range(steps):
        op = rng.integers(0, 10)
        try:
            if op < 2 or not live:
                mgr.add_seq(next_id, int(rng.integers(0, 70)))
                live.append(next_id)
                next_id += 1
            elif op < 4 and len(live) < max_seqs:
                mgr.fork(live[int(rng.integers(len(live)))], next_id)
                live.append(next_id)
                next_id += 1
            elif op < 9:
                mgr.append_slot(live[int(rng.integers(len(live)))])
            else:
                s = live.pop(int(rng.integers(len(live))))
                mgr.free_seq(s)
        except AllocError as e:
            assert e.status == "OUT_OF_BLOCKS"
        yield live


def test_waste_only_in_last_block_and_refcount_conservation():
    rng = np.random.default_rng(5)
    bs = 16
    mgr = BlockManager(96, bs, free_order=rng.permutation(96))
    for live in random_trace(mgr, rng, 600):
        held = [b for s in live for b in mgr.seq_blocks(s)]
        # every table entry is one reference
        assert sum(mgr.refcount) == len(held)
        # blocks are either free or referenced, never both
        assert len(set(held)) + mgr.num_free() == 96
        assert not (set(held) & set(mgr.free))
        for s in live:
            n, nb = mgr.seq_len(s), len(mgr.seq_blocks(s))
            assert nb == blocks_for(n, bs)
            assert nb * bs - n < bs           # only the last block has room left


def test_free_returns_every_block():
    rng = np.random.default_rng(6)
    mgr = BlockManager(64, 16, free_order=rng.permutation(64))
    live = []
    for live in random_trace(mgr, rng, 300):
        pass
    for s in list(live):
        mgr.free_seq(s)
    assert mgr.num_free() == 64
    assert sum(mgr.refcount) == 0


def test_parallel_samples_share_then_copy_on_write():
    bs = 16
    mgr = BlockManager(200, bs)
    mgr.add_seq(0, 1020)                     # 63 full blocks + a 12-token block
    for c in range(1, 8):
        mgr.fork(0, c)
    prompt = mgr.seq_blocks(0)
    assert all(mgr.refcount[b] == 8 for b in prompt)
    pairs = []
    for s in range(8):
        slot, src, dst = mgr.append_slot(s)
        if src >= 0:
            pairs.append((src, dst))
        assert slot % bs == 1020 % bs
    # reading: the last holder writes in place, so 8 samples make 7 copies
    assert len(pairs) == 7
    assert all(src == prompt[-1] for src, _ in pairs)
    assert len({dst for _, dst in pairs}) == 7
    assert mgr.refcount[prompt[-1]] == 1
    assert all(mgr.refcount[b] == 8 for b in prompt[:-1])   # full blocks stay shared
    # sharing saves memory: 8 samples hold 8·64 logical blocks in 63 + 8 physical ones
    assert 200 - mgr.num_free() == 63 + 8


def test_append_at_block_boundary_takes_fresh_block_without_copy():
    mgr = BlockManager(10, 16)
    mgr.add_seq(0, 32)
    mgr.fork(0, 1)
    slot, src, dst = mgr.append_slot(1)
    assert (src, dst) == (-1, -1)
    assert slot % 16 == 0 and slot // 16 not in mgr.seq_blocks(0)


def test_out_of_blocks_is_atomic():
    mgr = BlockManager(4, 16)
    mgr.add_seq(0, 40)                       # 3 blocks
    with pytest.raises(AllocError) as e:
        mgr.add_seq(1, 33)                   # needs 3, 1 left
    assert e.value.status == "OUT_OF_BLOCKS"
    assert mgr.num_free() == 1 and 1 not in mgr.seqs


def test_invalid_arguments():
    mgr = BlockManager(4, 16)
    with pytest.raises(AllocError):
        mgr.free_seq(3)
    with pytest.raises(AllocError):
        mgr.fork(0, 1)
    mgr.add_seq(0, 1)
    with pytest.raises(AllocError):
        mgr.add_seq(0, 1)
    with pytest.raises(AllocError):
        mgr.block_table([0], 0)
    with pytest.raises(AllocError):
        BlockManager(4, 16, free_order=[0, 1, 1, 2])


# ---------------------------------------------------------------------------
# prefix caching
# ---------------------------------------------------------------------------
def test_shared_system_prompt_hit_rate_closed_form():
    # n requests = k-block system prompt + a distinct 3-block suffix each:
    # the first misses everything, each later one hits exactly the k prompt blocks
    bs, k, n = 16, 5, 7
    rng = np.random.default_rng(0)
    system = list(rng.integers(0, 1000, k * bs))
    mgr = BlockManager(200, bs)
    for i in range(n):
        suffix = list(rng.integers(1000, 2000, 3 * bs))
        cached = mgr.add_seq_cached(i, system + suffix)
        assert cached == (0 if i == 0 else k * bs)
    queried, hits, cached_blocks, evicted = mgr.cache_stats()
    assert queried == n * (k + 3) and hits == (n - 1) * k
    assert hits / queried == pytest.approx((n - 1) * k / (n * (k + 3)))
    assert cached_blocks == k + 3 * n and evicted == 0
    # sharing: n sequences hold n*(k+3) logical blocks in k + 3n physical ones
    assert 200 - mgr.num_free() == k + 3 * n


def test_freed_prompt_stays_cached_then_hits():
    mgr = BlockManager(10, 4)
    toks = list(range(10))                  # 2 full blocks + 2 tokens
    assert mgr.add_seq_cached(0, toks) == 0
    mgr.free_seq(0)
    assert mgr.num_evictable() == 2 and mgr.num_free() == 8   # the partial block is not cached
    assert mgr.add_seq_cached(1, toks) == 8
    assert mgr.num_evictable() == 0


def test_lru_eviction_breaks_the_chain():
    mgr = BlockManager(4, 2)
    a = [1, 2, 3, 4]
    mgr.add_seq_cached(0, a)                # blocks 0, 1 cached
    mgr.free_seq(0)                         # evictable: 0 (older), 1
    mgr.add_seq_cached(1, [5, 6, 7, 8])     # takes free blocks 2, 3
    mgr.add_seq_cached(2, [9, 10])          # free list empty: evicts block 0 (a's first)
    assert mgr.seq_blocks(2) == [0]
    _, _, cached, evicted = mgr.cache_stats()
    assert evicted == 1 and cached == 4 - 1 + 1   # a's 2nd block, [5..8]'s two, [9,10]
    mgr.free_seq(2)
    # a's first block is gone, so its second (still cached) cannot be reached
    assert mgr.add_seq_cached(3, a) == 0


def test_prefix_cache_keeps_refcounts_and_blocks_consistent():
    rng = np.random.default_rng(9)
    bs = 4
    mgr = BlockManager(40, bs, free_order=rng.permutation(40))
    prompts = [list(rng.integers(0, 5, int(rng.integers(1, 30)))) for _ in range(6)]
    live = []
    for step in range(400):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                p = prompts[int(rng.integers(len(prompts)))]
                p = p + list(rng.integers(0, 5, int(rng.integers(0, 6))))
                mgr.add_seq_cached(step, p)
                live.append(step)
            elif op == 1:
                mgr.append_slot(live[int(rng.integers(len(live)))])
            else:
                mgr.free_seq(live.pop(int(rng.integers(len(live)))))
        except AllocError as e:
            assert e.status == "OUT_OF_BLOCKS"
        held = [b for s in live for b in mgr.seq_blocks(s)]
        assert sum(mgr.refcount) == len(held)
        assert len(set(held)) + mgr.num_free() + mgr.num_evictable() == 40
        for b in mgr.evictable:
            assert mgr.refcount[b] == 0 and b in mgr.cache_key
        for key, b in mgr.cache.items():
            assert mgr.cache_key[b] == key and len(key) % bs == 0


def test_append_slots_is_append_slot_in_order():
    """The batched form returns what one append_slot per id returns, in order,
    with the copy pairs of the appends that made one."""
    a, b = BlockManager(20, 4), BlockManager(20, 4)
    for m in (a, b):
        m.add_seq(1, 6)
        m.fork(1, 2)
        m.fork(1, 3)
    ids = [2, 3, 1, 2, 2, 3]
    slots, pairs = a.append_slots(ids)
    expect = [b.append_slot(i) for i in ids]
    assert slots == [s for s, _, _ in expect]
    assert pairs == [(s, d) for _, s, d in expect if s >= 0]
    assert len(pairs) == 2            # sequences 2 and 3 copy; 1, the last holder, writes in place
