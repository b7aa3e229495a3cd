"""The C++ host block allocator against the oracle block manager: identical
slots, copy pairs, tables, refcounts and free counts (bit-exact integer work)
on random operation traces, plus its error statuses."""

import numpy as np
import pytest

from oracle.block_manager import AllocError, BlockManager

pk = pytest.importorskip("paged_kv_cache_394_b200.pagedkv")

STATUS = {"INVALID_ARG": 1, "OUT_OF_BLOCKS": 5}


def both(oracle_call, lib_call):
    """Run one operation on both; they must agree on success, result and error."""
    try:
        expect = oracle_call()
        err = None
    except AllocError as e:
        expect, err = None, STATUS[e.status]
    try:
        got = lib_call()
        got_err = None
    except pk.PagedKVError as e:
        got, got_err = None, e.status
    assert got_err == err
    assert got == expect
    return err is None


@pytest.mark.parametrize("seed,num_blocks,bs", [(1, 40, 16), (2, 97, 32), (3, 12, 16), (4, 300, 16)])
def test_random_traces_match_oracle(seed, num_blocks, bs):
    rng = np.random.default_rng(seed)
    order = rng.permutation(num_blocks)
    ref = BlockManager(num_blocks, bs, free_order=order)
    lib = pk.BlockAllocator(num_blocks, bs, free_order=order)
    live, next_id = [], 0
    for _ in range(1500):
        op = int(rng.integers(0, 12))
        if op < 2 or not live:
            n = int(rng.integers(0, 5 * bs))
            if both(lambda: ref.add_seq(next_id, n), lambda: lib.add_seq(next_id, n)):
                live.append(next_id)
            next_id += 1
        elif op < 4:
            parent = live[int(rng.integers(len(live)))]
            if both(lambda: ref.fork(parent, next_id), lambda: lib.fork(parent, next_id)):
                live.append(next_id)
            next_id += 1
        elif op < 9:
            s = live[int(rng.integers(len(live)))]
            both(lambda: ref.append_slot(s), lambda: lib.append_slot(s))
        elif op < 10:
            batch = [live[int(i)] for i in rng.integers(0, len(live), size=int(rng.integers(1, 6)))]

            def ref_batch():
                slots, pairs = [], []
                for s in batch:
                    slot, a, b = ref.append_slot(s)
                    slots.append(slot)
                    if a >= 0:
                        pairs.append((a, b))
                return slots, pairs
            # a batch that runs out part-way leaves both in the same partial state
            try:
                expect = ref_batch()
            except AllocError as e:
                expect = e.status
            try:
                got = lib.append_slots(batch)
            except pk.PagedKVError as e:
                got = {1: "INVALID_ARG", 5: "OUT_OF_BLOCKS"}[e.status]
            assert got == expect
        elif op < 11:
            s = live.pop(int(rng.integers(len(live))))
            both(lambda: ref.free_seq(s), lambda: lib.free_seq(s))
        else:
            bogus = next_id + 1000
            both(lambda: ref.free_seq(bogus), lambda: lib.free_seq(bogus))
        # full state comparison
        assert lib.num_free() == ref.num_free()
        if live:
            mb = max(1, max(len(ref.seq_blocks(s)) for s in live))
            assert lib.block_table(live, mb) == ref.block_table(live, mb)
            assert lib.context_lens(live) == [ref.seq_len(s) for s in live]
    assert [lib.refcount(b) for b in range(num_blocks)] == ref.refcount
    tokens, blocks = lib.usage()
    if blocks:
        assert tokens / (blocks * bs) == pytest.approx(ref.physical_utilization(), abs=1e-15)


def test_parallel_sampling_scenario():
    lib = pk.BlockAllocator(200, 16)
    lib.add_seq(0, 1020)
    for c in range(1, 8):
        lib.fork(0, c)
    slots, pairs = lib.append_slots(list(range(8)))
    assert len(pairs) == 7 and len(set(d for _, d in pairs)) == 7
    assert all(s % 16 == 1020 % 16 for s in slots)
    assert lib.num_free() == 200 - 64 - 7


def test_error_statuses():
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator(0, 16)
    with pytest.raises(pk.PagedKVError):
        pk.BlockAllocator(4, 16, free_order=[0, 0, 1, 2])
    a = pk.BlockAllocator(2, 16)
    a.add_seq(7, 20)
    with pytest.raises(pk.PagedKVError) as e:
        a.add_seq(8, 1)
    assert e.value.status == pk.ERR_OUT_OF_BLOCKS
    with pytest.raises(pk.PagedKVError) as e:
        a.add_seq(7, 1)
    assert e.value.status == pk.ERR_INVALID_ARG
    with pytest.raises(pk.PagedKVError):
        a.block_table([7], 1)
    assert a.refcount(5) == -1 and a.seq_len(99) == -1
    assert a.seq_num_blocks(7) == 2


@pytest.mark.parametrize("seed,num_blocks,bs", [(11, 48, 4), (12, 120, 16), (13, 20, 2)])
def test_prefix_cache_traces_match_oracle(seed, num_blocks, bs):
    rng = np.random.default_rng(seed)
    order = rng.permutation(num_blocks)
    ref = BlockManager(num_blocks, bs, free_order=order)
    lib = pk.BlockAllocator(num_blocks, bs, free_order=order)
    # a few "system prompts" so that prefixes repeat, plus random tails
    bases = [list(rng.integers(0, 7, int(rng.integers(0, 6 * bs)))) for _ in range(5)]
    live, next_id = [], 0
    for _ in range(1200):
        op = int(rng.integers(0, 10))
        if op < 4 or not live:
            toks = bases[int(rng.integers(len(bases)))] + \
                list(rng.integers(0, 7, int(rng.integers(0, 2 * bs))))
            if both(lambda: ref.add_seq_cached(next_id, toks),
                    lambda: lib.add_seq_cached(next_id, toks)):
                live.append(next_id)
            next_id += 1
        elif op < 5:
            parent = live[int(rng.integers(len(live)))]
            if both(lambda: ref.fork(parent, next_id), lambda: lib.fork(parent, next_id)):
                live.append(next_id)
            next_id += 1
        elif op < 7:
            s = live[int(rng.integers(len(live)))]
            both(lambda: ref.append_slot(s), lambda: lib.append_slot(s))
        else:
            s = live.pop(int(rng.integers(len(live))))
            both(lambda: ref.free_seq(s), lambda: lib.free_seq(s))
        assert lib.num_free() == ref.num_free()
        assert lib.num_evictable() == ref.num_evictable()
        assert lib.cache_stats() == ref.cache_stats()
        if live:
            mb = max(1, max(len(ref.seq_blocks(s)) for s in live))
            assert lib.block_table(live, mb) == ref.block_table(live, mb)
    assert [lib.refcount(b) for b in range(num_blocks)] == ref.refcount
    q, h, _, ev = lib.cache_stats()
    assert h > 0 and ev > 0          # the trace exercised hits and evictions


def test_parallel_sampling_workload_layout_matches_oracle():
    """The full-size parallel-sampling workload (64 prompts x 8 samples, a
    1020-token prompt in blocks of 16) laid out by the C++ allocator and by
    the oracle block manager from the same free order: identical block
    tables, slots and copy pairs.  Each prompt's shared partial block is
    copied on write for the first 7 samples to append (the last writes in
    place), so the step carries 64 x 7 = 448 pairs."""
    from paged_kv_cache_394_b200 import workloads as W
    lib = W.make("prefix_share", allocator=pk.BlockAllocator)
    ref = W.make("prefix_share", allocator=BlockManager)
    assert np.array_equal(lib.block_tables, ref.block_tables)
    assert np.array_equal(lib.slot_mapping, ref.slot_mapping)
    assert np.array_equal(lib.cow_pairs, ref.cow_pairs)
    assert len(lib.cow_pairs) == 448
    bs, samples = lib.block_size, lib.notes["samples"]
    last = lib.notes["prompt_blocks"] - 1            # the partial prompt block
    for p in range(64):
        rows = lib.block_tables[p * samples:(p + 1) * samples]
        src = rows[-1, last]                          # the last sample kept the original
        pairs = lib.cow_pairs[7 * p:7 * p + 7]
        assert (pairs[:, 0] == src).all()
        assert list(pairs[:, 1]) == list(rows[:-1, last])
    assert len(set(lib.cow_pairs[:, 1].tolist())) == 448
    assert not set(lib.cow_pairs[:, 1].tolist()) & set(lib.cow_pairs[:, 0].tolist())
    # every new token lands past its sequence's prompt, in its own table row
    s = np.repeat(np.arange(lib.num_seqs), lib.context_lens - 1020)
    pos = np.concatenate([np.arange(1020, c) for c in lib.context_lens])
    assert np.array_equal(lib.slot_mapping,
                          lib.block_tables[s, pos // bs].astype(np.int64) * bs + pos % bs)
