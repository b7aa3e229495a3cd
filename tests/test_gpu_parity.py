"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

* reshape_and_cache and copy_blocks: bit-exact.
* paged_attn_decode: |gpu - ref| <= 2e-3 + 1e-2*|ref| elementwise.

Small cases are compared in full; the five named workloads run at full size in
the launch configuration the benchmark uses and are compared on sampled
(sequence, head) rows plus properties that hold at any size.
"""

import math

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import (DeviceWorkload, block_allocator, assert_close, dev_to_bits, oracle_caches, oracle_decode,
                     run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


RAGGED = [1, 5, 16, 17, 33, 100, 257, 600]


def small_workload(d, bs, g, dtype, lens=RAGGED, hkv=2, seed=7):
    return W.build_decode_workload(lens, g * hkv, hkv, d, bs, dtype,
                                   seed + d + bs + g + (dtype == "bf16"))


# ---------------------------------------------------------------------------
# bit-exact data movement
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,bs,dtype", [(64, 16, "fp16"), (128, 32, "bf16"), (128, 16, "fp16")])
def test_cache_write_bit_exact_small(pk, d, bs, dtype):
    w = small_workload(d, bs, 1, dtype)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    kc, vc = oracle_caches(w)
    assert np.array_equal(dev_to_bits(dw.k_cache), kc)
    assert np.array_equal(dev_to_bits(dw.v_cache), vc)


def test_copy_blocks_and_write_bit_exact(pk):
    w = W.build_prefix_share_workload(3, 4, 37, 5, 40, 8, 2, 64, 16, "bf16", seed=3,
                                      allocator=block_allocator)
    assert len(w.cow_pairs) == 3 * 3
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    kc, vc = oracle_caches(w)
    assert np.array_equal(dev_to_bits(dw.k_cache), kc)
    assert np.array_equal(dev_to_bits(dw.v_cache), vc)


def test_reshape_skips_negative_slots_and_flags_out_of_range(pk):
    w = small_workload(64, 16, 1, "fp16")
    dw = DeviceWorkload(w)
    before_k = dev_to_bits(dw.k_cache)
    slots = w.slot_mapping.copy()
    slots[0] = -1
    slots[1] = w.num_blocks * w.block_size          # one past the pool
    dw.slots = torch.from_numpy(slots).cuda()
    err = run_step(pk, dw, decode=False)
    assert err & pk.DEVERR_BAD_SLOT
    after_k = dev_to_bits(dw.k_cache)
    for t in (0, 1):
        b, o = divmod(int(w.slot_mapping[t]), w.block_size)
        assert np.array_equal(after_k[b, :, o], before_k[b, :, o])
    b, o = divmod(int(w.slot_mapping[2]), w.block_size)
    assert np.array_equal(after_k[b, :, o], w.key[2])


def test_copy_blocks_flags_bad_pairs(pk):
    w = small_workload(64, 16, 1, "fp16")
    dw = DeviceWorkload(w)
    before = dev_to_bits(dw.k_cache)
    pairs = torch.tensor([[0, 1], [-1, 2], [3, w.num_blocks]], dtype=torch.int64, device="cuda")
    pk.copy_blocks(dw.k_cache, dw.v_cache, pairs, dev_err=dw.err)
    torch.cuda.synchronize()
    assert int(dw.err.item()) & pk.DEVERR_BAD_PAIR
    after = dev_to_bits(dw.k_cache)
    assert np.array_equal(after[1], before[0])
    assert np.array_equal(after[2], before[2])


# ---------------------------------------------------------------------------
# decode: every built shape, single pass and split-K, compared in full
# ---------------------------------------------------------------------------
SHAPES = [(d, bs, g, dt) for d in (64, 128) for bs in (16, 32) for g in (1, 2, 4, 8)
          for dt in ("fp16", "bf16")]


@pytest.mark.parametrize("d,bs,g,dtype", SHAPES)
def test_decode_all_shapes(pk, d, bs, g, dtype):
    w = small_workload(d, bs, g, dtype)
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    for part in (0, 2 * bs, 128):
        dw = DeviceWorkload(w)
        assert run_step(pk, dw, partition_size=part) == 0
        assert_close(dev_to_bits(dw.out), ref, w)


def test_decode_many_partitions_ragged(pk):
    lens = [1, 511, 512, 513, 1500, 4097, 9000]
    w = W.build_decode_workload(lens, 8, 8, 128, 16, "fp16", 99)
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    for part in (0, 16, 512, 4096):
        dw = DeviceWorkload(w)
        assert run_step(pk, dw, partition_size=part) == 0
        assert_close(dev_to_bits(dw.out), ref, w)


# ---------------------------------------------------------------------------
# edge cases and the device error word
# ---------------------------------------------------------------------------
def test_empty_and_single_token_contexts(pk):
    w = W.build_decode_workload([1, 2, 1, 3], 4, 2, 128, 16, "bf16", 5, num_blocks=16)
    dw = DeviceWorkload(w)
    dw.lens = torch.tensor([0, 1, 1, 3], dtype=torch.int32, device="cuda")
    assert run_step(pk, dw) == 0
    out = dev_to_bits(dw.out)
    assert (out[0] == 0).all()                          # empty context -> zeros
    kc, vc = oracle_caches(w)
    for i in (1, 2):                                    # one token -> its value vector, exactly
        b = w.block_tables[i, 0]
        for h in range(4):
            assert np.array_equal(out[i, h], vc[b, h // 2, 0])


def test_zero_sequences_is_a_no_op(pk):
    q = torch.empty(0, 4, 64, dtype=torch.float16, device="cuda")
    kc = torch.zeros(4, 4, 16, 64, dtype=torch.float16, device="cuda")
    pk.paged_attn_decode(q, q, kc, kc, torch.zeros(0, 1, dtype=torch.int32, device="cuda"),
                         torch.zeros(0, dtype=torch.int32, device="cuda"), 0.1, 4, 16, 0)
    torch.cuda.synchronize()


def test_bad_block_id_is_reported_not_faulted(pk):
    w = small_workload(128, 16, 1, "fp16")
    dw = DeviceWorkload(w)
    tables = w.block_tables.copy()
    tables[6, 3] = w.num_blocks + 5
    tables[7, 0] = -7
    dw.tables = torch.from_numpy(tables).cuda()
    err = run_step(pk, dw)
    assert err & pk.DEVERR_BAD_BLOCK
    # the sequences without bad entries are still right
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc, pairs=[(s, h) for s in range(6) for h in range(2)])
    assert_close(dev_to_bits(dw.out), ref, w, pairs=[(s, h) for s in range(6) for h in range(2)])


def test_bad_context_len_is_reported(pk):
    w = small_workload(64, 16, 1, "fp16")
    dw = DeviceWorkload(w)
    lens = w.context_lens.copy()
    lens[0] = -3
    lens[1] = w.max_context_len + 1
    dw.lens = torch.from_numpy(lens).cuda()
    err = run_step(pk, dw)
    assert err & pk.DEVERR_BAD_CONTEXT
    assert (dev_to_bits(dw.out)[0] == 0).all()


def test_table_padding_is_never_read(pk):
    # entries past each sequence's last block are -1; no error may be raised
    w = small_workload(128, 32, 2, "bf16")
    assert (w.block_tables == -1).any()
    dw = DeviceWorkload(w)
    for part in (0, 32):
        assert run_step(pk, dw, partition_size=part) == 0


def test_placement_invariance_on_gpu(pk):
    w = small_workload(128, 16, 4, "bf16", seed=17)
    dw = DeviceWorkload(w)
    run_step(pk, dw)
    base = dev_to_bits(dw.out)
    rng = np.random.default_rng(0)
    perm = rng.permutation(w.num_blocks)
    moved = dict(vars(w))
    moved["k_cache"] = np.empty_like(w.k_cache)
    moved["v_cache"] = np.empty_like(w.v_cache)
    moved["k_cache"][perm] = w.k_cache
    moved["v_cache"][perm] = w.v_cache
    moved["block_tables"] = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)],
                                     -1).astype(np.int32)
    bs = w.block_size
    moved["slot_mapping"] = np.array([perm[s // bs] * bs + s % bs for s in w.slot_mapping])
    w2 = W.Workload(**moved)
    dw2 = DeviceWorkload(w2)
    run_step(pk, dw2)
    assert np.array_equal(dev_to_bits(dw2.out), base)


def test_host_buffer_step_matches_device_step(pk):
    w = W.build_prefix_share_workload(2, 4, 45, 3, 30, 16, 4, 128, 16, "fp16", seed=8,
                                      allocator=block_allocator)
    dw = DeviceWorkload(w)
    run_step(pk, dw)
    expect = dev_to_bits(dw.out)
    dw2 = DeviceWorkload(w)

    def pinned(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.view(dtype)))
        return t.pin_memory()
    out_h = torch.empty(w.q.shape, dtype=torch.int16).pin_memory()
    staging = torch.empty(pk.staging_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                           w.max_blocks_per_seq, len(w.slot_mapping),
                                           len(w.cow_pairs)), dtype=torch.uint8, device="cuda")
    pk.decode_step_host(out_h.view(torch.float16), pinned(w.q, np.int16).view(torch.float16),
                        pinned(w.key, np.int16).view(torch.float16),
                        pinned(w.value, np.int16).view(torch.float16), pinned(w.slot_mapping),
                        pinned(w.cow_pairs), pinned(w.block_tables), pinned(w.context_lens),
                        dw2.k_cache, dw2.v_cache, w.scale, w.max_context_len, staging,
                        dev_err=dw2.err)
    torch.cuda.synchronize()
    assert int(dw2.err.item()) == 0
    assert np.array_equal(out_h.numpy().view(np.uint16), expect)
    # compare bit patterns: the pools hold NaN poison, and NaN != NaN
    assert torch.equal(dw2.k_cache.view(torch.int16), dw.k_cache.view(torch.int16))
    assert torch.equal(dw2.v_cache.view(torch.int16), dw.v_cache.view(torch.int16))


# ---------------------------------------------------------------------------
# the named workloads at full size
# ---------------------------------------------------------------------------
def sample_pairs(w, n, seed):
    rng = np.random.default_rng(seed)
    lens = w.context_lens
    seqs = {int(np.argmax(lens)), int(np.argmin(lens))}
    seqs.update(int(s) for s in rng.integers(0, w.num_seqs, size=n))
    pairs = []
    for s in sorted(seqs):
        for h in sorted(set([0, w.num_heads - 1] + [int(x) for x in rng.integers(0, w.num_heads, 2)])):
            pairs.append((s, h))
    return pairs


@pytest.mark.parametrize("name", W.NAMES)
def test_named_workload(pk, name):
    # prefix_share: the C++ allocator forks the prompts and makes the copy pairs
    w = W.make(name, allocator=block_allocator)
    dw = DeviceWorkload(w)
    k_before = dw.k_cache.clone()
    err = run_step(pk, dw)
    assert err == 0
    # cache writes: every written slot holds its token, nothing else changed
    bs = w.block_size
    slots = torch.from_numpy(w.slot_mapping).cuda()
    blk, off = slots // bs, slots % bs
    written = dw.k_cache[blk, :, off, :]
    assert torch.equal(written.view(torch.int16).cpu(),
                       torch.from_numpy(w.key.view(np.int16)))
    assert torch.equal(dw.v_cache[blk, :, off, :].view(torch.int16).cpu(),
                       torch.from_numpy(w.value.view(np.int16)))
    mask = torch.ones(dw.k_cache.shape[0], bs, dtype=torch.bool, device="cuda")
    mask[blk, off] = False
    if len(w.cow_pairs):
        # each copied block equals its source as it was before the step,
        # at every offset this step did not write into the copy
        blk_c, off_c = blk.cpu(), off.cpu()
        for s_, d_ in w.cow_pairs.tolist():
            wr = torch.zeros(bs, dtype=torch.bool)
            wr[off_c[blk_c == d_]] = True
            keep = (~wr).cuda()
            assert torch.equal(dw.k_cache[d_][:, keep].view(torch.int16),
                               k_before[s_][:, keep].view(torch.int16))
            mask[d_] = False
    kb = k_before.view(torch.int16).permute(0, 2, 1, 3)[mask]
    ka = dw.k_cache.view(torch.int16).permute(0, 2, 1, 3)[mask]
    assert torch.equal(ka, kb)
    del k_before, kb, ka
    # decode on sampled rows
    pairs = sample_pairs(w, 6, seed=len(name))
    kc, vc = oracle_caches(w, inplace=True)
    ref = oracle_decode(w, kc, vc, pairs=pairs)
    assert_close(dev_to_bits(dw.out), ref, w, pairs=pairs)
    out = dev_to_bits(dw.out)
    from oracle.dtypes import widen
    assert np.isfinite(widen(out, w.dtype)).all()


def test_split_and_single_pass_agree_at_full_size(pk):
    w = W.make("llama7b")
    dw = DeviceWorkload(w)
    run_step(pk, dw, partition_size=0)
    single = dw.out.float().clone()
    for part in (256, 512):
        run_step(pk, dw, partition_size=part)
        split = dw.out.float()
        # both are within tolerance of the true values, so of each other twice that
        bound = 2 * (2e-3 + 1e-2 * single.abs())
        assert ((split - single).abs() <= bound).all()
    pairs = sample_pairs(w, 4, seed=1)
    kc, vc = oracle_caches(w, inplace=True)
    assert_close(dev_to_bits(dw.out), oracle_decode(w, kc, vc, pairs=pairs), w, pairs=pairs)
    assert math.isfinite(float(single.abs().max()))
