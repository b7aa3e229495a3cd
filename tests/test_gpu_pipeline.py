"""Pipelined host-buffer decode steps (pkv_decode_pipeline_*, through the C
ABI): overlapping step i+1's upload and step i-1's download with step i's
kernels must not change any result.  Every pipelined step's output must equal,
bit for bit, the one-call host step (pkv_decode_step_host) on the same host
inputs, and the caches must end as one serial step leaves them (the step's
block copies and cache writes are the same every time, so repeating them
changes nothing)."""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import DeviceWorkload, block_allocator, dev_to_bits

pytestmark = pytest.mark.gpu


def pinned(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.view(dtype))
    return torch.from_numpy(a).pin_memory()


@pytest.mark.parametrize("part", [0, 64])
def test_pipelined_steps_equal_serial_steps(part):
    from paged_kv_cache_394_b200 import pagedkv as pk
    # parallel sampling: copy pairs, cache writes and shared prompt blocks
    w = W.build_prefix_share_workload(3, 4, 45, 3, 30, 16, 4, 128, 16, "fp16", seed=23,
                                      allocator=block_allocator)
    f16 = torch.float16
    h_key = pinned(w.key, np.int16).view(f16)
    h_val = pinned(w.value, np.int16).view(f16)
    h_slots, h_pairs = pinned(w.slot_mapping), pinned(w.cow_pairs)
    h_tables, h_lens = pinned(w.block_tables), pinned(w.context_lens)
    rng = np.random.default_rng(3)
    # two query batches, alternated over the steps
    qs = [pinned(w.q, np.int16).view(f16),
          pinned(W._normal_bits(rng, w.q.shape, w.dtype), np.int16).view(f16)]
    t, p = len(w.slot_mapping), len(w.cow_pairs)

    # the reference: one-call host steps, one per query batch
    ref_dw = DeviceWorkload(w)
    staging1 = torch.empty(pk.staging_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                            w.max_blocks_per_seq, t, p),
                           dtype=torch.uint8, device="cuda")
    ws1 = pk.alloc_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                             w.max_context_len, part)
    expect = []
    for q in qs:
        out_h = torch.empty(w.q.shape, dtype=f16).pin_memory()
        pk.decode_step_host(out_h, q, h_key, h_val, h_slots, h_pairs, h_tables, h_lens,
                            ref_dw.k_cache, ref_dw.v_cache, w.scale, w.max_context_len, staging1,
                            workspace=ws1, partition_size=part, dev_err=ref_dw.err)
        torch.cuda.synchronize()
        expect.append(out_h.view(torch.int16).numpy().copy())
    assert int(ref_dw.err.item()) == 0
    assert not np.array_equal(expect[0], expect[1])

    dw = DeviceWorkload(w)
    stream = torch.cuda.Stream()
    staging = torch.empty(pk.DecodePipeline.staging_bytes(
        w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_blocks_per_seq, t, p),
        dtype=torch.uint8, device="cuda")
    ws = pk.alloc_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                            w.max_context_len, part)
    pipe = pk.DecodePipeline(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                             w.max_blocks_per_seq, t, p, f16, staging, stream=stream)
    n = 7
    outs = [torch.full(w.q.shape, -1, dtype=torch.int16).pin_memory().view(f16)
            for _ in range(n)]
    for i in range(n):
        pipe.step(outs[i], qs[i % 2], h_key, h_val, h_slots, h_pairs, h_tables, h_lens,
                  dw.k_cache, dw.v_cache, w.scale, w.max_context_len, workspace=ws,
                  partition_size=part, dev_err=dw.err)
    pipe.sync()
    torch.cuda.synchronize()
    pipe.close()
    assert int(dw.err.item()) == 0
    for i in range(n):
        assert np.array_equal(outs[i].view(torch.int16).numpy(), expect[i % 2]), i
    assert np.array_equal(dev_to_bits(dw.k_cache), dev_to_bits(ref_dw.k_cache))
    assert np.array_equal(dev_to_bits(dw.v_cache), dev_to_bits(ref_dw.v_cache))


def test_pipeline_join_orders_later_work():
    """Work enqueued on a stream after join() sees every step's output."""
    from paged_kv_cache_394_b200 import pagedkv as pk
    w = W.build_decode_workload([33, 400, 17, 128], 8, 2, 128, 16, "bf16", 29)
    dw = DeviceWorkload(w)
    bf = torch.bfloat16
    t = len(w.slot_mapping)
    staging = torch.empty(pk.DecodePipeline.staging_bytes(
        w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_blocks_per_seq, t, 0),
        dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    pipe = pk.DecodePipeline(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                             w.max_blocks_per_seq, t, 0, bf, staging, stream=stream)
    out_h = torch.empty(w.q.shape, dtype=bf).pin_memory()
    ws = pk.alloc_workspace(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                            w.max_context_len)   # four sequences: split-K
    empty_pairs = torch.zeros((0, 2), dtype=torch.int64).pin_memory()
    pipe.step(out_h, pinned(w.q, np.int16).view(bf), pinned(w.key, np.int16).view(bf),
              pinned(w.value, np.int16).view(bf), pinned(w.slot_mapping), empty_pairs,
              pinned(w.block_tables), pinned(w.context_lens), dw.k_cache, dw.v_cache, w.scale,
              w.max_context_len, workspace=ws, dev_err=dw.err)
    done = torch.cuda.Event()
    other = torch.cuda.Stream()
    pipe.join(other)
    done.record(other)
    done.synchronize()
    pipe.close()
    # the same step on the device path
    ref = DeviceWorkload(w)
    pk.reshape_and_cache(ref.key, ref.value, ref.k_cache, ref.v_cache, ref.slots, dev_err=ref.err)
    pk.paged_attn_decode(ref.out, ref.q, ref.k_cache, ref.v_cache, ref.tables, ref.lens, w.scale,
                         w.num_kv_heads, w.block_size, w.max_context_len, dev_err=ref.err)
    torch.cuda.synchronize()
    assert int(dw.err.item()) == 0 and int(ref.err.item()) == 0
    assert np.array_equal(out_h.view(torch.int16).numpy().view(np.uint16), dev_to_bits(ref.out))
