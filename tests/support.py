"""Helpers shared by the GPU tests: move a workload to the device, run its
step through the library's C ABI, and run the same step through the oracle.

The two sides share only the workload (drawn by paged_kv_cache_394_b200.
workloads); the device side uses the ctypes binding, the oracle side uses
oracle/ alone.
"""

import numpy as np
import torch

from oracle import attention as OA
from oracle import cache_ops as OC

# |gpu - ref| <= ATOL + RTOL * |ref| elementwise, against the float64 oracle
# before any rounding; covers bf16's half-ulp (2^-9 relative).
ATOL = 2e-3
RTOL = 1e-2


def block_allocator(num_blocks, block_size, free_order):
    """The library's C++ block allocator: it lays out the shared, copied and
    fresh blocks of the parallel-sampling workloads."""
    from paged_kv_cache_394_b200 import pagedkv as pk
    return pk.BlockAllocator(num_blocks, block_size, free_order)


def torch_dtype(w):
    return torch.float16 if w.dtype == "fp16" else torch.bfloat16


def bits_to_dev(a, w):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch_dtype(w))


def dev_to_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class DeviceWorkload:
    """The workload's tensors on the current CUDA device."""

    def __init__(self, w):
        self.w = w
        self.q = bits_to_dev(w.q, w)
        self.k_cache = bits_to_dev(w.k_cache, w)
        self.v_cache = bits_to_dev(w.v_cache, w)
        self.key = bits_to_dev(w.key, w)
        self.value = bits_to_dev(w.value, w)
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.pairs = torch.from_numpy(np.ascontiguousarray(w.cow_pairs)).cuda()
        self.tables = torch.from_numpy(w.block_tables).cuda()
        self.lens = torch.from_numpy(w.context_lens).cuda()
        self.out = torch.empty_like(self.q)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.qstart = (torch.from_numpy(w.query_start).cuda()
                       if w.query_start is not None else None)


def run_step(pk, dw, partition_size=None, decode=True):
    """copy_blocks -> reshape_and_cache -> paged_attn_decode on the device."""
    w = dw.w
    part = w.partition_size if partition_size is None else partition_size
    if len(w.cow_pairs):
        pk.copy_blocks(dw.k_cache, dw.v_cache, dw.pairs, dev_err=dw.err)
    if len(w.slot_mapping):
        pk.reshape_and_cache(dw.key, dw.value, dw.k_cache, dw.v_cache, dw.slots, dev_err=dw.err)
    if decode:
        pk.paged_attn_decode(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, w.scale,
                             w.num_kv_heads, w.block_size, w.max_context_len,
                             partition_size=part, dev_err=dw.err)
    torch.cuda.synchronize()
    return int(dw.err.item())


def run_prefill_step(pk, dw):
    """reshape_and_cache of the new tokens, then chunked-prefill attention."""
    w = dw.w
    pk.reshape_and_cache(dw.key, dw.value, dw.k_cache, dw.v_cache, dw.slots, dev_err=dw.err)
    pk.paged_attn_prefill(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, dw.qstart,
                          w.scale, w.num_kv_heads, w.block_size, w.max_context_len,
                          int(np.diff(w.query_start).max()), dev_err=dw.err)
    torch.cuda.synchronize()
    return int(dw.err.item())


def oracle_prefill(w, kc, vc, rows=None):
    return OA.paged_attention_prefill(w.q, kc, vc, w.block_tables, w.context_lens,
                                      w.query_start, w.scale, w.num_kv_heads, w.block_size,
                                      w.dtype, rows=rows)


def oracle_caches(w, inplace=False):
    kc, vc, bad1 = OC.copy_blocks(w.k_cache, w.v_cache, w.cow_pairs, inplace=inplace)
    kc, vc, bad2 = OC.reshape_and_cache(w.key, w.value, kc, vc, w.slot_mapping, w.block_size,
                                        inplace=inplace)
    assert not bad1 and not bad2
    return kc, vc


def oracle_decode(w, kc, vc, pairs=None):
    return OA.paged_attention_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale,
                                     w.num_kv_heads, w.block_size, w.dtype, pairs=pairs)


def widen_out(bits, w):
    from oracle.dtypes import widen
    return widen(bits, w.dtype)


def assert_close(got_bits, ref, w, pairs=None):
    """Elementwise |got - ref| <= ATOL + RTOL*|ref| on the compared rows."""
    got = widen_out(got_bits, w)
    if pairs is not None:
        idx = tuple(np.array(pairs).T)
        got, ref = got[idx], ref[idx]
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), "max excess %.3g at %s (got %r, ref %r)" % (
        (err - bound)[worst], worst, got[worst], ref[worst])
    return float(err.max())
