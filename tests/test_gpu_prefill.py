"""Chunked-prefill attention on the GPU (through the C ABI) against the
float64 oracle: |gpu - ref| <= 2e-3 + 1e-2*|ref| elementwise."""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import (DeviceWorkload, assert_close, dev_to_bits, oracle_caches, oracle_decode,
                     oracle_prefill, run_prefill_step, run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


HIST = [0, 5, 16, 40, 100, 0]
NEW = [1, 17, 16, 33, 64, 70]
SHAPES = [(d, bs, g, dt) for d in (64, 128) for bs in (16, 32) for g in (1, 2, 4, 8)
          for dt in ("fp16", "bf16")]


@pytest.mark.parametrize("d,bs,g,dtype", SHAPES)
def test_prefill_all_shapes(pk, d, bs, g, dtype):
    w = W.build_prefill_workload(HIST, NEW, 2 * g, 2, d, bs, dtype, seed=d + bs + g)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    kc, vc = oracle_caches(w)
    assert np.array_equal(dev_to_bits(dw.k_cache), kc)
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc), w)


def test_prefill_long_history_and_many_tiles(pk):
    w = W.build_prefill_workload([3000, 0, 777], [200, 300, 129], 16, 4, 128, 16, "bf16", seed=5)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    kc, vc = oracle_caches(w)
    rng = np.random.default_rng(0)
    rows = sorted({(int(t), int(h)) for t, h in zip(rng.integers(0, 629, 60), rng.integers(0, 16, 60))}
                  | {(0, 0), (199, 15), (200, 3), (628, 7)})
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc, rows), w, pairs=rows)


def test_single_query_prefill_matches_decode(pk):
    # one new token per sequence: prefill and decode compute the same thing
    w = W.build_decode_workload([5, 100, 257, 1000], 8, 2, 128, 16, "fp16", 21)
    w.query_start = np.arange(w.num_seqs + 1, dtype=np.int32)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    pre = dw.out.float().clone()
    dw2 = DeviceWorkload(w)
    assert run_step(pk, dw2) == 0
    ref = oracle_decode(w, *oracle_caches(w))
    assert_close(dev_to_bits(dw.out), ref, w)
    assert ((pre - dw2.out.float()).abs() <= 2 * (2e-3 + 1e-2 * dw2.out.float().abs())).all()


def test_prefill_empty_queries_and_bad_lengths(pk):
    w = W.build_prefill_workload([4, 10, 3], [3, 0, 5], 4, 4, 64, 16, "fp16", seed=2)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    kc, vc = oracle_caches(w)
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc), w)
    # query count above the context length is reported and skipped
    bad = w.query_start.copy()
    dw.qstart = torch.tensor([0, 3, 3, 8], dtype=torch.int32, device="cuda")
    dw.lens = torch.tensor([2, 10, 8], dtype=torch.int32, device="cuda")
    assert run_prefill_step(pk, dw) & pk.DEVERR_BAD_CONTEXT
    del bad


@pytest.mark.parametrize("name", W.PREFILL_NAMES)
def test_named_prefill_workload(pk, name):
    w = W.make(name)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    kc, vc = oracle_caches(w, inplace=True)
    rng = np.random.default_rng(7)
    t_total = int(w.query_start[-1])
    rows = sorted({(int(t), int(h)) for t, h in zip(rng.integers(0, t_total, 48),
                                                    rng.integers(0, w.num_heads, 48))}
                  | {(0, 0), (t_total - 1, w.num_heads - 1)})
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc, rows), w, pairs=rows)
    from oracle.dtypes import widen
    assert np.isfinite(widen(dev_to_bits(dw.out), w.dtype)).all()


def test_prefill_on_a_cached_prefix(pk):
    """Request B shares request A's first 64 tokens.  Its admission reuses A's
    four full blocks; B writes and prefills only its own 50 tokens, attending
    over A's cached K/V through its block table."""
    from oracle import attention as OA
    from oracle import cache_ops as OC
    bs, h, hkv, d, dtype = 16, 4, 2, 64, "fp16"
    rng = np.random.default_rng(3)
    n_blocks = 32
    alloc = pk.BlockAllocator(n_blocks, bs, free_order=rng.permutation(n_blocks))
    tok_a = list(rng.integers(0, 1000, 100))
    tok_b = tok_a[:64] + list(rng.integers(1000, 2000, 50))
    kv_a = W._normal_bits(rng, (2, 100, hkv, d), dtype)
    kv_b = W._normal_bits(rng, (2, 114, hkv, d), dtype)
    kv_b[:, :64] = kv_a[:, :64]                      # same prefix, same K/V
    q_b = W._normal_bits(rng, (50, h, d), dtype)

    assert alloc.add_seq_cached(0, tok_a) == 0
    assert alloc.add_seq_cached(1, tok_b) == 64       # A's first four blocks
    tables = np.array(alloc.block_table([0, 1], 8), dtype=np.int32)
    assert (tables[1, :4] == tables[0, :4]).all() and tables[1, 4] != tables[0, 4]

    def slots(row, positions):
        return np.array([row[p // bs] * bs + p % bs for p in positions], dtype=np.int64)
    slots_a = slots(tables[0], range(100))
    slots_b = slots(tables[1], range(64, 114))        # only B's own tokens

    nan = W.NAN_BITS[dtype]
    kc = np.full((n_blocks, hkv, bs, d), nan, np.uint16)
    vc = np.full_like(kc, nan)
    kc, vc, _ = OC.reshape_and_cache(kv_a[0], kv_a[1], kc, vc, slots_a, bs)
    kc, vc, _ = OC.reshape_and_cache(kv_b[0, 64:], kv_b[1, 64:], kc, vc, slots_b, bs)
    lens = np.array([114], dtype=np.int32)
    qs = np.array([0, 50], dtype=np.int32)
    ref = OA.paged_attention_prefill(q_b, kc, vc, tables[1:2], lens, qs, 1 / 8.0, hkv, bs, dtype)

    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.float16)
    dk = dev(np.full((n_blocks, hkv, bs, d), nan, np.uint16))
    dv = dev(np.full((n_blocks, hkv, bs, d), nan, np.uint16))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.reshape_and_cache(dev(kv_a[0]), dev(kv_a[1]), dk, dv, torch.from_numpy(slots_a).cuda(),
                         dev_err=err)
    pk.reshape_and_cache(dev(kv_b[0, 64:]), dev(kv_b[1, 64:]), dk, dv,
                         torch.from_numpy(slots_b).cuda(), dev_err=err)
    out = torch.empty(50, h, d, dtype=torch.float16, device="cuda")
    pk.paged_attn_prefill(out, dev(q_b), dk, dv, torch.from_numpy(tables[1:2]).cuda(),
                          torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), 1 / 8.0,
                          hkv, bs, 114, 50, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    from support import ATOL, RTOL
    from oracle.dtypes import widen
    g = widen(got, dtype)
    assert (np.abs(g - ref) <= ATOL + RTOL * np.abs(ref)).all()
