"""Decode with the CTAs taken in a caller-given sequence order
(pkv_paged_attn_decode_ordered, pkv_paged_attn_decode_fp8_ordered) or from a
host-planned work list (pkv_paged_attn_decode_planned, _fp8_planned): each
sequence's result is computed by the same CTAs with the same arithmetic, so
the output must equal the index-order decode bit for bit, and the oracle
within the usual tolerance.  A bad order entry or work item is reported,
not faulted."""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import (DeviceWorkload, assert_close, dev_to_bits, oracle_caches, oracle_decode,
                     run_step)
from test_gpu_fp8 import Fp8Device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


# G = 1 (CUDA cores) and G = 4 (tensor cores); one pass and split-K
CASES = [([5, 900, 17, 2100, 300, 1, 64, 1500], 8, 8, 16, "fp16", 4096),
         ([5, 900, 17, 2100, 300, 1, 64, 1500], 8, 8, 16, "fp16", 256),
         ([33, 700, 129, 1800, 0, 400], 16, 4, 32, "bf16", 4096),
         ([33, 700, 129, 1800, 0, 400], 16, 4, 32, "bf16", 128)]


@pytest.mark.parametrize("lens,h,hkv,bs,dtype,part", CASES)
def test_ordered_decode_equals_index_order(pk, lens, h, hkv, bs, dtype, part):
    w = W.build_decode_workload(lens, h, hkv, 128, bs, dtype, seed=sum(lens) % 97)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, partition_size=part) == 0
    plain = dev_to_bits(dw.out)
    order = pk.decode_order(w.context_lens).cuda()
    dw.out.zero_()
    pk.paged_attn_decode(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, w.scale,
                         w.num_kv_heads, w.block_size, w.max_context_len, partition_size=part,
                         dev_err=dw.err, seq_order=order)
    torch.cuda.synchronize()
    assert int(dw.err.item()) == 0
    assert np.array_equal(dev_to_bits(dw.out), plain)
    kc, vc = oracle_caches(w)
    assert_close(plain, oracle_decode(w, kc, vc), w)


@pytest.mark.parametrize("h,hkv", [(8, 8), (16, 4)])
def test_ordered_fp8_decode_equals_index_order(pk, h, hkv):
    w = W.build_decode_workload([5, 900, 17, 2100, 300, 1], h, hkv, 128, 16, "fp16", seed=5)
    dev = Fp8Device(pk, w)
    assert dev.step(pk) == 0
    plain = dev_to_bits(dev.out)
    order = pk.decode_order(w.context_lens).cuda()
    dev.out.zero_()
    pk.paged_attn_decode_fp8(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens, w.scale,
                             dev.ks, dev.vs, w.num_kv_heads, w.block_size, w.max_context_len,
                             dev_err=dev.err, seq_order=order)
    torch.cuda.synchronize()
    assert int(dev.err.item()) == 0
    assert np.array_equal(dev_to_bits(dev.out), plain)


def test_bad_order_entry_is_reported(pk):
    w = W.build_decode_workload([40, 300, 17], 4, 4, 128, 16, "fp16", seed=6)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw) == 0
    good = dev_to_bits(dw.out)
    order = torch.tensor([1, 7, 2], dtype=torch.int32, device="cuda")   # 7 is not a sequence
    pk.paged_attn_decode(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, w.scale,
                         w.num_kv_heads, w.block_size, w.max_context_len, dev_err=dw.err,
                         seq_order=order)
    torch.cuda.synchronize()
    assert int(dw.err.item()) & pk.DEVERR_BAD_ORDER
    out = dev_to_bits(dw.out)
    assert np.array_equal(out[1], good[1]) and np.array_equal(out[2], good[2])


# 16-bit: G = 1 and 4 at head_dim 128, G = 8 at 64; one pass and split-K
PLANNED = CASES + [([5, 900, 17, 2100, 300, 1, 64, 1500], 16, 2, 16, "bf16", 512, 64),
                   ([3000, 1, 2047, 2048, 2049, 4096], 8, 2, 32, "fp16", 2048, 128)]


@pytest.mark.parametrize("case", PLANNED)
def test_planned_decode_equals_index_order(pk, case):
    lens, h, hkv, bs, dtype, part = case[:6]
    d = case[6] if len(case) > 6 else 128
    w = W.build_decode_workload(lens, h, hkv, d, bs, dtype, seed=sum(lens) % 89)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, partition_size=part) == 0
    plain = dev_to_bits(dw.out)
    work = pk.decode_plan(w.context_lens, bs, part).cuda()
    dw.out.zero_()
    pk.paged_attn_decode(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, w.scale,
                         w.num_kv_heads, w.block_size, w.max_context_len, partition_size=part,
                         dev_err=dw.err, work=work)
    torch.cuda.synchronize()
    assert int(dw.err.item()) == 0
    assert np.array_equal(dev_to_bits(dw.out), plain)
    kc, vc = oracle_caches(w)
    assert_close(plain, oracle_decode(w, kc, vc), w)


@pytest.mark.parametrize("h,hkv,d,part", [(8, 8, 128, 0), (32, 8, 128, 0), (32, 8, 128, 512),
                                          (16, 4, 64, 256)])
def test_planned_fp8_decode_equals_index_order(pk, h, hkv, d, part):
    lens = [5, 900, 17, 2100, 300, 1, 4000, 2048]
    w = W.build_decode_workload(lens, h, hkv, d, 16, "bf16", seed=8)
    dev = Fp8Device(pk, w)
    part = part or pk.partition_size_fp8(len(lens), hkv, 16, w.max_context_len)
    assert dev.step(pk, decode=False) == 0
    pk.paged_attn_decode_fp8(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens, w.scale,
                             dev.ks, dev.vs, w.num_kv_heads, w.block_size, w.max_context_len,
                             partition_size=part, dev_err=dev.err)
    torch.cuda.synchronize()
    plain = dev_to_bits(dev.out)
    work = pk.decode_plan(w.context_lens, 16, part).cuda()
    dev.out.zero_()
    pk.paged_attn_decode_fp8(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens, w.scale,
                             dev.ks, dev.vs, w.num_kv_heads, w.block_size, w.max_context_len,
                             partition_size=part, dev_err=dev.err, work=work)
    torch.cuda.synchronize()
    assert int(dev.err.item()) == 0
    assert np.array_equal(dev_to_bits(dev.out), plain)


def test_plan_that_disagrees_with_the_lengths_is_reported(pk):
    lens = [40, 1300, 17, 600]
    w = W.build_decode_workload(lens, 8, 2, 128, 16, "fp16", seed=9)
    dw = DeviceWorkload(w)
    part = 512
    assert run_step(pk, dw, partition_size=part) == 0
    good = dev_to_bits(dw.out)

    def planned(work):
        dw.err.zero_()
        pk.paged_attn_decode(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, w.scale,
                             w.num_kv_heads, w.block_size, w.max_context_len,
                             partition_size=part, dev_err=dw.err, work=work.cuda())
        torch.cuda.synchronize()
        return int(dw.err.item())

    # planned for longer contexts: the extra items find nothing and report it;
    # every partition that exists is covered, so the results stand
    longer = pk.decode_plan([40, 1300, 17, 1100], 16, part)
    assert planned(longer) & pk.DEVERR_BAD_ORDER
    assert np.array_equal(dev_to_bits(dw.out), good)
    # planned for a shorter sequence 1: its second and third partitions are
    # missing; reported (its output is not to be trusted), the others exact
    shorter = pk.decode_plan([40, 500, 17, 600], 16, part)
    assert planned(shorter) & pk.DEVERR_BAD_ORDER
    out = dev_to_bits(dw.out)
    for i in (0, 2, 3):
        assert np.array_equal(out[i], good[i])
    # an item naming no sequence
    bad = pk.decode_plan(lens, 16, part)
    bad[-1, 0] = 9
    assert planned(bad) & pk.DEVERR_BAD_ORDER
