"""Planned prefill (pkv_prefill_plan + pkv_paged_attn_prefill_planned /
_fp8_planned) on the GPU: units cut into 2-4 key pieces whose partials a merge
kernel combines.  Against the float64 oracle with the prefill tolerance
|gpu - ref| <= 2e-3 + 1e-2*|ref|, and against the unplanned prefill (which
differs only by the merge's rounding).  Bad plans are reported, not faulted."""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import (DeviceWorkload, assert_close, dev_to_bits, oracle_caches, oracle_prefill,
                     run_prefill_step)
from test_gpu_fp8 import Fp8Device, oracle_codes, oracle_prefill8, run_prefill8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


def planned(pk, dw, plan, fp8=None):
    w = dw.w
    dw.out.zero_()
    dw.err.zero_()
    args = (dw.out, dw.q, fp8.k8 if fp8 else dw.k_cache, fp8.v8 if fp8 else dw.v_cache, dw.tables,
            dw.lens, dw.qstart if not fp8 else torch.from_numpy(w.query_start).cuda(), w.scale)
    if fp8:
        pk.paged_attn_prefill_fp8(*args, fp8.ks, fp8.vs, w.num_kv_heads, w.block_size,
                                  w.max_context_len, int(np.diff(w.query_start).max()),
                                  dev_err=dw.err, plan=plan.to("cuda"))
    else:
        pk.paged_attn_prefill(*args, w.num_kv_heads, w.block_size, w.max_context_len,
                              int(np.diff(w.query_start).max()), dev_err=dw.err,
                              plan=plan.to("cuda"))
    torch.cuda.synchronize()
    return int(dw.err.item())


def pieces_of(plan):
    return sorted(set(int(x) for x in plan.merges[:, 2].tolist()))


# (histories, new tokens, heads, kv heads, block size, dtype, SMs the plan
# spreads over: more SMs make smaller shares, so more pieces)
CASES = [([3000, 5, 700, 0], [200, 17, 64, 70], 8, 8, 16, "fp16", 148),
         ([3000, 5, 700, 0], [200, 17, 64, 70], 8, 2, 32, "bf16", 148),
         ([1500, 900, 40], [64, 33, 100], 16, 2, 16, "bf16", 1000),
         ([2100, 0, 333], [96, 120, 1], 8, 1, 32, "fp16", 1000)]


@pytest.mark.parametrize("case", CASES)
def test_planned_prefill_matches_oracle(pk, case):
    hist, new, h, hkv, bs, dtype, sms = case
    w = W.build_prefill_workload(hist, new, h, hkv, 128, bs, dtype, seed=sum(hist) % 101)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    plain = dw.out.float().clone()
    plan = pk.prefill_plan(w.query_start, w.context_lens, h, hkv, 128, sms)
    assert len(plan.merges) > 0, "the case must cut at least one unit"
    assert planned(pk, dw, plan) == 0
    kc, vc = oracle_caches(w)
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc), w)
    # the same attention, merged in another order: within the tolerance of each other
    got = dw.out.float()
    assert ((got - plain).abs() <= 2e-3 + 1e-2 * plain.abs()).all()


def test_planned_prefill_uses_up_to_four_pieces(pk):
    w = W.build_prefill_workload([4000, 64], [130, 10], 8, 2, 128, 16, "bf16", seed=4)
    plan = pk.prefill_plan(w.query_start, w.context_lens, 8, 2, 128, 1000)
    assert max(pieces_of(plan)) == 4
    dw = DeviceWorkload(w)
    pk.reshape_and_cache(dw.key, dw.value, dw.k_cache, dw.v_cache, dw.slots, dev_err=dw.err)
    assert planned(pk, dw, plan) == 0
    kc, vc = oracle_caches(w)
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc), w)


@pytest.mark.parametrize("name", W.PREFILL_NAMES)
def test_planned_named_prefill_workload(pk, name):
    w = W.make(name)
    if w.head_dim != 128:
        pytest.skip("planned prefill is head_dim 128")
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    plain = dw.out.float().clone()
    plan = pk.prefill_plan(w.query_start, w.context_lens, w.num_heads, w.num_kv_heads)
    assert planned(pk, dw, plan) == 0
    kc, vc = oracle_caches(w, inplace=True)
    rng = np.random.default_rng(9)
    t_total = int(w.query_start[-1])
    rows = sorted({(int(t), int(hh)) for t, hh in zip(rng.integers(0, t_total, 48),
                                                      rng.integers(0, w.num_heads, 48))}
                  | {(0, 0), (t_total - 1, w.num_heads - 1)})
    assert_close(dev_to_bits(dw.out), oracle_prefill(w, kc, vc, rows), w, pairs=rows)
    got = dw.out.float()
    assert ((got - plain).abs() <= 2e-3 + 1e-2 * plain.abs()).all()


@pytest.mark.parametrize("hkv,dtype", [(8, "fp16"), (2, "bf16")])
def test_planned_fp8_prefill(pk, hkv, dtype):
    w = W.build_prefill_workload([3000, 5, 700], [200, 17, 64], 8, hkv, 128, 16, dtype, seed=12)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    plain = dev.out.float().clone()
    plan = pk.prefill_plan(w.query_start, w.context_lens, 8, hkv, 128, 148)
    assert len(plan.merges) > 0
    assert planned(pk, dev, plan, fp8=dev) == 0
    kq, vq = oracle_codes(w)
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq), w)
    got = dev.out.float()
    assert ((got - plain).abs() <= 2e-3 + 1e-2 * plain.abs()).all()


def test_bad_plans_are_reported(pk):
    w = W.build_prefill_workload([3000, 5], [200, 17], 8, 2, 128, 16, "fp16", seed=13)
    dw = DeviceWorkload(w)
    assert run_prefill_step(pk, dw) == 0
    plan = pk.prefill_plan(w.query_start, w.context_lens, 8, 2, 128, 148)
    assert len(plan.merges) > 0
    # an item naming no sequence
    bad = pk.PrefillPlan(plan.work.clone(), plan.merges.clone(), plan.workspace_bytes)
    bad.work[0, 0] = 7
    assert planned(pk, dw, bad) & pk.DEVERR_BAD_ORDER
    # a history piece that reaches past the history
    bad = pk.PrefillPlan(plan.work.clone(), plan.merges.clone(), plan.workspace_bytes)
    i = int(np.nonzero((bad.work[:, 6] > 1).numpy() & (bad.work[:, 3] >= 0).numpy())[0][0])
    bad.work[i, 3] = 64 * 64
    assert planned(pk, dw, bad) & pk.DEVERR_BAD_ORDER
    # a plan made for other lengths: sequence 0's history shorter on the device
    lens = w.context_lens.copy()
    lens[0] = 300 + 200
    dw.lens = torch.from_numpy(lens).cuda()
    assert planned(pk, dw, plan) & pk.DEVERR_BAD_ORDER
