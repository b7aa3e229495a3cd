"""Parity of cascade decode (shared-prefix pass + per-sequence suffix +
merge, through the C ABI) with the float64 oracle's plain decode: the two
must agree, since cascade only changes which kernel reads which blocks.

|gpu - ref| <= 2e-3 + 1e-2*|ref| elementwise, as for plain decode.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import (DeviceWorkload, assert_close, block_allocator, dev_to_bits, oracle_caches,
                     oracle_decode, run_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


def run_cascade(pk, dw, group_start, shared_blocks, partition_size=0):
    w = dw.w
    gs = torch.from_numpy(np.asarray(group_start, np.int32)).cuda()
    sb = torch.from_numpy(np.asarray(shared_blocks, np.int32)).cuda()
    max_group = int(np.diff(group_start).max())
    pk.paged_attn_decode_cascade(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens, gs, sb,
                                 w.scale, w.num_kv_heads, w.block_size, w.max_context_len,
                                 max_group, int(np.max(shared_blocks)) if len(shared_blocks) else 0,
                                 partition_size=partition_size, dev_err=dw.err)
    torch.cuda.synchronize()
    return int(dw.err.item())


# (prompts, samples, prompt_len, heads, kv heads, block, dtype): partial and
# block-aligned prompts, every group size the grouped kernels serve
CASES = [(3, 4, 37, 8, 2, 16, "bf16"), (2, 8, 64, 8, 1, 16, "fp16"), (4, 2, 100, 4, 4, 32, "fp16"),
         (2, 3, 96, 16, 2, 32, "bf16"), (5, 1, 50, 2, 1, 16, "fp16"), (1, 16, 300, 8, 8, 16, "bf16")]


@pytest.mark.parametrize("prompts,samples,plen,h,hkv,bs,dtype",
                         CASES + [(1, 40, 70, 8, 2, 16, "bf16")])  # 40 x G 4: two 128-row tiles
def test_cascade_matches_oracle(pk, prompts, samples, plen, h, hkv, bs, dtype):
    w = W.build_prefix_share_workload(prompts, samples, plen, 5, 40, h, hkv, 128, bs, dtype,
                                      seed=plen + samples, allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    group_start, shared = W.cascade_groups(w)
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    for part in (0, bs):   # suffix in one partition, and in many
        dw.out.zero_()
        assert run_cascade(pk, dw, group_start, shared, partition_size=part) == 0
        assert_close(dev_to_bits(dw.out), ref, w)


# head_dim 64: the prefix pass is the mma.sync kernel in prefix mode; G = 1
# reads each member's own blocks on the CUDA cores, G >= 2 on the tensor cores
CASES_D64 = [(3, 4, 37, 8, 2, 16, "bf16"), (2, 8, 64, 4, 4, 32, "fp16"),
             (4, 2, 100, 16, 2, 16, "fp16"), (1, 16, 300, 8, 8, 32, "bf16"),
             (2, 16, 64, 16, 2, 16, "fp16")]   # 16 members x G 8: two 64-row tiles


@pytest.mark.parametrize("prompts,samples,plen,h,hkv,bs,dtype", CASES_D64)
def test_cascade_head_dim_64_matches_oracle(pk, prompts, samples, plen, h, hkv, bs, dtype):
    w = W.build_prefix_share_workload(prompts, samples, plen, 5, 40, h, hkv, 64, bs, dtype,
                                      seed=plen + samples + 64, allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    group_start, shared = W.cascade_groups(w)
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    for part in (0, bs):
        dw.out.zero_()
        assert run_cascade(pk, dw, group_start, shared, partition_size=part) == 0
        assert_close(dev_to_bits(dw.out), ref, w)


# E4M3 caches: (prompts, samples, prompt_len, heads, kv heads, head_dim, block, dtype)
CASES_FP8 = [(3, 4, 37, 8, 2, 128, 16, "bf16"), (2, 8, 64, 8, 1, 128, 32, "fp16"),
             (4, 2, 100, 4, 4, 128, 16, "fp16"), (3, 4, 37, 8, 2, 64, 16, "bf16"),
             (2, 8, 64, 4, 4, 64, 32, "fp16"), (1, 16, 300, 8, 8, 64, 16, "bf16"),
             (1, 40, 70, 8, 2, 128, 16, "bf16"),   # two 128-row tiles
             (2, 16, 64, 16, 2, 64, 16, "fp16")]   # two 64-row tiles


@pytest.mark.parametrize("prompts,samples,plen,h,hkv,d,bs,dtype", CASES_FP8)
def test_cascade_fp8_matches_oracle(pk, prompts, samples, plen, h, hkv, d, bs, dtype):
    """Cascade decode over E4M3 caches equals the oracle's decode over its own
    quantised caches (the plain E4M3 decode's reference)."""
    from test_gpu_fp8 import Fp8Device, oracle_codes, oracle_decode8
    w = W.build_prefix_share_workload(prompts, samples, plen, 5, 40, h, hkv, d, bs, dtype,
                                      seed=plen + samples + d, allocator=block_allocator)
    dev = Fp8Device(pk, w)
    assert dev.step(pk, decode=False) == 0
    kq, vq = oracle_codes(w)
    assert np.array_equal(dev.k8.cpu().numpy(), kq)
    ref = oracle_decode8(w, kq, vq)
    gs, shared = W.cascade_groups(w)
    gs_t = torch.from_numpy(np.asarray(gs, np.int32)).cuda()
    sb_t = torch.from_numpy(np.asarray(shared, np.int32)).cuda()
    for part in (0, bs):
        dev.out.zero_()
        pk.paged_attn_decode_cascade(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens, gs_t,
                                     sb_t, w.scale, w.num_kv_heads, w.block_size,
                                     w.max_context_len, int(np.diff(gs).max()),
                                     int(np.max(shared)), partition_size=part, dev_err=dev.err,
                                     k_scales=dev.ks, v_scales=dev.vs)
        torch.cuda.synchronize()
        assert int(dev.err.item()) == 0
        assert_close(dev_to_bits(dev.out), ref, w)


def test_cascade_fp8_reports_a_bad_scale(pk):
    from test_gpu_fp8 import Fp8Device
    w = W.build_prefix_share_workload(2, 4, 64, 5, 40, 4, 2, 128, 16, "fp16", seed=5,
                                      allocator=block_allocator)
    dev = Fp8Device(pk, w)
    assert dev.step(pk, decode=False) == 0
    gs, shared = W.cascade_groups(w)
    bad_v = torch.tensor([0.01, float("inf")], dtype=torch.float32, device="cuda")
    pk.paged_attn_decode_cascade(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens,
                                 torch.from_numpy(gs).cuda(), torch.from_numpy(shared).cuda(),
                                 w.scale, w.num_kv_heads, w.block_size, w.max_context_len,
                                 int(np.diff(gs).max()), int(np.max(shared)), dev_err=dev.err,
                                 k_scales=dev.ks, v_scales=bad_v)
    torch.cuda.synchronize()
    assert int(dev.err.item()) & pk.DEVERR_BAD_SCALE


def test_cascade_with_fewer_shared_blocks_and_singletons(pk):
    """Declaring less sharing than there is, or none, changes nothing."""
    w = W.build_prefix_share_workload(3, 4, 70, 5, 40, 8, 2, 128, 16, "fp16", seed=9,
                                      allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    gs, full = W.cascade_groups(w)
    for shared in (full - 2, np.array([0, 1, int(full[2])], np.int32)):
        assert run_cascade(pk, dw, gs, shared) == 0
        assert_close(dev_to_bits(dw.out), ref, w)
    singles = np.arange(w.num_seqs + 1, dtype=np.int32)   # every sequence its own group
    assert run_cascade(pk, dw, singles, np.zeros(w.num_seqs, np.int32)) == 0
    assert_close(dev_to_bits(dw.out), ref, w)
    assert run_cascade(pk, dw, singles, np.full(w.num_seqs, 3, np.int32)) == 0
    assert_close(dev_to_bits(dw.out), ref, w)


def test_cascade_equals_plain_decode_on_independent_sequences(pk):
    w = W.build_decode_workload([1, 5, 16, 17, 33, 100, 257, 600], 8, 2, 128, 16, "bf16", 12)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw) == 0
    plain = dw.out.clone()
    singles = np.arange(w.num_seqs + 1, dtype=np.int32)
    assert run_cascade(pk, dw, singles, np.zeros(w.num_seqs, np.int32)) == 0
    kc, vc = oracle_caches(w)
    assert_close(dev_to_bits(dw.out), oracle_decode(w, kc, vc), w)
    assert torch.isfinite(plain.float()).all()


def test_cascade_flags_a_member_shorter_than_its_prefix(pk):
    w = W.build_prefix_share_workload(2, 4, 64, 5, 40, 8, 2, 128, 16, "fp16", seed=4,
                                      allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    gs, _ = W.cascade_groups(w)
    lens = w.context_lens.copy()
    lens[1] = 20                                         # 20 tokens < 64 shared
    dw.lens = torch.from_numpy(lens).cuda()
    assert run_cascade(pk, dw, gs, np.array([4, 4], np.int32)) & pk.DEVERR_BAD_CONTEXT


def test_cascade_prefix_share_full_size(pk):
    """The parallel-sampling workload at full size (64 prompts x 8 samples),
    on sampled rows including the longest and shortest sequence."""
    w = W.make("prefix_share", allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    gs, shared = W.cascade_groups(w)
    assert run_cascade(pk, dw, gs, shared) == 0
    rng = np.random.default_rng(2)
    seqs = sorted({int(np.argmax(w.context_lens)), int(np.argmin(w.context_lens))}
                  | {int(s) for s in rng.integers(0, w.num_seqs, 6)})
    pairs = [(s, h) for s in seqs for h in (0, 7, 63)]
    kc, vc = oracle_caches(w, inplace=True)
    assert_close(dev_to_bits(dw.out), oracle_decode(w, kc, vc, pairs=pairs), w, pairs=pairs)
    assert torch.isfinite(dw.out.float()).all()


def test_cascade_clamps_device_sharing_to_the_host_bound(pk):
    """shared_blocks in device memory above the host's max_shared_blocks:
    with max_shared_blocks = 0 the prefix pass does not run, so the decode
    kernels must read every block themselves (never the stale workspace
    slot 0) and report PKV_DEVERR_BAD_CONTEXT; the result is still the
    plain decode."""
    w = W.build_prefix_share_workload(3, 4, 70, 5, 40, 8, 2, 128, 16, "fp16", seed=19,
                                      allocator=block_allocator)
    dw = DeviceWorkload(w)
    assert run_step(pk, dw, decode=False) == 0
    kc, vc = oracle_caches(w)
    ref = oracle_decode(w, kc, vc)
    gs, full = W.cascade_groups(w)
    gs_t = torch.from_numpy(gs).cuda()
    sb_t = torch.from_numpy(full).cuda()
    max_group = int(np.diff(gs).max())
    # a poisoned workspace: a merge that read slot 0 would turn the output NaN
    ws = torch.empty(pk.cascade_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads,
                                                w.head_dim, w.block_size, w.max_context_len, 0),
                     dtype=torch.uint8, device="cuda")
    ws.view(torch.float32).fill_(float("nan"))
    for bound in (0, 2):
        dw.err.zero_()
        dw.out.zero_()
        pk.paged_attn_decode_cascade(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens,
                                     gs_t, sb_t, w.scale, w.num_kv_heads, w.block_size,
                                     w.max_context_len, max_group, bound, workspace=ws,
                                     dev_err=dw.err)
        torch.cuda.synchronize()
        assert int(dw.err.item()) & pk.DEVERR_BAD_CONTEXT
        assert_close(dev_to_bits(dw.out), ref, w)
