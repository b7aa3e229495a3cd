"""Parity of the E4M3 cache path (through the C ABI) with the float64 oracle.

* reshape_and_cache_fp8 and copy_blocks on 1-byte caches: bit-exact codes.
* paged_attn_decode_fp8: |gpu - ref| <= 2e-3 + 1e-2*|ref| elementwise, where
  ref is float64 attention over the oracle's own dequantised codes.

The device caches are filled by the device's quantising write from the
workload's 16-bit pool; the oracle quantises the same 16-bit values itself.
"""

import numpy as np
import pytest
import torch

from oracle import cache_ops as OC
from oracle import fp8 as OF
from paged_kv_cache_394_b200 import workloads as W
from support import assert_close, bits_to_dev, block_allocator, dev_to_bits

pytestmark = pytest.mark.gpu

# Per-kv-head scales.  N(0,1) values reach about +-5.5: K scales around
# 0.0125 keep x / scale inside E4M3's range, V scales around 0.01 make the
# largest values saturate at 448.


def head_scales(base, hkv):
    """A different scale for every kv head: base * (0.8 .. 1.2)."""
    return (base * (0.8 + 0.4 * np.arange(hkv) / max(1, hkv - 1))).astype(np.float32)


def k_scales_for(w):
    return head_scales(0.0125, w.num_kv_heads)


def v_scales_for(w):
    return head_scales(0.01, w.num_kv_heads)


@pytest.fixture(scope="module")
def pk():
    from paged_kv_cache_394_b200 import pagedkv
    return pagedkv


def token_view(cache16):
    """[nb, hkv, bs, d] -> [nb*bs, hkv, d] (tokens in slot order)."""
    nb, hkv, bs, d = cache16.shape
    return cache16.permute(0, 2, 1, 3).reshape(nb * bs, hkv, d).contiguous()


class Fp8Device:
    """The workload on the device with E4M3 caches written by the device."""

    def __init__(self, pk, w, k_scales=None, v_scales=None):
        k_scales = k_scales_for(w) if k_scales is None else k_scales
        v_scales = v_scales_for(w) if v_scales is None else v_scales
        self.w = w
        self.ks = torch.from_numpy(np.asarray(k_scales, np.float32)).cuda()
        self.vs = torch.from_numpy(np.asarray(v_scales, np.float32)).cuda()
        k16, v16 = bits_to_dev(w.k_cache, w), bits_to_dev(w.v_cache, w)
        self.k8 = torch.empty(k16.shape, dtype=torch.uint8, device="cuda")
        self.v8 = torch.empty_like(self.k8)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        all_slots = torch.arange(w.num_blocks * w.block_size, dtype=torch.int64, device="cuda")
        pk.reshape_and_cache_fp8(token_view(k16), token_view(v16), self.k8, self.v8, all_slots,
                                 self.ks, self.vs, dev_err=self.err)
        del k16, v16
        self.q = bits_to_dev(w.q, w)
        self.key, self.value = bits_to_dev(w.key, w), bits_to_dev(w.value, w)
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.pairs = torch.from_numpy(np.ascontiguousarray(w.cow_pairs)).cuda()
        self.tables = torch.from_numpy(w.block_tables).cuda()
        self.lens = torch.from_numpy(w.context_lens).cuda()
        self.out = torch.empty_like(self.q)

    def step(self, pk, partition_size=None, decode=True):
        w = self.w
        part = w.partition_size if partition_size is None else partition_size
        if len(w.cow_pairs):
            pk.copy_blocks(self.k8, self.v8, self.pairs, dev_err=self.err)
        if len(w.slot_mapping):
            pk.reshape_and_cache_fp8(self.key, self.value, self.k8, self.v8, self.slots, self.ks,
                                     self.vs, dev_err=self.err)
        if decode:
            pk.paged_attn_decode_fp8(self.out, self.q, self.k8, self.v8, self.tables, self.lens,
                                     w.scale, self.ks, self.vs, w.num_kv_heads, w.block_size,
                                     w.max_context_len, partition_size=part, dev_err=self.err)
        torch.cuda.synchronize()
        return int(self.err.item())


def run_prefill8(pk, dev):
    """The quantising write of the new tokens, then E4M3 chunked prefill."""
    w = dev.w
    pk.reshape_and_cache_fp8(dev.key, dev.value, dev.k8, dev.v8, dev.slots, dev.ks, dev.vs,
                             dev_err=dev.err)
    qstart = torch.from_numpy(w.query_start).cuda()
    pk.paged_attn_prefill_fp8(dev.out, dev.q, dev.k8, dev.v8, dev.tables, dev.lens, qstart,
                              w.scale, dev.ks, dev.vs, w.num_kv_heads, w.block_size,
                              w.max_context_len, int(np.diff(w.query_start).max()),
                              dev_err=dev.err)
    torch.cuda.synchronize()
    return int(dev.err.item())


def oracle_prefill8(w, kq, vq, rows=None):
    return OF.paged_attention_prefill_fp8(w.q, kq, vq, w.block_tables, w.context_lens,
                                          w.query_start, w.scale, k_scales_for(w),
                                          v_scales_for(w), w.num_kv_heads, w.block_size,
                                          w.dtype, rows=rows)


def oracle_codes(w, k_scales=None, v_scales=None, blocks=None):
    """The oracle's E4M3 caches after the step: the pool quantised, the CoW
    copies, then the new tokens quantised into their slots.  With ``blocks``
    only those physical blocks of the pool are quantised (others stay 0)."""
    k_scale = k_scales_for(w) if k_scales is None else k_scales
    v_scale = v_scales_for(w) if v_scales is None else v_scales
    if blocks is None:
        kq = OF.quantize_cache(w.k_cache, w.dtype, k_scale)
        vq = OF.quantize_cache(w.v_cache, w.dtype, v_scale)
    else:
        kq = np.zeros(w.k_cache.shape, np.uint8)
        vq = np.zeros(w.v_cache.shape, np.uint8)
        kq[blocks] = OF.quantize_cache(w.k_cache[blocks], w.dtype, k_scale)
        vq[blocks] = OF.quantize_cache(w.v_cache[blocks], w.dtype, v_scale)
    kq, vq, bad = OC.copy_blocks(kq, vq, w.cow_pairs, inplace=True)
    assert not bad
    return OF.quantize_into_cache(w.key, w.value, kq, vq, w.slot_mapping, w.block_size, w.dtype,
                                  k_scale, v_scale)


def oracle_decode8(w, kq, vq, k_scales=None, v_scales=None, pairs=None):
    k_scale = k_scales_for(w) if k_scales is None else k_scales
    v_scale = v_scales_for(w) if v_scales is None else v_scales
    return OF.paged_attention_decode_fp8(w.q, kq, vq, w.block_tables, w.context_lens, w.scale,
                                         k_scale, v_scale, w.num_kv_heads, w.block_size,
                                         w.dtype, pairs=pairs)


RAGGED = [1, 5, 16, 17, 33, 100, 257, 600]
SHAPES = [(64, 16, 1, "fp16"), (64, 32, 2, "bf16"), (128, 16, 1, "bf16"), (128, 16, 4, "fp16"),
          (128, 32, 8, "bf16"), (128, 16, 8, "fp16"), (64, 16, 4, "bf16"), (128, 32, 2, "fp16")]


@pytest.mark.parametrize("d,bs,g,dtype", SHAPES)
def test_fp8_decode_small(pk, d, bs, g, dtype):
    w = W.build_decode_workload(RAGGED, 2 * g, 2, d, bs, dtype, 11 + d + bs + g)
    dev = Fp8Device(pk, w)
    kq, vq = oracle_codes(w)
    for part in (0, 2 * bs):   # one pass, and a split with many partitions and a ragged tail
        assert dev.step(pk, partition_size=part) == 0
        assert np.array_equal(dev.k8.cpu().numpy(), kq)
        assert np.array_equal(dev.v8.cpu().numpy(), vq)
        assert_close(dev_to_bits(dev.out), oracle_decode8(w, kq, vq), w)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_fp8_write_is_bit_exact_on_edge_values(pk, dtype):
    """Tiny (subnormal), huge (saturating), signed zeros, ties and NaN."""
    rng = np.random.default_rng(5)
    hkv, d, bs, nb = 2, 64, 16, 8
    t = nb * bs
    x = rng.standard_normal((t, hkv, d)).astype(np.float32)
    mags = np.array([1e-4, 1e-3, 0.02, 1.0, 50.0, 300.0], np.float32)
    x *= mags[rng.integers(0, len(mags), size=x.shape)]
    x[0, 0, :8] = [0.0, -0.0, 448.0, -448.0, 464.0, -1e4, 1.0625, 1.1875]
    x[0, 1, 0] = np.nan
    bits = W._to_bits(x, dtype)
    w16 = type("W", (), {"dtype": dtype})
    key = bits_to_dev(bits, w16)
    val = bits_to_dev(bits[::-1].copy(), w16)
    k8 = torch.zeros((nb, hkv, bs, d), dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    slots = np.random.default_rng(6).permutation(t).astype(np.int64)
    slots[7] = -1
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for ks, vs in ((np.ones(hkv, np.float32), np.ones(hkv, np.float32)),
                   (np.array([0.5, 0.75], np.float32), np.array([3.0, 0.3], np.float32))):
        pk.reshape_and_cache_fp8(key, val, k8, v8, torch.from_numpy(slots).cuda(),
                                 torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(),
                                 dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        zero = np.zeros((nb, hkv, bs, d), np.uint8)
        kq, vq = OF.quantize_into_cache(bits, bits[::-1].copy(), zero, zero, slots, bs, dtype,
                                        ks, vs)
        got_k = k8.cpu().numpy()
        # the skipped token's slot keeps what the previous round left there
        b7, o7 = divmod(int(np.setdiff1d(np.arange(t), slots)[0]), bs)
        kq[b7, :, o7], vq[b7, :, o7] = got_k[b7, :, o7], v8.cpu().numpy()[b7, :, o7]
        assert np.array_equal(got_k, kq)
        assert np.array_equal(v8.cpu().numpy(), vq)


def test_fp8_copy_blocks_bit_exact(pk):
    w = W.build_prefix_share_workload(3, 4, 37, 5, 40, 8, 2, 64, 16, "bf16", seed=3,
                                      allocator=block_allocator)
    assert len(w.cow_pairs) == 9
    dev = Fp8Device(pk, w)
    assert dev.step(pk) == 0
    kq, vq = oracle_codes(w)
    assert np.array_equal(dev.k8.cpu().numpy(), kq)
    assert np.array_equal(dev.v8.cpu().numpy(), vq)
    assert_close(dev_to_bits(dev.out), oracle_decode8(w, kq, vq), w)


def test_fp8_bad_slot_and_bad_block_are_reported(pk):
    w = W.build_decode_workload([5, 40], 2, 2, 64, 16, "fp16", 4)
    dev = Fp8Device(pk, w)
    slots = w.slot_mapping.copy()
    slots[0] = w.num_blocks * w.block_size
    dev.slots = torch.from_numpy(slots).cuda()
    assert dev.step(pk, decode=False) & pk.DEVERR_BAD_SLOT
    dev.err.zero_()
    tables = w.block_tables.copy()
    tables[1, 1] = w.num_blocks + 3
    dev.tables = torch.from_numpy(tables).cuda()
    dev.slots = torch.from_numpy(w.slot_mapping).cuda()
    assert dev.step(pk) & pk.DEVERR_BAD_BLOCK


def test_fp8_scales_fold_like_the_oracle(pk):
    """New scales with the old codes kept: K scales fold into the logits, V
    scales into the output, head by head (checked against the oracle)."""
    w = W.build_decode_workload([70, 300, 1], 8, 2, 128, 16, "bf16", 21)
    dev = Fp8Device(pk, w)
    assert dev.step(pk) == 0
    kq, vq = dev.k8.cpu().numpy(), dev.v8.cpu().numpy()
    ok, ov = oracle_codes(w)
    assert np.array_equal(kq, ok) and np.array_equal(vq, ov)
    ks2 = np.array([2.0, 0.5], np.float32) * k_scales_for(w)
    vs2 = np.array([0.25, 3.0], np.float32) * v_scales_for(w)
    dev.ks, dev.vs = torch.from_numpy(ks2).cuda(), torch.from_numpy(vs2).cuda()
    assert dev.step(pk) == 0   # the write re-quantises the new tokens with the new scales
    ok2, ov2 = OF.quantize_into_cache(w.key, w.value, ok, ov, w.slot_mapping, w.block_size,
                                      w.dtype, ks2, vs2)
    assert np.array_equal(dev.k8.cpu().numpy(), ok2)
    assert np.array_equal(dev.v8.cpu().numpy(), ov2)
    assert_close(dev_to_bits(dev.out), oracle_decode8(w, ok2, ov2, ks2, vs2), w)


def test_fp8_bad_scale_is_reported(pk):
    w = W.build_decode_workload([20, 9], 4, 2, 64, 16, "fp16", 8)
    dev = Fp8Device(pk, w)
    assert dev.step(pk) == 0
    before = dev.k8.clone()
    dev.ks = torch.tensor([0.01, float("nan")], device="cuda")
    err = dev.step(pk)
    assert err & pk.DEVERR_BAD_SCALE
    # the write skipped kv head 1 of the new tokens; head 0 was re-written as before
    assert torch.equal(dev.k8[:, 1], before[:, 1])


def sample_pairs(w, n, seed):
    rng = np.random.default_rng(seed)
    seqs = {int(np.argmax(w.context_lens)), int(np.argmin(w.context_lens))}
    seqs.update(int(s) for s in rng.integers(0, w.num_seqs, size=n))
    heads = sorted({0, w.num_heads - 1} | {int(x) for x in rng.integers(0, w.num_heads, 2)})
    return [(s, h) for s in sorted(seqs) for h in heads]


@pytest.mark.parametrize("name", ["llama7b", "gqa_chat"])
def test_fp8_named_workload_full_size(pk, name):
    """Full-size pools in the benchmark's launch configuration; codes and
    outputs compared on the blocks of sampled sequences."""
    w = W.make(name)
    dev = Fp8Device(pk, w)
    assert dev.step(pk) == 0
    pairs = sample_pairs(w, 4, seed=len(name))
    seqs = sorted({s for s, _ in pairs})
    blocks = np.unique(np.concatenate(
        [w.block_tables[s, :-(-int(w.context_lens[s]) // w.block_size)] for s in seqs]))
    kq, vq = oracle_codes(w, blocks=blocks)
    bt = torch.from_numpy(blocks).cuda()
    assert np.array_equal(dev.k8[bt].cpu().numpy(), kq[blocks])
    assert np.array_equal(dev.v8[bt].cpu().numpy(), vq[blocks])
    assert_close(dev_to_bits(dev.out), oracle_decode8(w, kq, vq, pairs=pairs), w, pairs=pairs)
    assert torch.isfinite(dev.out.float()).all()


PREFILL_HIST = [0, 5, 16, 40, 100, 0]
PREFILL_NEW = [1, 17, 16, 33, 64, 70]
PREFILL_SHAPES = [(16, 1, "fp16"), (32, 2, "bf16"), (16, 4, "bf16"), (32, 8, "fp16"),
                  (16, 8, "bf16"), (32, 1, "fp16"), (16, 2, "fp16"), (32, 4, "bf16")]


@pytest.mark.parametrize("bs,g,dtype", PREFILL_SHAPES)
def test_fp8_prefill_small(pk, bs, g, dtype):
    """Whole prompts and chunks on short and empty histories, every group size
    and block size, ragged query tiles (70 new tokens x G heads)."""
    w = W.build_prefill_workload(PREFILL_HIST, PREFILL_NEW, 2 * g, 2, 128, bs, dtype,
                                 seed=31 + bs + g)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    kq, vq = oracle_codes(w)
    assert np.array_equal(dev.k8.cpu().numpy(), kq)
    assert np.array_equal(dev.v8.cpu().numpy(), vq)
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq), w)


PREFILL_SHAPES_D64 = [(16, 1, "fp16"), (32, 2, "bf16"), (16, 4, "bf16"), (32, 8, "fp16"),
                      (16, 8, "bf16"), (32, 1, "bf16")]


@pytest.mark.parametrize("bs,g,dtype", PREFILL_SHAPES_D64)
def test_fp8_prefill_head_dim_64(pk, bs, g, dtype):
    """head_dim 64 runs the mma.sync kernel over codes widened to fp16 by its
    producer warp: the same cases as the tcgen05 kernel's."""
    w = W.build_prefill_workload(PREFILL_HIST, PREFILL_NEW, 2 * g, 2, 64, bs, dtype,
                                 seed=41 + bs + g)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    kq, vq = oracle_codes(w)
    assert np.array_equal(dev.k8.cpu().numpy(), kq)
    assert np.array_equal(dev.v8.cpu().numpy(), vq)
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq), w)


def test_fp8_prefill_head_dim_64_long_history_and_bad_block(pk):
    """A long history (many 16-key stages through the two widened stages) on
    sampled rows; then a table entry out of range is reported, not read."""
    w = W.build_prefill_workload([2000, 0, 333], [100, 150, 77], 8, 2, 64, 16, "bf16", seed=8)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    kq, vq = oracle_codes(w)
    rows = [(0, 0), (50, 3), (99, 7), (100, 1), (249, 6), (250, 2), (326, 5)]
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq, rows), w, pairs=rows)
    tables = w.block_tables.copy()
    tables[0, 3] = w.num_blocks + 5
    dev.tables = torch.from_numpy(tables).cuda()
    dev.err.zero_()
    assert run_prefill8(pk, dev) & pk.DEVERR_BAD_BLOCK


def test_fp8_prefill_long_history_sampled(pk):
    w = W.build_prefill_workload([3000, 0, 777], [200, 300, 129], 16, 4, 128, 16, "bf16", seed=6)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    kq, vq = oracle_codes(w)
    rng = np.random.default_rng(1)
    rows = sorted({(int(t), int(h)) for t, h in zip(rng.integers(0, 629, 40),
                                                    rng.integers(0, 16, 40))}
                  | {(0, 0), (199, 15), (200, 3), (628, 7)})
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq, rows), w, pairs=rows)


@pytest.mark.parametrize("d", [128, 64])
def test_fp8_prefill_of_one_token_matches_fp8_decode(pk, d):
    w = W.build_decode_workload(RAGGED, 8, 2, d, 16, "fp16", 23)
    w.query_start = np.arange(w.num_seqs + 1, dtype=np.int32)
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    kq, vq = oracle_codes(w)
    assert_close(dev_to_bits(dev.out), oracle_decode8(w, kq, vq), w)


def test_fp8_prefill_reports_a_bad_scale(pk):
    w = W.build_prefill_workload([4, 10], [3, 5], 4, 2, 128, 16, "fp16", seed=2)
    dev = Fp8Device(pk, w)
    dev.vs = torch.tensor([0.01, 0.0], dtype=torch.float32, device="cuda")
    assert run_prefill8(pk, dev) & pk.DEVERR_BAD_SCALE


def test_fp8_prefill_named_workload_sampled(pk):
    """The LLaMA-7B prefill batch at full size, on sampled rows."""
    w = W.make("llama7b_prefill")
    dev = Fp8Device(pk, w)
    assert run_prefill8(pk, dev) == 0
    rng = np.random.default_rng(4)
    total = int(w.query_start[-1])
    rows = sorted({(int(t), int(h)) for t, h in zip(rng.integers(0, total, 24),
                                                    rng.integers(0, w.num_heads, 24))}
                  | {(0, 0), (total - 1, w.num_heads - 1)})
    seq_of = np.repeat(np.arange(w.num_seqs), np.diff(w.query_start))
    seqs = sorted({int(seq_of[t]) for t, _ in rows})
    blocks = np.unique(np.concatenate(
        [w.block_tables[s, :-(-int(w.context_lens[s]) // w.block_size)] for s in seqs]))
    kq, vq = oracle_codes(w, blocks=blocks)
    assert_close(dev_to_bits(dev.out), oracle_prefill8(w, kq, vq, rows), w, pairs=rows)
    assert torch.isfinite(dev.out.float()).all()
