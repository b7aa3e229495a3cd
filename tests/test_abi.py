"""The C ABI library loads, exports every symbol include/pagedkv.h declares,
and validates arguments on the host (no GPU needed: every case below is
rejected before anything is enqueued)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_394_b200 import pagedkv
    return ctypes.CDLL(pagedkv.LIB_PATH)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(lib, n)]
    assert missing == []


def test_version_and_status_strings():
    from paged_kv_cache_394_b200 import pagedkv as pk
    assert "sm_100a" in pk.version()
    for s in range(6):
        assert pk._status_string(s).decode() != "unknown status"
    assert pk._status_string(99).decode() == "unknown status"


def test_host_validation_without_gpu():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    # reshape_and_cache: unsupported head_dim, negative tokens, null pointers
    assert pk._reshape_and_cache(null, null, null, null, null, 4, 2, 96, 16, 8, 0, null, null) == pk.ERR_UNSUPPORTED
    assert pk._reshape_and_cache(null, null, null, null, null, -1, 2, 64, 16, 8, 0, null, null) == pk.ERR_INVALID_ARG
    assert pk._reshape_and_cache(null, null, null, null, null, 4, 2, 64, 16, 8, 0, null, null) == pk.ERR_INVALID_ARG
    assert pk._reshape_and_cache(null, null, null, null, null, 0, 2, 64, 16, 8, 0, null, null) == pk.OK
    assert pk._reshape_and_cache(null, null, null, null, null, 4, 2, 64, 16, 8, 7, null, null) == pk.ERR_INVALID_ARG
    # misaligned pointers
    bad = ctypes.c_void_p(0x1008)
    good = ctypes.c_void_p(0x1000)
    assert pk._reshape_and_cache(bad, good, good, good, good, 4, 2, 64, 16, 8, 0, null, null) == pk.ERR_INVALID_ARG
    # copy_blocks
    assert pk._copy_blocks(null, null, null, 0, 2, 64, 16, 8, 0, null, null) == pk.OK
    assert pk._copy_blocks(null, null, null, 3, 2, 64, 16, 8, 0, null, null) == pk.ERR_INVALID_ARG
    assert pk._copy_blocks(good, good, good, 3, 2, 64, 24, 8, 0, null, null) == pk.ERR_UNSUPPORTED
    # decode: group 3 unsupported, heads not a multiple, partition not a multiple
    args = lambda **kw: dict(dict(s=2, h=6, hkv=2, d=64, bs=16, mb=4, mc=64, n=8, part=0), **kw)

    def dec(a, ptr=good, ws=None, wsb=0):
        return pk._paged_attn_decode(ptr, ptr, ptr, ptr, ptr, ptr, 0.125, a["s"], a["h"], a["hkv"],
                                     a["d"], a["bs"], a["mb"], a["mc"], a["n"], 0, a["part"], ws,
                                     wsb, null, null)
    assert dec(args()) == pk.ERR_UNSUPPORTED              # G = 3
    assert dec(args(h=5)) == pk.ERR_INVALID_ARG            # 5 % 2 != 0
    assert dec(args(h=4, part=24)) == pk.ERR_INVALID_ARG   # not a multiple of 16
    assert dec(args(h=4, mc=65)) == pk.ERR_INVALID_ARG     # > max_blocks * block_size
    assert dec(args(h=4, s=0)) == pk.OK
    assert dec(args(h=4), ptr=null) == pk.ERR_INVALID_ARG
    assert dec(args(h=4), ptr=bad) == pk.ERR_INVALID_ARG
    assert dec(args(h=4, part=16)) == pk.ERR_WORKSPACE     # split needs a workspace
    # non-finite scale
    assert pk._paged_attn_decode(good, good, good, good, good, good, float("nan"), 2, 4, 2, 64, 16,
                                 4, 64, 8, 0, 0, null, 0, null, null) == pk.ERR_INVALID_ARG


def test_partition_and_workspace_queries():
    from paged_kv_cache_394_b200 import pagedkv as pk
    # short contexts over many (sequence, kv head) units: single pass
    assert pk.partition_size(64, 32, 16, 2048) >= 2048
    assert pk.workspace_bytes(64, 32, 32, 128, 16, 2048) == 0
    # long contexts over few units: 4096-token partitions (E4M3: 2048)
    assert pk.partition_size(8, 40, 16, 32768) == 4096
    assert pk.partition_size_fp8(8, 40, 16, 32768) == 2048
    n = 8 * 40 * 16
    assert pk.workspace_bytes(8, 40, 40, 128, 16, 32768) >= n * (128 + 2) * 4
    # many units but long contexts: split too; a context that fits one
    # partition runs in one pass
    assert pk.partition_size(256, 8, 32, 4096) >= 4096     # enough units: one pass
    assert pk.partition_size_fp8(256, 8, 32, 4096) == 2048
    # the workspace covers the E4M3 rule's partitions too
    assert pk.workspace_bytes(256, 32, 8, 128, 32, 4096) >= 256 * 32 * 2 * 130 * 4
    assert pk.partition_size(4, 4, 16, 100) >= 100
    # few units: small partitions for parallelism, never below 256 tokens
    assert pk.partition_size(1, 8, 16, 2000) == 256
    # an explicit request is honoured
    assert pk.partition_size(64, 32, 16, 2048, 256) == 256
    assert pk.workspace_bytes(64, 32, 32, 128, 16, 2048, 256) >= 64 * 32 * 8 * 130 * 4
    assert pk.workspace_bytes(64, 32, 32, 128, 16, 2048, 24) == 0   # invalid request


def test_staging_bytes_covers_inputs():
    from paged_kv_cache_394_b200 import pagedkv as pk
    s, h, hkv, d, mb, t, p = 64, 32, 32, 128, 128, 64, 3
    need = 2 * s * h * d * 2 + 2 * t * hkv * d * 2 + t * 8 + p * 16 + s * mb * 4 + s * 4
    assert pk.staging_bytes(s, h, hkv, d, mb, t, p) >= need


def test_fp8_host_validation_without_gpu():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    good = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1008)
    rc8 = pk._reshape_and_cache_fp8
    # 16-bit sources only; E4M3 is a cache type, not an input type
    assert rc8(good, good, good, good, good, 4, 2, 64, 16, 8, pk.FP8_E4M3, good, good, null,
               null) == pk.ERR_INVALID_ARG
    # scale arrays are required
    assert rc8(good, good, good, good, good, 4, 2, 64, 16, 8, pk.FP16, null, good, null,
               null) == pk.ERR_INVALID_ARG
    assert rc8(good, good, good, good, good, 4, 2, 64, 16, 8, pk.FP16, good, null, null,
               null) == pk.ERR_INVALID_ARG
    assert rc8(null, null, null, null, null, 0, 2, 64, 16, 8, pk.BF16, null, null, null,
               null) == pk.OK
    assert rc8(null, null, null, null, null, 4, 2, 96, 16, 8, pk.FP16, good, good, null,
               null) == pk.ERR_UNSUPPORTED
    assert rc8(good, bad, good, good, good, 4, 2, 64, 16, 8, pk.FP16, good, good, null,
               null) == pk.ERR_INVALID_ARG
    # copy_blocks accepts the 1-byte cache type; unknown types are rejected
    assert pk._copy_blocks(null, null, null, 0, 2, 64, 16, 8, pk.FP8_E4M3, null, null) == pk.OK
    assert pk._copy_blocks(good, good, good, 1, 2, 64, 16, 8, 9, null, null) == pk.ERR_INVALID_ARG
    # the 16-bit scatter and decode still refuse the 1-byte type
    assert pk._reshape_and_cache(good, good, good, good, good, 4, 2, 64, 16, 8, pk.FP8_E4M3,
                                 null, null) == pk.ERR_INVALID_ARG

    def dec8(ks=good, vs=good, h=4, dt=pk.FP16, s=2, ptr=good):
        return pk._paged_attn_decode_fp8(ptr, ptr, ptr, ptr, ptr, ptr, 0.125, ks, vs, s, h, 2, 64,
                                         16, 4, 64, 8, dt, 0, null, 0, null, null)
    assert dec8(ks=null) == pk.ERR_INVALID_ARG
    assert dec8(vs=null) == pk.ERR_INVALID_ARG
    assert dec8(dt=pk.FP8_E4M3) == pk.ERR_INVALID_ARG     # q/out must be 16-bit
    assert dec8(h=6) == pk.ERR_UNSUPPORTED                 # G = 3
    assert dec8(s=0) == pk.OK
    assert dec8(ptr=bad) == pk.ERR_INVALID_ARG


def test_prefill_fp8_host_validation_without_gpu():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    good = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1008)

    def pre8(ks=good, vs=good, d=128, h=4, dt=pk.FP16, s=2, ptr=good):
        # out q k v tables lens qstart scale ks vs S T H Hkv D bs maxblk maxctx maxq nblk dt
        return pk._paged_attn_prefill_fp8(ptr, ptr, ptr, ptr, ptr, ptr, ptr, 0.125, ks, vs, s, 8,
                                          h, 2, d, 16, 4, 64, 4, 8, dt, null, null)
    assert pre8(d=96) == pk.ERR_UNSUPPORTED               # head_dim 64 or 128
    assert pre8(h=6) == pk.ERR_UNSUPPORTED                # G = 3
    assert pre8(ks=null) == pk.ERR_INVALID_ARG
    assert pre8(vs=null) == pk.ERR_INVALID_ARG
    assert pre8(dt=pk.FP8_E4M3) == pk.ERR_INVALID_ARG     # q/out must be 16-bit
    assert pre8(s=0) == pk.OK
    assert pre8(ptr=bad) == pk.ERR_INVALID_ARG


def test_binding_constants_match_the_header():
    """Status codes, dtype codes and device error bits of the binding equal
    the values include/pagedkv.h defines."""
    import re
    from paged_kv_cache_394_b200 import pagedkv as pk
    hdr = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    bits = dict((m.group(1), int(m.group(2))) for m in
                re.finditer(r"#define PKV_DEVERR_(\w+) (\d+)u", hdr))
    assert bits and all(getattr(pk, "DEVERR_" + k) == v for k, v in bits.items())
    for name, val in re.findall(r"PKV_((?:ERR_\w+|OK))\s*=\s*(\d+)", hdr):
        assert getattr(pk, name) == int(val), name
    for name, val in re.findall(r"PKV_(FP16|BF16|FP8_E4M3)\s*=\s*(\d+)", hdr):
        assert getattr(pk, name) == int(val), name


def test_cascade_host_validation_without_gpu():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    good = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1008)
    ws = pk.cascade_workspace_bytes(4, 8, 2, 128, 16, 256)
    assert ws > 0 and ws >= pk.workspace_bytes(4, 8, 2, 128, 16, 256)

    def cas(s=4, g=2, mgs=2, msb=4, d=128, ptr=good, gptr=good, wsb=ws, mc=256, part=0):
        return pk._paged_attn_decode_cascade(ptr, ptr, ptr, ptr, ptr, ptr, gptr, gptr, 0.125, s, g,
                                             mgs, msb, 8, 2, d, 16, 16, mc, 64, 0, part, good,
                                             wsb, null, null)
    assert cas(s=0) == pk.OK
    assert cas(d=96) == pk.ERR_UNSUPPORTED                 # head_dim 64 or 128
    assert cas(g=0) == pk.ERR_INVALID_ARG                  # sequences but no groups
    assert cas(msb=17) == pk.ERR_INVALID_ARG               # 17 * 16 > max_context_len
    assert cas(gptr=null) == pk.ERR_INVALID_ARG
    assert cas(wsb=ws - 16) == pk.ERR_WORKSPACE
    assert cas(ptr=bad) == pk.ERR_INVALID_ARG
    assert cas(part=24) == pk.ERR_INVALID_ARG              # not a multiple of block_size

    def cas8(s=4, d=64, ks=good, vs=good, dt=pk.BF16):
        return pk._paged_attn_decode_cascade_fp8(good, good, good, good, good, good, good, good,
                                                 0.125, ks, vs, s, 2, 2, 4, 8, 2, d, 16, 16, 256,
                                                 64, dt, 0, good, ws, null, null)
    assert cas8(s=0) == pk.OK
    assert cas8(d=96) == pk.ERR_UNSUPPORTED
    assert cas8(ks=null) == pk.ERR_INVALID_ARG
    assert cas8(vs=null) == pk.ERR_INVALID_ARG
    assert cas8(dt=pk.FP8_E4M3) == pk.ERR_INVALID_ARG      # q/out must be 16-bit


def test_pipeline_staging_and_host_validation_without_gpu():
    """Two staging areas, each holding a step at the maxima; bad arguments
    are refused before any stream or event is created."""
    from paged_kv_cache_394_b200 import pagedkv as pk
    s, h, hkv, d, mb, t, p = 64, 32, 32, 128, 128, 64, 3
    one = pk.staging_bytes(s, h, hkv, d, mb, t, p)
    assert pk.DecodePipeline.staging_bytes(s, h, hkv, d, mb, t, p) >= 2 * one
    assert pk.DecodePipeline.staging_bytes(s, 0, hkv, d, mb, t, p) == 0
    lib = ctypes.CDLL(pk.LIB_PATH)
    lib.pkv_decode_pipeline_create.argtypes = ([ctypes.c_void_p] + [ctypes.c_int] * 9 +
                                               [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p])
    h_out = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: every case fails first
    need = pk.DecodePipeline.staging_bytes(s, h, hkv, d, mb, t, p)
    args = [s, h, hkv, d, 16, mb, t, p, pk.FP16]
    assert lib.pkv_decode_pipeline_create(None, *args, fake, need, None) == pk.ERR_INVALID_ARG
    bad_heads = [s, h, 5, d, 16, mb, t, p, pk.FP16]          # 32 % 5 != 0
    assert lib.pkv_decode_pipeline_create(ctypes.byref(h_out), *bad_heads, fake, need,
                                          None) == pk.ERR_INVALID_ARG
    bad_dim = [s, h, hkv, 96, 16, mb, t, p, pk.FP16]
    assert lib.pkv_decode_pipeline_create(ctypes.byref(h_out), *bad_dim, fake, need,
                                          None) == pk.ERR_UNSUPPORTED
    assert lib.pkv_decode_pipeline_create(ctypes.byref(h_out), *args, None, need,
                                          None) == pk.ERR_INVALID_ARG
    assert lib.pkv_decode_pipeline_create(ctypes.byref(h_out), *args, fake, need - 16,
                                          None) == pk.ERR_WORKSPACE
    assert h_out.value is None
    lib.pkv_decode_pipeline_step.restype = ctypes.c_int
    assert lib.pkv_decode_pipeline_step(None, *([None] * 18)) == pk.ERR_INVALID_ARG


def test_testing_wait_hook_validates_on_the_host():
    from paged_kv_cache_394_b200 import pagedkv as pk
    for bad in (0, 2_000_000_001):
        with pytest.raises(pk.PagedKVError):
            pk.testing_decode_wait(bad, False)
    pk.testing_decode_wait(2_000_000_000, False)      # the default, accepted


@pytest.mark.parametrize("seed,n", [(0, 0), (1, 1), (2, 64), (3, 257), (4, 1000)])
def test_decode_order_is_longest_first_by_bucket(seed, n):
    """pkv_decode_order: a permutation; buckets of 256 tokens in descending
    order; index order inside a bucket (the definition, restated with a
    stable lexicographic sort)."""
    import numpy as np
    from paged_kv_cache_394_b200 import pagedkv as pk
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 40000, size=n).astype(np.int32)
    lens[: n // 3] = rng.integers(1000, 1300, size=n // 3)      # many ties in one bucket
    order = pk.decode_order(lens).numpy()
    assert sorted(order.tolist()) == list(range(n))
    expect = np.lexsort((np.arange(n), -(lens // 256)))
    assert np.array_equal(order, expect)


@pytest.mark.parametrize("seed,n,bs,part", [(0, 0, 16, 256), (1, 1, 16, 512), (2, 64, 32, 2048),
                                            (3, 257, 16, 1024), (4, 1000, 16, 4096),
                                            (5, 50, 16, 16)])
def test_decode_plan_lists_every_partition_longest_first(seed, n, bs, part):
    """pkv_decode_plan: exactly the (sequence, partition) items that exist,
    each once, with its sequence's partition count; descending in buckets
    of 256 tokens of the item's own length, (sequence, partition) order
    within a bucket (restated with a stable lexicographic sort)."""
    import numpy as np
    from paged_kv_cache_394_b200 import pagedkv as pk
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 9000, size=n).astype(np.int32)
    lens[: n // 4] = 0                                          # empty sequences: one item
    lens[n // 4: n // 2] = part * rng.integers(1, 4, size=n // 2 - n // 4)   # exact multiples
    work = pk.decode_plan(lens, bs, part).numpy()
    seqs, parts, counts, sizes = [], [], [], []
    for i, L in enumerate(lens.tolist()):
        nblk = -(-L // bs)
        np_ = max(1, -(-nblk // (part // bs)))
        for j in range(np_):
            seqs.append(i); parts.append(j); counts.append(np_)
            sizes.append(max(0, min(part, L - j * part)))
    seqs, parts, counts, sizes = map(np.asarray, (seqs, parts, counts, sizes))
    key = np.lexsort((parts, seqs, -(sizes // 256)))
    assert work.shape == (len(seqs), 2)
    assert np.array_equal(work[:, 0], seqs[key])
    assert np.array_equal(work[:, 1] & 0xFFFF, parts[key])
    assert np.array_equal(work[:, 1] >> 16, counts[key])


def test_decode_plan_and_planned_decode_validate_on_the_host():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    good = ctypes.c_void_p(0x1000)
    n = ctypes.c_int(-1)
    lens = (ctypes.c_int32 * 3)(100, 5000, 0)
    work = (ctypes.c_int32 * 8)()
    assert pk._decode_plan(lens, 3, 16, 2048, null, 0, ctypes.byref(n)) == pk.OK and n.value == 5
    assert pk._decode_plan(lens, 3, 16, 2048, work, 4, ctypes.byref(n)) == pk.ERR_INVALID_ARG
    assert pk._decode_plan(lens, 3, 16, 2048, work, 4, null) == pk.ERR_INVALID_ARG
    assert pk._decode_plan(lens, 3, 16, 24, work, 4, ctypes.byref(n)) == pk.ERR_INVALID_ARG
    assert pk._decode_plan(lens, 3, 16, 0, work, 4, ctypes.byref(n)) == pk.ERR_INVALID_ARG
    assert pk._decode_plan(null, 3, 16, 2048, work, 4, ctypes.byref(n)) == pk.ERR_INVALID_ARG
    assert pk._decode_plan(null, 0, 16, 2048, null, 0, ctypes.byref(n)) == pk.OK and n.value == 0
    long = (ctypes.c_int32 * 1)(16 * 65536)                    # 65536 partitions of one block
    assert pk._decode_plan(long, 1, 16, 16, null, 0, ctypes.byref(n)) == pk.ERR_UNSUPPORTED

    def dec(part, items=4, w=good, fp8=False):
        if fp8:
            return pk._paged_attn_decode_fp8_planned(good, good, good, good, good, good, w, items,
                                                     0.125, good, good, 2, 8, 2, 128, 16, 256,
                                                     4096, 512, 0, part, good, 1 << 30, null, null)
        return pk._paged_attn_decode_planned(good, good, good, good, good, good, w, items, 0.125,
                                             2, 8, 2, 128, 16, 256, 4096, 512, 0, part, good,
                                             1 << 30, null, null)
    for fp8 in (False, True):
        assert dec(0, fp8=fp8) == pk.ERR_INVALID_ARG                 # no partition size
        assert dec(2048, items=1, fp8=fp8) == pk.ERR_INVALID_ARG     # fewer items than sequences
        assert dec(2048, w=null, fp8=fp8) == pk.ERR_INVALID_ARG
        assert dec(2048, w=ctypes.c_void_p(0x1004), fp8=fp8) == pk.ERR_INVALID_ARG  # alignment
        assert dec(24, fp8=fp8) == pk.ERR_INVALID_ARG                # not a multiple of 16


@pytest.mark.parametrize("seed,n,h,hkv,sms", [(0, 4, 32, 32, 148), (1, 4, 32, 8, 148),
                                              (2, 1, 8, 8, 148), (3, 9, 16, 2, 20),
                                              (4, 30, 32, 8, 148), (5, 3, 8, 1, 4)])
def test_prefill_plan_covers_every_key_once(seed, n, h, hkv, sms):
    """pkv_prefill_plan: every (sequence, 256-row tile) unit with rows appears
    whole or as 2-4 pieces whose key ranges tile [0, causal end) in order:
    pieces before the last are whole 64-key tiles of history (every row sees
    them), the last starts inside the history; merge entries name exactly the
    cut units; items come longest first by the planner's cost."""
    import numpy as np
    from paged_kv_cache_394_b200 import pagedkv as pk
    rng = np.random.default_rng(seed)
    ql = rng.integers(0, 700, size=n)
    ql[0] = 512
    hist = rng.integers(0, 9000, size=n)
    qs = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    lens = (hist + ql).astype(np.int32)
    plan = pk.prefill_plan(qs, lens, h, hkv, 128, sms)
    work, merges = plan.work.numpy(), plan.merges.numpy()
    g = h // hkv
    units = {(s, t) for s in range(n) for t in range(-(-int(ql[s]) * g // 256))}
    seen = {}
    for it in work:
        seen.setdefault((int(it[0]), int(it[1])), []).append(it)
    assert set(seen) == units
    cut = set()
    for (s, t), its in seen.items():
        its = sorted(its, key=lambda it: it[4])
        pieces = int(its[0][6])
        assert [int(it[4]) for it in its] == list(range(pieces)) and 1 <= pieces <= 4
        assert all(int(it[6]) == pieces for it in its)
        if pieces == 1:
            assert (its[0][2], its[0][3]) == (0, -1)
            continue
        cut.add((s, t))
        assert len({int(it[5]) for it in its}) == 1
        kb = 0
        for it in its[:-1]:
            assert it[2] == kb and it[3] > kb and it[3] % 64 == 0 and it[3] <= hist[s]
            kb = int(it[3])
        assert its[-1][2] == kb and its[-1][3] == -1 and kb <= hist[s]
        m = int(its[0][5])
        assert tuple(merges[m][:3]) == (s, t, pieces)
    assert len(merges) == len(cut)
    if len(merges) == 0:
        assert plan.workspace_bytes == 0
    else:   # [merges][kv heads][256 rows][4 pieces] x (o, m, l) in fp32
        assert plan.workspace_bytes >= len(merges) * hkv * 256 * 4 * 130 * 4


def test_prefill_plan_splits_the_longest_unit():
    """Four sequences, one with a long history: only its units are cut, and
    its last query tile (the most keys) is among them."""
    import numpy as np
    from paged_kv_cache_394_b200 import pagedkv as pk
    ql = np.array([512, 512, 512, 512])
    hist = np.array([3000, 300, 100, 50])
    qs = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    plan = pk.prefill_plan(qs, (hist + ql).astype(np.int32), 32, 8, 128, 148)
    work = plan.work.numpy()
    assert len(plan.merges) > 0 and set(plan.merges.numpy()[:, 0]) == {0}
    assert any(it[0] == 0 and it[1] == 7 and it[6] > 1 for it in work)


def test_planned_prefill_validates_on_the_host():
    from paged_kv_cache_394_b200 import pagedkv as pk
    null = None
    good = ctypes.c_void_p(0x1000)
    n, m, wb = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    qs = (ctypes.c_int32 * 3)(0, 512, 1024)
    lens = (ctypes.c_int32 * 2)(4000, 600)
    assert pk._prefill_plan(qs, lens, 2, 8, 2, 64, 148, null, 0, ctypes.byref(n), null, 0,
                            ctypes.byref(m), null) == pk.ERR_UNSUPPORTED          # head_dim 64
    assert pk._prefill_plan(qs, lens, 2, 8, 2, 128, 0, null, 0, ctypes.byref(n), null, 0,
                            ctypes.byref(m), null) == pk.ERR_INVALID_ARG          # no SMs
    assert pk._prefill_plan(qs, lens, 2, 8, 2, 128, 148, null, 0, ctypes.byref(n), null, 0,
                            ctypes.byref(m), ctypes.byref(wb)) == pk.OK
    assert n.value >= 2 and m.value >= 1 and wb.value > 0
    work = (ctypes.c_int32 * (8 * n.value))()
    assert pk._prefill_plan(qs, lens, 2, 8, 2, 128, 148, work, n.value - 1, ctypes.byref(n),
                            null, 0, ctypes.byref(m), null) == pk.ERR_INVALID_ARG  # capacity

    def pre(d=128, ws=good, wsb=1 << 30, nm=1, merges=good):
        return pk._paged_attn_prefill_planned(good, good, good, good, good, good, good, good, 4,
                                              merges, nm, 0.125, 2, 1024, 8, 2, d, 16, 256, 4096,
                                              512, 512, 0, ws, wsb, null, null)
    assert pre(d=64) == pk.ERR_UNSUPPORTED
    assert pre(ws=null, wsb=0) == pk.ERR_WORKSPACE
    assert pre(wsb=1024) == pk.ERR_WORKSPACE
    assert pre(merges=null) == pk.ERR_INVALID_ARG
    assert pre(ws=ctypes.c_void_p(0x1008)) == pk.ERR_INVALID_ARG


def test_planners_edge_cases():
    """Empty batches, empty queries, histories too short to cut, and one
    huge history (at most four pieces, each history piece whole key tiles)."""
    import numpy as np
    from paged_kv_cache_394_b200 import pagedkv as pk
    # no sequences
    p = pk.prefill_plan(np.zeros(1, np.int32), np.zeros(0, np.int32), 8, 2)
    assert p.work.shape == (0, 8) and p.merges.shape == (0, 4) and p.workspace_bytes == 0
    assert pk.decode_plan(np.zeros(0, np.int32), 16, 256).shape == (0, 2)
    # sequences without new tokens have no units
    p = pk.prefill_plan(np.array([0, 0, 5, 5], np.int32), np.array([9, 20, 7], np.int32), 8, 2)
    assert sorted(set(p.work[:, 0].tolist())) == [1]
    # a history shorter than one key tile is never cut, however many SMs
    p = pk.prefill_plan(np.array([0, 300], np.int32), np.array([363], np.int32), 8, 2, 128, 10**6)
    assert len(p.merges) == 0
    # one huge history: cut, at most four pieces, history pieces whole tiles
    p = pk.prefill_plan(np.array([0, 64], np.int32), np.array([1_000_064], np.int32), 8, 8, 128, 148)
    w = p.work.numpy()
    assert len(p.merges) == 1 and (w[:, 6] <= 4).all() and (w[:, 6] >= 2).all()
    hist = w[w[:, 3] >= 0]
    assert (hist[:, 2] % 64 == 0).all() and (hist[:, 3] % 64 == 0).all()
    assert (hist[:, 3] <= 1_000_000).all()
    # decode: empty contexts still get one item each
    d = pk.decode_plan(np.array([0, 0, 40], np.int32), 16, 32).numpy()
    assert sorted(d[:, 0].tolist()) == [0, 1, 2, 2]
    assert (d[d[:, 0] < 2, 1] == (0 | (1 << 16))).all()
