"""The decode entry point that allocates nothing.

Some callers cannot allocate device memory: a plugin inside a host application
that owns every device allocation, or a serving loop that must not call
cudaMalloc once it runs, since cudaMalloc can synchronise the device.  For
them, pkv_paged_attn_decode_static_ws keeps its split-K scratch in a fixed
array inside the library.  These tests call it through the C ABI and check
its result against the ordinary entry point (which is given a caller-owned
workspace).  Both run the same kernels with the same partitions, so the two
outputs must agree bit for bit: a tolerance would hide a scratch-layout error
that happens to stay small.

The array exists once per CUDA context, so one test runs in a child process
that drives the CUDA driver API itself: the device's primary context first,
then a second context the child creates and makes current, then the primary
context again; each time the fixed-scratch call must equal the allocating one.

The file is collected last and needs no state from other tests: it passes
alone in a fresh process and after the rest of the suite.
"""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def device_inputs(w):
    tdt = torch.float16 if w.dtype == "fp16" else torch.bfloat16

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(tdt)
    return dict(q=up(w.q), k=up(w.k_cache), v=up(w.v_cache), key=up(w.key), value=up(w.value),
                slots=torch.from_numpy(w.slot_mapping).cuda(),
                tables=torch.from_numpy(w.block_tables).cuda(),
                lens=torch.from_numpy(w.context_lens).cuda())


def test_static_workspace_decode_matches_allocating_decode():
    from paged_kv_cache_394_b200 import pagedkv as pk
    from paged_kv_cache_394_b200 import workloads as W

    batches = [
        # long contexts: split-K with 512-token partitions
        W.build_decode_workload([9000, 17, 4096, 1, 2500, 600], 16, 8, 128, 16, "fp16", 11),
        # a different shape and dtype, forced split at 64 tokens
        W.build_decode_workload([300, 45, 129, 700], 8, 2, 64, 32, "bf16", 12),
    ]
    parts = [0, 64]
    for w, part in zip(batches, parts):
        need = pk.workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                                  w.block_size, w.max_context_len, part)
        assert 0 < need <= pk.STATIC_WORKSPACE_BYTES      # the split-K scratch is used
        d = device_inputs(w)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        # the step's new tokens first: until then their slots hold NaN poison
        pk.reshape_and_cache(d["key"], d["value"], d["k"], d["v"], d["slots"], dev_err=err)
        old = torch.empty_like(d["q"])
        new = torch.full_like(d["q"], float("nan"))
        pk.paged_attn_decode(old, d["q"], d["k"], d["v"], d["tables"], d["lens"], w.scale,
                             w.num_kv_heads, w.block_size, w.max_context_len,
                             partition_size=part, dev_err=err)
        pk.paged_attn_decode_static_ws(new, d["q"], d["k"], d["v"], d["tables"], d["lens"],
                                       w.scale, w.num_kv_heads, w.block_size, w.max_context_len,
                                       partition_size=part, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.isfinite(old.float()).all()
        assert torch.equal(new.view(torch.int16), old.view(torch.int16))


def test_static_workspace_rejects_oversized_requests():
    from paged_kv_cache_394_b200 import pagedkv as pk
    # 64 sequences x 32 heads x 64 partitions of 16 tokens needs far more than the array holds
    s, h, d, bs, ctx, part = 64, 32, 128, 16, 1024, 16
    assert pk.workspace_bytes(s, h, h, d, bs, ctx, part) > pk.STATIC_WORKSPACE_BYTES
    q = torch.zeros(s, h, d, dtype=torch.float16, device="cuda")
    kc = torch.zeros(8, h, bs, d, dtype=torch.float16, device="cuda")
    tables = torch.zeros(s, ctx // bs, dtype=torch.int32, device="cuda")
    lens = torch.ones(s, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedKVError) as e:
        pk.paged_attn_decode_static_ws(q, q, kc, kc, tables, lens, 0.1, h, bs, ctx,
                                       partition_size=part)
    assert e.value.status == pk.ERR_WORKSPACE


# The child: CUDA driver API through ctypes (torch never touches the device
# there), the library's C entry points through ctypes.  It prints one line per
# context and exits non-zero on the first mismatch or error.
CHILD = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from paged_kv_cache_394_b200 import workloads as W

cu = ctypes.CDLL("libcuda.so.1")
lib = ctypes.CDLL(sys.argv[2])
vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
for name, args in (("cuInit", [ctypes.c_uint]),
                   ("cuDeviceGet", [ctypes.POINTER(i32), i32]),
                   ("cuDevicePrimaryCtxRetain", [ctypes.POINTER(vp), i32]),
                   ("cuDevicePrimaryCtxRelease_v2", [i32]),
                   ("cuCtxCreate_v2", [ctypes.POINTER(vp), ctypes.c_uint, i32]),
                   ("cuCtxDestroy_v2", [vp]),
                   ("cuCtxSetCurrent", [vp]),
                   ("cuCtxSynchronize", []),
                   ("cuMemAlloc_v2", [ctypes.POINTER(ctypes.c_uint64), sz]),
                   ("cuMemFree_v2", [ctypes.c_uint64]),
                   ("cuMemsetD8_v2", [ctypes.c_uint64, ctypes.c_ubyte, sz]),
                   ("cuMemcpyHtoD_v2", [ctypes.c_uint64, vp, sz]),
                   ("cuMemcpyDtoH_v2", [vp, ctypes.c_uint64, sz])):
    getattr(cu, name).argtypes = args
    getattr(cu, name).restype = i32
lib.pkv_reshape_and_cache.argtypes = [vp] * 5 + [i32] * 6 + [vp, vp]
lib.pkv_paged_attn_workspace_bytes.argtypes = [i32] * 7
lib.pkv_paged_attn_workspace_bytes.restype = sz
lib.pkv_paged_attn_decode.argtypes = [vp] * 6 + [f32] + [i32] * 10 + [vp, sz, vp, vp]
lib.pkv_paged_attn_decode_static_ws.argtypes = [vp] * 6 + [f32] + [i32] * 10 + [vp, vp]
for f in (lib.pkv_reshape_and_cache, lib.pkv_paged_attn_decode,
          lib.pkv_paged_attn_decode_static_ws):
    f.restype = i32


def ck(r, what):
    if r != 0:
        sys.exit("%s returned %d" % (what, r))


w = W.build_decode_workload([900, 17, 300, 1, 64, 700], 8, 8, 128, 16, "fp16", 21)
part = 64                                   # split-K: the scratch holds partials
hkv, d, bs = w.num_kv_heads, w.head_dim, w.block_size
ws_bytes = lib.pkv_paged_attn_workspace_bytes(w.num_seqs, w.num_heads, hkv, d, bs,
                                              w.max_context_len, part)
assert ws_bytes > 0


def run_in_current_context(label):
    bufs = []

    def dev(nbytes, host=None):
        p = ctypes.c_uint64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), max(16, nbytes)), "cuMemAlloc")
        bufs.append(p.value)
        if host is not None:
            host = np.ascontiguousarray(host)
            ck(cu.cuMemcpyHtoD_v2(p.value, host.ctypes.data, host.nbytes), "cuMemcpyHtoD")
        return p.value

    q, kc, vc = dev(w.q.nbytes, w.q), dev(w.k_cache.nbytes, w.k_cache), dev(w.v_cache.nbytes, w.v_cache)
    key, val = dev(w.key.nbytes, w.key), dev(w.value.nbytes, w.value)
    slots = dev(w.slot_mapping.nbytes, w.slot_mapping)
    tables, lens = dev(w.block_tables.nbytes, w.block_tables), dev(w.context_lens.nbytes, w.context_lens)
    out_a, out_b = dev(w.q.nbytes), dev(w.q.nbytes)
    ws, err = dev(ws_bytes), dev(4)
    ck(cu.cuMemsetD8_v2(err, 0, 4), "cuMemset")
    ck(cu.cuMemsetD8_v2(out_b, 0xFF, w.q.nbytes), "cuMemset")   # NaN until written
    ck(lib.pkv_reshape_and_cache(key, val, kc, vc, slots, len(w.slot_mapping), hkv, d, bs,
                                 w.num_blocks, 0, err, None), "reshape_and_cache")
    args = (q, kc, vc, tables, lens, w.scale, w.num_seqs, w.num_heads, hkv, d, bs,
            w.max_blocks_per_seq, w.max_context_len, w.num_blocks, 0, part)
    ck(lib.pkv_paged_attn_decode(out_a, *args, ws, ws_bytes, err, None), "decode")
    ck(lib.pkv_paged_attn_decode_static_ws(out_b, *args, err, None), "decode_static_ws")
    ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    a, b = np.empty_like(w.q), np.empty_like(w.q)
    e = np.zeros(1, dtype=np.uint32)
    ck(cu.cuMemcpyDtoH_v2(a.ctypes.data, out_a, a.nbytes), "cuMemcpyDtoH")
    ck(cu.cuMemcpyDtoH_v2(b.ctypes.data, out_b, b.nbytes), "cuMemcpyDtoH")
    ck(cu.cuMemcpyDtoH_v2(e.ctypes.data, err, 4), "cuMemcpyDtoH")
    for p in bufs:
        ck(cu.cuMemFree_v2(p), "cuMemFree")
    if e[0] != 0:
        sys.exit("%s: device error word %d" % (label, e[0]))
    if not np.isfinite(a.view(np.float16).astype(np.float32)).all():
        sys.exit("%s: allocating decode gave non-finite output" % label)
    if not np.array_equal(a, b):
        sys.exit("%s: fixed-scratch decode differs from the allocating decode" % label)
    print(label, "ok", flush=True)


ck(cu.cuInit(0), "cuInit")
devn = i32()
ck(cu.cuDeviceGet(ctypes.byref(devn), 0), "cuDeviceGet")
primary = vp()
ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), devn), "cuDevicePrimaryCtxRetain")
ck(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
run_in_current_context("primary context")
other = vp()
ck(cu.cuCtxCreate_v2(ctypes.byref(other), 0, devn), "cuCtxCreate")   # now current
run_in_current_context("second context")
ck(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
run_in_current_context("primary context again")
ck(cu.cuCtxDestroy_v2(other), "cuCtxDestroy")
ck(cu.cuDevicePrimaryCtxRelease_v2(devn), "cuDevicePrimaryCtxRelease")
"""


def test_static_workspace_decode_in_each_cuda_context():
    from paged_kv_cache_394_b200 import pagedkv as pk
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, pk.library_path()],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.split("\n")[:3] == ["primary context ok", "second context ok",
                                        "primary context again ok"]
