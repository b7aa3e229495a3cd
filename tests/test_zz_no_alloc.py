"""The decode entry point that allocates nothing.

Some callers cannot allocate device memory: a plugin inside a host application
that owns every device allocation, or a serving loop that must not call
cudaMalloc once it runs, since cudaMalloc can synchronise the device.  For
them, pkv_paged_attn_decode_static_ws keeps its split-K scratch in a fixed
array inside the library.  This test calls it through the C ABI twice in a
row, on two different batches, and checks each result against the ordinary
entry point (which is given a torch-allocated workspace), within the parity
tolerance used everywhere else: |new - old| <= 2e-3 + 1e-2*|old|.

It sits in a file of its own, collected last, and needs no state from other
tests: it passes alone in a fresh process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


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
        old32, new32 = old.float(), new.float()
        assert torch.isfinite(old32).all() and torch.isfinite(new32).all()
        assert ((new32 - old32).abs() <= ATOL + RTOL * old32.abs()).all()


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
