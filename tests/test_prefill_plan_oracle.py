"""The planned prefill's decomposition, checked in float64 on the CPU: for
every unit pkv_prefill_plan cuts, the oracle's partial summaries over the
pieces' key ranges, merged by the oracle's partition combine, equal the
oracle's causal prefill row for row (the pieces cover each row's visible keys
exactly once, and no history piece holds a key a row may not see)."""

import numpy as np
import pytest

from oracle import attention as OA
from oracle import cache_ops as OC
from oracle.dtypes import widen
from paged_kv_cache_394_b200 import workloads as W

ROWS = 256   # (token, head) rows of a planned unit: two query tiles of 128


@pytest.mark.parametrize("hist,new,h,hkv,bs", [([700, 5, 300], [40, 17, 64], 8, 2, 16),
                                               ([1000, 0], [9, 70], 4, 4, 32),
                                               ([2000], [3], 8, 1, 16)])
def test_plan_pieces_recombine_to_the_prefill(hist, new, h, hkv, bs):
    from paged_kv_cache_394_b200 import pagedkv as pk
    w = W.build_prefill_workload(hist, new, h, hkv, 128, bs, "fp16", seed=sum(hist) % 89)
    plan = pk.prefill_plan(w.query_start, w.context_lens, h, hkv, 128, 1000)
    work = plan.work.numpy()
    assert len(plan.merges) > 0
    # the step's cache write first: the new tokens' K/V join the pool
    kc, vc, bad = OC.reshape_and_cache(w.key, w.value, w.k_cache, w.v_cache, w.slot_mapping, bs)
    assert not bad
    ref = OA.paged_attention_prefill(w.q, kc, vc, w.block_tables, w.context_lens,
                                     w.query_start, w.scale, hkv, bs, w.dtype)
    assert np.isfinite(ref).all()
    g_size = h // hkv
    checked = 0
    for merge in range(len(plan.merges)):
        its = sorted((it for it in work if it[6] > 1 and it[5] == merge), key=lambda it: it[4])
        s, tile = int(its[0][0]), int(its[0][1])
        q0 = int(w.query_start[s])
        q_len = int(w.query_start[s + 1]) - q0
        c = int(w.context_lens[s])
        for kvh in range(hkv):
            keys = OA.gather_kv(kc, w.block_tables[s], c, kvh, bs, w.dtype)
            vals = OA.gather_kv(vc, w.block_tables[s], c, kvh, bs, w.dtype)
            for row in range(tile * ROWS, min(q_len * g_size, (tile + 1) * ROWS)):
                j, g = divmod(row, g_size)
                pos = c - q_len + j
                head = kvh * g_size + g
                qvec = widen(w.q[q0 + j, head], w.dtype)
                parts = []
                for it in its:
                    kb = int(it[2])
                    ke = pos + 1 if it[3] < 0 else int(it[3])
                    assert ke <= pos + 1          # a history piece is visible to every row
                    parts.append(OA.partition_summary(qvec, keys[kb:ke], vals[kb:ke], w.scale))
                got = OA.combine_partitions(parts)
                np.testing.assert_allclose(got, ref[q0 + j, head], rtol=1e-12, atol=1e-12)
                checked += 1
    assert checked > 0
