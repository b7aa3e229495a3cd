"""The continuous-batching driver, replayed step by step through the oracle.

Every step's decisions (admissions, forks, frees) are mirrored in the oracle
block manager, which must produce the same slots and copy-on-write pairs; the
oracle cache ops apply the same host-drawn inputs; the oracle's prefill and
decode outputs must match the GPU's within 2e-3 + 1e-2*|ref|; at the end the
two pools are identical bit for bit and every block is free again.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import ATOL, RTOL

pytestmark = pytest.mark.gpu


def close(got_t, ref):
    from oracle.dtypes import widen
    got = widen(got_t.view(torch.int16).cpu().numpy().view(np.uint16), "fp16")
    assert np.isfinite(got).all()
    assert (np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)).all()


def test_continuous_batching_matches_oracle_replay():
    from oracle import attention as OA
    from oracle import cache_ops as OC
    from oracle.block_manager import BlockManager
    from paged_kv_cache_394_b200 import engine as E

    bs, h, hkv, d, nb = 16, 4, 2, 64, 96
    rng = np.random.default_rng(3)
    order = rng.permutation(nb)
    draws = {}

    def values(kind, shape):
        bits = W._normal_bits(rng, shape, "fp16")
        draws[kind] = bits
        return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.float16)

    b = E.ContinuousBatcher(nb, bs, h, hkv, d, max_num_seqs=6, max_num_batched_tokens=160,
                            max_model_len=256, free_order=order, values=values)
    trace = E.synthetic_trace(5, 10, mean_interarrival=1.0, prompt_median=40,
                              output_range=(2, 8), max_prompt=100)
    trace[3].samples = 3
    trace[7].samples = 2
    for r in trace:
        b.submit(r)
    ref = BlockManager(nb, bs, free_order=order)
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    steps = cows = decoded = 0
    while not b.idle():
        draws.clear()
        rec = b.step()
        steps += 1
        slots = []
        for sid, plen in rec.admitted:
            ref.add_seq(sid, plen)
            row = ref.seq_blocks(sid)
            slots += [row[t // bs] * bs + t % bs for t in range(plen)]
        pairs = []
        for sid in rec.decoded:
            slot, a, c = ref.append_slot(sid)
            slots.append(slot)
            if a >= 0:
                pairs.append((a, c))
        assert slots == list(rec.slots)
        assert pairs == [tuple(x) for x in rec.cow_pairs]
        cows += len(pairs)
        if pairs:
            OC.copy_blocks(kc, vc, np.array(pairs), inplace=True)
        if slots:
            OC.reshape_and_cache(draws["key"], draws["value"], kc, vc, np.array(slots), bs,
                                 inplace=True)
        if rec.admitted:
            ids = [sid for sid, _ in rec.admitted]
            lens = np.array([pl for _, pl in rec.admitted])
            tables = np.array(ref.block_table(ids, b.max_blocks), dtype=np.int32)
            qs = np.concatenate([[0], np.cumsum(lens)])
            close(b.last_outputs["prefill"][2],
                  OA.paged_attention_prefill(draws["q_prefill"], kc, vc, tables, lens, qs,
                                             b.scale, hkv, bs, "fp16"))
        if rec.decoded:
            decoded += len(rec.decoded)
            tables = np.array(ref.block_table(rec.decoded, b.max_blocks), dtype=np.int32)
            lens = np.array([ref.seq_len(s) for s in rec.decoded])
            close(b.last_outputs["decode"][2],
                  OA.paged_attention_decode(draws["q_decode"], kc, vc, tables, lens, b.scale,
                                            hkv, bs, "fp16"))
        for sid in rec.finished:
            ref.free_seq(sid)
        for parent, child in rec.forked:
            ref.fork(parent, child)
        assert b.alloc.num_free() == ref.num_free()
    assert cows >= 3 and decoded > 0 and steps > 5
    assert b.alloc.num_free() == nb and ref.num_free() == nb
    assert np.array_equal(b.k_cache.view(torch.int16).cpu().numpy().view(np.uint16), kc)
    assert np.array_equal(b.v_cache.view(torch.int16).cpu().numpy().view(np.uint16), vc)
