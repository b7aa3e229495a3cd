"""A whole decode step captured in a CUDA graph and replayed: the entry
points enqueue work only on the caller's stream and allocate nothing (the
allocation-free decode keeps its split-K scratch in the library), so the
captured step replays with new inputs and still matches the oracle."""

import numpy as np
import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import DeviceWorkload, assert_close, bits_to_dev, dev_to_bits, oracle_caches, oracle_decode

pytestmark = pytest.mark.gpu


def test_decode_step_replays_from_a_cuda_graph():
    from paged_kv_cache_394_b200 import pagedkv as pk
    w = W.build_decode_workload([5, 17, 300, 900, 33, 64], 8, 2, 128, 16, "bf16", 31)
    dw = DeviceWorkload(w)
    stream = torch.cuda.Stream()
    part = 256   # forces split-K: partition kernel + reduce inside the graph

    def step():
        pk.reshape_and_cache(dw.key, dw.value, dw.k_cache, dw.v_cache, dw.slots, dev_err=dw.err,
                             stream=stream)
        pk.paged_attn_decode_static_ws(dw.out, dw.q, dw.k_cache, dw.v_cache, dw.tables, dw.lens,
                                       w.scale, w.num_kv_heads, w.block_size, w.max_context_len,
                                       partition_size=part, dev_err=dw.err, stream=stream)
    with torch.cuda.stream(stream):
        step()                     # first call outside capture (caches the scratch address)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    # new queries, replayed through the captured graph
    rng = np.random.default_rng(5)
    for _ in range(2):
        new_q = W._normal_bits(rng, w.q.shape, w.dtype)
        dw.q.copy_(bits_to_dev(new_q, w))
        g.replay()
        torch.cuda.synchronize()
        w.q = new_q
        kc, vc = oracle_caches(w)
        assert_close(dev_to_bits(dw.out), oracle_decode(w, kc, vc), w)
    assert int(dw.err.item()) == 0
