"""Failure detection on the GPU without a fault: a decode kernel's bounded
wait for its own loads runs out, the kernel reports PKV_DEVERR_TIMEOUT and
returns, and the CUDA context stays usable.

The wait is made to run out on purpose through the library's testing hook
(pkv_testing_decode_wait): the first CTA withholds its first load, so one
warp waits on a barrier that nothing completes.  The wait is bounded by 1 ms
here; the warp then drains its other loads (bounded by 2 s, the one that was
never issued takes all of it) and the kernel finishes.  A normal decode
afterwards must run clean and match the oracle."""

import pytest
import torch

from paged_kv_cache_394_b200 import workloads as W
from support import DeviceWorkload, assert_close, dev_to_bits, oracle_caches, oracle_decode, run_step

pytestmark = pytest.mark.gpu

DEFAULT_WAIT_NS = 2_000_000_000


# G = 1 runs the CUDA-core kernel, G = 4 the tensor-core kernel; each single
# pass (one 1024-token partition) and split-K (64-token partitions)
@pytest.mark.parametrize("heads,kv_heads,part", [(4, 4, 1024), (4, 4, 64), (8, 2, 1024),
                                                 (8, 2, 64)])
def test_wait_that_runs_out_reports_timeout(heads, kv_heads, part):
    from paged_kv_cache_394_b200 import pagedkv as pk
    w = W.build_decode_workload([300, 45, 129, 700], heads, kv_heads, 128, 16, "fp16", 41)
    dw = DeviceWorkload(w)
    try:
        pk.testing_decode_wait(1_000_000, True)
        run_step(pk, dw, partition_size=part)
        torch.cuda.synchronize()
    finally:
        pk.testing_decode_wait(DEFAULT_WAIT_NS, False)
    assert int(dw.err.item()) & pk.DEVERR_TIMEOUT
    # the context is intact: the same step again runs clean and is right
    dw2 = DeviceWorkload(w)
    assert run_step(pk, dw2, partition_size=part) == 0
    kc, vc = oracle_caches(w)
    assert_close(dev_to_bits(dw2.out), oracle_decode(w, kc, vc), w)

