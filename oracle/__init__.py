"""CPU oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, float64 restatement of what the paged-KV-cache
hot path computes.  It exists so that the CUDA library can be checked against
something obviously correct.  Only the test suite, the smoke check in
``__graft_entry__.smoke`` and the CPU-baseline leg of ``bench.py`` may import
it.  The library (``paged_kv_cache_394_b200``) never imports it, never calls
it, and has no CPU fallback of any kind; the two share no code.

Sources, cited by page title and section throughout:

* [csdn] devpress.csdn.net, "vLLM镜像深度优化：PagedAttention助力大模型推理效率飞跃"
* [cortexgrid] aidocs.cortexgrid.cn/docs/0a2c4066ef83, vLLM explainer with an FAQ
* [betteryeah] betteryeah.com, "vLLM是什么？完整解析高性能LLM推理引擎的技术原理与部署实践"

Modules:

* ``attention``      paged decode attention (direct and partitioned forms) and
                     chunked-prefill attention
* ``cache_ops``      the cache-write scatter and the copy-on-write block copy
* ``block_manager``  the page allocator: free list, refcounts, sharing, CoW,
                     prefix caching
* ``dtypes``         exact widening of fp16/bf16 bit patterns to float64
* ``fp8``            the E4M3 cache: encode / decode, the quantising write,
                     decode and prefill over dequantised codes
"""

from . import attention, block_manager, cache_ops, dtypes, fp8  # noqa: F401
