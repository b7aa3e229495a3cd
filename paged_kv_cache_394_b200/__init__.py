"""B200-native paged KV cache: PagedAttention decode, cache-write scatter,
copy-on-write block copy and a host block allocator with prefix caching; also
chunked-prefill attention, cascade decode over shared prefixes, an 8-bit
(E4M3) cache and a continuous-batching step driver.

The compute runs in hand-written CUDA kernels for sm_100a behind the C ABI of
``libpagedkv.so`` (declared in ``include/pagedkv.h``).  ``pagedkv`` is the thin
ctypes binding over it; importing it loads the library and raises if the
library is missing.  ``workloads`` draws seeded synthetic inputs; ``engine``
drives iteration-level batching through the binding.

Submodules are imported lazily so that drawing inputs does not require the
compiled library.
"""

__all__ = ["pagedkv", "workloads", "engine"]
