"""B200-native paged KV cache: PagedAttention decode, cache-write scatter,
copy-on-write block copy and a host block allocator.

The compute runs in hand-written CUDA kernels for sm_100a behind the C ABI of
``libpagedkv.so`` (declared in ``include/pagedkv.h``).  ``pagedkv`` is the thin
ctypes binding over it; importing it loads the library and raises if the
library is missing.  ``workloads`` draws seeded synthetic inputs.

Submodules are imported lazily so that drawing inputs does not require the
compiled library.
"""

__all__ = ["pagedkv", "workloads"]
