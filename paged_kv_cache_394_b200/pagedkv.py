"""Thin ctypes binding of ``libpagedkv.so`` (declared in include/pagedkv.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Device tensors are torch tensors (torch supplies device memory
and streams); their pointers, shapes and the current CUDA stream are passed
through the C ABI.  Importing this module loads the library and raises
``ImportError`` if it has not been built — there is no fallback.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libpagedkv.so is not built (run `python -m paged_kv_cache_394_b200.build`)")
_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_OUT_OF_BLOCKS = range(6)
FP16, BF16, FP8_E4M3 = 0, 1, 2
(DEVERR_BAD_BLOCK, DEVERR_BAD_SLOT, DEVERR_BAD_PAIR, DEVERR_BAD_CONTEXT, DEVERR_TIMEOUT,
 DEVERR_BAD_SCALE, DEVERR_BAD_ORDER) = (1, 2, 4, 8, 16, 32, 64)

_vp, _i, _i64, _f, _sz, _u = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_size_t, ctypes.c_uint)


def _proto(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_lib_version = _proto("pkv_version", ctypes.c_char_p)
_status_string = _proto("pkv_status_string", ctypes.c_char_p, _i)
_last_cuda_error = _proto("pkv_last_cuda_error", _i)
_reshape_and_cache = _proto("pkv_reshape_and_cache", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                            _i, _i, _vp, _vp)
_copy_blocks = _proto("pkv_copy_blocks", _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp)
_partition_size = _proto("pkv_paged_attn_partition_size", _i, _i, _i, _i, _i, _i)
_partition_size_fp8 = _proto("pkv_paged_attn_partition_size_fp8", _i, _i, _i, _i, _i, _i)
_workspace_bytes = _proto("pkv_paged_attn_workspace_bytes", _sz, _i, _i, _i, _i, _i, _i, _i)
_paged_attn_decode = _proto("pkv_paged_attn_decode", _i, _vp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i,
                            _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp)
_paged_attn_decode_static_ws = _proto("pkv_paged_attn_decode_static_ws", _i, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                     _vp)
STATIC_WORKSPACE_BYTES = 16 << 20
_cascade_workspace_bytes = _proto("pkv_paged_attn_cascade_workspace_bytes", _sz, _i, _i, _i, _i,
                                  _i, _i, _i)
_paged_attn_decode_cascade = _proto("pkv_paged_attn_decode_cascade", _i, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _i, _i, _vp, _sz, _vp, _vp)
_paged_attn_decode_cascade_fp8 = _proto("pkv_paged_attn_decode_cascade_fp8", _i, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i,
                                        _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp)
_reshape_and_cache_fp8 = _proto("pkv_reshape_and_cache_fp8", _i, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                _i, _i, _i, _i, _vp, _vp, _vp, _vp)
_paged_attn_decode_fp8 = _proto("pkv_paged_attn_decode_fp8", _i, _vp, _vp, _vp, _vp, _vp, _vp, _f,
                                _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp,
                                _vp)
_paged_attn_prefill = _proto("pkv_paged_attn_prefill", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _f, _i,
                             _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp)
_paged_attn_prefill_fp8 = _proto("pkv_paged_attn_prefill_fp8", _i, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _f, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                 _vp, _vp)
_staging_bytes = _proto("pkv_decode_step_staging_bytes", _sz, _i, _i, _i, _i, _i, _i, _i)
_decode_step_host = _proto("pkv_decode_step_host", _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp,
                           _vp, _vp, _vp, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz,
                           _vp, _sz, _vp, _vp)
_decode_order = _proto("pkv_decode_order", _i, _vp, _i, _vp)
_paged_attn_decode_ordered = _proto("pkv_paged_attn_decode_ordered", _i, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz,
                                    _vp, _vp)
_paged_attn_decode_fp8_ordered = _proto("pkv_paged_attn_decode_fp8_ordered", _i, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp, _f, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                        _i, _i, _i, _i, _vp, _sz, _vp, _vp)
_decode_plan = _proto("pkv_decode_plan", _i, _vp, _i, _i, _i, _vp, _i, _vp)
_paged_attn_decode_planned = _proto("pkv_paged_attn_decode_planned", _i, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _i, _f, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                    _sz, _vp, _vp)
_paged_attn_decode_fp8_planned = _proto("pkv_paged_attn_decode_fp8_planned", _i, _vp, _vp, _vp,
                                        _vp, _vp, _vp, _vp, _i, _f, _vp, _vp, _i, _i, _i, _i, _i,
                                        _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp)
_prefill_plan = _proto("pkv_prefill_plan", _i, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp,
                       _i, _vp, _vp)
_paged_attn_prefill_planned = _proto("pkv_paged_attn_prefill_planned", _i, _vp, _vp, _vp, _vp,
                                     _vp, _vp, _vp, _vp, _i, _vp, _i, _f, _i, _i, _i, _i, _i, _i,
                                     _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp)
_paged_attn_prefill_fp8_planned = _proto("pkv_paged_attn_prefill_fp8_planned", _i, _vp, _vp, _vp,
                                         _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _f, _vp, _vp, _i,
                                         _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp,
                                         _vp)
_testing_decode_wait = _proto("pkv_testing_decode_wait", _i, ctypes.c_uint64, _i)
_pipeline_staging_bytes = _proto("pkv_decode_pipeline_staging_bytes", _sz, _i, _i, _i, _i, _i, _i,
                                 _i)
_pipeline_create = _proto("pkv_decode_pipeline_create", _i, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                          _vp, _sz, _vp)
_pipeline_step = _proto("pkv_decode_pipeline_step", _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i,
                        _vp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _sz, _vp)
_pipeline_join = _proto("pkv_decode_pipeline_join", _i, _vp, _vp)
_pipeline_sync = _proto("pkv_decode_pipeline_sync", _i, _vp)
_pipeline_destroy = _proto("pkv_decode_pipeline_destroy", None, _vp)
_alloc_create = _proto("pkv_alloc_create", _vp, _i, _i, _vp)
_alloc_destroy = _proto("pkv_alloc_destroy", None, _vp)
_alloc_add_seq = _proto("pkv_alloc_add_seq", _i, _vp, _i64, _i64)
_alloc_fork = _proto("pkv_alloc_fork", _i, _vp, _i64, _i64)
_alloc_append_slot = _proto("pkv_alloc_append_slot", _i, _vp, _i64, _vp, _vp, _vp)
_alloc_append_slots = _proto("pkv_alloc_append_slots", _i, _vp, _vp, _i, _vp, _vp, _vp, _vp)
_alloc_free_seq = _proto("pkv_alloc_free_seq", _i, _vp, _i64)
_alloc_block_table = _proto("pkv_alloc_block_table", _i, _vp, _vp, _i, _i, _vp)
_alloc_context_lens = _proto("pkv_alloc_context_lens", _i, _vp, _vp, _i, _vp)
_alloc_num_free = _proto("pkv_alloc_num_free", _i, _vp)
_alloc_refcount = _proto("pkv_alloc_refcount", _i, _vp, _i)
_alloc_seq_len = _proto("pkv_alloc_seq_len", _i64, _vp, _i64)
_alloc_seq_num_blocks = _proto("pkv_alloc_seq_num_blocks", _i, _vp, _i64)
_alloc_usage = _proto("pkv_alloc_usage", _i, _vp, _vp, _vp)
_alloc_add_seq_cached = _proto("pkv_alloc_add_seq_cached", _i, _vp, _i64, _vp, _i64, _vp)
_alloc_cache_stats = _proto("pkv_alloc_cache_stats", _i, _vp, _vp, _vp, _vp, _vp)
_alloc_num_evictable = _proto("pkv_alloc_num_evictable", _i, _vp)


class PagedKVError(RuntimeError):
    def __init__(self, status, where):
        msg = "%s: %s" % (where, _status_string(status).decode())
        if status == ERR_CUDA:
            msg += " (cudaError %d)" % _last_cuda_error()
        super().__init__(msg)
        self.status = status


def _check(status, where):
    if status != OK:
        raise PagedKVError(status, where)


def version():
    return _lib_version().decode()


def library_path():
    return LIB_PATH


def _dtype_code(t):
    if t.dtype == torch.float16:
        return FP16
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("expected float16 or bfloat16, got %s" % t.dtype)


def _cache_dtype_code(t):
    """Element type of a cache: 16-bit, or E4M3 codes held as uint8 / float8_e4m3fn."""
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return FP8_E4M3
    return _dtype_code(t)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name, dtype=None):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, dev_err=None, stream=None):
    """Write the new tokens' K/V ([T, Hkv, D]) into their slots of the caches."""
    for n, t in (("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    num_blocks, hkv, bs, d = k_cache.shape
    t = key.shape[0]
    if key.shape != (t, hkv, d) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if slot_mapping.shape != (t,):
        raise ValueError("slot_mapping must be [num_tokens]")
    _check(_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                              _ptr(slot_mapping), t, hkv, d, bs, num_blocks,
                              _dtype_code(k_cache), _ptr(dev_err), _stream(stream)),
           "reshape_and_cache")


def copy_blocks(k_cache, v_cache, block_mapping, dev_err=None, stream=None):
    """Copy whole blocks (K and V) for each (src, dst) row of block_mapping [P, 2]."""
    _dev(k_cache, "k_cache")
    _dev(v_cache, "v_cache")
    _dev(block_mapping, "block_mapping", torch.int64)
    num_blocks, hkv, bs, d = k_cache.shape
    p = block_mapping.shape[0] if block_mapping.numel() else 0
    if block_mapping.numel() and block_mapping.shape != (p, 2):
        raise ValueError("block_mapping must be [num_pairs, 2]")
    if v_cache.dtype != k_cache.dtype or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must match")
    _check(_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), p, hkv, d, bs,
                        num_blocks, _cache_dtype_code(k_cache), _ptr(dev_err), _stream(stream)),
           "copy_blocks")


def partition_size(num_seqs, num_kv_heads, block_size, max_context_len, requested=0):
    return _partition_size(num_seqs, num_kv_heads, block_size, max_context_len, requested)


def partition_size_fp8(num_seqs, num_kv_heads, block_size, max_context_len, requested=0):
    """The partition paged_attn_decode_fp8 uses (E4M3 caches)."""
    return _partition_size_fp8(num_seqs, num_kv_heads, block_size, max_context_len, requested)


def workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                    partition_size=0):
    return _workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_context_len, partition_size)


def alloc_workspace(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                    partition_size=0, device=None):
    n = workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                        max_context_len, partition_size)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def decode_order(context_lens):
    """Longest-first sequence order (int32 host tensor) for a host tensor or
    array of context lengths; see pkv_decode_order."""
    lens = torch.as_tensor(context_lens, dtype=torch.int32).contiguous()
    if lens.is_cuda:
        raise ValueError("context_lens must be on the host")
    order = torch.empty_like(lens)
    _check(_decode_order(_ptr(lens), lens.numel(), _ptr(order)), "decode_order")
    return order


def decode_plan(context_lens, block_size, partition_size):
    """Work list (int32 host tensor [items, 2]) of the (sequence, partition)
    items a decode with this partition size has, longest first, for a host
    tensor or array of context lengths; see pkv_decode_plan."""
    lens = torch.as_tensor(context_lens, dtype=torch.int32).contiguous()
    if lens.is_cuda:
        raise ValueError("context_lens must be on the host")
    n = ctypes.c_int(0)
    _check(_decode_plan(_ptr(lens), lens.numel(), block_size, partition_size, None, 0,
                        ctypes.byref(n)), "decode_plan")
    work = torch.empty((n.value, 2), dtype=torch.int32)
    _check(_decode_plan(_ptr(lens), lens.numel(), block_size, partition_size, _ptr(work),
                        n.value, ctypes.byref(n)), "decode_plan")
    return work


def _work_arg(work, partition_size):
    _dev(work, "work", torch.int32)
    if work.dim() != 2 or work.shape[1] != 2 or not work.is_contiguous():
        raise ValueError("work must be a contiguous [items, 2] list from decode_plan")
    if partition_size <= 0:
        raise ValueError("a planned decode takes the partition size it was planned with")
    return work.shape[0]


def paged_attn_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                      block_size, max_context_len, partition_size=0, workspace=None,
                      dev_err=None, stream=None, seq_order=None, work=None):
    """Paged decode attention; writes out [S, H, D].  With ``seq_order`` (a
    device int32 permutation, e.g. decode_order's) the CTAs take the
    sequences in that order; with ``work`` (the device copy of decode_plan's
    list for ``partition_size``) one CTA per item and kv head.  See
    include/pagedkv.h."""
    if work is not None and seq_order is not None:
        raise ValueError("give seq_order or work, not both")
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    s, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if q.dtype != k_cache.dtype or out.dtype != q.dtype:
        raise TypeError("q, out and caches must share a dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    if workspace is None:
        need = workspace_bytes(s, h, hkv, d, bs, max_context_len, partition_size)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if need else None
        if workspace is not None and stream is not None:
            workspace.record_stream(stream)   # the temporary must outlive the launch
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if work is not None:
        n = _work_arg(work, partition_size)
        _check(_paged_attn_decode_planned(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(block_tables), _ptr(context_lens), _ptr(work), n,
                                          float(scale), s, h, hkv, d, bs, block_tables.shape[1],
                                          max_context_len, num_blocks, _dtype_code(q),
                                          partition_size, ws_ptr, ws_bytes, _ptr(dev_err),
                                          _stream(stream)),
               "paged_attn_decode_planned")
        return
    if seq_order is not None:
        _dev(seq_order, "seq_order", torch.int32)
        if seq_order.shape != (s,):
            raise ValueError("seq_order must be [S]")
        _check(_paged_attn_decode_ordered(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(block_tables), _ptr(context_lens), _ptr(seq_order),
                                          float(scale), s, h, hkv, d, bs, block_tables.shape[1],
                                          max_context_len, num_blocks, _dtype_code(q),
                                          partition_size, ws_ptr, ws_bytes, _ptr(dev_err),
                                          _stream(stream)),
               "paged_attn_decode_ordered")
        return
    _check(_paged_attn_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                              _ptr(block_tables), _ptr(context_lens), float(scale), s, h, hkv, d,
                              bs, block_tables.shape[1], max_context_len, num_blocks,
                              _dtype_code(q), partition_size, ws_ptr, ws_bytes, _ptr(dev_err),
                              _stream(stream)),
           "paged_attn_decode")


def fp8_scales(scales, num_kv_heads, device=None):
    """Per-kv-head E4M3 scales as the float32 device tensor [num_kv_heads] the
    library reads: a number is repeated, a tensor is checked and returned."""
    if isinstance(scales, torch.Tensor):
        _dev(scales, "scales", torch.float32)
        if scales.shape != (num_kv_heads,):
            raise ValueError("scales must be [num_kv_heads]")
        return scales
    return torch.full((num_kv_heads,), float(scales), dtype=torch.float32,
                      device=device or "cuda")


def _scales_for(k_scales, v_scales, hkv, device, stream):
    ks, vs = fp8_scales(k_scales, hkv, device), fp8_scales(v_scales, hkv, device)
    if stream is not None:   # a temporary must outlive the launch on that stream
        ks.record_stream(stream)
        vs.record_stream(stream)
    return ks, vs


def cascade_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                            max_context_len, partition_size=0):
    return _cascade_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    max_context_len, partition_size)


def paged_attn_decode_cascade(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                              shared_blocks, scale, num_kv_heads, block_size, max_context_len,
                              max_group_size, max_shared_blocks, partition_size=0,
                              workspace=None, dev_err=None, stream=None, k_scales=None,
                              v_scales=None):
    """Decode for groups of sequences sharing their first shared_blocks[g]
    blocks (members consecutive, group g = group_start[g] .. group_start[g+1]-1).
    Same result as paged_attn_decode; with E4M3 caches (uint8 codes and
    k_scales / v_scales given) as paged_attn_decode_fp8.  See include/pagedkv.h."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    for n, t in (("block_tables", block_tables), ("context_lens", context_lens),
                 ("group_start", group_start), ("shared_blocks", shared_blocks)):
        _dev(t, n, torch.int32)
    s, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    fp8 = _cache_dtype_code(k_cache) == FP8_E4M3
    if fp8 != (k_scales is not None) or (k_scales is None) != (v_scales is None):
        raise TypeError("E4M3 caches take k_scales and v_scales; 16-bit caches take neither")
    if (v_cache.dtype != k_cache.dtype or out.dtype != q.dtype
            or (not fp8 and q.dtype != k_cache.dtype)):
        raise TypeError("q, out and caches must share a dtype (E4M3 caches: uint8 codes)")
    g = shared_blocks.shape[0]
    if group_start.shape != (g + 1,):
        raise ValueError("group_start must be [num_groups + 1]")
    if workspace is None:
        need = cascade_workspace_bytes(s, h, hkv, d, bs, max_context_len, partition_size)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        if stream is not None:
            workspace.record_stream(stream)   # the temporary must outlive the launch
    ws_bytes = workspace.numel() * workspace.element_size()
    if fp8:
        ks, vs = _scales_for(k_scales, v_scales, hkv, q.device, stream)
        _check(_paged_attn_decode_cascade_fp8(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            _ptr(context_lens), _ptr(group_start), _ptr(shared_blocks), float(scale), _ptr(ks),
            _ptr(vs), s, g, max_group_size, max_shared_blocks, h, hkv, d, bs,
            block_tables.shape[1], max_context_len, num_blocks, _dtype_code(q), partition_size,
            _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream)),
            "paged_attn_decode_cascade_fp8")
        return
    _check(_paged_attn_decode_cascade(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(block_tables), _ptr(context_lens), _ptr(group_start),
                                      _ptr(shared_blocks), float(scale), s, g, max_group_size,
                                      max_shared_blocks, h, hkv, d, bs, block_tables.shape[1],
                                      max_context_len, num_blocks, _dtype_code(q), partition_size,
                                      _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream)),
           "paged_attn_decode_cascade")


def reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scales, v_scales,
                          dev_err=None, stream=None):
    """Quantise the new tokens' K/V ([T, Hkv, D], 16-bit) to E4M3 codes of
    x / scale[h] and write them into their slots of the uint8 caches.
    ``k_scales`` / ``v_scales``: float32 device tensors [Hkv] (see fp8_scales)."""
    for n, t in (("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    if _cache_dtype_code(k_cache) != FP8_E4M3 or v_cache.dtype != k_cache.dtype:
        raise TypeError("E4M3 caches must be uint8 (or float8_e4m3fn)")
    num_blocks, hkv, bs, d = k_cache.shape
    t = key.shape[0]
    if key.shape != (t, hkv, d) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if value.dtype != key.dtype:
        raise TypeError("key and value must share a dtype")
    if slot_mapping.shape != (t,):
        raise ValueError("slot_mapping must be [num_tokens]")
    ks, vs = _scales_for(k_scales, v_scales, hkv, key.device, stream)
    _check(_reshape_and_cache_fp8(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(slot_mapping), t, hkv, d, bs, num_blocks, _dtype_code(key),
                                  _ptr(ks), _ptr(vs), _ptr(dev_err), _stream(stream)),
           "reshape_and_cache_fp8")


def paged_attn_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale, k_scales,
                          v_scales, num_kv_heads, block_size, max_context_len, partition_size=0,
                          workspace=None, dev_err=None, stream=None, seq_order=None, work=None):
    """Paged decode attention over E4M3 caches (values = code * scale of the
    kv head); q and out are 16-bit.  ``seq_order`` and ``work`` as for
    paged_attn_decode.  See include/pagedkv.h."""
    if work is not None and seq_order is not None:
        raise ValueError("give seq_order or work, not both")
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    s, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if _cache_dtype_code(k_cache) != FP8_E4M3 or v_cache.dtype != k_cache.dtype:
        raise TypeError("E4M3 caches must be uint8 (or float8_e4m3fn)")
    if out.dtype != q.dtype:
        raise TypeError("q and out must share a dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    if workspace is None:
        need = workspace_bytes(s, h, hkv, d, bs, max_context_len, partition_size)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device) if need else None
        if workspace is not None and stream is not None:
            workspace.record_stream(stream)   # the temporary must outlive the launch
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ks, vs = _scales_for(k_scales, v_scales, hkv, q.device, stream)
    if work is not None:
        n = _work_arg(work, partition_size)
        _check(_paged_attn_decode_fp8_planned(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                              _ptr(block_tables), _ptr(context_lens), _ptr(work),
                                              n, float(scale), _ptr(ks), _ptr(vs), s, h, hkv, d,
                                              bs, block_tables.shape[1], max_context_len,
                                              num_blocks, _dtype_code(q), partition_size, ws_ptr,
                                              ws_bytes, _ptr(dev_err), _stream(stream)),
               "paged_attn_decode_fp8_planned")
        return
    if seq_order is not None:
        _dev(seq_order, "seq_order", torch.int32)
        if seq_order.shape != (s,):
            raise ValueError("seq_order must be [S]")
        _check(_paged_attn_decode_fp8_ordered(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                              _ptr(block_tables), _ptr(context_lens),
                                              _ptr(seq_order), float(scale), _ptr(ks), _ptr(vs),
                                              s, h, hkv, d, bs, block_tables.shape[1],
                                              max_context_len, num_blocks, _dtype_code(q),
                                              partition_size, ws_ptr, ws_bytes, _ptr(dev_err),
                                              _stream(stream)),
               "paged_attn_decode_fp8_ordered")
        return
    _check(_paged_attn_decode_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(block_tables), _ptr(context_lens), float(scale),
                                  _ptr(ks), _ptr(vs), s, h, hkv, d, bs,
                                  block_tables.shape[1], max_context_len, num_blocks,
                                  _dtype_code(q), partition_size, ws_ptr, ws_bytes,
                                  _ptr(dev_err), _stream(stream)),
           "paged_attn_decode_fp8")


def paged_attn_decode_static_ws(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                num_kv_heads, block_size, max_context_len, partition_size=0,
                                dev_err=None, stream=None):
    """paged_attn_decode with its split-K scratch in the library's fixed device
    array (no allocation anywhere).  For callers that cannot allocate device
    memory; see include/pagedkv.h for the size limit and the sharing rules."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    s, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if q.dtype != k_cache.dtype or out.dtype != q.dtype:
        raise TypeError("q, out and caches must share a dtype")
    _check(_paged_attn_decode_static_ws(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_tables), _ptr(context_lens), float(scale), s,
                                        h, hkv, d, bs, block_tables.shape[1], max_context_len,
                                        num_blocks, _dtype_code(q), partition_size,
                                        _ptr(dev_err), _stream(stream)),
           "paged_attn_decode_static_ws")


class PrefillPlan:
    """A planned prefill's work list (pkv_prefill_plan): ``work`` [items, 8] and
    ``merges`` [entries, 4] int32 host tensors, ``workspace_bytes``."""

    def __init__(self, work, merges, workspace_bytes):
        self.work, self.merges, self.workspace_bytes = work, merges, workspace_bytes

    def to(self, device):
        """The lists on the device, for paged_attn_prefill(plan=...)."""
        return PrefillPlan(self.work.to(device), self.merges.to(device), self.workspace_bytes)


def prefill_plan(query_start, context_lens, num_heads, num_kv_heads, head_dim=128, num_sms=148):
    """Plan a prefill from host lengths (query_start [S+1], context_lens [S]);
    see pkv_prefill_plan."""
    qs = torch.as_tensor(query_start, dtype=torch.int32).contiguous()
    lens = torch.as_tensor(context_lens, dtype=torch.int32).contiguous()
    if qs.is_cuda or lens.is_cuda:
        raise ValueError("query_start and context_lens must be on the host")
    s = lens.numel()
    if qs.numel() != s + 1:
        raise ValueError("query_start must be [S+1]")
    n, m, wb = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_size_t(0)
    args = (_ptr(qs), _ptr(lens), s, num_heads, num_kv_heads, head_dim, num_sms)
    _check(_prefill_plan(*args, None, 0, ctypes.byref(n), None, 0, ctypes.byref(m),
                         ctypes.byref(wb)), "prefill_plan")
    work = torch.zeros((n.value, 8), dtype=torch.int32)
    merges = torch.zeros((m.value, 4), dtype=torch.int32)
    _check(_prefill_plan(*args, _ptr(work), n.value, ctypes.byref(n), _ptr(merges), m.value,
                         ctypes.byref(m), ctypes.byref(wb)), "prefill_plan")
    return PrefillPlan(work, merges, wb.value)


def _plan_args(plan, workspace, device, stream):
    _dev(plan.work, "plan.work", torch.int32)
    _dev(plan.merges, "plan.merges", torch.int32)
    if workspace is None and plan.workspace_bytes:
        workspace = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=device)
        if stream is not None:
            workspace.record_stream(stream)   # the temporary must outlive the launch
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return (_ptr(plan.work), plan.work.shape[0], _ptr(plan.merges) if plan.merges.numel() else None,
            plan.merges.shape[0]), (_ptr(workspace), nbytes, workspace)


def paged_attn_prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start, scale,
                       num_kv_heads, block_size, max_context_len, max_query_len, dev_err=None,
                       stream=None, plan=None, workspace=None):
    """Chunked-prefill attention; q/out are [T, H, D], query_start [S+1].  With
    ``plan`` (prefill_plan(...).to(device)) the planned prefill, with its
    partials in ``workspace`` (allocated if None).  See include/pagedkv.h."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(query_start, "query_start", torch.int32)
    t, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    s = context_lens.shape[0]
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if query_start.shape != (s + 1,) or block_tables.shape[0] != s:
        raise ValueError("query_start must be [S+1], block_tables [S, max_blocks]")
    if q.dtype != k_cache.dtype or out.dtype != q.dtype:
        raise TypeError("q, out and caches must share a dtype")
    if plan is not None:
        pa, (ws_ptr, ws_bytes, _ws) = _plan_args(plan, workspace, q.device, stream)
        _check(_paged_attn_prefill_planned(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                           _ptr(block_tables), _ptr(context_lens),
                                           _ptr(query_start), *pa, float(scale), s, t, h, hkv, d,
                                           bs, block_tables.shape[1], max_context_len,
                                           max_query_len, num_blocks, _dtype_code(q), ws_ptr,
                                           ws_bytes, _ptr(dev_err), _stream(stream)),
               "paged_attn_prefill_planned")
        return
    _check(_paged_attn_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                               _ptr(block_tables), _ptr(context_lens), _ptr(query_start),
                               float(scale), s, t, h, hkv, d, bs, block_tables.shape[1],
                               max_context_len, max_query_len, num_blocks, _dtype_code(q),
                               _ptr(dev_err), _stream(stream)),
           "paged_attn_prefill")


def paged_attn_prefill_fp8(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                           scale, k_scales, v_scales, num_kv_heads, block_size, max_context_len,
                           max_query_len, dev_err=None, stream=None, plan=None, workspace=None):
    """Chunked-prefill attention over E4M3 caches (values = code * scale of the
    kv head); q and out are 16-bit.  ``plan`` and ``workspace`` as for
    paged_attn_prefill.  See include/pagedkv.h."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, n)
    _dev(block_tables, "block_tables", torch.int32)
    _dev(context_lens, "context_lens", torch.int32)
    _dev(query_start, "query_start", torch.int32)
    t, h, d = q.shape
    num_blocks, hkv, bs, dk = k_cache.shape
    s = context_lens.shape[0]
    if (hkv, bs, dk) != (num_kv_heads, block_size, d) or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if query_start.shape != (s + 1,) or block_tables.shape[0] != s:
        raise ValueError("query_start must be [S+1], block_tables [S, max_blocks]")
    if _cache_dtype_code(k_cache) != FP8_E4M3 or v_cache.dtype != k_cache.dtype:
        raise TypeError("E4M3 caches must be uint8 (or float8_e4m3fn)")
    if out.dtype != q.dtype:
        raise TypeError("q and out must share a dtype")
    ks, vs = _scales_for(k_scales, v_scales, hkv, q.device, stream)
    if plan is not None:
        pa, (ws_ptr, ws_bytes, _ws) = _plan_args(plan, workspace, q.device, stream)
        _check(_paged_attn_prefill_fp8_planned(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                               _ptr(block_tables), _ptr(context_lens),
                                               _ptr(query_start), *pa, float(scale), _ptr(ks),
                                               _ptr(vs), s, t, h, hkv, d, bs,
                                               block_tables.shape[1], max_context_len,
                                               max_query_len, num_blocks, _dtype_code(q), ws_ptr,
                                               ws_bytes, _ptr(dev_err), _stream(stream)),
               "paged_attn_prefill_fp8_planned")
        return
    _check(_paged_attn_prefill_fp8(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(block_tables), _ptr(context_lens), _ptr(query_start),
                                   float(scale), _ptr(ks), _ptr(vs), s, t, h, hkv, d, bs,
                                   block_tables.shape[1], max_context_len, max_query_len,
                                   num_blocks, _dtype_code(q), _ptr(dev_err), _stream(stream)),
           "paged_attn_prefill_fp8")


def testing_decode_wait(wait_ns, withhold_first_load=False):
    """Testing hook: the decode kernels' bound on a wait for their own loads,
    and whether the first CTA withholds its first load so that the wait runs
    out (see include/pagedkv.h).  Restore with (2_000_000_000, False)."""
    _check(_testing_decode_wait(int(wait_ns), 1 if withhold_first_load else 0),
           "testing_decode_wait")


def staging_bytes(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                  num_new_tokens, num_pairs):
    return _staging_bytes(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                          num_new_tokens, num_pairs)


def decode_step_host(out_host, q_host, key_host, value_host, slot_mapping_host,
                     block_mapping_host, block_tables_host, context_lens_host, k_cache, v_cache,
                     scale, max_context_len, staging, workspace=None, partition_size=0,
                     dev_err=None, stream=None):
    """One whole step from host tensors (pinned for async copies); see the header."""
    _dev(k_cache, "k_cache")
    _dev(v_cache, "v_cache")
    _dev(staging, "staging")
    for n, t in (("out_host", out_host), ("q_host", q_host), ("key_host", key_host),
                 ("value_host", value_host), ("slot_mapping_host", slot_mapping_host),
                 ("block_mapping_host", block_mapping_host),
                 ("block_tables_host", block_tables_host),
                 ("context_lens_host", context_lens_host)):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous host tensor" % n)
    s, h, d = q_host.shape
    num_blocks, hkv, bs, _ = k_cache.shape
    t = key_host.shape[0]
    p = block_mapping_host.shape[0] if block_mapping_host.numel() else 0
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_decode_step_host(_ptr(out_host), _ptr(q_host), _ptr(key_host), _ptr(value_host),
                             _ptr(slot_mapping_host), t, _ptr(block_mapping_host), p,
                             _ptr(block_tables_host), _ptr(context_lens_host), _ptr(k_cache),
                             _ptr(v_cache), float(scale), s, h, hkv, d, bs,
                             block_tables_host.shape[1], max_context_len, num_blocks,
                             _dtype_code(k_cache), partition_size, _ptr(staging),
                             staging.numel() * staging.element_size(), ws_ptr, ws_bytes,
                             _ptr(dev_err), _stream(stream)),
           "decode_step_host")


def _host(t, name):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous host tensor" % name)


class DecodePipeline:
    """Consecutive decode steps from host tensors, overlapped across an upload,
    a compute and a download stream (``pkv_decode_pipeline_*``; see the
    header).  ``staging`` is a device uint8 tensor of at least
    ``DecodePipeline.staging_bytes(...)`` bytes; ``stream`` the compute stream."""

    @staticmethod
    def staging_bytes(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                      max_new_tokens, max_pairs):
        return _pipeline_staging_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                       max_blocks_per_seq, max_new_tokens, max_pairs)

    def __init__(self, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                 max_blocks_per_seq, max_new_tokens, max_pairs, dtype, staging, stream=None):
        _dev(staging, "staging")
        self._staging = staging                 # kept alive with the pipeline
        self._stream = torch.cuda.current_stream() if stream is None else stream
        h = ctypes.c_void_p()
        _check(_pipeline_create(ctypes.byref(h), num_seqs, num_heads, num_kv_heads, head_dim,
                                block_size, max_blocks_per_seq, max_new_tokens, max_pairs,
                                _dtype_code(torch.empty(0, dtype=dtype)), _ptr(staging),
                                staging.numel() * staging.element_size(),
                                ctypes.c_void_p(self._stream.cuda_stream)),
               "decode_pipeline_create")
        self._h = h

    def step(self, out_host, q_host, key_host, value_host, slot_mapping_host, block_mapping_host,
             block_tables_host, context_lens_host, k_cache, v_cache, scale, max_context_len,
             workspace=None, partition_size=0, dev_err=None):
        for n, t in (("out_host", out_host), ("q_host", q_host), ("key_host", key_host),
                     ("value_host", value_host), ("slot_mapping_host", slot_mapping_host),
                     ("block_mapping_host", block_mapping_host),
                     ("block_tables_host", block_tables_host),
                     ("context_lens_host", context_lens_host)):
            _host(t, n)
        _dev(k_cache, "k_cache")
        _dev(v_cache, "v_cache")
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        p = block_mapping_host.shape[0] if block_mapping_host.numel() else 0
        _check(_pipeline_step(self._h, _ptr(out_host), _ptr(q_host), _ptr(key_host),
                              _ptr(value_host), _ptr(slot_mapping_host), key_host.shape[0],
                              _ptr(block_mapping_host), p, _ptr(block_tables_host),
                              _ptr(context_lens_host), _ptr(k_cache), _ptr(v_cache), float(scale),
                              max_context_len, k_cache.shape[0], partition_size, _ptr(workspace),
                              ws_bytes, _ptr(dev_err)),
               "decode_pipeline_step")

    def join(self, stream=None):
        _check(_pipeline_join(self._h, _stream(stream)), "decode_pipeline_join")

    def sync(self):
        _check(_pipeline_sync(self._h), "decode_pipeline_sync")

    def close(self):
        if self._h:
            _pipeline_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class BlockAllocator:
    """Host block allocator (free list, refcounts, fork, copy-on-write)."""

    def __init__(self, num_blocks, block_size, free_order=None):
        self._order = None
        if free_order is not None:
            self._order = (ctypes.c_int32 * num_blocks)(*[int(b) for b in free_order])
        self._h = _alloc_create(num_blocks, block_size, self._order)
        if not self._h:
            raise PagedKVError(ERR_INVALID_ARG, "BlockAllocator")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            _alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id, num_tokens):
        _check(_alloc_add_seq(self._h, seq_id, num_tokens), "add_seq")

    def fork(self, parent, child):
        _check(_alloc_fork(self._h, parent, child), "fork")

    def append_slot(self, seq_id):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_alloc_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                  ctypes.byref(dst)), "append_slot")
        return slot.value, src.value, dst.value

    def append_slots(self, seq_ids):
        n = len(seq_ids)
        ids = (ctypes.c_int64 * max(n, 1))(*seq_ids)
        slots = (ctypes.c_int64 * max(n, 1))()
        pairs = (ctypes.c_int64 * max(2 * n, 2))()
        ncow, done = ctypes.c_int(), ctypes.c_int()
        _check(_alloc_append_slots(self._h, ids, n, slots, pairs, ctypes.byref(ncow),
                                   ctypes.byref(done)), "append_slots")
        return list(slots[:n]), [(pairs[2 * k], pairs[2 * k + 1]) for k in range(ncow.value)]

    def free_seq(self, seq_id):
        _check(_alloc_free_seq(self._h, seq_id), "free_seq")

    def block_table(self, seq_ids, max_blocks):
        n = len(seq_ids)
        ids = (ctypes.c_int64 * max(n, 1))(*seq_ids)
        out = (ctypes.c_int32 * max(n * max_blocks, 1))()
        _check(_alloc_block_table(self._h, ids, n, max_blocks, out), "block_table")
        flat = list(out[:n * max_blocks])
        return [flat[i * max_blocks:(i + 1) * max_blocks] for i in range(n)]

    def context_lens(self, seq_ids):
        n = len(seq_ids)
        ids = (ctypes.c_int64 * max(n, 1))(*seq_ids)
        out = (ctypes.c_int32 * max(n, 1))()
        _check(_alloc_context_lens(self._h, ids, n, out), "context_lens")
        return list(out[:n])

    def num_free(self):
        return _alloc_num_free(self._h)

    def refcount(self, block):
        return _alloc_refcount(self._h, block)

    def seq_len(self, seq_id):
        return _alloc_seq_len(self._h, seq_id)

    def seq_num_blocks(self, seq_id):
        return _alloc_seq_num_blocks(self._h, seq_id)

    def usage(self):
        tokens, blocks = ctypes.c_int64(), ctypes.c_int64()
        _check(_alloc_usage(self._h, ctypes.byref(tokens), ctypes.byref(blocks)), "usage")
        return tokens.value, blocks.value

    def add_seq_cached(self, seq_id, token_ids):
        """Admit a prompt, reusing cached full blocks; returns cached token count."""
        n = len(token_ids)
        arr = (ctypes.c_int32 * max(n, 1))(*[int(t) for t in token_ids])
        cached = ctypes.c_int64()
        _check(_alloc_add_seq_cached(self._h, seq_id, arr, n, ctypes.byref(cached)),
               "add_seq_cached")
        return cached.value

    def cache_stats(self):
        """(full blocks looked up, hits, blocks cached now, blocks evicted)."""
        vals = [ctypes.c_int64() for _ in range(4)]
        _check(_alloc_cache_stats(self._h, *[ctypes.byref(v) for v in vals]), "cache_stats")
        return tuple(v.value for v in vals)

    def num_evictable(self):
        return _alloc_num_evictable(self._h)
