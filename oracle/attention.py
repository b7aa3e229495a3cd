"""Paged decode attention in float64 — the oracle.  TEST INFRASTRUCTURE ONLY.

What the pages fix (sources named in the package docstring):

* A Transformer decoding autoregressively keeps a Key and a Value vector for
  every past token so they are not recomputed ([csdn], section
  "内存困局的破局者：PagedAttention 是如何工作的？").
* That KV cache is cut into fixed-size pages, usually 16 or 32 tokens each,
  which need not be contiguous; a lightweight page table records which
  physical block holds each logical page ([csdn] "分页式KV缓存：让显存利用接近
  理论极限"; [betteryeah] §2.2 "PagedAttention的分页机制"; [cortexgrid] FAQ
  answer on how the cache is split into blocks and mapped by a block table).
* When attention runs, the kernel assembles the data it needs from the page
  table across non-contiguous regions, and this is transparent to the model
  ([csdn] "分页式KV缓存").  Paged attention therefore has to equal ordinary
  attention over the tokens gathered back into logical order.
* A sequence of length L needs L×d of cache per attention head ([betteryeah]
  §2.1 "传统注意力机制的内存瓶颈").

Readings taken where the pages are silent:

* The attention itself is the textbook single-query form
  ``softmax(scale · q·Kᵀ) · V`` with ``scale`` supplied by the caller.
* Grouped-query attention: with ``G = num_heads / num_kv_heads``, query head
  ``h`` reads kv head ``h // G`` (consecutive query heads share a kv head).
* ``context_lens[i]`` counts every cached token of sequence ``i``, including
  the token whose K/V the same step has just written.
* Logical token ``t`` of a sequence lives in physical block
  ``block_table[t // block_size]`` at offset ``t % block_size``.
* ``context_len == 0`` yields an all-zero output row.
* The long-context form cuts the context into partitions and combines the
  per-partition (max, exp-sum, unnormalised output) triples; it must agree
  with the direct form up to float64 rounding.

Layouts (row-major):  q ``[S, H, D]``; k_cache / v_cache
``[num_blocks, H_kv, block_size, D]``; block_tables int32 ``[S, max_blocks]``;
context_lens int32 ``[S]``.  16-bit tensors are uint16 bit patterns (see
``oracle.dtypes``).  Results are float64 and are not rounded.
"""

import numpy as np

from .dtypes import widen


def kv_head_of(head, num_heads, num_kv_heads):
    """Grouped-query mapping: with G = num_heads / num_kv_heads, query head
    ``head`` reads kv head ``head // G``."""
    return head // (num_heads // num_kv_heads)


def token_location(table_row, t, block_size):
    """Physical (block, offset) of logical token(s) ``t`` through the page table."""
    t = np.asarray(t)
    return table_row[t // block_size], t % block_size


def gather_kv(cache_bits, table_row, context_len, kv_head, block_size, dtype):
    """Assemble one sequence's keys (or values) for one kv head, in logical order.

    Returns float64 ``[context_len, D]``.  Only table entries below
    ``ceil(context_len / block_size)`` are ever read.
    """
    t = np.arange(int(context_len))
    blocks, offsets = token_location(np.asarray(table_row), t, block_size)
    return widen(cache_bits[blocks, kv_head, offsets, :], dtype)


def attend(qvec, keys, values, scale):
    """Textbook single-query attention: ``softmax(scale·keys·q) · values``.

    ``qvec`` [D], ``keys``/``values`` [C, D], all float64.  C == 0 gives zeros.
    """
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1], dtype=np.float64)
    logits = scale * (keys @ qvec)
    weights = np.exp(logits - logits.max())
    probs = weights / weights.sum()
    return probs @ values


def paged_attention_decode(q_bits, k_cache_bits, v_cache_bits, block_tables,
                           context_lens, scale, num_kv_heads, block_size, dtype,
                           pairs=None):
    """Paged decode attention for every (sequence, query head), in float64.

    ``pairs``: optional iterable of (seq, head) to compute; rows not computed
    are NaN.  That lets full-size workloads be checked on a sample of outputs.
    """
    num_seqs, num_heads, head_dim = q_bits.shape
    if num_heads % num_kv_heads:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    if pairs is None:
        pairs = [(s, h) for s in range(num_seqs) for h in range(num_heads)]
    out = np.full((num_seqs, num_heads, head_dim), np.nan, dtype=np.float64)
    gathered = {}
    for s, h in pairs:
        g = kv_head_of(h, num_heads, num_kv_heads)
        if (s, g) not in gathered:
            gathered[(s, g)] = (
                gather_kv(k_cache_bits, block_tables[s], context_lens[s], g, block_size, dtype),
                gather_kv(v_cache_bits, block_tables[s], context_lens[s], g, block_size, dtype),
            )
        keys, values = gathered[(s, g)]
        out[s, h] = attend(widen(q_bits[s, h], dtype), keys, values, scale)
    return out


def partition_summary(qvec, keys, values, scale):
    """One partition's (max logit m, exp-sum l, unnormalised output o).

    m = max_t x_t, l = Σ_t exp(x_t − m), o = Σ_t exp(x_t − m)·V_t with
    x_t = scale·q·K_t.  An empty partition gives (−inf, 0, 0).
    """
    if keys.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(values.shape[1], dtype=np.float64)
    logits = scale * (keys @ qvec)
    m = logits.max()
    w = np.exp(logits - m)
    return m, w.sum(), w @ values


def combine_partitions(summaries):
    """Merge per-partition (m, l, o) triples into the attention output.

    M = max_p m_p;  out = Σ_p e^{m_p−M}·o_p / Σ_p e^{m_p−M}·l_p.
    Empty partitions (m = −inf) carry zero weight; all-empty gives zeros.
    """
    ms = np.array([m for m, _, _ in summaries], dtype=np.float64)
    if len(ms) == 0 or not np.isfinite(ms).any():
        dim = summaries[0][2].shape[0] if summaries else 0
        return np.zeros(dim, dtype=np.float64)
    big_m = ms.max()
    weights = np.exp(ms - big_m)
    num = sum(w * o for w, (_, _, o) in zip(weights, summaries))
    den = sum(w * l for w, (_, l, _) in zip(weights, summaries))
    return num / den


def paged_attention_decode_partitioned(q_bits, k_cache_bits, v_cache_bits,
                                       block_tables, context_lens, scale,
                                       num_kv_heads, block_size, dtype,
                                       partition_size, pairs=None):
    """Long-context form: attention per partition of ``partition_size`` tokens,
    then the max / sum / output reduce of ``combine_partitions``.

    Mathematically identical to ``paged_attention_decode``; the two differ
    only by float64 rounding.
    """
    if partition_size <= 0:
        raise ValueError("partition_size must be positive")
    num_seqs, num_heads, head_dim = q_bits.shape
    if num_heads % num_kv_heads:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    if pairs is None:
        pairs = [(s, h) for s in range(num_seqs) for h in range(num_heads)]
    out = np.full((num_seqs, num_heads, head_dim), np.nan, dtype=np.float64)
    for s, h in pairs:
        g = kv_head_of(h, num_heads, num_kv_heads)
        keys = gather_kv(k_cache_bits, block_tables[s], context_lens[s], g, block_size, dtype)
        values = gather_kv(v_cache_bits, block_tables[s], context_lens[s], g, block_size, dtype)
        qvec = widen(q_bits[s, h], dtype)
        c = int(context_lens[s])
        starts = range(0, c, partition_size)
        summaries = [partition_summary(qvec, keys[a:a + partition_size],
                                       values[a:a + partition_size], scale)
                     for a in starts]
        out[s, h] = combine_partitions(summaries) if summaries else np.zeros(head_dim)
    return out


def paged_attention_prefill(q_bits, k_cache_bits, v_cache_bits, block_tables, context_lens,
                            query_start, scale, num_kv_heads, block_size, dtype, rows=None):
    """Chunked-prefill attention over the paged cache, in float64.

    Sequence i contributes q_len_i = query_start[i+1] - query_start[i] query
    tokens: the last q_len_i of its context_lens[i] cached tokens (the step
    has already written their K/V).  Its j-th query sits at position
    p = C_i - q_len_i + j and attends causally to tokens 0..p, as every token of
    an autoregressive model does when its own K/V are computed ([csdn]
    "内存困局的破局者": each generated token's K and V join the cache).

    q_bits: uint16 [T, H, D] with T = query_start[-1] (queries of all sequences
    packed in order).  Returns float64 [T, H, D]; ``rows`` (iterable of
    (token, head)) restricts the computation, other rows are NaN.
    """
    total, num_heads, head_dim = q_bits.shape
    if num_heads % num_kv_heads:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    query_start = np.asarray(query_start, dtype=np.int64)
    seq_of = np.repeat(np.arange(len(query_start) - 1), np.diff(query_start))
    if rows is None:
        rows = [(t, h) for t in range(total) for h in range(num_heads)]
    out = np.full((total, num_heads, head_dim), np.nan, dtype=np.float64)
    gathered = {}
    for t, h in rows:
        s = int(seq_of[t])
        c = int(context_lens[s])
        q_len = int(query_start[s + 1] - query_start[s])
        pos = c - q_len + (t - int(query_start[s]))
        g = kv_head_of(h, num_heads, num_kv_heads)
        if (s, g) not in gathered:
            gathered[(s, g)] = (
                gather_kv(k_cache_bits, block_tables[s], c, g, block_size, dtype),
                gather_kv(v_cache_bits, block_tables[s], c, g, block_size, dtype),
            )
        keys, values = gathered[(s, g)]
        out[t, h] = attend(widen(q_bits[t, h], dtype), keys[:pos + 1], values[:pos + 1], scale)
    return out
