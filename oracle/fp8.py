"""FP8 E4M3 encoding of the KV cache — the oracle.  TEST INFRASTRUCTURE ONLY.

The pages mention quantised inference only in passing ([csdn] "量化模型优先考虑边缘
场景"; [betteryeah] §4.2 "启用量化推理"), so the format is the plainest modern
reading: the OCP 8-bit floating point "E4M3" (sign bit, 4 exponent bits with
bias 7, 3 mantissa bits; subnormals; no infinities; 0x7F / 0xFF are NaN;
largest finite value 448), with one float scale per kv head of each cache
(equal entries give one scale per cache):
    code = E4M3(x / scale[h]),   value = decode(code) * scale[h].

Readings taken:
* x / scale is computed in float32 (the precision the GPU uses), then
  rounded to E4M3 by round-to-nearest-even.
* Magnitudes that round above 448 saturate to +-448 (a cache must not hold
  NaN for finite inputs); NaN stays NaN (0x7F).
"""

import numpy as np

E4M3_MAX = 448.0


def e4m3_encode(x32):
    """float32 array -> uint8 E4M3 codes (RNE, saturating)."""
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    nan = np.isnan(x)
    sign = np.signbit(x)
    a = np.where(nan, 0.0, np.abs(x))
    # spacing of representable values around |x|: 2^(e-3) for the binade
    # [2^e, 2^(e+1)), e >= -6; subnormals share the spacing 2^-9 of e = -6
    e = np.floor(np.log2(np.where(a > 0, a, 1.0))).clip(-6, 8)
    quantum = 2.0 ** (e - 3)
    v = np.rint(a / quantum) * quantum        # round half to even
    v = np.minimum(v, E4M3_MAX)
    # encode the (exactly representable) rounded magnitude
    e2 = np.floor(np.log2(np.where(v > 0, v, 1.0))).clip(-6, 8)
    normal = v >= 2.0 ** -6
    exp_field = np.where(normal, e2 + 7, 0).astype(np.int64)
    man = np.where(normal, v / 2.0 ** e2 * 8 - 8, v / 2.0 ** -9).astype(np.int64)
    code = (exp_field << 3) | man
    out[...] = code
    out[sign] |= 0x80
    out[nan] = 0x7F
    return out


def e4m3_decode(codes):
    """uint8 E4M3 codes -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(ef == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (ef - 7))
    val = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def quantize(bits16, dtype, scale):
    """16-bit values -> E4M3 codes of value / scale (float32 division);
    ``scale`` is a number or an array that broadcasts against the values."""
    from .dtypes import widen
    x32 = widen(bits16, dtype).astype(np.float32)
    return e4m3_encode(x32 / np.asarray(scale, dtype=np.float32))


def dequantize(codes, scale):
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float32).astype(np.float64)


def per_head(scales, num_kv_heads):
    """A scale per kv head as float32 [num_kv_heads] (a number is repeated)."""
    s = np.asarray(scales, dtype=np.float32).reshape(-1)
    return np.repeat(s, num_kv_heads) if s.size == 1 else s


def quantize_cache(cache_bits, dtype, scales):
    """A whole 16-bit cache [N, Hkv, bs, D] -> codes, kv head h by scales[h]."""
    s = per_head(scales, cache_bits.shape[1])
    return quantize(cache_bits, dtype, s[None, :, None, None])


def quantize_into_cache(key_bits, value_bits, k_codes, v_codes, slot_mapping, block_size, dtype,
                        k_scales, v_scales):
    """The quantising cache write: kv head h of token t's K (V) becomes
    E4M3(x / k_scales[h]) (E4M3(x / v_scales[h])) in slot ``slot_mapping[t]``
    of copies of the code caches; negative slots are skipped.  Same placement
    as the 16-bit write (block = slot // block_size, offset = slot % block_size)."""
    k_out = np.array(k_codes, copy=True)
    v_out = np.array(v_codes, copy=True)
    hkv = key_bits.shape[1]
    kq = quantize(key_bits, dtype, per_head(k_scales, hkv)[None, :, None])
    vq = quantize(value_bits, dtype, per_head(v_scales, hkv)[None, :, None])
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        block, offset = divmod(int(slot), block_size)
        k_out[block, :, offset, :] = kq[t]
        v_out[block, :, offset, :] = vq[t]
    return k_out, v_out


def paged_attention_decode_fp8(q_bits, k_codes, v_codes, block_tables, context_lens, scale,
                               k_scales, v_scales, num_kv_heads, block_size, dtype, pairs=None):
    """Paged decode attention over E4M3 caches: the textbook single-query
    attention of ``oracle.attention`` over the gathered tokens' values
    decode(code) * scale of their kv head, in float64.  ``pairs`` as in
    ``oracle.attention.paged_attention_decode``."""
    from .attention import attend, kv_head_of, token_location
    from .dtypes import widen
    num_seqs, num_heads, head_dim = q_bits.shape
    ks, vs = per_head(k_scales, num_kv_heads), per_head(v_scales, num_kv_heads)
    if pairs is None:
        pairs = [(s, h) for s in range(num_seqs) for h in range(num_heads)]
    out = np.full((num_seqs, num_heads, head_dim), np.nan, dtype=np.float64)
    for s, h in pairs:
        g = kv_head_of(h, num_heads, num_kv_heads)
        blocks, offsets = token_location(np.asarray(block_tables[s]),
                                         np.arange(int(context_lens[s])), block_size)
        keys = dequantize(k_codes[blocks, g, offsets, :], ks[g])
        values = dequantize(v_codes[blocks, g, offsets, :], vs[g])
        out[s, h] = attend(widen(q_bits[s, h], dtype), keys, values, scale)
    return out


def paged_attention_prefill_fp8(q_bits, k_codes, v_codes, block_tables, context_lens, query_start,
                                scale, k_scales, v_scales, num_kv_heads, block_size, dtype,
                                rows=None):
    """Chunked-prefill attention over E4M3 caches: for new token j of sequence
    s, at position p = C_s - q_len_s + j, the textbook attention of
    ``oracle.attention`` over tokens 0..p with values decode(code) * scale of
    their kv head, in float64 (the causal reading of
    ``oracle.attention.paged_attention_prefill``).  ``rows`` (iterable of
    (token, head)) restricts the computation; other rows are NaN."""
    from .attention import attend, kv_head_of, token_location
    from .dtypes import widen
    total, num_heads, head_dim = q_bits.shape
    ks, vs = per_head(k_scales, num_kv_heads), per_head(v_scales, num_kv_heads)
    query_start = np.asarray(query_start, dtype=np.int64)
    seq_of = np.repeat(np.arange(len(query_start) - 1), np.diff(query_start))
    if rows is None:
        rows = [(t, h) for t in range(total) for h in range(num_heads)]
    out = np.full((total, num_heads, head_dim), np.nan, dtype=np.float64)
    for t, h in rows:
        s = int(seq_of[t])
        c = int(context_lens[s])
        pos = c - int(query_start[s + 1] - query_start[s]) + (t - int(query_start[s]))
        g = kv_head_of(h, num_heads, num_kv_heads)
        blocks, offsets = token_location(np.asarray(block_tables[s]), np.arange(pos + 1),
                                         block_size)
        keys = dequantize(k_codes[blocks, g, offsets, :], ks[g])
        values = dequantize(v_codes[blocks, g, offsets, :], vs[g])
        out[t, h] = attend(widen(q_bits[t, h], dtype), keys, values, scale)
    return out
