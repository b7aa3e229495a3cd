"""Cache-write scatter and copy-on-write block copy — the oracle.
TEST INFRASTRUCTURE ONLY.

What the pages fix (sources named in the package docstring):

* The cache keeps K and V per token ([csdn], section
  "内存困局的破局者：PagedAttention 是如何工作的？"), in fixed-size pages that
  are found through a page table ([csdn] "分页式KV缓存"; [betteryeah] §2.2).
  Writing a new token's K/V therefore means storing it at its page and offset.
* Samples of one prompt share that prompt's cached pages through the block
  table; physical blocks carry reference counts, and when several holders must
  modify a block, copy-on-write makes a private copy ([cortexgrid] FAQ answer
  on parallel sampling).  The copy is of the whole block.

Readings taken where the pages are silent:

* A slot is ``physical_block * block_size + offset`` (int64); a negative slot
  marks a padding token that is not written.
* A copy pair (src, dst) copies every kv head, every offset and every
  dimension of the K block and of the V block.  Pairs are applied in order.

Both operations are pure data movement; results must match bit for bit, so
they work on the uint16 bit patterns and never widen to float.
"""

import numpy as np


def reshape_and_cache(key_bits, value_bits, k_cache_bits, v_cache_bits, slot_mapping,
                      block_size, inplace=False):
    """Scatter new tokens' K/V into copies of the caches (or into the given
    arrays when ``inplace``, which spares a copy of very large pools).

    key_bits, value_bits: uint16 ``[T, H_kv, D]``; caches uint16
    ``[num_blocks, H_kv, block_size, D]``; slot_mapping int64 ``[T]``.
    Returns ``(k_cache, v_cache, out_of_range)`` where ``out_of_range`` lists
    the token indices whose slot lay beyond the pool (those are skipped).
    """
    k_out = k_cache_bits if inplace else np.array(k_cache_bits, copy=True)
    v_out = v_cache_bits if inplace else np.array(v_cache_bits, copy=True)
    num_slots = k_out.shape[0] * block_size
    bad = []
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        if slot >= num_slots:
            bad.append(t)
            continue
        block, offset = divmod(int(slot), block_size)
        k_out[block, :, offset, :] = key_bits[t]
        v_out[block, :, offset, :] = value_bits[t]
    return k_out, v_out, bad


def copy_blocks(k_cache_bits, v_cache_bits, block_mapping, inplace=False):
    """Copy whole physical blocks, K and V, for each (src, dst) pair in order
    (into copies of the caches, or into the given arrays when ``inplace``).

    Returns ``(k_cache, v_cache, out_of_range)``; pairs with an index outside
    the pool are skipped and listed.
    """
    k_out = k_cache_bits if inplace else np.array(k_cache_bits, copy=True)
    v_out = v_cache_bits if inplace else np.array(v_cache_bits, copy=True)
    num_blocks = k_out.shape[0]
    bad = []
    for p, (src, dst) in enumerate(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2)):
        if not (0 <= src < num_blocks and 0 <= dst < num_blocks):
            bad.append(p)
            continue
        k_out[dst] = k_out[src]
        v_out[dst] = v_out[src]
    return k_out, v_out, bad
