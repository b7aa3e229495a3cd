"""Page (block) manager — the oracle for the host block allocator.
TEST INFRASTRUCTURE ONLY.

What the pages fix (sources named in the package docstring):

* Pages are handed out on demand: a new request takes free pages at once and
  a sequence gains pages as it grows ([csdn] "分页式KV缓存" benefit list;
  [betteryeah] §2.2 "PagedAttention的分页机制": only the needed pages are
  allocated or released as a sequence's length changes).
* When a sequence finishes, its pages are marked free for reuse ([csdn]
  "典型工作流程拆解", step 7).
* Only the last page of a sequence can be partly empty, so waste stays under
  4 % ([cortexgrid] intro and FAQ answers).
* Parallel samples share the prompt's pages through the block table; physical
  blocks are reference-counted, and a block that several holders must modify
  is copied on write ([cortexgrid] FAQ answer on parallel sampling); sequences
  with a common prompt point at the same first pages ([csdn] "分页式KV缓存").
* Worked example: three sequences of 100, 300 and 500 tokens, each given a
  contiguous 500-token reservation, use (100+300+500)/(500×3) = 60 % of it
  ([betteryeah] §2.1 "传统注意力机制的内存瓶颈").

Readings taken where the pages are silent:

* The free list is a FIFO queue: allocation takes the front, release appends
  at the back.  Its initial order is an input (identity if none is given),
  so a shuffled pool is reproducible on both sides.
* ``add_seq`` takes ceil(n / block_size) blocks at once, or none if the pool
  is short.
* Copy-on-write triggers on an append into a partly filled last block whose
  refcount exceeds one: a fresh block is taken, the pair (old, new) is
  returned for the device copy, the old block's refcount drops by one and the
  sequence's table points at the new block.  The last remaining holder
  (refcount 1) writes in place, so n samples of one prompt make n−1 copies.
* An append at a block boundary takes a fresh block and needs no copy.
* Freeing walks the sequence's blocks front to back; each block whose
  refcount reaches zero is appended to the free queue.

Prefix caching (the ``enable_prefix_caching`` switch and the ``cache_hit_rate``
metric of [csdn]; sequences with a common prompt pointing at the same first
pages, [csdn] "分页式KV缓存"):

* A full block is identified by the exact token sequence from the start of
  its sequence through its last token.  ``add_seq_cached`` looks the prompt's
  full blocks up in order and reuses the cached ones up to the first miss;
  every freshly taken full block is registered under its prefix unless that
  prefix is already cached (a prefix keeps its first registered block while
  that block stays cached; such a block becomes unreachable when an earlier
  block of its prefix is evicted, and reachable again once that earlier
  prefix is re-registered).  Partial blocks are never cached.
* A cached block whose refcount drops to zero stays cached and becomes
  evictable, least recently released first.  Allocation takes the free queue
  first, then evicts the oldest evictable block (dropping its cache entry).
* Hit rate = full blocks found / full blocks looked up.
"""

from collections import deque


class AllocError(Exception):
    """Raised with ``status`` "INVALID_ARG" or "OUT_OF_BLOCKS"."""

    def __init__(self, status, msg=""):
        super().__init__("%s: %s" % (status, msg))
        self.status = status


def blocks_for(num_tokens, block_size):
    """Number of pages a sequence of ``num_tokens`` tokens occupies."""
    return -(-num_tokens // block_size)


class BlockManager:
    def __init__(self, num_blocks, block_size, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocError("INVALID_ARG", "num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise AllocError("INVALID_ARG", "free_order must be a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(order)
        self.refcount = [0] * num_blocks
        self.seqs = {}  # seq_id -> {"blocks": [..], "tokens": n}
        self.cache = {}         # full token prefix (tuple) -> block
        self.cache_key = {}     # block -> its prefix key
        self.evictable = []     # cached blocks with refcount 0, oldest first
        self.queried = 0
        self.hits = 0
        self.evicted = 0

    # -- queries ---------------------------------------------------------
    def num_free(self):
        return len(self.free)

    def num_evictable(self):
        return len(self.evictable)

    def seq_blocks(self, seq_id):
        return list(self.seqs[seq_id]["blocks"])

    def seq_len(self, seq_id):
        return self.seqs[seq_id]["tokens"]

    # -- operations ------------------------------------------------------
    def _take(self):
        if self.free:
            b = self.free.popleft()
        elif self.evictable:
            b = self.evictable.pop(0)
            del self.cache[self.cache_key.pop(b)]
            self.evicted += 1
        else:
            raise AllocError("OUT_OF_BLOCKS", "pool exhausted")
        self.refcount[b] = 1
        return b

    def _available(self):
        return len(self.free) + len(self.evictable)

    def _release(self, b):
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            if b in self.cache_key:
                self.evictable.append(b)
            else:
                self.free.append(b)

    def add_seq(self, seq_id, num_tokens):
        if seq_id in self.seqs or num_tokens < 0:
            raise AllocError("INVALID_ARG", "bad seq id or length")
        need = blocks_for(num_tokens, self.block_size)
        if need > self._available():
            raise AllocError("OUT_OF_BLOCKS", "need %d, have %d" % (need, self._available()))
        self.seqs[seq_id] = {"blocks": [self._take() for _ in range(need)],
                             "tokens": num_tokens}

    def fork(self, parent, child):
        if parent not in self.seqs or child in self.seqs:
            raise AllocError("INVALID_ARG", "bad parent or child id")
        p = self.seqs[parent]
        for b in p["blocks"]:
            self.refcount[b] += 1
        self.seqs[child] = {"blocks": list(p["blocks"]), "tokens": p["tokens"]}

    def append_slot(self, seq_id):
        """Reserve the slot of the sequence's next token.

        Returns ``(slot, cow_src, cow_dst)``; the cow pair is (-1, -1) when no
        copy is needed.
        """
        if seq_id not in self.seqs:
            raise AllocError("INVALID_ARG", "unknown seq id")
        seq = self.seqs[seq_id]
        pos = seq["tokens"]
        offset = pos % self.block_size
        cow_src = cow_dst = -1
        if offset == 0:
            if not self._available():
                raise AllocError("OUT_OF_BLOCKS", "pool exhausted")
            seq["blocks"].append(self._take())
        else:
            last = seq["blocks"][-1]
            if self.refcount[last] > 1:
                if not self._available():
                    raise AllocError("OUT_OF_BLOCKS", "pool exhausted")
                fresh = self._take()
                self.refcount[last] -= 1
                seq["blocks"][-1] = fresh
                cow_src, cow_dst = last, fresh
        seq["tokens"] = pos + 1
        return seq["blocks"][-1] * self.block_size + offset, cow_src, cow_dst

    def append_slots(self, seq_ids):
        """append_slot for each id in order; returns (slots, copy pairs made)."""
        slots, pairs = [], []
        for s in seq_ids:
            slot, src, dst = self.append_slot(s)
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        return slots, pairs

    def free_seq(self, seq_id):
        if seq_id not in self.seqs:
            raise AllocError("INVALID_ARG", "unknown seq id")
        for b in self.seqs.pop(seq_id)["blocks"]:
            self._release(b)

    def add_seq_cached(self, seq_id, tokens):
        """Admit a sequence whose prompt is ``tokens``, reusing cached full
        blocks of its longest cached prefix.  Returns the number of prompt
        tokens whose K/V are already cached."""
        tokens = [int(t) for t in tokens]
        if seq_id in self.seqs:
            raise AllocError("INVALID_ARG", "bad seq id")
        bs = self.block_size
        n = len(tokens)
        nfull = n // bs
        need = blocks_for(n, bs)
        hits = []
        for k in range(nfull):
            b = self.cache.get(tuple(tokens[:(k + 1) * bs]))
            if b is None:
                break
            hits.append(b)
        reclaimed = sum(1 for b in hits if self.refcount[b] == 0)
        if need - len(hits) > self._available() - reclaimed:
            raise AllocError("OUT_OF_BLOCKS", "pool exhausted")
        self.queried += nfull
        self.hits += len(hits)
        for b in hits:
            if self.refcount[b] == 0:
                self.evictable.remove(b)
            self.refcount[b] += 1
        blocks = list(hits)
        for k in range(len(hits), need):
            b = self._take()
            if k < nfull:
                key = tuple(tokens[:(k + 1) * bs])
                if key not in self.cache:
                    self.cache[key] = b
                    self.cache_key[b] = key
            blocks.append(b)
        self.seqs[seq_id] = {"blocks": blocks, "tokens": n}
        return len(hits) * bs

    def cache_stats(self):
        """(full blocks looked up, hits, blocks cached now, blocks evicted)."""
        return self.queried, self.hits, len(self.cache), self.evicted

    def block_table(self, seq_ids, max_blocks):
        """Rows of physical block ids, padded with -1."""
        rows = []
        for s in seq_ids:
            if s not in self.seqs:
                raise AllocError("INVALID_ARG", "unknown seq id")
            blocks = self.seqs[s]["blocks"]
            if len(blocks) > max_blocks:
                raise AllocError("INVALID_ARG", "table row too short")
            rows.append(blocks + [-1] * (max_blocks - len(blocks)))
        return rows

    # -- memory accounting ------------------------------------------------
    def physical_utilization(self):
        """Cached tokens / slots of allocated blocks, each physical slot counted once.

        A block's occupancy is the largest number of its slots any holder has
        filled (holders of a shared block agree on its shared slots).
        """
        occupied = {}
        for seq in self.seqs.values():
            n = seq["tokens"]
            for k, b in enumerate(seq["blocks"]):
                fill = min(self.block_size, n - k * self.block_size)
                occupied[b] = max(occupied.get(b, 0), fill)
        if not occupied:
            return 1.0
        return sum(occupied.values()) / (len(occupied) * self.block_size)


def contiguous_utilization(lengths, reserved_len):
    """Share of a per-sequence contiguous reservation actually used.

    The conventional scheme reserves ``reserved_len`` tokens for every
    sequence, so utilization = Σ L_i / (n · reserved_len) ([betteryeah] §2.1).
    """
    lengths = [int(x) for x in lengths]
    return sum(lengths) / (len(lengths) * reserved_len)


def paged_utilization(lengths, block_size):
    """Share of allocated page slots actually used: Σ L_i / (Σ ceil(L_i/bs)·bs)."""
    lengths = [int(x) for x in lengths]
    return sum(lengths) / (sum(blocks_for(n, block_size) for n in lengths) * block_size)
