"""Oracle: block allocator and per-sequence block tables.

TEST INFRASTRUCTURE ONLY.  Plain Python restatement of the pages' memory
manager, used to check the CUDA path's host manager.  Nothing in the product
imports this module.

Sources (page title, section):
* "Paged Attention" (velog @junegood), 구현 세부사항 / 메모리 할당자: a block
  allocator hands out a free physical block id (``allocate_block``) and takes
  a freed one back into the reuse pool (``free_block``).
* same page, 작동 예시 and 동적 할당: a sequence gets a new physical block only
  when its last block is full; the logical->physical map grows one entry at a
  time (block ids 3, 7, 2 in the page's trace).
* same page, 메모리 공유 (Copy-on-Write): beams share the prompt's pages and
  each continues on a page of its own.
* "09. PagedAttention" (119-ai-studio), 해법: 페이지처럼 나눠 담기: logical
  blocks map to physical blocks through a per-request block table; only the
  last block of a request may be partly filled.
* "KV Cache & PagedAttention" studynote (agnusdei1207), Ⅱ 핵심 원리: shared
  blocks are copied when one sharer diverges (copy-on-write).

Readings where the pages are silent:
* the free pool is first-in-first-out; a freed block goes to the back;
* sharing is counted per block (reference count); ``free_block`` drops one
  reference and returns the block to the pool when the count reaches zero;
* appending token position p of a sequence: if p is a multiple of the block
  size a new block is taken; otherwise the token goes into the last block,
  and if that block is shared (count > 1) it is first copied to a fresh block
  (copy-on-write), the sequence's reference to the old one is dropped and its
  table points at the copy.  The slot is ``table[p // bs] * bs + p % bs``.
"""
from __future__ import annotations

from collections import deque


class OutOfBlocks(RuntimeError):
    pass


class BlockStateError(RuntimeError):
    pass


class BlockAllocator:
    """Free pool + reference counts over ``num_blocks`` physical blocks.

    ``free_order`` lists the ids handed out first; ids of the pool that are
    not listed start held (count 1) by an outside owner.  ``None`` = all ids
    free in ascending order.
    """

    def __init__(self, num_blocks: int, free_order=None):
        if num_blocks <= 0:
            raise ValueError("num_blocks must be positive")
        self.num_blocks = num_blocks
        if free_order is None:
            free_order = range(num_blocks)
        seen = set()
        for b in free_order:
            if not (0 <= b < num_blocks) or b in seen:
                raise ValueError(f"bad free_order entry {b}")
            seen.add(b)
        self.free = deque(int(b) for b in free_order)
        self.refcount = [0 if b in seen else 1 for b in range(num_blocks)]

    def allocate_block(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free physical block")
        b = self.free.popleft()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def incref(self, b: int) -> None:
        if self.refcount[b] <= 0:
            raise BlockStateError(f"block {b} is not allocated")
        self.refcount[b] += 1

    def free_block(self, b: int) -> None:
        if self.refcount[b] <= 0:
            raise BlockStateError(f"block {b} freed while free")
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self.free.append(b)

    def num_free(self) -> int:
        return len(self.free)


class BlockManager:
    """Per-sequence logical->physical block tables on top of an allocator."""

    def __init__(self, allocator: BlockAllocator, block_size: int):
        self.alloc = allocator
        self.bs = block_size
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        # prefix cache (off unless enabled): whole token prefix -> block
        self.cache = None
        self.cache_of: dict[int, tuple] = {}
        self.lru: list[int] = []            # cached blocks, least recently used first
        self.cache_stats = dict(hits=0, misses=0, evictions=0)

    # ---------------------------------------------------------------- prefix caching
    # "vLLM PagedAttention" studynote (prefix caching) and "09. PagedAttention"
    # (119-ai-studio, 다음 장): full blocks of a prompt are reused by a later
    # prompt with the same leading tokens.  Keys here are the exact token
    # tuples of the whole prefix up to each block's end.  Reading of what the
    # pages leave open (the plainest one): the cache keeps one reference per
    # cached block; only full prompt blocks are cached, one block per prefix;
    # lookup walks the leading full blocks until the first miss and never
    # serves the block holding the prompt's last token (that token must be
    # computed); when the free pool is empty the least recently used cached
    # block that nothing else references is freed first.
    def enable_prefix_cache(self) -> None:
        if self.tables:
            raise BlockStateError("enable the cache before adding sequences")
        self.cache = {}

    def _uncache(self, b: int) -> None:
        del self.cache[self.cache_of.pop(b)]
        self.lru.remove(b)
        self.alloc.free_block(b)

    def _new_block(self) -> int:
        if self.alloc.num_free() == 0 and self.cache is not None:
            for b in list(self.lru):
                if self.alloc.refcount[b] == 1:
                    self._uncache(b)
                    self.cache_stats["evictions"] += 1
                    break
        return self.alloc.allocate_block()

    def add_seq_prompt(self, seq: int, tokens):
        """New sequence holding the prompt ``tokens``.  Returns (slots, cached)
        with slot -1 for the ``cached`` leading tokens served from the cache."""
        if self.cache is None:
            raise BlockStateError("prefix cache not enabled")
        tokens = [int(t) for t in tokens]
        bs, n = self.bs, len(tokens)
        self.add_seq(seq)
        table = self.tables[seq]
        # the last prompt token is always computed (the first generated token
        # needs its attention output), so a prompt of whole blocks looks up
        # all but its last block
        hit, full = 0, n // bs
        lookable = (n - 1) // bs if n else 0
        while hit < lookable:
            b = self.cache.get(tuple(tokens[:(hit + 1) * bs]))
            if b is None:
                break
            self.alloc.incref(b)
            self.lru.remove(b)
            self.lru.append(b)
            table.append(b)
            hit += 1
        self.lens[seq] = hit * bs
        registered = []
        try:
            for i in range(hit * bs, n):
                if i % bs == 0:
                    table.append(self._new_block())
                self.lens[seq] = i + 1
                key = tuple(tokens[:i + 1])
                if (i + 1) % bs == 0 and key not in self.cache:
                    b = table[-1]
                    self.cache[key] = b
                    self.cache_of[b] = key
                    self.lru.append(b)
                    self.alloc.incref(b)
                    registered.append(b)
        except OutOfBlocks:
            for b in registered:
                self._uncache(b)
            for b in table:
                self.alloc.free_block(b)
            del self.tables[seq], self.lens[seq]
            raise
        self.cache_stats["hits"] += hit
        self.cache_stats["misses"] += full - hit
        slots = [-1] * (hit * bs) + [table[i // bs] * bs + i % bs for i in range(hit * bs, n)]
        return slots, hit * bs

    def add_seq(self, seq: int) -> None:
        if seq in self.tables:
            raise BlockStateError(f"sequence {seq} exists")
        self.tables[seq] = []
        self.lens[seq] = 0

    def append(self, seq: int):
        """Append one token.  Returns (slot, cow) with cow = (src, dst) or None."""
        table = self.tables[seq]
        p = self.lens[seq]
        cow = None
        if p % self.bs == 0:
            table.append(self._new_block())
        else:
            last = table[-1]
            if self.alloc.refcount[last] > 1:
                new = self._new_block()
                self.alloc.free_block(last)
                table[-1] = new
                cow = (last, new)
        self.lens[seq] = p + 1
        return table[p // self.bs] * self.bs + p % self.bs, cow

    def fork(self, parent: int, child: int) -> None:
        if child in self.tables:
            raise BlockStateError(f"sequence {child} exists")
        for b in self.tables[parent]:
            self.alloc.incref(b)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]

    def free_seq(self, seq: int) -> None:
        for b in self.tables.pop(seq):
            self.alloc.free_block(b)
        del self.lens[seq]

    def table_rows(self, seqs, max_blocks: int):
        """Block-table rows padded with -1, and the lengths, for ``seqs``."""
        rows, lens = [], []
        for s in seqs:
            t = self.tables[s]
            if len(t) > max_blocks:
                raise ValueError("table longer than max_blocks")
            rows.append(t + [-1] * (max_blocks - len(t)))
            lens.append(self.lens[s])
        return rows, lens
