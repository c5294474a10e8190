"""Reference block manager.  TEST INFRASTRUCTURE ONLY.

Follows "KV 缓存与分页注意力":

* §像内存分页 - the KV pool is cut into equal blocks; a sequence's logical
  blocks are contiguous to it, its physical blocks may sit anywhere.
* §块表 - one block table per sequence; each entry records the physical block
  of a logical block and how many of its slots are filled.  A new physical
  block is allocated only when every earlier block is full, so a sequence
  wastes less than one block.  When a sequence finishes its blocks go back to
  the pool.
* FAQ "KV 缓存的写时复制是什么？" (§08 共用，写时复制) - when a sample is about to
  write into a shared block, the system first copies that block, writes into
  the copy, and lowers the original's count by one.

and "读懂PagedAttention", §同一提示生成两个回答的假想例子: two samples from one
prompt point their tables at the same input blocks; if the shared last input
block still has room and other references remain, it is copied on write
before the new token goes in; full shared blocks stay shared; only blocks that
must separate are copied (or a fresh block is taken); unreferenced blocks are
reclaimed.

Readings of what the pages leave open:

* Free-block policy: a FIFO queue, initialised to a given order (identity =
  "blocks assigned in arrival order"); allocation pops the front; a block whose
  count drops to zero is pushed to the back; a freed sequence releases its
  blocks in logical order.
* Copy-on-write: on append into a last block that is partially filled and has
  refcount > 1, pop a new block, record (old -> new), decrement the old
  block's count, put the new block into the table, then write.  With
  refcount == 1 the write goes in place, so of n sharers the first n-1 to
  write copy and the last one writes into the original.
* Batched appends are processed in the given order; a batch is all-or-nothing
  (on NO_BLOCKS nothing changes), mirroring the all-or-nothing rule for a
  sequence's blocks in §放不下的时候.

Automatic prefix caching (§后来的做法: each full block is hashed over its own
tokens and everything before it, and a new request that starts the same way
uses the existing blocks; it saves prompt processing only).  Readings:

* Only full blocks of a prompt are registered; the key of block i is FNV-1a 64
  (the published Fowler-Noll-Vo 1a hash: offset basis 14695981039346656037,
  prime 1099511628211, one byte at a time) over the key of block i-1 (8 bytes
  little endian, 0 for block 0) followed by block i's token ids (4 bytes
  little endian each); a key hit is confirmed against the stored token ids.
* A new prompt takes over the longest run of leading full blocks that hit;
  the first miss ends the run.  A hit on a freed block takes it back out of
  the free queue.  Blocks freed by their last user stay registered until they
  are handed out again as fresh blocks.
"""

from __future__ import annotations

import collections
import copy
from typing import Dict, List, Optional, Sequence, Tuple

OK = "OK"
INVALID_ARG = "INVALID_ARG"
NO_BLOCKS = "NO_BLOCKS"
UNKNOWN_SEQ = "UNKNOWN_SEQ"
SEQ_EXISTS = "SEQ_EXISTS"


class AllocError(Exception):
    def __init__(self, status: str, msg: str = ""):
        super().__init__(f"{status}: {msg}")
        self.status = status


FNV_OFFSET = 14695981039346656037
FNV_PRIME = 1099511628211


def fnv1a64(data: bytes) -> int:
    h = FNV_OFFSET
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & 0xFFFFFFFFFFFFFFFF
    return h


def block_key(parent: int, tokens: Sequence[int]) -> int:
    data = parent.to_bytes(8, "little") + b"".join(
        (int(t) & 0xFFFFFFFF).to_bytes(4, "little") for t in tokens)
    return fnv1a64(data)


class BlockManager:
    """Block tables, fill counts, refcounts and a FIFO free queue."""

    def __init__(self, num_blocks: int, block_size: int, order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocError(INVALID_ARG, "num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if order is None:
            order = range(self.num_blocks)
        order = [int(b) for b in order]
        if sorted(order) != list(range(self.num_blocks)):
            raise AllocError(INVALID_ARG, "free order must be a permutation of 0..num_blocks-1")
        self.free = collections.deque(order)
        self.refcount = [0] * self.num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.lengths: Dict[int, int] = {}
        self.cow_count = 0
        self.caching = False
        self.registered: Dict[int, tuple] = {}   # block -> (key, tokens)
        self.by_key: Dict[int, int] = {}
        self.hit_tokens = 0

    # -- helpers -----------------------------------------------------------
    def _fill_last(self, seq: int) -> int:
        """Filled slots in the last block: length - (blocks - 1) * bs, 0 if no blocks."""
        n = len(self.tables[seq])
        if n == 0:
            return 0
        return self.lengths[seq] - (n - 1) * self.block_size

    def _pop(self) -> int:
        b = self.free.popleft()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        self._unregister(b)          # handed out fresh: its old contents go
        return b

    def _unregister(self, b: int) -> None:
        if b in self.registered:
            key, _ = self.registered.pop(b)
            if self.by_key.get(key) == b:
                del self.by_key[key]

    def set_prefix_caching(self, on: bool) -> None:
        self.caching = bool(on)
        if not on:
            self.registered.clear()
            self.by_key.clear()

    def alloc_prefix(self, seq: int, tokens: Sequence[int]):
        """Admission with the prompt's token ids.  Returns (slots, n_cached)."""
        tokens = [int(t) for t in tokens]
        n = len(tokens)
        if not self.caching:
            return self.alloc(seq, n), 0
        if seq in self.tables:
            raise AllocError(SEQ_EXISTS, str(seq))
        bs = self.block_size
        need = (n + bs - 1) // bs
        full = n // bs
        keys, hits = [], []
        parent = 0
        hitting = True
        for i in range(full):
            blk = tokens[i * bs:(i + 1) * bs]
            key = block_key(parent, blk)
            keys.append(key)
            parent = key
            if hitting:
                b = self.by_key.get(key)
                if b is not None and self.registered[b][1] == blk:
                    hits.append(b)
                else:
                    hitting = False
        free_hits = sum(1 for b in hits if self.refcount[b] == 0)
        if need - len(hits) > len(self.free) - free_hits:
            raise AllocError(NO_BLOCKS, "prefix admission")
        table = []
        for b in hits:
            if self.refcount[b] == 0:
                self.free.remove(b)
            self.refcount[b] += 1
            table.append(b)
        for i in range(len(hits), need):
            b = self._pop()
            table.append(b)
            if i < full and keys[i] not in self.by_key:
                self.registered[b] = (keys[i], tokens[i * bs:(i + 1) * bs])
                self.by_key[keys[i]] = b
        self.tables[seq] = table
        self.lengths[seq] = n
        self.hit_tokens += len(hits) * bs
        return [table[t // bs] * bs + t % bs for t in range(n)], len(hits) * bs

    def _release(self, b: int) -> None:
        self.refcount[b] -= 1
        assert self.refcount[b] >= 0
        if self.refcount[b] == 0:
            self.free.append(b)

    # -- calls ---------------------------------------------------------------
    def alloc(self, seq: int, n_tokens: int) -> List[int]:
        """Admit a new sequence with n_tokens prompt tokens; returns their slots
        (physical block * bs + offset) in token order."""
        if n_tokens < 0:
            raise AllocError(INVALID_ARG, "n_tokens < 0")
        if seq in self.tables:
            raise AllocError(SEQ_EXISTS, str(seq))
        bs = self.block_size
        need = (n_tokens + bs - 1) // bs
        if need > len(self.free):
            raise AllocError(NO_BLOCKS, f"need {need}, free {len(self.free)}")
        table = [self._pop() for _ in range(need)]
        self.tables[seq] = table
        self.lengths[seq] = n_tokens
        return [table[t // bs] * bs + t % bs for t in range(n_tokens)]

    def append(self, seq: int) -> Tuple[int, int, int]:
        """Reserve the slot of one new token.  Returns (slot, cow_src, cow_dst);
        cow_src = cow_dst = -1 when no copy is needed."""
        if seq not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(seq))
        bs = self.block_size
        table = self.tables[seq]
        fill = self._fill_last(seq)
        src = dst = -1
        if not table or fill == bs:
            if not self.free:
                raise AllocError(NO_BLOCKS, "append needs a fresh block")
            table.append(self._pop())
            fill = 0
        elif self.refcount[table[-1]] > 1:
            if not self.free:
                raise AllocError(NO_BLOCKS, "copy-on-write needs a block")
            old = table[-1]
            new = self._pop()
            self.refcount[old] -= 1     # still > 0: other sharers hold it
            table[-1] = new
            src, dst = old, new
            self.cow_count += 1
        slot = table[-1] * bs + fill
        self.lengths[seq] += 1
        return slot, src, dst

    def append_batch(self, seqs: Sequence[int]) -> Tuple[List[int], List[Tuple[int, int]]]:
        """append() for each sequence in order; all-or-nothing.  Returns the
        slots (one per entry) and the copy-on-write pairs in the order made."""
        saved = self._snapshot()
        slots: List[int] = []
        pairs: List[Tuple[int, int]] = []
        try:
            for s in seqs:
                slot, src, dst = self.append(int(s))
                slots.append(slot)
                if src >= 0:
                    pairs.append((src, dst))
        except AllocError:
            self._restore(saved)
            raise
        return slots, pairs

    def fork(self, parent: int, child: int) -> None:
        """The child's table points at the parent's blocks; every block's count
        goes up by one."""
        if parent not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(parent))
        if child in self.tables:
            raise AllocError(SEQ_EXISTS, str(child))
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1

    def free_seq(self, seq: int) -> None:
        """A finished sequence gives its blocks back, in logical order; a block
        returns to the free queue when its count reaches zero."""
        if seq not in self.tables:
            raise AllocError(UNKNOWN_SEQ, str(seq))
        for b in self.tables.pop(seq):
            self._release(b)
        del self.lengths[seq]

    def export(self, seqs: Sequence[int], max_blocks: int):
        """Block tables [n][max_blocks] padded with -1, context lengths and the
        fill of each last block."""
        tables, lens, fills = [], [], []
        for s in seqs:
            s = int(s)
            if s not in self.tables:
                raise AllocError(UNKNOWN_SEQ, str(s))
            t = self.tables[s]
            if len(t) > max_blocks:
                raise AllocError(INVALID_ARG, "max_blocks too small")
            tables.append(t + [-1] * (max_blocks - len(t)))
            lens.append(self.lengths[s])
            fills.append(self._fill_last(s))
        return tables, lens, fills

    def stats(self) -> dict:
        bs = self.block_size
        used = sum(1 for r in self.refcount if r > 0)
        # a block's fill is the same for every sequence that references it
        fill_of: Dict[int, int] = {}
        for s, t in self.tables.items():
            for i, b in enumerate(t):
                f = bs if i < len(t) - 1 else self._fill_last(s)
                fill_of[b] = f
        return {
            "num_blocks": self.num_blocks,
            "block_size": bs,
            "free_blocks": len(self.free),
            "used_blocks": used,
            "num_seqs": len(self.tables),
            "stored_slots": sum(fill_of.values()),
            "logical_tokens": sum(self.lengths.values()),
            "table_slots": sum(len(t) for t in self.tables.values()) * bs,
            "cow_count": self.cow_count,
            "prefix_hit_tokens": self.hit_tokens,
            "cached_blocks": len(self.registered),
        }

    # -- snapshots for all-or-nothing batches -------------------------------
    def _snapshot(self):
        return (collections.deque(self.free), list(self.refcount),
                copy.deepcopy(self.tables), dict(self.lengths), self.cow_count,
                dict(self.registered), dict(self.by_key))

    def _restore(self, snap) -> None:
        (self.free, self.refcount, self.tables, self.lengths, self.cow_count,
         self.registered, self.by_key) = snap
