"""Block pool and per-sequence block tables (oracle; test infrastructure only).

From page 3, section "PagedAttention原理：从操作系统虚拟内存借鉴的智慧":

* the KV cache is cut into fixed-size blocks of 16 or 32 tokens; a sequence
  takes blocks only as it grows and returns them all when it finishes
  ("按需分配，消除内部碎片");
* several sequences may share physical blocks through a reference count
  ("跨请求共享");
* free blocks form a linked list, so alloc and free are O(1) and no device
  allocation happens per request ("空闲块以链表形式组织，分配和释放均为O(1)操作").

Page 1, section "2. PagedAttention的革命性设计" adds that waste is confined to
a sequence's last block.

Readings where the pages are silent (all deterministic, so block tables can be
compared bit for bit):

* the free list is a LIFO stack; ``initial_order`` seeds it so that successive
  allocations return ``initial_order[0], initial_order[1], ...``; a block whose
  count drops to zero is pushed on top;
* appending logical position ``pos`` (block size BS): if ``pos % BS == 0`` a
  new block is allocated for logical block ``pos // BS``; otherwise, if the
  last block is shared (count > 1), a fresh block is allocated, the pair
  (old, new) is reported for a block copy, the old block loses one reference
  and the table entry is replaced (copy-on-write); the slot is then
  ``table[pos // BS] * BS + pos % BS``;
* errors: allocating from an empty pool is ``OOM``; taking or dropping a
  reference of a free block, or dropping a reference below zero, is ``STATE``.
"""

from __future__ import annotations


class PoolError(Exception):
    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind


class BlockPool:
    def __init__(self, num_blocks: int, initial_order=None):
        if num_blocks <= 0:
            raise PoolError("ARG", "num_blocks must be positive")
        order = list(range(num_blocks)) if initial_order is None else [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise PoolError("ARG", "initial_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.refcnt = [0] * num_blocks
        # stack: the top (end of the list) is the next block handed out
        self.free = list(reversed(order))

    # --- O(1) primitives -------------------------------------------------
    def alloc(self) -> int:
        if not self.free:
            raise PoolError("OOM", "no free block")
        b = self.free.pop()
        self.refcnt[b] = 1
        return b

    def incref(self, b: int) -> None:
        self._check(b)
        if self.refcnt[b] == 0:
            raise PoolError("STATE", f"incref of free block {b}")
        self.refcnt[b] += 1

    def decref(self, b: int) -> None:
        self._check(b)
        if self.refcnt[b] == 0:
            raise PoolError("STATE", f"decref of free block {b}")
        self.refcnt[b] -= 1
        if self.refcnt[b] == 0:
            self.free.append(b)

    def refcount(self, b: int) -> int:
        self._check(b)
        return self.refcnt[b]

    def num_free(self) -> int:
        return len(self.free)

    def free_list(self):
        """Blocks in the order successive allocations would return them."""
        return list(reversed(self.free))

    def _check(self, b: int) -> None:
        if not (0 <= b < self.num_blocks):
            raise PoolError("ARG", f"block {b} out of range")

    # --- sequences -------------------------------------------------------
    def seq_append(self, row: list, pos: int, block_size: int):
        """Append logical position ``pos`` to a sequence whose table is ``row``.

        ``row`` holds the sequence's physical blocks in logical order and has
        exactly ceil(pos / block_size) entries before the call. Returns
        (slot, cow_src, cow_dst) with -1 for "no copy".
        """
        lb, off = divmod(pos, block_size)
        if len(row) != -(-pos // block_size):
            raise PoolError("ARG", "table length does not match position")
        cow_src = cow_dst = -1
        if off == 0:
            row.append(self.alloc())
        else:
            old = row[lb]
            if self.refcnt[old] > 1:
                new = self.alloc()
                self.decref(old)
                row[lb] = new
                cow_src, cow_dst = old, new
        return row[lb] * block_size + off, cow_src, cow_dst

    def seq_extend(self, row: list, start_pos: int, n_tokens: int, block_size: int):
        """Append positions start_pos .. start_pos + n_tokens - 1; returns (slots, cow pairs)."""
        slots, cows = [], []
        for pos in range(start_pos, start_pos + n_tokens):
            slot, cs, cd = self.seq_append(row, pos, block_size)
            slots.append(slot)
            if cs >= 0:
                cows.append((cs, cd))
        return slots, cows

    def fork(self, row: list) -> list:
        """A new sequence sharing every block of ``row`` (reference counts + 1)."""
        for b in row:
            self.incref(b)
        return list(row)

    def free_seq(self, row: list) -> None:
        """Release a finished sequence: drop one reference of each of its blocks."""
        for b in row:
            self.decref(b)
        row.clear()

    def batch_append(self, rows, positions, block_size: int):
        """One decode step's bookkeeping for a batch, sequence by sequence in order.

        Returns (slots, cow_pairs, table_updates) where table_updates lists
        (seq, logical_block, physical_block) for every table entry written.
        """
        slots, cows, updates = [], [], []
        for s, (row, pos) in enumerate(zip(rows, positions)):
            slot, cs, cd = self.seq_append(row, pos, block_size)
            slots.append(slot)
            if cs >= 0:
                cows.append((cs, cd))
            if pos % block_size == 0 or cs >= 0:
                updates.append((s, pos // block_size, row[pos // block_size]))
        return slots, cows, updates


def reorder(pool: BlockPool, rows: list, lens: list, parents) -> tuple:
    """Beam re-selection: new sequence i continues old sequence parents[i].

    Page 1 «突破GPU内存瓶颈：vLLM与PagedAttention技术深度解析», section "5. 高级应用场景"
    (beam search: the beams share their common blocks). Reading: every new row is a
    copy of its parent's row and takes one reference per block; then every old row
    drops its references, so a beam chosen k times holds its blocks k times and a
    beam chosen 0 times returns its private blocks. Returns (new rows, new lens).
    """
    new_rows = [list(rows[p]) for p in parents]
    new_lens = [lens[p] for p in parents]
    for r in new_rows:
        for b in r:
            pool.incref(b)
    for r in rows:
        for b in r:
            pool.decref(b)
    return new_rows, new_lens
