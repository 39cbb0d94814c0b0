"""Prefix cache over full KV blocks (oracle; test infrastructure only).

Page 3 «内存优化：KV Cache管理、PagedAttention原理与内存池配置», section
"案例与场景": with prefix caching on, the KV blocks of a common prefix get a global
hash index; a new request whose prefix matches cached blocks reuses those physical
blocks and allocates blocks only for its new tokens. Section "误区与复盘" (误区3):
it only works when the prefixes match exactly -- a random number or a timestamp in
the system prompt destroys the hit rate -- and the table costs host memory.

Readings (the pages give no more detail):

* only full blocks are cached; block k of a prompt is reusable iff the prompt's
  tokens [0, (k+1)*BS) equal those of the cached block's sequence (exact prefix
  match, so the KV computed for them is the same);
* lookup walks the prompt's full blocks in order and stops at the first miss;
  every hit takes one more reference on the block;
* the index holds one reference of its own on every block it lists, so a cached
  block survives the sequences that wrote it; ``evict`` drops, oldest insertion
  first, index entries whose block nobody else holds, and ``clear`` drops all.

The oracle keys the dictionary by the whole token prefix itself -- the plain
definition -- with no hashing.
"""

from __future__ import annotations

from .pool import BlockPool


class PrefixCache:
    def __init__(self, block_size: int):
        self.bs = block_size
        self.entries = {}            # tuple(prefix tokens) -> block
        self.order = []              # insertion order of the keys

    def __len__(self):
        return len(self.entries)

    def match(self, pool: BlockPool, tokens, row: list) -> int:
        """Append to `row` every leading full block of `tokens` found in the cache
        (taking a reference on each); returns how many were found."""
        n = 0
        for k in range(len(tokens) // self.bs):
            key = tuple(tokens[:(k + 1) * self.bs])
            b = self.entries.get(key)
            if b is None:
                break
            pool.incref(b)
            row.append(b)
            n += 1
        return n

    def insert(self, pool: BlockPool, tokens, row) -> int:
        """List every full block of a sequence (tokens laid out from position 0 in
        the blocks of `row`) that the cache does not hold yet; the cache takes a
        reference on each. Returns how many were added."""
        added = 0
        for k in range(len(tokens) // self.bs):
            key = tuple(tokens[:(k + 1) * self.bs])
            if key in self.entries:
                continue
            b = row[k]
            pool.incref(b)
            self.entries[key] = b
            self.order.append(key)
            added += 1
        return added

    def evict(self, pool: BlockPool, max_blocks: int) -> int:
        """Drop up to max_blocks entries whose block only the cache holds, oldest first."""
        n = 0
        keep = []
        for key in self.order:
            b = self.entries[key]
            if n < max_blocks and pool.refcnt[b] == 1:
                pool.decref(b)
                del self.entries[key]
                n += 1
            else:
                keep.append(key)
        self.order = keep
        return n

    def clear(self, pool: BlockPool) -> int:
        n = len(self.order)
        for key in self.order:
            pool.decref(self.entries[key])
        self.entries.clear()
        self.order.clear()
        return n
