"""Float64 CPU oracle for the paged-KV-cache decode hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow, obviously-correct restatement of what the method computes,
written from the three source pages:

* page 1 -- "突破GPU内存瓶颈：vLLM与PagedAttention技术深度解析" (ocdem.com);
* page 2 -- the untitled lshu.cn article whose first section is
  "1. 为什么vLLM能实现24倍推理加速";
* page 3 -- "内存优化：KV Cache管理、PagedAttention原理与内存池配置" (5688vip.com).

It shares no code, header, table or constant with the CUDA library in
``paged_kv_cache_436_b200``; neither side imports the other. The seeded input
generators in ``synthetic`` (which hold none of the method's arithmetic) are the
only code both sides use.

Modules:

* ``codecs``     -- bit-level decoders for binary16, bfloat16 and OCP E4M3, and
  the E4M3 round-to-nearest-even saturating encoder;
* ``attention``  -- paged single-query decode attention in float64;
* ``cache_ops``  -- the KV-cache slot write and the block copy, as array ops;
* ``pool``       -- the block pool (O(1) LIFO free list + refcounts) and the
  per-sequence append with copy-on-write;
* ``accounting`` -- the KV-size closed form and the per-step byte counts.
"""

from . import codecs, attention, cache_ops, pool, accounting  # noqa: F401
