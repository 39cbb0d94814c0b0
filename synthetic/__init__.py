"""Seeded synthetic workloads for the paged decode path.

This module holds recipes (shapes, context lengths, seeded permutations) and
random draws only -- none of the method's arithmetic. Both the oracle-side
tests and the CUDA-side tests and benchmark take their inputs from here.

The five workloads mirror the shapes of the source pages' measurements:

* ``tiny``          -- 4 sequences, 4 heads, head_dim 64, fp16, lengths {1,17,50,100},
                       a 32-block pool handed out in a seeded random order;
* ``llama7b_step``  -- the LLaMA-7B / A10G serving test of page 1, section
                       "3. 实战性能对比" (20 concurrent, prompt 128 +- 50,
                       output 256 +- 100): 20 sequences, 32/32 heads, fp16;
* ``llama13b_mix``  -- the 24-hour stress mix of page 2, section "5.3 极限压力测试"
                       (50% 128 / 30% 1K / 20% 8K tokens) on a LLaMA-13B shape:
                       256 sequences, 40/40 heads, bf16;
* ``gqa_prefix``    -- the prefix-caching case of page 3, section "案例与场景"
                       (Llama-3-8B, 64 concurrent, 1000-token history): 32 query /
                       8 kv heads, bf16, one 1000-token prefix shared by all 64;
* ``long_fp8``      -- the long-text FP8 row of page 2, section "5.1 长文本处理基准",
                       pushed to 32K tokens: 8 x 32768 tokens, 32/32 heads,
                       block size 32, E4M3 cache with one scale per tensor, bf16 q/out.

Public datasets are not used: every tensor is drawn from N(0, 1).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 4360


@dataclass
class Workload:
    name: str
    index: int                  # 1-based position in the list below
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    kv_dtype: str               # "f16" | "bf16" | "e4m3"
    q_dtype: str                # "f16" | "bf16"
    context_lens: list          # L_s, including the token decoded this step
    num_blocks: int             # physical blocks in the pool
    initial_order: list         # seeded permutation of range(num_blocks)
    scale: float
    seed: int
    prefix_len: int = 0         # tokens shared by every sequence (gqa_prefix)
    private_lens: list = field(default_factory=list)   # gqa_prefix: tokens after the prefix
    extra_slots: list = field(default_factory=list)    # tiny: slots in blocks no sequence holds
    beam_width: int = 0         # beam workloads: sequences r*width .. r*width+width-1 are one request

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_context_len(self) -> int:
        return max(self.context_lens) if self.context_lens else 0

    def max_blocks_per_seq(self, extra_tokens: int = 0) -> int:
        return -(-(self.max_context_len + extra_tokens) // self.block_size)


def _pool_size(context_lens, block_size, factor=1.1) -> int:
    need = sum(-(-L // block_size) for L in context_lens)
    return int(math.ceil(factor * need))


def make(name: str) -> Workload:
    """The named workload, fully determined by its seed."""
    idx = {n: i + 1 for i, n in enumerate(NAMES)}[name]
    seed = SEED_BASE + idx
    rng = np.random.default_rng(seed)
    if name == "tiny":
        lens = [1, 17, 50, 100]
        nb = 32
        order = rng.permutation(nb).tolist()
        w = Workload(name, idx, 4, 4, 4, 64, 16, "f16", "f16", lens, nb, order, 1.0 / 8.0, seed)
        # 4 distinct slots inside blocks that no sequence holds once the
        # sequences have taken their blocks in table order (14 blocks)
        used = sum(-(-L // 16) for L in lens)
        free_blocks = order[used:]
        cand = np.array([b * 16 + o for b in free_blocks for o in range(16)])
        w.extra_slots = sorted(rng.choice(cand, size=4, replace=False).tolist())
        return w
    if name == "llama7b_step":
        S = 20
        lens = (rng.integers(78, 179, size=S) + rng.integers(156, 357, size=S)).tolist()
        nb = _pool_size(lens, 16)
        order = rng.permutation(nb).tolist()
        return Workload(name, idx, S, 32, 32, 128, 16, "f16", "f16", lens, nb, order,
                        1.0 / math.sqrt(128), seed)
    if name == "llama13b_mix":
        classes = [128] * 128 + [1024] * 77 + [8192] * 51
        base = rng.permutation(np.array(classes))
        lens = (base + rng.integers(0, 16, size=len(base))).tolist()
        nb = _pool_size(lens, 16)
        order = rng.permutation(nb).tolist()
        return Workload(name, idx, 256, 40, 40, 128, 16, "bf16", "bf16", lens, nb, order,
                        1.0 / math.sqrt(128), seed)
    if name == "gqa_prefix":
        S, prefix = 64, 1000
        priv = rng.integers(1, 257, size=S).tolist()
        lens = [prefix + p for p in priv]
        need = -(-prefix // 16) + sum(-(-L // 16) - prefix // 16 for L in lens)
        nb = int(math.ceil(1.1 * need))
        order = rng.permutation(nb).tolist()
        return Workload(name, idx, S, 32, 8, 128, 16, "bf16", "bf16", lens, nb, order,
                        1.0 / math.sqrt(128), seed, prefix_len=prefix, private_lens=priv)
    if name == "long_fp8":
        S, L = 8, 32768
        lens = [L] * S
        nb = _pool_size(lens, 32)
        order = rng.permutation(nb).tolist()
        return Workload(name, idx, S, 32, 32, 128, 32, "e4m3", "bf16", lens, nb, order,
                        1.0 / math.sqrt(128), seed)
    raise KeyError(name)


NAMES = ["tiny", "llama7b_step", "llama13b_mix", "gqa_prefix", "long_fp8"]


def custom(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, q_dtype,
           context_lens, seed, pool_factor=1.25, scale=None) -> Workload:
    """A workload of arbitrary shape (fuzz and edge-case tests)."""
    rng = np.random.default_rng(seed)
    nb = max(1, _pool_size(list(context_lens) + [1], block_size, pool_factor) + 2)
    order = rng.permutation(nb).tolist()
    return Workload("custom", 0, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                    kv_dtype, q_dtype, list(context_lens), nb, order,
                    scale if scale is not None else 1.0 / math.sqrt(head_dim), seed)


# --------------------------------------------------------------------------
# random draws (torch generators: CPU for small tensors, CUDA for large ones)
# --------------------------------------------------------------------------

_TORCH_DT = {"f16": "float16", "bf16": "bfloat16"}


def _torch():
    import torch
    return torch


def normal_codes(shape, dtype: str, seed: int, device="cpu"):
    """N(0, 1) values rounded to fp16 / bf16 by torch; returned as int16 codes."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x.to(getattr(torch, _TORCH_DT[dtype])).view(torch.int16)


def normal_values(shape, dtype: str, seed: int, device="cpu"):
    """N(0, 1) values as a torch fp16 / bf16 tensor."""
    torch = _torch()
    return normal_codes(shape, dtype, seed, device).view(getattr(torch, _TORCH_DT[dtype]))


def normal_e4m3_codes(shape, seed: int, device="cpu", chunk=1 << 26):
    """E4M3 codes of N(0, 1) draws divided by a per-tensor scale amax / 448.

    The draws are cast by torch's float8_e4m3fn conversion (a library routine),
    so the cache contents come from neither the oracle's nor the kernels'
    encoder. Returns (codes as a uint8 tensor, scale as a Python float).
    """
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.uint8, device=device)
    amax = 0.0
    # two passes with the same seed: amax first, then the cast
    for start in range(0, n, chunk):
        m = min(chunk, n - start)
        x = torch.randn(m, generator=g, device=device, dtype=torch.float32)
        amax = max(amax, float(x.abs().max()))
    scale = amax / 448.0
    g.manual_seed(seed)
    for start in range(0, n, chunk):
        m = min(chunk, n - start)
        x = torch.randn(m, generator=g, device=device, dtype=torch.float32)
        y = (x / scale).clamp_(-448.0, 448.0)
        out[start:start + m] = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return out.view(*shape), float(scale)


def fill_normal_(t, dtype: str, seed: int, chunk=1 << 26):
    """Fill a contiguous fp16/bf16 tensor (any device) with seeded N(0, 1) values,
    chunk by chunk (bounded temporary memory)."""
    torch = _torch()
    g = torch.Generator(device=t.device)
    g.manual_seed(seed)
    flat = t.view(-1)
    target = getattr(torch, _TORCH_DT[dtype])
    for start in range(0, flat.numel(), chunk):
        m = min(chunk, flat.numel() - start)
        x = torch.randn(m, generator=g, device=t.device, dtype=torch.float32)
        flat[start:start + m].copy_(x.to(target).view(t.dtype))
    return t


def step_inputs(w: Workload, step: int, device="cpu"):
    """The query and the new token's K/V of every sequence at a given step.

    q: [S, Hq, D] (q dtype); k_new, v_new: [S, Hkv, D] (q dtype; an E4M3 cache is
    written from the query dtype)."""
    base = w.seed * 1000 + 17 * step
    q = normal_values((w.num_seqs, w.num_q_heads, w.head_dim), w.q_dtype, base + 1, device)
    k = normal_values((w.num_seqs, w.num_kv_heads, w.head_dim), w.q_dtype, base + 2, device)
    v = normal_values((w.num_seqs, w.num_kv_heads, w.head_dim), w.q_dtype, base + 3, device)
    return q, k, v


def subset(w: Workload, n_seqs: int) -> Workload:
    """The first n_seqs sequences of a workload, with a pool re-sized to 1.1x their
    need and a fresh seeded permutation (smaller device footprint, same shapes)."""
    if n_seqs >= w.num_seqs:
        return w
    rng = np.random.default_rng(w.seed + 1000 * n_seqs)
    lens = list(w.context_lens[:n_seqs])
    nb = _pool_size(lens, w.block_size)
    return Workload(f"{w.name}[:{n_seqs}]", w.index, n_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                    w.block_size, w.kv_dtype, w.q_dtype, lens, nb, rng.permutation(nb).tolist(), w.scale,
                    w.seed, w.prefix_len, list(w.private_lens[:n_seqs]), [], w.beam_width)


def grown(w: Workload, tokens: int) -> Workload:
    """The same workload with room for `tokens` more tokens per sequence: the pool
    gains S * ceil(tokens / BS) blocks, handed out (in a seeded order) after the
    recipe's own blocks."""
    extra = w.num_seqs * (-(-tokens // w.block_size))
    if extra == 0:
        return w
    rng = np.random.default_rng(w.seed + 77)
    order = list(w.initial_order) + (w.num_blocks + rng.permutation(extra)).tolist()
    return Workload(w.name, w.index, w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                    w.kv_dtype, w.q_dtype, list(w.context_lens), w.num_blocks + extra, order, w.scale,
                    w.seed, w.prefix_len, list(w.private_lens), list(w.extra_slots), w.beam_width)


# --------------------------------------------------------------------------
# beam search (page 1, section "5. 高级应用场景": width-5 beam search)
# --------------------------------------------------------------------------

BEAM_PARENT_WEIGHTS = (0.40, 0.25, 0.15, 0.12, 0.08)


def beam_workload(num_requests=16, width=5, prompt=1024, num_heads=40, head_dim=128, block_size=16,
                  kv_dtype="bf16", growth=256, seed=4369) -> Workload:
    """`num_requests` prompts of `prompt` + U[0,15] tokens, each decoded by `width`
    beams (sequence r * width + j is beam j of request r). The pool holds one copy of
    every prompt plus room for `growth` private tokens per beam."""
    rng = np.random.default_rng(seed)
    plens = (prompt + rng.integers(0, 16, size=num_requests)).tolist()
    lens = [L for L in plens for _ in range(width)]
    need = sum(-(-L // block_size) for L in plens) + num_requests * width * (-(-growth // block_size) + 1)
    nb = int(math.ceil(1.1 * need))
    return Workload("beam%d" % width, 0, num_requests * width, num_heads, num_heads, head_dim, block_size,
                    kv_dtype, kv_dtype, lens, nb, rng.permutation(nb).tolist(), 1.0 / math.sqrt(head_dim), seed,
                    beam_width=width)


def beam_parents(num_requests: int, width: int, step: int, seed: int):
    """Seeded beam re-selection of one step: new beam j of request r continues old
    beam parents[r * width + j] (same request; beams ranked by index, the better
    ones chosen more often; sorted, as a top-k selection would list them)."""
    rng = np.random.default_rng(seed * 7919 + step)
    out = []
    for r in range(num_requests):
        picks = np.sort(rng.choice(width, size=width, p=BEAM_PARENT_WEIGHTS[:width]))
        out += (r * width + picks).tolist()
    return out
