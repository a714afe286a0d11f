"""Seeded synthetic inputs for paged decode attention.

This module only *draws inputs*: sequence lengths, a block allocator that
places each sequence's blocks in a pool, the per-token K/V rows to append,
slot numbers and queries.  It holds none of the method's arithmetic (no
append, no quantisation, no attention) and imports neither the CUDA library
nor the oracle, so both sides of every parity check consume identical inputs.

Workload shapes follow the pages' models ("LLM推理显存优化KV Cache管理3大策略"
(mlqm.cn) §1-§5: Llama-2 7B/13B/70B; "生产级 LLM 推理的 KV 缓存优化" (GPUYard)
§2: 70B with 8 KV heads, head_dim 128; "大模型推理加速实战…" (yunthe.com):
block_size 16, 13B at batch 32 x 2048).  The data are synthetic (N(0,1)
values); no model weights or prompts are involved.

Conventions:
  * ``context_lens[s]`` is the number of tokens the decode step attends
    over.  The pool is pre-filled with the first ``ctx - 1`` tokens and the
    step appends token ``ctx - 1`` (so the appended token is attended).
  * A slot number is ``physical_block * block_size + offset``.
  * Unused block-table entries hold ``pad_entry`` (default -1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

__all__ = ["BlockAllocator", "Workload", "CONFIGS", "make_workload", "make_custom",
           "workload_seed", "canonical_name"]


class BlockAllocator:
    """Fixed-size block pool with a free list and reference counts.

    Mirrors the pages' block manager (mlqm.cn §2 Block/BlockTable: a block
    carries a ref_count, a table maps logical to physical blocks; yunthe.com:
    blocks are allocated on demand and returned when a sequence ends).  The
    free list is a seeded permutation of the pool, so allocation order places
    blocks at random physical positions.
    """

    def __init__(self, num_blocks: int, generator: Optional[torch.Generator] = None):
        if num_blocks <= 0:
            raise ValueError("num_blocks must be positive")
        self.num_blocks = num_blocks
        if generator is None:
            order = list(range(num_blocks))
        else:
            order = torch.randperm(num_blocks, generator=generator).tolist()
        # pop() takes from the end: reverse so the first drawn id comes first
        self._free: List[int] = list(reversed(order))
        self.ref_count: List[int] = [0] * num_blocks

    @property
    def num_free(self) -> int:
        return len(self._free)

    def allocate(self) -> int:
        if not self._free:
            raise MemoryError("block pool exhausted")
        b = self._free.pop()
        self.ref_count[b] = 1
        return b

    def share(self, block: int) -> int:
        if self.ref_count[block] <= 0:
            raise ValueError(f"block {block} is not allocated")
        self.ref_count[block] += 1
        return block

    def free(self, block: int) -> None:
        if self.ref_count[block] <= 0:
            raise ValueError(f"double free of block {block}")
        self.ref_count[block] -= 1
        if self.ref_count[block] == 0:
            self._free.append(block)


@dataclass
class Workload:
    """One decode step's inputs plus the pre-fill that populates the pool."""

    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    cache_dtype: str            # "f32" | "bf16" | "i8" | "fp8"
    input_dtype: torch.dtype    # dtype of q and of the K/V rows to append
    softmax_scale: float
    context_lens: torch.Tensor  # int32 [B]
    block_tables: torch.Tensor  # int32 [B, max_blocks_per_seq]
    prefill_slots: torch.Tensor  # int64 [T_pre]
    prefill_k: torch.Tensor     # [T_pre, n_kv, d] input_dtype
    prefill_v: torch.Tensor
    q: torch.Tensor             # [B, n_q, d] input_dtype
    new_k: torch.Tensor         # [B, n_kv, d] input_dtype
    new_v: torch.Tensor
    new_slots: torch.Tensor     # int64 [B]
    allocator: BlockAllocator = field(repr=False, default=None)
    meta: Dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.num_seqs else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def cache_elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2, "i8": 1, "fp8": 1}[self.cache_dtype]

    def kv_bytes(self) -> int:
        """Algorithmic KV bytes one decode call reads (K and V, plus INT8 scales)."""
        toks = int(self.context_lens.to(torch.int64).sum().item())
        per_tok_head = 2 * self.head_dim * self.cache_elem_bytes()
        if self.cache_dtype in ("i8", "fp8"):
            per_tok_head += 2 * 4
        return toks * self.num_kv_heads * per_tok_head


def _randn(shape, gen, dtype, outlier_prob=0.0, outlier_mult=8.0):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if outlier_prob > 0.0:
        mask = torch.rand(shape, generator=gen) < outlier_prob
        x = torch.where(mask, x * outlier_mult, x)
    return x.to(dtype)


def make_custom(name: str, context_lens: List[int], num_q_heads: int, num_kv_heads: int,
                head_dim: int, block_size: int, cache_dtype: str, seed: int,
                input_dtype: torch.dtype = torch.bfloat16, softmax_scale: Optional[float] = None,
                pool_factor: float = 1.2, min_pool: int = 0, shared_prefix: int = 0,
                outlier_prob: float = 0.0, pad_entry: int = -1, extra_table_cols: int = 0,
                randomize: bool = True, placement_seed: Optional[int] = None) -> Workload:
    """Builds a workload from explicit lengths.

    ``shared_prefix`` > 0 (a multiple of block_size) makes every sequence
    start with the same physical prefix blocks (ref_count = num_seqs); the
    prefix tokens are pre-filled once.  ``context_lens`` then counts prefix
    plus suffix.
    """
    if cache_dtype not in ("f32", "bf16", "i8", "fp8"):
        raise ValueError(cache_dtype)
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    if shared_prefix % block_size:
        raise ValueError("shared prefix must be block aligned")
    B = len(context_lens)
    lens = [int(c) for c in context_lens]
    if any(c < 0 for c in lens):
        raise ValueError("negative context length")
    if shared_prefix and any(c <= shared_prefix for c in lens):
        raise ValueError("each sequence needs at least one suffix token")
    gen = torch.Generator().manual_seed(seed)

    def nblk(n):
        return (n + block_size - 1) // block_size

    prefix_blocks = shared_prefix // block_size
    need = prefix_blocks + sum(nblk(c) - prefix_blocks for c in lens) if shared_prefix else \
        sum(nblk(c) for c in lens)
    num_blocks = max(int(math.ceil(pool_factor * need)), need, min_pool, 1)
    place_gen = gen if placement_seed is None else torch.Generator().manual_seed(placement_seed)
    alloc = BlockAllocator(num_blocks, place_gen if randomize else None)

    max_blocks = max([nblk(c) for c in lens] + [1]) + extra_table_cols
    tables = torch.full((B, max_blocks), pad_entry, dtype=torch.int32)

    shared = [alloc.allocate() for _ in range(prefix_blocks)]
    for b in shared[:]:
        for _ in range(B - 1):
            alloc.share(b)

    pre_slots: List[torch.Tensor] = []
    pre_k: List[torch.Tensor] = []
    pre_v: List[torch.Tensor] = []
    q_rows, nk_rows, nv_rows, new_slots = [], [], [], []
    if shared_prefix:
        sg = torch.Generator().manual_seed(seed * 7919 + 17)
        slots = torch.tensor([shared[t // block_size] * block_size + t % block_size
                              for t in range(shared_prefix)], dtype=torch.int64)
        pre_slots.append(slots)
        pre_k.append(_randn((shared_prefix, num_kv_heads, head_dim), sg, input_dtype, outlier_prob))
        pre_v.append(_randn((shared_prefix, num_kv_heads, head_dim), sg, input_dtype, outlier_prob))

    for s, ctx in enumerate(lens):
        own = [alloc.allocate() for _ in range(nblk(ctx) - prefix_blocks)] if ctx else []
        table = shared + own
        tables[s, :len(table)] = torch.tensor(table, dtype=torch.int32) if table else tables[s, :0]
        sg = torch.Generator().manual_seed(seed * 1_000_003 + s)
        first = shared_prefix
        n_pre = max(ctx - 1 - first, 0)
        if n_pre:
            toks = range(first, first + n_pre)
            pre_slots.append(torch.tensor([table[t // block_size] * block_size + t % block_size
                                           for t in toks], dtype=torch.int64))
            pre_k.append(_randn((n_pre, num_kv_heads, head_dim), sg, input_dtype, outlier_prob))
            pre_v.append(_randn((n_pre, num_kv_heads, head_dim), sg, input_dtype, outlier_prob))
        q_rows.append(_randn((num_q_heads, head_dim), sg, input_dtype))
        nk_rows.append(_randn((num_kv_heads, head_dim), sg, input_dtype, outlier_prob))
        nv_rows.append(_randn((num_kv_heads, head_dim), sg, input_dtype, outlier_prob))
        if ctx:
            t = ctx - 1
            new_slots.append(table[t // block_size] * block_size + t % block_size)
        else:
            new_slots.append(-1)  # nothing to append for an empty sequence

    def cat(xs, shape_tail, dtype):
        return torch.cat(xs) if xs else torch.zeros((0, *shape_tail), dtype=dtype)

    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(head_dim)
    return Workload(
        name=name, num_seqs=B, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
        cache_dtype=cache_dtype, input_dtype=input_dtype, softmax_scale=scale,
        context_lens=torch.tensor(lens, dtype=torch.int32), block_tables=tables,
        prefill_slots=cat(pre_slots, (), torch.int64),
        prefill_k=cat(pre_k, (num_kv_heads, head_dim), input_dtype),
        prefill_v=cat(pre_v, (num_kv_heads, head_dim), input_dtype),
        q=torch.stack(q_rows) if q_rows else torch.zeros((0, num_q_heads, head_dim), dtype=input_dtype),
        new_k=torch.stack(nk_rows) if nk_rows else torch.zeros((0, num_kv_heads, head_dim), dtype=input_dtype),
        new_v=torch.stack(nv_rows) if nv_rows else torch.zeros((0, num_kv_heads, head_dim), dtype=input_dtype),
        new_slots=torch.tensor(new_slots, dtype=torch.int64),
        allocator=alloc,
        meta={"seed": seed, "shared_prefix": shared_prefix, "outlier_prob": outlier_prob},
    )


# The five workloads: name -> (description, builder).  Seeds are 439_000 + index.
CONFIGS = {
    "tiny": "batch 4, ctx {17,33,64,100}, 4 q / 2 kv heads, d 64, bs 16, fp32, 64-block pool",
    "llama2-7b-mha": "batch 8, ctx 4096, 32 q = 32 kv heads, d 128, bf16, bs 16, pool 1.2x",
    "llama2-70b-gqa": "batch 16, ctx U[1024,32768], 64 q / 8 kv heads, d 128, bf16, bs 16, pool 1.2x",
    "llama2-13b-int8": "batch 32, ctx 2048, 40 q = 40 kv heads, d 128, int8 cache (bf16 in, 1% x8 outliers), bs 16",
    "shared-prefix": "64 seqs, 4096-token shared prefix + U[64,512] suffix, 32 q / 8 kv heads, d 128, bf16, bs 16|256",
}

_ALIASES = {"1": "tiny", "2": "llama2-7b-mha", "3": "llama2-70b-gqa", "4": "llama2-13b-int8",
            "5": "shared-prefix"}


def canonical_name(name: str) -> str:
    return _ALIASES.get(str(name), name)


def workload_seed(name: str) -> int:
    """Base seed of a named workload: 439_000 + its index (1-based)."""
    return 439_000 + list(CONFIGS).index(canonical_name(name)) + 1


def make_workload(name: str, block_size: Optional[int] = None, batch: Optional[int] = None,
                  data_seed: Optional[int] = None, **kw) -> Workload:
    """The named workload.  ``batch`` truncates the batch (for sampled checks);
    ``data_seed`` re-draws the values (and placement) keeping every shape and
    length of the workload."""
    name = canonical_name(name)
    seed = workload_seed(name)
    gen = torch.Generator().manual_seed(seed)
    if name == "tiny":
        lens = [17, 33, 64, 100]
        wl = dict(num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=block_size or 16,
                  cache_dtype="f32", input_dtype=torch.float32, softmax_scale=1.0 / 8.0,
                  pool_factor=1.0, min_pool=64)
    elif name == "llama2-7b-mha":
        lens = [4096] * 8
        wl = dict(num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=block_size or 16,
                  cache_dtype="bf16")
    elif name == "llama2-70b-gqa":
        lens = torch.randint(1024, 32768 + 1, (16,), generator=gen).tolist()
        wl = dict(num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=block_size or 16,
                  cache_dtype="bf16")
    elif name == "llama2-13b-int8":
        lens = [2048] * 32
        wl = dict(num_q_heads=40, num_kv_heads=40, head_dim=128, block_size=block_size or 16,
                  cache_dtype="i8", outlier_prob=0.01)
    elif name == "shared-prefix":
        suffix = torch.randint(64, 512 + 1, (64,), generator=gen).tolist()
        lens = [4096 + s for s in suffix]
        wl = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=block_size or 16,
                  cache_dtype="bf16", shared_prefix=4096)
    else:
        raise KeyError(name)
    if batch is not None:
        lens = lens[:batch]
    wl.update(kw)
    return make_custom(name, lens, seed=seed if data_seed is None else data_seed, **wl)
