"""Seeded synthetic inputs for attention over a paged KV cache.

This module is shared by the tests, the bench and the oracle checks. It holds
none of the attention arithmetic: it only draws random numbers and runs a small
host-side block allocator that hands out physical blocks and writes per-sequence
block tables, the way the pages describe the memory-management layer:

* KV cache cut into fixed-size blocks, physical blocks handed out from a pool
  ("FlashAttention y PagedAttention: dos soluciones para dos cuellos de botella
  distintos", PagedAttention / "Cómo funciona", steps 1-3);
* sequences with a common prompt point at the same physical blocks (same page,
  step 4, and the conceptual block table under "En código");
* block size 16 as the general recommendation, 8..128 in the sweep ("Flash
  Attention vs Paged Attention：大语言模型注意力计算的内存管理革命", 块大小优化策略).

Layouts (fixed by the C ABI in include/pa.h):
  q            [N, Hq, D] (decode) or [N, C, Hq, D] (prefill chunk)
  k_cache      [P, Hkv, B, D]   one (block, kv-head) page is B*D contiguous
  v_cache      [P, Hkv, B, D]
  block_tables int32 [N, max_blocks]  (-1 past the sequence's last block)
  context_lens int32 [N]          tokens each query may attend to, the new
                                  tokens of this step included
  k_new/v_new  [T, Hkv, D], new_seq/new_pos int32 [T]: the tokens this step
               appends (their cache slots are poisoned until the append)

Poisoning: in correctness runs every pool block no sequence owns, and every
slot at or past a sequence's valid length, holds NaN (or +-65504), so that a
stray read shows up in the output instead of hiding behind a plausible value.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class PagedBatch:
    """One batch of paged-attention inputs, all on one device."""

    name: str
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    new_seq: torch.Tensor
    new_pos: torch.Tensor
    block_size: int
    scale: float
    chunk: int  # query tokens per sequence (1 = decode)
    info: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def num_kv_heads(self) -> int:
        return int(self.k_cache.shape[1])

    @property
    def head_dim(self) -> int:
        return int(self.k_cache.shape[3])

    @property
    def num_q_heads(self) -> int:
        return int(self.q.shape[-2])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def to(self, device) -> "PagedBatch":
        out = PagedBatch(**{k: (v.to(device) if isinstance(v, torch.Tensor) else v)
                            for k, v in self.__dict__.items()})
        out.info = dict(self.info)
        return out


# --------------------------------------------------------------------------
# Host block allocator
# --------------------------------------------------------------------------

class BlockAllocator:
    """Hands out physical block ids from a seeded random permutation of a pool.

    Unlike the toy class on the pages (one logical->physical dict, a free list),
    it keeps one table per sequence and lets a group of sequences hold the same
    ids for a common prefix. Ids come out of a shuffled pool so that logical
    neighbours are never physical neighbours.
    """

    def __init__(self, pool_blocks: int, gen: torch.Generator):
        self.pool_blocks = pool_blocks
        self.free = torch.randperm(pool_blocks, generator=gen).tolist()
        self.owned: set[int] = set()

    def take(self, n: int) -> list[int]:
        if n > len(self.free):
            raise RuntimeError(f"pool exhausted: want {n}, have {len(self.free)}")
        ids, self.free = self.free[:n], self.free[n:]
        self.owned.update(ids)
        return ids


def blocks_for(n_tokens: int, block_size: int) -> int:
    return (n_tokens + block_size - 1) // block_size


def build_tables(lens: list[int], block_size: int, gen: torch.Generator,
                 pool_factor: float = 1.25, shared_prefix_tokens: int = 0,
                 shared_group: int = 0, min_pool: int = 0):
    """Per-sequence block tables for sequences of `lens` tokens.

    Sequences 0..shared_group-1 hold the same physical ids for their first
    shared_prefix_tokens tokens (which must be a multiple of block_size).
    Returns (block_tables int32 [N, max_blocks], pool_blocks, allocator).
    """
    assert shared_prefix_tokens % block_size == 0
    n_shared = shared_prefix_tokens // block_size
    need = []
    for i, L in enumerate(lens):
        nb = blocks_for(L, block_size)
        if i < shared_group:
            assert L >= shared_prefix_tokens
            nb -= n_shared
        need.append(nb)
    total = sum(need) + (n_shared if shared_group else 0)
    pool = max(int(math.ceil(pool_factor * total)), total, min_pool, 1)
    alloc = BlockAllocator(pool, gen)
    shared_ids = alloc.take(n_shared) if shared_group else []
    max_blocks = max(1, max(blocks_for(L, block_size) for L in lens))
    bt = torch.full((len(lens), max_blocks), -1, dtype=torch.int32)
    for i, L in enumerate(lens):
        ids = (shared_ids if i < shared_group else []) + alloc.take(need[i])
        if ids:
            bt[i, : len(ids)] = torch.tensor(ids, dtype=torch.int32)
    return bt, pool, alloc


def _randn(shape, gen, dtype, std=1.0, chunk_rows=4096):
    """N(0, std^2) samples in `dtype`, drawn in fp32 row chunks (bounded temp memory)."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=gen, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[r0:r1].copy_(x)
    return out


def poison_pool(k_cache, v_cache, block_tables, valid_lens, block_size, value=float("nan")):
    """Fill every slot that no sequence may read with `value`.

    A slot is readable iff it holds position < valid_lens[b] of some sequence b.
    Blocks owned by nobody are poisoned whole; inside owned blocks the slots past
    the owner's valid length are poisoned. Shared blocks are full by construction.
    """
    P = k_cache.shape[0]
    readable = torch.zeros((P, block_size), dtype=torch.bool)
    bt = block_tables.tolist()
    for b, L in enumerate(valid_lens):
        for j in range(blocks_for(L, block_size)):
            n = min(block_size, L - j * block_size)
            readable[bt[b][j], :n] = True
    mask = ~readable  # [P, B]
    m4 = mask[:, None, :, None].expand_as(k_cache)
    k_cache.masked_fill_(m4, value)
    v_cache.masked_fill_(m4, value)


def make_batch(name: str, lens: list[int], *, num_q_heads: int, num_kv_heads: int,
               head_dim: int, block_size: int, dtype: str, seed: int, chunk: int = 1,
               q_std: float = 1.0, pool_factor: float = 1.25, shared_prefix_tokens: int = 0,
               shared_group: int = 0, poison: float | None = float("nan"),
               min_pool: int = 0, scale: float | None = None) -> PagedBatch:
    """Build a batch on the CPU.

    lens[b] is the context length after this step's append (context_lens).
    The step appends the last `chunk` tokens of every sequence (positions
    lens[b]-chunk .. lens[b]-1): their K/V rows are in k_new/v_new and their
    cache slots are poisoned until the append writes them.
    """
    gen = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    N = len(lens)
    bt, pool, alloc = build_tables(lens, block_size, gen, pool_factor,
                                   shared_prefix_tokens, shared_group, min_pool)
    k_cache = _randn((pool, num_kv_heads, block_size, head_dim), gen, dt)
    v_cache = _randn((pool, num_kv_heads, block_size, head_dim), gen, dt)
    if chunk == 1:
        q = _randn((N, num_q_heads, head_dim), gen, dt, q_std)
    else:
        q = _randn((N * chunk, num_q_heads, head_dim), gen, dt, q_std).view(N, chunk, num_q_heads, head_dim)
    new_seq, new_pos = [], []
    for b, L in enumerate(lens):
        c = min(chunk, L)
        new_seq += [b] * c
        new_pos += list(range(L - c, L))
    T = len(new_seq)
    k_new = _randn((max(T, 1), num_kv_heads, head_dim), gen, dt)[:T]
    v_new = _randn((max(T, 1), num_kv_heads, head_dim), gen, dt)[:T]
    if poison is not None:
        prior = [L - min(chunk, L) for L in lens]
        poison_pool(k_cache, v_cache, bt, prior, block_size, poison)
    return PagedBatch(
        name=name, q=q, k_cache=k_cache, v_cache=v_cache, block_tables=bt,
        context_lens=torch.tensor(lens, dtype=torch.int32), k_new=k_new, v_new=v_new,
        new_seq=torch.tensor(new_seq, dtype=torch.int32),
        new_pos=torch.tensor(new_pos, dtype=torch.int32), block_size=block_size,
        scale=(1.0 / math.sqrt(head_dim)) if scale is None else scale, chunk=chunk,
        info=dict(seed=seed, dtype=dtype, pool_blocks=pool, q_std=q_std,
                  shared_prefix_tokens=shared_prefix_tokens, shared_group=shared_group,
                  owned_blocks=len(alloc.owned)))


# --------------------------------------------------------------------------
# The five workloads (seeds 0..4 in this order)
# --------------------------------------------------------------------------

def tiny_fp32(poison=float("nan")) -> PagedBatch:
    """4 sequences of {1,7,16,33} tokens, 2 q heads on 1 KV head, D=64, B=16, pool of 16."""
    return make_batch("tiny_fp32", [1, 7, 16, 33], num_q_heads=2, num_kv_heads=1, head_dim=64,
                      block_size=16, dtype="f32", seed=0, pool_factor=1.0, min_pool=16,
                      poison=poison)


def llama_decode_lens(num_seqs=64, lo=512, hi=4096, seed=1) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (num_seqs,), generator=g).tolist()


def llama_decode(num_seqs=64, lo=512, hi=4096, block_size=16, dtype="f16",
                 poison=float("nan"), seed=1) -> PagedBatch:
    """Llama-3-8B-shaped single-layer decode: 32 q / 8 KV heads, D=128, L ~ U[lo, hi]."""
    lens = llama_decode_lens(num_seqs, lo, hi, seed + 1000)
    return make_batch("llama_decode", lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=block_size, dtype=dtype, seed=seed, poison=poison)


def long_context(num_seqs=4, context_len=100_000, block_size=16, dtype="f16",
                 poison=float("nan"), seed=2) -> PagedBatch:
    """Long-context split-KV decode: 4 x 100k tokens, q ~ N(0, 2) for a peaky softmax."""
    return make_batch("long_context", [context_len] * num_seqs, num_q_heads=32, num_kv_heads=8,
                      head_dim=128, block_size=block_size, dtype=dtype, seed=seed,
                      q_std=math.sqrt(2.0), pool_factor=1.0, poison=poison)


def chat_trace_lens(num_seqs=256, median=300.0, sigma=1.0, lo=16, hi=8192,
                    shared_prefix=1024, shared_group=128, seed=3) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    x = torch.empty(num_seqs, dtype=torch.float64).log_normal_(math.log(median), sigma, generator=g)
    lens = x.round().clamp(lo, hi).to(torch.int64).tolist()
    for i in range(shared_group):
        lens[i] = min(hi, shared_prefix + lens[i])
    return lens


def chat_trace(block_size=16, num_seqs=256, dtype="f16", poison=float("nan"), seed=3) -> PagedBatch:
    """High-concurrency chat trace: lognormal lengths, half the batch sharing a 1024-token prefix."""
    shared_group = num_seqs // 2
    lens = chat_trace_lens(num_seqs, shared_group=shared_group, seed=seed + 1000)
    return make_batch(f"chat_trace_B{block_size}", lens, num_q_heads=32, num_kv_heads=8,
                      head_dim=128, block_size=block_size, dtype=dtype, seed=seed,
                      shared_prefix_tokens=1024, shared_group=shared_group, poison=poison)


def prefill_lens(num_seqs=8, lo=2048, hi=8192, chunk=512, seed=4) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    ctx = torch.randint(lo, hi + 1, (num_seqs,), generator=g)
    return (ctx + chunk).tolist()


def prefill_chunk(num_seqs=8, chunk=512, lo=2048, hi=8192, block_size=16, dtype="bf16",
                  poison=float("nan"), seed=4) -> PagedBatch:
    """Chunked prefill: `chunk` new causal query tokens after a paged context ~ U[lo, hi]."""
    lens = prefill_lens(num_seqs, lo, hi, chunk, seed + 1000)
    return make_batch("prefill_chunk", lens, num_q_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=block_size, dtype=dtype, seed=seed, chunk=chunk, poison=poison)


# --------------------------------------------------------------------------
# Byte and flop accounting (used by the bench and its unit tests)
# --------------------------------------------------------------------------

def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V rows of one token across all layers."""
    return num_layers * num_kv_heads * head_dim * 2 * elem_bytes


def decode_kv_bytes(context_lens, num_kv_heads: int, head_dim: int, elem_bytes: int,
                    block_tables=None, block_size: int | None = None, unique: bool = False) -> int:
    """Algorithmic K+V bytes one decode pass must read.

    logical: every sequence's own tokens; unique: a physical slot read by
    several sequences (a shared prefix) is counted once.
    """
    lens = [int(x) for x in context_lens]
    per_token = num_kv_heads * head_dim * 2 * elem_bytes
    if not unique:
        return sum(lens) * per_token
    slots = set()
    bt = block_tables.tolist()
    for b, L in enumerate(lens):
        for j in range(blocks_for(L, block_size)):
            n = min(block_size, L - j * block_size)
            slots.update((bt[b][j], r) for r in range(n))
    return len(slots) * per_token


def prefill_flops(context_lens, chunk: int, num_q_heads: int, head_dim: int) -> int:
    """Useful tensor flops of a causal chunk: 2 matmuls x 2 flop x visible keys per query row."""
    total = 0
    for L in context_lens:
        L = int(L)
        visible = sum(L - chunk + i + 1 for i in range(chunk))
        total += 4 * num_q_heads * head_dim * visible
    return total
