"""Host-side block manager: per-sequence block tables over a shared pool, with reference counts.

This is the memory-management layer the kernels read through ("FlashAttention
y PagedAttention", PagedAttention "Cómo funciona", steps 1-4):
  * the cache is cut into fixed-size blocks; a sequence's table maps logical
    block j (tokens j*B .. j*B+B-1) to a physical block;
  * blocks are handed out on demand, one more only when the last one is full;
  * sequences with a common prefix point at the same physical blocks
    (fork), and a sequence that writes into a shared block first gets its own
    copy of it (copy-on-write);
  * blocks are returned to the pool when no sequence holds them any more
    ("Flash Attention vs Paged Attention", Paged Attention的内存管理创新).

Unlike the pages' toy class (one logical->physical dict and a free list, no
sharing), every sequence has its own table and every physical block a
reference count. The manager only does bookkeeping; the copy itself is
pa_copy_blocks on the pairs it returns, and the slot of each new token goes
to pa_reshape_and_cache (or pa_decode_append writes it).
"""
from __future__ import annotations

import torch


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_list = list(range(num_blocks - 1, -1, -1))  # pop() hands out low ids first
        self.refcount = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lengths: dict[int, int] = {}

    # -- pool ---------------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self.free_list)

    def _take(self) -> int:
        if not self.free_list:
            raise OutOfBlocks("no free physical block")
        b = self.free_list.pop()
        self.refcount[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.refcount[b] -= 1
        assert self.refcount[b] >= 0
        if self.refcount[b] == 0:
            self.free_list.append(b)

    # -- sequences ----------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> list[int]:
        """New sequence holding num_tokens tokens (its prompt): ceil(n / B) fresh blocks."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        need = (num_tokens + self.block_size - 1) // self.block_size
        if need > self.num_free:
            raise OutOfBlocks(f"need {need} blocks, {self.num_free} free")
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lengths[seq] = num_tokens
        return list(self.tables[seq])

    def fork(self, parent: int, child: int) -> list[int]:
        """child starts as parent: same tokens, same physical blocks (reference counts + 1)."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        table = list(self.tables[parent])
        for b in table:
            self.refcount[b] += 1
        self.tables[child] = table
        self.lengths[child] = self.lengths[parent]
        return list(table)

    def append_slot(self, seq: int) -> tuple[int, tuple[int, int] | None]:
        """Reserve the slot of seq's next token; returns (slot, copy_pair or None).

        A new block is taken when the last one is full (or there is none). If
        the token lands in a block other sequences still share, that block is
        copied first: copy_pair = (shared block, private copy) for
        pa_copy_blocks, and seq's table now points at the copy.
        """
        table = self.tables[seq]
        pos = self.lengths[seq]
        j, off = divmod(pos, self.block_size)
        pair = None
        if j == len(table):
            table.append(self._take())
        elif self.refcount[table[j]] > 1:
            src = table[j]
            dst = self._take()
            self._release(src)
            table[j] = dst
            pair = (src, dst)
        self.lengths[seq] = pos + 1
        return table[j] * self.block_size + off, pair

    def free(self, seq: int) -> None:
        for b in self.tables.pop(seq):
            self._release(b)
        del self.lengths[seq]

    # -- views ----------------------------------------------------------------
    def block_table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def tables_tensor(self, seqs: list[int], max_blocks: int | None = None) -> torch.Tensor:
        """int32 [len(seqs), max_blocks] block tables, -1 past each sequence's blocks."""
        width = max_blocks if max_blocks is not None else max((len(self.tables[s]) for s in seqs), default=1)
        out = torch.full((len(seqs), max(width, 1)), -1, dtype=torch.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            if len(t) > width:
                raise ValueError(f"sequence {s} has {len(t)} blocks > {width}")
            if t:
                out[i, : len(t)] = torch.tensor(t, dtype=torch.int32)
        return out

    def check(self) -> None:
        """Invariants: reference counts equal table references; free blocks are unreferenced."""
        counts = [0] * self.num_blocks
        for t in self.tables.values():
            for b in t:
                counts[b] += 1
        assert counts == self.refcount, "reference counts out of sync"
        assert sorted(self.free_list) == [b for b in range(self.num_blocks) if counts[b] == 0]
        for s, t in self.tables.items():
            assert len(t) == (self.lengths[s] + self.block_size - 1) // self.block_size
