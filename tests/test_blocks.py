"""Host block manager (reference counts, fork, copy-on-write, release) on the CPU."""
import json
import os

import pytest

from paged_kv_cache_475_b200.blocks import BlockManager, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_on_demand_allocation():
    m = BlockManager(8, 16)
    m.allocate(0, 60)                      # 60 tokens occupy 4 blocks of 16
    assert len(m.block_table(0)) == 4 and m.num_free == 4
    slots = [m.append_slot(0)[0] for _ in range(4)]   # tokens 60..63 fill block 3
    assert len(m.block_table(0)) == 4
    assert slots == [m.block_table(0)[3] * 16 + o for o in (12, 13, 14, 15)]
    m.append_slot(0)                       # token 64 opens block 4
    assert len(m.block_table(0)) == 5 and m.num_free == 3
    m.check()


def test_fork_shares_and_copy_on_write():
    m = BlockManager(10, 16)
    m.allocate(1, 40)                      # blocks a, b, c (c half full)
    m.fork(1, 2)
    assert m.block_table(1) == m.block_table(2)
    shared_last = m.block_table(1)[2]
    assert m.refcount[shared_last] == 2
    slot, pair = m.append_slot(2)          # token 40 of seq 2 lands in the shared block
    assert pair is not None and pair[0] == shared_last
    assert m.block_table(2)[2] == pair[1] != shared_last
    assert slot == pair[1] * 16 + 8
    assert m.refcount[shared_last] == 1 and m.refcount[pair[1]] == 1
    slot1, pair1 = m.append_slot(1)        # seq 1 now owns its block alone: no copy
    assert pair1 is None and slot1 == shared_last * 16 + 8
    assert m.block_table(1)[:2] == m.block_table(2)[:2]   # full prefix blocks still shared
    m.check()


def test_pages_block_table_example():
    """request_1 -> [3, 7, 12] and request_2 -> [3, 7, 9] share blocks 3 and 7 (a common 32-token prompt)."""
    with open(os.path.join(GOLDEN, "block_table_example.json")) as f:
        g = json.load(f)
    B = g["block_size"]
    m = BlockManager(13, B)
    m.free_list = [b for b in range(12, -1, -1) if b not in (3, 7, 12, 9)] + [9, 12, 7, 3]
    m.allocate(1, 32)                      # the shared prompt: blocks 3 and 7
    m.fork(1, 2)
    m.append_slot(1)                       # token 32 of request_1 opens a new block
    m.append_slot(2)
    assert m.block_table(1) == g["block_tables"]["request_1"]
    assert m.block_table(2) == g["block_tables"]["request_2"]
    assert sorted(b for b in range(13) if m.refcount[b] == 2) == g["shared_blocks"]
    m.check()


def test_free_returns_blocks_only_when_unreferenced():
    m = BlockManager(6, 8)
    m.allocate(0, 20)
    m.fork(0, 1)
    m.free(0)
    assert m.num_free == 3                 # seq 1 still holds the 3 blocks
    m.free(1)
    assert m.num_free == 6
    m.check()


def test_out_of_blocks():
    m = BlockManager(2, 8)
    m.allocate(0, 16)
    with pytest.raises(OutOfBlocks):
        m.append_slot(0)
    with pytest.raises(OutOfBlocks):
        m.allocate(1, 1)


def test_tables_tensor_padding():
    m = BlockManager(8, 4)
    m.allocate(0, 9)
    m.allocate(1, 1)
    t = m.tables_tensor([0, 1])
    assert t.shape == (2, 3) and t[1, 1:].tolist() == [-1, -1]


def test_random_operation_sequences_keep_the_invariants():
    """Random allocate / fork / append / free sequences against a model of each sequence's tokens: the
    reference counts always equal the table references, a token's slot never moves, two live
    sequences never write the same slot, and a copy-on-write pair always copies the block the
    sequence was reading into a private one."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    ops = st.lists(st.tuples(st.sampled_from(["alloc", "fork", "append", "free"]), st.integers(0, 7),
                             st.integers(0, 7), st.integers(0, 70)), max_size=60)

    @settings(max_examples=150, deadline=None)
    @given(ops)
    def run(seq_ops):
        B = 8
        m = BlockManager(48, B)
        content = {}   # seq -> list of (physical block, offset) of its tokens, logical order
        for op, a, b, n in seq_ops:
            try:
                if op == "alloc" and a not in m.tables:
                    m.allocate(a, n)
                    t = m.block_table(a)
                    content[a] = [(t[p // B], p % B) for p in range(n)]
                elif op == "fork" and a in m.tables and b not in m.tables:
                    m.fork(a, b)
                    content[b] = list(content[a])
                elif op == "append" and a in m.tables:
                    before = list(content[a])
                    slot, pair = m.append_slot(a)
                    t = m.block_table(a)
                    pos = len(before)
                    assert slot == t[pos // B] * B + pos % B
                    if pair is not None:
                        src, dst = pair
                        assert src != dst and m.refcount[dst] == 1 and t[pos // B] == dst
                        # the tokens already in the copied block move to the private copy
                        before = [(dst if blk == src and i // B == pos // B else blk, off)
                                  for i, (blk, off) in enumerate(before)]
                    content[a] = before + [(slot // B, slot % B)]
                    # no other live sequence may own the slot just written
                    for s, toks in content.items():
                        if s != a:
                            assert (slot // B, slot % B) not in toks
                elif op == "free" and a in m.tables:
                    m.free(a)
                    del content[a]
            except OutOfBlocks:
                pass
            m.check()
            for s, toks in content.items():
                t = m.block_table(s)
                assert [(t[i // B], i % B) for i in range(len(toks))] == toks

    run()
