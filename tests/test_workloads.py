"""The seeded input generators (workloads.py) on the CPU.

Every parity test and the bench draw their inputs here, so the generators are
checked against the rules they promise: block tables that only share the
intended prefix blocks, poison on exactly the slots no sequence may read, the
append slots of the step, the length recipes of the five workloads, and
determinism per seed.
"""
import math

import numpy as np
import torch

import workloads as W


def _readable_slots(batch, lens):
    """(block, slot) pairs sequence b may read: positions < lens[b]."""
    B = batch.block_size
    bt = batch.block_tables.tolist()
    out = set()
    for b, L in enumerate(lens):
        for pos in range(L):
            out.add((bt[b][pos // B], pos % B))
    return out


def test_block_tables_are_valid_and_private_unless_shared():
    lens = [300, 200, 129, 50, 1, 16, 17]
    b = W.make_batch("t", lens, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16, dtype="f16", seed=3,
                     shared_prefix_tokens=128, shared_group=3)
    bt = b.block_tables
    P = b.num_blocks
    owners = {}
    for s, L in enumerate(lens):
        nb = W.blocks_for(L, 16)
        row = bt[s].tolist()
        assert all(0 <= x < P for x in row[:nb])
        assert all(x == -1 for x in row[nb:])
        for j, x in enumerate(row[:nb]):
            owners.setdefault(x, set()).add((s, j))
    shared = {x for x, o in owners.items() if len(o) > 1}
    # exactly the first 8 logical blocks of sequences 0..2, the same ids in the same order
    assert shared == set(bt[0, :8].tolist())
    assert torch.equal(bt[0, :8], bt[1, :8]) and torch.equal(bt[0, :8], bt[2, :8])
    for x in shared:
        assert owners[x] == {(s, j) for s in range(3) for j in range(8) if bt[s, j].item() == x}
    assert b.info["pool_blocks"] >= math.ceil(1.25 * (sum(W.blocks_for(L, 16) for L in lens) - 2 * 8))


def test_poison_marks_exactly_the_unreadable_slots():
    lens = [1, 15, 16, 17, 100, 33]
    for B in (8, 16, 32):
        b = W.make_batch("t", lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=B, dtype="f32", seed=5)
        prior = [L - 1 for L in lens]  # the step's own tokens are not in the cache yet
        readable = _readable_slots(b, prior)
        k = b.k_cache.numpy()
        for blk in range(b.num_blocks):
            for slot in range(B):
                finite = np.isfinite(k[blk, :, slot, :]).all()
                assert finite == ((blk, slot) in readable), (B, blk, slot)
        assert np.isnan(b.v_cache.numpy()).any() and np.isfinite(b.k_new.numpy()).all()


def test_append_slots_are_the_last_chunk_positions():
    lens = [520, 600, 3, 512]
    b = W.make_batch("t", lens, num_q_heads=4, num_kv_heads=1, head_dim=64, block_size=16, dtype="bf16", seed=7,
                     chunk=4)
    assert b.q.shape == (4, 4, 4, 64)
    want_seq, want_pos = [], []
    for s, L in enumerate(lens):
        c = min(4, L)
        want_seq += [s] * c
        want_pos += list(range(L - c, L))
    assert b.new_seq.tolist() == want_seq and b.new_pos.tolist() == want_pos
    assert b.k_new.shape == (len(want_seq), 1, 64)
    # every append slot is poisoned before the step
    B = b.block_size
    for s, p in zip(want_seq, want_pos):
        blk = b.block_tables[s, p // B].item()
        assert torch.isnan(b.k_cache[blk, :, p % B].float()).all()


def test_same_seed_same_batch_and_rank_offsets_differ():
    a = W.make_batch("t", [40, 70], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, dtype="f16", seed=11)
    b = W.make_batch("t", [40, 70], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, dtype="f16", seed=11)
    c = W.make_batch("t", [40, 70], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, dtype="f16", seed=111)
    for name in ("q", "k_cache", "v_cache", "block_tables", "k_new", "v_new"):
        x, y = getattr(a, name), getattr(b, name)
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.float16 else x,
                           y.view(torch.int16) if y.dtype == torch.float16 else y), name
    assert not torch.equal(a.q, c.q)


def test_workload_length_recipes():
    llama = W.llama_decode_lens(seed=1001)
    assert len(llama) == 64 and min(llama) >= 512 and max(llama) <= 4096
    assert sum(llama) == 154001  # the visible tokens the Llama-config byte accounting is quoted on
    chat = W.chat_trace_lens(seed=1003)
    assert len(chat) == 256 and min(chat) >= 16 and max(chat) <= 8192
    assert all(L >= 1024 + 16 for L in chat[:128])  # the sharers hold the 1024-token prompt plus their own
    own = [L - 1024 for L in chat[:128]] + chat[128:]
    assert 200 < float(np.median(own)) < 450  # lognormal around 300
    pre = W.prefill_lens(seed=1004)
    assert len(pre) == 8 and all(2048 + 512 <= L <= 8192 + 512 for L in pre)


def test_tiny_and_byte_accounting():
    t = W.tiny_fp32()
    assert t.context_lens.tolist() == [1, 7, 16, 33] and t.num_blocks == 16
    assert t.q.dtype == torch.float32 and t.num_q_heads == 2 and t.num_kv_heads == 1 and t.head_dim == 64
    # 128 KiB of K+V per token for 32 layers x 8 KV heads x 128 dims x fp16
    assert W.kv_bytes_per_token(32, 8, 128, 2) == 128 * 1024
