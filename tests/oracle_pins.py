"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each pin takes the oracle module as an argument so that tests/test_oracle.py
can run it on the real oracle and, with a planted mistake, on a mutated one
(tests/test_oracle_mutants.py): every plausible slip (a dropped scale, a
wrong head or block index, an off-by-one causal limit, a merge that forgets a
weight) must make at least one pin fail.

Nothing here calls the CUDA library. Independent ways of computing the same
thing used below:
  * walk_sequence: reads the pool token by token (no page gather);
  * torch.nn.functional.scaled_dot_product_attention in float64 (library);
  * a pure-Python brute force with math.exp over the token walk;
  * closed forms: uniform scores -> mean of V; dominant key -> its V row;
    one token -> V[0];
  * invariants: block permutation, shared vs private blocks, eq. (4) block sums.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def walk_sequence(cache, bt_row, n, kv_head):
    """Token-by-token read of one sequence: logical block t // B, row t % B (float64)."""
    B = cache.shape[2]
    rows = [cache[int(bt_row[t // B]), kv_head, t % B].to(torch.float64) for t in range(n)]
    if not rows:
        return torch.zeros((0, cache.shape[3]), dtype=torch.float64)
    return torch.stack(rows)


def small_decode(seed=11, dtype="f32", D=64, Hq=4, Hkv=2, B=16, lens=(1, 5, 16, 17, 40)):
    return W.make_batch("pin", list(lens), num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                        block_size=B, dtype=dtype, seed=seed)


def small_prefill(seed=12, dtype="f32", D=64, Hq=4, Hkv=2, B=8, lens=(9, 20, 33), C=6):
    return W.make_batch("pin", list(lens), num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                        block_size=B, dtype=dtype, seed=seed, chunk=C)


def appended(P, b):
    """The batch's caches after the oracle's own append (slots from the oracle)."""
    slots = P.slot_mapping(b.block_tables, b.new_seq, b.new_pos, b.block_size)
    return P.reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache, slots)


# ----------------------------------------------------------------------------
# Pins
# ----------------------------------------------------------------------------

def pin_uniform_scores_mean_of_v(P):
    """q = 0: every visible key has the same score, so the output is the mean of V."""
    for b in (small_decode(), small_prefill()):
        kc, vc = appended(P, b)
        q = torch.zeros_like(b.q)
        out = P.attention(q, kc, vc, b.block_tables, b.context_lens, b.scale)
        G = b.num_q_heads // b.num_kv_heads
        C = b.chunk
        out4 = out[:, None] if C == 1 else out
        for s in range(b.num_seqs):
            L = int(b.context_lens[s])
            for h in range(b.num_q_heads):
                Vs = walk_sequence(vc, b.block_tables[s], L, h // G).numpy()
                for i in range(C):
                    n = L - C + i + 1
                    np.testing.assert_allclose(out4[s, i, h], Vs[:n].mean(0), rtol=0, atol=1e-12)


def pin_dominant_key(P):
    """q = lam * K[j]: key j's score dominates by hundreds, so the output is V[j]."""
    b = small_decode(seed=21, lens=(3, 16, 33, 50))
    kc, vc = appended(P, b)
    G = b.num_q_heads // b.num_kv_heads
    gen = torch.Generator().manual_seed(5)
    q = torch.zeros_like(b.q)
    target = {}
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        for h in range(b.num_q_heads):
            Ks = walk_sequence(kc, b.block_tables[s], L, h // G)
            j = int(torch.randint(0, L, (1,), generator=gen))
            q[s, h] = (60.0 * Ks[j]).to(q.dtype)
            target[(s, h)] = walk_sequence(vc, b.block_tables[s], L, h // G)[j].numpy()
    out = P.attention(q, kc, vc, b.block_tables, b.context_lens, b.scale)
    for (s, h), v in target.items():
        np.testing.assert_allclose(out[s, h], v, rtol=0, atol=1e-9)


def pin_single_token(P):
    """L = 1: the softmax over one key is 1, so the output is that key's V row exactly."""
    b = small_decode(seed=31, lens=(1, 1, 1))
    kc, vc = appended(P, b)
    out = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    G = b.num_q_heads // b.num_kv_heads
    for s in range(3):
        for h in range(b.num_q_heads):
            v0 = walk_sequence(vc, b.block_tables[s], 1, h // G)[0].numpy()
            assert np.array_equal(out[s, h], v0)


def pin_block_permutation(P):
    """Relabelling physical blocks (pool and tables together) leaves the output bit-identical."""
    for b in (small_decode(seed=41), small_prefill(seed=42)):
        kc, vc = appended(P, b)
        ref = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
        Pn = kc.shape[0]
        perm = torch.randperm(Pn, generator=torch.Generator().manual_seed(7))
        kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
        kc2[perm] = kc
        vc2[perm] = vc
        bt = b.block_tables.clone().long()
        bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
        out = P.attention(b.q, kc2, vc2, bt2, b.context_lens, b.scale)
        assert np.array_equal(ref, out)


def pin_shared_vs_private(P):
    """Sequences reading a shared prefix through the same block ids equal private copies."""
    lens = [48, 40, 70, 19]
    b = W.make_batch("shared", lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=8,
                     dtype="f16", seed=51, shared_prefix_tokens=16, shared_group=3,
                     pool_factor=2.0)
    kc, vc = appended(P, b)
    ref = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    bt = b.block_tables.clone()
    used = set(bt[bt >= 0].tolist())
    spare = [i for i in range(kc.shape[0]) if i not in used]
    kc2, vc2 = kc.clone(), vc.clone()
    for s in (1, 2):  # give sequences 1 and 2 private copies of the shared blocks
        for j in range(2):
            src, dst = int(bt[s, j]), spare.pop()
            kc2[dst], vc2[dst] = kc[src], vc[src]
            bt[s, j] = dst
    assert bt[0, 0] != bt[1, 0]
    out = P.attention(b.q, kc2, vc2, bt, b.context_lens, b.scale)
    assert np.array_equal(ref, out)


def pin_eq4_block_sums(P):
    """[FvP] eq. (4): attention as per-block softmax sums equals the token-wise sum.

    Partitions of one block (P = B), of several blocks, and of the whole
    sequence, merged with the log-sum-exp rule, all give the direct result;
    the merge does not depend on the order of the partitions.
    """
    b = small_decode(seed=61, lens=(1, 9, 16, 31, 64, 77))
    kc, vc = appended(P, b)
    ref = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    for part in (b.block_size, 2 * b.block_size, 80):
        o, m, l = P.splitkv_partials(b.q, kc, vc, b.block_tables, b.context_lens, b.scale, part)
        np.testing.assert_allclose(P.merge(o, m, l), ref, rtol=0, atol=1e-12)
        perm = np.random.default_rng(3).permutation(o.shape[2])
        np.testing.assert_allclose(P.merge(o[:, :, perm], m[:, :, perm], l[:, :, perm]), ref,
                                   rtol=0, atol=1e-12)


def pin_partials_closed_form(P):
    """A single partition's state: l_p = sum exp(s - m_p) >= 1 and o_p / l_p = the attention."""
    b = small_decode(seed=62, lens=(5, 33))
    kc, vc = appended(P, b)
    ref = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    o, m, l = P.splitkv_partials(b.q, kc, vc, b.block_tables, b.context_lens, b.scale, 64)
    assert o.shape[2] == 1
    assert (l[:, :, 0] >= 1.0).all()
    np.testing.assert_allclose(o[:, :, 0] / l[:, :, 0, None], ref, rtol=0, atol=1e-12)
    # m_p is the largest scaled score of the partition
    G = b.num_q_heads // b.num_kv_heads
    for s in range(2):
        L = int(b.context_lens[s])
        for h in range(b.num_q_heads):
            Ks = walk_sequence(kc, b.block_tables[s], L, h // G).numpy()
            smax = max(b.scale * float(np.dot(Ks[t], b.q[s, h].double().numpy())) for t in range(L))
            assert abs(m[s, h, 0] - smax) < 1e-12


def pin_merge_empty(P):
    """Empty partitions (l = 0) drop out; a row with none is zero."""
    rng = np.random.default_rng(0)
    o = rng.standard_normal((2, 3, 4, 8))
    m = rng.standard_normal((2, 3, 4))
    l = rng.uniform(1, 3, (2, 3, 4))
    ref = P.merge(o[:, :, :2], m[:, :, :2], l[:, :, :2])
    o2, m2, l2 = o.copy(), m.copy(), l.copy()
    o2[:, :, 2:], m2[:, :, 2:], l2[:, :, 2:] = 0.0, -np.inf, 0.0
    np.testing.assert_allclose(P.merge(o2, m2, l2), ref, rtol=0, atol=1e-14)
    l3 = np.zeros_like(l)
    assert not P.merge(o2, m2, l3).any()
    # one live partition: the output is o/l regardless of m
    np.testing.assert_allclose(P.merge(o[:, :, :1], m[:, :, :1] + 50.0, l[:, :, :1]),
                               o[:, :, 0] / l[:, :, 0, None], rtol=1e-14, atol=0)


def pin_torch_sdpa(P):
    """torch's CPU scaled_dot_product_attention in float64 on independently walked K/V."""
    for b in (small_decode(seed=71, dtype="f16"), small_prefill(seed=72, dtype="bf16")):
        kc, vc = appended(P, b)
        out = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
        q4 = b.q[:, None] if b.chunk == 1 else b.q
        G = b.num_q_heads // b.num_kv_heads
        C = b.chunk
        for s in range(b.num_seqs):
            L = int(b.context_lens[s])
            Ks = torch.stack([walk_sequence(kc, b.block_tables[s], L, kh) for kh in range(b.num_kv_heads)])
            Vs = torch.stack([walk_sequence(vc, b.block_tables[s], L, kh) for kh in range(b.num_kv_heads)])
            Ks = Ks.repeat_interleave(G, dim=0)[None]       # [1, Hq, L, D]
            Vs = Vs.repeat_interleave(G, dim=0)[None]
            qs = q4[s].to(torch.float64).transpose(0, 1)[None]  # [1, Hq, C, D]
            pos = torch.arange(L - C, L)[:, None]
            mask = torch.arange(L)[None, :] <= pos          # [C, L]
            ref = F.scaled_dot_product_attention(qs, Ks, Vs, attn_mask=mask, scale=b.scale)
            ref = ref[0].transpose(0, 1).numpy()            # [C, Hq, D]
            got = out[s][None] if C == 1 else out[s]
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_brute_force(P):
    """Pure-Python loops over a token-by-token walk of the pool, math.exp, no arrays."""
    b = small_prefill(seed=81, D=8, Hq=4, Hkv=2, B=4, lens=(3, 6, 11), C=3)
    kc, vc = appended(P, b)
    out = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    B, G = b.block_size, b.num_q_heads // b.num_kv_heads
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        for i in range(b.chunk):
            for h in range(b.num_q_heads):
                qv = [float(x) for x in b.q[s, i, h]]
                n = L - b.chunk + i + 1
                scores = []
                for t in range(n):
                    blk, r = int(b.block_tables[s][t // B]), t % B
                    kv = [float(x) for x in kc[blk, h // G, r]]
                    scores.append(b.scale * sum(a * c for a, c in zip(qv, kv)))
                mx = max(scores)
                ws = [math.exp(x - mx) for x in scores]
                tot = sum(ws)
                for d in range(b.head_dim):
                    acc = 0.0
                    for t in range(n):
                        blk, r = int(b.block_tables[s][t // B]), t % B
                        acc += ws[t] * float(vc[blk, h // G, r, d])
                    assert abs(out[s, i, h, d] - acc / tot) < 1e-12


def pin_prefill_rows_are_truncated_decodes(P):
    """Query i of a chunk equals a decode over the first L-C+i+1 tokens; C = 1 is decode."""
    b = small_prefill(seed=91, lens=(12, 30), C=5)
    kc, vc = appended(P, b)
    out = P.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale)
    for i in range(b.chunk):
        lens_i = b.context_lens - b.chunk + i + 1
        dec = P.attention(b.q[:, i], kc, vc, b.block_tables, lens_i, b.scale)
        assert np.array_equal(out[:, i], dec)


def pin_page_example_slots(P):
    """The pages' block-table example: slots follow the hand-worked ranges; shared blocks agree."""
    with open(os.path.join(GOLDEN, "block_table_example.json")) as f:
        g = json.load(f)
    B = g["block_size"]
    names = ["request_1", "request_2"]
    bt = torch.tensor([g["block_tables"][n] for n in names], dtype=torch.int32)
    seq = torch.tensor([0] * 48 + [1] * 48, dtype=torch.int32)
    pos = torch.tensor(list(range(48)) * 2, dtype=torch.int32)
    slots = P.slot_mapping(bt, seq, pos, B)
    expect = []
    for n in names:
        for p0, p1, first in g["expected_slot_ranges_by_hand"][n]:
            expect += list(range(first, first + (p1 - p0)))
    assert slots.tolist() == expect
    # both requests see the same 32-token prefix through blocks 3 and 7
    gen = torch.Generator().manual_seed(1)
    kc = torch.randn(13, 1, B, 16, generator=gen, dtype=torch.float64)
    vc = torch.randn(13, 1, B, 16, generator=gen, dtype=torch.float64)
    q = torch.randn(1, 2, 16, generator=gen, dtype=torch.float64).expand(2, 2, 16).contiguous()
    lens = torch.tensor([32, 32], dtype=torch.int32)
    out = P.attention(q, kc, vc, bt, lens, 0.25)
    assert np.array_equal(out[0], out[1])
    lens = torch.tensor([48, 48], dtype=torch.int32)
    out = P.attention(q, kc, vc, bt, lens, 0.25)
    assert not np.allclose(out[0], out[1])


def pin_cache_write(P):
    """Append: written rows equal the new rows bit for bit, other slots keep their bits, slot < 0 writes nothing."""
    b = small_prefill(seed=101, dtype="bf16", lens=(7, 19, 26), C=4)
    slots = P.slot_mapping(b.block_tables, b.new_seq, b.new_pos, b.block_size)
    slots = slots.copy()
    slots[1] = -1
    kc, vc = P.reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache, slots)
    B = b.block_size
    touched = set()
    for t, s in enumerate(slots.tolist()):
        if s < 0:
            continue
        touched.add((s // B, s % B))
        assert torch.equal(kc[s // B, :, s % B].view(torch.int16), b.k_new[t].view(torch.int16))
        assert torch.equal(vc[s // B, :, s % B].view(torch.int16), b.v_new[t].view(torch.int16))
        # the slot is the new token's own position in its sequence
        seq, pos = int(b.new_seq[t]), int(b.new_pos[t])
        assert int(b.block_tables[seq][pos // B]) == s // B and pos % B == s % B
    mask = torch.ones(kc.shape[0], B, dtype=torch.bool)
    for blk, r in touched:
        mask[blk, r] = False
    same = kc.view(torch.int16)[:, :, :][mask[:, None, :, None].expand_as(kc)]
    orig = b.k_cache.view(torch.int16)[mask[:, None, :, None].expand_as(kc)]
    assert torch.equal(same, orig)
    assert len(set(slots[slots >= 0].tolist())) == int((slots >= 0).sum())


def pin_bytes_per_token(P=None):
    """128 KiB of KV per token for the Llama-3-8B-class shape on the pages."""
    with open(os.path.join(GOLDEN, "kv_bytes_per_token.json")) as f:
        g = json.load(f)
    per = W.kv_bytes_per_token(g["num_layers"], g["num_kv_heads"], g["head_dim"], g["elem_bytes"])
    assert per == g["kv_bytes_per_token"] == 128 * 1024
    gib = per * g["tokens"] / 2**30
    assert abs(gib - 12.207) < 1e-3 and abs(gib - g["page_quote_gib"]) < 0.7


def pin_copy_blocks(P):
    """Block copies: destination blocks take the source blocks' bits, every other block keeps its own."""
    gen = torch.Generator().manual_seed(9)
    sk = torch.randn(6, 2, 4, 8, generator=gen).to(torch.bfloat16)
    sv = torch.randn(6, 2, 4, 8, generator=gen).to(torch.bfloat16)
    dk = torch.randn(5, 2, 4, 8, generator=gen).to(torch.bfloat16)
    dv = torch.randn(5, 2, 4, 8, generator=gen).to(torch.bfloat16)
    src, dst = [4, 0, 4], [1, 3, 0]
    ok_, ov_ = P.copy_blocks(dk, dv, sk, sv, src, dst)
    for s_, d_ in zip(src, dst):
        assert torch.equal(ok_[d_].view(torch.int16), sk[s_].view(torch.int16))
        assert torch.equal(ov_[d_].view(torch.int16), sv[s_].view(torch.int16))
    for d_ in (2, 4):
        assert torch.equal(ok_[d_].view(torch.int16), dk[d_].view(torch.int16))


def pin_step_appends_then_attends(P):
    """step(): the step's new rows land in their slots before attention reads them.

    The pin appends on its own: for every new token t of sequence s at
    position pos, the row (block_tables[s][pos // B], pos % B) of every KV head
    takes k_new[t] / v_new[t] ([FvP] 内存管理机制, left-to-right fill; [FP]
    PagedAttention steps 1-3). The slots those rows occupy are NaN-poisoned in
    the input pools, so attending over the caches as they were before the
    append gives NaN rows. step() must return those caches bit for bit, the
    slots block * B + pos % B, and the attention of the appended caches.
    """
    for b in (small_decode(seed=111), small_prefill(seed=112), small_decode(seed=113, dtype="f16", B=8)):
        out, kc, vc, slots = P.step(b)
        B = b.block_size
        kc2, vc2 = b.k_cache.clone(), b.v_cache.clone()
        expect_slots = []
        for t in range(b.new_seq.shape[0]):
            s_, pos = int(b.new_seq[t]), int(b.new_pos[t])
            blk = int(b.block_tables[s_][pos // B])
            kc2[blk, :, pos % B] = b.k_new[t]
            vc2[blk, :, pos % B] = b.v_new[t]
            expect_slots.append(blk * B + pos % B)
        assert list(np.asarray(slots).tolist()) == expect_slots
        ib = torch.int32 if kc.dtype == torch.float32 else torch.int16
        assert torch.equal(kc.view(ib), kc2.view(ib)) and torch.equal(vc.view(ib), vc2.view(ib))
        assert np.isfinite(out).all()
        ref = P.attention(b.q, kc2, vc2, b.block_tables, b.context_lens, b.scale)
        assert np.array_equal(out, ref)


def pin_step_partition_branch(P):
    """step(batch, partition=S) evaluates the split partials with that S and merges them ([FvP] eq. (4)).

    The partials are watched on their way through the module: step() must ask
    for partitions of exactly S tokens over the appended caches (finite, since
    the pre-append pools hold NaN in the new slots), and the merged rows equal
    the single-pass rows for S = B (one block per partition) and S = 512 (one
    partition per sequence).
    """
    b = small_decode(seed=121, lens=(1, 9, 16, 31, 64, 77))
    ref, *_ = P.step(b)
    real = P.splitkv_partials
    for S in (b.block_size, 512):
        seen = []

        def spy(q, k_cache, v_cache, block_tables, context_lens, scale, partition, num_parts=None):
            r = real(q, k_cache, v_cache, block_tables, context_lens, scale, partition, num_parts)
            seen.append((partition, bool(np.isfinite(r[0]).all())))
            return r

        P.splitkv_partials = spy
        try:
            out, *_ = P.step(b, partition=S)
        finally:
            P.splitkv_partials = real
        assert seen == [(S, True)], seen
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


ALL_PINS = [
    pin_uniform_scores_mean_of_v, pin_dominant_key, pin_single_token, pin_block_permutation,
    pin_shared_vs_private, pin_eq4_block_sums, pin_partials_closed_form, pin_merge_empty,
    pin_torch_sdpa, pin_brute_force, pin_prefill_rows_are_truncated_decodes,
    pin_page_example_slots, pin_cache_write, pin_copy_blocks, pin_step_appends_then_attends,
    pin_step_partition_branch,
]
