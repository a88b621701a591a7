"""fp64 CPU oracle for attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import, call or execute anything in oracle/.
The product path (the CUDA library in paged_kv_cache_475_b200 and its Python
binding) never imports it and has no CPU fallback. The oracle shares no code,
constants or helpers with the CUDA path; the seeded input generator
(workloads.py) is the only module both sides use, and it holds no attention
arithmetic.

It is plain and slow on purpose: each sequence's pages are first copied into a
contiguous K/V array through the block table, then textbook softmax attention
runs in float64 on that copy. Inputs (f32/f16/bf16) are up-cast to float64
exactly; nothing is rounded on the way out.

Sources (web pages on paged KV caches, cited by title and section):
 [FP]  "FlashAttention y PagedAttention: dos soluciones para dos cuellos de
       botella distintos" (reactapp.top; Russian and German copies are
       line-for-line translations)
 [FvP] "Flash Attention vs Paged Attention：大语言模型注意力计算的内存管理革命"
       (ewbang.com)
 [PR]  "Cómo PagedAttention y RadixAttention optimizan el manejo del KV cache
       en LLMs" (transformaciondigital.pe)

Readings where the pages are silent or garbled (each one restated in the
design notes):
 * scale: [FvP] 算法原理 prints the scale garbled; the plain reading is
   1/sqrt(d), and the caller passes it explicitly.
 * GQA: query head h reads KV head h // (Hq/Hkv) (contiguous groups).
 * eq. (4) of [FvP] prints the causal block limit as [i/B]; it is read as
   ceil(i/B), with the last block cut at token i.
 * prefill positions: context_lens counts the chunk; query i of a C-token
   chunk sits at position L-C+i and sees keys 0..L-C+i.
 * empty context: L = 0 gives a zero output row (so does a chunk query at a
   negative position, L < C); an empty split partition has
   m = -inf, l = 0, o = 0 and drops out of the merge.
 * split partials: o_p is unnormalised, m_p is in natural-log units of the
   scaled score.

Pins (tests/test_oracle.py, run with -m "not gpu"): uniform scores -> mean of
V; one dominant key -> its V row; L=1 -> V[0]; random permutation of physical
blocks and shared vs private blocks leave the output unchanged; eq. (4)
block-wise sums equal the direct sum; torch's CPU scaled_dot_product_attention
in float64 on independently gathered tensors; a pure-Python brute force that
walks the pool token by token; the pages' worked block-table example.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _as_i64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.int64).numpy()
    return np.asarray(x, dtype=np.int64)


def _as_f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _cpu(x: torch.Tensor) -> torch.Tensor:
    return x.detach().to("cpu")


# --------------------------------------------------------------------------
# Cache write
# --------------------------------------------------------------------------

def slot_mapping(block_tables, seq_idx, positions, block_size: int) -> np.ndarray:
    """Flat cache slot of each new token.

    [FvP] 内存管理机制: logical blocks fill left to right, so the token at
    position pos sits in logical block pos // B at offset pos % B. [FP]
    PagedAttention "Cómo funciona" step 2 / [PR] step 2: the sequence's block
    table turns the logical block into a physical one. The flat slot index is
    physical_block * B + pos % B. A negative sequence index marks padding and
    gets slot -1.
    """
    bt = _as_i64(block_tables)
    seq = _as_i64(seq_idx)
    pos = _as_i64(positions)
    out = np.full(seq.shape[0], -1, dtype=np.int64)
    for i in range(seq.shape[0]):
        b, p = int(seq[i]), int(pos[i])
        if b < 0:
            continue
        logical_block, offset = p // block_size, p % block_size
        physical_block = int(bt[b, logical_block])
        out[i] = physical_block * block_size + offset
    return out


def reshape_and_cache(k_new, v_new, k_cache, v_cache, slots):
    """Write each new token's K/V rows into its slot; returns updated copies.

    Cache layout [P, Hkv, B, D]: slot s is block s // B, row s % B, for every
    KV head. Slots < 0 are padding and write nothing. Values are copied bit
    for bit in their own dtype.
    """
    kc, vc = _cpu(k_cache).clone(), _cpu(v_cache).clone()
    kn, vn = _cpu(k_new), _cpu(v_new)
    B = kc.shape[2]
    for t, s in enumerate(_as_i64(slots).tolist()):
        if s < 0:
            continue
        kc[s // B, :, s % B, :] = kn[t]
        vc[s // B, :, s % B, :] = vn[t]
    return kc, vc


def copy_blocks(dst_k, dst_v, src_k, src_v, src_ids, dst_ids):
    """Whole-block copies; returns updated copies of the destination pools.

    [FP] PagedAttention "Cómo funciona" step 4 (copy-on-write of a shared
    block) and the swapping of [FvP] 恢复机制对比: block dst_ids[i] of the
    destination pool becomes block src_ids[i] of the source pool, bits
    unchanged, for K and V.
    """
    dk, dv = _cpu(dst_k).clone(), _cpu(dst_v).clone()
    sk, sv = _cpu(src_k), _cpu(src_v)
    for s_, d_ in zip(_as_i64(src_ids).tolist(), _as_i64(dst_ids).tolist()):
        dk[d_] = sk[s_]
        dv[d_] = sv[s_]
    return dk, dv


# --------------------------------------------------------------------------
# Gather + textbook attention
# --------------------------------------------------------------------------

def gather_sequence(cache, block_table_row, n_tokens: int, kv_head: int) -> np.ndarray:
    """Copy one sequence's pages, in logical order, into a contiguous [n, D] float64 array.

    [FP] PagedAttention "Cómo funciona" step 5 and [PR] step 2: the kernel
    looks the sequence's blocks up in its table and gathers the keys and
    values so that the sequence reads as contiguous.
    """
    c = _cpu(cache)
    B, D = c.shape[2], c.shape[3]
    if n_tokens == 0:
        return np.zeros((0, D))
    n_blocks = (n_tokens + B - 1) // B
    ids = torch.as_tensor(_as_i64(block_table_row)[:n_blocks])
    pages = c[ids, kv_head]                      # [n_blocks, B, D], logical order
    rows = pages.reshape(n_blocks * B, D)[:n_tokens]
    return _as_f64(rows)


def softmax_attention(q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
                      n_visible: np.ndarray) -> np.ndarray:
    """softmax(q K^T * scale) V, row by row; row r sees keys 0..n_visible[r]-1.

    [FP] "Por qué la atención sale cara": Attention(Q,K,V) = softmax(QK^T/sqrt(d)) V.
    Keys past n_visible (the causal limit) are left out of the softmax.
    A row that sees no key is all zeros.
    """
    out = np.zeros((q_rows.shape[0], V.shape[1]))
    for r in range(q_rows.shape[0]):
        n = int(n_visible[r])
        if n == 0:
            continue
        s = scale * (K[:n] @ q_rows[r])
        w = np.exp(s - s.max())
        w = w / w.sum()
        out[r] = w @ V[:n]
    return out


def _group(num_q_heads: int, num_kv_heads: int) -> int:
    if num_q_heads % num_kv_heads:
        raise ValueError("Hq must be a multiple of Hkv")
    return num_q_heads // num_kv_heads


def attention(q, k_cache, v_cache, block_tables, context_lens, scale: float,
              rows=None) -> np.ndarray:
    """Paged attention for a decode step or a causal prefill chunk, in float64.

    q is [N, Hq, D] (decode: one query per sequence at position L-1) or
    [N, C, Hq, D] (prefill chunk: query i at position L-C+i). Query head h
    reads KV head h // (Hq/Hkv). Query i sees keys 0..L-C+i (causal inside the
    chunk, everything before it); this is the causal block sum of [FvP]
    算法原理 eq. (4) with the last block cut at the query's own token.

    rows: optional list of (b, i, h) to compute only those output rows (for
    sampled parity at full sizes); returns [len(rows), D]. Otherwise returns
    an array shaped like q.
    """
    qq = _cpu(q)
    decode = qq.dim() == 3
    if decode:
        qq = qq[:, None]
    N, C, Hq, D = qq.shape
    Hkv = _cpu(k_cache).shape[1]
    G = _group(Hq, Hkv)
    lens = _as_i64(context_lens)
    bt = _as_i64(block_tables)

    wanted = {}
    if rows is None:
        for b in range(N):
            for h in range(Hq):
                wanted.setdefault((b, h // G), []).extend((i, h) for i in range(C))
        out = np.zeros((N, C, Hq, D))
    else:
        for (b, i, h) in rows:
            wanted.setdefault((b, h // G), []).append((i, h))
        out_rows = {}

    for (b, kvh), items in sorted(wanted.items()):
        L = int(lens[b])
        K = gather_sequence(k_cache, bt[b], L, kvh)
        V = gather_sequence(v_cache, bt[b], L, kvh)
        qrows = np.stack([_as_f64(qq[b, i, h]) for (i, h) in items])
        n_vis = np.array([max(0, L - C + i + 1) if L > 0 else 0 for (i, h) in items])
        o = softmax_attention(qrows, K, V, scale, n_vis)
        for r, (i, h) in enumerate(items):
            if rows is None:
                out[b, i, h] = o[r]
            else:
                out_rows[(b, i, h)] = o[r]
    if rows is not None:
        return np.stack([out_rows[tuple(r)] for r in rows]) if rows else np.zeros((0, D))
    return out[:, 0] if decode else out


# --------------------------------------------------------------------------
# Split-KV partials and their merge
# --------------------------------------------------------------------------

def num_partitions(max_context_len: int, partition: int) -> int:
    return max(1, (int(max_context_len) + partition - 1) // partition)


def splitkv_partials(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                     partition: int, num_parts: int | None = None):
    """Per-partition softmax state of a decode step.

    Partition p of sequence b covers tokens [p*P, min((p+1)*P, L)). For each
    (b, h, p): m = max of the scaled scores, l = sum exp(s - m), o = sum
    exp(s - m) V (unnormalised). These are the running max / running sum of
    [FP] "Cómo funciona" (online softmax), taken one partition at a time.
    Empty partitions: m = -inf, l = 0, o = 0.
    Returns o [N, Hq, NP, D], m [N, Hq, NP], l [N, Hq, NP].
    """
    qq = _cpu(q)
    N, Hq, D = qq.shape
    Hkv = _cpu(k_cache).shape[1]
    G = _group(Hq, Hkv)
    lens = _as_i64(context_lens)
    bt = _as_i64(block_tables)
    NP = num_parts if num_parts is not None else num_partitions(lens.max() if N else 0, partition)
    o = np.zeros((N, Hq, NP, D))
    m = np.full((N, Hq, NP), -np.inf)
    l = np.zeros((N, Hq, NP))
    for b in range(N):
        L = int(lens[b])
        for kvh in range(Hkv):
            K = gather_sequence(k_cache, bt[b], L, kvh)
            V = gather_sequence(v_cache, bt[b], L, kvh)
            for h in range(kvh * G, (kvh + 1) * G):
                qv = _as_f64(qq[b, h])
                for p in range(NP):
                    t0, t1 = p * partition, min((p + 1) * partition, L)
                    if t0 >= t1:
                        continue
                    s = scale * (K[t0:t1] @ qv)
                    m[b, h, p] = s.max()
                    e = np.exp(s - m[b, h, p])
                    l[b, h, p] = e.sum()
                    o[b, h, p] = e @ V[t0:t1]
    return o, m, l


def merge(part_o, part_m, part_l) -> np.ndarray:
    """Combine per-partition softmax states into the attention output.

    Log-sum-exp rule (the online-softmax update of [FP] "Cómo funciona",
    applied across partitions): M = max_p m_p over non-empty partitions,
    L = sum_p exp(m_p - M) l_p, out = sum_p exp(m_p - M) o_p / L. Partitions
    with l_p = 0 are skipped; a row with no non-empty partition is zero.
    """
    o, m, l = _as_f64(part_o), _as_f64(part_m), _as_f64(part_l)
    N, Hq, NP, D = o.shape
    out = np.zeros((N, Hq, D))
    for b in range(N):
        for h in range(Hq):
            live = [p for p in range(NP) if l[b, h, p] > 0]
            if not live:
                continue
            M = max(m[b, h, p] for p in live)
            num = np.zeros(D)
            den = 0.0
            for p in live:
                w = math.exp(m[b, h, p] - M)
                num += w * o[b, h, p]
                den += w * l[b, h, p]
            out[b, h] = num / den
    return out


# --------------------------------------------------------------------------
# One decode / prefill step as the library runs it: append, then attend
# --------------------------------------------------------------------------

def step(batch, partition: int | None = None):
    """Append the step's new tokens, then attend; returns (out, k_cache, v_cache, slots)."""
    slots = slot_mapping(batch.block_tables, batch.new_seq, batch.new_pos, batch.block_size)
    kc, vc = reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, slots)
    if partition is not None:
        o, m, l = splitkv_partials(batch.q, kc, vc, batch.block_tables, batch.context_lens,
                                   batch.scale, partition)
        out = merge(o, m, l)
    else:
        out = attention(batch.q, kc, vc, batch.block_tables, batch.context_lens, batch.scale)
    return out, kc, vc, slots
