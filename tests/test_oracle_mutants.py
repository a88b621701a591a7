"""Planted mistakes in the oracle (on the CPU) must each trip at least one pin.

Each mutant swaps one oracle function for a copy with one plausible slip in
it: a dropped scale, a wrong KV head, pages in the wrong order, an off-by-one
causal limit, a sign error, a merge that forgets a weight, a slot formula with
block and offset swapped, a cache write one row off, a merge in the wrong log
base, a slot that skips the block table, K and V swapped, a step that attends
before its append, ignores the split-KV partition or appends one position
late. The real oracle passes
every pin (tests/test_oracle.py); a pin set that let any of these through would
not be pinning the oracle.
"""
import numpy as np
import pytest
import torch

import oracle.paged_attention as P
from tests import oracle_pins as pins

_orig_gather = P.gather_sequence
_orig_softmax = P.softmax_attention


def gather_pages_reversed(cache, bt_row, n, kv_head):
    c = cache.detach().cpu()
    B = c.shape[2]
    nb = (n + B - 1) // B
    ids = torch.as_tensor(np.asarray(bt_row, dtype=np.int64)[:nb][::-1].copy())
    return c[ids, kv_head].reshape(nb * B, -1)[:n].to(torch.float64).numpy()


def gather_wrong_head(cache, bt_row, n, kv_head):
    return _orig_gather(cache, bt_row, n, (kv_head + 1) % cache.shape[1])


def gather_row_offset(cache, bt_row, n, kv_head):
    full = _orig_gather(cache, bt_row, ((n + cache.shape[2] - 1) // cache.shape[2]) * cache.shape[2], kv_head)
    return np.roll(full, 1, axis=0)[:n]


def softmax_no_scale(q, K, V, scale, n_vis):
    return _orig_softmax(q, K, V, 1.0, n_vis)


def softmax_causal_off_by_one(q, K, V, scale, n_vis):
    return _orig_softmax(q, K, V, scale, np.maximum(np.asarray(n_vis) - 1, 1))


def softmax_sign_flip(q, K, V, scale, n_vis):
    return _orig_softmax(q, K, V, -scale, n_vis)


def softmax_no_normalise(q, K, V, scale, n_vis):
    out = np.zeros((q.shape[0], V.shape[1]))
    for r in range(q.shape[0]):
        n = int(n_vis[r])
        if n:
            s = scale * (K[:n] @ q[r])
            out[r] = np.exp(s - s.max()) @ V[:n]
    return out


def merge_unweighted_l(part_o, part_m, part_l):
    o, m, l = (np.asarray(x, dtype=np.float64) for x in (part_o, part_m, part_l))
    N, H, NP, D = o.shape
    out = np.zeros((N, H, D))
    for b in range(N):
        for h in range(H):
            live = [p for p in range(NP) if l[b, h, p] > 0]
            if not live:
                continue
            M = max(m[b, h, p] for p in live)
            out[b, h] = sum(np.exp(m[b, h, p] - M) * o[b, h, p] for p in live) / sum(l[b, h, p] for p in live)
    return out


def slots_swapped(block_tables, seq_idx, positions, block_size):
    bt = np.asarray(block_tables, dtype=np.int64)
    out = np.full(len(seq_idx), -1, dtype=np.int64)
    for i, (b, p) in enumerate(zip(np.asarray(seq_idx).tolist(), np.asarray(positions).tolist())):
        if b >= 0:
            out[i] = int(bt[b, p % block_size if p % block_size < bt.shape[1] else 0]) * block_size + p // block_size
    return out


_orig_rc = P.reshape_and_cache


def cache_write_row_off(k_new, v_new, k_cache, v_cache, slots):
    B = k_cache.shape[2]
    s = np.asarray(slots, dtype=np.int64)
    shifted = np.where(s >= 0, (s // B) * B + (s % B + 1) % B, s)
    return _orig_rc(k_new, v_new, k_cache, v_cache, shifted)


def partials_normalised(q, k_cache, v_cache, bt, lens, scale, partition, num_parts=None):
    o, m, l = _orig_partials(q, k_cache, v_cache, bt, lens, scale, partition, num_parts)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = np.where(l[..., None] > 0, o / np.where(l > 0, l, 1)[..., None], 0.0)
    return o, m, l


_orig_partials = P.splitkv_partials
_orig_copy = P.copy_blocks


def copy_blocks_shifted(dst_k, dst_v, src_k, src_v, src_ids, dst_ids):
    return _orig_copy(dst_k, dst_v, src_k, src_v, [(int(s) + 1) % src_k.shape[0] for s in src_ids], dst_ids)

def merge_exp2_units(part_o, part_m, part_l):
    """Weights 2^(m_p - M) although m_p is in natural-log units (a units mix-up)."""
    o, m, l = (np.asarray(x, dtype=np.float64) for x in (part_o, part_m, part_l))
    N, H, NP, D = o.shape
    out = np.zeros((N, H, D))
    for b in range(N):
        for h in range(H):
            live = [p for p in range(NP) if l[b, h, p] > 0]
            if not live:
                continue
            M = max(m[b, h, p] for p in live)
            w = [2.0 ** (m[b, h, p] - M) for p in live]
            out[b, h] = sum(wi * o[b, h, p] for wi, p in zip(w, live)) / sum(wi * l[b, h, p] for wi, p in zip(w, live))
    return out


def slots_ignore_table(block_tables, seq_idx, positions, block_size):
    """Logical position used as the slot, block table skipped."""
    out = np.full(len(seq_idx), -1, dtype=np.int64)
    for i, (b, p) in enumerate(zip(np.asarray(seq_idx).tolist(), np.asarray(positions).tolist())):
        if b >= 0:
            out[i] = p
    return out


def cache_write_swaps_kv(k_new, v_new, k_cache, v_cache, slots):
    return _orig_rc(v_new, k_new, k_cache, v_cache, slots)


def step_attends_before_append(batch, partition=None):
    """Appends, but attends over the caches as they were before the append."""
    slots = P.slot_mapping(batch.block_tables, batch.new_seq, batch.new_pos, batch.block_size)
    kc, vc = P.reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, slots)
    if partition is not None:
        o, m, l = P.splitkv_partials(batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens,
                                     batch.scale, partition)
        return P.merge(o, m, l), kc, vc, slots
    out = P.attention(batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens, batch.scale)
    return out, kc, vc, slots


def step_ignores_partition(batch, partition=None):
    """Drops the split-KV branch: always the single pass."""
    return _orig_step(batch)


def step_partition_pre_append(batch, partition=None):
    """Split branch only: partials over the pre-append caches."""
    if partition is None:
        return _orig_step(batch)
    return step_attends_before_append(batch, partition)


def step_appends_next_position(batch, partition=None):
    """Writes each new token one position later than its own."""
    slots = P.slot_mapping(batch.block_tables, batch.new_seq, batch.new_pos + 1, batch.block_size)
    kc, vc = P.reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, slots)
    out = P.attention(batch.q, kc, vc, batch.block_tables, batch.context_lens, batch.scale)
    return out, kc, vc, slots


_orig_step = P.step

MUTANTS = {
    "step_attends_before_append": ("step", step_attends_before_append),
    "step_ignores_partition": ("step", step_ignores_partition),
    "step_partition_pre_append": ("step", step_partition_pre_append),
    "step_appends_next_position": ("step", step_appends_next_position),
    "merge_exp2_units": ("merge", merge_exp2_units),
    "slots_ignore_table": ("slot_mapping", slots_ignore_table),
    "cache_write_swaps_kv": ("reshape_and_cache", cache_write_swaps_kv),
    "pages_reversed": ("gather_sequence", gather_pages_reversed),
    "wrong_kv_head": ("gather_sequence", gather_wrong_head),
    "row_offset": ("gather_sequence", gather_row_offset),
    "no_scale": ("softmax_attention", softmax_no_scale),
    "causal_off_by_one": ("softmax_attention", softmax_causal_off_by_one),
    "sign_flip": ("softmax_attention", softmax_sign_flip),
    "no_normalise": ("softmax_attention", softmax_no_normalise),
    "merge_unweighted_l": ("merge", merge_unweighted_l),
    "slot_block_offset_swapped": ("slot_mapping", slots_swapped),
    "cache_write_row_off": ("reshape_and_cache", cache_write_row_off),
    "partials_normalised": ("splitkv_partials", partials_normalised),
    "copy_blocks_source_shifted": ("copy_blocks", copy_blocks_shifted),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(P, attr, fn)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(P)
        except Exception as e:  # an assertion or a shape/index error both count as caught
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"mutant {name} passed every pin"
