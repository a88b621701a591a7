"""One decode or prefill step through the C ABI, with preallocated buffers.

A step is what a serving loop runs per layer: map the step's new tokens to
cache slots (pa_slot_mapping), write their K/V rows (pa_reshape_and_cache),
then attend (pa_decode, or pa_decode_splitkv + pa_merge for long or few
contexts, or pa_prefill_chunk). Buffers are allocated once in the
constructor, so a step allocates nothing and can be replayed from a CUDA
graph. Every call goes to libpa.so; nothing here computes.
"""
from __future__ import annotations

import torch

from . import (pa_decode, pa_decode_append, pa_decode_shared_prefix, pa_decode_splitkv,
               pa_decode_splitkv_append, pa_merge, pa_prefill_chunk, pa_reshape_and_cache, pa_slot_mapping,
               pa_splitkv_num_partitions, splitkv_workspace)

NUM_SMS_B200 = 148


def choose_partition(num_seqs: int, num_kv_heads: int, max_context_len: int,
                     num_sms: int = NUM_SMS_B200) -> int | None:
    """Split-KV partition size for a decode batch, or None for the single-pass kernel.

    Single pass reads every page once and needs no workspace; it is chosen
    when there are enough (sequence, KV head) CTAs to fill the GPU and no
    context is very long. Otherwise the context is cut into 512-token
    partitions so that the work spreads over all SMs.
    """
    ctas = num_seqs * num_kv_heads
    if ctas >= 3 * num_sms and max_context_len <= 8192:
        return None
    return 512


class DecodeStep:
    """Append one token per sequence, then decode-attend over the paged cache.

    fused_append: with exactly one new token per sequence (token b of
    k_new/v_new is sequence b's newest, at position context_lens[b] - 1), the
    append is folded into the decode kernel (pa_decode_append, or
    pa_decode_splitkv_append + pa_merge when split). "auto" picks it whenever
    that holds by construction.

    shared_prefix=(prefix_len, group_size): sequences 0..group_size-1 share the
    blocks of their first prefix_len tokens; the step then runs the cascade of
    pa_decode_shared_prefix (prefix once per group on the tensor cores, every
    sequence's own tokens in one decode pass, then the merge of the group's
    rows), with the newest tokens' K/V written on the way.
    """

    def __init__(self, num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 max_context_len: int, dtype: torch.dtype, num_new_tokens: int | None = None,
                 partition: int | None | str = "auto", fused_append: bool | str = "auto",
                 shared_prefix: tuple[int, int] | None = None, device="cuda"):
        self.N, self.Hq, self.D = num_seqs, num_q_heads, head_dim
        self.shared_prefix = shared_prefix
        if shared_prefix is not None:
            prefix_len, _ = shared_prefix
            self.num_parts = 5  # up to 4 prefix key ranges + the suffix slot
            self.part_o = torch.empty((num_seqs, num_q_heads, self.num_parts, head_dim), dtype=torch.float32,
                                      device=device)
            self.part_m = torch.empty((num_seqs, num_q_heads, self.num_parts), dtype=torch.float32, device=device)
            self.part_l = torch.empty_like(self.part_m)
            self.out = torch.empty((num_seqs, num_q_heads, head_dim), dtype=dtype, device=device)
            self.fused = num_new_tokens is None or num_new_tokens == num_seqs
            self.partition = prefix_len
            self.launches_per_call = 3 if self.fused else 5
            self.slot_mapping = torch.empty(num_seqs if num_new_tokens is None else num_new_tokens,
                                            dtype=torch.int64, device=device)
            return
        if partition == "auto":
            partition = choose_partition(num_seqs, num_kv_heads, max_context_len)
        self.partition = partition
        one_per_seq = num_new_tokens is None or num_new_tokens == num_seqs
        self.fused = one_per_seq if fused_append == "auto" else bool(fused_append)
        if self.fused and not one_per_seq:
            raise ValueError("the fused append needs one new token per sequence")
        T = num_seqs if num_new_tokens is None else num_new_tokens
        self.slot_mapping = torch.empty(T, dtype=torch.int64, device=device)
        self.out = torch.empty((num_seqs, num_q_heads, head_dim), dtype=dtype, device=device)
        if partition:
            # one buffer sized by the library's own workspace query, carved into the three partial arrays
            self.num_parts = pa_splitkv_num_partitions(max_context_len, partition)
            self.part_o, self.part_m, self.part_l = splitkv_workspace(num_seqs, num_q_heads, head_dim,
                                                                      max_context_len, partition, device)
        self.launches_per_call = (2 if partition else 1) if self.fused else (4 if partition else 3)

    def __call__(self, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, new_seq, new_pos,
                 scale: float, stream=None):
        if self.shared_prefix is not None:
            prefix_len, group = self.shared_prefix
            if not self.fused:
                B = k_cache.shape[2]
                pa_slot_mapping(self.slot_mapping, block_tables, new_seq, new_pos, B, stream)
                pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, self.slot_mapping, stream)
            pa_decode_shared_prefix(self.out, q, k_new if self.fused else None, v_new if self.fused else None,
                                    k_cache, v_cache, block_tables, context_lens, prefix_len, group,
                                    self.part_o, self.part_m, self.part_l, scale, stream)
            return self.out
        if self.fused and self.partition:
            pa_decode_splitkv_append(self.part_o, self.part_m, self.part_l, q, k_new, v_new, k_cache, v_cache,
                                     block_tables, context_lens, self.partition, scale, stream)
            pa_merge(self.out, self.part_o, self.part_m, self.part_l, context_lens, self.partition, stream)
            return self.out
        if self.fused:
            pa_decode_append(self.out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, scale, stream)
            return self.out
        B = k_cache.shape[2]
        pa_slot_mapping(self.slot_mapping, block_tables, new_seq, new_pos, B, stream)
        pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, self.slot_mapping, stream)
        if self.partition:
            pa_decode_splitkv(self.part_o, self.part_m, self.part_l, q, k_cache, v_cache, block_tables,
                              context_lens, self.partition, scale, stream)
            pa_merge(self.out, self.part_o, self.part_m, self.part_l, context_lens, self.partition, stream)
        else:
            pa_decode(self.out, q, k_cache, v_cache, block_tables, context_lens, scale, stream)
        return self.out


class PrefillStep:
    """Append a C-token chunk per sequence, then causal chunk attention over the paged cache."""

    def __init__(self, num_seqs: int, chunk: int, num_q_heads: int, head_dim: int, dtype: torch.dtype,
                 num_new_tokens: int | None = None, device="cuda"):
        T = num_seqs * chunk if num_new_tokens is None else num_new_tokens
        self.slot_mapping = torch.empty(T, dtype=torch.int64, device=device)
        self.out = torch.empty((num_seqs, chunk, num_q_heads, head_dim), dtype=dtype, device=device)
        self.launches_per_call = 3

    def __call__(self, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, new_seq, new_pos,
                 scale: float, stream=None):
        B = k_cache.shape[2]
        pa_slot_mapping(self.slot_mapping, block_tables, new_seq, new_pos, B, stream)
        pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, self.slot_mapping, stream)
        pa_prefill_chunk(self.out, q, k_cache, v_cache, block_tables, context_lens, scale, stream)
        return self.out


def run_batch(batch, partition: int | None | str = "auto", fused_append: bool | str = "auto",
              shared_prefix: tuple[int, int] | None | str = None):
    """Run one step of a workloads.PagedBatch that lives on the GPU; returns the output tensor.

    shared_prefix="batch" takes (prefix tokens, group) from the batch's own generator settings.
    """
    if shared_prefix == "batch":
        sp, sg = batch.info.get("shared_prefix_tokens", 0), batch.info.get("shared_group", 0)
        shared_prefix = (sp, sg) if sp and sg else None
    if batch.chunk == 1:
        step = DecodeStep(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                          int(batch.context_lens.max().item()) if batch.num_seqs else 1, batch.q.dtype,
                          num_new_tokens=batch.new_seq.shape[0], partition=partition, fused_append=fused_append,
                          shared_prefix=shared_prefix)
    else:
        step = PrefillStep(batch.num_seqs, batch.chunk, batch.num_q_heads, batch.head_dim, batch.q.dtype,
                           num_new_tokens=batch.new_seq.shape[0])
    return step(batch.q, batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, batch.block_tables,
                batch.context_lens, batch.new_seq, batch.new_pos, batch.scale)
