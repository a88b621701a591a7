"""Parity at the full workload sizes, in the launch configuration bench.py times.

The Llama-3-8B-shaped decode and the chat trace (every block size of the
sweep) are compared in full; the 100k-token split-KV decode on two query heads of
every KV head of every sequence, and the chunked prefill on four rows of every
CTA (sequence, KV head, query tile), which the oracle computes one by one.
Pools are NaN-poisoned outside what each sequence may read.
"""
import pytest

import oracle
import workloads as W
from tests.gpu_common import assert_close, gather_rows, require_gpu, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def prefill_cta_rows(b, query_tile_rows=128):
    """Four output rows of every CTA of the prefill grid (sequence, KV head, 128-row query tile).

    A CTA's 128 rows are (query, head) pairs of one GQA group: query tile qt holds queries
    qt*128/G .. qt*128/G + 128/G - 1. Per CTA: its first query with the group's first head,
    its last query with the last head (both cross the causal diagonal tile), and two queries
    in between with the middle heads.
    """
    G = b.num_q_heads // b.num_kv_heads
    QT = query_tile_rows // G
    rows = []
    for s in range(b.num_seqs):
        for kvh in range(b.num_kv_heads):
            for qt in range((b.chunk + QT - 1) // QT):
                i0, i1 = qt * QT, min(b.chunk, qt * QT + QT) - 1
                picks = [(i0, 0), (i0 + (i1 - i0) // 3, 1 % G), (i0 + 2 * (i1 - i0) // 3, 2 % G), (i1, G - 1)]
                rows += [(s, i, kvh * G + g) for i, g in picks]
    return rows


@pytest.fixture(scope="module")
def llama():
    b = W.llama_decode()
    ref, *_ = oracle.step(b)
    return b, ref


@pytest.mark.parametrize("partition,fused", [("auto", "auto"), (None, False), (512, False)])
def test_llama_decode_full(llama, partition, fused):
    b, ref = llama
    out, _, flags = run_gpu(b, partition=partition, fused_append=fused)
    assert flags == 0
    assert_close(out, ref, "f16", f"llama decode partition={partition} fused={fused}")


def test_long_context_sampled():
    b = W.long_context()
    out, _, flags = run_gpu(b, partition="auto")
    assert flags == 0
    # the first and the last query head of every KV head (every blockIdx.y of the split grid), every sequence
    G = b.num_q_heads // b.num_kv_heads
    rows = [(s, 0, kvh * G + g) for s in range(b.num_seqs) for kvh in range(b.num_kv_heads) for g in (0, G - 1)]
    kc, vc = oracle.reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache,
                                      oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos, b.block_size))
    ref = oracle.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale, rows=rows)
    assert_close(gather_rows(out, rows, 1), ref, "f16", "100k split-KV")


@pytest.mark.parametrize("B", [8, 16, 32, 64, 128])
def test_chat_trace_full(B):
    b = W.chat_trace(block_size=B)
    ref, *_ = oracle.step(b)
    out, _, flags = run_gpu(b, partition="auto")
    assert flags == 0
    assert_close(out, ref, "f16", f"chat trace B={B}")
    out, _, flags = run_gpu(b, shared_prefix="batch")   # the cascade bench.py times
    assert flags == 0
    assert_close(out, ref, "f16", f"chat trace shared-prefix B={B}")


def test_prefill_chunk_sampled():
    b = W.prefill_chunk()
    out, _, flags = run_gpu(b)
    assert flags == 0
    rows = prefill_cta_rows(b)
    kc, vc = oracle.reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache,
                                      oracle.slot_mapping(b.block_tables, b.new_seq, b.new_pos, b.block_size))
    ref = oracle.attention(b.q, kc, vc, b.block_tables, b.context_lens, b.scale, rows=rows)
    assert_close(gather_rows(out, rows, b.chunk), ref, "bf16", "prefill chunk")
