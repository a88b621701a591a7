"""CUDA path vs the fp64 oracle on the same seeded inputs (element by element).

Cache write and slot indices: bit-exact. Attention outputs: max-abs <= 1e-2 and
mean-abs <= 1e-3 for fp16/bf16, max-abs <= 1e-5 for fp32. Invariants that the
pages fix (block relabelling, shared blocks) must hold bit for bit on the GPU,
since the kernels' reduction order does not depend on physical block ids.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_common import (assert_close, permute_pool, require_gpu, run_gpu, small_batch)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


# ---------------------------------------------------------------------------
# Cache write
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B", [8, 16, 32, 64, 128])
def test_slot_mapping_and_cache_write_bit_exact(B):
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=100 + B, B=B, chunk=5, lens=(5, 9, 40, 129, 300), dtype="bf16")
    g = b.to("cuda")
    # padding tokens (seq -1) mixed in
    seq = torch.cat([g.new_seq, torch.full((3,), -1, dtype=torch.int32, device="cuda")])
    pos = torch.cat([g.new_pos, torch.zeros(3, dtype=torch.int32, device="cuda")])
    slots = torch.empty(seq.shape[0], dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(slots, g.block_tables, seq, pos, B)
    ref_slots = oracle.slot_mapping(b.block_tables, seq.cpu(), pos.cpu(), B)
    assert slots.cpu().numpy().tolist() == ref_slots.tolist()
    kn = torch.cat([g.k_new, torch.zeros((3,) + tuple(g.k_new.shape[1:]), dtype=g.k_new.dtype, device="cuda")])
    vn = torch.cat([g.v_new, torch.zeros_like(kn[-3:])])
    pa.pa_reshape_and_cache(kn, vn, g.k_cache, g.v_cache, slots)
    torch.cuda.synchronize()
    kc, vc = oracle.reshape_and_cache(kn.cpu(), vn.cpu(), b.k_cache, b.v_cache, ref_slots)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16))
    assert pa.pa_read_error_flags() == 0


def test_cache_write_f32_and_out_of_pool_slot():
    import paged_kv_cache_475_b200 as pa
    b = W.tiny_fp32()
    g = b.to("cuda")
    slots = torch.tensor([3, -1, 16 * 16 + 5, 17], dtype=torch.int64, device="cuda")  # third is past the pool
    kn = torch.randn(4, 1, 64, device="cuda")
    vn = torch.randn(4, 1, 64, device="cuda")
    pa.pa_reshape_and_cache(kn, vn, g.k_cache, g.v_cache, slots)
    flags = pa.pa_read_error_flags()
    assert flags & pa.DEVERR_SLOT
    ok = torch.tensor([3, -1, -1, 17])
    kc, vc = oracle.reshape_and_cache(kn.cpu(), vn.cpu(), b.k_cache, b.v_cache, ok)
    assert torch.equal(g.k_cache.cpu().view(torch.int32), kc.view(torch.int32))
    assert torch.equal(g.v_cache.cpu().view(torch.int32), vc.view(torch.int32))


# ---------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------

def test_tiny_fp32_decode():
    b = W.tiny_fp32()
    ref, *_ = oracle.step(b)
    for part in (None, 16, 32):
        out, _, flags = run_gpu(b, partition=part)
        assert flags == 0
        assert_close(out, ref, "f32", f"tiny fp32 partition={part}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [8, 16, 32, 64, 128])
def test_decode_grid_f16(D, G, B):
    b = small_batch(seed=D * 1000 + G * 100 + B, D=D, G=G, B=B)
    ref, *_ = oracle.step(b)
    out, _, flags = run_gpu(b, partition=None, fused_append=False)
    assert flags == 0
    assert_close(out, ref, "f16", f"D={D} G={G} B={B}")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("B", [8, 16, 128])
def test_decode_append_fused(dtype, B):
    """pa_decode_append: the cache after the call equals the oracle's append bit for bit, and the
    output (whose newest token was poisoned before the call) matches the oracle."""
    b = small_batch(seed=17 + B, dtype=dtype, B=B, lens=(1, 15, 16, 17, 100, 333, 700))
    ref, kc, vc, _ = oracle.step(b)
    out, g, flags = run_gpu(b, partition=None, fused_append=True)
    assert flags == 0
    assert_close(out, ref, dtype, f"fused append {dtype} B={B}")
    iv = torch.int32 if dtype == "f32" else torch.int16
    assert torch.equal(g.k_cache.cpu().view(iv), kc.view(iv))
    assert torch.equal(g.v_cache.cpu().view(iv), vc.view(iv))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [8, 16, 128])
@pytest.mark.parametrize("D,G", [(128, 4), (64, 2), (128, 8)])
def test_decode_other_dtypes(dtype, B, D, G):
    b = small_batch(seed=7 + B + D + G, dtype=dtype, D=D, G=G, B=B)
    ref, *_ = oracle.step(b)
    out, _, flags = run_gpu(b, partition=None)
    assert flags == 0
    assert_close(out, ref, dtype, f"{dtype} D={D} G={G} B={B}")


@pytest.mark.parametrize("poison", [float("nan"), 65504.0, -65504.0])
def test_decode_poisoned_pool_is_never_read(poison):
    b = small_batch(seed=31, poison=poison, lens=(1, 2, 31, 33, 250))
    ref, *_ = oracle.step(b)
    for part in (None, 64):
        out, _, flags = run_gpu(b, partition=part)
        assert flags == 0
        assert_close(out, ref, "f16", f"poison={poison} partition={part}")


def test_decode_peaky_softmax():
    b = small_batch(seed=41, q_std=2.0 ** 0.5 * 3, lens=(64, 513, 1000))
    ref, *_ = oracle.step(b)
    out, _, _ = run_gpu(b, partition=None)
    assert_close(out, ref, "f16", "peaky")


def test_decode_empty_and_single_token():
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=51, lens=(1, 1, 5))
    g = b.to("cuda")
    g.context_lens[2] = 0  # an empty context: zero row, nothing read
    from paged_kv_cache_475_b200.step import run_batch
    out = run_batch(g, partition=None)
    torch.cuda.synchronize()
    assert not out[2].any()
    # one visible token: the softmax weight is exactly 1, so out equals V[0] bit for bit
    for s in (0, 1):
        blk = int(b.block_tables[s, 0])
        for h in range(b.num_q_heads):
            v0 = b.v_new[s, h // (b.num_q_heads // b.num_kv_heads)]
            assert torch.equal(out[s, h].cpu(), v0)
    assert pa.pa_read_error_flags() == 0


def test_decode_block_permutation_bit_identical():
    b = small_batch(seed=61, lens=(3, 100, 517, 999))
    out1, _, _ = run_gpu(b, partition=None)
    out2, _, _ = run_gpu(permute_pool(b), partition=None)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    out3, _, _ = run_gpu(b, partition=64)
    out4, _, _ = run_gpu(permute_pool(b, seed=9), partition=64)
    assert torch.equal(out3.view(torch.int16), out4.view(torch.int16))


def test_decode_shared_blocks_equal_private_copies():
    b = small_batch(seed=71, B=16, lens=(300, 200, 129, 50), shared_prefix_tokens=128, shared_group=3,
                    pool_factor=3.0)
    out1, _, _ = run_gpu(b, partition=None)
    # give sequences 1 and 2 private copies of the 8 shared blocks
    b2 = b.to("cpu")
    b2.k_cache, b2.v_cache, b2.block_tables = b.k_cache.clone(), b.v_cache.clone(), b.block_tables.clone()
    used = set(b.block_tables[b.block_tables >= 0].tolist())
    spare = [i for i in range(b.k_cache.shape[0]) if i not in used]
    assert len(spare) >= 16
    for s in (1, 2):
        for j in range(8):
            src, dst = int(b.block_tables[s, j]), spare.pop()
            b2.k_cache[dst], b2.v_cache[dst] = b.k_cache[src], b.v_cache[src]
            b2.block_tables[s, j] = dst
    out2, _, _ = run_gpu(b2, partition=None)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_decode_bad_block_id_sets_flag_without_fault():
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=81, lens=(40, 70, 90))
    ref, *_ = oracle.step(b)
    bad = b.to("cpu")
    bad.block_tables = b.block_tables.clone()
    bad.block_tables[0, 1] = b.k_cache.shape[0] + 5  # outside the pool
    for part in (None, 32):
        g = bad.to("cuda")
        pa.pa_read_error_flags(clear=True)
        # the append only touches each sequence's last block, not block 1 of sequence 0
        from paged_kv_cache_475_b200.step import run_batch
        out = run_batch(g, partition=part).cpu()
        flags = pa.pa_read_error_flags(clear=True)
        assert flags & pa.DEVERR_BLOCK_ID
        assert_close(out[1:], ref[1:], "f16", "unaffected sequences")


# ---------------------------------------------------------------------------
# Split-KV partials and merge
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("partition", [16, 64, 512, 4096])
@pytest.mark.parametrize("B", [8, 16, 128])
@pytest.mark.parametrize("fused", [True, False])
def test_splitkv_partials_and_merge(partition, B, fused):
    """Split-KV step with the cache write separate (pa_reshape_and_cache) or folded into the
    partition holding each sequence's newest token (pa_decode_splitkv_append): the cache equals
    the oracle's append bit for bit, the merged output and the partials match the oracle."""
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=91 + partition + B, B=B, lens=(1, 16, 17, 511, 512, 513, 1400))
    out, g, flags = run_gpu(b, partition=partition, fused_append=fused)
    assert flags == 0
    ref, kc, vc, _ = oracle.step(b)
    assert_close(out, ref, "f16", f"merged partition={partition} B={B} fused={fused}")
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16))
    # the partials themselves
    NP = pa.pa_splitkv_num_partitions(int(b.context_lens.max()), partition)
    po, pm, pl = pa.splitkv_buffers(b.num_seqs, b.num_q_heads, b.head_dim, NP)
    pa.pa_decode_splitkv(po, pm, pl, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, partition, b.scale)
    torch.cuda.synchronize()
    o_ref, m_ref, l_ref = oracle.splitkv_partials(b.q, kc, vc, b.block_tables, b.context_lens, b.scale,
                                                  partition, NP)
    pm, pl, po = pm.cpu().double().numpy(), pl.cpu().double().numpy(), po.cpu().double().numpy()
    live = l_ref > 0
    assert (pl[~live] == 0).all() and np.isneginf(pm[~live]).all() and (po[~live] == 0).all()
    assert np.abs(pm[live] - m_ref[live]).max() < 1e-4
    assert (np.abs(pl[live] - l_ref[live]) / l_ref[live]).max() < 1e-4
    on = po[live] / pl[live][:, None]
    on_ref = o_ref[live] / l_ref[live][:, None]
    assert np.abs(on - on_ref).max() < 1e-3


def test_merge_skips_partitions_past_context():
    import paged_kv_cache_475_b200 as pa
    N, Hq, NP, D = 3, 4, 5, 128
    gen = torch.Generator().manual_seed(3)
    o = torch.randn(N, Hq, NP, D, generator=gen)
    m = torch.randn(N, Hq, NP, generator=gen)
    l = torch.rand(N, Hq, NP, generator=gen) + 0.5
    lens = torch.tensor([64, 200, 0], dtype=torch.int32)  # partition 64 -> 1, 4, 0 partitions
    live_o, live_m, live_l = o.clone().double().numpy(), m.clone().double().numpy(), l.clone().double().numpy()
    for b_, npb in enumerate([1, 4, 0]):
        live_l[b_, :, npb:] = 0.0
    ref = oracle.merge(live_o, live_m, live_l)
    out = torch.empty(N, Hq, D, dtype=torch.float32, device="cuda")
    pa.pa_merge(out, o.cuda(), m.cuda(), l.cuda(), lens.cuda(), 64)
    torch.cuda.synchronize()
    assert np.abs(out.cpu().double().numpy() - ref).max() < 1e-5
    assert not out[2].any()


# ---------------------------------------------------------------------------
# Chunked prefill
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_prefill_grid(D, G, dtype):
    b = small_batch(seed=D + G * 10 + len(dtype), dtype=dtype, D=D, G=G, B=16, chunk=37,
                    lens=(37, 38, 100, 229, 500))
    ref, *_ = oracle.step(b)
    out, _, flags = run_gpu(b)
    assert flags == 0
    assert_close(out, ref, dtype, f"prefill D={D} G={G} {dtype}")


@pytest.mark.parametrize("B", [8, 32, 64, 128])
@pytest.mark.parametrize("C", [1, 16, 64, 130])
def test_prefill_blocks_and_chunks(B, C):
    b = small_batch(seed=B * 7 + C, dtype="bf16", D=128, G=4, B=B, chunk=C, lens=(C, C + 1, C + 63, C + 300))
    ref, *_ = oracle.step(b)
    out, _, flags = run_gpu(b)
    assert flags == 0
    assert_close(out, ref, "bf16", f"prefill B={B} C={C}")


def test_prefill_permutation_bit_identical():
    b = small_batch(seed=5, dtype="bf16", chunk=40, lens=(40, 90, 333))
    out1, _, _ = run_gpu(b)
    out2, _, _ = run_gpu(permute_pool(b))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_prefill_short_context_rows_are_zero():
    """L < C: the first C - L queries sit at negative positions and see nothing."""
    import paged_kv_cache_475_b200 as pa
    from paged_kv_cache_475_b200.step import PrefillStep
    b = small_batch(seed=6, dtype="bf16", chunk=20, lens=(20, 40))
    g = b.to("cuda")
    step = PrefillStep(b.num_seqs, b.chunk, b.num_q_heads, b.head_dim, g.q.dtype,
                       num_new_tokens=g.new_seq.shape[0])
    step(g.q, g.k_new, g.v_new, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.new_seq, g.new_pos,
         b.scale)
    lens = g.context_lens.clone()
    lens[0] = 12  # only 12 keys visible for sequence 0: queries 0..7 see nothing
    out = torch.empty_like(g.q)
    pa.pa_prefill_chunk(out, g.q, g.k_cache, g.v_cache, g.block_tables, lens, b.scale)
    torch.cuda.synchronize()
    assert not out[0, :8].any()
    _, kc, vc, _ = oracle.step(b)  # the oracle's own append
    rows = [(0, i, h) for i in range(20) for h in range(b.num_q_heads)]
    ref = oracle.attention(b.q, kc, vc, b.block_tables, lens.cpu(), b.scale, rows=rows)
    assert not ref[: 8 * b.num_q_heads].any()
    got = torch.stack([out[0, i, h].cpu() for (_, i, h) in rows])
    assert_close(got, ref, "bf16", "short context")


# ---------------------------------------------------------------------------
# Whole-block copies: copy-on-write and swap
# ---------------------------------------------------------------------------

def test_copy_blocks_copy_on_write_in_place():
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=301, dtype="bf16", lens=(40, 70, 90), poison=None)
    g = b.to("cuda")
    src = torch.tensor([int(b.block_tables[0, 0]), int(b.block_tables[1, 2]), 5], dtype=torch.int32)
    dst = torch.tensor([int(b.k_cache.shape[0]) - 1, int(b.k_cache.shape[0]) - 2, 6], dtype=torch.int32)
    pa.pa_copy_blocks(g.k_cache, g.v_cache, g.k_cache, g.v_cache, src.cuda(), dst.cuda())
    torch.cuda.synchronize()
    kc, vc = oracle.copy_blocks(b.k_cache, b.v_cache, b.k_cache, b.v_cache, src, dst)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16))
    assert pa.pa_read_error_flags() == 0


def test_copy_blocks_swap_out_and_in_through_pinned_host_memory():
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=302, dtype="f16", lens=(100, 333), poison=None, pool_factor=2.0)
    g = b.to("cuda")
    P = b.k_cache.shape[0]
    ids = b.block_tables[0, :7].clone()                       # sequence 0's blocks
    host_k = torch.zeros((8,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    slots = torch.arange(7, dtype=torch.int32).pin_memory()
    pa.pa_copy_blocks(host_k, host_v, g.k_cache, g.v_cache, ids.cuda(), slots)      # swap out
    torch.cuda.synchronize()
    hk, hv = oracle.copy_blocks(torch.zeros_like(host_k), torch.zeros_like(host_v), b.k_cache, b.v_cache, ids,
                                torch.arange(7))
    assert torch.equal(host_k.view(torch.int16), hk.view(torch.int16))
    assert torch.equal(host_v.view(torch.int16), hv.view(torch.int16))
    used = set(b.block_tables[b.block_tables >= 0].tolist())
    new_ids = torch.tensor([i for i in range(P) if i not in used][:7], dtype=torch.int32)
    pa.pa_copy_blocks(g.k_cache, g.v_cache, host_k, host_v, slots, new_ids.cuda())  # swap in elsewhere
    torch.cuda.synchronize()
    assert torch.equal(g.k_cache[new_ids.long()].cpu().view(torch.int16), b.k_cache[ids.long()].view(torch.int16))
    # the sequence reads the same context through its updated table
    ref, *_ = oracle.step(b)
    g.block_tables[0, :7] = new_ids.cuda()
    from paged_kv_cache_475_b200.step import run_batch
    out = run_batch(g, partition=None, fused_append=False).cpu()
    assert_close(out, ref, "f16", "after swap in")
    assert pa.pa_read_error_flags() == 0


def test_copy_on_write_through_the_block_manager():
    """Two sequences share a half-full block; the second one's next token triggers a copy."""
    import paged_kv_cache_475_b200 as pa
    from paged_kv_cache_475_b200.blocks import BlockManager
    gen = torch.Generator().manual_seed(303)
    Hkv, Hq, D, B, P = 2, 8, 128, 16, 12
    m = BlockManager(P, B)
    m.allocate(0, 40)
    m.fork(0, 1)
    kc = torch.randn(P, Hkv, B, D, generator=gen).half()
    vc = torch.randn(P, Hkv, B, D, generator=gen).half()
    slot0, pair0 = m.append_slot(0)   # seq 0: first writer of the shared last block -> copy
    slot1, pair1 = m.append_slot(1)   # seq 1: now alone in the original block
    assert pair0 is not None and pair1 is None
    k_new = torch.randn(2, Hkv, D, generator=gen).half()
    v_new = torch.randn(2, Hkv, D, generator=gen).half()
    q = torch.randn(2, Hq, D, generator=gen).half()
    bt = m.tables_tensor([0, 1])
    lens = torch.tensor([41, 41], dtype=torch.int32)
    # oracle: copy, then write both new tokens, then attend
    okc, ovc = oracle.copy_blocks(kc, vc, kc, vc, [pair0[0]], [pair0[1]])
    okc, ovc = oracle.reshape_and_cache(k_new, v_new, okc, ovc, [slot0, slot1])
    ref = oracle.attention(q, okc, ovc, bt, lens, D ** -0.5)
    # library: pa_copy_blocks, pa_reshape_and_cache, pa_decode
    gk, gv = kc.cuda(), vc.cuda()
    pa.pa_copy_blocks(gk, gv, gk, gv, torch.tensor([pair0[0]], dtype=torch.int32).cuda(),
                      torch.tensor([pair0[1]], dtype=torch.int32).cuda())
    pa.pa_reshape_and_cache(k_new.cuda(), v_new.cuda(), gk, gv, torch.tensor([slot0, slot1]).cuda())
    out = torch.empty_like(q).cuda()
    pa.pa_decode(out, q.cuda(), gk, gv, bt.cuda(), lens.cuda(), D ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(gk.cpu().view(torch.int16), okc.view(torch.int16))
    assert_close(out.cpu(), ref, "f16", "copy on write")
    assert pa.pa_read_error_flags() == 0


# ---------------------------------------------------------------------------
# Shared-prefix (cascade) decode
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("B,prefix,G", [(16, 64, 4), (8, 128, 2), (32, 32, 8), (128, 128, 4)])
def test_decode_shared_prefix(dtype, B, prefix, G):
    lens = (prefix + 1, prefix + 40, prefix + 300, 17, prefix + 700, 90)
    b = small_batch(seed=400 + B + prefix, dtype=dtype, B=B, G=G, lens=lens, shared_prefix_tokens=prefix,
                    shared_group=3)
    ref, kc, vc, _ = oracle.step(b)
    for fused in (True, False):
        out, g, flags = run_gpu(b, fused_append=fused, shared_prefix="batch")
        assert flags == 0
        assert_close(out, ref, dtype, f"shared prefix {dtype} B={B} prefix={prefix} fused={fused}")
        assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))


def test_decode_shared_prefix_rejects_a_member_inside_the_prefix():
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=410, lens=(64, 100, 300), shared_prefix_tokens=64, shared_group=2)
    out, _, flags = run_gpu(b, shared_prefix="batch")   # sequence 0 ends exactly at the prefix end
    assert flags & pa.DEVERR_CONTEXT


# ---------------------------------------------------------------------------
# Copy-wait time-out
# ---------------------------------------------------------------------------

def test_copy_wait_times_out_sets_the_flag_and_the_context_stays_usable():
    """A wait for a copy that is never issued gives up, reports PA_DEVERR_WAIT and leaves nothing in flight.

    The self-test entry point arms warp 0 of the first CTA (KV head 0 of the longest sequence) for a tile
    whose copies never come, with a wait limit of 2e5 SM cycles (about 0.1 ms). Every other CTA runs as in
    pa_decode, so every other row must equal pa_decode's bit for bit; a plain decode afterwards must match
    the oracle with no flag set.
    """
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=420, lens=(1, 15, 100, 700, 333, 17), poison=None)  # unique longest: sequence 3
    g = b.to("cuda")
    pa.pa_read_error_flags(clear=True)
    ref_gpu = torch.empty_like(g.q)
    pa.pa_decode(ref_gpu, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale)
    assert pa.pa_read_error_flags() == 0

    starved = torch.full_like(g.q, float("nan"))
    pa.pa_decode_selftest_starved_wait(starved, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens,
                                       g.scale, wait_cycles=200_000)
    assert pa.pa_read_error_flags(clear=True) == pa.DEVERR_WAIT
    G = g.q.shape[1] // g.k_cache.shape[1]
    keep = torch.ones(g.q.shape[:2], dtype=torch.bool, device="cuda")
    keep[3, :G] = False
    assert torch.equal(starved[keep].view(torch.int16), ref_gpu[keep].view(torch.int16))

    again = torch.empty_like(g.q)
    pa.pa_decode(again, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale)
    assert pa.pa_read_error_flags() == 0
    assert torch.equal(again.view(torch.int16), ref_gpu.view(torch.int16))
    expect = oracle.attention(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    assert_close(again, expect, "f16", "decode after a timed-out wait")


# ---------------------------------------------------------------------------
# Non-finite values inside the visible context
# ---------------------------------------------------------------------------

def _plant(cache, bt, seq, pos, kvh, d, B):
    cache[int(bt[seq, pos // B]), kvh, pos % B, d] = float("nan")


def test_nan_in_a_visible_key_or_value_reaches_the_output_as_in_the_definition():
    """A NaN in a visible K row makes every score of that KV head's rows NaN, so the whole rows are NaN; a
    NaN in a visible V element makes that output dimension NaN. The oracle (the plain definition) says so;
    the kernels must agree, also where the NaN key is the only token of a warp's tiles (position 16 of a
    17-token context, position 0 of a 1-token one), through the single pass and through split-KV + merge.
    """
    import paged_kv_cache_475_b200 as pa
    b = small_batch(seed=421, lens=(1, 17, 40, 300, 64), poison=None)
    B = b.block_size
    _plant(b.k_cache, b.block_tables, 0, 0, 0, 5, B)      # sequence 0, its only key, KV head 0
    _plant(b.k_cache, b.block_tables, 1, 16, 1, 77, B)    # sequence 1, key 16 (alone in its tile), KV head 1
    _plant(b.v_cache, b.block_tables, 3, 123, 0, 9, B)    # sequence 3, value 123, KV head 0, dim 9
    expect = oracle.attention(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    assert np.isnan(expect[0, :4]).all() and np.isnan(expect[1, 4:]).all()
    assert np.isnan(expect[3, :4, 9]).all() and np.isfinite(np.delete(expect[3, :4], 9, axis=-1)).all()
    g = b.to("cuda")
    pa.pa_read_error_flags(clear=True)
    single = torch.empty_like(g.q)
    pa.pa_decode(single, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale)
    outs = {"single pass": single}
    for partition in (16, 128):
        nparts = pa.pa_splitkv_num_partitions(int(b.context_lens.max()), partition)
        po, pm, pl = pa.splitkv_buffers(b.num_seqs, b.num_q_heads, b.head_dim, nparts)
        merged = torch.empty_like(g.q)
        pa.pa_decode_splitkv(po, pm, pl, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, partition,
                             g.scale)
        pa.pa_merge(merged, po, pm, pl, g.context_lens, partition)
        outs[f"split {partition}"] = merged
    torch.cuda.synchronize()
    assert pa.pa_read_error_flags() == 0
    nan = np.isnan(expect)
    for what, out in outs.items():
        got = out.cpu().to(torch.float64).numpy()
        assert (np.isnan(got) == nan).all(), f"{what}: NaN pattern differs from the definition"
        err = np.abs(got[~nan] - expect[~nan])
        assert err.max() <= 1e-2 and err.mean() <= 1e-3, f"{what}: finite part off by {err.max():.3e}"


# ---------------------------------------------------------------------------
# Two rows per CTA (large batches of mostly short rows)
# ---------------------------------------------------------------------------

def _paired_lens(seed, n):
    g = np.random.default_rng(seed)
    lens = g.integers(1, 400, n)
    lens[:5] = (1, 2, 15, 16, 17)
    return tuple(int(x) for x in lens)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_decode_with_paired_rows(dtype, fused):
    """300 sequences x 8 KV heads is more than three waves of CTAs on a B200, so the single pass gives the
    CTAs past the longest eighth two rows each (two warps per row); 300 - 37 = 263 paired ranks leave the
    last CTA one empty row slot. Every row must match the oracle and the cache write must be bit-exact."""
    b = small_batch(seed=430, dtype=dtype, G=4, Hkv=8, B=16, lens=_paired_lens(430, 300))
    ref, kc, vc, _ = oracle.step(b)
    out, g, flags = run_gpu(b, partition=None, fused_append=fused)
    assert flags == 0
    assert_close(out, ref, dtype, f"paired rows {dtype} fused={fused}")
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16))


def test_shared_prefix_with_paired_rows():
    """The cascade's suffix pass pairs rows too: members (suffix only) and non-members mixed in pairs."""
    lens = tuple(64 + x if i < 120 else x for i, x in enumerate(_paired_lens(431, 300)))
    b = small_batch(seed=431, dtype="f16", G=4, Hkv=8, B=16, lens=lens, shared_prefix_tokens=64, shared_group=120)
    ref, kc, vc, _ = oracle.step(b)
    out, g, flags = run_gpu(b, fused_append=True, shared_prefix="batch")
    assert flags == 0
    assert_close(out, ref, "f16", "shared prefix with paired rows")
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
