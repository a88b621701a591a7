"""pa_decode_splitkv_noalloc: split-KV decode for callers that cannot allocate device memory.

Some callers cannot give this library a workspace for the split-KV partials:
a plugin or FFI host with no device allocator at hand, a serving runtime that
has already handed all free HBM to its KV block pool, or a latency-critical
loop that cannot pay for cudaMalloc's implicit device synchronisation. For
them the library keeps the partials in a fixed per-device array of its own.

This test calls that entry point through the C ABI (ctypes, no binding in
between) twice in a row. The first call has the larger footprint (more rows,
more partitions per row); the second is smaller and laid out differently
(another head count, head dim, block size, partition size and dtype), so any
partial it read without writing first would be the first call's. Each output
must equal, bit for bit, the workspace path (pa_decode_splitkv + pa_merge with
caller-allocated partials that start out NaN): both run the same kernels on
the same inputs. The second call is also checked against the fp64 oracle. A
request larger than the array is refused with PA_ERR_WORKSPACE. The file name
makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import oracle
import workloads as W
from tests.gpu_common import assert_close, require_gpu

pytestmark = pytest.mark.gpu

PA_ERR_WORKSPACE = -5
_DT = {torch.float16: 1, torch.bfloat16: 2}


def _lib():
    import paged_kv_cache_475_b200 as pa

    lib = ctypes.CDLL(pa.LIB_PATH)  # the library the binding has loaded
    lib.pa_decode_splitkv_noalloc.restype = ctypes.c_int
    lib.pa_noalloc_scratch_bytes.restype = ctypes.c_size_t
    return lib


def _noalloc(lib, out, b, partition, num_parts):
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.pa_decode_splitkv_noalloc(
        p(out), p(b.q), p(b.k_cache), p(b.v_cache), p(b.block_tables), ctypes.c_int(b.block_tables.shape[1]),
        p(b.context_lens), ctypes.c_int(b.num_seqs), ctypes.c_int(b.num_q_heads), ctypes.c_int(b.num_kv_heads),
        ctypes.c_int(b.head_dim), ctypes.c_int(b.block_size), ctypes.c_int(b.num_blocks), ctypes.c_int(partition),
        ctypes.c_int(num_parts), ctypes.c_float(b.scale), ctypes.c_int(_DT[b.q.dtype]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _workspace_path(b, partition, num_parts):
    import paged_kv_cache_475_b200 as pa

    po, pm, pl = pa.splitkv_buffers(b.num_seqs, b.num_q_heads, b.head_dim, num_parts)
    for t in (po, pm, pl):
        t.fill_(float("nan"))  # a partial read before it is written would show
    out = torch.empty_like(b.q)
    pa.pa_decode_splitkv(po, pm, pl, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, partition, b.scale)
    pa.pa_merge(out, po, pm, pl, b.context_lens, partition)
    return out


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    require_gpu()
    lib = _lib()
    assert lib.pa_noalloc_scratch_bytes() == 16 << 20
    # (batch, partition): first the larger footprint (3 x 32 rows x 36 partitions of 256 tokens, D = 128),
    # then a smaller one laid out differently (4 x 8 rows x 5 partitions of 512 tokens, D = 64, bf16)
    first = W.make_batch("noalloc_a", [9000, 4000, 17], num_q_heads=32, num_kv_heads=8, head_dim=128,
                         block_size=32, dtype="f16", seed=202, poison=None)
    second = W.make_batch("noalloc_b", [1, 300, 1200, 2500], num_q_heads=8, num_kv_heads=4, head_dim=64,
                          block_size=16, dtype="bf16", seed=201, poison=None)
    for k, (b_cpu, partition) in enumerate([(first, 256), (second, 512)]):
        b = b_cpu.to("cuda")
        num_parts = (int(b.context_lens.max()) + partition - 1) // partition
        out = torch.full_like(b.q, float("nan"))
        assert _noalloc(lib, out, b, partition, num_parts) == 0
        ref = _workspace_path(b, partition, num_parts)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {k}: differs from the workspace path"
        if k == 1:
            expect = oracle.attention(b_cpu.q, b_cpu.k_cache, b_cpu.v_cache, b_cpu.block_tables, b_cpu.context_lens,
                                      b_cpu.scale)
            assert_close(out, expect, "bf16", "noalloc second call vs oracle")


def test_noalloc_refuses_requests_larger_than_its_array():
    require_gpu()
    lib = _lib()
    b = W.make_batch("noalloc_big", [64, 64], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                     dtype="f16", seed=203, poison=None).to("cuda")
    out = torch.empty_like(b.q)
    # 2 x 8 rows x 100000 partitions x 130 floats is far more than 16 MiB
    assert _noalloc(lib, out, b, 512, 100_000) == PA_ERR_WORKSPACE
