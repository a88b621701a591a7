"""Python binding of libpa.so, the paged-KV attention library for B200 (sm_100a).

Argument marshalling only: every function here checks the torch tensors it is
given (device, dtype, contiguity), derives the sizes the C ABI wants from
their shapes, and calls the entry point of the same name in libpa.so on the
current CUDA stream. All arithmetic runs in the library's CUDA kernels; there
is no CPU fallback. Importing the package fails loudly if libpa.so is missing
(build it with `python paged_kv_cache_475_b200/build.py`).

The C declarations and their contracts are in include/pa.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa.so")  # the in-tree build, always

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python paged_kv_cache_475_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
PA_ERR_CUDA = -6
_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}

DEVERR_BLOCK_ID = 0x1
DEVERR_CONTEXT = 0x2
DEVERR_SLOT = 0x4
DEVERR_WAIT = 0x8
DEVERR_POSITION = 0x10
DEVERR_SETUP = 0x20

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_SIGS = {
    "pa_slot_mapping": [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _vp],
    "pa_reshape_and_cache": [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp],
    "pa_copy_blocks": [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp],
    "pa_decode": [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp],
    "pa_decode_selftest_starved_wait": [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                                        ctypes.c_longlong, _vp],
    "pa_decode_append": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp],
    "pa_decode_shared_prefix": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                _vp, _vp, _i, _f, _i, _vp],
    "pa_splitkv_num_partitions": [_i, _i],
    "pa_splitkv_workspace_bytes": [_i, _i, _i, _i, _i],
    "pa_decode_splitkv": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                          _i, _vp],
    "pa_decode_splitkv_append": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i,
                                 _i, _f, _i, _vp],
    "pa_merge": [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp],
    "pa_prefill_chunk": [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp],
    "pa_decode_splitkv_noalloc": [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                                  _vp],
    "pa_noalloc_scratch_bytes": [],
    "pa_read_error_flags": [ctypes.POINTER(ctypes.c_uint32), _i],
    "pa_status_string": [_i],
    "pa_last_cuda_error": [],
    "pa_version": [],
    "pa_trace_clear": [],
    "pa_trace_read": [_vp, _i],
}
for _name, _args in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = {"pa_status_string": ctypes.c_char_p, "pa_last_cuda_error": ctypes.c_char_p,
                   "pa_noalloc_scratch_bytes": _sz, "pa_splitkv_workspace_bytes": _sz}.get(_name, _i)


class PagedAttentionError(RuntimeError):
    pass


def _check(status: int, name: str) -> None:
    if status != 0:
        msg = f"{name}: {_lib.pa_status_string(status).decode()}"
        if status == PA_ERR_CUDA:
            msg += f" [{_lib.pa_last_cuda_error().decode()}]"
        raise PagedAttentionError(msg)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, dim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}; the kernels run on the current device cuda:"
                         f"{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got {t.dim()}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def version() -> int:
    return _lib.pa_version()


def pa_splitkv_num_partitions(max_context_len: int, partition_size: int) -> int:
    return _lib.pa_splitkv_num_partitions(int(max_context_len), int(partition_size))


def pa_splitkv_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                               partition_size: int) -> int:
    """Bytes of one buffer holding part_o, part_m and part_l (layout in include/pa.h); 0 if invalid."""
    return _lib.pa_splitkv_workspace_bytes(int(num_seqs), int(num_q_heads), int(head_dim), int(max_context_len),
                                           int(partition_size))


def pa_slot_mapping(slot_mapping, block_tables, seq_idx, positions, block_size: int, stream=None):
    """slot_mapping[t] = block_tables[seq_idx[t]][positions[t] // B] * B + positions[t] % B (int64)."""
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(seq_idx, "seq_idx", torch.int32, 1)
    _need(positions, "positions", torch.int32, 1)
    T = slot_mapping.shape[0]
    if seq_idx.shape[0] != T or positions.shape[0] != T:
        raise ValueError("slot_mapping, seq_idx and positions must have the same length")
    _check(_lib.pa_slot_mapping(_ptr(slot_mapping), _ptr(block_tables), block_tables.shape[1], _ptr(seq_idx),
                                _ptr(positions), T, block_tables.shape[0], int(block_size), _stream(stream)),
           "pa_slot_mapping")


def pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping, stream=None):
    """Write k_new/v_new [T, Hkv, D] into k_cache/v_cache [P, Hkv, B, D] at slot_mapping (int64 [T])."""
    for n, t in (("k_new", k_new), ("v_new", v_new)):
        _need(t, n, k_cache.dtype, 3)
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, n, None, 4)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    P, Hkv, B, D = k_cache.shape
    T = slot_mapping.shape[0]
    if v_cache.shape != k_cache.shape or k_new.shape != (T, Hkv, D) or v_new.shape != (T, Hkv, D):
        raise ValueError("shape mismatch between new rows, caches and slot_mapping")
    _check(_lib.pa_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                     T, P, Hkv, D, B, _dtype_code(k_cache), _stream(stream)),
           "pa_reshape_and_cache")


def pa_copy_blocks(dst_k, dst_v, src_k, src_v, src_block_ids, dst_block_ids, stream=None):
    """dst[dst_block_ids[i]] = src[src_block_ids[i]] for K and V pools [P, Hkv, B, D].

    Pools may be CUDA tensors or pinned host tensors (device-addressable); the
    id tensors (int32) likewise. Copy-on-write: dst pools = src pools.
    """
    for n, t in (("dst_k", dst_k), ("dst_v", dst_v), ("src_k", src_k), ("src_v", src_v)):
        if not isinstance(t, torch.Tensor) or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous [P, Hkv, B, D] tensor")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{n} must be a CUDA tensor or pinned host memory")
        if t.is_cuda and t.device.index != torch.cuda.current_device():
            raise ValueError(f"{n} is on {t.device}, not on the current device")
    for n, t in (("src_block_ids", src_block_ids), ("dst_block_ids", dst_block_ids)):
        if t.dtype != torch.int32 or t.dim() != 1 or not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{n} must be int32 [n], on the GPU or pinned")
    if dst_k.shape[1:] != src_k.shape[1:] or dst_v.shape != dst_k.shape or src_v.shape != src_k.shape:
        raise ValueError("pool shapes differ")
    if dst_k.dtype != src_k.dtype:
        raise ValueError("pool dtypes differ")
    n = src_block_ids.shape[0]
    if dst_block_ids.shape[0] != n:
        raise ValueError("id arrays differ in length")
    _, Hkv, B, D = src_k.shape
    _check(_lib.pa_copy_blocks(_ptr(dst_k), _ptr(dst_v), dst_k.shape[0], _ptr(src_k), _ptr(src_v), src_k.shape[0],
                               _ptr(src_block_ids), _ptr(dst_block_ids), n, Hkv, D, B, _dtype_code(src_k),
                               _stream(stream)), "pa_copy_blocks")


def _cache_dims(q, k_cache, v_cache, block_tables, context_lens):
    _need(k_cache, "k_cache", q.dtype, 4)
    _need(v_cache, "v_cache", q.dtype, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    P, Hkv, B, D = k_cache.shape
    N = context_lens.shape[0]
    if block_tables.shape[0] != N:
        raise ValueError("block_tables and context_lens disagree on the number of sequences")
    return P, Hkv, B, D, N


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float, stream=None):
    """out[N, Hq, D] = paged attention of q[N, Hq, D] over each sequence's context."""
    _need(q, "q", None, 3)
    _need(out, "out", q.dtype, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    if q.shape[0] != N or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q/out must be [N, Hq, D]")
    _check(_lib.pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                          block_tables.shape[1], _ptr(context_lens), N, q.shape[1], Hkv, D, B, P, float(scale),
                          _dtype_code(q), _stream(stream)), "pa_decode")


def pa_decode_selftest_starved_wait(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                    wait_cycles: int, stream=None):
    """pa_decode with one copy wait that must time out (PA_DEVERR_WAIT); a self-test, not attention."""
    _need(q, "q", None, 3)
    _need(out, "out", q.dtype, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    if q.shape[0] != N or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q/out must be [N, Hq, D]")
    _check(_lib.pa_decode_selftest_starved_wait(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), N, q.shape[1], Hkv, D, B, P, float(scale), _dtype_code(q), int(wait_cycles),
        _stream(stream)), "pa_decode_selftest_starved_wait")


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, scale: float,
                     stream=None):
    """Write each sequence's newest token (k_new/v_new [N, Hkv, D], position L-1) into its slot, then decode."""
    _need(q, "q", None, 3)
    _need(out, "out", q.dtype, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    for n, t in (("k_new", k_new), ("v_new", v_new)):
        _need(t, n, q.dtype, 3)
        if t.shape != (N, Hkv, D):
            raise ValueError(f"{n} must be [N, Hkv, D]")
    if q.shape[0] != N or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q/out must be [N, Hq, D]")
    _check(_lib.pa_decode_append(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), N, q.shape[1], Hkv,
                                 D, B, P, float(scale), _dtype_code(q), _stream(stream)), "pa_decode_append")


def pa_decode_splitkv(part_o, part_m, part_l, q, k_cache, v_cache, block_tables, context_lens,
                      partition_size: int, scale: float, stream=None):
    """Per-partition (o, m, l) of a decode step; part_o [N, Hq, NP, D], part_m/part_l [N, Hq, NP] fp32."""
    _need(q, "q", None, 3)
    _need(part_o, "part_o", torch.float32, 4)
    _need(part_m, "part_m", torch.float32, 3)
    _need(part_l, "part_l", torch.float32, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    NP = part_o.shape[2]
    if part_o.shape != (N, q.shape[1], NP, D) or part_m.shape != (N, q.shape[1], NP) or part_l.shape != part_m.shape:
        raise ValueError("partial buffers must be [N, Hq, NP, D] and [N, Hq, NP]")
    _check(_lib.pa_decode_splitkv(_ptr(part_o), _ptr(part_m), _ptr(part_l), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), N, q.shape[1],
                                  Hkv, D, B, P, int(partition_size), NP, float(scale), _dtype_code(q),
                                  _stream(stream)), "pa_decode_splitkv")


def pa_decode_shared_prefix(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, prefix_len: int,
                            group_size: int, part_o, part_m, part_l, scale: float, stream=None):
    """Decode where sequences 0..group_size-1 share their first prefix_len tokens' blocks (cascade:
    prefix once on the tensor cores, suffixes split-KV, merge). k_new/v_new may be None (no append)."""
    _need(q, "q", None, 3)
    _need(out, "out", q.dtype, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        for n, t in (("k_new", k_new), ("v_new", v_new)):
            _need(t, n, q.dtype, 3)
            if t.shape != (N, Hkv, D):
                raise ValueError(f"{n} must be [N, Hkv, D]")
    _need(part_o, "part_o", torch.float32, 4)
    _need(part_m, "part_m", torch.float32, 3)
    _need(part_l, "part_l", torch.float32, 3)
    NP = part_o.shape[2]
    if part_o.shape != (N, q.shape[1], NP, D) or part_m.shape != (N, q.shape[1], NP) or part_l.shape != part_m.shape:
        raise ValueError("partial buffers must be [N, Hq, NP, D] and [N, Hq, NP]")
    _check(_lib.pa_decode_shared_prefix(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), N, q.shape[1],
                                        Hkv, D, B, P, int(prefix_len), int(group_size), _ptr(part_o), _ptr(part_m),
                                        _ptr(part_l), NP, float(scale), _dtype_code(q), _stream(stream)),
           "pa_decode_shared_prefix")


def pa_decode_splitkv_append(part_o, part_m, part_l, q, k_new, v_new, k_cache, v_cache, block_tables,
                             context_lens, partition_size: int, scale: float, stream=None):
    """pa_decode_splitkv plus the write of each sequence's newest K/V row (k_new/v_new [N, Hkv, D])."""
    _need(q, "q", None, 3)
    _need(part_o, "part_o", torch.float32, 4)
    _need(part_m, "part_m", torch.float32, 3)
    _need(part_l, "part_l", torch.float32, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    for n, t in (("k_new", k_new), ("v_new", v_new)):
        _need(t, n, q.dtype, 3)
        if t.shape != (N, Hkv, D):
            raise ValueError(f"{n} must be [N, Hkv, D]")
    NP = part_o.shape[2]
    if part_o.shape != (N, q.shape[1], NP, D) or part_m.shape != (N, q.shape[1], NP) or part_l.shape != part_m.shape:
        raise ValueError("partial buffers must be [N, Hq, NP, D] and [N, Hq, NP]")
    _check(_lib.pa_decode_splitkv_append(_ptr(part_o), _ptr(part_m), _ptr(part_l), _ptr(q), _ptr(k_new), _ptr(v_new),
                                         _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
                                         _ptr(context_lens), N, q.shape[1], Hkv, D, B, P, int(partition_size), NP,
                                         float(scale), _dtype_code(q), _stream(stream)), "pa_decode_splitkv_append")


def pa_merge(out, part_o, part_m, part_l, context_lens, partition_size: int, stream=None):
    """Combine split-KV partials into out [N, Hq, D] (dtype of out)."""
    _need(out, "out", None, 3)
    _need(part_o, "part_o", torch.float32, 4)
    _need(part_m, "part_m", torch.float32, 3)
    _need(part_l, "part_l", torch.float32, 3)
    _need(context_lens, "context_lens", torch.int32, 1)
    N, Hq, NP, D = part_o.shape
    if out.shape != (N, Hq, D) or part_m.shape != (N, Hq, NP) or part_l.shape != (N, Hq, NP):
        raise ValueError("shape mismatch between out and partials")
    _check(_lib.pa_merge(_ptr(out), _ptr(part_o), _ptr(part_m), _ptr(part_l), _ptr(context_lens), N, Hq, D,
                         int(partition_size), NP, _dtype_code(out), _stream(stream)), "pa_merge")


def pa_prefill_chunk(out, q, k_cache, v_cache, block_tables, context_lens, scale: float, stream=None):
    """out[N, C, Hq, D] = causal paged attention of a C-token chunk per sequence (f16/bf16)."""
    _need(q, "q", None, 4)
    _need(out, "out", q.dtype, 4)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    if q.shape[0] != N or q.shape[3] != D or out.shape != q.shape:
        raise ValueError("q/out must be [N, C, Hq, D]")
    _check(_lib.pa_prefill_chunk(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                 block_tables.shape[1], _ptr(context_lens), N, q.shape[1], q.shape[2], Hkv, D, B,
                                 P, float(scale), _dtype_code(q), _stream(stream)), "pa_prefill_chunk")


def pa_decode_splitkv_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, partition_size: int,
                              num_partitions: int, scale: float, stream=None):
    """Split-KV decode + merge into out [N, Hq, D] with the partials in the library's fixed
    per-device array (no workspace from the caller); see include/pa.h for its limits."""
    _need(q, "q", None, 3)
    _need(out, "out", q.dtype, 3)
    P, Hkv, B, D, N = _cache_dims(q, k_cache, v_cache, block_tables, context_lens)
    if q.shape[0] != N or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q/out must be [N, Hq, D]")
    _check(_lib.pa_decode_splitkv_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                          block_tables.shape[1], _ptr(context_lens), N, q.shape[1], Hkv, D, B, P,
                                          int(partition_size), int(num_partitions), float(scale), _dtype_code(q),
                                          _stream(stream)), "pa_decode_splitkv_noalloc")


def pa_noalloc_scratch_bytes() -> int:
    return _lib.pa_noalloc_scratch_bytes()


def trace_clear() -> None:
    """Zero the timeline records (builds with PA_TRACE=1 only; see include/pa.h)."""
    _check(_lib.pa_trace_clear(), "pa_trace_clear")


def trace_read(max_records: int = 1 << 16):
    """Timeline records of the last traced launch as a numpy structured array (PA_TRACE=1 builds only)."""
    import numpy as np

    dt = np.dtype([("t_start", "<u8"), ("t_first", "<u8"), ("t_end", "<u8"), ("smid", "<i4"), ("seq", "<i4"),
                   ("kv_head", "<i4"), ("part", "<i4"), ("tokens", "<i4"), ("kind", "<i4")])
    buf = np.zeros(max_records, dtype=dt)
    _check(_lib.pa_trace_read(ctypes.c_void_p(buf.ctypes.data), int(max_records)), "pa_trace_read")
    return buf


def pa_read_error_flags(clear: bool = True) -> int:
    """Device error word (PA_DEVERR_* bits) of the current device; synchronises."""
    v = ctypes.c_uint32(0)
    _check(_lib.pa_read_error_flags(ctypes.byref(v), 1 if clear else 0), "pa_read_error_flags")
    return v.value


def splitkv_workspace(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int, partition_size: int,
                      device="cuda"):
    """(part_o, part_m, part_l) carved out of ONE caller-owned buffer of pa_splitkv_workspace_bytes bytes,
    at the offsets include/pa.h gives (each part starts on a 256-byte boundary)."""
    total = pa_splitkv_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, partition_size)
    if total == 0:
        raise ValueError("invalid split-KV workspace shape")
    NP = pa_splitkv_num_partitions(max_context_len, partition_size)
    cells = num_seqs * num_q_heads * NP
    o_bytes = (cells * head_dim * 4 + 255) // 256 * 256
    ml_bytes = (cells * 4 + 255) // 256 * 256
    if o_bytes + 2 * ml_bytes != total:
        raise RuntimeError("pa_splitkv_workspace_bytes disagrees with the documented layout")
    buf = torch.empty(total, dtype=torch.uint8, device=device)
    part_o = buf[:cells * head_dim * 4].view(torch.float32).view(num_seqs, num_q_heads, NP, head_dim)
    part_m = buf[o_bytes:o_bytes + cells * 4].view(torch.float32).view(num_seqs, num_q_heads, NP)
    part_l = buf[o_bytes + ml_bytes:o_bytes + ml_bytes + cells * 4].view(torch.float32).view(num_seqs, num_q_heads, NP)
    return part_o, part_m, part_l


def splitkv_buffers(num_seqs: int, num_q_heads: int, head_dim: int, num_partitions: int, device="cuda"):
    """Allocate (part_o, part_m, part_l) for pa_decode_splitkv (caller-owned workspace)."""
    part_o = torch.empty((num_seqs, num_q_heads, num_partitions, head_dim), dtype=torch.float32, device=device)
    part_m = torch.empty((num_seqs, num_q_heads, num_partitions), dtype=torch.float32, device=device)
    part_l = torch.empty_like(part_m)
    return part_o, part_m, part_l
