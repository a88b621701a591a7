"""Shared helpers of the GPU parity tests: run the CUDA path, compare with the oracle."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import workloads as W

# Tolerances: fp16/bf16 outputs vs the fp64 oracle, fp32 tiny config.
TOL_HALF_MAX, TOL_HALF_MEAN = 1e-2, 1e-3
TOL_F32_MAX = 1e-5


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA GPU (run with -m 'not gpu' on a CPU-only machine)")


def run_gpu(batch_cpu, partition="auto", fused_append="auto", shared_prefix=None):
    """One step of the batch on the GPU through the C ABI; returns (out, gpu_batch, error_flags)."""
    import paged_kv_cache_475_b200 as pa
    from paged_kv_cache_475_b200.step import run_batch

    pa.pa_read_error_flags(clear=True)
    g = batch_cpu.to("cuda")
    out = run_batch(g, partition, fused_append, shared_prefix)
    torch.cuda.synchronize()
    flags = pa.pa_read_error_flags(clear=True)
    return out.cpu(), g, flags


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype: str, what: str = ""):
    g = got.detach().cpu().to(torch.float64).numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    if dtype == "f32":
        assert err.max() <= TOL_F32_MAX, f"{what}: max abs err {err.max():.3e} > {TOL_F32_MAX}"
    else:
        assert err.max() <= TOL_HALF_MAX, f"{what}: max abs err {err.max():.3e} > {TOL_HALF_MAX}"
        assert err.mean() <= TOL_HALF_MEAN, f"{what}: mean abs err {err.mean():.3e} > {TOL_HALF_MEAN}"
    return float(err.max()), float(err.mean())


def small_batch(seed, dtype="f16", D=128, G=4, B=16, Hkv=2, lens=(1, 15, 16, 17, 100, 333, 700), chunk=1,
                poison=float("nan"), q_std=1.0, shared_prefix_tokens=0, shared_group=0, pool_factor=1.25):
    return W.make_batch(f"small_s{seed}", list(lens), num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D,
                        block_size=B, dtype=dtype, seed=seed, chunk=chunk, poison=poison, q_std=q_std,
                        shared_prefix_tokens=shared_prefix_tokens, shared_group=shared_group,
                        pool_factor=pool_factor)


def permute_pool(batch, seed=7):
    """The same batch with its physical blocks relabelled by a random permutation."""
    P = batch.k_cache.shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed))
    b2 = batch.to("cpu")
    b2.k_cache = torch.empty_like(batch.k_cache)
    b2.v_cache = torch.empty_like(batch.v_cache)
    b2.k_cache[perm] = batch.k_cache
    b2.v_cache[perm] = batch.v_cache
    bt = batch.block_tables.long()
    b2.block_tables = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
    return b2


def sample_rows(batch, n, seed=0):
    """Spread (b, i, h) rows over sequences, heads and chunk positions (first and last included)."""
    g = torch.Generator().manual_seed(seed)
    rows = []
    N, C, Hq = batch.num_seqs, batch.chunk, batch.num_q_heads
    for b in range(N):
        rows.append((b, C - 1, 0))
        rows.append((b, 0, Hq - 1))
    while len(rows) < n:
        rows.append((int(torch.randint(N, (1,), generator=g)), int(torch.randint(C, (1,), generator=g)),
                     int(torch.randint(Hq, (1,), generator=g))))
    return rows[:max(n, 2 * N)]


def gather_rows(out: torch.Tensor, rows, chunk: int):
    if chunk == 1:
        return torch.stack([out[b, h] for (b, i, h) in rows])
    return torch.stack([out[b, i, h] for (b, i, h) in rows])


def ln2():
    return math.log(2.0)
