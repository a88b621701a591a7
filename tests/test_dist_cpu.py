"""Multi-rank host logic of bench.py on the CPU (gloo, 2 ranks, 127.0.0.1).

bench.py shards by batch: every rank builds its own batch (seed offset by rank),
times its own steps, and rank 0 reports the summed bytes over the max time. This
checks that the ranks really get different batches, that the reductions give the
max time and the summed work, and that the weak-scaling value follows from them.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads as W

    b = W.make_batch("dist", W.llama_decode_lens(8, 64, 512, seed=1000 + 100 * rank), num_q_heads=8,
                     num_kv_heads=2, head_dim=64, block_size=16, dtype="f16", seed=1 + 100 * rank, poison=None)
    acct = bench.workload_bytes(b)
    fake_ms = 2.0 + rank  # rank 1 is the slow one
    t_max = bench.max_over_ranks(fake_ms, world, device="cpu")
    total = bench.sum_over_ranks(acct["kv_logical"], world, device="cpu")
    checksum = float(b.k_cache.float().sum())
    out[rank] = (t_max, total, acct["kv_logical"], checksum)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_reductions():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (t0, tot0, b0, c0), (t1, tot1, b1, c1) = out[0], out[1]
    assert t0 == t1 == 3.0                      # max over ranks
    assert tot0 == tot1 == b0 + b1              # summed work
    assert b0 != b1 and c0 != c1                # different batches per rank
    value = tot0 / (t0 / 1e3) / 1e9             # GB/s as bench.py reports it
    assert value == pytest.approx((b0 + b1) / 3e-3 / 1e9)
