"""Throughput bench of the paged-KV attention library on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload llama_decode|long_context|chat_trace|prefill_chunk]
                [--block-size B] [--partition auto|none|<tokens>] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the hot path over one batch: map the step's new tokens
to cache slots, write their K/V rows into the paged cache, then attend
(single-pass decode, or split-KV + merge, or the chunked prefill). The headline
workload is the Llama-3-8B-shaped single-layer decode (64 sequences, 32 q / 8
KV heads, head dim 128, block size 16, context lengths uniform in
[512, 4096], fp16). Inputs are synthetic and resident in HBM before timing;
the KV read per step (~0.6 GB) is larger than the 126 MB L2, so no flush is
needed between steps.

A default run (one GPU) also times the other workloads and puts them in a
"workloads" object of the same JSON line: the 4 x 100k split-KV decode, the
256-sequence chat trace (shared-prefix cascade, with the block-size sweep
8..128), the bf16 chunked prefill and the block swap. The headline value is
K timed steps, with a "sustained" run of the same step for about two seconds
beside it for the clock record; every other entry's value comes from one
timed region of about two seconds of steps (--sustain-seconds), whose clock
record has >= 10 samples under load, with its first K steps as "burst". Each
entry carries its roofline, end-to-end figure and clocks.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch
(weak scaling, no collective on the data path); the step time is the max
over ranks and the value counts every rank's bytes.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-KV decode attention achieved HBM GB/s (% of peak) and seq-steps/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0  # the same pool, seconds-long, under the 1000 W cap

WORKLOAD_DESC = {
    "llama_decode": "Llama-3-8B-shaped single-layer paged decode fp16: batch 64, 32 q / 8 KV heads, head_dim 128, "
                    "block_size 16, context_lens U[512,4096], pool 1.25x shuffled, one appended token per sequence",
    "long_context": "long-context split-KV paged decode fp16: batch 4 x 100000 tokens, 32 q / 8 KV heads, "
                    "head_dim 128, block_size 16, 512-token partitions + merge, q ~ N(0,2)",
    "chat_trace": "chat-trace paged decode fp16: batch 256, lognormal context_lens (median 300, sigma 1, "
                  "clipped [16,8192]), half sharing a 1024-token prefix, 32 q / 8 KV heads, head_dim 128",
    "prefill_chunk": "chunked prefill bf16: batch 8, 512 causal query tokens after a paged context U[2048,8192], "
                     "32 q / 8 KV heads, head_dim 128, block_size 16",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama_decode", choices=list(WORKLOAD_DESC) + ["block_swap"])
    ap.add_argument("--block-size", type=int, default=16)
    ap.add_argument("--partition", default="auto")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=16.0,
                    help="budget of the cpu_baseline samples (half with every core, half with one)")
    ap.add_argument("--sustain-seconds", type=float, default=2.0,
                    help="length of the extra run of each step that the clock record samples")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only --workload (by default the Llama decode line also carries the long-context, "
                         "chat-trace (with the block-size sweep) and prefill workloads)")
    ap.add_argument("--reference-seconds", type=float, default=100.0,
                    help="budget of the whole --impl reference run (sets its sample size)")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    a.all_workloads = not a.headline_only and int(os.environ.get("WORLD_SIZE", "1")) == 1
    return a


def make_workload(name, block_size, seed_offset=0, poison=None):
    import workloads as W

    if name == "llama_decode":
        return W.llama_decode(block_size=block_size, poison=poison, seed=1 + seed_offset)
    if name == "long_context":
        return W.long_context(block_size=block_size, poison=poison, seed=2 + seed_offset)
    if name == "chat_trace":
        return W.chat_trace(block_size=block_size, poison=poison, seed=3 + seed_offset)
    return W.prefill_chunk(block_size=block_size, poison=poison, seed=4 + seed_offset)


def workload_bytes(batch):
    """Algorithmic HBM bytes of one step (dict): the minimum a perfect kernel moves."""
    import workloads as W

    esz = batch.k_cache.element_size()
    Hkv, D = batch.num_kv_heads, batch.head_dim
    kv_logical = W.decode_kv_bytes(batch.context_lens.tolist(), Hkv, D, esz)
    kv_unique = W.decode_kv_bytes(batch.context_lens.tolist(), Hkv, D, esz, batch.block_tables,
                                  batch.block_size, unique=True)
    q_out = 2 * batch.q.numel() * esz
    nb = sum(W.blocks_for(int(L), batch.block_size) for L in batch.context_lens.tolist())
    tables = nb * 4 + batch.num_seqs * 4
    T = batch.new_seq.shape[0]
    append = 2 * 2 * T * Hkv * D * esz + T * (8 + 8)  # new rows read + written, slots
    return dict(kv_logical=kv_logical, kv_unique=kv_unique, q_out=q_out, tables=tables, append=append,
                attend_logical=kv_logical + q_out + tables, attend_unique=kv_unique + q_out + tables)



def workload_config(name, batch_cpu, partition_arg, world):
    """The line's `config`: the workload and its sizes only, the same for both arms (the reference arm
    builds it from the same batch without loading the library); how a step runs it is in `step_plan`."""
    acct = workload_bytes(batch_cpu)
    cascade = name == "chat_trace" and partition_arg == "auto"
    return {
        "workload": WORKLOAD_DESC[name], "num_seqs": batch_cpu.num_seqs, "block_size": batch_cpu.block_size,
        "head_dim": batch_cpu.head_dim, "num_q_heads": batch_cpu.num_q_heads,
        "num_kv_heads": batch_cpu.num_kv_heads,
        "l2": "inputs larger than L2 (KV read per step >> 126 MB), no flush" if not cascade else
              "unique KV (522 MB) larger than L2, no flush; the shared prefix is read once per step by design",
        "kv_bytes_logical_per_rank": acct["kv_logical"], "kv_bytes_unique_per_rank": acct["kv_unique"],
        "parallelism": f"dp{world} (independent batches per GPU)",
    }

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def measured_peaks_sustained_tflops():
    """The seconds-long cuBLAS bf16 figure (for a kernel timed inside a long run), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return d["bf16_tflops_sustained"]
    return FALLBACK_BF16_TFLOPS_SUSTAINED


def kernel_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    if d.get("source_sha256") != source_hash(d.get("sources", [])):
        return None
    return d.get("dram_bytes_per_launch")


def source_hash(files):
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons around timed regions.

    Each sample carries nvidia-smi's own timestamp. summary(t0, t1) keeps the
    samples that fall inside one region (widened by one sampling period on
    each side, so that a region shorter than the period still gets the samples
    that bracket it), after waiting up to a second for the first sample after
    the region so that one always exists. mark() names the region stop()
    summarises.
    """

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.2

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(int(self.PERIOD_S * 1000))], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        deadline = time.time() + 5.0  # the first sample before any timing starts
        while time.time() < deadline and not self._rows():
            time.sleep(0.05)

    def _rows(self):
        import datetime

        rows = []
        with open(self.f.name) as fh:
            for line in fh.read().splitlines():
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        return rows

    def mark(self, t0, t1):
        """Host wall-clock bounds of the timed region (time.time() before its first launch, after its sync)."""
        self.window = (t0, t1)

    def summary(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        deadline = time.time() + 1.0
        while time.time() < deadline and not any(r[0] >= t1 for r in self._rows()):
            time.sleep(0.05)
        rows = self._rows()
        inside = [r for r in rows if t0 - self.PERIOD_S <= r[0] <= t1 + self.PERIOD_S]
        if not inside:  # the sample nearest the region
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:1]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = {n for r in inside for n, v in zip(names, r[3]) if v.lower() == "active"}
        sm = [r[1] for r in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max((r[2] for r in inside),
                                                                                     default=None),
                "reasons": sorted(reasons), "samples": len(sm)}

    def stop(self):
        t0, t1 = self.window if self.window else (0.0, float("inf"))
        out = self.summary(t0, t1)
        self.close()
        return out

    def close(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            os.unlink(self.f.name)
            self.proc = None


def dist_init(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x, world, device="cuda"):
    import torch

    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device="cuda"):
    import torch

    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------------------
# CPU side: the oracle on a bounded sample (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_sample(batch, n_seqs):
    """A sub-batch of the first n_seqs sequences (same tables, same pool)."""
    import copy

    s = copy.copy(batch)
    s.q = batch.q[:n_seqs]
    s.block_tables = batch.block_tables[:n_seqs]
    s.context_lens = batch.context_lens[:n_seqs]
    keep = batch.new_seq < n_seqs
    s.new_seq, s.new_pos = batch.new_seq[keep], batch.new_pos[keep]
    s.k_new, s.v_new = batch.k_new[keep], batch.v_new[keep]
    return s


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def usable_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class host_threads:
    """Caps the host threads the oracle may use (BLAS pools and torch's intra-op pool) inside a with block."""

    def __init__(self, n):
        self.n = n

    def __enter__(self):
        import torch

        self.torch_prev = torch.get_num_threads()
        torch.set_num_threads(self.n)
        try:
            from threadpoolctl import threadpool_limits

            self.ctl = threadpool_limits(limits=self.n)
        except Exception:  # noqa: BLE001
            self.ctl = None
        return self

    def __exit__(self, *exc):
        import torch

        torch.set_num_threads(self.torch_prev)
        if self.ctl is not None:
            self.ctl.restore_original_limits()


def time_oracle(batch_cpu, budget_s, prefill=False):
    """Run the oracle step on growing samples until the budget is spent; returns (bytes_or_flops/s, info)."""
    import oracle
    import workloads as W

    n = 1
    done_units, spent, seqs_done, steps = 0.0, 0.0, 0, 0
    while spent < budget_s and n <= batch_cpu.num_seqs:
        s = oracle_sample(batch_cpu, n)
        t0 = time.perf_counter()
        oracle.step(s)
        dt = time.perf_counter() - t0
        if prefill:
            units = W.prefill_flops(s.context_lens.tolist(), s.chunk, s.num_q_heads, s.head_dim)
        else:
            units = W.decode_kv_bytes(s.context_lens.tolist(), s.num_kv_heads, s.head_dim, s.k_cache.element_size())
        done_units += units
        spent += dt
        seqs_done += n
        steps += 1
        if dt * 2 < budget_s - spent:
            n = min(batch_cpu.num_seqs, n * 2)
    return done_units / spent, dict(seconds=round(spent, 2), seqs=seqs_done, samples=steps)


def cpu_baseline(batch_cpu, budget_s, prefill, scale, unit):
    """The oracle as it stands, on the host: with every usable core, then with one."""
    cores = usable_cores()
    with host_threads(cores):
        v_all, info_all = time_oracle(batch_cpu, budget_s / 2, prefill)
    with host_threads(1):
        v_one, info_one = time_oracle(batch_cpu, budget_s / 2, prefill)
    return {
        "value": v_all / scale, "unit": unit, "cores": cores, "kind": "oracle",
        "all_cores": {"value": v_all / scale, "threads": cores, **info_all},
        "one_core": {"value": v_one / scale, "threads": 1, **info_one},
        "cpu_model": cpu_model(), "cpu_count": os.cpu_count(),
        "sample": "fp64 numpy oracle step (append + attention) on the first 1, 2, 4, ... sequences of the same "
                  f"batch: {info_all['seqs']} sequences in {info_all['seconds']} s with {cores} threads (BLAS and "
                  f"torch pools), {info_one['seqs']} in {info_one['seconds']} s with 1. The oracle's per-row "
                  "matrix-vector loop is mostly single-threaded, so the two figures are close.",
    }


def run_reference(args):
    """--impl reference: the fp64 CPU oracle, as it stands, on a bounded sample of the workload."""
    import torch  # noqa: F401

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    prefill = args.workload == "prefill_chunk"
    batch = make_workload(args.workload, args.block_size)
    per_step_budget = max(0.05, args.reference_seconds / (args.steps + args.warmup))
    # one sample size sized to the per-step budget
    import oracle
    import workloads as W

    n = 1
    while True:
        s = oracle_sample(batch, n)
        t0 = time.perf_counter()
        oracle.step(s)
        dt = time.perf_counter() - t0
        if dt * 2 > per_step_budget or n >= batch.num_seqs:
            break
        n = min(batch.num_seqs, n * 2)
    sample = oracle_sample(batch, n)
    for _ in range(args.warmup):
        oracle.step(sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.step(sample)
    dt = time.perf_counter() - t0
    if prefill:
        units = W.prefill_flops(sample.context_lens.tolist(), sample.chunk, sample.num_q_heads, sample.head_dim)
        value, unit = units * args.steps / dt / 1e12, "TFLOP/s"
    else:
        units = W.decode_kv_bytes(sample.context_lens.tolist(), sample.num_kv_heads, sample.head_dim,
                                  sample.k_cache.element_size())
        value, unit = units * args.steps / dt / 1e9, "GB/s"
    import torch as _t

    threads = _t.get_num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args.workload, batch, args.partition, args.gpus),
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(), "cpu_count": os.cpu_count(),
                         "sample": f"first {n} of {batch.num_seqs} sequences per step, fp64 numpy"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ---------------------------------------------------------------------------
# GPU side
# ---------------------------------------------------------------------------

def measure(name, block_size, partition_arg, K, W, rank, world, sampler, do_e2e=True, sustain_s=2.0,
            cpu_budget_s=0.0, long_timed=False):
    """Time one workload's step and return the fields of its JSON entry.

    Default (the headline): K timed steps give the value; a separate ~sustain_s run of the same step gives
    the clock record under load ("sustained"). long_timed (the other workloads): K steps first ("burst"),
    then the value, kernel time and clock record all come from one timed region of ~sustain_s worth of
    steps, so the clock sampler sees >= 10 samples under load; the tensor-bound roofline then uses the
    sustained bf16 peak. Both end with K end-to-end steps from host buffers."""
    import torch

    import paged_kv_cache_475_b200 as pa
    import workloads as Wl
    from paged_kv_cache_475_b200.step import DecodeStep, PrefillStep

    prefill = name == "prefill_chunk"
    batch_cpu = make_workload(name, block_size, seed_offset=100 * rank)
    batch = batch_cpu.to("cuda")
    acct = workload_bytes(batch_cpu)
    part = None
    sp = None
    if prefill:
        step = PrefillStep(batch.num_seqs, batch.chunk, batch.num_q_heads, batch.head_dim, batch.q.dtype,
                           num_new_tokens=batch.new_seq.shape[0])
        partition = None
    else:
        part = "auto" if partition_arg == "auto" else (None if partition_arg == "none" else int(partition_arg))
        # chat trace: half the batch shares a 1024-token prompt -> the shared-prefix cascade
        sp = (batch_cpu.info["shared_prefix_tokens"], batch_cpu.info["shared_group"]) \
            if name == "chat_trace" and partition_arg == "auto" else None
        step = DecodeStep(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                          int(batch_cpu.context_lens.max()), batch.q.dtype,
                          num_new_tokens=batch.new_seq.shape[0], partition=part, shared_prefix=sp)
        partition = step.partition
    stream = torch.cuda.current_stream()
    args_step = (batch.q, batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, batch.block_tables,
                 batch.context_lens, batch.new_seq, batch.new_pos, batch.scale)

    fused = (not prefill) and step.fused
    cascade = (not prefill) and getattr(step, "shared_prefix", None) is not None
    # A step that is one launch (or the cascade's fixed sequence) is timed by
    # one event at its end; its duration is the interval from the previous
    # step's end event (the timed region's start for the first step), which
    # includes the launch gap. An event pair around every launch would add
    # its own stream operations to each step.
    end_only = cascade or (fused and not partition)

    def run_step(ev=None):
        if cascade:
            step(*args_step)
            if ev is not None:
                ev[1].record(stream)
            return
        if fused and partition:
            if ev is not None:
                ev[0].record(stream)
            pa.pa_decode_splitkv_append(step.part_o, step.part_m, step.part_l, batch.q, batch.k_new, batch.v_new,
                                        batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens,
                                        partition, batch.scale)
            if ev is not None:
                ev[1].record(stream)
            pa.pa_merge(step.out, step.part_o, step.part_m, step.part_l, batch.context_lens, partition)
            return
        if fused:
            pa.pa_decode_append(step.out, batch.q, batch.k_new, batch.v_new, batch.k_cache, batch.v_cache,
                                batch.block_tables, batch.context_lens, batch.scale)
            if ev is not None:
                ev[1].record(stream)
            return
        B = batch.k_cache.shape[2]
        pa.pa_slot_mapping(step.slot_mapping, batch.block_tables, batch.new_seq, batch.new_pos, B)
        pa.pa_reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache, step.slot_mapping)
        if ev is not None:
            ev[0].record(stream)
        if prefill:
            pa.pa_prefill_chunk(step.out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                                batch.context_lens, batch.scale)
        elif partition:
            pa.pa_decode_splitkv(step.part_o, step.part_m, step.part_l, batch.q, batch.k_cache, batch.v_cache,
                                 batch.block_tables, batch.context_lens, partition, batch.scale)
        else:
            pa.pa_decode(step.out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens,
                         batch.scale)
        if ev is not None:
            ev[1].record(stream)
        if partition and not prefill:
            pa.pa_merge(step.out, step.part_o, step.part_m, step.part_l, batch.context_lens, partition)

    for _ in range(W):
        run_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    def timed_steps(n):
        """n steps in one timed region: (ms per step, max over ranks; mean dominant-kernel ms; wall window)."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        w0 = time.time()
        t_start.record(stream)
        for i in range(n):
            run_step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        w1 = time.time()
        barrier(world)
        torch.cuda.synchronize()
        ms = max_over_ranks(t_start.elapsed_time(t_end), world) / n
        if end_only:
            ends = [t_start] + [b for _, b in evs]
            km = statistics.mean(ends[i].elapsed_time(ends[i + 1]) for i in range(n))
        else:
            km = statistics.mean(a.elapsed_time(b) for a, b in evs)
        return ms, km, (w0, w1)

    # ---- the K timed steps ----------------------------------------------------
    ms_step, kern_ms, win_timed = timed_steps(K)
    n_long = int(min(200000, max(K, sustain_s / max(ms_step / 1e3, 1e-6))))
    n_long = int(max_over_ranks(n_long, world))
    burst = None
    n_sus = ms_sus = win_sus = None
    if long_timed:
        # ---- the entry's value: ~sustain_s of steps in one timed region ------------
        burst = {"steps": K, "ms_per_step": ms_step, "kernel_ms": kern_ms}
        ms_step, kern_ms, win_timed = timed_steps(n_long)
    else:
        # ---- the same step for ~sustain_s, so the clock record has samples under load
        n_sus = n_long
        s_start, s_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        s0 = time.time()
        s_start.record(stream)
        for _ in range(n_sus):
            run_step()
        s_end.record(stream)
        torch.cuda.synchronize()
        s1 = time.time()
        barrier(world)
        ms_sus = max_over_ranks(s_start.elapsed_time(s_end), world) / n_sus
        win_sus = (s0, s1)
    flags = pa.pa_read_error_flags(clear=True)

    hbm_peak, tf_peak, peak_src = measured_peaks()
    tf_peak_sus = measured_peaks_sustained_tflops()
    if prefill:
        flops = Wl.prefill_flops(batch_cpu.context_lens.tolist(), batch.chunk, batch.num_q_heads, batch.head_dim)
        units_rank, scale, unit = flops, 1e12, "TFLOP/s"
        achieved = flops / (kern_ms / 1e3) / 1e12
        peak_used = tf_peak_sus if long_timed else tf_peak
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak_used, "unit": "TFLOP/s",
                "frac": achieved / peak_used, "traffic": kernel_traffic("prefill_chunk"),
                "peak_source": (f"{peak_src} bf16 sustained (cuBLAS, seconds-long loop under the power cap)"
                                if long_timed else f"{peak_src} bf16 burst (cuBLAS)"),
                "kernel": "pa_prefill_chunk", "kernel_ms": kern_ms, "algorithmic_flops_per_launch": flops}
        if burst is not None:
            a = flops / (burst["kernel_ms"] / 1e3) / 1e12
            burst.update({"value": flops * world / (burst["ms_per_step"] / 1e3) / 1e12, "unit": unit,
                          "kernel_achieved": a, "roofline_frac": a / tf_peak,
                          "peak_source": f"{peak_src} bf16 burst (cuBLAS)"})
    else:
        units_rank, scale, unit = acct["kv_logical"], 1e9, "GB/s"
        kname = ("pa_decode_shared_prefix" if cascade else
                 ("pa_decode_splitkv_append" if partition else "pa_decode_append") if fused else
                 ("pa_decode_splitkv" if partition else "pa_decode"))
        attend_bytes = acct["attend_unique"] + (acct["append"] if fused else 0)
        achieved = attend_bytes / (kern_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": kernel_traffic(f"{kname}:{name}:B{block_size}"),
                "peak_source": f"{peak_src} HBM copy bandwidth", "kernel": kname, "kernel_ms": kern_ms,
                "algorithmic_bytes_per_launch": attend_bytes}
        if burst is not None:
            a = attend_bytes / (burst["kernel_ms"] / 1e3) / 1e9
            burst.update({"value": sum_over_ranks(units_rank, world) / (burst["ms_per_step"] / 1e3) / scale,
                          "unit": unit, "kernel_achieved": a, "roofline_frac": a / hbm_peak})
    value = sum_over_ranks(units_rank, world) / (ms_step / 1e3) / scale

    # ---- end to end: host buffers in, result out, through the C ABI -----------
    # Every step uploads its inputs (q, the new K/V rows, block tables, context
    # lengths, new-token indices) from pinned host memory and reads its output
    # back into pinned host memory. As in a serving loop, the transfers run on
    # their own streams and overlap the neighbouring steps' kernels: inputs and
    # outputs are double-buffered (two step objects, two device staging
    # buffers), and events order every buffer's reuse. The inputs travel as one
    # packed staging buffer (one upload per step).
    e2e = None
    if do_e2e:
        templates = [batch.q, batch.k_new, batch.v_new, batch.block_tables, batch.context_lens, batch.new_seq,
                     batch.new_pos]
        offs, off = [], 0
        for t in templates:
            off = (off + 255) // 256 * 256
            offs.append(off)
            off += t.numel() * t.element_size()
        staging_bytes = off
        host_in = torch.empty(staging_bytes, dtype=torch.uint8).pin_memory()
        for t, o in zip(templates, offs):  # the caller's inputs, in host memory
            n = t.numel() * t.element_size()
            host_in[o:o + n].copy_(t.cpu().contiguous().view(-1).view(torch.uint8))
        dev_in = [torch.empty(staging_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]

        def views(buf):
            out = []
            for t, o in zip(templates, offs):
                n = t.numel() * t.element_size()
                out.append(buf[o:o + n].view(t.dtype).view(t.shape))
            return out

        dev_views = [views(d) for d in dev_in]
        if prefill:
            steps = [PrefillStep(batch.num_seqs, batch.chunk, batch.num_q_heads, batch.head_dim, batch.q.dtype,
                                 num_new_tokens=batch.new_seq.shape[0]) for _ in range(2)]
        else:
            steps = [DecodeStep(batch.num_seqs, batch.num_q_heads, batch.num_kv_heads, batch.head_dim,
                                int(batch_cpu.context_lens.max()), batch.q.dtype,
                                num_new_tokens=batch.new_seq.shape[0], partition=part, shared_prefix=sp)
                     for _ in range(2)]
        host_out = [torch.empty(steps[k].out.shape, dtype=steps[k].out.dtype).pin_memory() for k in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in templates)
        d2h = host_out[0].numel() * host_out[0].element_size()
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_kern = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            s = i % 2
            up.wait_event(ev_kern[s])          # step i-2 no longer reads this staging buffer
            with torch.cuda.stream(up):
                dev_in[s].copy_(host_in, non_blocking=True)
            ev_up[s].record(up)
            stream.wait_event(ev_up[s])        # this step's inputs have landed
            stream.wait_event(ev_down[s])      # step i-2's output has been read back
            q, k_new, v_new, bt, lens, new_seq, new_pos = dev_views[s]
            out = steps[s](q, k_new, v_new, batch.k_cache, batch.v_cache, bt, lens, new_seq, new_pos, batch.scale)
            ev_kern[s].record(stream)
            down.wait_event(ev_kern[s])
            with torch.cuda.stream(down):
                host_out[s].copy_(out, non_blocking=True)
            ev_down[s].record(down)

        for i in range(W):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        for i in range(K):
            e2e_step(i)
        for s in range(2):
            stream.wait_event(ev_down[s])      # the last results are in host memory
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world) / K
        e2e = {"value": sum_over_ranks(units_rank, world) / (ms_e2e / 1e3) / scale, "unit": unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "transfers": "overlapped with compute (separate copy streams, double-buffered)"}
        flags |= pa.pa_read_error_flags(clear=True)

    cpu = None
    if cpu_budget_s > 0 and rank == 0 and world == 1:
        cpu = cpu_baseline(batch_cpu, cpu_budget_s, prefill, scale, unit)

    res = {
        "value": value, "unit": unit, "ms_per_step": ms_step, "steps": n_long if long_timed else K, "warmup": W,
        "dtype": batch_cpu.info["dtype"],
        "config": workload_config(name, batch_cpu, partition_arg if not prefill else "auto", world),
        "step_plan": {"partition": partition, "fused_append": fused,
                      "shared_prefix": list(step.shared_prefix) if cascade else None},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": step.launches_per_call * (n_long if long_timed else K),
        "device_error_flags": flags,
        "_windows": {"timed": win_timed},
    }
    if long_timed:
        res["burst"] = burst
    else:
        res["sustained"] = {"steps": n_sus, "ms_per_step": ms_sus,
                            "value": sum_over_ranks(units_rank, world) / (ms_sus / 1e3) / scale, "unit": unit}
        res["_windows"]["sustained"] = win_sus
    if cpu is not None:
        res["cpu_baseline"] = cpu
    if not prefill:
        res["seq_steps_per_s"] = batch.num_seqs * world / (ms_step / 1e3)
        res["pct_of_peak"] = 100.0 * value / (hbm_peak * world)
        if acct["kv_unique"] != acct["kv_logical"]:
            res["unique_bytes_frac"] = acct["attend_unique"] / (ms_step / 1e3) / 1e9 / hbm_peak
    del step, batch, args_step
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def measure_block_swap(K, W, rank, world, runs=64, run_blocks=32):
    """Block copies of the Llama-shaped pool (8 KV heads x 16 tokens x 128 dims, fp16: 64 KiB of K+V per
    block): swap-out to and swap-in from a pinned host pool through pa_copy_blocks (the kernel reads or
    writes host memory directly), the same bytes as one cudaMemcpyAsync per contiguous run of blocks, and
    a device-side copy-on-write of as many blocks. Every figure is bytes moved / CUDA-event time."""
    import torch

    import paged_kv_cache_475_b200 as pa

    Hkv, B, D = 8, 16, 128
    n = runs * run_blocks
    P_dev = 4 * n
    g = torch.Generator().manual_seed(5 + 100 * rank)
    kd = torch.randn((P_dev, Hkv, B, D), generator=g).to(torch.float16).cuda()
    vd = torch.randn((P_dev, Hkv, B, D), generator=g).to(torch.float16).cuda()
    kh = torch.empty((n, Hkv, B, D), dtype=torch.float16).pin_memory()
    vh = torch.empty((n, Hkv, B, D), dtype=torch.float16).pin_memory()
    starts = (torch.randperm(P_dev // run_blocks, generator=g)[:runs] * run_blocks).tolist()
    dev_ids = torch.tensor([s0 + j for s0 in starts for j in range(run_blocks)], dtype=torch.int32)
    host_ids = torch.arange(n, dtype=torch.int32)
    dev_ids_g, host_ids_g = dev_ids.cuda(), host_ids.cuda()
    block_bytes = 2 * Hkv * B * D * 2
    moved = n * block_bytes
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world) / K

    def out_kernel():
        pa.pa_copy_blocks(kh, vh, kd, vd, dev_ids_g, host_ids_g)

    def in_kernel():
        pa.pa_copy_blocks(kd, vd, kh, vh, host_ids_g, dev_ids_g)

    def out_memcpy():
        for r, s0 in enumerate(starts):
            h0 = r * run_blocks
            kh[h0:h0 + run_blocks].copy_(kd[s0:s0 + run_blocks], non_blocking=True)
            vh[h0:h0 + run_blocks].copy_(vd[s0:s0 + run_blocks], non_blocking=True)

    def in_memcpy():
        for r, s0 in enumerate(starts):
            h0 = r * run_blocks
            kd[s0:s0 + run_blocks].copy_(kh[h0:h0 + run_blocks], non_blocking=True)
            vd[s0:s0 + run_blocks].copy_(vh[h0:h0 + run_blocks], non_blocking=True)

    kd_one = kd[:n]
    cow_src = dev_ids_g
    cow_dst = torch.tensor([(int(i) + 2 * n) % P_dev for i in dev_ids], dtype=torch.int32).cuda()

    def cow_kernel():
        pa.pa_copy_blocks(kd, vd, kd, vd, cow_src, cow_dst)

    res = {}
    for name, fn in (("swap_out_kernel", out_kernel), ("swap_in_kernel", in_kernel),
                     ("swap_out_memcpy_per_run", out_memcpy), ("swap_in_memcpy_per_run", in_memcpy)):
        ms = timed(fn)
        res[name] = {"ms": ms, "GB/s": moved / (ms / 1e3) / 1e9}
    ms = timed(lambda: kh.copy_(kd_one, non_blocking=True))
    res["one_memcpy_d2h_half_bytes"] = {"ms": ms, "GB/s": moved / 2 / (ms / 1e3) / 1e9}
    ms = timed(lambda: kd_one.copy_(kh, non_blocking=True))
    res["one_memcpy_h2d_half_bytes"] = {"ms": ms, "GB/s": moved / 2 / (ms / 1e3) / 1e9}
    ms = timed(cow_kernel)
    hbm_peak, _, peak_src = measured_peaks()
    res["copy_on_write_device"] = {"ms": ms, "GB/s": 2 * moved / (ms / 1e3) / 1e9,
                                   "hbm_frac": 2 * moved / (ms / 1e3) / 1e9 / hbm_peak,
                                   "bytes": "read + write of every copied block"}
    flags = pa.pa_read_error_flags(clear=True)
    # the swapped-out blocks really are the device blocks, bit for bit
    out_kernel()
    torch.cuda.synchronize()
    ok = bool(torch.equal(kh.view(torch.int16), kd[dev_ids.long()].cpu().view(torch.int16)))
    res.update({"blocks": n, "runs": runs, "blocks_per_run": run_blocks, "bytes_per_direction": moved,
                "block_bytes": block_bytes, "bit_exact_roundtrip": ok, "device_error_flags": flags,
                "peak_source": peak_src,
                "pool": "Llama-shaped fp16 pool [P, 8, 16, 128] for K and for V; host pool pinned"})
    del kd, vd, kh, vh
    torch.cuda.empty_cache()
    return res


EXTRA_WORKLOADS = ("long_context", "chat_trace", "prefill_chunk")
SWEEP_BLOCK_SIZES = (8, 16, 32, 64, 128)


def run_ours(args):
    import torch

    world, rank, local = dist_init(args)
    if args.workload == "block_swap":  # the block copies alone (swap out / in, copy-on-write)
        r = measure_block_swap(args.steps, args.warmup, rank, world)
        if rank == 0:
            print(json.dumps({"workload": "block_swap", **r}))
        return
    sampler = ClockSampler(local)
    sampler.start()
    K, W = args.steps, args.warmup
    main = measure(args.workload, args.block_size, args.partition, K, W, rank, world, sampler,
                   do_e2e=not args.no_e2e, sustain_s=args.sustain_seconds,
                   cpu_budget_s=0.0 if args.no_cpu_baseline else args.cpu_seconds)
    extras = {}
    sweep = []
    if args.all_workloads and args.workload == "llama_decode":
        for name in EXTRA_WORKLOADS:
            extras[name] = measure(name, 16, "auto", K, W, rank, world, sampler, do_e2e=not args.no_e2e,
                                   sustain_s=args.sustain_seconds, long_timed=True)
        swap = measure_block_swap(K, W, rank, world)
        for B in SWEEP_BLOCK_SIZES:  # the pages' block-size question, on the chat trace (cascade)
            r = measure("chat_trace", B, "auto", K, W, rank, world, sampler, do_e2e=False, sustain_s=0.0)
            sweep.append({"block_size": B, "value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
                          "kernel_ms": r["roofline"]["kernel_ms"], "roofline_frac": r["roofline"]["frac"],
                          "device_error_flags": r["device_error_flags"], "_windows": r["_windows"]})

    def clocks_of(r):
        win = r.pop("_windows")
        r["clocks"] = sampler.summary(*win["timed"])
        if "sustained" in win and "sustained" in r:
            r["sustained"]["clocks"] = sampler.summary(*win["sustained"])
        return r

    clocks_of(main)
    for r in extras.values():
        clocks_of(r)
    for r in sweep:
        clocks_of(r)
    sampler.close()

    if rank == 0:
        line = {
            "metric": METRIC, "value": main["value"], "unit": main["unit"], "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": main["dtype"], "data": "synthetic", "config": main["config"],
            "step_plan": main["step_plan"],
            "roofline": main["roofline"], "cpu_baseline": main.get("cpu_baseline"), "e2e": main["e2e"],
            "gpu_launches": main["gpu_launches"],
            "clocks": main["clocks"], "sustained": main["sustained"],
            "device_error_flags": main["device_error_flags"],
        }
        for k in ("seq_steps_per_s", "pct_of_peak"):
            if k in main:
                line[k] = main[k]
        if extras:
            # every timed region of the line together (each entry also carries its own count)
            line["gpu_launches_all_timed_regions"] = main["gpu_launches"] + sum(
                r["gpu_launches"] for r in extras.values())
            line["workloads"] = {}
            for name, r in extras.items():
                r.pop("warmup", None)
                line["workloads"][name] = r
            line["workloads"]["chat_trace"]["block_size_sweep"] = sweep
            line["workloads"]["block_swap"] = swap
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
