"""Per-CTA timeline of one decode step (needs a build made with `build.py --trace`).

python -m paged_kv_cache_475_b200.trace --workload llama_decode|chat_trace|long_context|prefill_chunk [--out t.npz]

Runs a few warm-up steps of the workload (the same step bench.py times), then
one step with the timeline records cleared before it. For the decode
workloads it prints where the decode kernel's time goes: how long a CTA waits
from entry until its first tile has landed, how many CTAs each SM runs over
time, and how the kernel ends (the tail, when SMs run out of CTAs). For the
prefill chunk it prints the per-role timeline of one heavy CTA of the
tensor-core kernel: per 128-key tile, when each producer, the MMA thread and
two softmax warps reached each step, and the mean time between the steps.
The records are written to --out as a numpy archive for further study.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def summarize(rec, num_sms=148, bins=20):
    rec = rec[rec["t_start"] > 0]
    t0 = rec["t_start"].min()
    start = (rec["t_start"] - t0) / 1e3
    first = np.where(rec["t_first"] > 0, (rec["t_first"] - t0) / 1e3, np.nan)
    end = (rec["t_end"] - t0) / 1e3
    span = end.max()
    out = {"ctas": int(len(rec)), "span_us": float(span),
           "first_tile_after_entry_us": {q: float(np.nanpercentile(first - start, p))
                                         for q, p in (("p10", 10), ("median", 50), ("p90", 90))},
           "cta_life_us": {q: float(np.percentile(end - start, p)) for q, p in (("p10", 10), ("median", 50),
                                                                                 ("p90", 90), ("max", 100))},
           "last_cta_start_us": float(start.max())}
    # CTAs resident per SM over time, and the share of CTA-time spent before the first tile
    edges = np.linspace(0, span, bins + 1)
    occ = []
    for a, b in zip(edges[:-1], edges[1:]):
        live = (start < b) & (end > a)
        per_sm = np.bincount(rec["smid"][live], minlength=num_sms)
        occ.append(round(float(per_sm.mean()), 2))
    out["mean_ctas_per_sm_by_time_slice"] = occ
    life = (end - start).sum()
    out["share_of_cta_time_before_first_tile"] = float(np.nansum(first - start) / life)
    ends = np.sort(end)
    out["time_when_90pct_of_ctas_done_us"] = float(ends[int(0.9 * (len(ends) - 1))])
    return out


PREFILL_EVENTS = ["k_slot_free", "k_issued", "v_slot_free", "v_issued", "mma_k_full", "mma_s_issued",
                  "mma_v_full", "mma_p0_ready", "mma_p1_ready", "mma_pv_issued", "sm0_s_full", "sm0_p_stored",
                  "sm4_s_full", "sm4_p_stored", "k_rows_done", "k_expect_done", "k_atom0_issued"]


def summarize_prefill(rec):
    """Per-tile event times (us from the first event) of the traced prefill CTA, and mean step gaps."""
    ev = rec[rec["kind"] >= 100]
    if len(ev) == 0:
        return {"error": "no prefill records"}
    t0 = ev["t_start"].min()
    n = int(ev["seq"].max()) + 1
    tab = np.full((len(PREFILL_EVENTS), n), np.nan)
    for r in ev:
        tab[int(r["kind"]) - 100, int(r["seq"])] = (int(r["t_start"]) - t0) / 1e3
    E = {name: tab[i] for i, name in enumerate(PREFILL_EVENTS)}
    mid = slice(2, max(3, n - 2))  # steady state: drop the first and last tiles

    def gap(a, b, shift=0):  # mean of E[b][j + shift] - E[a][j]
        x = E[a][mid]
        idx = np.arange(n)[mid] + shift
        ok = idx < n
        y = np.full(x.shape, np.nan)
        y[ok] = E[b][idx[ok]]
        d = y - x
        # events this build does not record are NaN throughout: report NaN without a warning
        return float(np.nanmean(d)) if np.isfinite(d).any() else float("nan")

    period = np.diff(E["mma_s_issued"])
    return {
        "tiles": n, "period_us_median": float(np.nanmedian(period[mid])),
        "k_slot_free_to_issued": gap("k_slot_free", "k_issued"),
        "k_issued_to_mma_k_full": gap("k_issued", "mma_k_full"),
        "mma_k_full_to_s_issued": gap("mma_k_full", "mma_s_issued"),
        "mma_s_issued_to_sm0_s_full": gap("mma_s_issued", "sm0_s_full"),
        "sm0_s_full_to_p_stored": gap("sm0_s_full", "sm0_p_stored"),
        "sm4_s_full_to_p_stored": gap("sm4_s_full", "sm4_p_stored"),
        "sm0_p_stored_to_mma_p0_ready": gap("sm0_p_stored", "mma_p0_ready"),
        "mma_p1_ready_to_pv_issued": gap("mma_p1_ready", "mma_pv_issued"),
        "mma_s_issued_j_to_k_slot_free_j+2": gap("mma_s_issued", "k_slot_free", 2),
        "mma_pv_issued_j_to_mma_k_full_j+2": gap("mma_pv_issued", "mma_k_full", 2),
        "sm0_p_stored_j_to_sm0_s_full_j+1": gap("sm0_p_stored", "sm0_s_full", 1),
        "v_issued_to_mma_v_full": gap("v_issued", "mma_v_full"),
        "k_slot_free_to_rows_done": gap("k_slot_free", "k_rows_done"),
        "k_rows_done_to_expect_done": gap("k_rows_done", "k_expect_done"),
        "k_expect_done_to_atom0_issued": gap("k_expect_done", "k_atom0_issued"),
        "k_atom0_issued_to_issued": gap("k_atom0_issued", "k_issued"),
        "table_us": {k: [None if np.isnan(x) else round(float(x), 3) for x in v] for k, v in E.items()},
    }


def main():
    import json

    import torch

    import paged_kv_cache_475_b200 as pa
    import workloads as W
    from paged_kv_cache_475_b200.step import DecodeStep

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama_decode",
                    choices=["llama_decode", "chat_trace", "long_context", "prefill_chunk"])
    ap.add_argument("--partition", default="auto")
    ap.add_argument("--out", default=None)
    a = ap.parse_args()
    if a.workload == "prefill_chunk":
        from paged_kv_cache_475_b200.step import PrefillStep

        b = W.prefill_chunk(poison=None).to("cuda")
        step = PrefillStep(b.num_seqs, b.chunk, b.num_q_heads, b.head_dim, b.q.dtype,
                           num_new_tokens=b.new_seq.shape[0])
        args = (b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.new_seq, b.new_pos,
                b.scale)
        for _ in range(5):
            step(*args)
        torch.cuda.synchronize()
        pa.trace_clear()
        step(*args)
        rec = pa.trace_read()
        s = summarize_prefill(rec)
        s["workload"] = a.workload
        print(json.dumps(s))
        if a.out:
            np.savez(a.out, records=rec[rec["kind"] >= 100])
        return
    b = {"llama_decode": W.llama_decode, "chat_trace": W.chat_trace, "long_context": W.long_context}[a.workload](
        poison=None).to("cuda")
    sp = (b.info["shared_prefix_tokens"], b.info["shared_group"]) if a.workload == "chat_trace" else None
    part = "auto" if a.partition == "auto" else (None if a.partition == "none" else int(a.partition))
    step = DecodeStep(b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim, int(b.context_lens.max()), b.q.dtype,
                      num_new_tokens=b.new_seq.shape[0], partition=part, shared_prefix=sp)
    args = (b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.new_seq, b.new_pos,
            b.scale)
    for _ in range(5):
        step(*args)
    torch.cuda.synchronize()
    pa.trace_clear()
    step(*args)
    rec = pa.trace_read()
    s = summarize(rec)
    s["workload"] = a.workload
    print(json.dumps(s))
    if a.out:
        np.savez(a.out, records=rec[rec["t_start"] > 0])


if __name__ == "__main__":
    main()
