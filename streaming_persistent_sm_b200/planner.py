"""Composition planner: rank ways of cutting a program into launches.

"One Megakernel is Not Enough" (abstract; plain-language summary; Table I)
selects which contiguous regions of a model to fuse into persistent launches
and which to run conventionally, from existing measurements and a simulation
of tile and event graphs, without timing every candidate end to end.  This
module does the same for one program of this library (a decode step, or a
prefill):

  * measurements: one traced run of the monolith (per-tile busy times and the
    hop from a tile's last producer to its start) and the device's weight-load
    bandwidth per worker; one calibration point fixes the per-launch cost;
  * candidates: one persistent launch, 2-4 persistent regions cut at layer
    boundaries, or one conventional launch per op;
  * simulation: ``wpk_predict`` (native) list-schedules the compiled tile graph
    under each candidate (Table I's rows: tile-to-tile readiness, one or more
    staging slots per worker, a dispatch node per launch, synchronisation added
    to tile waits, waves of CTAs for conventional launches);
  * the candidates are ranked by predicted time.

Only argument marshalling and bookkeeping happen here; the simulation is in the
C library.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence

import numpy as np

from . import wpk as W


@dataclass
class Calibration:
    """Service costs of one program, from one traced monolith run."""

    service_ns: np.ndarray          # per tile: busy time once started
    load_ns: np.ndarray             # per tile: weight bytes / per-worker bandwidth
    sync_ns: float                  # median hop: last producer's end -> consumer's start
    first_chunk_ns: float = 1000.0  # issue -> first staged bytes landed
    dispatch_ns: float = 4000.0     # one launch (fixed by `fit_dispatch`)


@dataclass
class Candidate:
    name: str
    mode: int
    n_regions: int = 1
    region_cut: Sequence[int] = (0, 0, 0, 0)

    def as_kwargs(self) -> dict:
        cut = list(self.region_cut) + [0] * (4 - len(self.region_cut))
        return dict(mode=self.mode, n_regions=self.n_regions, region_cut=tuple(cut[:4]))


def calibrate(trace: np.ndarray, tile_bytes: np.ndarray, edges: np.ndarray, bytes_per_ns_per_worker: float,
              first_chunk_ns: float = 1000.0) -> Calibration:
    """Per-tile costs from a trace of the monolith (records in any order).

    service = end - start of each tile; load = its staged weight bytes over one
    worker's share of the load bandwidth; sync = the median, over tiles that
    waited for a predecessor (its last predecessor ended after the worker's
    previous tile did, so the worker was idle), of start - (latest predecessor
    end).  A tile that waited for its own worker measures the queue, not the
    hop, and is left out."""
    tr = np.sort(trace, order="tile")
    n = len(tr)
    start = tr["t_start_ns"].astype(np.float64)
    end = tr["t_end_ns"].astype(np.float64)
    service = np.maximum(end - start, 0.0)
    load = tile_bytes.astype(np.float64) / float(bytes_per_ns_per_worker)
    last_pred = np.full(n, -np.inf)
    if len(edges):
        np.maximum.at(last_pred, edges[:, 1], end[edges[:, 0]])
    # end of the previous tile on the same worker (tiles of a worker in start order)
    prev_end = np.full(n, -np.inf)
    worker = tr["worker"].astype(np.int64)
    order = np.lexsort((start, worker))
    same = worker[order][1:] == worker[order][:-1]
    prev_end[order[1:][same]] = end[order[:-1][same]]
    waited = np.isfinite(last_pred) & (last_pred >= prev_end)
    hops = start[waited] - last_pred[waited]
    hops = hops[hops >= 0]
    sync = float(np.median(hops)) if len(hops) else 0.0
    return Calibration(service, load, sync, first_chunk_ns)


def predict(h, cal: Calibration, cand: Candidate, n_workers: int, n_sms: int, schedule: int, slots: int) -> float:
    """Predicted ns of one run of the selected program under `cand`."""
    return W.wpk_predict(h, cal.service_ns, cal.load_ns, n_workers=n_workers, n_sms=n_sms, schedule=schedule,
                         slots=slots, dispatch_ns=cal.dispatch_ns, sync_ns=cal.sync_ns,
                         first_chunk_ns=cal.first_chunk_ns, **cand.as_kwargs())


def fit_dispatch(h, cal: Calibration, cand: Candidate, measured_ns: float, n_workers: int, n_sms: int,
                 schedule: int, slots: int, hi_ns: float = 50_000.0) -> float:
    """The per-launch cost at which `cand` is predicted at `measured_ns`
    (bisection; the prediction grows with the dispatch cost)."""
    lo, hi = 0.0, hi_ns
    for _ in range(50):
        mid = 0.5 * (lo + hi)
        cal.dispatch_ns = mid
        if predict(h, cal, cand, n_workers, n_sms, schedule, slots) < measured_ns:
            lo = mid
        else:
            hi = mid
    cal.dispatch_ns = 0.5 * (lo + hi)
    return cal.dispatch_ns


def default_candidates(n_layers: int) -> List[Candidate]:
    """One persistent launch, two to four regions cut at even layer
    boundaries, and one conventional launch per op."""
    out = [Candidate("1 MK", W.WPK_MEGAKERNEL)]
    for r in (2, 3, 4):
        cuts = [round(i * n_layers / r) for i in range(r)]
        out.append(Candidate(f"{r} MK (cuts {','.join(map(str, cuts))})", W.WPK_MEGAKERNEL, r, cuts))
    out.append(Candidate("per-op graph", W.WPK_PER_OP_GRAPH))
    return out


def rank(h, cal: Calibration, candidates: Sequence[Candidate], n_workers: int, n_sms: int, schedule: int,
         slots: int) -> List[Dict]:
    """Candidates with their predicted time, fastest first."""
    rows = [{"name": c.name, "candidate": c, "predicted_us": predict(h, cal, c, n_workers, n_sms, schedule, slots) / 1e3}
            for c in candidates]
    return sorted(rows, key=lambda r: r["predicted_us"])


# ---------------------------------------------------------------- the harness
def _time_program(eng, prompts, prefill: bool, steps: int, reps: int) -> float:
    """Median device time (ns) of one run of the program: a prefill, or one
    decode step (after a prefill, outside the timed region)."""
    import torch

    dev_prompts = torch.as_tensor(prompts, device="cuda")
    B, T = prompts.shape
    out = torch.empty(max(steps, 1) + 1, B, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    times = []
    for r in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if prefill:
            a.record(stream)
            W.wpk_prefill(eng.h, dev_prompts.data_ptr(), B, T, out[0].data_ptr(), 0, stream.cuda_stream)
            b.record(stream)
        else:
            W.wpk_prefill(eng.h, dev_prompts.data_ptr(), B, T, out[0].data_ptr(), 0, stream.cuda_stream)
            a.record(stream)
            for i in range(steps):
                W.wpk_step(eng.h, 0, out[i + 1].data_ptr(), 0, stream.cuda_stream)
            b.record(stream)
        torch.cuda.synchronize()
        if r:  # the first run warms up
            times.append(a.elapsed_time(b) * 1e6 / (1 if prefill else steps))
    return float(np.median(times))


def main(argv=None) -> int:
    """Trace the monolith of a workload's program, time its conventional
    (per-op) composition, predict every candidate and rank them; with
    --measure, also time every candidate and compare the two rankings."""
    import argparse
    import json
    import os
    import sys

    import torch

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama1b_prefill_b16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--measure", action="store_true", help="also time every candidate end to end")
    ap.add_argument("--steps", type=int, default=8, help="decode steps per timed run (decode workloads)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--json", default="")
    a = ap.parse_args(argv)
    wl = synth.WORKLOADS[a.workload]
    s = wl.model
    prefill = wl.steps == 0
    B, T = wl.batch, wl.prompt_len
    ctx = T + max(a.steps, 1) + 1
    weights = synth.cached_weights(s, seed=0)
    prompts = synth.make_prompts(s.vocab, B, T, wl.prompt_seed)
    sched = W.WPK_SCHED_STATIC
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peaks = os.path.join(root, "MEASURED_PEAKS.json")
    hbm_gbs = json.load(open(peaks))["hbm_gbs"] if os.path.exists(peaks) else 6650.0

    def engine(**kw):
        return W.Engine(s, weights, B, ctx, schedule=sched, **kw)

    # 1. the monolith, traced: per-tile service times
    eng = engine(trace=1)
    try:
        _time_program(eng, prompts, prefill, a.steps, 1)
        if prefill:
            W.wpk_select_program(eng.h, B, T)
        n = W.wpk_graph_stats_get(eng.h)["n_tiles"]
        tr = W.wpk_get_trace(eng.h, n)
        cal = calibrate(tr, W.wpk_get_tile_bytes(eng.h, n), W.wpk_get_edges(eng.h),
                        bytes_per_ns_per_worker=hbm_gbs / sms)
        n_workers = eng.stats["n_workers"]
    finally:
        eng.close()
    # 2. the conventional profile: the per-op composition, timed; it fixes the
    #    per-launch cost
    eng = engine(mode=W.WPK_PER_OP_GRAPH)
    try:
        per_op_ns = _time_program(eng, prompts, prefill, a.steps, a.reps)
        if prefill:
            W.wpk_select_program(eng.h, B, T)
        cands = default_candidates(s.n_layers)
        per_op = [c for c in cands if c.mode == W.WPK_PER_OP_GRAPH][0]
        fit_dispatch(eng.h, cal, per_op, per_op_ns, n_workers, sms, sched, 4)
        rows = rank(eng.h, cal, cands, n_workers, sms, sched, 4)
    finally:
        eng.close()
    # 3. optional validation: every candidate end to end
    if a.measure:
        for r in rows:
            c = r["candidate"]
            if c.mode == W.WPK_PER_OP_GRAPH:
                r["measured_us"] = per_op_ns / 1e3
                continue
            kw = dict(n_regions=c.n_regions, region_cut=tuple(c.region_cut)) if c.n_regions > 1 else {}
            e2 = engine(**kw)
            try:
                r["measured_us"] = _time_program(e2, prompts, prefill, a.steps, a.reps) / 1e3
            finally:
                e2.close()
        order = sorted(rows, key=lambda r: r["measured_us"])
        for i, r in enumerate(order):
            r["measured_rank"] = i + 1
    out = {"workload": wl.name, "program": "prefill" if prefill else "decode step", "sync_ns": cal.sync_ns,
           "dispatch_ns": cal.dispatch_ns, "per_op_measured_us": per_op_ns / 1e3,
           "candidates": [{k: v for k, v in r.items() if k != "candidate"} | {"predicted_rank": i + 1}
                          for i, r in enumerate(rows)]}
    if a.measure:
        out["winner_matches"] = rows[0]["name"] == min(rows, key=lambda r: r["measured_us"])["name"]
    print(json.dumps(out))
    if a.json:
        with open(a.json, "w") as f:
            json.dump(out, f, indent=1)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
