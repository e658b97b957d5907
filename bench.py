#!/usr/bin/env python
"""Benchmark of the persistent decode program on B200.

Default workload (N=1): the Llama-3.2-1B-shaped decoder (seeded random bf16
weights) at batch 1 - prefill of a 496-token uniform-random prompt to the first
token, then 128 greedy decode steps.  One bench step is that whole job; the
value is generated tokens per second over it (first token + 128 decode tokens
per sequence).  Decode-only workloads (batch 16/32/48, already prefilled) time
the 128 decode steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--mode megakernel|per_op_graph] [--impl ours|reference]

Multi-GPU: the sessions shard across GPUs with no exchange (replicas), one
process per GPU under torchrun; the value is the sum over ranks divided by the
slowest rank's time.  `--impl reference` times the float64 CPU oracle on the
host cores on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode step µs and tokens/s at batch 1–48; achieved HBM GB/s vs 8 TB/s peak"
KV_BYTES_PER_TOKEN = lambda s: 2 * s.n_layers * s.n_kv_heads * s.head_dim * 2  # K and V, bf16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama1b_b1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--mode", default="megakernel", choices=["megakernel", "per_op_graph"])
    ap.add_argument("--regions", default="", help="comma-separated region cuts, e.g. 0,8")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=None)
    ap.add_argument("--prompt-len", type=int, default=None, help="override the prompt length (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tile-bytes", type=int, default=0)
    ap.add_argument("--slot-bytes", type=int, default=0)
    ap.add_argument("--workers-per-sm", type=int, default=0)
    ap.add_argument("--lookahead", type=int, default=0)
    ap.add_argument("--schedule", default="static", choices=["queue", "static", "teams"])
    ap.add_argument("--prefill", default="auto", choices=["auto", "mma", "tokenwise"])
    ap.add_argument("--decode", default="auto", choices=["auto", "gemv", "mma"],
                    help="decode program: CUDA-core GEMV tiles or tensor-core tiles (auto: by batch)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--resident", action="store_true", help="one resident grid serves every decode step")
    ap.add_argument("--split-pages", type=int, default=0)
    ap.add_argument("--page-tokens", type=int, default=0, help="KV page size in tokens (0 = the plan's default)")
    ap.add_argument("--frame-chunks", type=int, default=0,
                    help="two-stage: split the batch into chunks whose backbone and head launches overlap")
    ap.add_argument("--head-workers", type=int, default=0, help="two-stage with --frame-chunks: the heads' workers")
    ap.add_argument("--capacity", action="store_true",
                    help="also measure the real-time capacity: the largest fixed cohort whose q-quantile step "
                         "time fits --period-ms")
    ap.add_argument("--period-ms", type=float, default=80.0, help="update period P of the capacity metric")
    ap.add_argument("--quantile", type=float, default=0.99, help="quantile q of the capacity metric")
    return ap.parse_args()


def profiled_traffic(kernel, B, mean_ctx):
    """DRAM bytes per launch of a decode program from the committed ncu summary
    of that kernel, scaled by the KV bytes to this run's batch and context - or
    None when no summary covers the kernel or its sources changed since the
    capture."""
    import glob
    import hashlib
    import re

    src = os.path.join(ROOT, "streaming_persistent_sm_b200", "csrc")
    sha = hashlib.sha1(b"".join(open(os.path.join(src, f), "rb").read()
                                for f in ("runtime.cu", "ptx.cuh", "wpk_internal.h"))).hexdigest()
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        m = {k: v for k, v in re.findall(r"^(\w+)(?:\([^)]*\))?: (\S+)$", open(p).read(), re.M)}
        if m.get("traffic_kernel") != kernel or m.get("source_sha1") != sha:
            continue
        kv = float(m["kv_bytes_per_token"])
        base = float(m["traffic_bytes_per_launch"]) - float(m["traffic_batch"]) * float(m["traffic_context"]) * kv
        return base + B * mean_ctx * kv
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1645.6)), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        load = [s for s, r in zip(sm, rows) if float(r[3]) > 250.0] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------- CPU reference --
def oracle_sample(wl, weights, n_steps: int = 2):
    """Time the float64 oracle on host cores: the workload's prefill and a few
    steps for one sequence; tokens/s extrapolated to the whole job."""
    return oracle_job_sample(wl, weights, n_steps)


def codes_per_step(model):
    """Tokens one sequence emits per step: one, or a frame of codebook codes."""
    return model.n_codebooks if hasattr(model, "backbone") else 1


def job_tokens(wl, decode_steps):
    """Tokens one bench step generates, and whether the prefill is part of it
    (decode-only workloads start from an already-prefilled prompt)."""
    with_prefill = not wl.name.startswith("llama1b_decode")
    return wl.batch * codes_per_step(wl.model) * ((1 if with_prefill else 0) + decode_steps), with_prefill


def oracle_job_sample(wl, weights, n_steps: int):
    """One sequence through the float64 oracle: (prefill seconds, median step
    seconds) - a decode step, or a two-stage frame."""
    import oracle

    s = wl.model
    if hasattr(s, "backbone"):
        ts = oracle.TwoStage(s, weights)
        prompts = synth.make_prompts(s.backbone.vocab, 1, wl.prompt_len, wl.prompt_seed)
        cache = ts.backbone.new_cache(1, wl.prompt_len + n_steps + 1)
        t0 = time.perf_counter()
        codes, _ = ts.prefill(cache, prompts)
        t_prefill = time.perf_counter() - t0
        times = []
        for _ in range(n_steps):
            t0 = time.perf_counter()
            codes, _ = ts.frame(cache, codes)
            times.append(time.perf_counter() - t0)
        return t_prefill, statistics.median(times)
    dec = oracle.Decoder(s, weights)
    prompts = synth.make_prompts(s.vocab, 1, wl.prompt_len, wl.prompt_seed)
    cache = dec.new_cache(1, wl.prompt_len + n_steps + 1)
    t0 = time.perf_counter()
    tok = oracle.argmax_lowest(dec.prefill(cache, prompts))
    t_prefill = time.perf_counter() - t0
    times = []
    for _ in range(n_steps):
        t0 = time.perf_counter()
        tok = oracle.argmax_lowest(dec.step(cache, tok))
        times.append(time.perf_counter() - t0)
    return t_prefill, statistics.median(times)


def model_weight_bytes(model):
    """bf16 bytes of every tensor of the model (the tied LM head once)."""
    return 2 * sum(int(np.prod(shp)) for _, shp, _ in synth.tensor_specs(model))


def workload_config(wl, prompt_len, decode_steps, layers=0):
    """The workload a bench line measures - the same keys for both arms."""
    _, with_prefill = job_tokens(wl, decode_steps)
    wb = model_weight_bytes(wl.model)
    l2 = ("inputs larger than L2 (126 MB): %.2f GB of weights streamed from HBM per step" % (wb / 1e9)
          if wb > 126e6 else "weights fit in L2 (%.1f MB): latency-bound, no HBM claim" % (wb / 1e6))
    return {"workload": wl.name + (f" ({layers} layers)" if layers else ""), "batch": wl.batch,
            "prompt_len": prompt_len, "decode_steps": decode_steps,
            "timed": "prefill + decode steps" if with_prefill else "decode steps (prompt prefilled untimed)",
            "l2": l2}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[args.workload]
    decode_steps = wl.steps if args.decode_steps is None else args.decode_steps
    weights = synth.cached_weights(wl.model, seed=0)
    cores = os.cpu_count()
    # one prefill, then warm-up + timed steps (decode steps or frames)
    t_prefill, t_step = oracle_job_sample(wl, weights, args.warmup + args.steps)
    tokens, with_prefill = job_tokens(wl, decode_steps)
    per_seq = (t_prefill if with_prefill else 0.0) + decode_steps * t_step
    job_s = per_seq * wl.batch  # the oracle runs the sequences one after another
    value = tokens / job_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": job_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, wl.prompt_len, decode_steps),
        "decode_step_us": {"median": t_step * 1e6},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"float64 NumPy oracle, one sequence: prefill of {wl.prompt_len} tokens "
                                   f"({t_prefill:.2f} s) and {args.steps} timed decode steps (median "
                                   f"{t_step * 1e3:.0f} ms); one bench step = the whole job (prefill and "
                                   f"{decode_steps} steps for each of the {wl.batch} sequences), extrapolated"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- ours --
def prefill_flops(s, batch, prompt_len):
    """Algorithmic FLOPs of prefilling `batch` prompts of `prompt_len` tokens:
    every projection once per token, causal attention (QK^T and PV over the
    tokens at or before each query), the LM head at the last position."""
    q, kv = s.n_heads * s.head_dim, s.n_kv_heads * s.head_dim
    per_token = s.n_layers * (s.hidden * (q + 2 * kv) + q * s.hidden + 3 * s.ffn * s.hidden)
    attn = s.n_layers * 4 * s.n_heads * s.head_dim * prompt_len * (prompt_len + 1) // 2
    return 2 * per_token * batch * prompt_len + batch * attn + 2 * s.vocab * s.hidden * batch


def algorithmic_bytes_per_step(shape, weight_bytes, batch, ctx_len):
    """Weights once + KV read over ctx_len tokens + KV written for 1 token, per sequence."""
    kv = KV_BYTES_PER_TOKEN(shape)
    return weight_bytes + batch * (ctx_len * kv + kv)


def deadline_capacity(step_ms_by_n, period_ms, q):
    """Real-time capacity ("Why real-time inference wants a megakernel", "Real
    time changes the objective"): the largest number of live sessions N whose
    q-quantile update latency is within the period P - updates must keep
    finishing on time, so a mean or a throughput does not decide it.  Returns
    (N or 0 if none fits, {N: q-quantile ms})."""
    qs = {int(n): float(np.quantile(np.asarray(t, dtype=np.float64), q)) for n, t in step_ms_by_n.items() if len(t)}
    ok = [n for n, v in qs.items() if v <= period_ms]
    return (max(ok) if ok else 0), dict(sorted(qs.items()))


def measure_capacity(W, s, weights, prompt_len, sizes, steps, period_ms, q, seed):
    """Per-step device times of fixed cohorts of each size in `sizes` (a plan
    compiled for N sessions, all live, prompts prefilled untimed), and the
    deadline capacity they give."""
    import torch

    times = {}
    for n in sizes:
        eng = W.Engine(s, weights, n, prompt_len + steps + 1)
        try:
            prompts = synth.make_prompts(s.vocab, n, prompt_len, seed)
            eng.prefill_slots(0, prompts)
            out = torch.empty((steps, n), dtype=torch.int32, device="cuda")
            stream = torch.cuda.current_stream()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for i in range(steps):
                ev[i][0].record(stream)
                W.wpk_step(eng.h, 0, out[i].data_ptr(), 0, stream.cuda_stream)
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            times[n] = [a.elapsed_time(b) for a, b in ev[1:]]  # the first step warms up
        finally:
            eng.close()
    cap, by_n = deadline_capacity(times, period_ms, q)
    return {"period_ms": period_ms, "quantile": q, "capacity_sessions": cap, "step_ms_at_quantile": by_n,
            "sizes": list(sizes), "steps": steps - 1,
            "note": "largest cohort whose q-quantile step time fits the period; plans are capped at "
                    "128 sessions (the tensor-core decode's largest N)"}


def slowest_rank_ms(total_ms, world, device):
    """The job's time: the slowest rank's, agreed by every rank (each rank
    calls this once, after its timed region), then a barrier."""
    if world == 1:
        return total_ms
    import torch
    import torch.distributed as dist

    t = torch.tensor([total_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.barrier()
    return float(t.item())


def job_value(world, tokens_per_step, ms_per_step):
    """Whole-job throughput: the tokens of all ranks (each runs the same
    workload on its own sessions) over the slowest rank's time."""
    return world * tokens_per_step / (ms_per_step / 1e3)


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist

    from streaming_persistent_sm_b200 import wpk as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    wl = synth.WORKLOADS[args.workload]
    s = wl.model
    if args.layers:
        import dataclasses

        s = dataclasses.replace(s, n_layers=args.layers)
    B, T = wl.batch, (wl.prompt_len if args.prompt_len is None else args.prompt_len)
    decode_steps = wl.steps if args.decode_steps is None else args.decode_steps
    tokens_per_step, with_prefill = job_tokens(wl, decode_steps)
    two = hasattr(s, "backbone")
    K = codes_per_step(s)
    ctx = T + max(decode_steps, 1)
    weights = synth.cached_weights(s, seed=0)
    mode = W.WPK_MEGAKERNEL if args.mode == "megakernel" else W.WPK_PER_OP_GRAPH
    plan = dict(mode=mode, tile_bytes=args.tile_bytes, slot_bytes=args.slot_bytes,
                workers_per_sm=args.workers_per_sm, lookahead=args.lookahead,
                schedule={"static": W.WPK_SCHED_STATIC, "queue": W.WPK_SCHED_QUEUE,
                          "teams": W.WPK_SCHED_TEAMS}[args.schedule],
                prefill={"auto": W.WPK_PREFILL_AUTO, "mma": W.WPK_PREFILL_MMA,
                         "tokenwise": W.WPK_PREFILL_TOKENWISE}[args.prefill],
                decode={"auto": W.WPK_DECODE_AUTO, "gemv": W.WPK_DECODE_GEMV, "mma": W.WPK_DECODE_MMA}[args.decode],
                resident=1 if args.resident else 0,
                split_pages=args.split_pages, page_tokens=args.page_tokens, frame_chunks=args.frame_chunks,
                head_workers=args.head_workers)
    if args.regions:
        cuts = [int(x) for x in args.regions.split(",")]
        plan.update(n_regions=len(cuts), region_cut=tuple(cuts))
    eng = W.Engine(s, weights, B, ctx, **plan)
    stats = eng.stats
    prompts = synth.make_prompts(s.backbone.vocab if two else s.vocab, B, T, wl.prompt_seed + 17 * rank)
    prompts_dev = torch.as_tensor(prompts, device=dev)
    out_dev = torch.empty((max(decode_steps, 1) + 1, B) + ((K,) if two else ()), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    launches_per_decode = stats["n_regions"] if mode == W.WPK_MEGAKERNEL else stats["n_ops"]
    # chunked two-stage frame: a backbone + head pair per chunk of ceil(B / C) sequences
    chunks = args.frame_chunks if two and args.frame_chunks > 1 else 1
    rows = -(-B // chunks)
    n_chunks = -(-B // rows)
    prefill_tensor_cores = True
    try:
        W.wpk_select_program(eng.h, rows, T)
        pst = W.wpk_graph_stats_get(eng.h)
        W.wpk_select_program(eng.h, 0, 0)
        launches_per_prefill = pst["n_regions"] if mode == W.WPK_MEGAKERNEL else pst["n_ops"]
    except W.WpkError:
        prefill_tensor_cores = False
        launches_per_prefill = T * launches_per_decode
    if two:  # the backbone, then the head's K steps of the frame
        launches_per_decode += K
        launches_per_prefill += K
    launches_per_decode *= n_chunks
    launches_per_prefill *= n_chunks

    def prefill():
        W.wpk_prefill(eng.h, prompts_dev.data_ptr(), B, T, out_dev[0].data_ptr(), 0, sp)

    def decode(ev=None):
        for i in range(decode_steps):
            if ev is not None:
                ev[i][0].record(stream)
            W.wpk_step(eng.h, 0, out_dev[i + 1].data_ptr(), 0, sp)
            if ev is not None:
                ev[i][1].record(stream)

    def job(ev=None, pev=None):
        if with_prefill:
            if pev is not None:
                pev[0].record(stream)
            prefill()
            if pev is not None:
                pev[1].record(stream)
        else:
            prefill()  # untimed part of decode-only workloads is excluded below
        decode(ev)

    # decode-only workloads: the prompt is prefilled outside the timed region
    mk = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        job()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms, dec_us, pre_ms = [], [], []
    with ClockSampler(local) as clk:
        if with_prefill:
            t0, t1 = mk(), mk()
            evs = [[[mk(), mk()] for _ in range(decode_steps)] for _ in range(args.steps)]
            pevs = [[mk(), mk()] for _ in range(args.steps)]
            torch.cuda.synchronize()
            t0.record(stream)
            for k in range(args.steps):
                job(evs[k], pevs[k])
            t1.record(stream)
            torch.cuda.synchronize()
            total_ms = t0.elapsed_time(t1)
            for k in range(args.steps):
                pre_ms.append(pevs[k][0].elapsed_time(pevs[k][1]))
                dec_us += [a.elapsed_time(b) * 1e3 for a, b in evs[k]]
        else:
            total_ms = 0.0
            for k in range(args.steps):
                prefill()
                evs = [[mk(), mk()] for _ in range(decode_steps)]
                t0, t1 = mk(), mk()
                t0.record(stream)
                decode(evs)
                t1.record(stream)
                torch.cuda.synchronize()
                total_ms += t0.elapsed_time(t1)
                dec_us += [a.elapsed_time(b) * 1e3 for a, b in evs]
    total_ms = slowest_rank_ms(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_value(world, tokens_per_step, ms_per_step)

    # roofline of the dominant kernel (the persistent decode program): bytes per
    # launch over the launch durations measured above
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    # the decode program's kernel: tensor-core decode tiles (op codes from 16 on) run in their own kernel
    mma_decode = bool((W.wpk_get_tile_ops(eng.h, stats["n_tiles"]) >= W.OP_NAMES.index("b_qkv")).any())
    kernel_name = ("wpk_persistent" if mode == W.WPK_MEGAKERNEL else "wpk_per_op") + ("_mma" if mma_decode else "") + "_kernel"
    decode_summary = None
    if decode_steps > 0:
        dec_ctx = [T + i for i in range(decode_steps)]  # tokens already cached at each decode step
        if two:  # a frame: backbone step + K head steps (head weights, output head k, head KV)
            hs = s.head
            head_w = 2 * hs.n_layers * (hs.hidden * (hs.n_heads + 2 * hs.n_kv_heads) * hs.head_dim
                                        + hs.n_heads * hs.head_dim * hs.hidden + 3 * hs.ffn * hs.hidden)
            head_bytes = sum(head_w + 2 * s.codebook_vocab * hs.hidden + B * (k + 1) * KV_BYTES_PER_TOKEN(hs)
                             for k in range(K))
            algo_dec = [algorithmic_bytes_per_step(s.backbone, stats["weight_bytes"], B, c) + head_bytes
                        for c in dec_ctx]
        else:
            algo_dec = [algorithmic_bytes_per_step(s, stats["weight_bytes"], B, c) for c in dec_ctx]
        # the dominant kernel is the decode program (one launch per step): its
        # algorithmic bytes per launch over the launch times measured above
        launch_bytes = sum(algo_dec)
        launch_ms = sum(dec_us) / 1e3 / args.steps
        achieved_gbs = launch_bytes / (launch_ms / 1e3) / 1e9
        dec_gbs = statistics.mean(algo_dec) / (statistics.median(dec_us) / 1e6) / 1e9
        decode_summary = {"median": statistics.median(dec_us), "p95": float(np.percentile(dec_us, 95)),
                          "achieved_gbs": dec_gbs, "frac_of_8tbs": dec_gbs / 8000.0}
        # DRAM traffic per launch from the committed capture (plain decoder, one
        # launch per step; None for other programs or after a kernel change)
        traffic = (profiled_traffic(kernel_name, B, statistics.mean(dec_ctx)) if not two
                   and mode == W.WPK_MEGAKERNEL and stats["n_regions"] == 1 and not args.layers else None)
        roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                    "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)", "kernel": kernel_name}
    else:
        # prefill only: the prefill program dominates and is a dense contraction;
        # algorithmic FLOPs (one bf16 product per weight and token) over its time
        flops = prefill_flops(s, B, T)
        achieved_tf = flops / (statistics.median(pre_ms) / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": achieved_tf / tc_peak, "traffic": None,
                    "peak_source": f"{peak_kind} cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)",
                    "kernel": "wpk_prefill_kernel" if mode == W.WPK_MEGAKERNEL else "wpk_prefill_op_kernel",
                    "flops_per_launch": flops}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "accum_dtype": "fp32", "data": "synthetic",
        "config": workload_config(wl, T, decode_steps, args.layers),
        "plan": {"schedule": args.schedule,
                 "mode": args.mode + (" (resident grid)" if args.resident else ""),
                 "regions": stats["n_regions"], "tiles_per_step": stats["n_tiles"],
                 "prefill": "tensor-core prefill program" if prefill_tensor_cores else "token by token",
                 "workers": stats["n_workers"], "lookahead": args.lookahead or "library default (4)",
                 **({"codes_per_frame": K, "tokens": "codebook codes (a frame per sequence per step)"}
                    if two else {}),
                 **({"frame_chunks": n_chunks, "backbone_workers": stats["n_workers"],
                     "head_workers": args.head_workers or (torch.cuda.get_device_properties(dev).multi_processor_count
                                                           * max(1, args.workers_per_sm) - stats["n_workers"])}
                    if chunks > 1 else {})},
        "decode_step_us": decode_summary,
        "ttft_ms": statistics.median(pre_ms) if pre_ms else None,
        "roofline": roofline,
        "gpu_launches": args.steps * ((launches_per_prefill if with_prefill else 0) + launches_per_decode * decode_steps),
        "clocks": clk.summary(),
    }

    # end to end through the C ABI with host buffers: pinned prompt -> device,
    # prefill + decode, tokens -> pinned host, all inside the timed region
    host_prompt = torch.from_numpy(prompts).pin_memory()
    host_out = torch.empty(tuple(out_dev[: decode_steps + 1].shape), dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    e2e_runs = max(1, min(args.steps, 3))
    t0 = time.perf_counter()
    for _ in range(e2e_runs):
        prompts_dev.copy_(host_prompt, non_blocking=True)
        prefill()
        decode()
        host_out.copy_(out_dev[: decode_steps + 1], non_blocking=True)
        torch.cuda.synchronize()
    e2e_s = slowest_rank_ms((time.perf_counter() - t0) / e2e_runs * 1e3, world, dev) / 1e3
    line["e2e"] = {"value": job_value(world, tokens_per_step, e2e_s * 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(host_prompt.numel() * 4),
                   "d2h_bytes_per_step": int(host_out.numel() * 4)}

    if args.capacity and not two:
        line["capacity"] = measure_capacity(W, s, weights, T, (1, 8, 16, 32, 48, 64, 96, 128), 17,
                                            args.period_ms, args.quantile, wl.prompt_seed)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_pre, t_step = oracle_sample(wl, weights, n_steps=2)
        per_seq = (t_pre if with_prefill else 0.0) + decode_steps * t_step
        cpu_value = tokens_per_step / (per_seq * B)
        what = "frames" if two else "decode steps"
        line["cpu_baseline"] = {
            "value": cpu_value, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"float64 NumPy oracle, one sequence: {T}-token prefill ({t_pre:.1f} s) + 2 {what} "
                      f"(median {t_step:.2f} s); extrapolated to {decode_steps} {what} and {B} sequences"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    eng.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
