"""Shared helpers for GPU-vs-oracle parity tests (teacher-forced).

Tolerances (the decode step's contract): per step and batch row,
max |logit difference| <= 2e-2 and relative L2 <= 1e-2; the GPU's greedy token
must equal the oracle's argmax unless the oracle's top-2 logits are closer than
2e-2 (then either of the near-tied tokens is accepted).  The oracle consumes
the GPU's tokens, so a legitimate near-tie never cascades.
"""
from __future__ import annotations

import numpy as np

MAX_ABS = 2e-2
REL_L2 = 1e-2
TIE_GAP = 2e-2


def check_logits(gpu: np.ndarray, ref: np.ndarray, tokens: np.ndarray, where: str = "") -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{where}: non-finite GPU logits"
    worst = {"max_abs": 0.0, "rel_l2": 0.0, "ties": 0}
    for b in range(ref.shape[0]):
        d = gpu[b] - ref[b]
        max_abs = float(np.max(np.abs(d)))
        rel = float(np.linalg.norm(d) / np.linalg.norm(ref[b]))
        worst["max_abs"] = max(worst["max_abs"], max_abs)
        worst["rel_l2"] = max(worst["rel_l2"], rel)
        assert max_abs <= MAX_ABS, f"{where} row {b}: max|dlogit| {max_abs:.3g} > {MAX_ABS}"
        assert rel <= REL_L2, f"{where} row {b}: rel L2 {rel:.3g} > {REL_L2}"
        check_token(int(tokens[b]), ref[b], f"{where} row {b}", worst)
    return worst


def check_token(tok: int, ref_row: np.ndarray, where: str = "", stats: dict | None = None) -> None:
    order = np.argsort(-ref_row, kind="stable")
    top, second = int(order[0]), int(order[1])
    gap = float(ref_row[top] - ref_row[second])
    if tok == int(np.argmax(ref_row)):
        return
    assert gap < TIE_GAP, f"{where}: token {tok} != oracle argmax {top} (gap {gap:.3g})"
    assert ref_row[top] - ref_row[tok] < TIE_GAP, f"{where}: token {tok} is not one of the near-tied maxima"
    if stats is not None:
        stats["ties"] += 1


def run_teacher_forced(engine, dec, prompts: np.ndarray, steps: int, max_context: int, check_every: int = 1,
                       rows=None):
    """Prefill + `steps` greedy decode steps on the GPU, each compared with the
    oracle fed the GPU's previous tokens.  ``rows`` restricts the oracle to a
    subset of batch rows (rows are independent; the oracle runs them as a
    batch of their own)."""
    B = prompts.shape[0]
    rows = list(range(B)) if rows is None else list(rows)
    first, lg = engine.prefill(prompts, want_logits=True)
    first = first.cpu().numpy()
    lg = lg.cpu().numpy()
    cache = dec.new_cache(len(rows), max_context)
    ref = dec.prefill(cache, prompts[rows])
    worst = [check_logits(lg[rows], ref, first[rows], "prefill")]
    tok = first
    for s in range(steps):
        out, lg = engine.step(None, want_logits=True)
        out = out.cpu().numpy()
        ref = dec.step(cache, tok[rows])
        if s % check_every == 0 or s == steps - 1:
            worst.append(check_logits(lg.cpu().numpy()[rows], ref, out[rows], f"step {s}"))
        tok = out
    return worst
