"""The resident grid: one cooperative launch serves many steps, driven by a
doorbell in mapped host memory (tiny decoder shape, parity against the oracle).
"""
import time

import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import check_logits, run_teacher_forced

pytestmark = pytest.mark.gpu

S = synth.TINY
CTX = 64


@pytest.fixture(scope="module")
def weights():
    return synth.make_weights(S, seed=0)


@pytest.fixture(scope="module")
def dec(weights):
    return oracle.Decoder(S, weights)


def _prompts(B, T, seed=synth.WORKLOADS["tiny"].prompt_seed):
    return synth.make_prompts(S.vocab, B, T, seed)


@pytest.mark.parametrize("B,schedule", [(1, W.WPK_SCHED_QUEUE), (1, W.WPK_SCHED_STATIC), (3, W.WPK_SCHED_QUEUE),
                                        (16, W.WPK_SCHED_STATIC)])
def test_resident_prefill_and_steps(weights, dec, B, schedule):
    eng = W.Engine(S, weights, B, CTX, resident=1, schedule=schedule)
    try:
        run_teacher_forced(eng, dec, _prompts(B, 20, seed=B), steps=16, max_context=CTX)
    finally:
        eng.close()


def test_resident_grid_survives_idle_exit_and_new_prefill(weights, dec):
    # a 20 ms wait bound gives a 400 ms idle limit: the grid leaves while the
    # host sleeps and the next step launches a new one; a new prefill stops
    # the grid and the following steps start another
    eng = W.Engine(S, weights, 1, CTX, resident=1, wait_timeout_ns=20_000_000)
    try:
        p = _prompts(1, 12, seed=21)
        first, lg = eng.prefill(p, want_logits=True)
        cache = dec.new_cache(1, CTX)
        check_logits(lg.cpu().numpy(), dec.prefill(cache, p), first.cpu().numpy(), "prefill")
        tok = first.cpu().numpy()
        for i in range(6):
            if i == 3:
                time.sleep(0.6)
            out, lg = eng.step(tok, want_logits=True)
            check_logits(lg.cpu().numpy(), dec.step(cache, tok), out.cpu().numpy(), f"step {i}")
            tok = out.cpu().numpy()
        run_teacher_forced(eng, dec, _prompts(1, 9, seed=22), steps=4, max_context=CTX)
    finally:
        eng.close()


def test_resident_trace_respects_every_edge(weights):
    eng = W.Engine(S, weights, 1, CTX, resident=1, trace=1)
    try:
        st = eng.stats
        eng.prefill(_prompts(1, 20), want_logits=False)
        for _ in range(3):
            eng.step()
        tr = W.wpk_get_trace(eng.h, st["n_tiles"])  # stops the grid first
        assert sorted(tr["tile"].tolist()) == list(range(st["n_tiles"]))
        assert set(tr["epoch"].tolist()) == {3}  # the last of three steps on one grid
        e = W.wpk_get_edges(eng.h)
        done, start = tr["ev_done"].astype(np.int64), tr["ev_start"].astype(np.int64)
        idx = np.empty(st["n_tiles"], dtype=np.int64)
        idx[tr["tile"]] = np.arange(st["n_tiles"])
        assert np.all(done[idx[e[:, 0]]] < start[idx[e[:, 1]]])
    finally:
        eng.close()


def test_resident_stall_is_reported_and_poisons(weights):
    eng = W.Engine(S, weights, 1, CTX, resident=1, wait_timeout_ns=20_000_000)
    try:
        eng.prefill(_prompts(1, 4), want_logits=False)
        eng.step()
        W.wpk_debug_break_counter(eng.h, 3)
        with pytest.raises(W.WpkError) as ei:
            eng.step()
        assert ei.value.code in (W.WPK_ERR_POISONED, W.WPK_ERR_TIMEOUT)
        assert W.wpk_get_error_info(eng.h)["code"] == W.WPK_ERR_TIMEOUT
    finally:
        eng.close()
    eng2 = W.Engine(S, weights, 1, CTX, resident=1)
    try:
        first, _ = eng2.prefill(_prompts(1, 4))
        eng2.step()
        assert 0 <= int(first.cpu()[0]) < S.vocab
    finally:
        eng2.close()
