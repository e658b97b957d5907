"""GPU parity of the decode program against the CPU oracle (tiny decoder shape).

Every check goes through the C ABI (``libwpk.so``) via the thin ctypes binding.
"""
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


PLANS = {
    "megakernel": dict(),
    "fewer_workers": dict(n_workers=37),
    "regions3": dict(n_regions=3, region_cut=(0, 1, 2, 0)),
    "per_op_graph": dict(mode=W.WPK_PER_OP_GRAPH),
    "small_tiles_one_slot": dict(tile_bytes=4096, slot_bytes=16384, lookahead=1),
    "two_stage_ring": dict(slot_bytes=32768, lookahead=2),
    "split2_page32": dict(page_tokens=32, split_pages=2),
    "tokenwise_prefill": dict(prefill=W.WPK_PREFILL_TOKENWISE),
    "static_schedule": dict(schedule=W.WPK_SCHED_STATIC),
    "team_schedule": dict(schedule=W.WPK_SCHED_TEAMS),
    "team_schedule_few_workers": dict(schedule=W.WPK_SCHED_TEAMS, n_workers=5),
}


@pytest.mark.parametrize("name", sorted(PLANS))
def test_tiny_prefill_and_16_steps(weights, dec, name):
    eng = W.Engine(S, weights, 1, CTX, **PLANS[name])
    try:
        run_teacher_forced(eng, dec, _prompts(1, 32), steps=16, max_context=CTX)
    finally:
        eng.close()


def test_tiny_prefill_attention_split_along_keys(weights, dec):
    # 2 x 2 (sequence, kv head) pairs x 3 query blocks of 64 tokens are fewer
    # tiles than the workers, so the prefill's causal attention is split along
    # the keys (128 per split) and the last split to finish combines them
    eng = W.Engine(S, weights, 2, 256)
    try:
        run_teacher_forced(eng, dec, _prompts(2, 190, seed=7), steps=3, max_context=256)
    finally:
        eng.close()


def test_tiny_batch3_ragged_tail(weights, dec):
    # 3 sequences; prompt of 37 tokens ends inside the second 32-token page
    eng = W.Engine(S, weights, 3, 96, page_tokens=32)
    try:
        run_teacher_forced(eng, dec, _prompts(3, 37, seed=5), steps=12, max_context=96)
    finally:
        eng.close()


def test_tiny_batch_smaller_than_plan(weights, dec):
    eng = W.Engine(S, weights, 4, CTX)
    try:
        run_teacher_forced(eng, dec, _prompts(2, 10, seed=6), steps=4, max_context=CTX)
    finally:
        eng.close()


def test_block_table_permutation_does_not_change_results(weights, dec):
    eng = W.Engine(S, weights, 2, 128, page_tokens=16)
    try:
        nb = 2 * (128 // 16)
        W.wpk_set_block_table(eng.h, np.random.default_rng(3).permutation(nb).astype(np.int32).reshape(2, -1))
        run_teacher_forced(eng, dec, _prompts(2, 40, seed=8), steps=6, max_context=128)
    finally:
        eng.close()


def test_explicit_input_tokens_and_context_limit(weights, dec):
    eng = W.Engine(S, weights, 1, 12)
    try:
        p = _prompts(1, 8, seed=9)
        first, lg = eng.prefill(p, want_logits=True)
        cache = dec.new_cache(1, 12)
        check_logits(lg.cpu().numpy(), dec.prefill(cache, p), first.cpu().numpy(), "prefill")
        for tok in (5, 1000, 77, 0):  # caller-chosen tokens instead of feedback
            out, lg = eng.step(np.array([tok], dtype=np.int32), want_logits=True)
            check_logits(lg.cpu().numpy(), dec.step(cache, np.array([tok])), out.cpu().numpy(), f"tok {tok}")
        with pytest.raises(W.WpkError) as ei:
            eng.step()
        assert ei.value.code == W.WPK_ERR_SHAPE
    finally:
        eng.close()


def test_trace_respects_every_edge_and_prefetches(weights):
    eng = W.Engine(S, weights, 1, CTX, trace=1)
    try:
        st = eng.stats
        eng.prefill(_prompts(1, 20), want_logits=False)
        eng.step()
        import torch

        torch.cuda.synchronize()
        tr = W.wpk_get_trace(eng.h, st["n_tiles"])
        assert sorted(tr["tile"].tolist()) == list(range(st["n_tiles"]))  # each tile ran once
        e = W.wpk_get_edges(eng.h)
        done, start, issue = tr["ev_done"].astype(np.int64), tr["ev_start"].astype(np.int64), tr["ev_issue"].astype(np.int64)
        idx = np.empty(st["n_tiles"], dtype=np.int64)
        idx[tr["tile"]] = np.arange(st["n_tiles"])
        u, v = idx[e[:, 0]], idx[e[:, 1]]
        assert np.all(done[u] < start[v]), "a tile started before one of its producers finished"
        # weight prefetch: some staging copies were issued before a producer finished
        assert np.any(issue[v] < done[u])
        assert np.all(issue <= start) and np.all(start < done)
        assert len(set(tr["worker"].tolist())) > 1
    finally:
        eng.close()


def test_team_schedule_trace_respects_every_dataflow_edge(weights):
    # the team schedule signals once per worker and op (and not at all where a
    # worker's own stream keeps the order): every edge of the full dataflow
    # graph (taken from a static plan of the same step) must still hold in the
    # traced run
    eng = W.Engine(S, weights, 2, CTX, trace=1, schedule=W.WPK_SCHED_TEAMS, n_workers=24)
    full = W.wpk_build_graph(W.model_cfg(S), W.plan_cfg(2, CTX, schedule=W.WPK_SCHED_STATIC, n_workers=24))
    try:
        st = eng.stats
        eng.prefill(_prompts(2, 20), want_logits=False)
        eng.step()
        eng.step()
        import torch

        torch.cuda.synchronize()
        tr = W.wpk_get_trace(eng.h, st["n_tiles"])
        assert sorted(tr["tile"].tolist()) == list(range(st["n_tiles"]))
        e_full = W.wpk_get_edges(full)
        assert W.wpk_graph_stats_get(eng.h)["n_signals"] < W.wpk_graph_stats_get(full)["n_signals"]
        done, start = tr["ev_done"].astype(np.int64), tr["ev_start"].astype(np.int64)
        idx = np.empty(st["n_tiles"], dtype=np.int64)
        idx[tr["tile"]] = np.arange(st["n_tiles"])
        assert np.all(done[idx[e_full[:, 0]]] < start[idx[e_full[:, 1]]])
        # each worker ran its tiles in ticket order
        for w in set(tr["worker"].tolist()):
            mine = np.sort(tr["tile"][tr["worker"] == w])
            assert np.all(np.diff(start[idx[mine]]) > 0)
    finally:
        eng.close()
        W.wpk_destroy(full)


def test_stalled_dependency_times_out_and_poisons_handle(weights):
    eng = W.Engine(S, weights, 1, CTX, wait_timeout_ns=20_000_000)
    try:
        eng.prefill(_prompts(1, 4), want_logits=False)
        W.wpk_debug_break_counter(eng.h, 3)
        eng.step()
        info = W.wpk_get_error_info(eng.h)
        assert info["code"] == W.WPK_ERR_TIMEOUT
        # the first waiter to give up records itself: the broken counter or a
        # counter downstream of it, in either case one that was never satisfied
        assert info["counter"] >= 3 and info["observed"] < info["target"]
        with pytest.raises(W.WpkError) as ei:
            eng.step()
        assert ei.value.code == W.WPK_ERR_POISONED
    finally:
        eng.close()
    # the GPU context is still usable afterwards
    eng2 = W.Engine(S, weights, 1, CTX)
    try:
        first, _ = eng2.prefill(_prompts(1, 4))
        assert 0 <= int(first.cpu()[0]) < S.vocab
    finally:
        eng2.close()


def test_out_of_range_token_is_reported(weights):
    eng = W.Engine(S, weights, 1, CTX)
    try:
        eng.prefill(_prompts(1, 4))
        eng.step(np.array([S.vocab + 5], dtype=np.int32))
        info = W.wpk_get_error_info(eng.h)
        assert info["code"] == W.WPK_ERR_INVALID_ARG
    finally:
        eng.close()
