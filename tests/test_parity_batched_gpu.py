"""GPU parity of the batched decode program (tensor-core tiles, more than 8
sequences per step) against the CPU oracle, tiny decoder shape.

The step's sequences are the N dimension of tcgen05 tiles whose M dimension is
128 weight rows; O and down projections are split along K and summed in fp32.
Every check goes through the C ABI.
"""
import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import run_teacher_forced

pytestmark = pytest.mark.gpu

S = synth.TINY
CTX = 96


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
    "static_schedule": dict(schedule=W.WPK_SCHED_STATIC),
    "per_op_graph": dict(mode=W.WPK_PER_OP_GRAPH),
    "regions3": dict(n_regions=3, region_cut=(0, 1, 2, 0)),
    "fewer_workers": dict(n_workers=29),
    "page32_split1": dict(page_tokens=32, split_pages=1),
    "two_stage_ring": dict(slot_bytes=32768, lookahead=2),
    "team_schedule": dict(schedule=W.WPK_SCHED_TEAMS),
}


@pytest.mark.parametrize("name", sorted(PLANS))
def test_batched_decode_b16(weights, dec, name):
    eng = W.Engine(S, weights, 16, CTX, **PLANS[name])
    try:
        assert "b_qkv" in [W.OP_NAMES[o] for o in W.wpk_get_tile_ops(eng.h, eng.stats["n_tiles"])]
        run_teacher_forced(eng, dec, _prompts(16, 21, seed=11), steps=10, max_context=CTX)
    finally:
        eng.close()


@pytest.mark.parametrize("plan_b,active,T", [(16, 13, 30), (9, 9, 17), (32, 32, 40), (48, 33, 9)])
def test_batched_decode_ragged(weights, dec, plan_b, active, T):
    # active batch below the plan and below the padded MMA N; prompts end
    # inside a page
    eng = W.Engine(S, weights, plan_b, CTX)
    try:
        run_teacher_forced(eng, dec, _prompts(active, T, seed=plan_b + active), steps=6, max_context=CTX)
    finally:
        eng.close()


def test_batched_decode_at_the_maximum_batch(weights, dec):
    # the largest tensor-core N: a plan of 128 sequences (two 128-row hi/lo
    # images per stage), 117 of them active, prompts ending inside a page
    eng = W.Engine(S, weights, 128, CTX, decode=W.WPK_DECODE_MMA)
    try:
        assert "b_qkv" in [W.OP_NAMES[o] for o in W.wpk_get_tile_ops(eng.h, eng.stats["n_tiles"])]
        run_teacher_forced(eng, dec, _prompts(117, 23, seed=117), steps=6, max_context=CTX)
    finally:
        eng.close()


def test_batched_decode_matches_gemv_program(weights):
    # the tensor-core and the CUDA-core decode programs agree with each other
    # as closely as each agrees with the oracle
    p = _prompts(12, 16, seed=3)
    out = {}
    for mode in (W.WPK_DECODE_MMA, W.WPK_DECODE_GEMV):
        eng = W.Engine(S, weights, 12, 64, decode=mode)
        try:
            eng.prefill(p)
            logits = []
            for tok in (3, 700, 42):
                _, lg = eng.step(np.full(12, tok, dtype=np.int32), want_logits=True)
                logits.append(lg.cpu().numpy())
            out[mode] = np.stack(logits)
        finally:
            eng.close()
    d = np.abs(out[W.WPK_DECODE_MMA] - out[W.WPK_DECODE_GEMV])
    assert d.max() < 2e-2, d.max()


def test_batched_trace_respects_every_edge(weights):
    eng = W.Engine(S, weights, 16, CTX, trace=1)
    try:
        st = eng.stats
        eng.prefill(_prompts(16, 20), want_logits=False)
        eng.step()
        import torch

        torch.cuda.synchronize()
        tr = W.wpk_get_trace(eng.h, st["n_tiles"])
        assert sorted(tr["tile"].tolist()) == list(range(st["n_tiles"]))
        e = W.wpk_get_edges(eng.h)
        done, start = tr["ev_done"].astype(np.int64), tr["ev_start"].astype(np.int64)
        idx = np.empty(st["n_tiles"], dtype=np.int64)
        idx[tr["tile"]] = np.arange(st["n_tiles"])
        assert np.all(done[idx[e[:, 0]]] < start[idx[e[:, 1]]])
    finally:
        eng.close()


def test_batched_out_of_range_token_is_reported(weights):
    eng = W.Engine(S, weights, 16, CTX)
    try:
        eng.prefill(_prompts(16, 4))
        toks = np.zeros(16, dtype=np.int32)
        toks[7] = S.vocab + 1
        eng.step(toks)
        assert W.wpk_get_error_info(eng.h)["code"] == W.WPK_ERR_INVALID_ARG
    finally:
        eng.close()
