"""GPU parity on the Llama-3.2-1B-shaped decoder (full size, seeded random init).

Prefill of the 496-token prompt (first token), then greedy decode steps, each
teacher-forced against the float64 oracle on all 128256 logits.  Batched runs
check rows {0, B/2, B-1} with the oracle (rows are independent).
"""
import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import run_teacher_forced

pytestmark = pytest.mark.gpu

S = synth.LLAMA_1B


@pytest.fixture(scope="module")
def weights():
    return synth.cached_weights(S, seed=0)


@pytest.fixture(scope="module")
def dec(weights):
    return oracle.Decoder(S, weights)


def test_llama1b_b1_prefill_and_steps(weights, dec):
    # the bench's job in the bench's launch configuration (static schedule):
    # prefill and all 128 steps, to context 623, so the attention splits past
    # the 512- and 576-token page boundaries hold data; every 8th step and the
    # last are compared on all 128256 logits (the oracle runs every step)
    wl = synth.WORKLOADS["llama1b_b1"]
    ctx = wl.prompt_len + wl.steps
    eng = W.Engine(S, weights, 1, ctx, schedule=W.WPK_SCHED_STATIC)
    try:
        prompts = synth.make_prompts(S.vocab, 1, wl.prompt_len, wl.prompt_seed)
        worst = run_teacher_forced(eng, dec, prompts, steps=wl.steps, max_context=ctx, check_every=8)
        assert len(worst) == 1 + wl.steps // 8 + (1 if (wl.steps - 1) % 8 else 0)
        print("worst per checked step:", worst)
    finally:
        eng.close()


def test_llama1b_b1_per_op_graph(weights, dec):
    wl = synth.WORKLOADS["llama1b_b1"]
    ctx = wl.prompt_len + wl.steps
    eng = W.Engine(S, weights, 1, ctx, mode=W.WPK_PER_OP_GRAPH)
    try:
        prompts = synth.make_prompts(S.vocab, 1, 64, wl.prompt_seed)
        run_teacher_forced(eng, dec, prompts, steps=3, max_context=ctx)
    finally:
        eng.close()


@pytest.mark.parametrize("B,decode", [(16, W.WPK_DECODE_MMA), (16, W.WPK_DECODE_GEMV), (48, W.WPK_DECODE_MMA)])
def test_llama1b_batched_sampled_rows(weights, dec, B, decode):
    wl = synth.WORKLOADS[f"llama1b_decode_b{B}"]
    ctx = wl.prompt_len + wl.steps
    eng = W.Engine(S, weights, B, ctx, decode=decode)
    try:
        prompts = synth.make_prompts(S.vocab, B, wl.prompt_len, wl.prompt_seed)
        run_teacher_forced(eng, dec, prompts, steps=3, max_context=ctx, rows=[0, B // 2, B - 1])
    finally:
        eng.close()


def test_llama1b_decode_b32_sampled_rows(weights, dec):
    # the C3 shape at batch 32 in the bench's configuration (tensor-core
    # decode, static schedule): 24 steps, rows {0, 16, 31}
    wl = synth.WORKLOADS["llama1b_decode_b32"]
    B = wl.batch
    ctx = wl.prompt_len + wl.steps
    eng = W.Engine(S, weights, B, ctx, schedule=W.WPK_SCHED_STATIC)
    try:
        assert "b_qkv" in [W.OP_NAMES[o] for o in W.wpk_get_tile_ops(eng.h, eng.stats["n_tiles"])]
        prompts = synth.make_prompts(S.vocab, B, wl.prompt_len, wl.prompt_seed)
        run_teacher_forced(eng, dec, prompts, steps=24, max_context=ctx, check_every=4, rows=[0, B // 2, B - 1])
    finally:
        eng.close()


def test_llama1b_prefill_b32_sampled_rows(weights, dec):
    # the C4 shape at its largest batch: 32 prompts of 496 tokens (15872 rows)
    wl = synth.WORKLOADS["llama1b_prefill_b32"]
    B = wl.batch
    eng = W.Engine(S, weights, B, wl.prompt_len + 4)
    try:
        prompts = synth.make_prompts(S.vocab, B, wl.prompt_len, wl.prompt_seed)
        run_teacher_forced(eng, dec, prompts, steps=1, max_context=wl.prompt_len + 4, rows=[0, B // 2, B - 1])
    finally:
        eng.close()


@pytest.mark.parametrize("plan", [{}, dict(frame_chunks=2)])
def test_two_stage_1b_shape_b32_sampled_rows(plan):
    # the C5 shape: the 1B backbone, a 4-layer h1024 head, 16 codebooks of 2048,
    # batch 32 (tensor-core decode for both), 200-token prompts, two frames;
    # chunked: two pairs of 16 sequences, row 16 is the second chunk's first
    from tests.test_two_stage_gpu import _check_frame_shape

    s = synth.TWO_STAGE
    w = synth.cached_weights(s, seed=0)
    ora = oracle.TwoStage(s, w)
    wl = synth.WORKLOADS["two_stage_b32"]
    B, T, rows = wl.batch, wl.prompt_len, [0, 16, 31]
    eng = W.Engine(s, w, B, T + 4, **plan)
    try:
        prompts = synth.make_prompts(s.backbone.vocab, B, T, wl.prompt_seed)
        codes, lg = eng.prefill(prompts, want_logits=True)
        codes, lg = codes.cpu().numpy(), lg.cpu().numpy()
        cache = ora.backbone.new_cache(len(rows), T + 4)
        _, ref = ora.prefill(cache, prompts[rows], forced=codes[rows])
        _check_frame_shape(s, codes[rows], lg[rows], ref, "prefill")
        for f in range(2):
            prev = codes
            out, lg = eng.step(want_logits=True)
            codes, lg = out.cpu().numpy(), lg.cpu().numpy()
            _, ref = ora.frame(cache, prev[rows], forced=codes[rows])
            _check_frame_shape(s, codes[rows], lg[rows], ref, f"frame {f}")
    finally:
        eng.close()
