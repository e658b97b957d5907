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
    wl = synth.WORKLOADS["llama1b_b1"]
    ctx = wl.prompt_len + wl.steps
    eng = W.Engine(S, weights, 1, ctx)
    try:
        prompts = synth.make_prompts(S.vocab, 1, wl.prompt_len, wl.prompt_seed)
        worst = run_teacher_forced(eng, dec, prompts, steps=6, max_context=ctx)
        print("worst per step:", worst)
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
