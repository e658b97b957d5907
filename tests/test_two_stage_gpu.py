"""GPU parity of the two-stage streaming model (backbone + codebook head) against
the oracle's TwoStage, teacher-forced with the GPU's codes.

The composition (projection, head inputs, output heads, next-frame input) is
this repository's reading of a two-stage streaming model.  The oracle's
implementation of it is pinned against transformers' Llama layers in
tests/test_oracle_pins.py.
"""
import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import check_logits

pytestmark = pytest.mark.gpu

S = synth.TINY_TWO_STAGE


@pytest.fixture(scope="module")
def weights():
    return synth.make_weights(S, seed=0)


@pytest.fixture(scope="module")
def ora(weights):
    return oracle.TwoStage(S, weights)


def _check_frame_shape(shape, gpu_codes, gpu_logits, ref_logits, where):
    for k in range(shape.n_codebooks):
        check_logits(gpu_logits[:, k], ref_logits[:, k], gpu_codes[:, k], f"{where} codebook {k}")


def _check_frame(gpu_codes, gpu_logits, ref_logits, where):
    _check_frame_shape(S, gpu_codes, gpu_logits, ref_logits, where)


@pytest.mark.parametrize("B,plan", [(1, {}), (3, {}), (16, {}), (12, dict(schedule=W.WPK_SCHED_STATIC)),
                                    (2, dict(n_regions=2, region_cut=(0, 1, 0, 0))),
                                    # chunked frames: backbone and head launches overlap on two streams
                                    (3, dict(frame_chunks=2)), (5, dict(frame_chunks=3, head_workers=40)),
                                    (16, dict(frame_chunks=2, schedule=W.WPK_SCHED_STATIC))])
def test_two_stage_prefill_and_frames(weights, ora, B, plan):
    T, frames, ctx = 17, 6, 32
    eng = W.Engine(S, weights, B, ctx, **plan)
    try:
        prompts = synth.make_prompts(S.backbone.vocab, B, T, 40 + B)
        codes, lg = eng.prefill(prompts, want_logits=True)
        codes, lg = codes.cpu().numpy(), lg.cpu().numpy()
        assert codes.shape == (B, S.n_codebooks) and lg.shape == (B, S.n_codebooks, S.codebook_vocab)
        cache = ora.backbone.new_cache(B, ctx)
        _, ref = ora.prefill(cache, prompts, forced=codes)
        _check_frame(codes, lg, ref, "prefill")
        for f in range(frames):
            prev = codes
            out, lg = eng.step(want_logits=True)  # input: the previous frame's codes
            codes, lg = out.cpu().numpy(), lg.cpu().numpy()
            _, ref = ora.frame(cache, prev, forced=codes)
            _check_frame(codes, lg, ref, f"frame {f}")
    finally:
        eng.close()


@pytest.mark.parametrize("plan", [{}, dict(frame_chunks=2)])
def test_two_stage_explicit_codes_are_the_next_input(weights, ora, plan):
    B, T, ctx = 2, 9, 16
    eng = W.Engine(S, weights, B, ctx, **plan)
    try:
        prompts = synth.make_prompts(S.backbone.vocab, B, T, 7)
        codes, _ = eng.prefill(prompts)
        cache = ora.backbone.new_cache(B, ctx)
        ora.prefill(cache, prompts, forced=codes.cpu().numpy())
        chosen = np.array([[1, 2, 3, 4], [255, 0, 17, 9]], dtype=np.int32)
        out, lg = eng.step(chosen, want_logits=True)
        _, ref = ora.frame(cache, chosen, forced=out.cpu().numpy())
        _check_frame(out.cpu().numpy(), lg.cpu().numpy(), ref, "explicit")
        bad = chosen.copy()
        bad[1, 2] = S.codebook_vocab  # out of range code
        eng.step(bad)
        assert W.wpk_get_error_info(eng.h)["code"] == W.WPK_ERR_INVALID_ARG
    finally:
        eng.close()
