"""The allocation-free decode step, checked against the ordinary one.

Some callers cannot allocate device memory when they step the model: a host
application that reserves the whole device pool up front and gives plugins no
allocator, or a real-time loop that must never enter an allocator.  They use
wpk_step_noalloc, whose activation scratch is a static device array inside the
library instead of a caller-allocated buffer.  This file calls it through the
C ABI twice in a row and compares logits and tokens with wpk_step on an
identical handle, within the parity tolerance of the other GPU tests.  It is
named to be collected last, so a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import check_logits

pytestmark = pytest.mark.gpu

S = synth.TINY


def test_noalloc_step_matches_step_on_two_calls_in_a_row():
    import torch

    w = synth.make_weights(S, seed=0)
    prompts = synth.make_prompts(S.vocab, 2, 24, seed=1000)
    ref = W.Engine(S, w, 2, 64)
    eng = W.Engine(S, w, 2, 64)
    try:
        first_ref, _ = ref.prefill(prompts)
        first, _ = eng.prefill(prompts)
        tok = first_ref.clone()
        stream = torch.cuda.current_stream().cuda_stream
        for call in range(2):
            out_ref, lg_ref = ref.step(tok, want_logits=True)
            out = torch.empty(2, dtype=torch.int32, device="cuda")
            lg = torch.empty((2, S.vocab), dtype=torch.float32, device="cuda")
            W.wpk_step_noalloc(eng.h, tok.data_ptr(), out.data_ptr(), lg.data_ptr(), stream)
            torch.cuda.synchronize()
            check_logits(lg.cpu().numpy(), lg_ref.cpu().numpy(), out.cpu().numpy(), f"call {call}")
            tok = out_ref.clone()
    finally:
        ref.close()
        eng.close()


def test_noalloc_step_on_the_1b_shape_with_the_default_plan():
    # the default plan prefills on tensor cores, whose scratch is far larger
    # than the static array; only the decode step's scratch moves there
    import torch

    s = synth.LLAMA_1B
    w = synth.cached_weights(s, seed=0)
    prompts = synth.make_prompts(s.vocab, 1, 64, seed=1001)
    ref = W.Engine(s, w, 1, 624)
    eng = W.Engine(s, w, 1, 624)
    try:
        _, _, scratch = W.wpk_workspace_size(eng.h)
        assert scratch > (8 << 20)  # the whole plan would not fit
        first_ref, _ = ref.prefill(prompts)
        eng.prefill(prompts)
        tok = first_ref.clone()
        stream = torch.cuda.current_stream().cuda_stream
        for call in range(2):
            out_ref, lg_ref = ref.step(tok, want_logits=True)
            out = torch.empty(1, dtype=torch.int32, device="cuda")
            lg = torch.empty((1, s.vocab), dtype=torch.float32, device="cuda")
            W.wpk_step_noalloc(eng.h, tok.data_ptr(), out.data_ptr(), lg.data_ptr(), stream)
            torch.cuda.synchronize()
            check_logits(lg.cpu().numpy(), lg_ref.cpu().numpy(), out.cpu().numpy(), f"call {call}")
            tok = out_ref.clone()
    finally:
        ref.close()
        eng.close()


def test_noalloc_step_rejects_plans_larger_than_the_static_array():
    # 2048 sequences of the tiny shape need ~16 MiB of scratch (> 8 MiB)
    eng = W.Engine(S, synth.make_weights(S, seed=0), 2048, 64)
    try:
        with pytest.raises(W.WpkError) as ei:
            W.wpk_step_noalloc(eng.h)
        assert ei.value.code == W.WPK_ERR_SHAPE
    finally:
        eng.close()
