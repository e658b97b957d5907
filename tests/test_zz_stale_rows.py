"""Regression: pages are staged before the step writes its own token's K/V row,
so the staged copy of that row is stale.  Fill every caller-owned buffer with
NaN before loading; no NaN may reach the results (GEMV and tensor-core decode)."""
import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import run_teacher_forced

pytestmark = pytest.mark.gpu

S = synth.TINY


@pytest.mark.parametrize("B,page", [(3, 32), (1, 64), (16, 32)])
def test_nan_filled_buffers_do_not_leak(B, page):
    import torch

    w = synth.make_weights(S, seed=0)
    dec = oracle.Decoder(S, w)
    model, plan = W.model_cfg(S), W.plan_cfg(B, 96, page_tokens=page)
    h = W.wpk_build_graph(model, plan)
    eng = None
    try:
        wb, kb, sb = W.wpk_workspace_size(h)
        dev = torch.device("cuda", 0)
        bufs = [torch.full((max(n, 256) // 4,), float("nan"), dtype=torch.float32, device=dev) for n in (wb, kb, sb)]
        eng = W.Engine.__new__(W.Engine)  # an Engine over these NaN-filled buffers
        eng.torch, eng.shape, eng.plan, eng.h, eng.max_batch, eng.batch = torch, S, plan, h, B, 0
        eng._tok_shape, eng._logit_shape = (), (S.vocab,)
        eng.dev_weights, eng.dev_kv, eng.dev_scratch = bufs
        hw = W._HostWeights(S, w)
        W.wpk_load_weights(h, hw.struct, bufs[0].data_ptr(), bufs[1].data_ptr(), bufs[2].data_ptr(), eng._stream())
        run_teacher_forced(eng, dec, synth.make_prompts(S.vocab, B, 37, 5), steps=8, max_context=96)
    finally:
        if eng is not None:
            eng.close()  # destroys the handle once
        else:
            W.wpk_destroy(h)
