"""Fixed-cohort serving on the GPU ("Why real-time inference wants a megakernel",
"The cohort is known"): sequences are admitted into slots of a plan compiled for
a session capacity, each slot keeps its own context length, idle slots are
masked, and a step runs the whole cohort.  Every live slot is checked against
the oracle running that sequence alone (teacher-forced, the parity bar of the
other tests); idle slots must output -1 and keep their state.
"""
import numpy as np
import pytest

import oracle
import synth
from streaming_persistent_sm_b200 import wpk as W
from tests.parity import check_logits

pytestmark = pytest.mark.gpu

S = synth.TINY
CTX = 80


@pytest.fixture(scope="module")
def weights():
    return synth.make_weights(S, seed=0)


@pytest.fixture(scope="module")
def dec(weights):
    return oracle.Decoder(S, weights)


class Slot:
    """One sequence run alone by the oracle."""

    def __init__(self, dec, prompt):
        self.dec = dec
        self.cache = dec.new_cache(1, CTX)
        self.ref = dec.prefill(self.cache, prompt[None, :])
        self.n = prompt.shape[0]

    def step(self, tok):
        self.ref = self.dec.step(self.cache, np.array([tok], dtype=np.int32))
        self.n += 1


def _check(lg, out, slots, where):
    for b, sl in slots.items():
        check_logits(lg[b:b + 1], sl.ref, out[b:b + 1], f"{where} slot {b}")


@pytest.mark.parametrize("capacity,decode", [(4, W.WPK_DECODE_GEMV), (16, W.WPK_DECODE_MMA)])
def test_slots_admitted_masked_and_resumed(weights, dec, capacity, decode):
    eng = W.Engine(S, weights, capacity, CTX, decode=decode)
    try:
        pa = synth.make_prompts(S.vocab, 1, 20, 11)[0]
        pb = synth.make_prompts(S.vocab, 1, 13, 12)[0]
        pc = synth.make_prompts(S.vocab, 1, 7, 13)[0]
        # admit two sequences of different lengths into slots 0 and 2
        first_a, lg_a = eng.prefill_slots(0, pa[None, :], want_logits=True)
        first_b, lg_b = eng.prefill_slots(2, pb[None, :], want_logits=True)
        live = {0: Slot(dec, pa), 2: Slot(dec, pb)}
        check_logits(lg_a.cpu().numpy(), live[0].ref, first_a.cpu().numpy(), "prefill slot 0")
        check_logits(lg_b.cpu().numpy(), live[2].ref, first_b.cpu().numpy(), "prefill slot 2")
        last = {0: int(first_a[0]), 2: int(first_b[0])}

        def step(where):
            out, lg = eng.step(want_logits=True)
            out, lg = out.cpu().numpy(), lg.cpu().numpy()
            for b in live:
                live[b].step(last[b])
            _check(lg, out, live, where)
            for b in range(capacity):
                if b not in live:
                    assert out[b] == -1, f"{where}: idle slot {b} produced {out[b]}"
            for b in live:
                last[b] = int(out[b])
            return out

        for i in range(4):
            step(f"step {i}")
        # slot 0 idles for two steps: it outputs -1 and its sequence is frozen
        mask = np.zeros(capacity, dtype=np.int32)
        mask[2] = 1
        W.wpk_set_active_slots(eng.h, mask)
        frozen = live.pop(0)
        for i in range(2):
            step(f"slot 0 idle, step {i}")
        # admit a third sequence into slot 1 while slot 2 runs on
        first_c, lg_c = eng.prefill_slots(1, pc[None, :], want_logits=True)
        live[1] = Slot(dec, pc)
        check_logits(lg_c.cpu().numpy(), live[1].ref, first_c.cpu().numpy(), "prefill slot 1")
        last[1] = int(first_c[0])
        step("after admitting slot 1")
        # slot 0 resumes where it stopped
        mask = np.zeros(capacity, dtype=np.int32)
        mask[[0, 1, 2]] = 1
        W.wpk_set_active_slots(eng.h, mask)
        live[0] = frozen
        for i in range(3):
            step(f"three slots, step {i}")
        # each slot's own context: prompt + the steps it was live for
        assert {b: s.n for b, s in live.items()} == {0: 20 + 4 + 3, 1: 7 + 1 + 3, 2: 13 + 4 + 2 + 1 + 3}
    finally:
        eng.close()


def test_a_slot_that_was_never_filled_cannot_go_live(weights):
    eng = W.Engine(S, weights, 4, CTX)
    try:
        eng.prefill_slots(0, synth.make_prompts(S.vocab, 1, 5, 3))
        with pytest.raises(W.WpkError) as ei:
            W.wpk_set_active_slots(eng.h, np.array([1, 1, 0, 0], dtype=np.int32))
        assert ei.value.code == W.WPK_ERR_INVALID_ARG
    finally:
        eng.close()


def test_a_live_slot_stops_at_the_context_limit(weights):
    eng = W.Engine(S, weights, 2, 12)
    try:
        eng.prefill_slots(1, synth.make_prompts(S.vocab, 1, 10, 4))
        eng.step()
        eng.step()  # slot 1 now holds 12 tokens
        with pytest.raises(W.WpkError) as ei:
            eng.step()
        assert ei.value.code == W.WPK_ERR_SHAPE
    finally:
        eng.close()
