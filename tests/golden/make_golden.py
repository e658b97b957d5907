"""Write the oracle regression fixtures in this folder.

It calls only the oracle (``oracle/``) and the seeded input generators
(``synth/``).  The fixtures record what the float64 oracle computes for a few
small seeded cases, so that a later change to the oracle's arithmetic shows up
as a failed comparison and has to be justified.  They pin the oracle to its own
past, not to an outside fact: the outside pins are the closed forms, invariants
and the float64 Hugging Face Llama comparison in ``tests/test_oracle_pins.py``.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
SAMPLE = [0, 1, 17, 255, 511, 1023]  # logit columns recorded per row


def decoder_case():
    """Tiny decoder: 2 sequences, a 9-token prompt, then 3 greedy steps."""
    s = synth.TINY
    w = synth.make_weights(s, seed=0)
    dec = oracle.Decoder(s, w)
    prompts = synth.make_prompts(s.vocab, 2, 9, seed=7)
    cache = dec.new_cache(2, 16)
    lg = dec.prefill(cache, prompts)
    rows = []
    for step in range(4):
        tok = oracle.argmax_lowest(lg)
        m = lg.max(1)
        lse = np.log(np.exp(lg - m[:, None]).sum(1)) + m
        rows.append({"step": step, "tokens": tok.tolist(), "logits_sample": lg[:, SAMPLE].tolist(),
                     "logsumexp": lse.tolist()})
        if step < 3:
            lg = dec.step(cache, tok)
    return {"case": "tiny decoder, weights seed 0, prompts seed 7 (2 x 9 tokens), prefill then 3 greedy steps",
            "shape": "TINY", "sample_columns": SAMPLE, "steps": rows}


def two_stage_case():
    """Tiny two-stage model: 2 sequences, a 5-token prompt, the first frame and one more."""
    s = synth.TINY_TWO_STAGE
    w = synth.make_weights(s, seed=0)
    ts = oracle.TwoStage(s, w)
    prompts = synth.make_prompts(s.backbone.vocab, 2, 5, seed=11)
    cache = ts.backbone.new_cache(2, 8)
    codes, lg = ts.prefill(cache, prompts)
    frames = [{"frame": 0, "codes": np.asarray(codes).tolist(), "logits_k0_sample": lg[:, 0, :8].tolist()}]
    codes2, lg2 = ts.frame(cache, np.asarray(codes))
    frames.append({"frame": 1, "codes": np.asarray(codes2).tolist(), "logits_k0_sample": lg2[:, 0, :8].tolist()})
    return {"case": "tiny two-stage model, weights seed 0, prompts seed 11 (2 x 5 tokens), two frames",
            "shape": "TINY_TWO_STAGE", "frames": frames}


def main():
    out = {"decoder": decoder_case(), "two_stage": two_stage_case()}
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
