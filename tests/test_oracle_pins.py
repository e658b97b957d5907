"""Pins for the CPU oracle: each check compares it with something other than
itself (a closed form, an invariant, a library routine, or an independent
implementation), chosen so that a plausible slip (a sign, an index, a
transposed operand, a dropped term) fails at least one of them."""
import math

import numpy as np
import pytest

import oracle
from oracle import llama as L
import synth

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------- bf16 --
def _torch_bf16(x32: np.ndarray) -> np.ndarray:
    import torch

    return torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()


def test_round_bf16_matches_torch_on_all_tie_classes():
    # Random fp32 bit patterns plus every low-half pattern that decides RNE.
    hi = RNG.integers(0x0001, 0x7F7F, size=4000, dtype=np.uint32)
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF], dtype=np.uint32)
    bits = (hi[:, None] << 16 | lows[None, :]).ravel()
    sign = RNG.integers(0, 2, size=bits.size, dtype=np.uint32) << 31
    x32 = (bits | sign).view(np.float32)
    got = oracle.round_bf16(x32.astype(np.float64))
    np.testing.assert_array_equal(got, _torch_bf16(x32))


def test_round_bf16_hand_values():
    one = 1.0
    assert oracle.round_bf16(np.array(one + 2 ** -8)) == 1.0            # tie -> even (1.0)
    assert oracle.round_bf16(np.array(one + 3 * 2 ** -8)) == one + 2 ** -6  # tie -> even (mantissa 2)
    assert oracle.round_bf16(np.array(one + 2 ** -8 + 2 ** -20)) == one + 2 ** -7
    assert oracle.round_bf16(np.array(-3.0)) == -3.0
    assert oracle.round_bf16(np.array(0.0)) == 0.0


def test_bf16_widening_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x3C23], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.bf16_to_f64(bits), [1.0, -1.0, 3.140625, 0.0, 2.0 ** -7 * (1 + 35 / 128)])


# ------------------------------------------------------------------ RMSNorm --
def test_rmsnorm_output_rms_closed_form():
    x = RNG.standard_normal((5, 64)) * 3.0
    eps = 1e-2
    y = oracle.rmsnorm(x, np.ones(64), eps)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12)


def test_rmsnorm_gain_and_scale_invariance():
    x = RNG.standard_normal((3, 32))
    g = RNG.standard_normal(32)
    y = oracle.rmsnorm(x, g, 0.0)
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, g, 0.0), y, rtol=1e-12)
    np.testing.assert_allclose(y / g, oracle.rmsnorm(x, np.ones(32), 0.0), rtol=1e-10)
    # a constant vector normalises to all ones
    np.testing.assert_allclose(oracle.rmsnorm(np.full((1, 8), -4.0), np.ones(8), 0.0), -np.ones((1, 8)))


# --------------------------------------------------------------------- RoPE --
def test_rope_is_a_rotation_by_position_for_d2():
    # d = 2: one pair, inv_0 = 1, so position p rotates by p radians, counter-clockwise.
    for p in [0, 1, 3, 17]:
        e0 = oracle.rope_apply(np.array([[[1.0, 0.0]]]), np.array([p]), 10000.0)[0, 0]
        e1 = oracle.rope_apply(np.array([[[0.0, 1.0]]]), np.array([p]), 10000.0)[0, 0]
        np.testing.assert_allclose(e0, [math.cos(p), math.sin(p)], atol=1e-15)
        np.testing.assert_allclose(e1, [-math.sin(p), math.cos(p)], atol=1e-15)


def test_rope_pairs_half_apart_and_frequency_formula():
    # d = 4, theta = 100: inv = [1, 100^(-1/2) = 0.1]; pairs are (0, 2) and (1, 3).
    x = np.zeros((1, 1, 4))
    x[0, 0, 1] = 1.0
    y = oracle.rope_apply(x, np.array([10]), 100.0)[0, 0]
    np.testing.assert_allclose(y, [0.0, math.cos(1.0), 0.0, math.sin(1.0)], atol=1e-15)
    np.testing.assert_allclose(oracle.rope_inv_freq(64, 500000.0)[[0, 1, 31]],
                               [1.0, 500000.0 ** (-2 / 64), 500000.0 ** (-62 / 64)], rtol=1e-15)


def test_rope_norm_identity_and_relative_position():
    d = 64
    q = RNG.standard_normal((1, 1, d))
    k = RNG.standard_normal((1, 1, d))
    np.testing.assert_array_equal(oracle.rope_apply(q, np.array([0]), 1e4), q)
    for p in [1, 100, 623]:
        r = oracle.rope_apply(q, np.array([p]), 5e5)
        pair = lambda a: a[..., :32] ** 2 + a[..., 32:] ** 2
        np.testing.assert_allclose(pair(r), pair(q), rtol=1e-12)
    dot = lambda m, n: float(np.sum(oracle.rope_apply(q, np.array([m]), 1e4) *
                                    oracle.rope_apply(k, np.array([n]), 1e4)))
    assert dot(7, 3) == pytest.approx(dot(107, 103), rel=1e-9)
    assert dot(7, 3) != pytest.approx(dot(7, 4), rel=1e-3)


# ------------------------------------------------------------ softmax, silu --
def test_softmax_closed_forms():
    s = RNG.standard_normal((4, 9)) * 5
    np.testing.assert_allclose(oracle.softmax(s).sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.softmax(np.full((1, 5), 3.3)), np.full((1, 5), 0.2))
    np.testing.assert_allclose(oracle.softmax(np.array([[0.0, math.log(2.0)]])), [[1 / 3, 2 / 3]])
    np.testing.assert_allclose(oracle.softmax(s + 100.0), oracle.softmax(s), rtol=1e-12)


def test_silu_closed_forms():
    assert oracle.silu(np.array(0.0)) == 0.0
    z = RNG.standard_normal(100) * 4
    np.testing.assert_allclose(oracle.silu(z) - oracle.silu(-z), z, atol=1e-14)
    assert oracle.silu(np.array(math.log(3.0))) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    assert oracle.silu(np.array(-40.0)) == pytest.approx(0.0, abs=1e-15)


# ---------------------------------------------------------------- attention --
def test_attention_single_token_returns_v():
    q = RNG.standard_normal((1, 4, 64))
    k = RNG.standard_normal((1, 2, 64))
    v = RNG.standard_normal((1, 2, 64))
    o = oracle.attention(q, k, v, np.array([0]), np.array([0]))
    np.testing.assert_allclose(o[0, [0, 1]], v[0, [0, 0]], rtol=1e-15)
    np.testing.assert_allclose(o[0, [2, 3]], v[0, [1, 1]], rtol=1e-15)


def test_attention_two_keys_weights_three_to_one():
    # scores differ by ln 3 -> softmax weights 3/4 and 1/4 (scale 1/sqrt(d) with d = 4 is 1/2)
    d = 4
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 2.0
    k = np.zeros((2, 1, d)); k[0, 0, 0] = math.log(3.0)
    v = RNG.standard_normal((2, 1, d))
    o = oracle.attention(q, k, v, np.array([1]), np.array([0, 1]))
    np.testing.assert_allclose(o[0, 0], 0.75 * v[0, 0] + 0.25 * v[1, 0], rtol=1e-14)


def test_attention_causal_mask_and_gqa_equals_repeated_mha():
    T, hq, hkv, d = 6, 8, 2, 16
    q = RNG.standard_normal((T, hq, d))
    k = RNG.standard_normal((T, hkv, d))
    v = RNG.standard_normal((T, hkv, d))
    pos = np.arange(T)
    o = oracle.attention(q, k, v, pos, pos)
    o_mha = oracle.attention(q, np.repeat(k, hq // hkv, axis=1), np.repeat(v, hq // hkv, axis=1), pos, pos)
    np.testing.assert_allclose(o, o_mha, rtol=1e-14)
    # the first query sees only the first key
    np.testing.assert_allclose(o[0, 0], v[0, 0], rtol=1e-14)
    np.testing.assert_allclose(o[0, hq - 1], v[0, hkv - 1], rtol=1e-14)


def test_argmax_lowest_index_on_ties():
    np.testing.assert_array_equal(oracle.argmax_lowest(np.array([[1.0, 3.0, 3.0, 2.0], [5, 5, 5, 5]])), [1, 0])


# ----------------------------------------------------------- whole decoder --
TINY = synth.TINY


@pytest.fixture(scope="module")
def tiny_weights():
    return synth.make_weights(TINY, seed=0)


def _hf_model(weights):
    import torch
    from transformers import LlamaConfig, LlamaForCausalLM

    s = TINY
    cfg = LlamaConfig(vocab_size=s.vocab, hidden_size=s.hidden, intermediate_size=s.ffn,
                      num_hidden_layers=s.n_layers, num_attention_heads=s.n_heads,
                      num_key_value_heads=s.n_kv_heads, head_dim=s.head_dim, rms_norm_eps=s.rms_eps,
                      rope_theta=s.rope_theta, tie_word_embeddings=True, max_position_embeddings=4096,
                      attention_bias=False, mlp_bias=False)
    m = LlamaForCausalLM(cfg).double().eval()
    f = lambda n: torch.from_numpy(oracle.bf16_to_f64(weights[n]))
    names = {"model.embed_tokens.weight": "embed", "model.norm.weight": "final_norm"}
    for l in range(s.n_layers):
        p, q = f"model.layers.{l}.", f"layers.{l}."
        names.update({p + "self_attn.q_proj.weight": q + "wq", p + "self_attn.k_proj.weight": q + "wk",
                      p + "self_attn.v_proj.weight": q + "wv", p + "self_attn.o_proj.weight": q + "wo",
                      p + "mlp.gate_proj.weight": q + "w_gate", p + "mlp.up_proj.weight": q + "w_up",
                      p + "mlp.down_proj.weight": q + "w_down", p + "input_layernorm.weight": q + "attn_norm",
                      p + "post_attention_layernorm.weight": q + "ffn_norm"})
    sd = m.state_dict()
    with torch.no_grad():
        for hf, ours in names.items():
            sd[hf].copy_(f(ours))
        m.lm_head.weight.copy_(f("embed"))
    return m


def _hf_logits(m, tokens):
    import torch

    with torch.no_grad():
        return m(torch.from_numpy(np.asarray(tokens, dtype=np.int64))).logits.numpy()


def _oracle_seq_logits(dec, tokens):
    """Oracle logits at every prompt position (prefill of the first token, then steps)."""
    B, T = tokens.shape
    cache = dec.new_cache(B, 128)
    out = [dec.prefill(cache, tokens[:, :1])]
    for t in range(1, T):
        out.append(dec.step(cache, tokens[:, t]))
    return np.stack(out, axis=1)


def test_decoder_matches_transformers_llama_fp64(tiny_weights):
    tokens = synth.make_prompts(TINY.vocab, 2, 12, seed=7)
    hf = _hf_logits(_hf_model(tiny_weights), tokens)
    dec = oracle.Decoder(TINY, tiny_weights, round_kv=False)
    ours = _oracle_seq_logits(dec, tokens)
    # transformers evaluates its RoPE cos/sin in float32 even in a float64
    # model, so the two agree to ~1e-7 rather than to float64 rounding; every
    # structural slip planted below moves the logits by more than 1e-3.
    np.testing.assert_allclose(ours, hf, atol=2e-6, rtol=0)
    # also the one-shot prefill of the whole prompt
    cache = dec.new_cache(2, 64)
    np.testing.assert_allclose(dec.prefill(cache, tokens), hf[:, -1], atol=2e-6, rtol=0)


PLANTED = {
    "rope_sign": lambda: _patch(L, "rope_apply", lambda x, pos, th: _rope_neg(x, pos, th)),
    "gqa_modulo": lambda: _patch(L, "attention", _attention_modulo),
    "silu_is_relu": lambda: _patch(L, "silu", lambda z: np.maximum(z, 0.0)),
    "rmsnorm_no_eps": lambda: _patch(L, "rmsnorm", lambda x, g, eps: x / np.sqrt(np.mean(x * x, -1, keepdims=True) + 1.0) * g),
}


def _patch(mod, name, fn):
    old = getattr(mod, name)
    setattr(mod, name, fn)
    return lambda: setattr(mod, name, old)


_orig_rope = L.rope_apply
_orig_attention = L.attention


def _rope_neg(x, pos, theta):
    return _orig_rope(x, -np.asarray(pos), theta)


def _attention_modulo(q, k, v, qp, kp):
    hq, hkv = q.shape[1], k.shape[1]
    perm = [h % hkv for h in range(hq)]
    kk = k[:, perm]
    vv = v[:, perm]
    return _orig_attention(q, kk, vv, qp, kp)


@pytest.mark.parametrize("mistake", sorted(PLANTED))
def test_planted_mistakes_are_caught_by_the_transformers_pin(tiny_weights, mistake):
    """A deliberate slip planted in the oracle (CPU only) must break the cross-check."""
    tokens = synth.make_prompts(TINY.vocab, 1, 8, seed=3)
    hf = _hf_logits(_hf_model(tiny_weights), tokens)
    undo = PLANTED[mistake]()
    try:
        dec = oracle.Decoder(TINY, tiny_weights, round_kv=False)
        ours = _oracle_seq_logits(dec, tokens)
    finally:
        undo()
    assert np.max(np.abs(ours - hf)) > 1e-3


def test_prefill_equals_incremental_decode(tiny_weights):
    dec = oracle.Decoder(TINY, tiny_weights)
    tokens = synth.make_prompts(TINY.vocab, 2, 20, seed=11)
    c1 = dec.new_cache(2, 64)
    full = dec.prefill(c1, tokens)
    inc = _oracle_seq_logits(dec, tokens)[:, -1]
    np.testing.assert_allclose(full, inc, atol=1e-6, rtol=0)


def test_batch_rows_are_independent(tiny_weights):
    dec = oracle.Decoder(TINY, tiny_weights)
    tokens = synth.make_prompts(TINY.vocab, 3, 10, seed=12)
    cb = dec.new_cache(3, 64)
    lb = dec.prefill(cb, tokens)
    sb = dec.step(cb, np.array([5, 6, 7]))
    for b in range(3):
        c = dec.new_cache(1, 64)
        np.testing.assert_allclose(dec.prefill(c, tokens[b:b + 1]), lb[b:b + 1], atol=1e-12, rtol=0)
        np.testing.assert_allclose(dec.step(c, np.array([5 + b])), sb[b:b + 1], atol=1e-12, rtol=0)


def test_paged_cache_equals_contiguous_bit_exact(tiny_weights):
    dec = oracle.Decoder(TINY, tiny_weights)
    tokens = synth.make_prompts(TINY.vocab, 2, 40, seed=13)
    contiguous = dec.new_cache(2, 128, page_tokens=128)
    perm = np.random.default_rng(5).permutation(2 * 8).reshape(2, 8)
    paged = dec.new_cache(2, 128, page_tokens=16, block_table=perm)
    a = dec.prefill(contiguous, tokens)
    b = dec.prefill(paged, tokens)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(dec.step(contiguous, tokens[:, 0]), dec.step(paged, tokens[:, 0]))


def test_kv_cache_values_are_bf16(tiny_weights):
    dec = oracle.Decoder(TINY, tiny_weights)
    c = dec.new_cache(1, 64)
    dec.prefill(c, synth.make_prompts(TINY.vocab, 1, 5, seed=2))
    k, v = c.read(0, 0, 5)
    np.testing.assert_array_equal(oracle.round_bf16(k), k)
    np.testing.assert_array_equal(oracle.round_bf16(v), v)


def test_context_limit_is_enforced(tiny_weights):
    dec = oracle.Decoder(TINY, tiny_weights)
    c = dec.new_cache(1, 4, page_tokens=4)
    with pytest.raises(ValueError):
        dec.prefill(c, np.zeros((1, 5), dtype=np.int32))


# --------------------------------------------------------- two-stage model --
def _small_two_stage():
    bb = synth.ModelShape(n_layers=1, hidden=128, n_heads=2, n_kv_heads=1, head_dim=64, ffn=256, vocab=300)
    hd = synth.ModelShape(n_layers=1, hidden=64, n_heads=2, n_kv_heads=1, head_dim=32, ffn=128, vocab=50,
                          tied_embedding=False)
    return synth.TwoStageShape(backbone=bb, head=hd, n_codebooks=4, codebook_vocab=50)


def test_two_stage_teacher_forcing_with_own_codes_is_identity():
    s = _small_two_stage()
    w = synth.make_weights(s, seed=0)
    ts = oracle.TwoStage(s, w)
    prompts = synth.make_prompts(300, 2, 6, seed=4)
    c1 = ts.backbone.new_cache(2, 16)
    codes, logits = ts.prefill(c1, prompts)
    c2 = ts.backbone.new_cache(2, 16)
    codes_f, logits_f = ts.prefill(c2, prompts, forced=codes)
    np.testing.assert_array_equal(codes, codes_f)
    np.testing.assert_array_equal(logits, logits_f)
    assert codes.shape == (2, 4) and codes.max() < 50
    nxt, _ = ts.frame(c1, codes)
    assert c1.length.tolist() == [7, 7] and nxt.shape == (2, 4)


def test_two_stage_head_position0_reads_projected_state():
    # With one codebook the head's output depends on the backbone state only through W_proj.
    s = _small_two_stage()
    w = synth.make_weights(s, seed=0)
    ts = oracle.TwoStage(s, w)
    h = RNG.standard_normal((1, 128))
    c_a, l_a = ts.head_frame(h)
    ts.proj = np.zeros_like(ts.proj)
    c_b, l_b = ts.head_frame(h)
    assert not np.allclose(l_a[:, 0], l_b[:, 0])



# ---- the two-stage model against transformers' Llama run on input vectors ----
def _hf_llama_body(shape, weights, prefix):
    """transformers' LlamaModel in float64 carrying one decoder's layers and
    final norm; it is driven through inputs_embeds, so its own embedding
    table is never read."""
    import torch
    from transformers import LlamaConfig, LlamaModel

    cfg = LlamaConfig(vocab_size=8, hidden_size=shape.hidden, intermediate_size=shape.ffn,
                      num_hidden_layers=shape.n_layers, num_attention_heads=shape.n_heads,
                      num_key_value_heads=shape.n_kv_heads, head_dim=shape.head_dim, rms_norm_eps=shape.rms_eps,
                      rope_theta=shape.rope_theta, max_position_embeddings=4096, attention_bias=False,
                      mlp_bias=False)
    m = LlamaModel(cfg).double().eval()
    f = lambda n: torch.from_numpy(oracle.bf16_to_f64(weights[prefix + n]))
    names = {"norm.weight": "final_norm"}
    for l in range(shape.n_layers):
        p, q = f"layers.{l}.", f"layers.{l}."
        names.update({p + "self_attn.q_proj.weight": q + "wq", p + "self_attn.k_proj.weight": q + "wk",
                      p + "self_attn.v_proj.weight": q + "wv", p + "self_attn.o_proj.weight": q + "wo",
                      p + "mlp.gate_proj.weight": q + "w_gate", p + "mlp.up_proj.weight": q + "w_up",
                      p + "mlp.down_proj.weight": q + "w_down", p + "input_layernorm.weight": q + "attn_norm",
                      p + "post_attention_layernorm.weight": q + "ffn_norm"})
    sd = m.state_dict()
    with torch.no_grad():
        for hf, ours in names.items():
            sd[hf].copy_(f(ours))
    return m


def _hf_two_stage_logits(s, weights, prompts, frame_codes):
    """Per-frame head logits [B][K][V] from two transformers models.

    The backbone runs once over the prompt's embeddings followed by each
    frame's input sum_k frame_embed_k[c_k] (frame f's state is at position
    T - 1 + f).  For every frame the head runs from position 0 on
    [W_proj . state, head_embed_1[c_0], ..., head_embed_(K-1)[c_(K-2)]]."""
    import torch

    f64 = lambda n: oracle.bf16_to_f64(weights[n])
    K = s.n_codebooks
    B, T = prompts.shape
    seq = [f64("backbone.embed")[prompts]]
    for codes in frame_codes[:-1]:
        seq.append(sum(f64(f"frame_embed.{k}")[codes[:, k]] for k in range(K))[:, None, :])
    bb = _hf_llama_body(s.backbone, weights, "backbone.")
    hd = _hf_llama_body(s.head, weights, "head.")
    with torch.no_grad():
        hid = bb(inputs_embeds=torch.from_numpy(np.concatenate(seq, axis=1))).last_hidden_state.numpy()
        out = []
        for f, codes in enumerate(frame_codes):
            xs = [hid[:, T - 1 + f] @ f64("proj").T]
            xs += [f64(f"head_embed.{k}")[codes[:, k - 1]] for k in range(1, K)]
            y = hd(inputs_embeds=torch.from_numpy(np.stack(xs, axis=1))).last_hidden_state.numpy()
            out.append(np.stack([y[:, k] @ f64(f"out_head.{k}").T for k in range(K)], axis=1))
    return out


def _oracle_two_stage_frames(ts, prompts, n_frames):
    cache = ts.backbone.new_cache(prompts.shape[0], prompts.shape[1] + n_frames)
    codes, lg = ts.prefill(cache, prompts)
    out = [(codes, lg)]
    for _ in range(n_frames - 1):
        codes, lg = ts.frame(cache, codes)
        out.append((codes, lg))
    return out


@pytest.fixture(scope="module")
def two_stage_case():
    s = synth.TINY_TWO_STAGE
    return s, synth.make_weights(s, seed=0), synth.make_prompts(s.backbone.vocab, 2, 6, seed=5)


def test_two_stage_matches_transformers_llama_fp64(two_stage_case):
    """The oracle's two-stage composition (projection, head inputs, per-frame
    head cache, output heads, next-frame input) against an independent build
    of the same definition from transformers' float64 Llama."""
    s, w, prompts = two_stage_case
    ours = _oracle_two_stage_frames(oracle.TwoStage(s, w, round_kv=False), prompts, 3)
    ref = _hf_two_stage_logits(s, w, prompts, [c for c, _ in ours])
    for f, ((codes, lg), r) in enumerate(zip(ours, ref)):
        np.testing.assert_allclose(lg, r, atol=2e-6, rtol=0, err_msg=f"frame {f}")
        assert (codes == oracle.argmax_lowest(r.reshape(-1, r.shape[-1])).reshape(codes.shape)).all()


class _HeadCacheKept(oracle.TwoStage):
    """Planted slip: the head's cache runs on across frames."""

    def head_frame(self, h, forced=None):
        kept = getattr(self, "_kept", None)
        orig = self.head.new_cache
        if kept is None:
            kept = self._kept = orig(h.shape[0], 4 * self.s.n_codebooks, page_tokens=self.s.n_codebooks)
        self.head.new_cache = lambda *a, **k: kept
        try:
            return super().head_frame(h, forced)
        finally:
            self.head.new_cache = orig


class _HeadTableShifted(oracle.TwoStage):
    """Planted slip: head step k looks code c_(k-1) up in the table of step
    k + 1 (the last step wraps to table 1)."""

    def __init__(self, *a, **k):
        super().__init__(*a, **k)
        self.head_embed = [None] + self.head_embed[2:] + [self.head_embed[1]]


class _FrameInputFirstCode(oracle.TwoStage):
    """Planted slip: the next frame's input is frame_embed_0[c_0] alone."""

    def frame(self, cache, prev_codes, forced=None):
        x = self.frame_embed[0][np.asarray(prev_codes[:, 0], dtype=np.int64)]
        hid = self.backbone.forward_hidden(cache, x[:, None, :])
        return self.head_frame(hid[:, 0, :], forced)


@pytest.mark.parametrize("cls", [_HeadCacheKept, _HeadTableShifted, _FrameInputFirstCode])
def test_planted_two_stage_slips_are_caught(two_stage_case, cls):
    s, w, prompts = two_stage_case
    ours = _oracle_two_stage_frames(cls(s, w, round_kv=False), prompts, 3)
    ref = _hf_two_stage_logits(s, w, prompts, [c for c, _ in ours])
    assert max(np.max(np.abs(lg - r)) for (_, lg), r in zip(ours, ref)) > 1e-3


def test_oracle_matches_its_regression_fixture():
    """The oracle still computes what tests/golden/make_golden.py recorded
    (a regression guard on the oracle's arithmetic; the outside pins are the
    tests above)."""
    import importlib.util
    import json
    import os

    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(here, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(os.path.join(here, "oracle_regression.json")) as f:
        want = json.load(f)
    got = {"decoder": mg.decoder_case(), "two_stage": mg.two_stage_case()}
    for a, b in zip(want["decoder"]["steps"], got["decoder"]["steps"]):
        assert a["tokens"] == b["tokens"], a["step"]
        np.testing.assert_allclose(b["logits_sample"], a["logits_sample"], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(b["logsumexp"], a["logsumexp"], rtol=1e-9, atol=1e-12)
    for a, b in zip(want["two_stage"]["frames"], got["two_stage"]["frames"]):
        assert a["codes"] == b["codes"], a["frame"]
        np.testing.assert_allclose(b["logits_k0_sample"], a["logits_k0_sample"], rtol=1e-9, atol=1e-12)
