"""Plain float64 forward pass of a Llama-style decoder (TEST INFRASTRUCTURE ONLY).

What is computed, and where it comes from:

* The unit of work is one recurring model update: a decode step that consumes
  one token per sequence and advances resident state (the attention cache),
  and the prompt prefill that produces the first token ("Why real-time
  inference wants a megakernel", section "Real time changes the objective";
  "Persistent threads and megakernels", section 3, Figs. 2-3: one token, batch
  one).  The model family is Llama 3.2 1B with a 496-token prompt ("One
  Megakernel is Not Enough", Table III).
* The decode step reads the key/value cache of earlier tokens ("Persistent
  threads and megakernels", section 6).  The pages print no forward-pass
  formula, so the standard Llama definition is written out here, with the
  readings below.

Readings taken where the pages are silent:
  RMSNorm  a = x / sqrt(mean(x^2) + eps) * g            (no bias, no scale on x)
  RoPE     rotate-half pairs (i, i + d/2), inv_i = theta^(-2i/d), 0-based
           positions, no frequency scaling
  GQA      q-head h reads kv-head h // (n_heads / n_kv_heads)
  attention scores q.k / sqrt(d), causal including the current token,
           softmax with max subtraction
  KV cache keys (after RoPE) and values are rounded to bf16 (RNE) when stored
  FFN      down(silu(gate(f)) * up(f)), silu(z) = z / (1 + e^-z)
  head     logits = E . RMSNorm(x; g_final) with the tied embedding E
  argmax   lowest index wins ties
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# bf16 <-> float64
# ----------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits.  For x = m * 2^E with m in [0.5, 1) the bf16
    spacing is 2^(E-8); below the smallest normal (2^-126) the spacing stays
    2^-133.  Scaling by a power of two is exact, and np.rint rounds half to
    even, so the result is the correctly rounded bf16 value (finite inputs in
    bf16 range).
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.rint(x / q) * q


# ----------------------------------------------------------------------------
# Primitives
# ----------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """inv_i = theta^(-2i/d) for i in [0, d/2)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-(2.0 * i) / head_dim)


def rope_apply(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE.

    x: [..., T, H, d]; pos: [..., T] integer positions.  Pair (i, i + d/2) at
    position p is rotated by the angle p * inv_i:
        (x_i, x_{i+d/2}) -> (x_i cos - x_{i+d/2} sin, x_{i+d/2} cos + x_i sin)
    """
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, theta)  # [..., T, d/2]
    c = np.cos(ang)[..., None, :]
    s = np.sin(ang)[..., None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray,
              k_pos: np.ndarray) -> np.ndarray:
    """Causal grouped-query attention for one sequence.

    q: [Tq, Hq, d], k/v: [Tk, Hkv, d]; q_pos [Tq], k_pos [Tk].  Query at
    position p attends to keys with position <= p.  Returns [Tq, Hq, d].
    """
    tq, hq, d = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(d)
    mask = k_pos[None, :] <= q_pos[:, None]                        # [Tq, Tk]
    for h in range(hq):
        g = h // group
        s = (q[:, h, :] @ k[:, g, :].T) * scale                    # [Tq, Tk]
        s = np.where(mask, s, -np.inf)
        out[:, h, :] = softmax(s, axis=-1) @ v[:, g, :]
    return out


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Index of the maximum along the last axis; the lowest index wins ties."""
    return np.argmax(logits, axis=-1).astype(np.int32)


# ----------------------------------------------------------------------------
# Paged KV cache
# ----------------------------------------------------------------------------

class KVCache:
    """Keys/values per layer in fixed-size pages addressed through a block table.

    k_pool/v_pool: [n_layers][n_blocks][page_tokens][n_kv_heads][d] float64
    block_table:   [batch][max_blocks] page ids; sequence b's token t lives in
                   page block_table[b][t // page_tokens], row t % page_tokens.
    A single page of max_context tokens per sequence is the contiguous layout.
    """

    def __init__(self, n_layers: int, batch: int, max_context: int, n_kv_heads: int,
                 head_dim: int, page_tokens: int = 64,
                 block_table: Optional[np.ndarray] = None):
        self.page = page_tokens
        self.max_blocks = -(-max_context // page_tokens)
        if block_table is None:
            block_table = np.arange(batch * self.max_blocks, dtype=np.int64).reshape(batch, self.max_blocks)
        self.block_table = np.asarray(block_table, dtype=np.int64)
        n_blocks = int(self.block_table.max()) + 1
        shape = (n_layers, n_blocks, page_tokens, n_kv_heads, head_dim)
        self.k_pool = np.zeros(shape)
        self.v_pool = np.zeros(shape)
        self.length = np.zeros(batch, dtype=np.int64)   # tokens stored per sequence
        self.max_context = max_context

    def write(self, layer: int, b: int, positions: np.ndarray, k: np.ndarray, v: np.ndarray) -> None:
        for i, t in enumerate(positions):
            if t >= self.max_context:
                raise ValueError("context limit exceeded")
            blk = self.block_table[b, t // self.page]
            self.k_pool[layer, blk, t % self.page] = k[i]
            self.v_pool[layer, blk, t % self.page] = v[i]

    def read(self, layer: int, b: int, n: int):
        t = np.arange(n)
        blk = self.block_table[b, t // self.page]
        return self.k_pool[layer, blk, t % self.page], self.v_pool[layer, blk, t % self.page]


# ----------------------------------------------------------------------------
# Decoder
# ----------------------------------------------------------------------------

class Decoder:
    """A Llama-style decoder over bf16 weights held as float64.

    ``weights`` maps names (see ``synth.decoder_tensor_specs``) to bf16 bit
    patterns; matmul weights are [out][in].  ``prefix`` selects a sub-model.
    """

    def __init__(self, shape, weights: Dict[str, np.ndarray], prefix: str = "",
                 round_kv: bool = True, with_embed: bool = True):
        self.s = shape
        self.round_kv = round_kv
        w = lambda n: bf16_to_f64(weights[prefix + n])
        self.embed = w("embed") if with_embed else None
        self.layers = []
        for l in range(shape.n_layers):
            p = f"layers.{l}."
            self.layers.append({n: w(p + n) for n in
                                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")})
        self.final_norm = w("final_norm")
        if with_embed:
            self.lm_head = self.embed if shape.tied_embedding else w("lm_head")

    def new_cache(self, batch: int, max_context: int, page_tokens: int = 64,
                  block_table: Optional[np.ndarray] = None) -> KVCache:
        return KVCache(self.s.n_layers, batch, max_context, self.s.n_kv_heads, self.s.head_dim,
                       page_tokens, block_table)

    # -- one layer over T new tokens per sequence --------------------------------
    def _layer(self, l: int, x: np.ndarray, cache: KVCache, pos0: np.ndarray) -> np.ndarray:
        s, W = self.s, self.layers[l]
        B, T, _ = x.shape
        a = rmsnorm(x, W["attn_norm"], s.rms_eps)
        q = (a @ W["wq"].T).reshape(B, T, s.n_heads, s.head_dim)
        k = (a @ W["wk"].T).reshape(B, T, s.n_kv_heads, s.head_dim)
        v = (a @ W["wv"].T).reshape(B, T, s.n_kv_heads, s.head_dim)
        o = np.empty((B, T, s.n_heads, s.head_dim))
        for b in range(B):
            qpos = pos0[b] + np.arange(T)
            qb = rope_apply(q[b], qpos, s.rope_theta)
            kb = rope_apply(k[b], qpos, s.rope_theta)
            vb = v[b]
            if self.round_kv:
                kb, vb = round_bf16(kb), round_bf16(vb)
            cache.write(l, b, qpos, kb, vb)
            n = pos0[b] + T
            K, V = cache.read(l, b, n)
            o[b] = attention(qb, K, V, qpos, np.arange(n))
        x = x + o.reshape(B, T, -1) @ W["wo"].T
        f = rmsnorm(x, W["ffn_norm"], s.rms_eps)
        hdn = silu(f @ W["w_gate"].T) * (f @ W["w_up"].T)
        return x + hdn @ W["w_down"].T

    def forward_hidden(self, cache: KVCache, x: np.ndarray) -> np.ndarray:
        """Run all layers over new inputs x [B][T][hidden] at the cache's next
        positions; returns the final-normed hidden state [B][T][hidden]."""
        B, T, _ = x.shape
        pos0 = cache.length[:B].copy()
        for l in range(self.s.n_layers):
            x = self._layer(l, x, cache, pos0)
        cache.length[:B] = pos0 + T
        return rmsnorm(x, self.final_norm, self.s.rms_eps)

    def embed_tokens(self, tokens: np.ndarray) -> np.ndarray:
        return self.embed[np.asarray(tokens, dtype=np.int64)]

    def prefill(self, cache: KVCache, tokens: np.ndarray) -> np.ndarray:
        """Prompt prefill: tokens [B][T] -> logits at the last prompt position [B][V]."""
        hid = self.forward_hidden(cache, self.embed_tokens(tokens))
        return hid[:, -1, :] @ self.lm_head.T

    def step(self, cache: KVCache, tokens: np.ndarray) -> np.ndarray:
        """One decode step: tokens [B] (one per sequence) -> logits [B][V]."""
        hid = self.forward_hidden(cache, self.embed_tokens(np.asarray(tokens)[:, None]))
        return hid[:, 0, :] @ self.lm_head.T


# ----------------------------------------------------------------------------
# Two-stage streaming model (backbone + codebook head)
# ----------------------------------------------------------------------------

class TwoStage:
    """Backbone decoder feeding a small decoder that emits one token per codebook.

    Per frame and sequence: h = RMSNorm(backbone state; g_final);
    p = W_proj . h; head position 0 reads p, head position k (1..K-1) reads
    head_embed_k[c_{k-1}]; c_k = argmax(out_head_k . RMSNorm(y_k; g_head_final)).
    The head's cache restarts every frame.  The next backbone input is
    sum_k frame_embed_k[c_k].  This composition is this repository's reading of
    a two-stage streaming model (the pages name such models but print none).
    The tests check this implementation of it against one assembled from
    transformers' Llama layers.
    """

    def __init__(self, shape, weights: Dict[str, np.ndarray], round_kv: bool = True):
        self.s = shape
        self.backbone = Decoder(shape.backbone, weights, "backbone.", round_kv)
        self.head = Decoder(shape.head, weights, "head.", round_kv, with_embed=False)
        self.proj = bf16_to_f64(weights["proj"])
        self.head_embed = [None] + [bf16_to_f64(weights[f"head_embed.{k}"]) for k in range(1, shape.n_codebooks)]
        self.out_head = [bf16_to_f64(weights[f"out_head.{k}"]) for k in range(shape.n_codebooks)]
        self.frame_embed = [bf16_to_f64(weights[f"frame_embed.{k}"]) for k in range(shape.n_codebooks)]

    def head_frame(self, h: np.ndarray, forced: Optional[np.ndarray] = None):
        """h [B][backbone hidden] -> (codes [B][K], logits [B][K][codebook_vocab]).

        With ``forced`` [B][K], the head is conditioned on those codes instead
        of its own argmax (teacher forcing); the returned codes are still the
        oracle's own argmax."""
        s = self.s
        B = h.shape[0]
        cache = self.head.new_cache(B, s.n_codebooks, page_tokens=s.n_codebooks)
        codes = np.zeros((B, s.n_codebooks), dtype=np.int32)
        logits = np.zeros((B, s.n_codebooks, s.codebook_vocab))
        x = h @ self.proj.T
        for k in range(s.n_codebooks):
            if k > 0:
                prev = forced[:, k - 1] if forced is not None else codes[:, k - 1]
                x = self.head_embed[k][np.asarray(prev, dtype=np.int64)]
            y = self.head.forward_hidden(cache, x[:, None, :])[:, 0, :]
            logits[:, k] = y @ self.out_head[k].T
            codes[:, k] = argmax_lowest(logits[:, k])
        return codes, logits

    def prefill(self, cache: KVCache, tokens: np.ndarray, forced=None):
        hid = self.backbone.forward_hidden(cache, self.backbone.embed_tokens(tokens))
        return self.head_frame(hid[:, -1, :], forced)

    def frame(self, cache: KVCache, prev_codes: np.ndarray, forced=None):
        x = sum(self.frame_embed[k][np.asarray(prev_codes[:, k], dtype=np.int64)]
                for k in range(self.s.n_codebooks))
        hid = self.backbone.forward_hidden(cache, x[:, None, :])
        return self.head_frame(hid[:, 0, :], forced)
