"""Seeded synthetic inputs for the Llama-style decoder workloads.

This module only draws numbers: random-init bf16 weights and uniform random
prompt ids.  It holds none of the model's arithmetic, so both the CPU oracle
(``oracle/``) and the CUDA path can be fed from it without sharing any code.

Workload shapes follow the recurring-update workloads of the pages: a tiny
Llama-style decoder, a Llama-3.2-1B-shaped decoder (the 496-token prompt is the
Llama 3.2 1B evaluation shape of "One Megakernel is Not Enough", Table III) and
a two-stage streaming model (backbone + codebook head) standing in for the
streaming TTS models of the same paper.

Weight recipe: every matmul weight and embedding is drawn N(0, 0.02) in fp32
and rounded to bf16 (round-to-nearest-even, done by torch's dtype conversion);
RMSNorm gains are 1.0.  Each tensor gets its own child of
``numpy.random.SeedSequence(seed)``, spawned in the fixed name order that
``tensor_specs`` returns, so a tensor's values do not depend on which other
tensors are generated.  Prompts are uniform ids in [0, vocab) from a separate
seed, one row per sequence.
"""
from __future__ import annotations

import concurrent.futures as _fut
import os
from dataclasses import dataclass, field, asdict
from typing import Dict, List, Optional, Tuple

import numpy as np

BF16_ONE = np.uint16(0x3F80)
INIT_STD = 0.02


@dataclass(frozen=True)
class ModelShape:
    """Shape of a Llama-style decoder (no biases, tied or untied embedding)."""

    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    tied_embedding: bool = True

    def as_dict(self) -> dict:
        return asdict(self)


@dataclass(frozen=True)
class TwoStageShape:
    """Backbone decoder + codebook head decoder (the two-stage streaming model)."""

    backbone: ModelShape
    head: ModelShape
    n_codebooks: int = 16
    codebook_vocab: int = 2048


TINY = ModelShape(n_layers=2, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64,
                  ffn=704, vocab=1024, rms_eps=1e-5, rope_theta=10000.0)
LLAMA_1B = ModelShape(n_layers=16, hidden=2048, n_heads=32, n_kv_heads=8, head_dim=64,
                      ffn=8192, vocab=128256, rms_eps=1e-5, rope_theta=500000.0)
# The codebook head: 4 layers, hidden 1024, 16 q heads / 4 kv heads, FFN 4096.
# Its "vocab" field is the codebook vocabulary; it has no token embedding of
# its own (inputs are the projected backbone state or a codebook embedding).
CODEBOOK_HEAD = ModelShape(n_layers=4, hidden=1024, n_heads=16, n_kv_heads=4, head_dim=64,
                           ffn=4096, vocab=2048, rms_eps=1e-5, rope_theta=500000.0,
                           tied_embedding=False)
TWO_STAGE = TwoStageShape(backbone=LLAMA_1B, head=CODEBOOK_HEAD)
# a small two-stage model for parity tests: the tiny backbone, a 2-layer head
TINY_HEAD = ModelShape(n_layers=2, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=512, vocab=256,
                       rms_eps=1e-5, rope_theta=10000.0, tied_embedding=False)
TINY_TWO_STAGE = TwoStageShape(backbone=TINY, head=TINY_HEAD, n_codebooks=4, codebook_vocab=256)


@dataclass(frozen=True)
class Workload:
    name: str
    model: object
    batch: int
    prompt_len: int
    steps: int
    prompt_seed: int


# The five workloads (weights seed 0; prompt seed 1000 + workload index).
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", TINY, 1, 32, 16, 1000),
    "llama1b_b1": Workload("llama1b_b1", LLAMA_1B, 1, 496, 128, 1001),
    "llama1b_decode_b16": Workload("llama1b_decode_b16", LLAMA_1B, 16, 496, 128, 1002),
    "llama1b_decode_b32": Workload("llama1b_decode_b32", LLAMA_1B, 32, 496, 128, 1002),
    "llama1b_decode_b48": Workload("llama1b_decode_b48", LLAMA_1B, 48, 496, 128, 1002),
    "llama1b_prefill_b1": Workload("llama1b_prefill_b1", LLAMA_1B, 1, 496, 0, 1003),
    "llama1b_prefill_b16": Workload("llama1b_prefill_b16", LLAMA_1B, 16, 496, 0, 1003),
    "llama1b_prefill_b32": Workload("llama1b_prefill_b32", LLAMA_1B, 32, 496, 0, 1003),
    "two_stage_b32": Workload("two_stage_b32", TWO_STAGE, 32, 200, 64, 1004),
}


def decoder_tensor_specs(m: ModelShape, prefix: str = "", with_embed: bool = True,
                         with_final_norm: bool = True) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, kind) for every tensor of a decoder, in generation order.

    Matmul weights are stored [out_features][in_features]; kind is "normal"
    (N(0, 0.02) -> bf16) or "ones" (RMSNorm gain 1.0).
    """
    h, q, kv = m.hidden, m.n_heads * m.head_dim, m.n_kv_heads * m.head_dim
    specs: List[Tuple[str, Tuple[int, ...], str]] = []
    if with_embed:
        specs.append((prefix + "embed", (m.vocab, h), "normal"))
    for l in range(m.n_layers):
        p = f"{prefix}layers.{l}."
        specs += [
            (p + "attn_norm", (h,), "ones"),
            (p + "wq", (q, h), "normal"),
            (p + "wk", (kv, h), "normal"),
            (p + "wv", (kv, h), "normal"),
            (p + "wo", (h, q), "normal"),
            (p + "ffn_norm", (h,), "ones"),
            (p + "w_gate", (m.ffn, h), "normal"),
            (p + "w_up", (m.ffn, h), "normal"),
            (p + "w_down", (h, m.ffn), "normal"),
        ]
    if with_final_norm:
        specs.append((prefix + "final_norm", (h,), "ones"))
    if with_embed and not m.tied_embedding:
        specs.append((prefix + "lm_head", (m.vocab, h), "normal"))
    return specs


def tensor_specs(model) -> List[Tuple[str, Tuple[int, ...], str]]:
    if isinstance(model, ModelShape):
        return decoder_tensor_specs(model)
    assert isinstance(model, TwoStageShape)
    bb, hd = model.backbone, model.head
    specs = decoder_tensor_specs(bb, "backbone.")
    specs.append(("proj", (hd.hidden, bb.hidden), "normal"))          # backbone -> head
    for k in range(1, model.n_codebooks):                               # previous-codebook inputs
        specs.append((f"head_embed.{k}", (model.codebook_vocab, hd.hidden), "normal"))
    specs += decoder_tensor_specs(hd, "head.", with_embed=False)
    for k in range(model.n_codebooks):                                  # one output head per codebook
        specs.append((f"out_head.{k}", (model.codebook_vocab, hd.hidden), "normal"))
    for k in range(model.n_codebooks):                                  # next-frame backbone input
        specs.append((f"frame_embed.{k}", (model.codebook_vocab, bb.hidden), "normal"))
    return specs


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _draw(seed_seq: np.random.SeedSequence, shape, kind) -> np.ndarray:
    if kind == "ones":
        return np.full(shape, BF16_ONE, dtype=np.uint16)
    rng = np.random.default_rng(seed_seq)
    a = rng.standard_normal(int(np.prod(shape)), dtype=np.float32)
    a *= np.float32(INIT_STD)
    return _to_bf16_bits(a).reshape(shape)


def make_weights(model, seed: int = 0, threads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """All tensors of ``model`` as bf16 bit patterns (``np.uint16``), by name."""
    specs = tensor_specs(model)
    children = np.random.SeedSequence(seed).spawn(len(specs))
    threads = threads or min(8, os.cpu_count() or 1)
    out: Dict[str, np.ndarray] = {}
    with _fut.ThreadPoolExecutor(threads) as ex:
        futs = {ex.submit(_draw, c, shp, kind): name for (name, shp, kind), c in zip(specs, children)}
        for f, name in futs.items():
            out[name] = f.result()
    return {name: out[name] for name, _, _ in specs}


def make_prompts(vocab: int, batch: int, length: int, seed: int) -> np.ndarray:
    """Uniform random token ids in [0, vocab), shape [batch][length], int32."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=(batch, length), dtype=np.int64).astype(np.int32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a bit shift, no rounding)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


_CACHE_DIR_ENV = "WPK_WEIGHT_CACHE"


def cached_weights(model, seed: int = 0) -> Dict[str, np.ndarray]:
    """``make_weights`` with an optional on-disk cache (directory in $WPK_WEIGHT_CACHE)."""
    d = os.environ.get(_CACHE_DIR_ENV)
    if not d:
        return make_weights(model, seed)
    import hashlib

    digest = hashlib.sha1(repr(model).encode()).hexdigest()[:12]
    key = f"{type(model).__name__}_{digest}_s{seed}.npz"
    path = os.path.join(d, key)
    if os.path.exists(path):
        with np.load(path) as z:
            return {k: z[k] for k in z.files}
    w = make_weights(model, seed)
    os.makedirs(d, exist_ok=True)
    np.savez(path + ".tmp.npz", **w)
    os.replace(path + ".tmp.npz", path)
    return w
