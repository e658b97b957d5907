"""ctypes binding of ``libwpk.so`` with the same entry-point names as ``include/wpk.h``.

Argument marshalling only: every step of the decode/prefill path runs in the
library's CUDA kernels.  Loading fails loudly when the library is missing;
there is no fallback.  ``Engine`` adds torch-owned device buffers around a
handle (PyTorch is used for device memory and streams only).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwpk.so")

WPK_OK = 0
WPK_ERR_INVALID_ARG = -1
WPK_ERR_CUDA = -2
WPK_ERR_TIMEOUT = -3
WPK_ERR_NOT_LOADED = -4
WPK_ERR_SHAPE = -5
WPK_ERR_UNSUPPORTED = -6
WPK_ERR_POISONED = -7
WPK_MEGAKERNEL = 0
WPK_PER_OP_GRAPH = 1
WPK_SCHED_QUEUE = 0
WPK_SCHED_STATIC = 1
WPK_SCHED_TEAMS = 2
WPK_PREFILL_AUTO = 0
WPK_PREFILL_MMA = 1
WPK_PREFILL_TOKENWISE = 2
WPK_DECODE_AUTO = 0
WPK_DECODE_GEMV = 1
WPK_DECODE_MMA = 2

OP_NAMES = ["embed", "qkv", "attn", "o", "gate_up", "down", "lm_head", "final",
            "p_embed", "norm", "mma_qkv", "mma_o", "mma_gate_up", "mma_down", "p_attn", "gather",
            "b_qkv", "b_o", "b_gate_up", "b_down", "b_lm_head"]

_ERR_NAMES = {0: "OK", -1: "INVALID_ARG", -2: "CUDA", -3: "TIMEOUT", -4: "NOT_LOADED", -5: "SHAPE",
              -6: "UNSUPPORTED", -7: "POISONED"}


class WpkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"wpk error {code} ({_ERR_NAMES.get(code, '?')}): {msg}")
        self.code = code


class wpk_model_cfg(C.Structure):
    pass


wpk_model_cfg._fields_ = [("n_layers", C.c_int), ("hidden", C.c_int), ("n_heads", C.c_int), ("n_kv_heads", C.c_int),
                          ("head_dim", C.c_int), ("ffn", C.c_int), ("vocab", C.c_int), ("rms_eps", C.c_float),
                          ("rope_theta", C.c_float), ("tied_embedding", C.c_int), ("n_codebooks", C.c_int),
                          ("codebook_vocab", C.c_int), ("head", C.POINTER(wpk_model_cfg))]


class wpk_plan_cfg(C.Structure):
    _fields_ = [("max_batch", C.c_int), ("max_context", C.c_int), ("page_tokens", C.c_int),
                ("n_workers", C.c_int), ("workers_per_sm", C.c_int), ("mode", C.c_int), ("resident", C.c_int),
                ("n_regions", C.c_int), ("region_cut", C.c_int * 4), ("trace", C.c_int),
                ("wait_timeout_ns", C.c_uint64), ("slot_bytes", C.c_int), ("tile_bytes", C.c_int),
                ("split_pages", C.c_int), ("lookahead", C.c_int), ("schedule", C.c_int), ("prefill", C.c_int),
                ("decode", C.c_int), ("frame_chunks", C.c_int), ("head_workers", C.c_int)]


_P16 = C.POINTER(C.c_uint16)


class wpk_layer_weights(C.Structure):
    _fields_ = [(n, _P16) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")]


class wpk_weights(C.Structure):
    _fields_ = [("embed", _P16), ("final_norm", _P16), ("lm_head", _P16), ("layers", C.POINTER(wpk_layer_weights)),
                ("proj", _P16), ("frame_embed", C.POINTER(_P16)), ("head_embed", C.POINTER(_P16)),
                ("out_head", C.POINTER(_P16)), ("head_layers", C.POINTER(wpk_layer_weights)),
                ("head_final_norm", _P16)]


class wpk_graph_stats(C.Structure):
    _fields_ = [("n_tiles", C.c_int64), ("n_counters", C.c_int64), ("n_edges", C.c_int64),
                ("n_signals", C.c_int64), ("n_ops", C.c_int64), ("n_workers", C.c_int64),
                ("weight_bytes", C.c_int64), ("region_begin", C.c_int64 * 5), ("n_regions", C.c_int64)]


class wpk_predict_cfg(C.Structure):
    _fields_ = [("mode", C.c_int), ("n_regions", C.c_int), ("region_cut", C.c_int * 4), ("n_workers", C.c_int),
                ("n_sms", C.c_int), ("schedule", C.c_int), ("slots", C.c_int), ("dispatch_ns", C.c_double),
                ("sync_ns", C.c_double), ("first_chunk_ns", C.c_double)]


class wpk_error_info(C.Structure):
    _fields_ = [("code", C.c_int32), ("tile", C.c_uint32), ("counter", C.c_uint32), ("epoch", C.c_uint32),
                ("observed", C.c_uint32), ("target", C.c_uint32)]


TRACE_DTYPE = np.dtype([("tile", "<u4"), ("worker", "<u2"), ("op", "<u2"), ("ev_issue", "<u4"),
                        ("ev_start", "<u4"), ("ev_done", "<u4"), ("epoch", "<u4"), ("t_claim_ns", "<u8"),
                        ("t_issued_ns", "<u8"), ("t_start_ns", "<u8"), ("t_data_ns", "<u8"), ("t_end_ns", "<u8")])
assert TRACE_DTYPE.itemsize == 64

# Every symbol include/wpk.h declares, with its ctypes signature.
_H = C.c_void_p
_SIGS = {
    "wpk_build_graph": (C.c_int, [C.POINTER(wpk_model_cfg), C.POINTER(wpk_plan_cfg), C.POINTER(_H)]),
    "wpk_workspace_size": (C.c_int, [_H, C.POINTER(C.c_size_t), C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)]),
    "wpk_load_weights": (C.c_int, [_H, C.POINTER(wpk_weights), C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "wpk_set_block_table": (C.c_int, [_H, C.POINTER(C.c_int32)]),
    "wpk_prefill": (C.c_int, [_H, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    "wpk_step": (C.c_int, [_H, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "wpk_graph_stats_get": (C.c_int, [_H, C.POINTER(wpk_graph_stats)]),
    "wpk_select_program": (C.c_int, [_H, C.c_int, C.c_int]),
    "wpk_get_edges": (C.c_int, [_H, C.POINTER(C.c_int32), C.c_int64, C.POINTER(C.c_int64)]),
    "wpk_get_tile_ops": (C.c_int, [_H, C.POINTER(C.c_int32), C.c_int64]),
    "wpk_verify_graph": (C.c_int, [_H]),
    "wpk_simulate": (C.c_int, [_H, C.c_int, C.c_int, C.c_uint64, C.c_int, C.c_int, C.POINTER(C.c_int32)]),
    "wpk_get_tile_bytes": (C.c_int, [_H, C.POINTER(C.c_int64), C.c_int64]),
    "wpk_prefill_slots": (C.c_int, [_H, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    "wpk_set_active_slots": (C.c_int, [_H, C.POINTER(C.c_int32), C.c_int]),
    "wpk_predict": (C.c_int, [_H, C.POINTER(C.c_double), C.POINTER(C.c_double), C.POINTER(wpk_predict_cfg),
                              C.POINTER(C.c_double)]),
    "wpk_get_trace": (C.c_int, [_H, C.c_void_p, C.c_size_t]),
    "wpk_get_error_info": (C.c_int, [_H, C.POINTER(wpk_error_info)]),
    "wpk_last_error": (C.c_char_p, [_H]),
    "wpk_destroy": (C.c_int, [_H]),
    "wpk_debug_break_counter": (C.c_int, [_H, C.c_int]),
    "wpk_step_noalloc": (C.c_int, [_H, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "wpk_debug_gemm": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                 C.c_void_p]),
}

_lib = None


def load_library(path: str = LIB_PATH) -> C.CDLL:
    """Load libwpk.so (raises if it was not built; there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m streaming_persistent_sm_b200.build`")
    lib = C.CDLL(path)
    for name, (res, args) in _SIGS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(rc: int, h=None):
    if rc != WPK_OK:
        msg = load_library().wpk_last_error(h).decode() if h else ""
        raise WpkError(rc, msg)


def model_cfg(shape) -> wpk_model_cfg:
    """A decoder shape, or a two-stage shape (backbone + codebook head)."""
    if hasattr(shape, "backbone"):
        head = model_cfg(shape.head)
        m = model_cfg(shape.backbone)
        m.n_codebooks = shape.n_codebooks
        m.codebook_vocab = shape.codebook_vocab
        m._head = head  # keep the head struct alive
        m.head = C.pointer(head)
        return m
    return wpk_model_cfg(shape.n_layers, shape.hidden, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.ffn,
                         shape.vocab, shape.rms_eps, shape.rope_theta, 1 if shape.tied_embedding else 0, 0, 0, None)


def plan_cfg(max_batch: int, max_context: int, mode: int = WPK_MEGAKERNEL, n_regions: int = 1,
             region_cut: Sequence[int] = (0, 0, 0, 0), trace: int = 0, wait_timeout_ns: int = 0,
             page_tokens: int = 0, n_workers: int = 0, workers_per_sm: int = 0, resident: int = 0,
             slot_bytes: int = 0, tile_bytes: int = 0, split_pages: int = 0, lookahead: int = 0,
             schedule: int = 0, prefill: int = 0, decode: int = 0, frame_chunks: int = 0,
             head_workers: int = 0) -> wpk_plan_cfg:
    cut = (C.c_int * 4)(*list(region_cut) + [0] * (4 - len(region_cut)))
    return wpk_plan_cfg(max_batch, max_context, page_tokens, n_workers, workers_per_sm, mode, resident, n_regions,
                        cut, trace, wait_timeout_ns, slot_bytes, tile_bytes, split_pages, lookahead, schedule,
                        prefill, decode, frame_chunks, head_workers)


# ----------------------------------------------------------- thin wrappers --
def wpk_build_graph(model: wpk_model_cfg, plan: wpk_plan_cfg) -> C.c_void_p:
    h = C.c_void_p()
    rc = load_library().wpk_build_graph(C.byref(model), C.byref(plan), C.byref(h))
    if rc != WPK_OK:
        raise WpkError(rc, load_library().wpk_last_error(None).decode())
    return h


def wpk_workspace_size(h):
    w, k, s = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(load_library().wpk_workspace_size(h, C.byref(w), C.byref(k), C.byref(s)), h)
    return w.value, k.value, s.value


def wpk_load_weights(h, weights: wpk_weights, dev_weights: int, dev_kv: int, dev_scratch: int, stream: int = 0):
    _check(load_library().wpk_load_weights(h, C.byref(weights), dev_weights, dev_kv, dev_scratch, stream), h)


def wpk_set_block_table(h, table: np.ndarray):
    t = np.ascontiguousarray(table, dtype=np.int32)
    _check(load_library().wpk_set_block_table(h, t.ctypes.data_as(C.POINTER(C.c_int32))), h)


def wpk_prefill(h, tokens_dev: int, batch: int, prompt_len: int, first_tok_dev: int, logits_dev: int = 0,
                stream: int = 0):
    _check(load_library().wpk_prefill(h, tokens_dev, batch, prompt_len, first_tok_dev, logits_dev or None,
                                      stream or None), h)


def wpk_step(h, in_tok_dev: int = 0, out_tok_dev: int = 0, logits_dev: int = 0, stream: int = 0):
    _check(load_library().wpk_step(h, in_tok_dev or None, out_tok_dev or None, logits_dev or None, stream or None), h)


def wpk_step_noalloc(h, in_tok_dev: int = 0, out_tok_dev: int = 0, logits_dev: int = 0, stream: int = 0):
    """wpk_step with the activation scratch in the library's static device array."""
    _check(load_library().wpk_step_noalloc(h, in_tok_dev or None, out_tok_dev or None, logits_dev or None,
                                           stream or None), h)


def wpk_debug_gemm(a_img_dev: int, b1_img_dev: int, b2_img_dev: int, d_dev: int, n_chunks: int, N: int,
                   bf16: bool = True, stream: int = 0):
    _check(load_library().wpk_debug_gemm(a_img_dev, b1_img_dev, b2_img_dev or None, d_dev, n_chunks, N,
                                         1 if bf16 else 0, stream or None))


def wpk_select_program(h, batch: int = 0, prompt_len: int = 0):
    _check(load_library().wpk_select_program(h, batch, prompt_len), h)


def wpk_graph_stats_get(h) -> dict:
    st = wpk_graph_stats()
    _check(load_library().wpk_graph_stats_get(h, C.byref(st)), h)
    d = {n: getattr(st, n) for n, _ in wpk_graph_stats._fields_ if n != "region_begin"}
    d["region_begin"] = list(st.region_begin)[: st.n_regions + 1]
    return d


def wpk_get_edges(h) -> np.ndarray:
    n = C.c_int64()
    _check(load_library().wpk_get_edges(h, None, 0, C.byref(n)), h)
    buf = np.zeros((n.value, 2), dtype=np.int32)
    _check(load_library().wpk_get_edges(h, buf.ctypes.data_as(C.POINTER(C.c_int32)), n.value, C.byref(n)), h)
    return buf


def wpk_get_tile_ops(h, n_tiles: int) -> np.ndarray:
    ops = np.zeros(n_tiles, dtype=np.int32)
    _check(load_library().wpk_get_tile_ops(h, ops.ctypes.data_as(C.POINTER(C.c_int32)), n_tiles), h)
    return ops


def wpk_verify_graph(h):
    _check(load_library().wpk_verify_graph(h), h)


def wpk_simulate(h, n_threads: int, n_epochs: int, seed: int, wait_ms: int = 5000, stuck_tile: int = -1,
                 n_tiles: int = 0):
    order = np.full(max(1, n_tiles * n_epochs), -1, dtype=np.int32)
    rc = load_library().wpk_simulate(h, n_threads, n_epochs, seed, wait_ms, stuck_tile,
                                     order.ctypes.data_as(C.POINTER(C.c_int32)) if n_tiles else None)
    return rc, order


def wpk_prefill_slots(h, tokens_dev: int, slot0: int, batch: int, prompt_len: int, first_tok_dev: int,
                      logits_dev: int = 0, stream: int = 0):
    _check(load_library().wpk_prefill_slots(h, tokens_dev, slot0, batch, prompt_len, first_tok_dev,
                                            logits_dev or None, stream or None), h)


def wpk_set_active_slots(h, active) -> None:
    a = np.ascontiguousarray(active, dtype=np.int32)
    _check(load_library().wpk_set_active_slots(h, a.ctypes.data_as(C.POINTER(C.c_int32)), len(a)), h)


def wpk_get_tile_bytes(h, n_tiles: int) -> np.ndarray:
    out = np.zeros(n_tiles, dtype=np.int64)
    _check(load_library().wpk_get_tile_bytes(h, out.ctypes.data_as(C.POINTER(C.c_int64)), n_tiles), h)
    return out


def wpk_predict(h, service_ns, load_ns, mode: int = 0, n_regions: int = 1, region_cut=(0, 0, 0, 0),
                n_workers: int = 148, n_sms: int = 148, schedule: int = 1, slots: int = 4, dispatch_ns: float = 0.0,
                sync_ns: float = 0.0, first_chunk_ns: float = 0.0) -> float:
    """Predicted ns of one run of the selected program under a composition."""
    sv = np.ascontiguousarray(service_ns, dtype=np.float64)
    ld = np.ascontiguousarray(load_ns, dtype=np.float64)
    cfg = wpk_predict_cfg(mode, n_regions, (C.c_int * 4)(*region_cut), n_workers, n_sms, schedule, slots,
                          dispatch_ns, sync_ns, first_chunk_ns)
    out = C.c_double()
    _check(load_library().wpk_predict(h, sv.ctypes.data_as(C.POINTER(C.c_double)),
                                      ld.ctypes.data_as(C.POINTER(C.c_double)), C.byref(cfg), C.byref(out)), h)
    return out.value


def wpk_get_trace(h, n_tiles: int) -> np.ndarray:
    buf = np.zeros(n_tiles, dtype=TRACE_DTYPE)
    _check(load_library().wpk_get_trace(h, buf.ctypes.data, buf.nbytes), h)
    return buf


def wpk_get_error_info(h) -> dict:
    e = wpk_error_info()
    _check(load_library().wpk_get_error_info(h, C.byref(e)), h)
    return {n: getattr(e, n) for n, _ in wpk_error_info._fields_}


def wpk_last_error(h) -> str:
    return load_library().wpk_last_error(h).decode()


def wpk_destroy(h):
    _check(load_library().wpk_destroy(h))


def wpk_debug_break_counter(h, counter: int):
    _check(load_library().wpk_debug_break_counter(h, counter), h)


# ------------------------------------------------------------------ Engine --
class _HostWeights:
    """Keeps the numpy arrays alive while their pointers are in a wpk_weights."""

    def __init__(self, shape, weights: Dict[str, np.ndarray], prefix: str = ""):
        self.arrays = []

        def ptr(name):
            a = np.ascontiguousarray(weights[name], dtype=np.uint16)
            self.arrays.append(a)
            return a.ctypes.data_as(_P16)

        def layers(s, pre):
            arr = (wpk_layer_weights * s.n_layers)()
            for l in range(s.n_layers):
                p = f"{pre}layers.{l}."
                for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down"):
                    setattr(arr[l], n, ptr(p + n))
            return arr

        if hasattr(shape, "backbone"):  # two-stage model
            bb, K = shape.backbone, shape.n_codebooks
            self.layers = layers(bb, "backbone.")
            self.head_layers = layers(shape.head, "head.")
            tables = lambda name, first: (_P16 * K)(*([None] * first + [ptr(f"{name}.{k}") for k in range(first, K)]))
            self.frame_embed, self.head_embed, self.out_head = (tables("frame_embed", 0), tables("head_embed", 1),
                                                                tables("out_head", 0))
            self.struct = wpk_weights(ptr("backbone.embed"), ptr("backbone.final_norm"), None, self.layers,
                                      ptr("proj"), self.frame_embed, self.head_embed, self.out_head,
                                      self.head_layers, ptr("head.final_norm"))
            return
        self.layers = layers(shape, prefix)
        self.struct = wpk_weights(ptr(prefix + "embed"), ptr(prefix + "final_norm"),
                                  ptr(prefix + "lm_head") if not shape.tied_embedding else None, self.layers)


class Engine:
    """A handle plus torch-owned device buffers (weights image, KV pages, scratch)."""

    def __init__(self, shape, weights: Dict[str, np.ndarray], max_batch: int, max_context: int, **plan_kw):
        import torch

        self.torch = torch
        self.shape = shape
        self.plan = plan_cfg(max_batch, max_context, **plan_kw)
        self.h = wpk_build_graph(model_cfg(shape), self.plan)
        self.stats = wpk_graph_stats_get(self.h)
        wb, kb, sb = wpk_workspace_size(self.h)
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev_weights = torch.empty(max(wb, 256), dtype=torch.uint8, device=dev)
        self.dev_kv = torch.empty(max(kb, 256), dtype=torch.uint8, device=dev)
        self.dev_scratch = torch.empty(max(sb, 256), dtype=torch.uint8, device=dev)
        hw = _HostWeights(shape, weights)
        wpk_load_weights(self.h, hw.struct, self.dev_weights.data_ptr(), self.dev_kv.data_ptr(),
                         self.dev_scratch.data_ptr(), self._stream())
        self.max_batch = max_batch
        self.batch = 0
        # outputs per sequence: a token and its logits, or (two-stage) the
        # frame's codes and their logits per codebook
        if hasattr(shape, "backbone"):
            self._tok_shape, self._logit_shape = (shape.n_codebooks,), (shape.n_codebooks, shape.codebook_vocab)
        else:
            self._tok_shape, self._logit_shape = (), (shape.vocab,)

    def _stream(self) -> int:
        return self.torch.cuda.current_stream().cuda_stream

    def prefill(self, tokens, want_logits: bool = False):
        torch = self.torch
        tok = torch.as_tensor(np.ascontiguousarray(tokens, dtype=np.int32)).cuda()
        B, T = tok.shape
        self.batch = B
        first = torch.empty((B,) + self._tok_shape, dtype=torch.int32, device=tok.device)
        logits = (torch.empty((B,) + self._logit_shape, dtype=torch.float32, device=tok.device)
                  if want_logits else None)
        wpk_prefill(self.h, tok.data_ptr(), B, T, first.data_ptr(), logits.data_ptr() if want_logits else 0,
                    self._stream())
        self._keep = tok
        return first, logits

    def prefill_slots(self, slot0: int, tokens, want_logits: bool = False):
        """Prefill len(tokens) new sequences into slots slot0.. of the cohort
        (every slot of the plan is stepped from now on; see wpk_prefill_slots)."""
        torch = self.torch
        tok = torch.as_tensor(np.ascontiguousarray(tokens, dtype=np.int32)).cuda()
        B, T = tok.shape
        self.batch = self.max_batch
        first = torch.empty((B,) + self._tok_shape, dtype=torch.int32, device=tok.device)
        logits = (torch.empty((B,) + self._logit_shape, dtype=torch.float32, device=tok.device)
                  if want_logits else None)
        wpk_prefill_slots(self.h, tok.data_ptr(), slot0, B, T, first.data_ptr(),
                          logits.data_ptr() if want_logits else 0, self._stream())
        self.torch.cuda.current_stream().synchronize()
        return first, logits

    def step(self, in_tok=None, want_logits: bool = False, out_tok=None, logits=None):
        torch = self.torch
        B = self.batch
        dev = torch.device("cuda", torch.cuda.current_device())
        itp = 0
        if in_tok is not None:
            it = in_tok if isinstance(in_tok, torch.Tensor) else torch.as_tensor(
                np.ascontiguousarray(in_tok, dtype=np.int32), device=dev)
            self._keep_in = it
            itp = it.data_ptr()
        if out_tok is None:
            out_tok = torch.empty((B,) + self._tok_shape, dtype=torch.int32, device=dev)
        if want_logits and logits is None:
            logits = torch.empty((B,) + self._logit_shape, dtype=torch.float32, device=dev)
        wpk_step(self.h, itp, out_tok.data_ptr(), logits.data_ptr() if logits is not None else 0, self._stream())
        return out_tok, logits

    def close(self):
        if self.h:
            wpk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
