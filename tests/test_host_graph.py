"""Host-side checks of the C ABI and the graph compiler (no GPU needed)."""
import os
import re

import numpy as np
import pytest

import synth
from streaming_persistent_sm_b200 import wpk as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(W.LIB_PATH):
        from streaming_persistent_sm_b200 import build

        build.build()
    return W.load_library()


def test_library_exports_every_declared_symbol(lib):
    header = open(os.path.join(ROOT, "include", "wpk.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+char\s*\*|int)\s*(wpk_\w+)\s*\(", header, re.M))
    assert len(declared) >= 16
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(W._SIGS), declared ^ set(W._SIGS)


def _graph(shape=synth.TINY, **kw):
    B = kw.pop("max_batch", 1)
    ctx = kw.pop("max_context", 64)
    return W.wpk_build_graph(W.model_cfg(shape), W.plan_cfg(B, ctx, **kw))


def test_tiny_graph_verifies_and_counters_dedup(lib):
    h = _graph()
    try:
        st = W.wpk_graph_stats_get(h)
        W.wpk_verify_graph(h)
        ops = W.wpk_get_tile_ops(h, st["n_tiles"])
        assert ops[0] == 0 and ops[-1] == 7  # embed first, final last
        # per layer: 1 QKV + one per kv head + O + gate/up + one per down K-chunk
        assert st["n_counters"] == synth.TINY.n_layers * (4 + synth.TINY.n_kv_heads) + 2
        # every tile but the last signals at least one counter (a k/v tile that
        # covers several kv heads signals each head's attention counter)
        assert st["n_signals"] >= st["n_tiles"] - 1
        assert st["weight_bytes"] == sum(np.prod(s) * 2 for n, s, k in synth.tensor_specs(synth.TINY) if k == "normal")
        edges = W.wpk_get_edges(h)
        assert np.all(edges[:, 0] < edges[:, 1])  # ticket order is topological
    finally:
        W.wpk_destroy(h)


@pytest.mark.parametrize("kw", [
    dict(max_batch=3, max_context=200, split_pages=2, page_tokens=32),
    dict(max_batch=2, max_context=130, page_tokens=32, tile_bytes=4096, slot_bytes=16384, lookahead=1),
    dict(max_batch=1, max_context=64, n_regions=3, region_cut=(0, 1, 2, 0)),
])
def test_graph_variants_verify(lib, kw):
    h = _graph(**kw)
    try:
        W.wpk_verify_graph(h)
        st = W.wpk_graph_stats_get(h)
        rb = st["region_begin"]
        assert rb[0] == 0 and rb[-1] == st["n_tiles"] and all(a < b for a, b in zip(rb, rb[1:]))
    finally:
        W.wpk_destroy(h)


def test_down_projection_uses_chunk_edges(lib):
    # the 1B shape splits the down projection in 4 K-chunks; each chunk's tiles
    # wait only for the gate/up tiles producing that chunk (finer edges)
    s = synth.ModelShape(n_layers=1, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=8192, vocab=512)
    h = _graph(s)
    try:
        W.wpk_verify_graph(h)
        st = W.wpk_graph_stats_get(h)
        ops = W.wpk_get_tile_ops(h, st["n_tiles"])
        e = W.wpk_get_edges(h)
        gu = np.flatnonzero(ops == 4)
        down = np.flatnonzero(ops == 5)
        preds_of_down = {v: set(e[e[:, 1] == v, 0]) for v in down}
        sizes = {len(p) for p in preds_of_down.values()}
        assert sizes == {len(gu) // 4}
        assert len({frozenset(p) for p in preds_of_down.values()}) == 4
    finally:
        W.wpk_destroy(h)


@pytest.mark.parametrize("threads,schedule", [(1, 0), (3, 0), (17, 0), (1, 1), (5, 1), (23, 1)])
def test_cpu_schedule_simulator_is_deadlock_free(lib, threads, schedule):
    h = _graph(max_batch=2, max_context=128, schedule=schedule)
    try:
        st = W.wpk_graph_stats_get(h)
        T = st["n_tiles"]
        rc, order = W.wpk_simulate(h, threads, 3, 42 + threads, 10000, -1, T)
        assert rc == 0, W.wpk_last_error(h)
        e = W.wpk_get_edges(h)
        for ep in range(3):
            pos = np.empty(T, dtype=np.int64)
            seg = order[ep * T:(ep + 1) * T]
            # a step starts only after the previous one completed (the doorbell),
            # so epoch ep's tiles are the ep-th block of completions
            pos[seg] = np.arange(T)
            assert sorted(seg.tolist()) == list(range(T))
            assert np.all(pos[e[:, 0]] < pos[e[:, 1]])
    finally:
        W.wpk_destroy(h)


def test_simulator_reports_stuck_producer_as_timeout(lib):
    h = _graph()
    try:
        rc, _ = W.wpk_simulate(h, 4, 1, 1, 200, 5, 0)
        assert rc == W.WPK_ERR_TIMEOUT
        assert "timed out" in W.wpk_last_error(h)
    finally:
        W.wpk_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(max_batch=0), dict(n_regions=5), dict(mode=7), dict(slot_bytes=1000),
    dict(n_regions=2, region_cut=(0, 9, 0, 0)), dict(split_pages=-1), dict(page_tokens=128), dict(decode=7),
    dict(decode=W.WPK_DECODE_MMA, max_batch=129),
])
def test_invalid_plans_are_rejected(lib, bad):
    with pytest.raises(W.WpkError):
        _graph(**bad)


def test_host_only_handle_refuses_device_calls(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("host-only behaviour")
    h = _graph()
    try:
        with pytest.raises(W.WpkError) as ei:
            W.wpk_step(h)
        assert ei.value.code == W.WPK_ERR_CUDA
    finally:
        W.wpk_destroy(h)


def test_llama1b_graph_shape(lib):
    h = _graph(synth.LLAMA_1B, max_batch=1, max_context=624)
    try:
        st = W.wpk_graph_stats_get(h)
        # 16 layers x (QKV + 8 kv heads + O + gate/up + 4 down chunks) + LM head + final
        assert st["n_counters"] == 16 * 15 + 2
        bf16_bytes = sum(np.prod(s) * 2 for n, s, k in synth.tensor_specs(synth.LLAMA_1B) if k == "normal")
        # matmul weights and the tied embedding, read once per step (norm gains excluded)
        assert st["weight_bytes"] == bf16_bytes == 2_471_493_632
    finally:
        W.wpk_destroy(h)


@pytest.mark.parametrize("B,T", [(1, 20), (2, 40), (3, 130)])
def test_prefill_program_verifies_and_simulates(lib, B, T):
    h = _graph(max_batch=3, max_context=160)
    try:
        W.wpk_select_program(h, B, T)
        st = W.wpk_graph_stats_get(h)
        ops = W.wpk_get_tile_ops(h, st["n_tiles"])
        names = [W.OP_NAMES[o] for o in ops]
        assert names[0] == "p_embed" and names[-1] == "final" and "mma_qkv" in names and "p_attn" in names
        W.wpk_verify_graph(h)
        rc, order = W.wpk_simulate(h, 7, 2, 3, 10000, -1, st["n_tiles"])
        assert rc == 0, W.wpk_last_error(h)
        e = W.wpk_get_edges(h)
        assert np.all(e[:, 0] < e[:, 1])
        # attention of a later query block waits for the K/V tiles of every earlier token block
        n_tb = -(-(B * T) // 128)
        # two RMSNorms per layer, each as 128 / 16 tiles of 16 rows per token block
        assert ops.tolist().count(W.OP_NAMES.index("norm")) == 2 * synth.TINY.n_layers * n_tb * (128 // 16)
        W.wpk_select_program(h, 0, 0)
        assert W.wpk_graph_stats_get(h)["n_tiles"] != st["n_tiles"]
    finally:
        W.wpk_destroy(h)


def test_tokenwise_prefill_plan_has_no_prefill_program(lib):
    h = _graph(prefill=W.WPK_PREFILL_TOKENWISE)
    try:
        with pytest.raises(W.WpkError) as ei:
            W.wpk_select_program(h, 1, 8)
        assert ei.value.code == W.WPK_ERR_UNSUPPORTED
    finally:
        W.wpk_destroy(h)


# ------------------------------------------------------- batched decode program
def _ops(h):
    st = W.wpk_graph_stats_get(h)
    return st, np.array([W.OP_NAMES[o] for o in W.wpk_get_tile_ops(h, st["n_tiles"])])


@pytest.mark.parametrize("B", [16, 12, 9])
def test_batched_decode_program_verifies_and_simulates(lib, B):
    # more than 8 sequences: the step runs on tensor-core tiles (AUTO)
    h = _graph(max_batch=B, max_context=160)
    try:
        st, names = _ops(h)
        for op in ("b_qkv", "b_o", "b_gate_up", "b_down", "b_lm_head"):
            assert op in names, op
        assert not {"qkv", "o", "gate_up", "down", "lm_head"} & set(names)
        assert names[0] == "embed" and names[-1] == "final"
        W.wpk_verify_graph(h)
        # same weight bytes as the GEMV program: every matrix once, LM head tied
        assert st["weight_bytes"] == sum(np.prod(s) * 2 for n, s, k in synth.tensor_specs(synth.TINY)
                                         if k == "normal")
        rc, order = W.wpk_simulate(h, 11, 2, 5, 10000, -1, st["n_tiles"])
        assert rc == 0, W.wpk_last_error(h)
        e = W.wpk_get_edges(h)
        T = st["n_tiles"]
        pos = np.empty(T, dtype=np.int64)
        pos[order[:T]] = np.arange(T)
        assert np.all(pos[e[:, 0]] < pos[e[:, 1]])
    finally:
        W.wpk_destroy(h)


def test_batched_decode_k_split_edges(lib):
    # each down tile waits only for the gate/up tiles of its K range (one gate/up
    # tile = 64 h features = one 64-column chunk), each O tile only for the
    # attention tiles of the heads in its K range
    s = synth.ModelShape(n_layers=1, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64, ffn=2048, vocab=512)
    h = _graph(s, max_batch=16, max_context=64, n_workers=64, tile_bytes=16384)
    try:
        W.wpk_verify_graph(h)
        st, names = _ops(h)
        e = W.wpk_get_edges(h)
        gu = set(np.flatnonzero(names == "b_gate_up"))
        down = np.flatnonzero(names == "b_down")
        attn = set(np.flatnonzero(names == "attn"))
        o = np.flatnonzero(names == "b_o")
        assert len(down) > 2 and len(o) > 2  # both projections are split along K
        pred_sets = []
        for v in down:
            p = set(e[e[:, 1] == v, 0])
            assert p <= gu and 0 < len(p) < len(gu)
            pred_sets.append(frozenset(p))
        assert len(set(pred_sets)) > 1
        for v in o:
            p = set(e[e[:, 1] == v, 0]) - set(np.flatnonzero(names == "embed"))
            assert p <= attn and 0 < len(p) <= len(attn)
    finally:
        W.wpk_destroy(h)


def test_decode_mode_selection(lib):
    for B, want in ((4, "lm_head"), (5, "b_lm_head"), (48, "b_lm_head")):
        h = _graph(max_batch=B, max_context=64)
        try:
            _, names = _ops(h)
            assert want in names and names[-2] == want
        finally:
            W.wpk_destroy(h)
    h = _graph(max_batch=32, max_context=64, decode=W.WPK_DECODE_GEMV)
    try:
        _, names = _ops(h)
        assert "lm_head" in names and "b_qkv" not in names
    finally:
        W.wpk_destroy(h)
    # shapes that are not multiples of the 128-row tensor-core tiles
    odd = synth.ModelShape(n_layers=1, hidden=192, n_heads=3, n_kv_heads=1, head_dim=64, ffn=320, vocab=300)
    with pytest.raises(W.WpkError) as ei:
        _graph(odd, max_batch=16, decode=W.WPK_DECODE_MMA)
    assert ei.value.code == W.WPK_ERR_UNSUPPORTED
    h = _graph(odd, max_batch=16)  # AUTO falls back to GEMV tiles
    try:
        _, names = _ops(h)
        assert "lm_head" in names
    finally:
        W.wpk_destroy(h)


def test_llama1b_batched_decode_graph_shape(lib):
    h = _graph(synth.LLAMA_1B, max_batch=48, max_context=624, n_workers=148)
    try:
        st, names = _ops(h)
        # the LM head's 128-row blocks: 128256 = 1002 x 128
        assert (names == "b_lm_head").sum() == 1002
        assert st["weight_bytes"] == 2_471_493_632
        # one attention tile per (sequence, kv head): 48 x 8 per layer
        assert (names == "attn").sum() == 16 * 48 * 8
        for op in ("b_qkv", "b_o", "b_down"):
            assert (names == op).sum() >= 16 * 128, op  # split along K: about one tile per worker
    finally:
        W.wpk_destroy(h)


def test_prefill_splits_o_and_down_along_k(lib):
    # one 128-token block gives only hidden/128 = 16 O and down row blocks:
    # both are split along K so every worker gets a tile, and each split waits
    # only for the producers of its K range
    h = _graph(synth.LLAMA_1B, max_batch=1, max_context=256, n_workers=148)
    try:
        W.wpk_select_program(h, 1, 128)
        st, names = _ops(h)
        n_o, n_down = (names == "mma_o").sum(), (names == "mma_down").sum()
        assert n_o >= 16 * 128 and n_down >= 16 * 128, (n_o, n_down)
        e = W.wpk_get_edges(h)
        gu = set(np.flatnonzero(names == "mma_gate_up"))
        for v in np.flatnonzero(names == "mma_down")[:64]:
            p = set(e[e[:, 1] == v, 0])
            assert p <= gu and len(p) < 128
    finally:
        W.wpk_destroy(h)


def test_two_stage_handle_host_side(lib):
    s = synth.TINY_TWO_STAGE
    h = W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(16, 64))
    try:
        W.wpk_verify_graph(h)  # the backbone program
        st, names = _ops(h)
        # the backbone's output head is the projection into the head's width
        bb = s.backbone
        matrices = sum(np.prod(x) * 2 for n, x, k in synth.tensor_specs(bb) if k == "normal" and n != "embed")
        assert st["weight_bytes"] == matrices + s.head.hidden * bb.hidden * 2
        wb, kb, sb = W.wpk_workspace_size(h)
        # every table is in the image: frame inputs, head inputs (K-1), output heads
        K, V = s.n_codebooks, s.codebook_vocab
        assert wb > (K * bb.hidden + (2 * K - 1) * s.head.hidden) * V * 2
    finally:
        W.wpk_destroy(h)
    bad = W.model_cfg(s)
    bad.n_codebooks = 17
    with pytest.raises(W.WpkError):
        W.wpk_build_graph(bad, W.plan_cfg(1, 64))
    with pytest.raises(W.WpkError):
        W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(1, 64, resident=1))


def test_two_stage_chunked_frame_host_side(lib):
    """frame_chunks = C builds C backbone + head pairs of ceil(B / C) sequences
    over one weight image; KV and scratch are the pairs' sums."""
    s = synth.TINY_TWO_STAGE
    # (the pairs of three decode on CUDA cores; so does the reference plan)
    one = W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(5, 64, n_workers=16, decode=W.WPK_DECODE_GEMV))
    per3 = W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(3, 64, n_workers=12))
    h = W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(5, 64, n_workers=16, frame_chunks=2, head_workers=4))
    try:
        W.wpk_verify_graph(h)
        st = W.wpk_graph_stats_get(h)
        assert st["n_workers"] == 12  # the backbones' share of the 16 workers
        wb1, _, _ = W.wpk_workspace_size(one)
        wb, kb, sb = W.wpk_workspace_size(h)
        _, kb3, sb3 = W.wpk_workspace_size(per3)
        assert wb == wb1  # one shared image
        assert kb == 2 * kb3 and sb == 2 * sb3  # two pairs of three sequences each
    finally:
        for x in (one, per3, h):
            W.wpk_destroy(x)
    for bad in (dict(frame_chunks=9), dict(frame_chunks=6), dict(frame_chunks=-1),
                dict(frame_chunks=2, head_workers=16), dict(head_workers=4)):
        with pytest.raises(W.WpkError):
            W.wpk_build_graph(W.model_cfg(s), W.plan_cfg(5, 64, n_workers=16, **bad))
    with pytest.raises(W.WpkError):  # a plain decoder has no frame
        W.wpk_build_graph(W.model_cfg(synth.TINY), W.plan_cfg(4, 64, frame_chunks=2))


@pytest.mark.parametrize("shape,B", [(synth.TINY, 1), (synth.TINY, 3), (synth.LLAMA_1B, 1)])
def test_team_schedule_streams_partition_the_step_and_drop_same_stream_edges(lib, shape, B):
    # "Why real-time inference wants a megakernel", "A concrete design": every op
    # goes to a team of workers, each worker walks its own stream, and only
    # dependencies between streams need a counter
    W_ = 16 if shape is synth.TINY else 148
    h = _graph(shape, max_batch=B, max_context=640 if shape is synth.LLAMA_1B else 64,
               schedule=W.WPK_SCHED_TEAMS, n_workers=W_)
    ref = _graph(shape, max_batch=B, max_context=640 if shape is synth.LLAMA_1B else 64,
                 schedule=W.WPK_SCHED_STATIC, n_workers=W_)
    try:
        st, st_ref = W.wpk_graph_stats_get(h), W.wpk_graph_stats_get(ref)
        assert st["n_tiles"] == st_ref["n_tiles"]
        # a worker signals once per op it served, not once per tile
        assert st["n_signals"] < st_ref["n_signals"]
        if shape is synth.TINY:
            W.wpk_verify_graph(h)  # stream order counts as an edge for the hazard check
            rc, order = W.wpk_simulate(h, W_, 3, 5, 10000, -1, st["n_tiles"])
            assert rc == 0, W.wpk_last_error(h)
            for e in range(3):  # every tile once per step
                assert sorted(order[e * st["n_tiles"]:(e + 1) * st["n_tiles"]].tolist()) == list(range(st["n_tiles"]))
            # a stuck tile is still caught (the embed tile: it signals the first layer)
            rc, _ = W.wpk_simulate(h, W_, 1, 5, 300, 0, 0)
            assert rc == W.WPK_ERR_TIMEOUT
        e = W.wpk_get_edges(h)
        assert np.all(e[:, 0] < e[:, 1])
    finally:
        W.wpk_destroy(h)
        W.wpk_destroy(ref)


def test_team_schedule_is_one_region_launched_per_step(lib):
    for kw in (dict(n_regions=2, region_cut=(0, 1, 0, 0)), dict(resident=1), dict(mode=W.WPK_PER_OP_GRAPH)):
        with pytest.raises(W.WpkError) as ei:
            _graph(schedule=W.WPK_SCHED_TEAMS, **kw)
        assert ei.value.code == W.WPK_ERR_UNSUPPORTED


def test_two_pass_gemv_tiles_fit_the_ring_in_whole_stages(lib):
    # Above 8 sequences a GEMV tile is read in several passes, so all its
    # chunks must be staged at once.  GEMV stages hold two 16 KB chunks: a
    # slot of nine chunks holds four stages, eight chunks.
    h = _graph(synth.LLAMA_1B, max_batch=16, max_context=640, decode=W.WPK_DECODE_GEMV, slot_bytes=9 * 16384)
    try:
        st = W.wpk_graph_stats_get(h)
        ops = W.wpk_get_tile_ops(h, st["n_tiles"])
        nbytes = W.wpk_get_tile_bytes(h, st["n_tiles"])
        gemv = np.isin(ops, [W.OP_NAMES.index(n) for n in ("qkv", "o", "gate_up", "down", "lm_head")])
        assert gemv.sum() > 0
        # every 1B GEMV row is 4 KB, so a chunk is exactly 16 KB
        assert nbytes[gemv].max() == 8 * 16384
    finally:
        W.wpk_destroy(h)
