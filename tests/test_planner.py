"""The composition planner's simulator (wpk_predict) against closed forms on
host-only graphs, and the planner's calibration from a synthetic trace.  No GPU.
"""
import numpy as np
import pytest

import synth
from streaming_persistent_sm_b200 import planner as PL
from streaming_persistent_sm_b200 import wpk as W

S = synth.TINY


@pytest.fixture(scope="module")
def h():
    W.load_library()
    hh = W.wpk_build_graph(W.model_cfg(S), W.plan_cfg(1, 64, schedule=W.WPK_SCHED_STATIC))
    yield hh
    W.wpk_destroy(hh)


def _groups(ops):
    """(begin, end) of each op group: maximal runs of one op (in ticket order,
    the compiler never puts two groups of one op next to each other)."""
    out, i = [], 0
    while i < len(ops):
        j = i
        while j < len(ops) and ops[j] == ops[i]:
            j += 1
        out.append((i, j))
        i = j
    return out


def _longest_path(n, edges, cost):
    """Longest path through the tile DAG with per-tile costs (brute force)."""
    preds = [[] for _ in range(n)]
    for u, v in edges:
        preds[v].append(u)
    fin = np.zeros(n)
    for t in range(n):
        fin[t] = max([fin[u] for u in preds[t]], default=0.0) + cost[t]
    return fin.max()


def test_one_worker_runs_every_tile_in_order(h):
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    sv = np.full(n, 1000.0)
    ld = np.zeros(n)
    for R, cuts in ((1, (0, 0, 0, 0)), (2, (0, 1, 0, 0))):
        t = W.wpk_predict(h, sv, ld, n_regions=R, region_cut=cuts, n_workers=1, dispatch_ns=500.0)
        assert t == pytest.approx(n * 1000.0 + R * 500.0)


def test_unbounded_workers_follow_the_critical_path(h):
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    e = W.wpk_get_edges(h)
    rng = np.random.default_rng(0)
    sv = rng.uniform(100.0, 5000.0, n)
    # (one slot: a worker holds one tile, so the queue gives every tile a worker)
    t = W.wpk_predict(h, sv, np.zeros(n), n_workers=n, schedule=W.WPK_SCHED_QUEUE, slots=1)
    assert t == pytest.approx(_longest_path(n, e, sv))
    # the static streams give worker w the tickets w, w + n, ...: also one each
    assert W.wpk_predict(h, sv, np.zeros(n), n_workers=n) == pytest.approx(t)
    # each counter wait adds the hop to the tile's ready time
    t_sync = W.wpk_predict(h, sv, np.zeros(n), n_workers=n, schedule=W.WPK_SCHED_QUEUE, slots=1, sync_ns=700.0)
    has_pred = np.zeros(n, dtype=bool)
    has_pred[e[:, 1]] = True
    assert t_sync == pytest.approx(_longest_path(n, e, sv + 700.0 * has_pred))


def test_conventional_launches_run_in_waves(h):
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    ops = W.wpk_get_tile_ops(h, n)
    sv = np.full(n, 2000.0)
    for sms in (1, 2, 3, 1000):
        t = W.wpk_predict(h, sv, np.zeros(n), mode=W.WPK_PER_OP_GRAPH, n_sms=sms, dispatch_ns=3000.0)
        want = sum(3000.0 + -(-(e - b) // sms) * 2000.0 for b, e in _groups(ops))
        assert t == pytest.approx(want), sms


def test_one_staging_slot_against_claim_ahead():
    # one worker, a load-bound stream: with one slot a tile's load starts when
    # the previous tile is done; with more slots the loads run back to back
    W.load_library()
    hh = W.wpk_build_graph(W.model_cfg(S), W.plan_cfg(1, 64))
    try:
        n = W.wpk_graph_stats_get(hh)["n_tiles"]
        sv, ld, f = np.full(n, 1000.0), np.full(n, 3000.0), 400.0
        one = W.wpk_predict(hh, sv, ld, n_workers=1, slots=1, first_chunk_ns=f)
        assert one == pytest.approx(n * max(f + 1000.0, 3000.0))
        two = W.wpk_predict(hh, sv, ld, n_workers=1, slots=2, first_chunk_ns=f)
        assert two == pytest.approx(n * 3000.0)  # the loads are the bound
        # compute-bound: the slot rule no longer matters once loads are short
        sv2, ld2 = np.full(n, 3000.0), np.full(n, 1000.0)
        assert W.wpk_predict(hh, sv2, ld2, n_workers=1, slots=1) == pytest.approx(n * 3000.0)
    finally:
        W.wpk_destroy(hh)


def test_bad_configurations_are_rejected(h):
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    sv, ld = np.ones(n), np.zeros(n)
    for kw in (dict(n_workers=0), dict(slots=0), dict(n_regions=5), dict(n_regions=2, region_cut=(0, 0, 0, 0)),
               dict(mode=7)):
        with pytest.raises(W.WpkError):
            W.wpk_predict(h, sv, ld, **kw)
    with pytest.raises(W.WpkError):
        W.wpk_predict(h, -sv, ld)


def test_calibration_from_a_synthetic_trace(h):
    # a trace written by hand: tile t runs [10 t, 10 t + 4] us, so every hop
    # from the latest producer is 6 us minus the producers' spacing
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    e = W.wpk_get_edges(h)
    tr = np.zeros(n, dtype=W.TRACE_DTYPE)
    tr["tile"] = np.arange(n)[::-1]  # records in any order
    tr["worker"] = (tr["tile"] % 7).astype(np.uint16)
    tr["t_start_ns"] = (10_000 * tr["tile"]).astype(np.uint64)
    tr["t_end_ns"] = tr["t_start_ns"] + 4_000
    cal = PL.calibrate(tr, np.full(n, 8192), e, bytes_per_ns_per_worker=4.096)
    assert np.allclose(cal.service_ns, 4000.0)
    assert np.allclose(cal.load_ns, 2000.0)
    start = 10_000.0 * np.arange(n)
    last = np.full(n, -np.inf)
    np.maximum.at(last, e[:, 1], start[e[:, 0]] + 4000.0)
    # tile t follows tile t - 7 on its worker; the hop counts only where the
    # last predecessor ended after that
    prev = np.where(np.arange(n) >= 7, start - 70_000.0 + 4000.0, -np.inf)
    ok = np.isfinite(last) & (last >= prev)
    hop = start[ok] - last[ok]
    assert cal.sync_ns == pytest.approx(np.median(hop[hop >= 0]))


def test_calibration_leaves_out_tiles_that_waited_for_their_worker(h):
    # one worker runs every tile back to back: no tile waited on a dependency,
    # so no hop is measured
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    e = W.wpk_get_edges(h)
    tr = np.zeros(n, dtype=W.TRACE_DTYPE)
    tr["tile"] = np.arange(n)
    tr["t_start_ns"] = (1000 * np.arange(n)).astype(np.uint64)
    tr["t_end_ns"] = tr["t_start_ns"] + 1000
    assert PL.calibrate(tr, np.zeros(n), e, bytes_per_ns_per_worker=1.0).sync_ns == 0.0


def test_dispatch_fit_and_ranking(h):
    n = W.wpk_graph_stats_get(h)["n_tiles"]
    cal = PL.Calibration(np.full(n, 1500.0), np.full(n, 500.0), sync_ns=800.0, first_chunk_ns=300.0)
    kw = dict(n_workers=8, n_sms=8, schedule=W.WPK_SCHED_STATIC, slots=4)
    per_op = PL.Candidate("per-op graph", W.WPK_PER_OP_GRAPH)
    cal.dispatch_ns = 2500.0
    target = PL.predict(h, cal, per_op, **kw)
    cal.dispatch_ns = 0.0
    assert PL.fit_dispatch(h, cal, per_op, target, **kw) == pytest.approx(2500.0, rel=1e-6)
    rows = PL.rank(h, cal, PL.default_candidates(S.n_layers)[:2] + [per_op], **kw)
    assert [r["predicted_us"] for r in rows] == sorted(r["predicted_us"] for r in rows)
    # more launches cost more dispatch nodes: one region beats two here
    names = [r["name"] for r in rows]
    assert names.index("1 MK") < names.index("2 MK (cuts 0,1)")
