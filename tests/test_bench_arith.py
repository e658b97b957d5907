"""The benchmark's roofline arithmetic on CPU: the algorithmic bytes and
FLOPs it divides by, the tokens it counts, and the scaling of profiled DRAM
traffic, each against figures worked out by hand for the 1B shape."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

S = synth.LLAMA_1B
W_BYTES = 2_471_493_632  # every bf16 matrix of the 1B shape once, the tied LM head included


def test_kv_bytes_per_token_of_the_1b_shape():
    # K and V, 16 layers, 8 kv heads of 64 dims, bf16
    assert bench.KV_BYTES_PER_TOKEN(S) == 2 * 16 * 8 * 64 * 2 == 32_768


def test_algorithmic_bytes_of_a_decode_step():
    # batch 1 at context 496: the weights, 496 cached tokens' KV read, one token's KV written
    assert bench.algorithmic_bytes_per_step(S, W_BYTES, 1, 496) == W_BYTES + 496 * 32_768 + 32_768 == 2_487_779_328
    # batch 16: the KV terms scale with the batch, the weights do not
    assert bench.algorithmic_bytes_per_step(S, W_BYTES, 16, 496) == W_BYTES + 16 * 497 * 32_768


def test_prefill_flops_of_the_1b_shape():
    h, q, kv, f, L, V, T = 2048, 2048, 512, 8192, 16, 128256, 496
    per_token = L * (h * (q + 2 * kv) + q * h + 3 * f * h)
    attn = L * 4 * 32 * 64 * T * (T + 1) // 2
    want = 2 * per_token * T + attn + 2 * V * h
    assert bench.prefill_flops(S, 1, T) == want
    assert want == pytest.approx(0.98e12, rel=0.01)
    # the batch multiplies every term
    assert bench.prefill_flops(S, 3, T) == 3 * want


def test_tokens_counted_per_bench_step():
    wl = synth.WORKLOADS["llama1b_b1"]
    assert bench.job_tokens(wl, 128) == (1 * (1 + 128), True)  # first token + 128 decode steps
    wl = synth.WORKLOADS["llama1b_decode_b16"]
    assert bench.job_tokens(wl, 128) == (16 * 128, False)  # the prompt is prefilled untimed
    wl = synth.WORKLOADS["two_stage_b32"]
    k = wl.model.n_codebooks
    assert bench.job_tokens(wl, 64) == (32 * k * 65, True)  # codes: K per frame and sequence


def test_profiled_traffic_scales_with_the_kv_bytes(tmp_path, monkeypatch):
    # a summary written for batch 2 at context 100: 1e9 bytes per launch
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = os.path.join(ROOT, "streaming_persistent_sm_b200", "csrc")
    import hashlib

    sha = hashlib.sha1(b"".join(open(os.path.join(src, f), "rb").read()
                                for f in ("runtime.cu", "ptx.cuh", "wpk_internal.h"))).hexdigest()
    (prof / "k.md").write_text("traffic_kernel: kern\ntraffic_bytes_per_launch: 1000000000\ntraffic_context: 100\n"
                               "traffic_batch: 2\nkv_bytes_per_token: 1000\n"
                               f"source_sha1(runtime.cu + ptx.cuh + wpk_internal.h): {sha}\n")
    os.makedirs(tmp_path / "streaming_persistent_sm_b200", exist_ok=True)
    os.symlink(src, tmp_path / "streaming_persistent_sm_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # weights part 1e9 - 2*100*1000; then 4 sequences at context 150
    assert bench.profiled_traffic("kern", 4, 150) == 1e9 - 2e5 + 4 * 150 * 1000
    assert bench.profiled_traffic("other_kernel", 4, 150) is None
    (prof / "k.md").write_text((prof / "k.md").read_text().replace(sha, "0" * 40))
    assert bench.profiled_traffic("kern", 4, 150) is None  # sources changed since the capture


def test_weight_bytes_match_the_compiled_decode_program():
    """The weight bytes the roofline counts are the ones the compiled b1
    program streams: every bf16 matrix once, the tied LM head included (the
    norm gains are not counted)."""
    from streaming_persistent_sm_b200 import wpk as W

    h = W.wpk_build_graph(W.model_cfg(S), W.plan_cfg(1, 640))
    try:
        st = W.wpk_graph_stats_get(h)
    finally:
        W.wpk_destroy(h)
    hd, q, kv, f, L, V = 2048, 2048, 512, 8192, 16, 128256
    matrices = 2 * (L * (hd * (q + 2 * kv) + q * hd + 3 * f * hd) + V * hd)
    assert st["weight_bytes"] == W_BYTES == matrices


def test_deadline_capacity_is_the_largest_cohort_within_the_period():
    import bench

    # per-size step times (ms): the q-quantile, not the mean, decides
    times = {1: [1.0] * 99 + [2.0], 8: [5.0] * 99 + [50.0], 16: [6.0] * 98 + [90.0, 95.0], 32: [70.0] * 100}
    cap, qs = bench.deadline_capacity(times, period_ms=80.0, q=0.99)
    assert qs[1] == pytest.approx(1.01) and qs[32] == pytest.approx(70.0)  # linear interpolation
    assert qs[16] > 80.0  # its mean is 7.7 ms, its 99th percentile misses the period
    assert cap == 32  # sizes need not be monotone; the largest that fits
    assert bench.deadline_capacity(times, period_ms=0.5, q=0.5) == (0, {1: 1.0, 8: 5.0, 16: 6.0, 32: 70.0})
    cap, _ = bench.deadline_capacity(times, period_ms=80.0, q=0.5)
    assert cap == 32
