"""The bench's counted work and its traffic bookkeeping, on the CPU: the FLOP
counts of the training step and the cached-KV prefill against a direct count
of allowed (query, key) pairs, the decode byte count against the used cache
rows, and the rule that a stored ncu traffic figure is dropped once the
kernel sources it was captured on change."""
import numpy as np

import bench
from io_aware_exact_21_b200.inputs import WORKLOADS


def _pairs(nq, nk, causal):
    i = np.arange(nq)[:, None] + (nk - nq)
    j = np.arange(nk)[None, :]
    allowed = np.ones((nq, nk), bool)
    if causal:
        allowed &= j <= i
    return int(allowed.sum())


def test_training_flops_are_the_dense_convention():
    # forward 4*d per (query, key) pair of the full square, halved when causal;
    # backward 2.5 x forward (five GEMMs)
    f, b = bench.flops(4, 16, 8192, 128, False)
    assert f == 4.0 * 4 * 16 * 8192 * 8192 * 128 and b == 2.5 * f
    fc, bc = bench.flops(4, 16, 8192, 128, True)
    assert fc == f / 2 and bc == b / 2
    # the halved count is within 1/N of the exact causal pair count
    n = 512
    exact = 4.0 * _pairs(n, n, True) * 64
    assert abs(bench.flops(1, 1, n, 64, True)[0] - exact) / exact < 1.0 / n


def test_cached_kv_flops_count_the_allowed_pairs():
    # Nq*Nk - Nq^2/2 pairs under the bottom-right causal mask (the triangle of
    # the last Nq positions halved, as in the self-attention count)
    for nq, nk in ((64, 256), (128, 128), (100, 1000)):
        exact = 4.0 * _pairs(nq, nk, True) * 128
        got = bench.flops_kv(1, 1, nq, nk, 128, True)
        assert abs(got - exact) / exact < 1.0 / nq
        assert bench.flops_kv(1, 1, nq, nk, 128, False) == 4.0 * nq * nk * 128


def _window_pairs(n, w):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    return int(((j <= i) & (j > i - w)).sum())


def test_packed_workload_flops_from_the_drawn_lengths():
    # a window counts its pairs exactly; causal alone uses n^2 / 2 per sequence
    for n in (1, 5, 127, 1024, 1025, 3000):
        assert bench.allowed_pairs(n, True, 1024) == _window_pairs(n, 1024)
        assert bench.allowed_pairs(n, True, 0) == 0.5 * n * n
        assert bench.allowed_pairs(n, False, 0) == n * n
    wl = WORKLOADS["varlen_window"]
    lens = [130, 2000, 4096]
    f, b = bench.workload_flops(wl, lens)
    assert f == 4.0 * wl.H * wl.d * sum(_window_pairs(n, 1024) for n in lens) and b == 2.5 * f
    wc = WORKLOADS["varlen_causal"]
    assert bench.workload_flops(wc, lens)[0] == 4.0 * wc.H * wc.d * sum(n * n / 2 for n in lens)


def test_decode_bytes_are_the_used_cache_rows():
    wl = WORKLOADS["decode"]
    lens = [4096, 5000, 8192] + [6000] * (wl.B - 3)
    kv = 2 * sum(lens) * wl.H * wl.d * 2
    qo = 2 * wl.B * wl.N * wl.H * wl.d * 2 + wl.B * wl.H * wl.N * 4
    assert bench.decode_bytes(wl, lens) == kv + qo


def test_traffic_figure_is_dropped_when_its_sources_change(monkeypatch, tmp_path):
    # a stored figure is reported only while the hash of its sources matches
    entry = bench.TRAFFIC["dkdv"]
    current = bench.source_hash(entry["sources"])
    monkeypatch.setitem(bench.TRAFFIC, "dkdv", dict(entry, sha=current))
    assert bench.traffic_for("dkdv") == entry["bytes_per_launch"]
    monkeypatch.setitem(bench.TRAFFIC, "dkdv", dict(entry, sha="0" * 16))
    assert bench.traffic_for("dkdv") is None
    # and only for the workload it was captured on
    monkeypatch.setitem(bench.TRAFFIC, "dkdv", dict(entry, sha=current))
    assert bench.traffic_for("dkdv", "decode") is None


def test_cpu_baseline_repeats_until_the_time_floor(monkeypatch):
    # the cpu_baseline leg repeats the oracle sample with a new seed each
    # time and reports the rate over all samples
    calls = []

    def fake(seed=5):
        calls.append(seed)
        return 2.0 * len(calls), "one sample", 4, 1.0     # rate, description, threads, seconds

    monkeypatch.setattr(bench, "oracle_sample_kv", fake)
    rate, desc, threads = bench.cpu_baseline_sample("prefill_kv", min_secs=3.0)
    assert calls == [5, 6, 7]
    assert rate == (2.0 + 4.0 + 6.0) / 3.0 and threads == 4
    assert "3 such samples" in desc and "3.0 s in total" in desc


def test_source_hash_ignores_comments_only():
    # a comment or blank-line edit keeps the hash (the compiler sees the same
    # code); any change to code, including inside a string, does not
    base = 'int a = 1;  // the count\nconst char* s = "x // y";\n'
    assert bench.strip_comments(base) == bench.strip_comments(
        '/* header */\nint a = 1;\n\nconst char* s = "x // y";  // note\n')
    assert bench.strip_comments(base) != bench.strip_comments(base.replace("1;", "2;"))
    assert bench.strip_comments(base) != bench.strip_comments(base.replace("x // y", "x // z"))

