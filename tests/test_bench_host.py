"""Host-side helpers of bench.py (no GPU): the kernel-launch count it claims per step, and the
comment-insensitive source digests that decide whether a measured DRAM-traffic figure still
belongs to the kernel source it was captured from."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    sys.argv = ["bench"]
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench as b

    return b


def test_launch_count_follows_batching(bench):
    from entropy_coded_lossless_b200 import inputs

    c4k = {"chunk_symbols": 4096}
    # KV cache: 64 large segments, one encoder batch: histogram, build, write, scan x3, header,
    # compaction, check, decode
    assert bench.kernel_launches_per_step(inputs.kv_cache_segments(), c4k) == 10
    # 1024 small tensors: two histogram launches, the LG-table fill, two encoder batches
    act = [(i * 65536, 65536) for i in range(1024)]
    assert bench.kernel_launches_per_step(act, c4k) == 2 + 1 + 1 + 3 + 1 + 2 + 2 * 2
    # a kind change starts a new encoder batch: large, small, large -> three batches
    mixed = [(0, 1 << 20), (1 << 20, 4096), (2 << 20, 1 << 20)]
    assert bench.kernel_launches_per_step(mixed, c4k) == 1 + 1 + 3 + 1 + 2 + 2 * 3
    assert bench.kernel_launches_per_step([], c4k) == 0


def test_source_digest_ignores_comments(bench, tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    a.write_text("int f(int x) {\n  return x + 1;  // one more\n}\n")
    b.write_text("/* header */\nint f(int x) {\n\n  return x + 1;\n}\n")
    assert bench.source_digest(str(a)) == bench.source_digest(str(b))
    b.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.source_digest(str(a)) != bench.source_digest(str(b))


def test_measured_traffic_entries_are_well_formed(bench):
    for name, m in bench.MEASURED_TRAFFIC.items():
        assert set(m) == {"bytes_per_symbol", "source", "sha256_prefix"}, name
        assert os.path.exists(os.path.join(ROOT, "entropy_coded_lossless_b200", "csrc", m["source"])), name
        assert 0 < m["bytes_per_symbol"] < 8 and len(m["sha256_prefix"]) == 16, name
    # a stale digest yields no traffic figure rather than a wrong one
    saved = dict(bench.MEASURED_TRAFFIC["decode_kernel"])
    try:
        bench.MEASURED_TRAFFIC["decode_kernel"]["sha256_prefix"] = "0" * 16
        assert bench.measured_traffic(["decode_kernel"], 1 << 20) is None
    finally:
        bench.MEASURED_TRAFFIC["decode_kernel"] = saved


def test_rate_report_on_oracle_streams(bench, orc):
    """bench.py's host rate report (Shannonic §4 Theorem 1 terms, §5 %diff) read from an SHN1 stream
    the oracle wrote: its RP equals the oracle's own payload bit count, its entropy and Theorem-1
    terms equal the independent fp64 helpers of tests/spec.py on each segment's histogram and table,
    and the decomposition closes: RP - H = D_KL + offset excess + spread excess."""
    import numpy as np

    from entropy_coded_lossless_b200 import inputs
    from tests import spec

    x1 = inputs.laplace_int8(150_000, 7.258, seed=21).numpy()
    x2 = inputs.laplace_int8(90_001, 2.0, seed=22).numpy()
    x = np.concatenate([x1, x2])
    segs = [(0, x1.size), (x1.size, x2.size)]
    p = {"K": 16, "log2L": 7, "chunk_symbols": 4096, "states_per_chunk": 4}
    stream, stats = orc.encode(x, 16, 7, 4, 4096, segments=segs)
    hist = np.stack([np.ctypeslib.as_array(s.hist) for s in stats])
    r = bench.rate_report(stream, segs, p, hist)
    payload = sum(s.payload_bits for s in stats)
    assert abs(r["payload"] - payload / x.size) < 1e-12
    st = spec.parse_stream(stream)
    want = {"H": 0.0, "HP": 0.0, "DKL": 0.0, "offset": 0.0}
    for i, (o, n) in enumerate(segs):
        t = spec.theorem1_terms(hist[i], st["segments"][i]["lo"], st["segments"][i]["f"], 7)
        for k in want:
            want[k] += t[k] * n / x.size
    t1 = r["theorem1"]
    assert abs(t1["H"] - want["H"]) < 1e-9 and abs(r["entropy"] - want["H"]) < 1e-9
    assert abs(t1["H_P"] - want["HP"]) < 1e-9
    assert abs(t1["D_KL_P_Q"] - want["DKL"]) < 1e-9
    assert abs(t1["offset_bits"] - want["offset"]) < 1e-9
    closure = t1["D_KL_P_Q"] + t1["offset_excess"] + t1["spread_excess"]
    assert abs((r["payload"] - r["entropy"]) - closure) < 1e-9
    assert abs(t1["spread_excess"]) < 0.01  # Theorem 1 holds to within 0.01 bit
    # the per-segment mask selects segment 1 alone
    r2 = bench.rate_report(stream, segs, p, hist, mask=[False, True])
    assert abs(r2["payload"] - stats[1].payload_bits / x2.size) < 1e-12
