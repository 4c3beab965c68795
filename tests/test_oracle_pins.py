"""Pins of the CPU oracle against what the mathematics and the paper fix (no GPU).

"Shannonic: Efficient Entropy-Optimal Compression for ML Workloads" (MLSys 2026 notes):
  §4.1 DP range selection   → brute force over every contiguous partition of small alphabets,
                               compared on the real-valued objective (fp64 log2).
  §4.1 state counts          → brute force over every composition of L for tiny K, L.
  fixed-point log2           → bound against math.log2, exact at powers of two.
  §4.2 Algorithm 2           → round trip; K=1 (raw offsets, pins the bit order); forced uniform
                               table (every symbol exactly 4+4 bits); a single distinct value
                               (0 payload bits); an independent bit-by-bit reader of the SHN1 format.
  §4 Theorem 1               → rate closes to the closed form within 0.01 bit; the i.i.d. rate
                               matches the exact stationary rate of the tANS state chain.
  §4 Condition 3             → its sign predicts which of Shannonic / plain tANS is shorter.
  §5 "within 1% of H"        → K=16, L=128 on the ~5.3-bit distributions.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from entropy_coded_lossless_b200 import inputs
from tests import spec


# ----------------------------------------------------------------------------------------------
# fixed-point log2


def test_lg_exact_at_powers_of_two(orc):
    for k in range(32):
        assert orc.lg(1 << k) == k << 24
    assert orc.lg(0) == 0


def test_lg_bound_against_log2(orc):
    rng = np.random.default_rng(0)
    ns = list(range(1, 5000)) + [int(v) for v in rng.integers(1, 1 << 32, 20000, dtype=np.uint64)]
    ns += [(1 << k) + d for k in range(2, 32) for d in (-1, 1) if (1 << k) + d < (1 << 32)]
    worst = 0.0
    for n in ns:
        err = math.log2(n) - orc.lg(n) / 2.0 ** 24
        assert err > -1e-12, n
        worst = max(worst, err)
    assert worst < 2.0 ** -24 * (1 + 2.0 ** -6), worst


# ----------------------------------------------------------------------------------------------
# histogram


def test_histogram_matches_bincount(orc):
    rng = np.random.default_rng(1)
    x = rng.integers(-128, 128, 100_003).astype(np.int8)
    h = orc.histogram(x)
    ref = np.bincount(x.view(np.uint8) ^ 0x80, minlength=256)
    assert (h == ref).all() and h.sum() == x.size


# ----------------------------------------------------------------------------------------------
# DP range selection vs brute force


def _all_partitions(A, K):
    for cuts in itertools.combinations(range(1, A), K - 1):
        yield [0, *cuts, A]


def _random_hist(rng, A):
    kind = rng.integers(0, 4)
    if kind == 0:
        h = rng.integers(0, 1000, A)
    elif kind == 1:
        h = rng.integers(0, 3, A) * rng.integers(0, 50, A)
    elif kind == 2:
        c = rng.integers(0, A)
        h = (1000 * np.exp(-np.abs(np.arange(A) - c) / rng.uniform(0.5, 4))).astype(np.int64)
    else:
        h = np.zeros(A, np.int64)
        h[rng.integers(0, A, 3)] = rng.integers(1, 10_000, 3)
    return h.astype(np.uint64)


@pytest.mark.parametrize("A", [4, 6, 9, 12, 16])
def test_dp_is_optimal_by_brute_force(orc, A):
    rng = np.random.default_rng(100 + A)
    for _ in range(12):
        h = _random_hist(rng, A)
        n = int(h.sum())
        for K in range(1, min(A, 6) + 1):
            lo, cost = orc.partition(h, K)
            bounds = [int(v) for v in lo] + [A]
            assert bounds[0] == 0 and all(a < b for a, b in zip(bounds[:-1], bounds[1:]))
            got = spec.ideal_partition_cost_bits(h, bounds)
            best = min(spec.ideal_partition_cost_bits(h, p) for p in _all_partitions(A, K))
            # fixed-point log2 is within 2^-24 bit per value of the real one
            assert got <= best + 2 * n * 2.0 ** -24 + 1e-9, (h, K, bounds)
            assert abs(cost / 2.0 ** 24 - got) <= 2 * n * 2.0 ** -24 + 1e-6


def test_dp_special_cases(orc):
    rng = np.random.default_rng(7)
    h = rng.integers(0, 100, 256).astype(np.uint64)
    lo, _ = orc.partition(h, 1)
    assert list(lo) == [0]
    lo, _ = orc.partition(h, 256)
    assert list(lo) == list(range(256))
    # all-zero histogram: every partition costs 0, smallest-j tie-break gives lo = 0..K-1
    lo, cost = orc.partition(np.zeros(256, np.uint64), 16)
    assert cost == 0 and list(lo) == list(range(16))


def test_dp_uniform_histogram_value(orc):
    # every partition into power-of-two-width ranges costs exactly 8n bits in total coded size;
    # the DP objective is 8n - n*log2(n) up to LG rounding
    h = np.full(256, 1000, np.uint64)
    n = 256000
    lo, cost = orc.partition(h, 16)
    total_bits = cost / 2.0 ** 24 + n * math.log2(n)
    assert abs(total_bits - 8 * n) < 1e-3 * n


# ----------------------------------------------------------------------------------------------
# state counts vs brute force


def _compositions(total, parts):
    if parts == 1:
        yield (total,)
        return
    for first in range(total + 1):
        for rest in _compositions(total - first, parts - 1):
            yield (first,) + rest


@pytest.mark.parametrize("R", [2, 3, 4])
def test_normalize_is_optimal_by_brute_force(orc, R):
    L = 1 << R
    rng = np.random.default_rng(R)
    for _ in range(40):
        K = int(rng.integers(1, 5))
        N = rng.integers(0, 1000, K).astype(np.uint64)
        if rng.random() < 0.3:
            N[rng.integers(0, K)] = 0
        if (N > 0).sum() == 0 or (N > 0).sum() > L:
            continue
        f = orc.normalize(N, R)
        assert f.sum() == L and ((f > 0) == (N > 0)).all()

        def obj(fv):
            return sum(float(N[k]) * math.log2(fv[k]) for k in range(K) if N[k] > 0)

        best = max(obj(c) for c in _compositions(L, K) if all((c[k] > 0) == (N[k] > 0) for k in range(K)))
        assert obj(f) >= best - 1e-6 * max(1.0, abs(best))


def test_normalize_invariants_large(orc):
    rng = np.random.default_rng(5)
    for R in (4, 7, 10, 12):
        for _ in range(10):
            K = int(rng.integers(1, 64))
            N = (rng.pareto(1.2, K) * 1000).astype(np.uint64)
            N[rng.random(K) < 0.2] = 0
            if (N > 0).sum() == 0:
                N[0] = 1
            if (N > 0).sum() > 1 << R:
                with pytest.raises(orc.OracleError):
                    orc.normalize(N, R)
                continue
            f = orc.normalize(N, R)
            assert f.sum() == 1 << R and ((f > 0) == (N > 0)).all()
    f = orc.normalize(np.zeros(5, np.uint64), 7)
    assert list(f) == [128, 0, 0, 0, 0]


# ----------------------------------------------------------------------------------------------
# tables


def test_tables_structure_and_inverse(orc):
    rng = np.random.default_rng(11)
    for R in (4, 7, 8, 10):
        L = 1 << R
        for K in (1, 3, 16):
            N = rng.integers(0, 500, K).astype(np.uint64)
            N[0] = max(int(N[0]), 1)
            f = orc.normalize(N, R)
            lo = np.sort(rng.choice(np.arange(1, 256), K - 1, replace=False)) if K > 1 else np.zeros(0)
            lo = np.concatenate([[0], lo]).astype(np.uint16)
            t = orc.tables(lo, f, R)
            spread = np.array(t.spread[:L])
            assert (np.bincount(spread, minlength=K)[:K] == f).all()
            # the spread and decode rows equal an independent reading of SHN1 format §5
            s_ref, dec_ref = spec.spec_tables([int(v) for v in lo], [int(v) for v in f], R)
            assert list(spread) == s_ref
            assert [(t.dec_sym[i], t.dec_nb[i], t.dec_next[i]) for i in range(L)] == dec_ref
            # encoder transition followed by the decoder row returns the original state
            for s in range(K):
                if f[s] == 0:
                    continue
                for X in range(L, 2 * L):
                    nb = 0
                    while (X >> nb) >= 2 * int(f[s]):
                        nb += 1
                    Xn = t.enc[t.cumul[s] + (X >> nb) - int(f[s])]
                    slot = Xn - L
                    assert t.dec_sym[slot] == s and t.dec_nb[slot] == nb
                    assert L + t.dec_next[slot] + (X & ((1 << nb) - 1)) == X


# ----------------------------------------------------------------------------------------------
# encoder / decoder


def _roundtrip(orc, x, **kw):
    stream, stats = orc.encode(x, **kw)
    rc, y = orc.decode(stream)
    assert rc == 0
    assert np.array_equal(y, np.asarray(x).view(np.uint8).reshape(-1))
    return stream, stats


def test_roundtrip_many(orc):
    rng = np.random.default_rng(3)
    for trial in range(30):
        n = int(rng.integers(0, 3000))
        b = float(rng.choice([0.3, 2.0, 7.0, 60.0]))
        x = inputs.laplace_int8(n, b, seed=trial).numpy()
        K = int(rng.choice([1, 2, 8, 16, 32]))
        R = int(rng.choice([4, 5, 7, 8, 10]))
        if K > (1 << R):
            continue
        S = int(rng.choice([1, 2, 4, 8, 16]))
        C = int(rng.choice([128, 256, 1024]))
        cuts = sorted(rng.integers(0, n + 1, int(rng.integers(0, 4))).tolist()) if n else []
        b_ = [0, *cuts, n]
        segs = [(a, c - a) for a, c in zip(b_[:-1], b_[1:])]
        _roundtrip(orc, x, K=K, R=R, S=S, C=C, segments=segs)


def test_roundtrip_plain_tans_and_full_alphabet(orc):
    x = np.arange(-128, 128, dtype=np.int8).repeat(40)
    np.random.default_rng(0).shuffle(x)
    _roundtrip(orc, x, K=256, R=10, S=4, C=1024)
    _roundtrip(orc, x, K=16, R=7, S=4, C=1024)


def test_k1_payload_is_reversed_raw_bytes(orc):
    # K=1: one range [0,256), w=8, f=L, nb=0: each chunk holds the offsets u_{c-1} .. u_0 as
    # whole bytes, then S zero states of R bits, then the sentinel
    x = inputs.laplace_int8(3000, 20.0, seed=9).numpy()
    stream, stats = orc.encode(x, K=1, R=7, S=4, C=1024)
    st = spec.parse_stream(stream)
    u = x.view(np.uint8) ^ 0x80
    for c in range(3):
        words = spec.chunk_words(st, 0, c)
        seg = u[spec.chunk_positions(x.size, 1024, c)]
        raw = words.tobytes()
        assert raw[: seg.size] == seg[::-1].tobytes()
        rest = int.from_bytes(raw[seg.size:], "little")
        assert rest == 1 << (4 * 7)  # zero states, sentinel right after them
    assert stats[0].payload_bits == 8 * x.size


def test_forced_uniform_table_costs_exactly_8_bits(orc):
    # 16 ranges of width 16 with f=8 at L=128: x in [8,16) so nb = 7-3 = 4, w = 4
    x = inputs.laplace_int8(5000, 40.0, seed=2).numpy()
    lo = np.arange(0, 256, 16, dtype=np.uint16)
    f = np.full(16, 8, np.uint32)
    stream, stats = orc.encode(x, K=16, R=7, S=4, C=1024, lo=lo, f=f)
    assert stats[0].payload_bits == 8 * x.size
    rc, y = orc.decode(stream)
    assert rc == 0 and np.array_equal(y, x.view(np.uint8))


def test_single_value_has_empty_payload(orc):
    x = np.full(10_000, -3, np.int8)
    stream, stats = _roundtrip(orc, x, K=16, R=7, S=4, C=1024)
    assert stats[0].payload_bits == 0


def test_chunk_mapping_partitions_each_segment():
    """SHN1 format §6: the chunks of a segment hold every symbol exactly once, at most C each, and in
    a full group of 32 the k-th pieces of the chunks are 512 consecutive symbols."""
    for n, C in [(0, 128), (1, 128), (128, 128), (129, 128), (5000, 256), (32 * 256, 256), (33 * 256 + 7, 256),
                 (70 * 1024 + 3, 1024), (1_000_003, 4096)]:
        nch = -(-n // C)
        seen = np.zeros(n, np.int64)
        for c in range(nch):
            pos = spec.chunk_positions(n, C, c)
            assert 0 < len(pos) <= C
            seen[pos] += 1
        assert (seen == 1).all()
        if n >= 32 * C:
            firsts = [spec.chunk_positions(n, C, c)[16 * 3] for c in range(32)]
            assert firsts == list(range(firsts[0], firsts[0] + 512, 16))


def test_independent_reader_decodes_oracle_stream(orc):
    rng = np.random.default_rng(4)
    for trial in range(4):
        x = inputs.laplace_int8(700, float(rng.choice([1.0, 6.0, 30.0])), seed=50 + trial).numpy()
        K, R, S = [(16, 7, 4), (8, 5, 2), (256, 8, 1), (3, 4, 16)][trial]
        stream, _ = orc.encode(x, K=K, R=R, S=S, C=256, segments=[(0, 300), (300, 400)])
        st = spec.parse_stream(stream)
        assert st["stream_bytes"] == len(stream) and len(stream) % 16 == 0
        u = x.view(np.uint8) ^ 0x80
        for si, sg in enumerate(st["segments"]):
            nch = -(-sg["n"] // 256)
            for c in range(nch):
                pos = sg["out_offset"] + np.array(spec.chunk_positions(sg["n"], 256, c), dtype=np.int64)
                got, ok = spec.spec_decode_chunk(spec.chunk_words(st, si, c), sg["lo"], sg["f"], R, S, pos.size)
                assert ok and got == u[pos].tolist()


def test_corruption_is_reported(orc):
    """Structural damage (header, index, sentinel, truncation) is always an error. A flipped
    payload bit is caught when it disturbs the tANS state chain (end-state / position check);
    a flip inside a raw offset field only changes that value, since offsets carry no redundancy."""
    x = inputs.laplace_int8(20_000, 7.0, seed=1).numpy()
    stream, _ = orc.encode(x, K=16, R=7, S=4, C=1024)
    st = spec.parse_stream(stream)
    assert orc.decode(stream[:100])[0] != 0
    assert orc.decode(stream[: st["payload_offset"] + 64])[0] != 0
    bad = stream.copy()
    bad[0] ^= 1
    assert orc.decode(bad)[0] != 0
    bad = stream.copy()
    bad[st["index_offset"] + 4 * 3: st["index_offset"] + 4 * 4] = 0xFF
    assert orc.decode(bad)[0] != 0
    # remove chunk 2's sentinel word
    sg = st["segments"][0]
    end = st["payload_offset"] + sg["payload_start"] + 4 * int(st["index"][3])
    bad = stream.copy()
    bad[end - 4:end] = 0
    assert orc.decode(bad)[0] != 0
    rng = np.random.default_rng(0)
    detected = 0
    trials = 60
    for _ in range(trials):
        bad = stream.copy()
        pos = int(rng.integers(st["payload_offset"], len(stream) - 16))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        rc, y = orc.decode(bad)
        detected += rc != 0
    assert detected >= int(0.25 * trials)


# ----------------------------------------------------------------------------------------------
# rates: Theorem 1, the exact tANS chain rate, Condition 3, "within 1% of H"


def _rate(orc, x, **kw):
    stream, stats = orc.encode(x, **kw)
    bits = sum(s.payload_bits for s in stats)
    return bits / x.size, stream, stats


def test_theorem1_closure_config1(orc):
    x = inputs.laplace_int8(65536, inputs.LAPLACE_B_FOR_ENTROPY[5.3], seed=0).numpy()
    rp, _, stats = _rate(orc, x, K=16, R=7, S=4, C=4096)
    st = stats[0]
    th = spec.theorem1_terms(np.array(st.hist[:]), list(st.lo[:16]), list(st.f[:16]), 7)
    assert abs(rp - th["CL"]) <= 0.01
    assert rp <= 1.01 * th["H"]


def test_theorem1_closure_and_target_weight_like(orc):
    x = inputs.weight_like_int8(seed=1).numpy()
    rp, _, stats = _rate(orc, x, K=16, R=7, S=4, C=4096, threads=4)
    st = stats[0]
    th = spec.theorem1_terms(np.array(st.hist[:]), list(st.lo[:16]), list(st.f[:16]), 7)
    assert abs(rp - th["CL"]) <= 0.01
    assert rp <= 1.01 * th["H"]
    # §4 Condition 3 vs the measured plain tANS (K=256 identity ranges, L=1024)
    rp_t, _, stats_t = _rate(orc, x, K=256, R=10, S=4, C=4096, threads=4)
    th_t = spec.theorem1_terms(np.array(stats_t[0].hist[:]), list(range(256)), list(stats_t[0].f[:256]), 10)
    lhs = th_t["DKL"] - th["DKL"]
    rhs = th["offset"] - th["H_given_P"]
    assert (lhs > rhs) == (rp < rp_t)
    assert rp < rp_t


def test_theorem1_closure_activation_tensors(orc):
    x, segs, fam = inputs.activation_batch_int8(n_tensors=12, n=65536, seed=3)
    x = x.numpy()
    stream, stats = orc.encode(x, K=16, R=7, S=4, C=4096, segments=segs, threads=4)
    for st in stats:
        th = spec.theorem1_terms(np.array(st.hist[:]), list(st.lo[:16]), list(st.f[:16]), 7)
        assert abs(st.payload_bits / 65536 - th["CL"]) <= 0.01


def _chain_rate(t, P, R):
    """Exact expected renormalisation bits per symbol of the encoder's state chain (i.i.d. ranges)."""
    L = 1 << R
    K = len(P)
    T = np.zeros((L, L))
    bits = np.zeros(L)
    for s in range(K):
        if P[s] == 0:
            continue
        fs = int(t.f[s])
        for X in range(L, 2 * L):
            nb = 0
            while (X >> nb) >= 2 * fs:
                nb += 1
            Xn = t.enc[t.cumul[s] + (X >> nb) - fs]
            T[X - L, Xn - L] += P[s]
            bits[X - L] += P[s] * nb
    pi = np.full(L, 1.0 / L)
    for _ in range(5000):
        pi = pi @ T
    return float(pi @ bits)


def test_iid_rate_matches_exact_chain_rate(orc):
    n = 1 << 20
    x = inputs.laplace_int8(n, inputs.LAPLACE_B_FOR_ENTROPY[5.3], seed=21).numpy()
    rp, _, stats = _rate(orc, x, K=16, R=7, S=1, C=65536)
    st = stats[0]
    lo = list(st.lo[:16])
    f = list(st.f[:16])
    h = np.array(st.hist[:], dtype=np.float64)
    bounds = lo + [256]
    P = np.array([h[bounds[k]:bounds[k + 1]].sum() for k in range(16)]) / n
    t = orc.tables(np.array(lo, np.uint16), np.array(f, np.uint32), 7)
    expect = _chain_rate(t, P, 7) + sum(P[k] * spec.width_bits(lo, k) for k in range(16))
    # per-symbol bit count has std < 3 bits; 4 sigma of the mean, plus the per-chunk start transient
    assert abs(rp - expect) <= 4 * 3.0 / math.sqrt(n) + 0.002


@pytest.mark.parametrize("H", [5.3])
def test_rate_within_one_percent_k16_l128(orc, H):
    x = inputs.laplace_int8(1 << 20, inputs.LAPLACE_B_FOR_ENTROPY[H], seed=4).numpy()
    rp, _, stats = _rate(orc, x, K=16, R=7, S=4, C=4096, threads=4)
    h = spec.entropy_bits(np.array(stats[0].hist[:]))
    assert rp <= 1.01 * h, (rp, h)


def test_worked_example_accounting_closes():
    """The §4 worked example's printed numbers obey the Theorem 1 decomposition used by
    spec.theorem1_terms: tANS = H + D_KL(p||q); Shannonic = H + D_KL(P||Q) + (offset − H(p|P))."""
    g = {}
    for line in open(__file__.replace("test_oracle_pins.py", "golden/worked_example.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, v = line.split("=")
            g[k.strip()] = float(v)
    assert abs(g["H"] + g["tans_quant_loss"] - g["tans_L1024_bits"]) <= 0.001
    assert abs(g["H"] + g["shannonic_quant_loss"] + g["shannonic_offset_cost"] - g["shannonic_K16_L128_bits"]) <= 0.0015
    # the same decomposition holds exactly on a synthetic histogram
    x = inputs.laplace_int8(50_000, 5.0, seed=8).numpy()
    hist = np.bincount(x.view(np.uint8) ^ 0x80, minlength=256)
    lo = [0, 100, 120, 124, 126, 127, 128, 129, 130, 132, 136, 140, 150, 170, 200, 230]
    f = [1, 4, 6, 8, 14, 16, 20, 16, 14, 8, 6, 5, 4, 3, 2, 1]
    th = spec.theorem1_terms(hist, lo, f, 7)
    assert abs(th["CL"] - (th["H"] + th["DKL"] + (th["offset"] - th["H_given_P"]))) < 1e-9
    assert th["offset"] >= th["H_given_P"] - 1e-12
