"""The CUDA kernels compute some steps in a different order or form than the oracle does. These CPU
tests restate those forms in Python, from their description in the kernel sources, and check them
against the oracle on random inputs, so that each reformulation is shown to give the oracle's
result exactly (the GPU parity tests then check the kernels themselves):

* the greedy state allocation with cached per-range gains and a per-lane tournament
  (build_tables.cu, normalize_warp, used at L <= 128) against the oracle's sequential greedy;
* the same allocation computed as a threshold on the gains (build_tables.cu, normalize_block, used
  from L = 256: bisection on the M-th largest gain, per-range counts from an estimate corrected in
  unit steps, ties in range order) against the oracle's sequential greedy, and the premise that
  makes it exact: the fixed-point LG differences never increase;
* the range DP restricted to the end points that can still lie on a split into K non-empty
  ranges (build_tables.cu) against the oracle's full DP;
* the decoder's ring-refill quad index, kept in 32 bits (decode.cu), against the plain formula;
* the encoder's bias trick for the renormalisation shift (encode.cu) against its definition;
* the decoder's multiply-high field extractions (decode.cu) against plain shifts;
* the decoder's per-slot table construction (modular inverse of the spread step, binary search,
  rank count; decode.cu) against the oracle's tables.
"""
import numpy as np
import pytest

INF = 1 << 80


def lg_table(orc, L):
    return [orc.lg(f) for f in range(L + 2)]


def tournament_greedy(N, R, lgf):
    """Lane l holds ranges l + 32 r (r < kPer); every lane caches the gain of each of its ranges and
    its best (largest gain, then smallest k, by a left-priority tournament); a step is a warp argmax
    over the lanes' bests (largest gain, then smallest k); only the winner's gain is recomputed."""
    K = len(N)
    L = 1 << R
    kper = 1 if K <= 32 else 2 if K <= 64 else 4 if K <= 128 else 8
    n = [int(N[k]) if k < K else 0 for k in range(32 * kper)]
    f = [1 if v > 0 else 0 for v in n]
    if sum(n) == 0:
        out = [0] * K
        out[0] = L
        return out

    def gain(k):
        return n[k] * (lgf[f[k] + 1] - lgf[f[k]]) if n[k] > 0 and f[k] < L else 0

    G = [gain(k) for k in range(32 * kper)]

    def lane_best(lane):
        gv = [G[lane + 32 * r] for r in range(kper)]
        kv = [lane + 32 * r for r in range(kper)]
        w = 1
        while w < kper:
            for r in range(0, kper - w, 2 * w):
                if gv[r + w] > gv[r]:
                    gv[r], kv[r] = gv[r + w], kv[r + w]
            w *= 2
        return gv[0], (kv[0] if gv[0] > 0 else None)

    best = [lane_best(lane) for lane in range(32)]
    for _ in range(L - sum(f)):
        top = max(g for g, _ in best)
        win = min(k for g, k in best if g == top and k is not None)
        f[win] += 1
        G[win] = gain(win)
        best[win & 31] = lane_best(win & 31)
    return f[:K]


@pytest.mark.parametrize("seed", range(40))
def test_tournament_greedy_matches_oracle(orc, seed):
    """The kernel uses this form at L <= 128 (so K <= 128)."""
    rng = np.random.default_rng(seed)
    K = int(rng.choice([1, 3, 16, 31, 33, 64, 100, 128]))
    R = int(rng.integers(max(4, int(np.ceil(np.log2(K)))), 8))
    top = min(1 << int(rng.choice([6, 20, 31])), (1 << 32) // (K + 1))  # the total stays below 2^32
    pool = rng.integers(1, top, 4)  # few distinct counts: many ties
    N = rng.choice(np.concatenate([[0, 0, 1], pool]), K).astype(np.uint64)
    if int((N > 0).sum()) > (1 << R):
        N[(1 << R):] = 0
    expect = orc.normalize(N, R)
    got = tournament_greedy(N, R, lg_table(orc, 1 << R))
    assert list(expect) == got


def threshold_allocation(N, R, lgf):
    """The kernel's form: every range with a count starts with one state; the M = L - nonzero further
    states are the M first elements (k, f) in the order (gain down, k up, f up), gain =
    N_k (LG(f+1) - LG(f)) for f = 1 .. L-1: all elements above the M-th largest gain v, found by
    bisection on the gain, then the elements equal to v in range order. A range's count above a
    trial value starts from N 2^24 / (tau ln 2) and is corrected in unit steps."""
    K = len(N)
    L = 1 << R
    n = [int(v) for v in N]
    nonzero = sum(1 for v in n if v > 0)
    if nonzero == 0:
        return [L] + [0] * (K - 1)
    M = L - nonzero

    def gain(k, f):
        return n[k] * (lgf[f + 1] - lgf[f])

    def count_gt(k, tau):
        if n[k] == 0:
            return 0
        est = float(np.float32(n[k]) * np.float32(24204406.32) / np.float32(max(tau, 1)))
        f = L - 1 if est >= L - 1 else int(est)
        while f + 1 <= L - 1 and gain(k, f + 1) > tau:
            f += 1
        while f >= 1 and gain(k, f) <= tau:
            f -= 1
        return f

    f = [1 if v > 0 else 0 for v in n]
    if M > 0:
        lo, hi = 0, max(gain(k, 1) for k in range(K) if n[k] > 0)
        while hi - lo > 1:
            mid = lo + (hi - lo) // 2
            if sum(count_gt(k, mid) for k in range(K)) >= M:
                lo = mid
            else:
                hi = mid
        v = hi
        above = [count_gt(k, v) for k in range(K)]
        r = M - sum(above)
        seen = 0
        for k in range(K):
            e = count_gt(k, v - 1) - above[k]
            take = 0 if seen >= r else min(e, r - seen)
            seen += e
            if n[k] > 0:
                f[k] = 1 + above[k] + take
    return f


def test_lg_differences_never_increase(orc):
    """The premise of the threshold form: LG(f+1) - LG(f) is non-increasing for f = 1 .. 4096, so
    every range's gain sequence is non-increasing (the greedy then takes each range's elements in
    order, and its picks are a prefix of one global order)."""
    lgf = lg_table(orc, 4096)
    d = [lgf[f + 1] - lgf[f] for f in range(1, 4097)]
    assert all(d[i + 1] <= d[i] for i in range(len(d) - 1))
    assert any(d[i + 1] == d[i] for i in range(len(d) - 1))  # equal neighbours exist: ties within a range


@pytest.mark.parametrize("seed", range(60))
def test_threshold_allocation_matches_oracle(orc, seed):
    rng = np.random.default_rng(seed)
    K = int(rng.choice([1, 3, 16, 31, 33, 64, 100, 129, 200, 256]))
    R = int(rng.integers(max(4, int(np.ceil(np.log2(K)))), 13))
    top = min(1 << int(rng.choice([6, 20, 31])), (1 << 32) // (K + 1))  # the total stays below 2^32
    mode = seed % 3
    if mode == 0:  # few distinct counts: many ties between ranges
        pool = rng.integers(1, top, 4)
        N = rng.choice(np.concatenate([[0, 0, 1], pool]), K).astype(np.uint64)
    elif mode == 1:
        N = rng.integers(0, top, K).astype(np.uint64)
    else:  # one dominant range: thousands of states on it, where neighbouring gains can be equal
        N = rng.integers(0, 4, K).astype(np.uint64)
        N[rng.integers(0, K)] = top
    if int((N > 0).sum()) > (1 << R):
        N[(1 << R):] = 0
    expect = orc.normalize(N, R)
    got = threshold_allocation(N, R, lg_table(orc, 1 << R))
    assert list(expect) == got


def banded_dp(orc, h, K):
    """The kernel's layer order: D[i][k] = min over j in [k-1, i-1] of D[j][k-1] + Cost(j, i), ties to
    the smallest j, computed only for k <= i <= 256 - (K - k); backtrack from D[256][K]."""
    A = len(h)
    pre = np.concatenate([[0], np.cumsum(h.astype(np.int64))])
    lgs = {}

    def cost(j, i):
        c = int(pre[i] - pre[j])
        if c == 0:
            return 0
        if c not in lgs:
            lgs[c] = orc.lg(c)
        width = i - j
        w = 0 if width <= 1 else int(width - 1).bit_length()
        return c * ((w << 24) - lgs[c])

    prev = [0] + [INF] * A
    arg = []
    for k in range(1, K + 1):
        cur = [INF] * (A + 1)
        a_k = {}
        for i in range(k, A - (K - k) + 1):
            best, bj = INF, None
            for j in range(k - 1, i):
                if prev[j] >= INF:
                    continue
                v = prev[j] + cost(j, i)
                if v < best:
                    best, bj = v, j
            cur[i], a_k[i] = best, bj
        arg.append(a_k)
        prev = cur
    lo, i = [0] * K, A
    for k in range(K, 0, -1):
        j = arg[k - 1][i]
        lo[k - 1] = j
        i = j
    return lo, prev[A]


@pytest.mark.parametrize("seed,K", [(0, 1), (1, 2), (2, 5), (3, 8), (4, 12), (5, 15), (6, 16)])
def test_banded_dp_matches_oracle_small_alphabet(orc, seed, K):
    # a 16-symbol alphabet keeps the pure-Python DP fast while every band edge is exercised
    rng = np.random.default_rng(100 + seed)
    h = rng.choice([0, 0, 1, 7, 1000, 123456], 16).astype(np.uint64)
    lo_o, cost_o = orc.partition(h, K)
    lo, cost = banded_dp(orc, h, K)
    assert cost == cost_o and lo == [int(v) for v in lo_o]


def test_banded_dp_matches_oracle_full_alphabet(orc):
    rng = np.random.default_rng(7)
    v = np.clip(np.round(rng.laplace(0, 9, 20000)), -128, 127).astype(np.int64) + 128
    h = np.bincount(v, minlength=256).astype(np.uint64)
    for K in (250, 255, 256):  # narrow bands, where the restriction drops most cells
        lo_o, cost_o = orc.partition(h, K)
        lo, cost = banded_dp(orc, h, K)
        assert cost == cost_o and lo == [int(x) for x in lo_o], K


def test_refill_quad_index_in_32_bits():
    """quad((cb / 4 + t)) = (cb / 4 + t) >> 2 equals (cb >> 4) + (((cb >> 2) & 3) + t) >> 2 for 4-byte
    aligned chunk starts cb anywhere below 32 GiB and window words t, negative ones included (Python
    >> floors like an arithmetic shift)."""
    rng = np.random.default_rng(3)
    cbs = [4 * int(x) for x in rng.integers(0, (32 << 30) // 4, 2000)] + [0, 4, 8, 12, (32 << 30) - 4]
    for cb in cbs:
        for t in (-3, -1, 0, 1, 2, 3, 5, 1000, 16383):
            plain = ((cb >> 2) + t) >> 2
            split = (cb >> 4) + ((((cb >> 2) & 3) + t) >> 2)
            assert plain == split
            assert -(1 << 31) <= (cb >> 4) < (1 << 31)  # the quad base itself fits the int32 it is kept in


def test_encoder_bias_trick_gives_the_defined_shift():
    """The encoder takes nb = (X + bias) >> 16 with bias = ((R - a) << 16) - (f << (R - a)),
    a = floor(log2 f); the oracle takes nb by its definition, the smallest shift with X >> nb < 2f.
    Exhaustive over every count f and state X in [L, 2L) for L = 16 ... 4096."""
    for R in range(4, 13):
        L = 1 << R
        X = np.arange(L, 2 * L, dtype=np.int64)
        for f in range(1, L + 1):
            a = f.bit_length() - 1
            bias = ((R - a) << 16) - (f << (R - a))
            nb = (X + bias) >> 16
            assert np.all((X >> nb) < 2 * f) and np.all((X >> nb) >= f), (R, f)
            # smallest such shift: one bit less would leave the state at or above 2f
            assert np.all((nb == 0) | ((X >> np.maximum(nb - 1, 0)) >= 2 * f)), (R, f)


def test_decoder_multiply_high_field_extraction():
    """The decoder reads the fields of a table entry's second word with multiply-highs: y >> 8 as
    mulhi(y, 2^24), (y >> 16) + a as mad.hi(y, 2^16, a), and the signed top byte added to the bit
    position as mad.hi.s32(y, 2^8, p). Checked against the plain shifts on random words."""
    rng = np.random.default_rng(11)
    for y in [int(v) for v in rng.integers(0, 1 << 32, 5000, dtype=np.uint64)] + [0, 0xFFFFFFFF, 0x80000000, 0x7FFFFFFF]:
        assert (y * (1 << 24)) >> 32 == y >> 8
        a = int(rng.integers(0, 1 << 16))
        assert ((y * (1 << 16)) >> 32) + a == (y >> 16) + a
        ys = y - (1 << 32) if y >> 31 else y          # the word as a signed 32-bit value
        p = int(rng.integers(0, 1 << 20))
        top = (y >> 24) - 256 if (y >> 24) & 0x80 else (y >> 24)  # (int8)(y >> 24)
        assert ((ys * 256) >> 32) + p == p + top


def gpu_decode_slot(i, R, f, cumul):
    """The decoder's table build computes each slot independently: the placement index tau of slot
    i from the modular inverse of the spread step, the range of tau by binary search over the
    cumulative counts, the slot's rank among its range's slots by counting placements below i."""
    L = 1 << R
    step = (L >> 1) + (L >> 3) + 3
    inv = pow(step, -1, 1 << 32)
    tau = (i * inv) & (L - 1)
    a, b = 0, len(f) - 1
    while a < b:
        m = (a + b + 1) >> 1
        if cumul[m] <= tau:
            a = m
        else:
            b = m - 1
    s = a
    rank = sum(1 for u in range(cumul[s], cumul[s] + f[s]) if ((u * step) & (L - 1)) < i)
    x = f[s] + rank
    nb = R - (x.bit_length() - 1)
    return s, nb, (x << nb) - L


@pytest.mark.parametrize("seed", range(12))
def test_decoder_slot_construction_matches_oracle_tables(orc, seed):
    rng = np.random.default_rng(500 + seed)
    R = int(rng.integers(4, 11))
    L = 1 << R
    K = int(rng.integers(1, min(L, 256) + 1))
    f = np.zeros(K, np.int64)  # a random composition of L into K parts, empty ranges allowed
    for u in rng.integers(0, K, L):
        f[u] += 1
    lo = np.sort(rng.choice(np.arange(1, 256), K - 1, replace=False)) if K > 1 else np.zeros(0, int)
    lo = np.concatenate([[0], lo]).astype(np.uint16)
    t = orc.tables(lo, f.astype(np.uint32), R)
    cumul = np.concatenate([[0], np.cumsum(f)])[:K].tolist()
    fl = f.tolist()
    for i in range(L):
        s, nb, nxt = gpu_decode_slot(i, R, fl, cumul)
        assert (s, nb, nxt) == (t.dec_sym[i], t.dec_nb[i], t.dec_next[i]), (R, K, i)
