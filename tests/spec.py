"""Independent pure-Python reading of the SHN1 format specification and the paper's rate formulas, for tests.

Nothing here imports the oracle or the CUDA binding. It is a second, deliberately naive
implementation of the stream layout (SHN1 format §6), the tables (§5) and the decoder (§7), used on
small inputs to pin the oracle's bit order and field layout, plus fp64 helpers for the rate
measurements of "Shannonic: Efficient Entropy-Optimal Compression for ML Workloads" (§4 Theorem 1,
§5 %diff).
"""
import math
import struct

import numpy as np


def u32s(b):
    return np.frombuffer(bytes(b), dtype="<u4")


def parse_stream(buf):
    b = bytes(np.asarray(buf, dtype=np.uint8))
    (magic, ver, hbytes, nseg, K, R, S, C, tb, total_sym, total_ch, index_off, payload_off,
     stream_bytes) = struct.unpack_from("<IHHIHBBIIQQQQQ", b, 0)
    assert magic == 0x314E4853 and ver == 1 and hbytes == 64
    segs = []
    for s in range(nseg):
        n, out_off, pay_start, pay_words, first = struct.unpack_from("<QQQII", b, 64 + 32 * s)
        rec = 64 + 32 * nseg + tb * s
        f = list(struct.unpack_from(f"<{K}H", b, rec))
        lo = list(b[rec + 2 * K: rec + 3 * K])
        segs.append(dict(n=n, out_offset=out_off, payload_start=pay_start, payload_words=pay_words,
                         first_chunk=first, f=f, lo=lo))
    index = np.frombuffer(b, dtype="<u4", count=total_ch, offset=index_off) if total_ch else np.zeros(0, "<u4")
    return dict(K=K, R=R, S=S, C=C, table_bytes=tb, total_symbols=total_sym, total_chunks=total_ch,
                index_offset=index_off, payload_offset=payload_off, stream_bytes=stream_bytes,
                segments=segs, index=index, raw=b)


def chunk_positions(n, C, c):
    """SHN1 format §6: positions (relative to the segment start) of chunk c's symbols, in order."""
    nch = -(-n // C)
    grp, j = divmod(c, 32)
    m = min(32, nch - 32 * grp)
    base = 32 * grp * C
    ng = min(32 * (grp + 1) * C, n) - base
    P = -(-ng // 16)
    out = []
    for p in range(j, P, m):
        out.extend(base + 16 * p + t for t in range(16) if 16 * p + t < ng)
    return out


def chunk_words(st, seg_id, c):
    """Words of chunk c of segment seg_id (a numpy uint32 array)."""
    sg = st["segments"][seg_id]
    nch = -(-sg["n"] // st["C"])
    g = sg["first_chunk"] + c
    w0 = int(st["index"][g])
    w1 = int(st["index"][g + 1]) if c + 1 < nch else sg["payload_words"]
    start = st["payload_offset"] + sg["payload_start"] + 4 * w0
    return np.frombuffer(st["raw"], dtype="<u4", count=w1 - w0, offset=start)


def spec_tables(lo, f, R):
    """SHN1 format §5 written out directly: spread, decode rows (sym, nb, next) and encode rows."""
    L = 1 << R
    K = len(f)
    step = L // 2 + L // 8 + 3
    cumul = [sum(f[:k]) for k in range(K)]
    spread = [None] * L
    for k in range(K):
        for r in range(f[k]):
            spread[((cumul[k] + r) * step) % L] = k
    assert all(s is not None for s in spread)
    seen = [0] * K
    dec = []
    for i in range(L):
        s = spread[i]
        x = f[s] + seen[s]
        seen[s] += 1
        nb = R - (x.bit_length() - 1)
        dec.append((s, nb, (x << nb) - L))
    return spread, dec


def width_bits(lo, k):
    hi = lo[k + 1] if k + 1 < len(lo) else 256
    return (hi - lo[k] - 1).bit_length()


def spec_decode_chunk(words, lo, f, R, S, c):
    """SHN1 format §7 decoder, bit by bit. Returns (symbols u as a list, ok flag)."""
    L = 1 << R
    _, dec = spec_tables(lo, f, R)
    bits = []
    for w in words:
        for t in range(32):
            bits.append((int(w) >> t) & 1)
    P = max(i for i, v in enumerate(bits) if v)  # sentinel position

    def read(n):
        nonlocal P
        v = 0
        for t in range(n):
            v |= bits[P - n + t] << t
        P -= n
        return v

    X = [0] * S
    for q in range(S - 1, -1, -1):
        X[q] = L + read(R)
    out = []
    for i in range(c):
        q = i % S
        s, nb, nxt = dec[X[q] - L]
        r = read(nb)
        o = read(width_bits(lo, s))
        X[q] = L + nxt + r
        out.append((lo[s] + o) & 255)
    return out, (P == 0 and all(x == L for x in X))


def entropy_bits(hist):
    h = np.asarray(hist, dtype=np.float64)
    n = h.sum()
    p = h[h > 0] / n
    return float(-(p * np.log2(p)).sum())


def theorem1_terms(hist, lo, f, R):
    """§4 Theorem 1: CL = H(P) + D_KL(P||Q) + sum_k P_k w_k, with P the range probabilities,
    Q_k = f_k / L and w_k = ceil(log2 |R_k|). Also returns H(p) and H(p|P)."""
    h = np.asarray(hist, dtype=np.float64)
    n = h.sum()
    K = len(f)
    bounds = list(lo) + [256]
    P = np.array([h[bounds[k]:bounds[k + 1]].sum() for k in range(K)]) / n
    Q = np.asarray(f, dtype=np.float64) / (1 << R)
    w = np.array([width_bits(lo, k) for k in range(K)], dtype=np.float64)
    nz = P > 0
    HP = float(-(P[nz] * np.log2(P[nz])).sum())
    D = float((P[nz] * np.log2(P[nz] / Q[nz])).sum())
    off = float((P * w).sum())
    H = entropy_bits(h)
    return dict(H=H, HP=HP, DKL=D, offset=off, H_given_P=H - HP, CL=HP + D + off)


def ideal_partition_cost_bits(hist, bounds):
    """Real-valued DP objective sum_k [c_k w_k - c_k log2 c_k] for ranges [bounds[k], bounds[k+1])."""
    tot = 0.0
    for a, b in zip(bounds[:-1], bounds[1:]):
        c = float(sum(hist[a:b]))
        w = (b - a - 1).bit_length()
        tot += c * w - (c * math.log2(c) if c > 0 else 0.0)
    return tot
