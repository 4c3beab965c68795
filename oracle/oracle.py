"""ctypes wrapper of the plain C oracle (oracle/shn_oracle.c) — TEST INFRASTRUCTURE ONLY.

Functions follow "Shannonic: Efficient Entropy-Optimal Compression for ML Workloads" (MLSys 2026
talk notes) §4.1 (histogram, DP range selection, tables) and §4.2 (Algorithm 2), with every open
detail fixed by the SHN1 format specification. Arrays are numpy; nothing here touches a GPU.
"""
import ctypes
import os

import numpy as np

from . import build as _build

ORC_OK, ORC_ERR_ARG, ORC_ERR_CAPACITY, ORC_ERR_CORRUPT, ORC_ERR_NOMEM = 0, 1, 2, 3, 4
MAX_L = 4096


class Segment(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_uint64), ("length", ctypes.c_uint64)]


class Params(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("R", ctypes.c_int32), ("S", ctypes.c_int32), ("C", ctypes.c_int32)]


class Tables(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int32),
        ("R", ctypes.c_int32),
        ("L", ctypes.c_int32),
        ("lo", ctypes.c_uint16 * 257),
        ("f", ctypes.c_uint32 * 256),
        ("cumul", ctypes.c_uint32 * 256),
        ("width_bits", ctypes.c_uint8 * 256),
        ("range_of", ctypes.c_uint8 * 256),
        ("spread", ctypes.c_uint16 * MAX_L),
        ("dec_sym", ctypes.c_uint16 * MAX_L),
        ("dec_nb", ctypes.c_uint8 * MAX_L),
        ("dec_next", ctypes.c_uint16 * MAX_L),
        ("enc", ctypes.c_uint16 * MAX_L),
    ]


class SegmentStats(ctypes.Structure):
    _fields_ = [
        ("dp_cost", ctypes.c_int64),
        ("payload_bits", ctypes.c_uint64),
        ("payload_words", ctypes.c_uint64),
        ("hist", ctypes.c_uint64 * 256),
        ("lo", ctypes.c_uint16 * 256),
        ("f", ctypes.c_uint32 * 256),
    ]


class OracleError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"oracle {what} failed with code {code}")
        self.code = code


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.orc_lg.restype = i64
        L.orc_lg.argtypes = [u64]
        L.orc_histogram.restype = None
        L.orc_histogram.argtypes = [vp, u64, vp]
        L.orc_partition.restype = i32
        L.orc_partition.argtypes = [vp, i32, i32, vp, ctypes.POINTER(i64)]
        L.orc_normalize.restype = i32
        L.orc_normalize.argtypes = [vp, i32, i32, vp]
        L.orc_tables_init.restype = i32
        L.orc_tables_init.argtypes = [vp, vp, i32, i32, ctypes.POINTER(Tables)]
        L.orc_build_segment_tables.restype = i32
        L.orc_build_segment_tables.argtypes = [vp, i32, i32, ctypes.POINTER(Tables), ctypes.POINTER(i64)]
        L.orc_encode_chunk.restype = i64
        L.orc_encode_chunk.argtypes = [ctypes.POINTER(Tables), i32, vp, ctypes.c_uint32, vp, u64, ctypes.POINTER(u64)]
        L.orc_decode_chunk.restype = i32
        L.orc_decode_chunk.argtypes = [ctypes.POINTER(Tables), i32, vp, u64, ctypes.c_uint32, vp]
        L.orc_stream_bound.restype = u64
        L.orc_stream_bound.argtypes = [ctypes.POINTER(Params), vp, i32]
        L.orc_encode_stream.restype = i32
        L.orc_encode_stream.argtypes = [vp, vp, i32, ctypes.POINTER(Params), i32, vp, u64, ctypes.POINTER(u64), vp]
        L.orc_encode_stream_with_tables.restype = i32
        L.orc_encode_stream_with_tables.argtypes = [
            vp, vp, i32, ctypes.POINTER(Params), vp, vp, i32, vp, u64, ctypes.POINTER(u64), vp]
        L.orc_decode_stream.restype = i32
        L.orc_decode_stream.argtypes = [vp, u64, i32, vp, u64, ctypes.POINTER(u64)]
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(0)


def _u8(x):
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint8:
        a = a.view(np.uint8) if a.dtype == np.int8 else a.astype(np.uint8)
    return a


def lg(n: int) -> int:
    """SHN1 format §2 fixed-point log2 (24 fraction bits)."""
    return int(lib().orc_lg(int(n)))


def histogram(x) -> np.ndarray:
    """256-bin histogram over symbols u = byte ^ 0x80."""
    a = _u8(x).reshape(-1)
    h = np.zeros(256, np.uint64)
    lib().orc_histogram(_ptr(a), a.size, _ptr(h))
    return h


def partition(hist, K: int):
    """DP range selection over an alphabet of len(hist) symbols. Returns (lo[K], dp_cost)."""
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    lo = np.zeros(K, np.uint16)
    cost = ctypes.c_int64(0)
    rc = lib().orc_partition(_ptr(h), h.size, K, _ptr(lo), ctypes.byref(cost))
    if rc:
        raise OracleError(rc, "partition")
    return lo, int(cost.value)


def normalize(N, R: int) -> np.ndarray:
    n = np.ascontiguousarray(N, dtype=np.uint64)
    f = np.zeros(n.size, np.uint32)
    rc = lib().orc_normalize(_ptr(n), n.size, R, _ptr(f))
    if rc:
        raise OracleError(rc, "normalize")
    return f


def tables(lo, f, R: int) -> Tables:
    lo_a = np.ascontiguousarray(lo, dtype=np.uint16)
    f_a = np.ascontiguousarray(f, dtype=np.uint32)
    t = Tables()
    rc = lib().orc_tables_init(_ptr(lo_a), _ptr(f_a), lo_a.size, R, ctypes.byref(t))
    if rc:
        raise OracleError(rc, "tables_init")
    return t


def segment_tables(hist, K: int, R: int):
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    t = Tables()
    cost = ctypes.c_int64(0)
    rc = lib().orc_build_segment_tables(_ptr(h), K, R, ctypes.byref(t), ctypes.byref(cost))
    if rc:
        raise OracleError(rc, "build_segment_tables")
    return t, int(cost.value)


def encode_chunk(t: Tables, S: int, x):
    a = _u8(x).reshape(-1)
    cap = (S * t.R + a.size * (t.R + 8) + 1 + 31) // 32 + 1
    w = np.zeros(cap, np.uint32)
    bits = ctypes.c_uint64(0)
    n = lib().orc_encode_chunk(ctypes.byref(t), S, _ptr(a), a.size, _ptr(w), cap, ctypes.byref(bits))
    if n < 0:
        raise OracleError(-n, "encode_chunk")
    return w[:n].copy(), int(bits.value)


def decode_chunk(t: Tables, S: int, words, c: int):
    w = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(c, np.uint8)
    rc = lib().orc_decode_chunk(ctypes.byref(t), S, _ptr(w), w.size, c, _ptr(out))
    return rc, out


def _segs(segments, n):
    if segments is None:
        segments = [(0, n)]
    arr = (Segment * max(1, len(segments)))()
    for i, (o, l) in enumerate(segments):
        arr[i].offset, arr[i].length = int(o), int(l)
    return arr, len(segments)


def stream_bound(K, R, S, C, segments) -> int:
    segs, ns = _segs(segments, 0)
    p = Params(K, R, S, C)
    return int(lib().orc_stream_bound(ctypes.byref(p), segs, ns))


def encode(x, K=16, R=7, S=4, C=4096, segments=None, threads=1, lo=None, f=None):
    """Encode the INT8 array x into an SHN1 stream. Returns (stream uint8 array, per-segment stats)."""
    a = _u8(x).reshape(-1)
    segs, ns = _segs(segments, a.size)
    p = Params(K, R, S, C)
    cap = int(lib().orc_stream_bound(ctypes.byref(p), segs, ns))
    if cap == 0:
        raise OracleError(ORC_ERR_ARG, "stream_bound")
    out = np.zeros(cap, np.uint8)
    nbytes = ctypes.c_uint64(0)
    stats = (SegmentStats * max(1, ns))()
    if lo is None:
        rc = lib().orc_encode_stream(_ptr(a), segs, ns, ctypes.byref(p), threads, _ptr(out), cap,
                                     ctypes.byref(nbytes), stats)
    else:
        lo_a = np.ascontiguousarray(lo, dtype=np.uint16).reshape(-1)
        f_a = np.ascontiguousarray(f, dtype=np.uint32).reshape(-1)
        rc = lib().orc_encode_stream_with_tables(_ptr(a), segs, ns, ctypes.byref(p), _ptr(lo_a), _ptr(f_a),
                                                 threads, _ptr(out), cap, ctypes.byref(nbytes), stats)
    if rc:
        raise OracleError(rc, "encode_stream")
    return out[: nbytes.value].copy(), [stats[i] for i in range(ns)]


def decode(stream, threads=1, capacity=None):
    """Decode an SHN1 stream. Returns (status code, uint8 output)."""
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    nsym = ctypes.c_uint64(0)
    if capacity is None:
        lib().orc_decode_stream(_ptr(s), s.size, threads, ctypes.c_void_p(0), 0, ctypes.byref(nsym))
        capacity = int(nsym.value)
    out = np.zeros(max(1, capacity), np.uint8)
    rc = lib().orc_decode_stream(_ptr(s), s.size, threads, _ptr(out), capacity, ctypes.byref(nsym))
    return rc, out[: min(capacity, int(nsym.value))]


def cpu_count() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
