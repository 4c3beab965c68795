"""The C-ABI library loads without a GPU and exports every entry point include/shn.h declares;
host-only queries agree with the format (SHN1 format §6) as the oracle computes it. No CUDA calls."""
import os
import re

import pytest

from entropy_coded_lossless_b200 import build as shn_build
from entropy_coded_lossless_b200 import shn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", hdr)).read()
            names += re.findall(r"^[a-z_0-9 ]+[ *]+(shn_\w+)\(", txt, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    shn_build.build()
    return shn.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(shn.EXPORTED)


def test_version_and_status_strings(lib):
    assert shn.version() == 0x00010000
    for code in range(8):
        assert shn.status_string(code) != "unknown status"


def test_param_checks(lib):
    P = shn.CodecParams
    assert shn.check_params(P()) == 0
    for bad in [P(K=0), P(K=257, log2L=12), P(log2L=3), P(log2L=13), P(K=32, log2L=4), P(chunk_symbols=100),
                P(chunk_symbols=65536 + 128), P(states_per_chunk=3), P(states_per_chunk=32)]:
        assert shn.check_params(bad) == shn.SHN_ERR_INVALID_ARG, bad
    assert shn.table_bytes(P()) == shn.TABLE_BYTES


@pytest.mark.parametrize("K,R,S,C", [(16, 7, 4, 4096), (1, 4, 1, 128), (256, 10, 16, 65536), (32, 8, 2, 1024)])
def test_encode_bound_matches_format(lib, orc, K, R, S, C):
    segs = [(0, 65536), (65536, 0), (65536, 12345), (77881, 1)]
    p = shn.CodecParams(K, R, C, S)
    assert shn.encode_bound(p, segs) == orc.stream_bound(K, R, S, C, segs)
    wmin, wfull = shn.encode_workspace_bytes_min(p, segs), shn.encode_workspace_bytes(p, segs)
    assert 256 <= wmin < wfull
    # the single-pass slots hold every chunk at its worst case: the bound's payload, give or take
    # the rounding of each slot to 4 words and of each region to 256 bytes
    payload_bound = orc.stream_bound(K, R, S, C, segs) - orc.stream_bound(K, R, S, C, [])
    assert wfull - wmin >= payload_bound - 16 * len(segs) - 4096
    assert shn.decode_workspace_bytes(p) == 256


def test_oversized_segment_rejected(lib):
    p = shn.CodecParams()
    assert shn.encode_bound(p, [(0, 1 << 32)]) == 0


def test_offload_queries_and_host_checks(lib, orc):
    """Host-side logic of the offload entry points, no CUDA call: workspace query, and the checks
    shn_decode_from_host makes on the host streams before it enqueues anything."""
    import ctypes

    import numpy as np

    p = shn.CodecParams(16, 7, 4096, 4)
    segs = [(0, 1 << 20), (1 << 20, 5000), (1 << 20 | 5000, 3 << 20)]
    ends = [1, 3]
    w = shn.offload_workspace_bytes(p, segs, ends)
    # at least two staging streams of the larger batch and its single-pass encoder workspace
    assert w >= 2 * shn.encode_bound(p, segs[1:]) + shn.encode_workspace_bytes(p, segs[1:])
    assert shn.offload_workspace_bytes(p, segs, [2, 1]) == 0  # batch ends must not decrease

    x = np.zeros(1000, np.int8)
    stream, _ = orc.encode(x, K=16, R=7, S=4, C=4096)
    L = shn.lib()
    fake_dev = 1 << 20  # never dereferenced: every check below fails before a CUDA call

    def call(buf, nbytes, out_cap, staging_bytes):
        arr = np.ascontiguousarray(buf)
        ptrs = (ctypes.c_void_p * 1)(arr.ctypes.data)
        sizes = (ctypes.c_size_t * 1)(nbytes)
        offs = (ctypes.c_size_t * 1)(0)
        return L.shn_decode_from_host(ptrs, sizes, 1, ctypes.byref(p.c()), fake_dev, staging_bytes, fake_dev, 256,
                                      fake_dev, offs, out_cap, None, None)

    bad = stream.copy()
    bad[0] ^= 0xFF
    assert call(bad, stream.size, 1000, 1 << 20) == shn.SHN_ERR_CORRUPT
    assert call(stream, 10, 1000, 1 << 20) == shn.SHN_ERR_CORRUPT  # shorter than a header
    assert call(stream, stream.size, 999, 1 << 20) == shn.SHN_ERR_CAPACITY
    assert call(stream, stream.size, 1000, stream.size) == shn.SHN_ERR_WORKSPACE  # room for one stream only


def test_static_encoder_host_checks(lib):
    """shn_encode_static makes shn_encode's host checks before anything else, with no CUDA call:
    a stream whose worst case passes 16 GiB (32-bit word offsets inside a payload) is refused even
    when its chunk count fits the static scratch; so are a missing segment array and misaligned
    pointers. The same oversized request is refused by shn_encode."""
    import ctypes

    L = shn.lib()
    p = shn.CodecParams(16, 7, 65536, 4)
    seg = (1 << 32) - 1
    segs = [(i * seg, seg) for i in range(3)]  # about 196,608 chunks of 65,536 symbols
    chunks = sum(-(-n // p.chunk_symbols) for _, n in segs)
    assert chunks < shn.encode_static_max_chunks()
    assert shn.encode_bound(p, segs) > (16 << 30)
    arr = shn._segments(segs)
    fake = 1 << 20  # a 256-byte aligned stand-in for device pointers: never dereferenced
    pc = ctypes.byref(p.c())

    def static(h_segs, n_segs, status=fake, out=fake):
        return L.shn_encode_static(fake, h_segs, n_segs, fake, pc, out, 1 << 40, fake, status, None)

    assert static(arr, 3) == shn.SHN_ERR_INVALID_ARG
    assert L.shn_encode(fake, arr, 3, fake, pc, fake, 1 << 40, fake, 1 << 40, fake, None) == shn.SHN_ERR_INVALID_ARG
    small = shn._segments([(0, 4096)])
    assert static(None, 1) == shn.SHN_ERR_INVALID_ARG
    assert static(small, 1, status=fake + 4) == shn.SHN_ERR_INVALID_ARG
    assert static(small, 1, out=fake + 8) == shn.SHN_ERR_INVALID_ARG
    # too many chunks for the static scratch (but a stream well within 16 GiB)
    p128 = shn.CodecParams(16, 7, 128, 4)
    many = shn._segments([(0, (shn.encode_static_max_chunks() + 1) * 128)])
    assert L.shn_encode_static(fake, many, 1, fake, ctypes.byref(p128.c()), fake, 1 << 40, fake, fake,
                               None) == shn.SHN_ERR_CAPACITY


def test_segment_list_marshalled_once(lib):
    """shn.Segments holds the C array a call takes; the binding passes it through unchanged (a
    codec reuses it on every call), and its sizes agree with a plain list's."""
    pairs = [(0, 5000), (5000, 0), (12_345, 77), (1 << 33, 4096 * 3 + 1)]
    sg = shn.Segments(pairs)
    assert len(sg) == len(pairs) and list(sg) == pairs
    arr = shn._segments(sg)
    assert arr is sg.arr and shn._segments(sg) is arr
    assert [(arr[i].offset, arr[i].length) for i in range(len(pairs))] == pairs
    p = shn.CodecParams(16, 7, 4096, 4)
    assert shn.encode_bound(p, sg) == shn.encode_bound(p, pairs) > 0
    assert shn.encode_workspace_bytes(p, sg) == shn.encode_workspace_bytes(p, pairs) > 0
    empty = shn.Segments([])
    assert len(empty) == 0 and len(shn._segments(empty)) == 1  # the C array is never empty
