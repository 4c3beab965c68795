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
