"""shn_encode_static: the encoder for callers that cannot allocate device memory.

Such callers (allocator hooks, out-of-memory handlers, plugins whose host owns all device memory)
cannot hand the library a workspace, so this entry point keeps its scratch in a fixed array inside
libshn itself. Its stream must be byte-identical to shn_encode's — the tolerance for all integer
work in these tests is zero — and the shared array must not leak one call's state into the next,
so the test makes two calls in a row with different inputs and compares each with shn_encode.
This file is collected last on purpose; it passes alone and after the other tests.
"""
import numpy as np
import pytest
import torch

from entropy_coded_lossless_b200 import inputs, shn

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shn.lib()


def _workspace_encoder(x, segs, p):
    codec = shn.Codec(segs, p)
    codec.compress(x)
    st, det = codec.status("enc")
    assert st == 0, (st, det)
    n = int(codec.out_bytes.item())
    return codec, codec.stream_buf[:n].clone()


def _static_encoder(x, segs, p, tables):
    out = shn.empty_aligned(shn.encode_bound(p, segs), DEV, 16)
    out_bytes = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.full((2,), -1, dtype=torch.int32, device=DEV)
    shn.shn_encode_static(x, segs, tables, p, out, out_bytes, status)
    torch.cuda.synchronize()
    return out[: int(out_bytes.item())].clone(), status.cpu().tolist()


def test_static_scratch_encoder_matches_workspace_encoder():
    p = shn.CodecParams(16, 7, 4096, 4)
    calls = [
        # many chunks and segments first, then fewer: stale scratch from the first call would show
        (inputs.activation_batch_int8(256, 65536, seed=3, device=DEV)[0],
         [(i * 65536, 65536) for i in range(256)]),
        (inputs.laplace_int8(1_000_003, 7.258, seed=11, device=DEV), [(0, 600_001), (600_001, 400_002)]),
    ]
    for x, segs in calls:
        codec, ref = _workspace_encoder(x, segs, p)
        got, status = _static_encoder(x, segs, p, codec.tables)
        assert status[0] == 0, status
        assert got.numel() == ref.numel()
        assert torch.equal(got, ref)
        # and it decodes back to the input
        out = torch.empty(codec.n_symbols, dtype=torch.uint8, device=DEV)
        codec.decode(got, got.numel(), out)
        assert codec.status("dec")[0] == 0
        expect = torch.cat([x.view(torch.uint8)[o:o + n] for o, n in segs])
        assert torch.equal(out, expect)


@pytest.mark.parametrize("K,R,C", [(16, 7, 65536), (256, 10, 4096)])
def test_static_scratch_encoder_other_params(K, R, C):
    """Long chunks (65,536 symbols) and plain tANS at L = 1024, each on two ragged segments: the
    static path gives shn_encode's bytes for them too."""
    p = shn.CodecParams(K, R, C, 4)
    x = inputs.laplace_int8(300_007, 20.0, seed=K + R, device=DEV)
    segs = [(0, 200_003), (200_003, 100_004)]
    for _ in range(2):
        codec, ref = _workspace_encoder(x, segs, p)
        got, status = _static_encoder(x, segs, p, codec.tables)
        assert status[0] == 0, status
        assert torch.equal(got, ref)


def test_static_scratch_encoder_rejects_too_many_chunks():
    p = shn.CodecParams(16, 7, 128, 4)
    n = (shn.encode_static_max_chunks() + 1) * 128
    segs = [(0, n)]
    x = torch.zeros(16, dtype=torch.int8, device=DEV)  # never read: the call fails on the host
    tables = shn.empty_aligned(shn.TABLE_BYTES, DEV)
    out = shn.empty_aligned(1 << 20, DEV, 16)
    out_bytes = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.zeros(2, dtype=torch.int32, device=DEV)
    with pytest.raises(shn.ShnError) as e:
        shn.shn_encode_static(x, segs, tables, p, out, out_bytes, status)
    assert e.value.code == shn.SHN_ERR_CAPACITY
