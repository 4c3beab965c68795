"""Compressed offload and pipelined reload: shn_encode writing its stream straight into pinned host
memory, shn_offload copying each batch's stream out with the copy engine (both byte-identical to
the oracle's streams), and shn_decode_from_host restoring the tensor from several host streams while
copies and decodes overlap."""
import numpy as np
import pytest
import torch

from entropy_coded_lossless_b200 import inputs, shn

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shn.lib()


def offload(x_dev, batches, p):
    """Encode each batch of segments into its own pinned host stream; returns (streams, sizes)."""
    streams, sizes = [], []
    for segs in batches:
        codec = shn.Codec(segs, p)
        codec.histogram(x_dev)
        codec.build()
        host = torch.empty(codec.bound, dtype=torch.uint8, pin_memory=True)
        shn.shn_encode(x_dev, segs, codec.tables, p, codec.work_enc, host, codec.out_bytes)
        torch.cuda.synchronize()
        assert codec.status("enc")[0] == 0
        streams.append(host)
        sizes.append(int(codec.out_bytes.item()))
    return streams, sizes


@pytest.mark.parametrize("K,R,S,C", [(16, 7, 4, 4096), (256, 10, 2, 1024)])
def test_offload_to_host_and_pipelined_reload(orc, K, R, S, C):
    rng = np.random.default_rng(R)
    n = 1_500_007
    x = inputs.laplace_int8(n, 7.0, seed=K)
    cuts = sorted(set([0, n] + rng.integers(0, n, 6).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    batches = [segs[0:2], segs[2:3], segs[3:]]
    p = shn.CodecParams(K, R, C, S)
    x_dev = x.to(DEV)
    streams, sizes = offload(x_dev, batches, p)
    xb = x.numpy().view(np.uint8)
    for segs_b, h, nb in zip(batches, streams, sizes):  # what crossed the link is the oracle's stream
        ref, _ = orc.encode(xb, K=K, R=R, S=S, C=C, segments=segs_b, threads=8)
        assert nb == ref.size and np.array_equal(h[:nb].numpy(), ref)
    offsets = np.cumsum([0] + [sum(ln for _, ln in b) for b in batches])[:-1].tolist()
    staging = shn.empty_aligned(2 * max(-(-s // 16) * 16 for s in sizes), DEV, 16)
    work = shn.empty_aligned(256, DEV)
    out = torch.zeros(n, dtype=torch.uint8, device=DEV)
    copy_stream = torch.cuda.Stream()
    shn.shn_decode_from_host(streams, sizes, p, staging, work, out, offsets,
                             torch.cuda.current_stream(), copy_stream)
    assert shn.shn_get_device_status(work)[0] == 0
    expect = np.concatenate([xb[o:o + ln] for b in batches for o, ln in b])
    assert np.array_equal(out.cpu().numpy(), expect)


@pytest.mark.parametrize("K,R,S,C", [(16, 7, 4, 4096), (32, 9, 8, 512)])
def test_pipelined_offload_and_reload(orc, K, R, S, C):
    """shn_offload: every batch's stream, copied out by the copy engine, is the oracle's stream for
    that batch; shn_decode_from_host restores the tensor from them."""
    rng = np.random.default_rng(K + R)
    n = 2_000_003
    x = inputs.laplace_int8(n, 5.0, seed=R)
    cuts = sorted(set([0, n] + rng.integers(0, n, 9).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    ends = [2, 3, 5, 7, len(segs)]  # five batches, one with a single segment
    p = shn.CodecParams(K, R, C, S)
    x_dev = x.to(DEV)
    work = shn.empty_aligned(shn.offload_workspace_bytes(p, segs, ends), DEV)
    h_out = torch.empty(n * 2 + (1 << 20), dtype=torch.uint8, pin_memory=True)
    copy_stream = torch.cuda.Stream()
    offs, sizes = shn.shn_offload(x_dev, segs, ends, p, work, h_out, torch.cuda.current_stream(), copy_stream)
    copy_stream.synchronize()
    xb = x.numpy().view(np.uint8)
    batches = [segs[a:b] for a, b in zip([0] + ends[:-1], ends)]
    streams = []
    for segs_b, o, nb in zip(batches, offs, sizes):
        ref, _ = orc.encode(xb, K=K, R=R, S=S, C=C, segments=segs_b, threads=8)
        assert o % 16 == 0 and nb == ref.size and np.array_equal(h_out[o:o + nb].numpy(), ref)
        streams.append(h_out[o:o + nb])
    out_offsets = np.cumsum([0] + [sum(ln for _, ln in b) for b in batches])[:-1].tolist()
    staging = shn.empty_aligned(2 * max(-(-v // 16) * 16 for v in sizes), DEV, 16)
    dwork = shn.empty_aligned(256, DEV)
    out = torch.zeros(n, dtype=torch.uint8, device=DEV)
    shn.shn_decode_from_host(streams, sizes, p, staging, dwork, out, out_offsets, torch.cuda.current_stream(),
                             copy_stream)
    assert shn.shn_get_device_status(dwork)[0] == 0
    assert np.array_equal(out.cpu().numpy(), np.concatenate([xb[o:o + ln] for b in batches for o, ln in b]))
    with pytest.raises(shn.ShnError) as e:  # host buffer too small for the streams
        shn.shn_offload(x_dev, segs, ends, p, work, h_out[: sizes[0] + 16])
    assert e.value.code == shn.SHN_ERR_CAPACITY


def test_reload_rejects_bad_host_streams():
    p = shn.CodecParams(16, 7, 1024, 4)
    x_dev = inputs.laplace_int8(100_000, 7.0, seed=1).to(DEV)
    streams, sizes = offload(x_dev, [[(0, 100_000)]], p)
    staging = shn.empty_aligned(2 * 16 * (-(-sizes[0] // 16)), DEV, 16)
    work = shn.empty_aligned(256, DEV)
    out = torch.zeros(100_000, dtype=torch.uint8, device=DEV)
    bad = streams[0].clone().pin_memory()
    bad[0] ^= 0xFF  # not an SHN1 header
    with pytest.raises(shn.ShnError) as e:
        shn.shn_decode_from_host([bad], sizes, p, staging, work, out, [0])
    assert e.value.code == shn.SHN_ERR_CORRUPT
    with pytest.raises(shn.ShnError) as e:  # output range past the end
        shn.shn_decode_from_host(streams, sizes, p, staging, work, out[:99_999], [0])
    assert e.value.code == shn.SHN_ERR_CAPACITY
    with pytest.raises(shn.ShnError) as e:  # staging smaller than two streams
        shn.shn_decode_from_host(streams, sizes, p, staging[:sizes[0]], work, out, [0])
    assert e.value.code == shn.SHN_ERR_WORKSPACE
