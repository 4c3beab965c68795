"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Bar (integer/byte work): bit-exact histograms, identical range bounds, state counts and DP values,
byte-identical SHN1 streams, byte-identical decoded tensors, and cross decoding (oracle stream →
GPU decoder, GPU stream → oracle decoder). The full-size KV cache (2 GiB) and 1 GiB sweep stream are
compared whole: every histogram, table record and stream byte against the oracle run on all host
threads. The 3 GiB and 8.4 GiB cases, where host memory is the limit, are checked on sampled chunks
the oracle recomputes one by one, plus the round-trip property on the device.
"""
import numpy as np
import pytest
import torch

from entropy_coded_lossless_b200 import inputs, shn
from tests import spec

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shn.lib()


def gpu_pipeline(x_cpu, segs, p: shn.CodecParams, single_pass=True):
    """histogram → tables → encode → decode on the device; returns host copies."""
    x = x_cpu.to(DEV) if isinstance(x_cpu, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(x_cpu)).to(DEV)
    codec = shn.Codec(segs, p, single_pass=single_pass)
    codec.compress(x)
    st, det = codec.status("enc")
    assert st == 0, (st, det)
    nbytes = int(codec.out_bytes.item())
    stream = codec.stream_buf[:nbytes]
    out = torch.empty(codec.n_symbols, dtype=torch.uint8, device=DEV)
    codec.decode(stream, nbytes, out)
    dst, ddet = codec.status("dec")
    assert dst == 0, (dst, ddet)
    hist = codec.hist[: 256 * max(1, len(segs))].cpu().numpy().astype(np.uint64).reshape(-1, 256)
    tables = [codec.table_fields(i) for i in range(len(segs))]
    return dict(stream=stream.cpu().numpy(), out=out.cpu().numpy(), hist=hist, tables=tables, codec=codec)


def check_parity(orc, x_np, segs, p: shn.CodecParams, threads=8, single_pass=True):
    g = gpu_pipeline(x_np, segs, p, single_pass)
    xb = np.ascontiguousarray(x_np).view(np.uint8).reshape(-1)
    # histograms
    for i, (o, n) in enumerate(segs):
        assert np.array_equal(g["hist"][i], orc.histogram(xb[o:o + n])), f"hist seg {i}"
    # tables
    ref_stream, ref_stats = orc.encode(xb, K=p.K, R=p.log2L, S=p.states_per_chunk, C=p.chunk_symbols,
                                       segments=segs, threads=threads)
    for i, st in enumerate(ref_stats):
        t = g["tables"][i]
        assert t["status"] == 0
        assert t["lo"] == list(st.lo[: p.K]), f"lo seg {i}"
        assert t["f"] == list(st.f[: p.K]), f"f seg {i}"
        assert t["dp_cost"] == st.dp_cost, f"dp seg {i}"
    # streams byte for byte
    assert g["stream"].size == ref_stream.size
    if not np.array_equal(g["stream"], ref_stream):
        diff = np.nonzero(g["stream"] != ref_stream)[0]
        raise AssertionError(f"streams differ at {diff[:10]} of {ref_stream.size}")
    # decoded bytes, and cross decoding
    out_sel = np.concatenate([xb[o:o + n] for o, n in segs]) if segs else np.zeros(0, np.uint8)
    assert np.array_equal(g["out"], out_sel)
    rc, y = orc.decode(g["stream"], threads=threads)
    assert rc == 0 and np.array_equal(y, out_sel)
    return g, ref_stream


def gpu_decode(stream_np, p, n_out):
    comp = shn.empty_aligned(stream_np.size, DEV, 16)
    comp.copy_(torch.from_numpy(stream_np))
    out = torch.zeros(max(1, n_out), dtype=torch.uint8, device=DEV)
    work = shn.empty_aligned(shn.decode_workspace_bytes(p), DEV)
    shn.shn_decode(comp, stream_np.size, p, work, out[:n_out] if n_out else out[:0])
    st, det = shn.shn_get_device_status(work)
    return st, out[:n_out].cpu().numpy()


# ----------------------------------------------------------------------------------------------


def test_config1_laplace(orc):
    x = inputs.laplace_int8(65536, inputs.LAPLACE_B_FOR_ENTROPY[5.3], seed=0).numpy()
    check_parity(orc, x, [(0, x.size)], shn.CodecParams(16, 7, 4096, 4))


def test_config2_weight_like(orc):
    x = inputs.weight_like_int8(seed=1).numpy()
    check_parity(orc, x, [(0, x.size)], shn.CodecParams(16, 7, 4096, 4))


def test_int4_weights(orc):
    """INT4 group-quantised weights, one value per byte: a 16-symbol alphabet inside the byte one."""
    x = inputs.int4_weight_like(512, 2048, seed=6).numpy()
    g, _ = check_parity(orc, x, [(0, x.size)], shn.CodecParams(16, 7, 4096, 4))
    st = spec.parse_stream(g["stream"])
    assert st["segments"][0]["payload_words"] * 32 < 4 * x.size  # below 4 bits per weight


def test_config2_plain_tans_l1024(orc):
    """The comparator of the weight-tensor config: plain tANS (K = 256 identity ranges) at L = 1024,
    bit-exact on the GPU, and (as on the pages) longer than Shannonic K = 16, L = 128."""
    x = inputs.weight_like_int8(seed=1).numpy()
    g_tans, _ = check_parity(orc, x, [(0, x.size)], shn.CodecParams(256, 10, 4096, 4))
    g_sh = gpu_pipeline(x, [(0, x.size)], shn.CodecParams(16, 7, 4096, 4))
    pay = lambda g: spec.parse_stream(g["stream"])["segments"][0]["payload_words"]
    assert pay(g_sh) < pay(g_tans)


@pytest.mark.parametrize("K,R,S,C", [(256, 9, 4, 1024), (16, 10, 2, 4096), (200, 11, 8, 256), (256, 12, 1, 128),
                                     (3, 12, 16, 1024), (32, 9, 4, 65536)])
def test_large_state_counts(orc, K, R, S, C):
    """L = 512 ... 4096: fields up to R + 8 bits, fewer table copies; two symbols per window position
    where R plus the widest offset fits 16 bits (K = 256, 200, 32 here), one otherwise (K = 3); ragged
    segments so tiles straddle segments (plain per-segment tables)."""
    rng = np.random.default_rng(K + 7 * R)
    n = 200_003
    x = inputs.laplace_int8(n, float(rng.choice([3.0, 20.0, 97.0])), seed=K * R).numpy()
    cuts = sorted(set([0, n] + rng.integers(0, n, 4).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    check_parity(orc, x, segs, shn.CodecParams(K, R, C, S))


@pytest.mark.parametrize("R", [9, 10, 11, 12])
def test_large_tables_mixed_field_widths(orc, R):
    """One L > 256 stream whose segment tables differ in their widest offset field: a near-uniform
    segment (ranges of ~16 symbols) beside a peaked one (its empty tails become ranges of > 64
    symbols), and small segments. With 128-symbol chunks the two large segments fill whole decoder
    tiles (one replicated table) and the small ones share tiles (several tables). Encoder blocks
    choose paired or single field appends per table, decoder tiles per set of tables; the stream
    must not depend on either choice."""
    sizes_b = [(150_000, 97.17), (150_000, 0.7), (3_000, 97.17), (2_500, 0.7), (40_000, 20.0), (777, 0.7)]
    x = np.concatenate([inputs.laplace_int8(n, b, seed=10 * R + i).numpy() for i, (n, b) in enumerate(sizes_b)])
    cuts = np.cumsum([0] + [n for n, _ in sizes_b])
    segs = [(int(a), int(b - a)) for a, b in zip(cuts[:-1], cuts[1:])]
    g, _ = check_parity(orc, x, segs, shn.CodecParams(16, R, 128, 4))
    widest = []
    for t in g["tables"]:
        lo = list(t["lo"]) + [256]
        widest.append(max(int(np.ceil(np.log2(b - a))) if b - a > 1 else 0 for a, b in zip(lo[:-1], lo[1:])))
    if R in (10, 11):  # both kinds of table are present
        assert min(widest) + R <= 16 < max(widest) + R, widest


def test_config4_activation_batch_full(orc):
    x, segs, _ = inputs.activation_batch_int8(1024, 65536, seed=3)
    check_parity(orc, x.numpy(), segs, shn.CodecParams(16, 7, 4096, 4), threads=32)


@pytest.mark.parametrize("K,R,S,C", [(1, 4, 1, 128), (2, 5, 2, 256), (8, 6, 8, 1024), (32, 8, 16, 384),
                                     (16, 7, 4, 128), (64, 8, 4, 4096), (3, 4, 16, 65536)])
def test_params_and_ragged_segments(orc, K, R, S, C):
    rng = np.random.default_rng(K * 100 + R)
    n = 300_001
    x = inputs.laplace_int8(n, float(rng.choice([1.5, 7.0, 40.0])), seed=K + R).numpy()
    cuts = sorted(set([0, n] + rng.integers(0, n, 5).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    segs.insert(2, (segs[1][0], 0))  # an empty segment
    segs.append((n - 77, 77))       # overlapping, short, unaligned
    check_parity(orc, x, segs, shn.CodecParams(K, R, C, S))


@pytest.mark.parametrize("n_tables", [1, 18, 19, 37, 38, 74, 75, 160])
def test_table_build_cluster_sizes(orc, n_tables):
    """The table build runs a cluster of 8, 4 or 2 blocks per table, or one block, by how many
    tables the launch has (the largest cluster that still gives every block an SM: on 148 SMs the
    switches fall between 18 and 19, 37 and 38, 74 and 75 tables); every table record and the
    stream must equal the oracle's whichever is taken. Segments of different lengths and
    entropies, two of them beyond 2^17 symbols (LG computed, not looked up)."""
    rng = np.random.default_rng(n_tables)
    lens = rng.integers(2_000, 40_000, n_tables)
    lens[0], lens[-1] = 150_000, 200_000
    parts = [inputs.laplace_int8(int(n), float(rng.choice([0.8, 3.0, 7.0, 40.0])), seed=1000 + i).numpy()
             for i, n in enumerate(lens)]
    x = np.concatenate(parts)
    ends = np.cumsum(lens)
    segs = [(int(e - n), int(n)) for e, n in zip(ends, lens)]
    check_parity(orc, x, segs, shn.CodecParams(16, 7, 1024, 4))
    if n_tables in (19, 38, 160):  # the threshold allocation (L >= 256): clusters of 4 and 2, one block
        check_parity(orc, x, segs, shn.CodecParams(32, 9, 1024, 4))


def test_degenerate_inputs(orc):
    p = shn.CodecParams(16, 7, 1024, 4)
    single = np.full(5000, -7, np.int8)
    allv = np.tile(np.arange(-128, 128, dtype=np.int8), 40)
    np.random.default_rng(1).shuffle(allv)
    x = np.concatenate([single, allv, np.zeros(1, np.int8)])
    segs = [(0, 5000), (5000, allv.size), (x.size - 1, 1)]
    g, _ = check_parity(orc, x, segs, p)
    st = spec.parse_stream(g["stream"])
    assert st["segments"][0]["payload_words"] == 5  # one value: states + sentinel only
    # plain tANS (K = 256 identity ranges) at L = 256
    check_parity(orc, allv, [(0, allv.size)], shn.CodecParams(256, 8, 1024, 4))


def test_empty_stream(orc):
    p = shn.CodecParams()
    codec = shn.Codec([], p)
    x = torch.zeros(16, dtype=torch.int8, device=DEV)
    codec.encode(x)
    assert codec.status("enc")[0] == 0
    n = int(codec.out_bytes.item())
    ref, _ = orc.encode(np.zeros(0, np.int8), segments=[])
    assert n == ref.size == 64
    assert np.array_equal(codec.stream_buf[:n].cpu().numpy(), ref)
    st, out = gpu_decode(ref, p, 0)
    assert st == 0


def test_oracle_stream_decoded_by_gpu(orc):
    x = inputs.laplace_int8(200_000, 3.0, seed=5).numpy()
    for K, R, S, C in [(16, 7, 4, 4096), (8, 8, 2, 1024), (32, 6, 16, 128)]:
        ref, _ = orc.encode(x, K=K, R=R, S=S, C=C, segments=[(0, 123_457), (123_457, 76_543)])
        st, out = gpu_decode(ref, shn.CodecParams(K, R, C, S), x.size)
        assert st == 0 and np.array_equal(out, x.view(np.uint8))


def test_sweep_points_small(orc):
    n = 1 << 20
    for i, pt in enumerate(inputs.sweep_points()):
        if pt["L"] > 256:
            continue
        x = inputs.laplace_int8(n, pt["b"], seed=4 + i).numpy()
        check_parity(orc, x, [(0, n)], shn.CodecParams(pt["K"], int(np.log2(pt["L"])), pt["C"], 4), threads=16)


# ---- full-size workloads: sampled chunks against the oracle + device round trip -------------


def _sampled_chunk_check(orc, x_dev, segs, p, g_stream, n_samples=24, seed=0):
    st = spec.parse_stream(g_stream)
    rng = np.random.default_rng(seed)
    for _ in range(n_samples):
        si = int(rng.integers(0, len(segs)))
        o, n = segs[si]
        sg = st["segments"][si]
        nch = -(-n // p.chunk_symbols)
        c = int(rng.integers(0, nch))
        pos = torch.tensor(spec.chunk_positions(n, p.chunk_symbols, c), dtype=torch.int64, device=x_dev.device)
        chunk = x_dev[o + pos].cpu().numpy().view(np.uint8)
        t = orc.tables(np.array(sg["lo"], np.uint16), np.array(sg["f"], np.uint32), p.log2L)
        words, _ = orc.encode_chunk(t, p.states_per_chunk, chunk)
        assert np.array_equal(spec.chunk_words(st, si, c), words), (si, c)


def _full_size(orc, x_dev, segs, p, table_check_segs):
    codec = shn.Codec(segs, p)
    codec.compress(x_dev)
    st, det = codec.status("enc")
    assert st == 0, (st, det)
    nbytes = int(codec.out_bytes.item())
    out = torch.empty(codec.n_symbols, dtype=torch.uint8, device=DEV)
    codec.decode(codec.stream_buf[:nbytes], nbytes, out)
    assert codec.status("dec")[0] == 0
    assert torch.equal(out, x_dev.view(torch.uint8)), "device round trip"
    # histograms and tables of sampled segments against the oracle
    hist = codec.hist.view(-1, 256).cpu().numpy().astype(np.uint64)
    for si in table_check_segs:
        o, n = segs[si]
        seg_np = x_dev[o:o + n].cpu().numpy().view(np.uint8)
        h = orc.histogram(seg_np)
        assert np.array_equal(hist[si], h)
        t, cost = orc.segment_tables(h, p.K, p.log2L)
        f = codec.table_fields(si)
        assert f["lo"] == list(t.lo[: p.K]) and f["f"] == list(t.f[: p.K]) and f["dp_cost"] == cost
    stream = codec.stream_buf[:nbytes].cpu().numpy()
    _sampled_chunk_check(orc, x_dev, segs, p, stream)
    return nbytes


def _full_size_whole(orc, x_dev, segs, p):
    """Whole-workload parity at full size, in the launch configuration bench.py times: the GPU's
    histograms, table records (lo, f, DP value) and stream against the oracle's, every byte; the
    device round trip; and the oracle decoding the GPU's stream."""
    codec = shn.Codec(segs, p)
    codec.compress(x_dev)
    st, det = codec.status("enc")
    assert st == 0, (st, det)
    nbytes = int(codec.out_bytes.item())
    out = torch.empty(codec.n_symbols, dtype=torch.uint8, device=DEV)
    codec.decode(codec.stream_buf[:nbytes], nbytes, out)
    assert codec.status("dec")[0] == 0
    assert torch.equal(out, x_dev.view(torch.uint8)), "device round trip"
    del out
    xb = x_dev.view(torch.uint8).cpu().numpy()
    threads = max(8, orc.cpu_count())
    ref, stats = orc.encode(xb, K=p.K, R=p.log2L, S=p.states_per_chunk, C=p.chunk_symbols, segments=segs,
                            threads=threads)
    hist = codec.hist.view(-1, 256).cpu().numpy().astype(np.uint64)
    for si, stt in enumerate(stats):
        assert np.array_equal(hist[si], np.ctypeslib.as_array(stt.hist)), f"hist seg {si}"
        f = codec.table_fields(si)
        assert f["lo"] == list(stt.lo[: p.K]) and f["f"] == list(stt.f[: p.K]), f"table seg {si}"
        assert f["dp_cost"] == stt.dp_cost, f"dp seg {si}"
    got = codec.stream_buf[:nbytes].cpu().numpy()
    assert got.size == ref.size, (got.size, ref.size)
    if not np.array_equal(got, ref):
        diff = np.nonzero(got != ref)[0]
        raise AssertionError(f"streams differ at {diff[:10]} of {ref.size}")
    del ref
    rc, y = orc.decode(got, threads=threads)
    assert rc == 0 and np.array_equal(y, xb)
    return nbytes


def test_config3_kv_cache_full(orc):
    x = inputs.kv_cache_int8(seed=2, device=DEV)
    segs = inputs.kv_cache_segments()
    nbytes = _full_size_whole(orc, x, segs, shn.CodecParams(16, 7, 4096, 4))
    assert nbytes < x.numel()


@pytest.mark.parametrize("H", [2.0, 4.0, 5.3, 7.9])
def test_config5_full_gib(orc, H):
    x = inputs.sweep_stream_int8(H, seed=4, device=DEV)
    _full_size_whole(orc, x, [(0, x.numel())], shn.CodecParams(16, 7, 4096, 4))


def test_segments_beyond_2gib(orc):
    """3 GiB in two segments, the second starting past 2^31 bytes and the stream running past 2^32
    bits, with a ragged tail: 64-bit offsets throughout (an int32 overflow anywhere in the path
    would show here as a wrong histogram, a failed round trip or a sampled chunk that differs)."""
    n1, n2 = (1 << 31) + 48, (1 << 30) + 12_345
    x = inputs.laplace_int8(n1 + n2, inputs.LAPLACE_B_FOR_ENTROPY[5.3], seed=12, device=DEV)
    nbytes = _full_size(orc, x, [(0, n1), (n1, n2)], shn.CodecParams(16, 7, 4096, 4), table_check_segs=[0, 1])
    assert nbytes > (1 << 31)

def test_stream_beyond_8gib(orc):
    """8.4 GiB of near-uniform bytes (H = 7.9 bits) in three segments: a stream of ~8.3 GiB, past
    where byte offsets divided by 4 leave 32-bit signed range. The encoder accepts any input whose
    worst-case bound (15 bits per value at L = 128) stays within 16 GiB, i.e. up to ~8.5 GiB, and
    near-incompressible input gives a stream of about its own size."""
    n = int(2.8 * (1 << 30)) & ~15
    segs = [(0, n), (n, n), (2 * n, n + 12_345)]
    x = inputs.laplace_int8(3 * n + 12_345, inputs.LAPLACE_B_FOR_ENTROPY[7.9], seed=13, device=DEV)
    nbytes = _full_size(orc, x, segs, shn.CodecParams(16, 7, 4096, 4), table_check_segs=[2])
    assert nbytes > (8 << 30)

# ---- errors reported on the device ------------------------------------------------------------


def test_decoder_reports_corruption(orc):
    p = shn.CodecParams(16, 7, 1024, 4)
    x = inputs.laplace_int8(50_000, 7.0, seed=1).numpy()
    ref, _ = orc.encode(x, K=16, R=7, S=4, C=1024)
    st_ = spec.parse_stream(ref)
    assert gpu_decode(ref, p, x.size)[0] == 0
    bad = ref.copy()
    bad[0] ^= 1
    assert gpu_decode(bad, p, x.size)[0] == shn.SHN_ERR_CORRUPT
    bad = ref.copy()
    bad[st_["index_offset"] + 8: st_["index_offset"] + 12] = 0xFF
    assert gpu_decode(bad, p, x.size)[0] == shn.SHN_ERR_CORRUPT
    end = st_["payload_offset"] + 4 * int(st_["index"][3])
    bad = ref.copy()
    bad[end - 4:end] = 0
    assert gpu_decode(bad, p, x.size)[0] == shn.SHN_ERR_CORRUPT
    # truncated stream, wrong parameters, too small output
    assert gpu_decode(ref[:-64], p, x.size)[0] == shn.SHN_ERR_CORRUPT
    assert gpu_decode(ref, shn.CodecParams(16, 7, 1024, 2), x.size)[0] == shn.SHN_ERR_CORRUPT
    assert gpu_decode(ref, p, x.size - 1)[0] == shn.SHN_ERR_CAPACITY
    # random payload bit flips: never a fault; detected when the state chain is disturbed
    rng = np.random.default_rng(0)
    detected = 0
    for _ in range(40):
        bad = ref.copy()
        pos = int(rng.integers(st_["payload_offset"], ref.size - 16))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        st, _ = gpu_decode(bad, p, x.size)
        assert st in (0, shn.SHN_ERR_CORRUPT)
        detected += st != 0
    assert detected >= 10


@pytest.mark.parametrize("K,R,S,C", [(16, 7, 4, 4096), (5, 10, 2, 1024), (64, 8, 16, 384)])
def test_two_pass_mode(orc, K, R, S, C):
    """With the minimal workspace the encoder sizes every chunk first and writes it in place; the
    stream is the same bytes as the oracle's (and the single-pass mode's)."""
    rng = np.random.default_rng(K * R)
    n = 250_001
    x = inputs.laplace_int8(n, float(rng.choice([2.0, 9.0, 60.0])), seed=R).numpy()
    cuts = sorted(set([0, n] + rng.integers(0, n, 3).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    p = shn.CodecParams(K, R, C, S)
    assert shn.encode_workspace_bytes_min(p, segs) < shn.encode_workspace_bytes(p, segs)
    check_parity(orc, x, segs, p, single_pass=False)


@pytest.mark.parametrize("single_pass", [True, False])
def test_encoder_reports_capacity(single_pass):
    p = shn.CodecParams(16, 7, 4096, 4)
    x = inputs.laplace_int8(100_000, 7.0, seed=2).to(DEV)
    segs = [(0, x.numel())]
    codec = shn.Codec(segs, p, single_pass=single_pass)
    codec.histogram(x)
    codec.build()
    small = shn.empty_aligned(20_000, DEV, 16)
    shn.shn_encode(x, segs, codec.tables, p, codec.work_enc, small, codec.out_bytes)
    st, _ = codec.status("enc")
    assert st == shn.SHN_ERR_CAPACITY
    assert int(codec.out_bytes.item()) > 20_000
    with pytest.raises(shn.ShnError):
        shn.shn_encode(x, segs, codec.tables, p, codec.work_enc, small[:10], codec.out_bytes)


@pytest.mark.parametrize("single_pass", [True, False])
def test_encoder_rejects_foreign_table(single_pass):
    # a table built for a one-value segment cannot code other symbols: device status, no fault
    p = shn.CodecParams(16, 7, 4096, 4)
    a = torch.full((8192,), 3, dtype=torch.int8, device=DEV)
    b = inputs.laplace_int8(8192, 7.0, seed=3).to(DEV)
    codec = shn.Codec([(0, 8192)], p, single_pass=single_pass)
    codec.histogram(a)
    codec.build()
    codec.encode(b)
    assert codec.status("enc")[0] == shn.SHN_ERR_INVALID_ARG
