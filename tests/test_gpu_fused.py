"""Decode fused with dequantisation (shn_decode_bf16) against a plain PyTorch CPU reference of the
same op: bf16_rn(float32(int8) * float32(scale[i >> log2_group])), compared bit for bit."""
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


def reference_bf16(x_int8: torch.Tensor, scales: torch.Tensor, log2_group: int) -> torch.Tensor:
    idx = torch.arange(x_int8.numel()) >> log2_group
    return (x_int8.cpu().float() * scales.cpu()[idx]).to(torch.bfloat16)


def fused(x: torch.Tensor, segs, p, scales, log2_group, n_scales=None):
    codec = shn.Codec(segs, p)
    xd = x.to(DEV)
    codec.compress(xd)
    assert codec.status("enc")[0] == 0
    nbytes = int(codec.out_bytes.item())
    out = torch.empty(codec.n_symbols, dtype=torch.bfloat16, device=DEV)
    sc = scales.to(DEV)[: n_scales if n_scales is not None else scales.numel()]
    shn.shn_decode_bf16(codec.stream_buf, nbytes, p, sc, log2_group, codec.work_dec, out)
    return codec.status("dec"), out.cpu()


def test_kv_cache_groups_of_128():
    shape = (2, 2, 2, 2, 512, 128)  # 4 segments of 262,144 values
    x = inputs.kv_cache_int8(seed=5, shape=shape)
    scales = inputs.kv_cache_scales(seed=5, shape=shape)
    (st, det), y = fused(x, inputs.kv_cache_segments(shape), shn.CodecParams(16, 7, 4096, 4), scales, 7)
    assert st == 0, (st, det)
    ref = reference_bf16(x, scales, 7)
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("K,R,S,C,lg", [(256, 10, 4, 1024, 4), (16, 7, 2, 384, 5), (8, 12, 16, 128, 9)])
def test_other_params_and_short_last_piece(K, R, S, C, lg):
    rng = np.random.default_rng(K + R)
    # every segment but the last has a length that is a multiple of 16; the last one is ragged
    lens = [16 * int(v) for v in rng.integers(1, 4000, 3)] + [int(rng.integers(1, 70_000))]
    n = sum(lens)
    x = inputs.laplace_int8(n, 9.0, seed=R)
    scales = torch.rand(((n - 1) >> lg) + 1, generator=torch.Generator().manual_seed(R)) * 0.1 + 1e-3
    segs, o = [], 0
    for ln in lens:
        segs.append((o, ln))
        o += ln
    (st, det), y = fused(x, segs, shn.CodecParams(K, R, C, S), scales, lg)
    assert st == 0, (st, det)
    assert torch.equal(y.view(torch.int16), reference_bf16(x, scales, lg).view(torch.int16))


def test_fused_decode_reports_bad_arguments():
    x = inputs.laplace_int8(50_000, 9.0, seed=1)
    p = shn.CodecParams(16, 7, 1024, 4)
    scales = torch.ones((50_000 >> 7) + 1)
    (st, _), _ = fused(x, [(0, 50_000)], p, scales, 7, n_scales=10)  # too few scales
    assert st == shn.SHN_ERR_CAPACITY
    (st, _), _ = fused(x, [(0, 100), (100, 49_900)], p, scales, 7)  # second segment starts at 100
    assert st == shn.SHN_ERR_UNSUPPORTED
