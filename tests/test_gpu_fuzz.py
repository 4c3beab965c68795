"""Seeded fuzz: random parameters, value distributions and segment layouts, every stream compared
with the oracle's byte for byte and decoded back (both encoder modes, both decode outputs)."""
import numpy as np
import pytest
import torch

from entropy_coded_lossless_b200 import inputs, shn
from tests.test_gpu_parity import check_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shn.lib()


def random_tensor(rng, n):
    kind = rng.integers(0, 5)
    if kind == 0:
        return inputs.laplace_int8(n, float(rng.choice([0.5, 2.0, 9.0, 60.0])), seed=int(rng.integers(1 << 30))).numpy()
    if kind == 1:  # a few distinct values
        vals = rng.integers(-128, 128, int(rng.integers(1, 6))).astype(np.int8)
        return vals[rng.integers(0, vals.size, n)]
    if kind == 2:  # uniform bytes
        return rng.integers(-128, 128, n).astype(np.int8)
    if kind == 3:  # ReLU-like: half zeros
        x = np.clip(np.round(rng.normal(0, 20, n)), -128, 127).astype(np.int8)
        x[x < 0] = 0
        return x
    return inputs.int4_weight_like(4, max(64, (n // 4) // 64 * 64), seed=int(rng.integers(1 << 30))).numpy()[:n]


@pytest.mark.parametrize("case", range(24))
def test_fuzz(orc, case):
    rng = np.random.default_rng(1000 + case)
    R = int(rng.integers(4, 13))
    K = int(min(rng.choice([1, 2, 3, 8, 16, 32, 100, 256]), 1 << R))
    S = int(rng.choice([1, 2, 4, 8, 16]))
    C = int(rng.choice([128, 384, 1024, 4096, 16384]))
    n = int(rng.integers(1, 400_000))
    x = random_tensor(rng, n)
    n = x.size
    cuts = sorted(set([0, n] + rng.integers(0, n, int(rng.integers(0, 6))).tolist()))
    segs = [(a, b - a) for a, b in zip(cuts[:-1], cuts[1:])]
    if rng.random() < 0.3:
        segs.append((int(rng.integers(0, n)), 0))  # an empty segment
    p = shn.CodecParams(K, R, C, S)
    check_parity(orc, x, segs, p, single_pass=bool(rng.random() < 0.7))
