"""GPU parity of the tiled encode (d > 128) against the oracle (B200).

Same checks as the fused path: codes bit-exact outside the 1e-5 band around a boundary (standardised
units), in-band mismatches below 1e-4 of all coordinates, fp16 norms / gammas exact up to the
one-ulp midpoint rule, signs checked against the oracle's second stage on the GPU's indices.
"""
import numpy as np
import pytest

import workloads as W
from test_gpu_encode_decode import check_mse, check_prod

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiled_mse_d256(dev, bits, dtype):
    x = W.gaussian(1000, 256, seed=bits, tag=W.TAG_X)
    if dtype == "bf16":
        x = W.round_to_bf16(x)
    st = check_mse(x, 256, bits, torch.float32 if dtype == "f32" else torch.bfloat16, dev, decode=False)
    print("tiled mse d256", bits, dtype, st)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiled_prod_d256(dev, bits, dtype):
    x = W.gaussian(700, 256, seed=10 + bits, tag=W.TAG_X)
    if dtype == "bf16":
        x = W.round_to_bf16(x)
    st = check_prod(x, 256, bits, torch.float32 if dtype == "f32" else torch.bfloat16, dev, decode=False)
    print("tiled prod d256", bits, dtype, st)


def test_tiled_vector_search_shape(dev):
    # the vector-search recipe: unit-norm fp32 rows, d = 1536, Algorithm 2 at 4 bits
    x = W.unit_rows(2000, 1536, seed=0)
    st = check_prod(x, 1536, 4, torch.float32, dev, decode=False)
    print("tiled prod d1536", st)


@pytest.mark.parametrize("d", [3072, 4096])
def test_tiled_prod_largest_d(dev, d):
    # the largest dimensions (the exact-gamma fix-up holds a batch's codebook values of all d
    # coordinates in shared memory: eight vectors at a time up to d = 3072, four above)
    x = W.gaussian(700, d, seed=d, tag=W.TAG_X)
    st = check_prod(x, d, 3, torch.float32, dev, decode=False)
    print("tiled prod", d, st)


def test_tiled_prod_many_fixup_batches(dev):
    # enough rows that every fix-up block claims several chunks of flag words and fills batches
    # across chunk boundaries (about 4 % of the gammas lie near an fp16 rounding midpoint)
    x = W.gaussian(120_000, 256, seed=77, tag=W.TAG_X)
    st = check_prod(x, 256, 3, torch.float32, dev, decode=False)
    print("tiled prod d256 n120000", st)


def test_tiled_mse_d1536_bf16(dev):
    x = W.round_to_bf16(W.gaussian(300, 1536, seed=3, tag=W.TAG_X))
    st = check_mse(x, 1536, 3, torch.bfloat16, dev, decode=False)
    print("tiled mse d1536", st)


@pytest.mark.parametrize("n", [1, 129, 385])
def test_tiled_ragged_and_zero_vectors(dev, n):
    x = W.gaussian(n, 384, seed=n, tag=W.TAG_X)
    x[:: 7] = 0.0                                   # zero vectors follow the documented convention
    check_mse(x, 384, 3, torch.float32, dev, decode=False)
    check_prod(x, 384, 3, torch.float32, dev, decode=False)


def test_tiled_extreme_magnitudes(dev):
    x = W.gaussian(260, 256, seed=9, tag=W.TAG_X)
    x[0::3] *= 1e-30
    x[1::3] *= 1e30
    check_prod(x, 256, 3, torch.float32, dev, decode=False)
