"""GPU parity of the mixed-width format (a bit width per group of 32 rotated coordinates) against
the oracle (B200).

Encode (tq_encode_mse_mixed): every index equals the oracle's except next to a decision boundary of
its own group's codebook (1e-5 on the standardised coordinate, fewer than 1e-4 of all coordinates),
norms exact up to the fp16 midpoint rule; a map with one width everywhere gives exactly the words of
tq_encode_mse. Decode (tq_decode_mixed): the oracle's fp64 dequantisation of the GPU's own codes
within 1e-3 normwise (the split-fp16 products put it near 1e-6).
"""
import numpy as np
import pytest

import workloads as W
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import BAND, MAX_MISMATCH_FRACTION, check_fp16, normwise_rel, np_f16, np_u32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def rot_for(d, dev):
    Pi, S = W.rotation(d), W.jl_matrix(d)
    return Pi, tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))


def check_mixed_codes(gwords, ora, gb, d):
    gi = Q.unpack_mixed(gwords, gb)
    oi = ora["idx"]
    mism = gi != oi
    nm = int(mism.sum())
    if nm:
        v, j = np.nonzero(mism)
        assert np.all(np.abs(gi[v, j] - oi[v, j]) == 1), "mismatched indices are not neighbours"
        for vv, jj in zip(v, j):
            t = lloyd_max(d, gb[jj // 32]).t32.astype(np.float64)
            k = min(gi[vv, jj], oi[vv, jj])
            assert np.sqrt(d) * abs(ora["y"][vv, jj] - t[k]) < BAND
    assert nm <= MAX_MISMATCH_FRACTION * oi.size
    return nm


@pytest.mark.parametrize("d,gb", [(128, [3, 3, 2, 2]), (128, [4, 1, 2, 3]), (64, [2, 3]), (64, [1, 4]),
                                  (96, [4, 4, 1])])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mixed_encode_decode(dev, d, gb, dtype):
    n = 5000
    x = W.kv_block(1, n, d, 3, 20.0, 0.5, seed=d + sum(gb), tag=W.TAG_K)[0]
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Pi, rot = rot_for(d, dev)
    codes = torch.empty((n, sum(gb)), dtype=torch.int32, device=dev)
    norms = torch.empty((n,), dtype=torch.float16, device=dev)
    tq.tq_encode_mse_mixed(gb, torch.from_numpy(x).to(dev).to(dt), rot, codes, norms)
    tq.tq_sync_check()
    cbs = {b: lloyd_max(d, b) for b in set(gb)}
    ora = Q.encode_mse_mixed(x, Pi, cbs, gb)
    nm = check_mixed_codes(np_u32(codes), ora, gb, d)
    check_fp16(np_f16(norms), ora["n"], "norms")
    for odt in (torch.float32, torch.bfloat16):
        out = torch.empty((n, d), dtype=odt, device=dev)
        tq.tq_decode_mixed(gb, rot, codes, norms, out)
        tq.tq_sync_check()
        want = Q.decode_mixed(np_u32(codes), np_f16(norms), Pi, cbs, gb)
        rel = normwise_rel(out.float().cpu().numpy(), want)
        tol = 1e-3 if odt == torch.float32 else 1e-3 + 2.0 ** -8
        print("mixed", d, gb, dtype, odt, "code mismatches", nm, "decode max rel", rel.max())
        assert rel.max() <= tol
        if odt == torch.float32:
            assert rel.max() <= 1e-5


@pytest.mark.parametrize("d,b", [(128, 3), (64, 2), (128, 4)])
def test_mixed_uniform_map_equals_plain_encode(dev, d, b):
    n = 777
    x = W.gaussian(n, d, seed=b)
    Pi, rot = rot_for(d, dev)
    gb = [b] * (d // 32)
    c1 = torch.empty((n, sum(gb)), dtype=torch.int32, device=dev)
    n1 = torch.empty((n,), dtype=torch.float16, device=dev)
    tq.tq_encode_mse_mixed(gb, torch.from_numpy(x).to(dev), rot, c1, n1)
    c2, n2 = tq.empty_mse(n, d, b)
    tq.tq_encode_mse(tq.tq_codebook_init(d, b), torch.from_numpy(x).to(dev), rot, c2, n2)
    tq.tq_sync_check()
    assert torch.equal(c1.view(-1), c2.view(-1)) and torch.equal(n1, n2)
