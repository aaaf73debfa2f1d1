"""The vector-search workload at full size on the GPU, checked on samples against the oracle.

Database: 1,000,000 unit-norm fp32 rows, d = 1536 (seeded Gaussian blocks of 4096 rows, drawn one
block at a time so any block can be regenerated alone), Algorithm 2 at 4 bits (3-bit codebook +
residual signs); 1024 unit-norm queries; top-10 by inner-product estimate from the codes.

Checked: codes / signs / norms / gammas of 2000 sampled vectors (the encode parity rules), and the
top-10 ids of 6 sampled queries against the oracle's explicit scores <q, x_hat> over the whole
database (dequantised block by block in fp64), with the top-k tie rule.
"""
import time

import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import check_codes, check_fp16, check_signs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")

N, D, NQ, K, BITS = 1_000_000, 1536, 1024, 10, 4
BLK = 4096


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def test_vector_search_full_size(dev):
    Pi, S = W.rotation(D), W.jl_matrix(D)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    cb = tq.tq_codebook_init(D, BITS - 1)
    x = torch.empty((N, D), dtype=torch.float32, device=dev)
    t0 = time.time()
    for b0 in range(0, N, BLK):
        r = min(BLK, N - b0)
        x[b0:b0 + r] = torch.from_numpy(W.unit_rows_block(b0 // BLK, BLK, D)[:r]).to(dev)
    print(f"database generated in {time.time() - t0:.1f} s")
    codes, signs, norms, gammas = tq.empty_prod(N, D, BITS)
    ws = torch.empty(tq.tq_encode_workspace_bytes(N, D, 2), dtype=torch.uint8, device=dev)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record()
    tq.tq_encode_prod(cb, x, rot, codes, signs, norms, gammas, ws=ws)
    e1.record()
    qh = W.unit_rows(NQ, D, seed=2)
    q = torch.from_numpy(qh).to(dev)
    ids = torch.empty((NQ, K), dtype=torch.int32, device=dev)
    vals = torch.empty((NQ, K), dtype=torch.float32, device=dev)
    sws = torch.empty(tq.tq_scores_workspace_bytes(NQ, N, D, K), dtype=torch.uint8, device=dev)
    tq.tq_scores(cb, q, rot, codes, norms, signs, gammas, scores=None, k=K, topk_ids=ids, topk_scores=vals, ws=sws)
    e2.record()
    tq.tq_sync_check()
    print(f"encode {e0.elapsed_time(e1):.1f} ms, scores + top-{K} {e1.elapsed_time(e2):.1f} ms")
    del x, ws, sws

    ocb = lloyd_max(D, BITS - 1)
    codes_h = codes.cpu().numpy().view(np.uint32)
    signs_h = signs.cpu().numpy().view(np.uint32)
    norms_h = norms.cpu().numpy()
    gammas_h = gammas.cpu().numpy()

    # encode parity on sampled vectors (regenerating only their blocks)
    rng = np.random.default_rng(123)
    sample = np.sort(rng.choice(N, 2000, replace=False))
    xs = np.stack([W.unit_rows_block(i // BLK, BLK, D)[i % BLK] for i in sample])
    ora = Q.encode_prod(xs, Pi, S, ocb)
    st = check_codes(codes_h[sample], ora["idx"], ora["y"], ocb.t32, BITS - 1, D)
    gidx = Q.unpack_planes(codes_h[sample], BITS - 1)
    ora2 = Q.residual_signs(ora["u"], gidx, ora["n"], Pi, S, ocb)
    st["signs"] = check_signs(signs_h[sample], ora2["z"], ora2["s"], ora2["gamma"], D)
    check_fp16(norms_h[sample], ora["n"], "norms")
    check_fp16(gammas_h[sample], ora2["gamma"], "gammas")
    print("sampled encode parity", st)

    # top-10 of sampled queries against the oracle's explicit scores over the whole database
    qs = np.sort(rng.choice(NQ, 6, replace=False))
    want = np.empty((len(qs), N))
    t0 = time.time()
    for b0 in range(0, N, 2 * BLK):
        r = min(2 * BLK, N - b0)
        sl = slice(b0, b0 + r)
        xh = Q.decode(codes_h[sl], norms_h[sl], Pi, ocb, signs_h[sl], gammas_h[sl], S)
        want[:, sl] = OA.scores(qh[qs], xh)
    print(f"oracle scores over the database in {time.time() - t0:.1f} s")
    oi, os_ = OA.topk(want, K)
    rms = np.sqrt(np.mean(want ** 2, axis=1))
    got_ids = ids.cpu().numpy()[qs]
    for r_, qi in enumerate(qs):
        got = set(int(i) for i in got_ids[r_])
        assert len(got) == K
        for i in got - set(int(i) for i in oi[r_]):
            assert want[r_, i] >= os_[r_, -1] - 1e-3 * rms[r_], (qi, i)
    print("top-10 of sampled queries match the oracle")
