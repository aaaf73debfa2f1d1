"""GPU parity of tq_scores (inner-product scores from the codes, top-k) against the oracle (B200).

The database codes are made by the oracle's encoder (so the large-d cases do not depend on the
GPU encoder); the oracle then dequantises them explicitly and takes plain fp64 dot products with
the queries. Tolerances: scores 1e-3 relative, normwise per query row; top-k ids compared as sets,
a mismatch allowed only where the oracle's score of the GPU's id is within 1e-3 RMS(row) of the
oracle's k-th score.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import normwise_rel

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def database(n, d, cbits, alg2, seed, dev):
    """Unit-norm Gaussian database encoded by the oracle; returns host arrays and device tensors."""
    Pi, S = W.rotation(d), W.jl_matrix(d)
    x = W.unit_rows(n, d, seed=seed) if n > 0 else np.zeros((0, d))
    cb = lloyd_max(d, cbits)
    if alg2:
        e = Q.encode_prod(x, Pi, S, cb)
    else:
        e = Q.encode_mse(x, Pi, cb)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    db = dict(Pi=Pi, S=S, cb=cb, rot=rot, n=n, d=d, alg2=alg2,
              codes=t(e["codes"].astype(np.uint32), np.int32), norms=t(e["norms"], np.int16).view(torch.float16),
              e=e)
    if alg2:
        db["signs"] = t(e["signs"].astype(np.uint32), np.int32)
        db["gammas"] = t(e["gammas"], np.int16).view(torch.float16)
    else:
        db["signs"] = db["gammas"] = None
    return db


def oracle_scores(db, qh):
    e = db["e"]
    if db["alg2"]:
        xh = Q.decode(e["codes"], e["norms"], db["Pi"], db["cb"], e["signs"], e["gammas"], db["S"])
    else:
        xh = Q.decode(e["codes"], e["norms"], db["Pi"], db["cb"])
    return OA.scores(qh, xh)


def gpu_scores(db, q, k=0, want_scores=True, dev=None):
    nq = q.shape[0]
    cbt = tq.tq_codebook_init(db["d"], db["cb"].bits)
    sc = torch.full((nq, db["n"]), float("nan"), device=dev) if want_scores else None
    ids = torch.full((nq, k), -7, dtype=torch.int32, device=dev) if k else None
    vals = torch.full((nq, k), float("nan"), device=dev) if k else None
    tq.tq_scores(cbt, q, db["rot"], db["codes"], db["norms"], db["signs"], db["gammas"], scores=sc, k=k,
                 topk_ids=ids, topk_scores=vals)
    tq.tq_sync_check()
    return (sc.cpu().numpy() if sc is not None else None,
            ids.cpu().numpy() if k else None, vals.cpu().numpy() if k else None)


def check_topk(ids, vals, want_scores, k):
    oi, os_ = OA.topk(want_scores, k)
    rms = np.sqrt(np.mean(want_scores ** 2, axis=1))
    for r in range(want_scores.shape[0]):
        got = set(int(i) for i in ids[r] if i >= 0)
        assert len(got) == min(k, want_scores.shape[1])
        for i in got - set(int(i) for i in oi[r]):
            assert want_scores[r, i] >= os_[r, -1] - 1e-3 * rms[r], (r, i)
        # the reported scores are the GPU's scores of those ids, in descending order
        v = vals[r][: len(got)]
        assert np.all(np.diff(v) <= 0)


def queries(nq, d, seed=5):
    return W.unit_rows(nq, d, seed=seed)


@pytest.mark.parametrize("cbits,alg2", [(1, False), (2, False), (3, False), (4, False), (1, True), (2, True),
                                        (3, True)])
def test_scores_d128(dev, cbits, alg2):
    d, n, nq = 128, 1000, 7
    db = database(n, d, cbits, alg2, seed=cbits + 10 * alg2, dev=dev)
    qh = queries(nq, d)
    got, ids, vals = gpu_scores(db, torch.from_numpy(qh.astype(np.float32)).to(dev), k=10, dev=dev)
    want = oracle_scores(db, qh)
    rel = max(normwise_rel(got[r], want[r]) for r in range(nq))
    print("scores d128", cbits, alg2, "max rel", rel)
    assert rel <= 1e-3
    check_topk(ids, vals, want, 10)


@pytest.mark.parametrize("d,n,nq", [(64, 300, 130), (192, 129, 1), (1536, 600, 40)])
def test_scores_shapes(dev, d, n, nq):
    db = database(n, d, 3, True, seed=d, dev=dev)
    qh = queries(nq, d, seed=d + 1)
    q = torch.from_numpy(qh.astype(np.float32)).to(dev).to(torch.bfloat16)
    got, ids, vals = gpu_scores(db, q, k=10, dev=dev)
    want = oracle_scores(db, q.float().cpu().numpy())
    rel = max(normwise_rel(got[r], want[r]) for r in range(nq))
    print("scores", (d, n, nq), "max rel", rel)
    assert rel <= 1e-3
    check_topk(ids, vals, want, min(10, n))


def test_topk_chunked_without_scores(dev):
    # more database vectors than one score chunk: the running top-k is merged across chunks
    d, n, nq, k = 64, 70000, 3, 16
    db = database(n, d, 2, True, seed=3, dev=dev)
    qh = queries(nq, d, seed=4)
    _, ids, vals = gpu_scores(db, torch.from_numpy(qh.astype(np.float32)).to(dev), k=k, want_scores=False, dev=dev)
    want = oracle_scores(db, qh)
    check_topk(ids, vals, want, k)


def test_topk_fewer_vectors_than_k(dev):
    d, n, nq, k = 128, 5, 2, 10
    db = database(n, d, 2, False, seed=6, dev=dev)
    qh = queries(nq, d, seed=7)
    got, ids, vals = gpu_scores(db, torch.from_numpy(qh.astype(np.float32)).to(dev), k=k, dev=dev)
    want = oracle_scores(db, qh)
    for r in range(nq):
        assert sorted(ids[r][:n].tolist()) == sorted(np.argsort(-want[r])[:n].tolist())
        assert np.all(ids[r][n:] == -1) and np.all(np.isneginf(vals[r][n:]))


def test_empty_database(dev):
    d, nq, k = 128, 3, 4
    db = database(0, d, 2, False, seed=8, dev=dev)
    q = torch.from_numpy(queries(nq, d).astype(np.float32)).to(dev)
    _, ids, vals = gpu_scores(db, q, k=k, want_scores=False, dev=dev)
    assert np.all(ids == -1) and np.all(np.isneginf(vals))
