"""GPU parity of tq_attend_prefill (causal multi-query attention over the packed cache) against the
oracle (B200).

The cache [B][Hkv][T] is encoded on the GPU; its last Qn slots are the new tokens, and query token j
attends the tokens t <= T - Qn + j. The oracle dequantises the GPU's own packed bytes and evaluates
the causal softmax per query in fp64 (techblog-plum page, notes on many queries over the cache;
aiboss88 page, attention on the quantised cache). Tolerance: 1e-3 relative, normwise per output
vector.
"""
import math

import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from parity import normwise_rel
from test_gpu_attend_multichunk import Cache, chunk_plan

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")

D = 128


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def run_prefill(cache, q_np, dev):
    B, Qn, Hq, _ = q_np.shape
    q = torch.from_numpy(q_np).to(dev).to(torch.bfloat16)
    out = torch.full((B, Qn, Hq, D), float("nan"), dtype=torch.float32, device=dev)
    tq.tq_attend_prefill(cache.cbk, cache.cbv, q, cache.rot, cache.kc, cache.view3(cache.kn), cache.vc,
                         cache.view3(cache.vn), out, v_signs=cache.vs, v_gammas=cache.view3(cache.vg),
                         k_signs=cache.ks, k_gammas=cache.view3(cache.kg))
    tq.tq_sync_check()
    return out.cpu().numpy()


def check(cache, q_np, got, label, slices=None):
    B, Qn, Hq, _ = q_np.shape
    grp = Hq // cache.Hkv
    worst = 0.0
    for s in (slices if slices is not None else range(B * cache.Hkv)):
        b, hk = divmod(s, cache.Hkv)
        kh, vh = cache.dequant_slice(s)
        want = OA.prefill_attend(q_np[b, :, hk * grp:(hk + 1) * grp].astype(np.float64), kh, vh, 1.0 / math.sqrt(D))
        g = got[b, :, hk * grp:(hk + 1) * grp]
        rel = normwise_rel(g.reshape(-1, D), want.reshape(-1, D))
        worst = max(worst, float(rel.max()))
        assert np.all(np.isfinite(g)), f"{label}: slice {s} has unwritten outputs"
        assert rel.max() <= 1e-3, f"{label}: slice {s} max rel {rel.max():.3g}"
    print(label, "max rel", worst)


@pytest.mark.parametrize("B,Hq,Hkv,Qn,T,k_alg2", [
    (2, 8, 2, 5, 700, False),      # 4 heads per KV head: 2 query tokens per pass, 3 passes
    (1, 8, 1, 3, 1000, False),     # 8 heads per KV head: 1 query token per pass
    (1, 2, 2, 16, 16, False),      # 1 head per KV head, T = Qn: pure causal self-attention
    (2, 4, 1, 7, 300, True),       # Algorithm 2 keys
    (1, 4, 2, 9, 129, False),      # 2 heads per KV head: 4 query tokens per pass
])
def test_prefill_small(dev, B, Hq, Hkv, Qn, T, k_alg2):
    cache = Cache(dev, B, Hkv, T, kb=3, vb=2 if not k_alg2 else 3, k_alg2=k_alg2)
    q_np = W.queries_bf16((B, Qn, Hq, D))
    got = run_prefill(cache, q_np, dev)
    check(cache, q_np, got, f"prefill {(B, Hq, Hkv, Qn, T, k_alg2)}")


def test_prefill_one_query_is_decode(dev):
    B, Hq, Hkv, T = 2, 8, 2, 333
    cache = Cache(dev, B, Hkv, T)
    q_np = W.queries_bf16((B, 1, Hq, D))
    got = run_prefill(cache, q_np, dev)
    dec = cache.attend(torch.from_numpy(q_np[:, 0]).to(dev).to(torch.bfloat16))
    assert np.array_equal(got[:, 0], dec)


def test_prefill_long_cache(dev):
    """130 new tokens at the end of a cache whose chunks are spread over all SMs (65 passes)."""
    B, Hq, Hkv = 1, 4, 1
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    T = nsm * 6 * 128 + 50
    Qn = 130
    assert chunk_plan(B, Hkv, T)[1] >= 6
    cache = Cache(dev, B, Hkv, T)
    q_np = W.queries_bf16((B, Qn, Hq, D))
    got = run_prefill(cache, q_np, dev)
    check(cache, q_np, got, "prefill long")
