"""GPU parity of tq_attend_decode against the oracle (B200).

The cache is encoded on the GPU (keys Algorithm 1, values Algorithm 2 unless stated); the oracle
dequantises the GPU's own packed bytes and evaluates softmax(q k_hat / sqrt(d)) v_hat in fp64, so
the comparison isolates the attention arithmetic. Tolerance: 1e-3 relative, normwise per output
vector.
"""
import math

import numpy as np
import pytest

import workloads as W
from oracle import attention as OA
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import normwise_rel, np_f16, np_u32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def make_cache(B, Hkv, T, d, kb, vb, v_alg2, dev, n_outlier=3, sigma=0.5, seed=0, k_alg2=False):
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    K = np.stack([W.kv_block(Hkv, T, d, n_outlier, 20.0, sigma, seed=seed, tag=W.TAG_K, batch_index=b)
                  for b in range(B)])
    V = np.stack([W.kv_block(Hkv, T, d, n_outlier, 20.0, sigma, seed=seed, tag=W.TAG_V, batch_index=b)
                  for b in range(B)])
    n = B * Hkv * T
    if k_alg2:
        cbk = tq.tq_codebook_init(d, kb - 1)
        kc, ks, kn, kg = tq.empty_prod(n, d, kb)
        tq.tq_encode_prod(cbk, torch.from_numpy(K.reshape(n, d)).to(dev).to(torch.bfloat16), rot, kc, ks, kn, kg)
    else:
        cbk = tq.tq_codebook_init(d, kb)
        kc, kn = tq.empty_mse(n, d, kb)
        ks = kg = None
        tq.tq_encode_mse(cbk, torch.from_numpy(K.reshape(n, d)).to(dev).to(torch.bfloat16), rot, kc, kn)
    if v_alg2:
        cbv = tq.tq_codebook_init(d, vb - 1)
        vc, vs, vn, vg = tq.empty_prod(n, d, vb)
        tq.tq_encode_prod(cbv, torch.from_numpy(V.reshape(n, d)).to(dev).to(torch.bfloat16), rot, vc, vs, vn, vg)
    else:
        cbv = tq.tq_codebook_init(d, vb)
        vc, vn = tq.empty_mse(n, d, vb)
        vs = vg = None
        tq.tq_encode_mse(cbv, torch.from_numpy(V.reshape(n, d)).to(dev).to(torch.bfloat16), rot, vc, vn)
    tq.tq_sync_check()
    return dict(Pi=Pi, S=S, rot=rot, cbk=cbk, cbv=cbv, kc=kc, kn=kn, ks=ks, kg=kg, vc=vc, vs=vs, vn=vn, vg=vg,
                n=n, kb=kb, vb=vb, v_alg2=v_alg2, k_alg2=k_alg2)


def oracle_attention(cache, q, B, Hq, Hkv, T, d, slices=None):
    Pi, S = cache["Pi"], cache["S"]
    n = cache["n"]
    kb, vb = cache["kb"], cache["vb"]
    k_alg2 = cache.get("k_alg2", False)
    kbits = kb - 1 if k_alg2 else kb
    okb = lloyd_max(d, kbits)
    ovb = lloyd_max(d, vb - 1) if cache["v_alg2"] else lloyd_max(d, vb)
    kc = np_u32(cache["kc"]).reshape(B, Hkv, T, d // 32, kbits)
    if k_alg2:
        ks = np_u32(cache["ks"]).reshape(B, Hkv, T, d // 32)
        kg = np_f16(cache["kg"]).reshape(B, Hkv, T)
    kn = np_f16(cache["kn"]).reshape(B, Hkv, T)
    vbits = vb - 1 if cache["v_alg2"] else vb
    vc = np_u32(cache["vc"]).reshape(B, Hkv, T, d // 32, vbits)
    vn = np_f16(cache["vn"]).reshape(B, Hkv, T)
    if cache["v_alg2"]:
        vs = np_u32(cache["vs"]).reshape(B, Hkv, T, d // 32)
        vg = np_f16(cache["vg"]).reshape(B, Hkv, T)
    grp = Hq // Hkv
    out = {}
    for (b, hk) in (slices or [(b, hk) for b in range(B) for hk in range(Hkv)]):
        if k_alg2:
            kh = Q.decode(kc[b, hk], kn[b, hk], Pi, okb, ks[b, hk], kg[b, hk], S)
        else:
            kh = Q.decode(kc[b, hk], kn[b, hk], Pi, okb)
        if cache["v_alg2"]:
            vh = Q.decode(vc[b, hk], vn[b, hk], Pi, ovb, vs[b, hk], vg[b, hk], S)
        else:
            vh = Q.decode(vc[b, hk], vn[b, hk], Pi, ovb)
        o = OA.softmax_attend(q[b, hk * grp:(hk + 1) * grp].astype(np.float64), kh, vh, 1.0 / math.sqrt(d))
        for h in range(grp):
            out[(b, hk * grp + h)] = o[h]
    return out


def run_attend(cache, q_np, B, Hq, Hkv, T, d, dev):
    q = torch.from_numpy(q_np).to(dev).to(torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    n = cache["n"]
    tq.tq_attend_decode(cache["cbk"], cache["cbv"], q, cache["rot"],
                        cache["kc"], cache["kn"].view(B, Hkv, T), cache["vc"], cache["vn"].view(B, Hkv, T), out,
                        v_signs=cache["vs"], v_gammas=cache["vg"], k_signs=cache.get("ks"), k_gammas=cache.get("kg"))
    tq.tq_sync_check()
    return out.cpu().numpy()


@pytest.mark.parametrize("B,Hq,Hkv,T", [(1, 4, 1, 128), (2, 8, 2, 300), (1, 4, 1, 1), (3, 8, 2, 129),
                                        (2, 16, 2, 1000)])
def test_attend_small(dev, B, Hq, Hkv, T):
    d = 128
    cache = make_cache(B, Hkv, T, d, 3, 2, True, dev)
    q_np = W.queries_bf16((B, Hq, d))
    got = run_attend(cache, q_np, B, Hq, Hkv, T, d, dev)
    want = oracle_attention(cache, q_np, B, Hq, Hkv, T, d)
    rel = np.array([normwise_rel(got[b, h], want[(b, h)]) for (b, h) in want])
    print("attend", (B, Hq, Hkv, T), "max rel", rel.max())
    assert rel.max() <= 1e-3


@pytest.mark.parametrize("kb,vb,v_alg2", [(1, 1, False), (2, 3, True), (3, 2, False), (2, 2, True), (1, 3, True)])
def test_attend_bit_widths(dev, kb, vb, v_alg2):
    B, Hq, Hkv, T, d = 2, 8, 2, 700, 128
    cache = make_cache(B, Hkv, T, d, kb, vb, v_alg2, dev)
    q_np = W.queries_bf16((B, Hq, d))
    got = run_attend(cache, q_np, B, Hq, Hkv, T, d, dev)
    want = oracle_attention(cache, q_np, B, Hq, Hkv, T, d)
    rel = np.array([normwise_rel(got[b, h], want[(b, h)]) for (b, h) in want])
    print("attend bits", (kb, vb, v_alg2), "max rel", rel.max())
    assert rel.max() <= 1e-3


@pytest.mark.parametrize("B,Hq,Hkv,T", [(2, 8, 2, 300), (1, 16, 2, 700)])
@pytest.mark.parametrize("kb,vb,v_alg2", [(3, 2, True), (2, 3, True), (3, 2, False)])
def test_attend_alg2_keys(dev, B, Hq, Hkv, T, kb, vb, v_alg2):
    # Algorithm 2 keys: scores carry the QJL term alpha gamma <S q, 2z - 1> of the unbiased estimate
    d = 128
    cache = make_cache(B, Hkv, T, d, kb, vb, v_alg2, dev, k_alg2=True)
    q_np = W.queries_bf16((B, Hq, d))
    got = run_attend(cache, q_np, B, Hq, Hkv, T, d, dev)
    want = oracle_attention(cache, q_np, B, Hq, Hkv, T, d)
    rel = np.array([normwise_rel(got[b, h], want[(b, h)]) for (b, h) in want])
    print("attend alg2 keys", (B, Hq, Hkv, T, kb, vb, v_alg2), "max rel", rel.max())
    assert rel.max() <= 1e-3
