"""GPU parity of tq_attend_append (append the new token's K / V, then attend) (B200).

A compact cache of T_cur + 1 tokens is encoded with the plain encoders; its first T_cur tokens are
copied into a larger cache of T_max slots per slice whose other slots hold a sentinel, and
tq_attend_append appends the last token's raw K / V (its prep kernel encodes them in fp64).
Checked:
  * the appended slot holds the oracle's encoding of that token (keys Algorithm 1, values
    Algorithm 2): codes and signs exact outside the 1e-5 band of a decision, fp16 norms / gammas
    exact up to the 2^-20 midpoint rule; earlier slots are unchanged and later slots still hold the
    sentinel;
  * the output equals tq_attend_decode over the first T_cur + 1 slots bit for bit (same kernels, same
    split of the chunks, the cache read with a slot stride);
  * the output matches the oracle's fp64 attention over the dequantised cache (1e-3 normwise).
"""
import numpy as np
import pytest

import workloads as W
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import check_codes, check_fp16, check_signs, normwise_rel, np_f16, np_u32
from test_gpu_attend import make_cache, oracle_attention

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")

SENTINEL = 0x5A5A5A5A


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


@pytest.mark.parametrize("B,Hq,Hkv,T_cur,T_max", [(2, 8, 2, 0, 5), (2, 8, 2, 127, 200), (1, 4, 1, 128, 129),
                                                 (2, 8, 2, 300, 1000), (1, 16, 2, 200, 260)])
def test_append_then_attend(dev, B, Hq, Hkv, T_cur, T_max):
    d, kb, vb = 128, 3, 2
    T = T_cur + 1
    cache = make_cache(B, Hkv, T, d, kb, vb, True, dev)
    G = d // 32
    # the raw K / V of the compact cache (same seeds as make_cache); the last token of each slice is new
    K = np.stack([W.kv_block(Hkv, T, d, 3, 20.0, 0.5, seed=0, tag=W.TAG_K, batch_index=b) for b in range(B)])
    V = np.stack([W.kv_block(Hkv, T, d, 3, 20.0, 0.5, seed=0, tag=W.TAG_V, batch_index=b) for b in range(B)])
    k_new = torch.from_numpy(np.ascontiguousarray(K[:, :, T_cur])).to(dev).to(torch.bfloat16)
    v_new = torch.from_numpy(np.ascontiguousarray(V[:, :, T_cur])).to(dev).to(torch.bfloat16)

    # the cache with T_max slots per slice: sentinel everywhere, then the first T_cur compact tokens
    def grow(compact, inner, dtype):
        x = torch.full((B, Hkv, T_max) + inner, SENTINEL if dtype == torch.int32 else 0, dtype=torch.int32,
                       device=dev)
        if dtype == torch.float16:
            x = torch.full((B, Hkv, T_max) + inner, 0x5A5A, dtype=torch.int16, device=dev).view(torch.float16)
        c = compact.view((B, Hkv, T) + inner)
        x[:, :, :T_cur] = c[:, :, :T_cur]
        return x
    kc = grow(cache["kc"], (G, kb), torch.int32)
    vc = grow(cache["vc"], (G, vb - 1), torch.int32)
    vs = grow(cache["vs"], (G,), torch.int32)
    kn = grow(cache["kn"], (), torch.float16)
    vn = grow(cache["vn"], (), torch.float16)
    vg = grow(cache["vg"], (), torch.float16)
    before = [t.clone() for t in (kc, vc, vs, kn, vn, vg)]

    q_np = W.queries_bf16((B, Hq, d))
    q = torch.from_numpy(q_np).to(dev).to(torch.bfloat16)
    out = torch.full((B, Hq, d), float("nan"), device=dev)
    tq.tq_attend_append(cache["cbk"], cache["cbv"], q, cache["rot"], k_new, v_new, T_cur,
                        kc.view(B, Hkv, T_max, -1), kn, vc.view(B, Hkv, T_max, -1), vs.view(B, Hkv, T_max, -1),
                        vn, vg, out)
    tq.tq_sync_check()

    # records: slot T_cur holds the oracle's encoding of the new token, the rest is as before
    Pi, S = cache["Pi"], cache["S"]
    kx = K[:, :, T_cur].reshape(B * Hkv, d)
    vx = V[:, :, T_cur].reshape(B * Hkv, d)
    okb, ovb = lloyd_max(d, kb), lloyd_max(d, vb - 1)
    ek = Q.encode_mse(kx, Pi, okb)
    ev = Q.encode_prod(vx, Pi, S, ovb)
    gk = np_u32(kc[:, :, T_cur].contiguous()).reshape(B * Hkv, G, kb)
    gv = np_u32(vc[:, :, T_cur].contiguous()).reshape(B * Hkv, G, vb - 1)
    check_codes(gk, ek["idx"], ek["y"], okb.t32, kb, d)
    check_codes(gv, ev["idx"], ev["y"], ovb.t32, vb - 1, d)
    gidx = Q.unpack_planes(gv, vb - 1)
    ev2 = Q.residual_signs(ev["u"], gidx, ev["n"], Pi, S, ovb)
    check_signs(np_u32(vs[:, :, T_cur].contiguous()).reshape(B * Hkv, G), ev2["z"], ev2["s"], ev2["gamma"], d)
    check_fp16(np_f16(kn[:, :, T_cur].contiguous()).reshape(-1), ek["n"], "key norms")
    check_fp16(np_f16(vn[:, :, T_cur].contiguous()).reshape(-1), ev["n"], "value norms")
    check_fp16(np_f16(vg[:, :, T_cur].contiguous()).reshape(-1), ev2["gamma"], "gammas")
    for now, was in zip((kc, vc, vs, kn, vn, vg), before):
        a = now.view(torch.int16) if now.dtype == torch.float16 else now
        b_ = was.view(torch.int16) if was.dtype == torch.float16 else was
        assert torch.equal(a[:, :, :T_cur], b_[:, :, :T_cur])
        assert torch.equal(a[:, :, T_cur + 1:], b_[:, :, T_cur + 1:])

    # the same attention over the first T_cur + 1 slots as a compact cache, bit for bit
    cut = lambda t: t[:, :, :T].contiguous()
    ckc, ckn, cvc, cvs, cvn, cvg = (cut(t) for t in (kc, kn, vc, vs, vn, vg))
    ref = torch.empty_like(out)
    tq.tq_attend_decode(cache["cbk"], cache["cbv"], q, cache["rot"], ckc.view(-1, G, kb), ckn, cvc.view(-1, G, vb - 1),
                        cvn, ref, v_signs=cvs.view(-1, G), v_gammas=cvg)
    tq.tq_sync_check()
    assert torch.equal(out, ref)

    # the oracle over the cache as the GPU wrote it
    grown = dict(cache, kc=ckc, kn=ckn, vc=cvc, vs=cvs, vn=cvn, vg=cvg)
    want = oracle_attention(grown, q_np, B, Hq, Hkv, T, d)
    got = out.cpu().numpy()
    rel = np.array([normwise_rel(got[b, h], want[(b, h)]) for (b, h) in want])
    print("append", (B, Hq, Hkv, T_cur, T_max), "max rel", rel.max())
    assert rel.max() <= 1e-3
