"""GPU parity of decode attention where every CTA walks many 128-token chunks (B200).

The attention main kernel splits the chunks of all (batch, KV head) slices evenly over one CTA per
SM, so a CTA walks a contiguous run of chunks that may start and end inside a slice, and the
combine kernel merges the per-CTA partial softmax states. These tests run that regime: the chunk
ring wraps many times, the TMEM and value-plane buffers alternate, the running maximum is rescaled
inside a CTA, and slices are split between CTAs. The oracle dequantises the GPU's own packed cache
and evaluates softmax(q k_hat / sqrt(d)) v_hat in fp64 per sampled slice (aiboss88 page: attention
evaluated on the quantised cache). Tolerance: 1e-3 relative, normwise per output vector.
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

D = 128
CHUNK = 128


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


def chunk_plan(B, Hkv, T):
    """The main kernel's split: chunks per slice, chunks per CTA, CTAs (one per SM at most)."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    nchunk = -(-T // CHUNK)
    total = B * Hkv * nchunk
    ncta = min(nsm, total)
    per_cta = -(-total // ncta)
    return nchunk, per_cta, -(-total // per_cta)


def split_slices(B, Hkv, T):
    """Slices whose chunks are shared by two or more CTAs."""
    nchunk, per_cta, _ = chunk_plan(B, Hkv, T)
    return [s for s in range(B * Hkv) if (s * nchunk) // per_cta != (s * nchunk + nchunk - 1) // per_cta]


class Cache:
    """A packed cache [B][Hkv][T] encoded on the GPU (keys Algorithm 1 or 2, values Algorithm 2)."""

    def __init__(self, dev, B, Hkv, T, kb=3, vb=2, k_alg2=False, host_recipe=True, seed=0):
        self.B, self.Hkv, self.T, self.kb, self.vb, self.k_alg2 = B, Hkv, T, kb, vb, k_alg2
        self.Pi, self.S = W.rotation(D), W.jl_matrix(D)
        self.rot = tq.tq_rotation_prepare(torch.from_numpy(self.Pi).to(dev), torch.from_numpy(self.S).to(dev))
        n = B * Hkv * T
        kbits = kb - 1 if k_alg2 else kb
        self.cbk = tq.tq_codebook_init(D, kbits)
        self.cbv = tq.tq_codebook_init(D, vb - 1)
        if k_alg2:
            self.kc, self.ks, self.kn, self.kg = tq.empty_prod(n, D, kb)
        else:
            (self.kc, self.kn), self.ks, self.kg = tq.empty_mse(n, D, kb), None, None
        self.vc, self.vs, self.vn, self.vg = tq.empty_prod(n, D, vb)
        # all slices are drawn first and encoded in one call per stage (the per-vector norm arrays of
        # a batch element need not start 16-byte aligned)
        per = Hkv * T
        K = torch.empty((n, D), dtype=torch.bfloat16, device=dev)
        V = torch.empty((n, D), dtype=torch.bfloat16, device=dev)
        for b in range(B):
            sl = slice(b * per, (b + 1) * per)
            if host_recipe:
                K[sl] = torch.from_numpy(W.kv_block(Hkv, T, D, 3, 20.0, 0.5, seed=seed, tag=W.TAG_K, batch_index=b)
                                         .reshape(per, D)).to(dev).to(torch.bfloat16)
                V[sl] = torch.from_numpy(W.kv_block(Hkv, T, D, 3, 20.0, 0.5, seed=seed, tag=W.TAG_V, batch_index=b)
                                         .reshape(per, D)).to(dev).to(torch.bfloat16)
            else:
                K[sl] = W.kv_slices_device(Hkv, T, D, 3, 20.0, 0.5, 1000 + 2 * b + seed, dev)
                V[sl] = W.kv_slices_device(Hkv, T, D, 3, 20.0, 0.5, 1001 + 2 * b + seed, dev)
        if k_alg2:
            tq.tq_encode_prod(self.cbk, K, self.rot, self.kc, self.ks, self.kn, self.kg)
        else:
            tq.tq_encode_mse(self.cbk, K, self.rot, self.kc, self.kn)
        tq.tq_encode_prod(self.cbv, V, self.rot, self.vc, self.vs, self.vn, self.vg)
        del K, V
        tq.tq_sync_check()
        self.okb = lloyd_max(D, kbits)
        self.ovb = lloyd_max(D, vb - 1)

    def view3(self, t):
        return None if t is None else t.view(self.B, self.Hkv, self.T)

    def attend(self, q, noalloc=False):
        B, Hq = q.shape[0], q.shape[1]
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
        f = tq.tq_attend_decode_noalloc if noalloc else tq.tq_attend_decode
        f(self.cbk, self.cbv, q, self.rot, self.kc, self.view3(self.kn), self.vc, self.view3(self.vn), out,
          v_signs=self.vs, v_gammas=self.view3(self.vg), k_signs=self.ks, k_gammas=self.view3(self.kg))
        tq.tq_sync_check()
        return out.cpu().numpy()

    def dequant_slice(self, s):
        """The oracle's k_hat, v_hat [T, d] of slice s = b * Hkv + hk from the GPU's packed bytes."""
        T = self.T
        sl = slice(s * T, (s + 1) * T)
        kbits = self.okb.bits
        kc = np_u32(self.kc[sl]).reshape(T, D // 32, kbits)
        kn = np_f16(self.kn[sl])
        if self.k_alg2:
            kh = Q.decode(kc, kn, self.Pi, self.okb, np_u32(self.ks[sl]), np_f16(self.kg[sl]), self.S)
        else:
            kh = Q.decode(kc, kn, self.Pi, self.okb)
        vh = Q.decode(np_u32(self.vc[sl]).reshape(T, D // 32, self.vb - 1), np_f16(self.vn[sl]), self.Pi, self.ovb,
                      np_u32(self.vs[sl]), np_f16(self.vg[sl]), self.S)
        return kh, vh

    def oracle(self, q_np, s, Hq):
        grp = Hq // self.Hkv
        b, hk = divmod(s, self.Hkv)
        kh, vh = self.dequant_slice(s)
        return OA.softmax_attend(q_np[b, hk * grp:(hk + 1) * grp].astype(np.float64), kh, vh, 1.0 / math.sqrt(D))


def check_slices(cache, q_np, got, slices, Hq, label):
    grp = Hq // cache.Hkv
    worst = 0.0
    for s in slices:
        b, hk = divmod(s, cache.Hkv)
        want = cache.oracle(q_np, s, Hq)
        rel = normwise_rel(got[b, hk * grp:(hk + 1) * grp], want)
        worst = max(worst, float(rel.max()))
        assert rel.max() <= 1e-3, f"{label}: slice {s} max rel {rel.max():.3g}"
    print(label, "slices", list(slices), "max rel", worst)
    return worst


def test_bench_shape_sampled(dev):
    """The benchmarked shape itself: B=16, Hq=32, Hkv=8, T=131072 (keys Algorithm 1 at 3 bits, values
    Algorithm 2 at 2 bits), every slice split between CTAs; the first and last slice and six seeded
    others are compared with the oracle."""
    B, Hq, Hkv, T = 16, 32, 8, 131072
    nchunk, per_cta, ncta = chunk_plan(B, Hkv, T)
    assert per_cta > 100                                  # hundreds of chunks per CTA
    cache = Cache(dev, B, Hkv, T, host_recipe=False)
    q_np = W.queries_bf16((B, Hq, D))
    got = cache.attend(torch.from_numpy(q_np).to(dev).to(torch.bfloat16))
    split = split_slices(B, Hkv, T)
    rng = np.random.default_rng(5)
    picks = sorted(set([0, B * Hkv - 1] + list(rng.choice(split, 6, replace=False))))
    check_slices(cache, q_np, got, picks, Hq, "bench shape")


def boost_late_tokens(cache, q_np, Hq, factor_margin=3.0):
    """Raises the key norm of one late token inside several CTAs' chunk runs (by a power of two, so the
    packed record stays exactly the encoding of the scaled vector) such that its logit for query
    head 0 of its slice exceeds every earlier logit of that run by about `factor_margin`: the running
    maximum must then be rescaled in the middle of a CTA's run."""
    B, Hkv, T = cache.B, cache.Hkv, cache.T
    nchunk, per_cta, ncta = chunk_plan(B, Hkv, T)
    grp = Hq // Hkv
    kn = cache.kn.view(torch.int16).cpu().numpy().view(np.float16).copy()
    boosted = []
    for s in range(B * Hkv):
        b, hk = divmod(s, Hkv)
        kh, _ = cache.dequant_slice(s)
        lg = kh @ q_np[b, hk * grp].astype(np.float64) / math.sqrt(D)
        c0 = s * nchunk
        for j in range(c0 // per_cta, (c0 + nchunk - 1) // per_cta + 1, max(1, ncta // 5)):
            lo = max(j * per_cta, c0) - c0
            hi = min((j + 1) * per_cta, c0 + nchunk) - c0
            if hi - lo < 4:
                continue
            t_lo, t_hi = (lo + (hi - lo) // 2) * CHUNK, min(hi * CHUNK, T)
            seg = lg[t_lo:t_hi]
            t = t_lo + int(np.argmax(seg))
            ell = lg[t]
            m_prev = lg[lo * CHUNK:t].max()
            if ell <= 0:
                continue
            k = max(1, math.ceil(math.log2((m_prev + factor_margin) / ell)))
            if float(kn[s * T + t]) * 2.0 ** k > 6e4:
                continue
            kn[s * T + t] = np.float16(float(kn[s * T + t]) * 2.0 ** k)
            boosted.append((s, t, k))
    cache.kn.copy_(torch.from_numpy(kn.view(np.int16)).view(torch.float16).to(cache.kn.device))
    return boosted


@pytest.mark.parametrize("Hq", [4, 8])
def test_many_chunks_per_cta(dev, Hq):
    """One slice of 148 * 24 * 128 + 37 tokens: every CTA walks 25 chunks (more than the chunk ring,
    the six-slot value-MMA ring and both TMEM buffers), the last chunk is ragged, and late tokens with
    boosted norms force running-maximum rescales inside CTAs. Hq = 4 and 8 cover both warp layouts."""
    B, Hkv = 1, 1
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    T = nsm * 24 * CHUNK + 37
    nchunk, per_cta, ncta = chunk_plan(B, Hkv, T)
    assert per_cta >= 25
    cache = Cache(dev, B, Hkv, T)
    q_np = W.queries_bf16((B, Hq, D))
    boosted = boost_late_tokens(cache, q_np, Hq)
    assert len(boosted) >= 3
    got = cache.attend(torch.from_numpy(q_np).to(dev).to(torch.bfloat16))
    check_slices(cache, q_np, got, [0], Hq, f"many chunks Hq={Hq} boosted={boosted}")


@pytest.mark.parametrize("Hq,kb,vb", [(4, 3, 2), (8, 3, 3)])
def test_many_chunks_alg2_keys(dev, Hq, kb, vb):
    """Algorithm 2 keys (2-bit codebook + QJL sign plane) over many chunks per CTA, several slices
    split between CTAs."""
    B, Hkv = 2, 1
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    T = nsm * 6 * CHUNK + 77
    cache = Cache(dev, B, Hkv, T, kb=kb, vb=vb, k_alg2=True)
    q_np = W.queries_bf16((B, Hq, D))
    boost_late_tokens(cache, q_np, Hq)
    got = cache.attend(torch.from_numpy(q_np).to(dev).to(torch.bfloat16))
    assert split_slices(B, Hkv, T)
    check_slices(cache, q_np, got, range(B * Hkv), Hq, f"alg2 keys Hq={Hq}")


def test_append_long_cache(dev):
    """tq_attend_append at T_cur = 131071 of T_max = 131072 slots, two KV heads: the new records are the
    oracle's encoding of the new token (band rule), no other slot changes, and the attention over the
    131072 filled slots matches the oracle."""
    from oracle import quant as Qo
    from parity import check_codes, check_fp16, check_signs
    B, Hq, Hkv, T = 1, 8, 2, 131072
    cache = Cache(dev, B, Hkv, T, host_recipe=False, seed=3)
    gen_k = W.kv_slices_device(Hkv, T, D, 3, 20.0, 0.5, 1000 + 3, dev).view(Hkv, T, D)
    gen_v = W.kv_slices_device(Hkv, T, D, 3, 20.0, 0.5, 1001 + 3, dev).view(Hkv, T, D)
    k_new = gen_k[:, T - 1].contiguous().view(B, Hkv, D)
    v_new = gen_v[:, T - 1].contiguous().view(B, Hkv, D)
    del gen_k, gen_v
    # wipe the last slot, then append it back
    for t in (cache.kc, cache.vc, cache.vs):
        t.view(B, Hkv, T, -1)[:, :, T - 1].zero_()
    for t in (cache.kn, cache.vn, cache.vg):
        t.view(B, Hkv, T)[:, :, T - 1].zero_()
    before = [t.clone() for t in (cache.kc, cache.kn, cache.vc, cache.vs, cache.vn, cache.vg)]
    q_np = W.queries_bf16((B, Hq, D))
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    tq.tq_attend_append(cache.cbk, cache.cbv, torch.from_numpy(q_np).to(dev).to(torch.bfloat16), cache.rot, k_new,
                        v_new, T - 1, cache.kc, cache.view3(cache.kn), cache.vc, cache.vs, cache.view3(cache.vn),
                        cache.view3(cache.vg), out)
    tq.tq_sync_check()
    for a, b_ in zip((cache.kc, cache.kn, cache.vc, cache.vs, cache.vn, cache.vg), before):
        a3, b3 = a.view(B, Hkv, T, -1), b_.view(B, Hkv, T, -1)
        assert torch.equal(a3[:, :, :T - 1], b3[:, :, :T - 1])
    kx = k_new.float().cpu().numpy().reshape(B * Hkv, D)
    vx = v_new.float().cpu().numpy().reshape(B * Hkv, D)
    ek = Qo.encode_mse(kx, cache.Pi, cache.okb)
    ev = Qo.encode_prod(vx, cache.Pi, cache.S, cache.ovb)
    last = lambda t, inner: t.view((B * Hkv, T) + inner)[:, T - 1].contiguous()
    gk = np_u32(last(cache.kc, (D // 32, 3)))
    gv = np_u32(last(cache.vc, (D // 32, 1)))
    check_codes(gk, ek["idx"], ek["y"], cache.okb.t32, 3, D)
    check_codes(gv, ev["idx"], ev["y"], cache.ovb.t32, 1, D)
    ev2 = Qo.residual_signs(ev["u"], Qo.unpack_planes(gv, 1), ev["n"], cache.Pi, cache.S, cache.ovb)
    check_signs(np_u32(last(cache.vs, (D // 32,))), ev2["z"], ev2["s"], ev2["gamma"], D)
    check_fp16(np_f16(last(cache.kn, ())), ek["n"], "key norms")
    check_fp16(np_f16(last(cache.vg, ())), ev2["gamma"], "gammas")
    got = out.cpu().numpy()
    check_slices(cache, q_np, got, range(B * Hkv), Hq, "append T_cur=131071")
