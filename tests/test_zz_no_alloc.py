"""tq_attend_decode_noalloc: the attention entry point whose scratch is the library's fixed device
array instead of a caller workspace.

Its output is checked against tq_attend_decode (caller workspace) on the same inputs, for two
calls in a row with different sizes (so a call that depended on what an earlier call left in the
shared array would show), and once more for the first case after the second. The tolerance is the
one the attention parity tests use: 1e-3 relative, normwise per output vector. The file is named
to be collected last, so it also runs after every other GPU test in the same process.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from parity import normwise_rel

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")

TOL = 1e-3


def _cache(B, Hkv, T, d, kb, vb, dev, seed):
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    n = B * Hkv * T
    K = np.concatenate([W.kv_block(Hkv, T, d, 3, 20.0, 0.5, seed=seed, tag=W.TAG_K, batch_index=b)
                        for b in range(B)]).reshape(n, d)
    V = np.concatenate([W.kv_block(Hkv, T, d, 3, 20.0, 0.5, seed=seed, tag=W.TAG_V, batch_index=b)
                        for b in range(B)]).reshape(n, d)
    cbk, cbv = tq.tq_codebook_init(d, kb), tq.tq_codebook_init(d, vb - 1)
    kc, kn = tq.empty_mse(n, d, kb)
    vc, vs, vn, vg = tq.empty_prod(n, d, vb)
    tq.tq_encode_mse(cbk, torch.from_numpy(K).to(dev).to(torch.bfloat16), rot, kc, kn)
    tq.tq_encode_prod(cbv, torch.from_numpy(V).to(dev).to(torch.bfloat16), rot, vc, vs, vn, vg)
    q = torch.from_numpy(W.queries_bf16((B, Hkv * 4, d), seed=seed)).to(dev).to(torch.bfloat16)
    return dict(B=B, Hkv=Hkv, T=T, d=d, rot=rot, cbk=cbk, cbv=cbv, kc=kc, kn=kn.view(B, Hkv, T), vc=vc, vs=vs,
                vn=vn.view(B, Hkv, T), vg=vg.view(B, Hkv, T), q=q)


def _attend(c, fn, **kw):
    out = torch.full((c["B"], c["q"].shape[1], c["d"]), float("nan"), dtype=torch.float32, device=c["q"].device)
    fn(c["cbk"], c["cbv"], c["q"], c["rot"], c["kc"], c["kn"], c["vc"], c["vn"], out,
       v_signs=c["vs"], v_gammas=c["vg"], **kw)
    return out


def _rel(got, want):
    g, w = got.cpu().numpy().reshape(-1, got.shape[-1]), want.cpu().numpy().reshape(-1, want.shape[-1])
    return max(normwise_rel(g[i], w[i]) for i in range(g.shape[0]))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(gpu_required):
    dev = torch.device("cuda")
    a = _cache(2, 2, 1000, 128, 3, 3, dev, seed=1)
    b = _cache(3, 4, 333, 128, 2, 2, dev, seed=2)
    assert tq.tq_attend_workspace_bytes(2, 8, 2, 1000, 128) <= tq.TQ_ATTEND_NOALLOC_MAX_BYTES
    # two calls in a row on the fixed scratch, then the first case again
    got_a = _attend(a, tq.tq_attend_decode_noalloc)
    got_b = _attend(b, tq.tq_attend_decode_noalloc)
    got_a2 = _attend(a, tq.tq_attend_decode_noalloc)
    tq.tq_sync_check()
    want_a = _attend(a, tq.tq_attend_decode)
    want_b = _attend(b, tq.tq_attend_decode)
    tq.tq_sync_check()
    for got, want in ((got_a, want_a), (got_b, want_b), (got_a2, want_a)):
        assert torch.isfinite(got).all()
        assert _rel(got, want) <= TOL


def test_noalloc_rejects_oversize():
    """Sizes whose scratch exceeds the fixed array are refused on the host, before any device work
    (so this runs without a GPU; the pointers are never dereferenced)."""
    L = tq.lib()
    B, Hq, Hkv, T, d = 64, 256, 32, 1 << 20, 128
    need = int(L.tq_attend_workspace_bytes(B, Hq, Hkv, T, d))
    assert need > tq.TQ_ATTEND_NOALLOC_MAX_BYTES
    cb = tq.Codebook()
    fake = ctypes.c_void_p(1 << 20)
    st = L.tq_attend_decode_noalloc(ctypes.byref(cb), ctypes.byref(cb), B, Hq, Hkv, T, d, fake, tq.TQ_BF16, fake,
                                    fake, fake, None, None, fake, fake, fake, fake, 0.1, fake, None)
    assert st == tq.TQ_ERR_WORKSPACE
    msg = L.tq_last_error().decode()
    assert str(need) in msg


@pytest.mark.gpu
def test_noalloc_many_chunks_per_cta(gpu_required):
    """A size where every CTA walks many chunks (B=2, Hq=32, Hkv=8, T=16384: 2048 chunks over the SMs),
    noalloc against the workspace entry point, twice in a row."""
    dev = torch.device("cuda")
    B, Hkv, T, d = 2, 8, 16384, 128
    Pi, S = W.rotation(d), W.jl_matrix(d)
    rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
    n = B * Hkv * T
    cbk, cbv = tq.tq_codebook_init(d, 3), tq.tq_codebook_init(d, 1)
    kc, kn = tq.empty_mse(n, d, 3)
    vc, vs, vn, vg = tq.empty_prod(n, d, 2)
    tq.tq_encode_mse(cbk, W.kv_slices_device(B * Hkv, T, d, 3, 20.0, 0.5, 21, dev), rot, kc, kn)
    tq.tq_encode_prod(cbv, W.kv_slices_device(B * Hkv, T, d, 3, 20.0, 0.5, 22, dev), rot, vc, vs, vn, vg)
    q = torch.from_numpy(W.queries_bf16((B, 32, d), seed=4)).to(dev).to(torch.bfloat16)
    c = dict(B=B, Hkv=Hkv, T=T, d=d, rot=rot, cbk=cbk, cbv=cbv, kc=kc, kn=kn.view(B, Hkv, T), vc=vc, vs=vs,
             vn=vn.view(B, Hkv, T), vg=vg.view(B, Hkv, T), q=q)
    got1 = _attend(c, tq.tq_attend_decode_noalloc)
    got2 = _attend(c, tq.tq_attend_decode_noalloc)
    want = _attend(c, tq.tq_attend_decode)
    tq.tq_sync_check()
    for got in (got1, got2):
        assert torch.isfinite(got).all()
        assert _rel(got, want) <= TOL


def test_noalloc_array_covers_the_decode_attention_workload():
    """The fixed array is sized for the decode-attention workload (B=16, Hq=32, Hkv=8, T=131072,
    d=128) with room to spare; a change to the workspace plan that outgrew it would fail here."""
    need = tq.tq_attend_workspace_bytes(16, 32, 8, 131072, 128)
    assert 0 < need <= tq.TQ_ATTEND_NOALLOC_MAX_BYTES
