"""Pins for the oracle's scores, decode attention and top-k (CPU only)."""
import math

import numpy as np
import pytest

from oracle import attention as A


def _loop_attention(q, k, v, scale):
    # textbook definition with pure-Python loops (tiny sizes only)
    H, d = len(q), len(q[0])
    T = len(k)
    out = []
    for h in range(H):
        logits = [sum(q[h][i] * k[t][i] for i in range(d)) * scale for t in range(T)]
        m = max(logits)
        w = [math.exp(l - m) for l in logits]
        s = sum(w)
        out.append([sum(w[t] * v[t][i] for t in range(T)) / s for i in range(d)])
    return np.array(out)


def test_attention_matches_loops():
    g = np.random.default_rng(0)
    B, Hq, Hkv, T, d = 2, 4, 2, 37, 8
    q = g.standard_normal((B, Hq, d))
    k = g.standard_normal((B, Hkv, T, d)) * 2
    v = g.standard_normal((B, Hkv, T, d))
    out = A.decode_attention(q, k, v, 1 / math.sqrt(d))
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            want = _loop_attention(q[b, h:h + 1].tolist(), k[b, hk].tolist(), v[b, hk].tolist(),
                                   1 / math.sqrt(d))
            assert np.allclose(out[b, h], want[0], rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    g = np.random.default_rng(1)
    d = 16
    q = g.standard_normal((3, d))
    v = g.standard_normal((5, d))
    # one token: output is that value
    assert np.allclose(A.softmax_attend(q, g.standard_normal((1, d)), v[:1], 0.3), v[:1].repeat(3, 0))
    # identical keys: the mean of the values
    k = np.repeat(g.standard_normal((1, d)), 5, axis=0)
    assert np.allclose(A.softmax_attend(q, k, v, 0.3), v.mean(0)[None].repeat(3, 0))
    # a dominant key: its value
    k = g.standard_normal((5, d)) * 0.01
    k[2] = q[0] * 1e3
    assert np.allclose(A.softmax_attend(q[:1], k, v, 1.0), v[2][None])
    # large logits do not overflow (max subtraction)
    assert np.all(np.isfinite(A.softmax_attend(q, k * 1e6, v, 1.0)))


def test_scores_are_dot_products():
    g = np.random.default_rng(2)
    q = g.standard_normal((3, 8))
    x = g.standard_normal((4, 8))
    s = A.scores(q, x)
    for i in range(3):
        for j in range(4):
            assert abs(s[i, j] - sum(q[i, t] * x[j, t] for t in range(8))) < 1e-12


def test_topk_brute_force_with_ties():
    s = np.array([[0.5, 0.9, 0.5, -1.0, 0.9, 0.1], [3, 3, 3, 3, 3, 3]], dtype=np.float64)
    ids, vals = A.topk(s, 3)
    for r in range(2):
        want = sorted(range(6), key=lambda j: (-s[r, j], j))[:3]
        assert list(ids[r]) == want
        assert list(vals[r]) == [s[r, j] for j in want]
    g = np.random.default_rng(3)
    s = g.integers(0, 20, size=(5, 200)).astype(np.float64)
    ids, _ = A.topk(s, 10)
    for r in range(5):
        assert list(ids[r]) == sorted(range(200), key=lambda j: (-s[r, j], j))[:10]


def test_prefill_brute_force_mask():
    """Causal multi-query attention against explicit loops with a mask matrix (tiny sizes)."""
    g = np.random.default_rng(3)
    T, Qn, H, d = 7, 4, 2, 5
    q = g.standard_normal((Qn, H, d))
    k = g.standard_normal((T, d))
    v = g.standard_normal((T, d))
    scale = 0.7
    got = A.prefill_attend(q, k, v, scale)
    for j in range(Qn):
        pos = T - Qn + j
        for h in range(H):
            logit = [sum(q[j, h, i] * k[t, i] for i in range(d)) * scale if t <= pos else -math.inf
                     for t in range(T)]
            m = max(logit)
            w = [math.exp(x - m) if x > -math.inf else 0.0 for x in logit]
            z = sum(w)
            want = [sum(w[t] * v[t, i] for t in range(T)) / z for i in range(d)]
            assert np.allclose(got[j, h], want, rtol=1e-12, atol=1e-12)


def test_prefill_special_cases():
    """One query is decode attention over the whole cache; with T = Q the first query sees only its
    own token (its output is that token's value); the last query always sees the whole cache."""
    g = np.random.default_rng(4)
    T, H, d = 9, 3, 6
    k, v = g.standard_normal((T, d)), g.standard_normal((T, d))
    q1 = g.standard_normal((1, H, d))
    assert np.allclose(A.prefill_attend(q1, k, v, 0.3)[0], A.softmax_attend(q1[0], k, v, 0.3), rtol=1e-14)
    qs = g.standard_normal((T, H, d))
    out = A.prefill_attend(qs, k, v, 0.3)
    assert np.allclose(out[0], np.broadcast_to(v[0], (H, d)), rtol=1e-14)
    assert np.allclose(out[-1], A.softmax_attend(qs[-1], k, v, 0.3), rtol=1e-14)
