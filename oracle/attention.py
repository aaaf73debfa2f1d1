"""Scores, decode attention and top-k over a TurboQuant-packed cache (oracle, fp64).

Sources: aiboss88 page, features and "dual-mode quantisation" -- an MSE mode
and an inner-product mode that gives unbiased attention-score estimates, with
attention computed on the quantised cache; same page, applications -- nearest
neighbour search in vector databases. ai-navigate-news page: keys use
Algorithm 1 (Q K^T), values use Algorithm 2 (attention weights times V).

Plain definitions, deliberately not the code-domain route of the CUDA path:

* score(q, v)  = <q, x_hat_v> with x_hat_v dequantised explicitly (``quant.decode``);
* attention    = softmax_t(<q, k_hat_t> * scale) weighted sum of v_hat_t, per
  (batch, query head), query head h reading KV head h // (Hq / Hkv);
  no causal mask (one decode query sees the whole cache);
* top-k        = the k largest scores, ties to the lower id, descending;
* prefill      = causal multi-query attention: the last Q cached tokens are the queries' own
  tokens, and query j attends the tokens up to and including its own position.
"""
from __future__ import annotations

import numpy as np


def scores(q: np.ndarray, xhat: np.ndarray) -> np.ndarray:
    """[Q, d] x [N, d] -> [Q, N] inner products in fp64."""
    return np.asarray(q, dtype=np.float64) @ np.asarray(xhat, dtype=np.float64).T


def softmax_attend(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, scale: float) -> np.ndarray:
    """q [H, d] against one KV head's khat, vhat [T, d] -> [H, d] (fp64, max-subtracted)."""
    logits = (np.asarray(q, dtype=np.float64) @ np.asarray(khat, dtype=np.float64).T) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(vhat, dtype=np.float64)


def prefill_attend(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, scale: float) -> np.ndarray:
    """Causal multi-query attention of one KV head: q [Q, H, d] are the queries of the last Q of the
    T cached tokens (khat, vhat [T, d]); query j sits at position T - Q + j and attends the tokens
    t <= T - Q + j. Returns [Q, H, d] (fp64)."""
    q = np.asarray(q, dtype=np.float64)
    Qn, T = q.shape[0], np.asarray(khat).shape[0]
    out = np.empty(q.shape, dtype=np.float64)
    for j in range(Qn):
        n = T - Qn + j + 1
        out[j] = softmax_attend(q[j], khat[:n], vhat[:n], scale)
    return out


def decode_attention(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, scale: float) -> np.ndarray:
    """q [B, Hq, d]; khat, vhat [B, Hkv, T, d] -> out [B, Hq, d] (GQA: h -> h // (Hq/Hkv))."""
    B, Hq, d = q.shape
    Hkv = khat.shape[1]
    grp = Hq // Hkv
    out = np.empty((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hkv):
            out[b, h * grp:(h + 1) * grp] = softmax_attend(q[b, h * grp:(h + 1) * grp],
                                                           khat[b, h], vhat[b, h], scale)
    return out


def topk(score_rows: np.ndarray, k: int, ids: np.ndarray | None = None):
    """Per row: the k best (score, id) pairs sorted by (-score, id)."""
    s = np.asarray(score_rows, dtype=np.float64)
    Q, N = s.shape
    if ids is None:
        ids = np.arange(N, dtype=np.int64)
    out_i = np.empty((Q, k), dtype=np.int64)
    out_s = np.empty((Q, k), dtype=np.float64)
    for r in range(Q):
        order = np.lexsort((ids, -s[r]))[:k]
        out_i[r] = ids[order]
        out_s[r] = s[r, order]
    return out_i, out_s
