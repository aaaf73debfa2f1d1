"""TurboQuant Algorithm 1 / Algorithm 2 encode, bit packing and decode (oracle, fp64).

Sources (page titles as listed in the oracle package docstring):

* ai-navigate-news page, "how it works (technical)": Algorithm 1 = random
  rotation -> Lloyd-Max scalar quantisation of the Beta-distributed coordinates
  -> inverse rotation, MSE-optimal. Algorithm 2 = Algorithm 1 at b-1 bits, then
  the residual r is encoded as sign(S r); inner products are unbiased.
  Same page, bit-packing paragraph: indices and signs packed into bytes, norms
  and residual norms ("gammas") kept as float16.
* aiboss88 page, "technical principles" / "two-stage residual correction":
  rotate, quantise each coordinate independently with a precomputed codebook,
  then a 1-bit quantised Johnson-Lindenstrauss transform of the residual
  removes the inner-product bias.

Readings where the pages are silent (each also listed in the design notes):

* Norms: the method is stated for unit vectors; x is normalised by n = ||x||,
  n is stored as fp16 (round to nearest even) and u = x / n (fp64 n) is encoded.
* The residual is taken in the original domain, r = u - Pi^T c[idx]
  (= Pi^T (y - c[idx]) for orthogonal Pi); S multiplies r ("sign(S r)").
  The techblog-plum page's conceptual sketch (residual in the rotated domain,
  no S, fixed 0.5 * sign on decode) is not followed.
* QJL scale: for a row s ~ N(0, I_d), E[s sign(<s, r>)] = sqrt(2/pi) r / ||r||,
  hence E[S^T sign(S r)] = d sqrt(2/pi) r / ||r|| and the unbiased decode is
  x_hat = n (Pi^T c[idx] + alpha * gamma * S^T (2z - 1)), alpha = sqrt(pi/2) / d,
  gamma = ||r||.
* Ties: idx_j = #{k : t_k < y_j} (an exact tie goes to the lower index); the
  QJL bit is z_j = [ (S r)_j >= 0 ] (sign(0) -> +1).
* Zero vector: n = 0 gives u = 0, y = 0, idx_j = L/2 - 1; for Algorithm 2 the
  residual is taken as 0 (gamma = 0, all sign bits 1). Decode returns 0.
* Non-finite input (the pages are silent; a policy of this library): a row with
  a NaN entry stores n = NaN, a row with an infinite entry and no NaN stores
  n = +Inf (the IEEE sum of squares), and either row is otherwise encoded as the
  zero vector (idx_j = L/2 - 1; gamma = 0 and all sign bits 1). Decode then
  returns non-finite values for it. A finite row whose norm exceeds the fp16
  range stores n = +Inf (round to nearest) with its ordinary codes.
* Packed layout (bit planes, one 32-bit word per 32 coordinates and plane):
  bit l of codes[v][g][p] is bit p of idx[v][32 g + l]; bit l of signs[v][g]
  is z[v][32 g + l]. Words are little-endian uint32.

The fp32 codebook (centroids c and boundaries t rounded to fp32) is what the
packed format means; the oracle quantises with those fp32 values upcast to fp64.
"""
from __future__ import annotations

import math

import numpy as np

from .codebook import Codebook


def qjl_alpha(d: int) -> float:
    """Scale of the QJL term: alpha = sqrt(pi/2) / d (derived, see module docstring)."""
    return math.sqrt(math.pi / 2.0) / d


# ---- packing ----------------------------------------------------------------------------------

def pack_planes(idx: np.ndarray, bits: int) -> np.ndarray:
    """idx [N, d] (ints in [0, 2^bits)) -> uint32 [N, d/32, bits] bit-plane words."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    assert d % 32 == 0
    g = idx.reshape(n, d // 32, 32)
    out = np.zeros((n, d // 32, bits), dtype=np.uint64)
    lane = np.arange(32, dtype=np.uint64)
    for p in range(bits):
        bitp = ((g >> p) & 1).astype(np.uint64)
        out[:, :, p] = np.sum(bitp << lane, axis=2)
    return out.astype(np.uint32)


def unpack_planes(words: np.ndarray, bits: int) -> np.ndarray:
    """uint32 [N, d/32, bits] -> idx [N, d] int64."""
    w = np.asarray(words, dtype=np.uint64)
    n, G, b = w.shape
    assert b == bits
    lane = np.arange(32, dtype=np.uint64)
    idx = np.zeros((n, G, 32), dtype=np.int64)
    for p in range(bits):
        idx |= (((w[:, :, p, None] >> lane) & 1).astype(np.int64) << p)
    return idx.reshape(n, G * 32)


def pack_signs(z: np.ndarray) -> np.ndarray:
    """z [N, d] bool -> uint32 [N, d/32]; bit l of word g is z[32 g + l]."""
    z = np.asarray(z, dtype=np.uint64)
    n, d = z.shape
    lane = np.arange(32, dtype=np.uint64)
    return np.sum(z.reshape(n, d // 32, 32) << lane, axis=2).astype(np.uint32)


def unpack_signs(words: np.ndarray) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint64)
    n, G = w.shape
    lane = np.arange(32, dtype=np.uint64)
    return (((w[:, :, None] >> lane) & 1) != 0).reshape(n, G * 32)


# ---- encode -----------------------------------------------------------------------------------

def normalise(x: np.ndarray):
    """n = ||x|| (fp64), fp16 copy of n (RNE), u = x / n; u = 0 for the zero vector and for a row
    with a non-finite entry (whose n is then NaN, or +Inf when no entry is NaN)."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        n = np.sqrt(np.sum(x * x, axis=1))
    ok = np.isfinite(n) & (n > 0)
    safe = np.where(ok, n, 1.0)
    with np.errstate(invalid="ignore", over="ignore"):
        u = np.where(ok[:, None], x / safe[:, None], 0.0)
        n16 = n.astype(np.float16)                       # above the fp16 range: +Inf
    return n, n16, u


def rotate(u: np.ndarray, Pi: np.ndarray) -> np.ndarray:
    """y = Pi u for each row u (Pi taken as its fp32 values, upcast)."""
    return u @ np.asarray(Pi, dtype=np.float64).T


def quantise(y: np.ndarray, cb: Codebook) -> np.ndarray:
    """idx_j = #{k : t_k < y_j} with the fp32 boundaries (upcast)."""
    t = cb.t32.astype(np.float64)
    return np.searchsorted(t, y, side="left").astype(np.int64)


def encode_mse(x: np.ndarray, Pi: np.ndarray, cb: Codebook) -> dict:
    """Algorithm 1. Returns codes [N, d/32, b] uint32, norms fp16 and the fp64 intermediates."""
    n, n16, u = normalise(x)
    y = rotate(u, Pi)
    idx = quantise(y, cb)
    return dict(codes=pack_planes(idx, cb.bits), norms=n16, n=n, u=u, y=y, idx=idx)


def residual_signs(u: np.ndarray, idx: np.ndarray, n: np.ndarray, Pi: np.ndarray, S: np.ndarray,
                   cb_bm1: Codebook) -> dict:
    """Second stage of Algorithm 2 for given first-stage indices: r = u - Pi^T c[idx],
    gamma = |r|, s = S r, z = [s >= 0] (zero vectors: r = 0)."""
    c = cb_bm1.c32.astype(np.float64)
    chat = c[idx]                                        # rotated-domain reconstruction
    Pi64 = np.asarray(Pi, dtype=np.float64)
    r = u - chat @ Pi64                                  # u - Pi^T c[idx], original domain
    nn = np.asarray(n)
    r[~(np.isfinite(nn) & (nn > 0))] = 0.0               # zero and non-finite rows: no residual
    gamma = np.sqrt(np.sum(r * r, axis=1))
    s = r @ np.asarray(S, dtype=np.float64).T            # S r
    z = s >= 0
    return dict(signs=pack_signs(z), gammas=gamma.astype(np.float16), gamma=gamma, r=r, s=s, z=z, chat=chat)


def encode_prod(x: np.ndarray, Pi: np.ndarray, S: np.ndarray, cb_bm1: Codebook) -> dict:
    """Algorithm 2 at b bits = Algorithm 1 at b-1 bits (``cb_bm1``) + QJL sign of S r.

    Returns codes [N, d/32, b-1], signs [N, d/32], norms fp16, gammas fp16 and intermediates.
    """
    e = encode_mse(x, Pi, cb_bm1)
    e.update(residual_signs(e["u"], e["idx"], e["n"], Pi, S, cb_bm1))
    return e


# ---- mixed widths per channel group ----------------------------------------------------------
# Reading (the scope table's "mixed / fractional bit widths per channel group"; the pages' only
# fractional figure, techblog-plum's "average 2.5 bit", is keys at 3 bits and values at 2): the d
# rotated coordinates form d/32 groups of 32 (the packing groups), and group g is quantised with
# the b_g-bit Lloyd-Max codebook of the same coordinate law f_d (after the rotation every coordinate
# has that law, so each group's own codebook is optimal for it). The record holds, group by group,
# that group's b_g bit-plane words, then the fp16 norm: 4 sum_g b_g + 2 bytes. Algorithm 1 only.

def pack_mixed(idx: np.ndarray, group_bits) -> np.ndarray:
    """idx [N, d] -> uint32 [N, sum(group_bits)]: group g's planes (pack_planes of its 32 columns)."""
    idx = np.asarray(idx, dtype=np.int64)
    parts = [pack_planes(idx[:, 32 * g:32 * g + 32], b).reshape(idx.shape[0], b) for g, b in enumerate(group_bits)]
    return np.concatenate(parts, axis=1)


def unpack_mixed(words: np.ndarray, group_bits) -> np.ndarray:
    """uint32 [N, sum(group_bits)] -> idx [N, 32 len(group_bits)]."""
    w = np.asarray(words, dtype=np.uint32)
    out, o = [], 0
    for b in group_bits:
        out.append(unpack_planes(w[:, o:o + b].reshape(w.shape[0], 1, b), b))
        o += b
    return np.concatenate(out, axis=1)


def encode_mse_mixed(x: np.ndarray, Pi: np.ndarray, cbs: dict, group_bits) -> dict:
    """Algorithm 1 with a bit width per group of 32 rotated coordinates (cbs: bits -> codebook)."""
    n, n16, u = normalise(x)
    y = rotate(u, Pi)
    idx = np.empty(y.shape, dtype=np.int64)
    for g, b in enumerate(group_bits):
        idx[:, 32 * g:32 * g + 32] = quantise(y[:, 32 * g:32 * g + 32], cbs[b])
    return dict(codes=pack_mixed(idx, group_bits), norms=n16, n=n, u=u, y=y, idx=idx)


def decode_mixed(codes: np.ndarray, norms16: np.ndarray, Pi: np.ndarray, cbs: dict, group_bits) -> np.ndarray:
    """x_hat = n Pi^T c_g[idx] with each group's own codebook."""
    idx = unpack_mixed(codes, group_bits)
    chat = np.empty(idx.shape, dtype=np.float64)
    for g, b in enumerate(group_bits):
        chat[:, 32 * g:32 * g + 32] = cbs[b].c32.astype(np.float64)[idx[:, 32 * g:32 * g + 32]]
    return np.asarray(norms16, dtype=np.float64)[:, None] * (chat @ np.asarray(Pi, dtype=np.float64))


# ---- decode -----------------------------------------------------------------------------------

def decode(codes: np.ndarray, norms16: np.ndarray, Pi: np.ndarray, cb: Codebook,
           signs: np.ndarray | None = None, gammas16: np.ndarray | None = None,
           S: np.ndarray | None = None) -> np.ndarray:
    """x_hat = n (Pi^T c[idx] + alpha gamma S^T (2z - 1)), the last term for Algorithm 2 only.

    ``cb`` is the codebook the codes were made with (b-1 bits for Algorithm 2); n and gamma are
    the stored fp16 values.
    """
    idx = unpack_planes(codes, cb.bits)
    c = cb.c32.astype(np.float64)
    Pi64 = np.asarray(Pi, dtype=np.float64)
    xh = c[idx] @ Pi64                                   # rows: Pi^T c[idx]
    if signs is not None:
        d = idx.shape[1]
        sgn = np.where(unpack_signs(signs), 1.0, -1.0)
        g = np.asarray(gammas16, dtype=np.float64)
        xh = xh + qjl_alpha(d) * g[:, None] * (sgn @ np.asarray(S, dtype=np.float64))
    return np.asarray(norms16, dtype=np.float64)[:, None] * xh
