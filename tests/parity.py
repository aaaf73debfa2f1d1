"""Comparison rules between the CUDA path and the oracle (test helper, CPU side).

Rules (the accepted tolerances for this method's outputs):
* codes and packed bytes bit-exact, except coordinates whose rotated value lies within 1e-5 of a
  decision boundary on the standardised scale sqrt(d) * y (the coordinate law has standard
  deviation 1/sqrt(d)); such mismatches must also be fewer than 1e-4 of all coordinates, and the
  two indices must be neighbours.
* QJL sign bits bit-exact, except where |(S r)_j| / |r| < 1e-5 ((S r)_j / |r| is standard normal).
* fp16 norms / residual norms equal, or one ulp apart only when the exact value sits within
  2^-20 (relative) of the fp16 rounding midpoint between the two.
* dequantised vectors, scores and attention outputs within 1e-3 relative, normwise (per vector /
  per score row / per output vector).
"""
from __future__ import annotations

import numpy as np

from oracle import quant as Q

BAND = 1e-5
MAX_MISMATCH_FRACTION = 1e-4


def np_u32(t) -> np.ndarray:
    """torch int32 tensor (uint32 bit patterns) -> numpy uint32."""
    return t.detach().cpu().numpy().view(np.uint32)


def np_f16(t) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float16)


def check_codes(gpu_words: np.ndarray, ora_idx: np.ndarray, ora_y: np.ndarray, t32: np.ndarray, bits: int, d: int):
    """Band rule for quantiser indices. Returns a stats dict; raises AssertionError on violation."""
    gi = Q.unpack_planes(gpu_words.reshape(ora_idx.shape[0], d // 32, bits), bits)
    oi = ora_idx
    mism = gi != oi
    nm = int(mism.sum())
    total = oi.size
    t = t32.astype(np.float64)
    stats = dict(total=total, mismatches=nm)
    if nm:
        v, j = np.nonzero(mism)
        a, b = gi[v, j], oi[v, j]
        assert np.all(np.abs(a - b) == 1), "mismatched indices are not neighbours"
        k = np.minimum(a, b)                    # boundary t[k] separates levels k and k+1
        dist = np.sqrt(d) * np.abs(ora_y[v, j] - t[k])
        stats["max_band_distance"] = float(dist.max())
        assert np.all(dist < BAND), f"code mismatch outside the band: {dist.max():.3g}"
    assert nm <= MAX_MISMATCH_FRACTION * total, f"{nm} code mismatches of {total}"
    # in-band population (for the report)
    dmin = np.min(np.abs(ora_y[..., None] - t[None, None, :]), axis=-1) * np.sqrt(d) if len(t) else None
    stats["in_band"] = int((dmin < BAND).sum()) if dmin is not None else 0
    return stats


def check_signs(gpu_words: np.ndarray, ora_z: np.ndarray, ora_s: np.ndarray, ora_gamma: np.ndarray, d: int):
    gz = Q.unpack_signs(gpu_words.reshape(ora_z.shape[0], d // 32))
    mism = gz != ora_z
    nm = int(mism.sum())
    stats = dict(total=ora_z.size, mismatches=nm)
    if nm:
        v, j = np.nonzero(mism)
        rel = np.abs(ora_s[v, j]) / np.maximum(ora_gamma[v], 1e-300)
        stats["max_band_distance"] = float(rel.max())
        assert np.all(rel < BAND), f"sign mismatch outside the band: {rel.max():.3g}"
    assert nm <= MAX_MISMATCH_FRACTION * ora_z.size, f"{nm} sign mismatches"
    return stats


def check_fp16(gpu16: np.ndarray, exact: np.ndarray, name: str, mid_tol: float = 2.0 ** -20):
    """fp16 values: equal to RNE(exact) or one ulp away within mid_tol (relative) of a rounding midpoint."""
    g = np.asarray(gpu16, dtype=np.float16)
    o = np.asarray(exact, dtype=np.float64).astype(np.float16)
    diff = g.view(np.uint16).astype(np.int64) - o.view(np.uint16).astype(np.int64)
    bad = diff != 0
    nb = int(bad.sum())
    if nb:
        assert np.all(np.abs(diff[bad]) == 1), f"{name}: fp16 values more than one ulp apart"
        lo = np.minimum(g[bad].astype(np.float64), o[bad].astype(np.float64))
        hi = np.maximum(g[bad].astype(np.float64), o[bad].astype(np.float64))
        mid = 0.5 * (lo + hi)
        ex = np.asarray(exact, dtype=np.float64)[bad]
        rel = np.abs(ex - mid) / np.abs(ex)
        assert np.all(rel <= mid_tol), \
            f"{name}: off-by-one not at a midpoint ({int((rel > mid_tol).sum())} of {nb}, max rel {rel.max():.3g})"
    return dict(total=g.size, off_by_one=nb)


def normwise_rel(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    num = np.linalg.norm(got - want, axis=-1)
    den = np.linalg.norm(want, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)
