"""Lloyd-Max codebook for one coordinate of a randomly rotated unit vector (oracle).

Source: aiboss88 page, "TurboQuant technical principles" -- after a random
rotation every coordinate follows a Beta-shaped law and the optimal scalar
quantiser is found once with the Lloyd-Max algorithm (continuous 1-D k-means);
techblog-plum page, "step 1: PolarQuant" -- the buckets are precomputed once,
so there is no inference-time cost.

Density. For u uniform on the unit sphere of R^d, one coordinate X has
    f_d(x) = C_d (1 - x^2)^((d-3)/2),   C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)),
and X^2 ~ Beta(1/2, (d-1)/2), so for t >= 0
    P(0 <= X <= t) = I_{t^2}(1/2, (d-1)/2) / 2,
and the first moment over a cell has the closed form
    int_a^b x f_d(x) dx = C_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1).

Lloyd-Max. Alternate (i) boundaries = midpoints of neighbouring centroids and
(ii) centroids = conditional means of their cells, until the centroids stop
moving. The density is symmetric, so only the positive half is iterated and
mirrored (t_{L/2} = 0 exactly); it is log-concave for d >= 3, so the fixed
point is unique.

Parity pins (tests/test_oracle_codebook.py): b=1 closed form E|X|; centroid
condition by independent adaptive quadrature; the large-d limit against Max's
Gaussian table; distortion inside the pages' [1, 2.7] x 4^-b band and 1.45x at
b=1.
"""
from __future__ import annotations

import math

import functools

import mpmath
import numpy as np
from scipy import special


@functools.lru_cache(maxsize=None)
def _log_cd(d: int) -> float:
    """log C_d; the gamma ratio is taken in 40-digit arithmetic (fp64 lgamma differences lose
    about log10(d) digits to cancellation)."""
    with mpmath.workdps(40):
        r = mpmath.gamma(mpmath.mpf(d) / 2) / (mpmath.sqrt(mpmath.pi) * mpmath.gamma(mpmath.mpf(d - 1) / 2))
        return float(mpmath.log(r))


def density(x, d: int):
    """f_d(x) on [-1, 1]."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(divide="ignore"):
        return np.exp(_log_cd(d) + 0.5 * (d - 3) * np.log1p(-x * x))


def mass(a: float, b: float, d: int) -> float:
    """P(a <= X <= b) for 0 <= a <= b <= 1."""
    p = (d - 1) / 2.0
    if b >= 1.0:
        # upper tail through the complementary function to avoid cancellation
        return 0.5 * special.betaincc(0.5, p, a * a) if a > 0 else 0.5
    return 0.5 * (special.betainc(0.5, p, b * b) - special.betainc(0.5, p, a * a))


def first_moment(a: float, b: float, d: int) -> float:
    """int_a^b x f_d(x) dx for 0 <= a <= b <= 1 (closed form)."""
    e = (d - 1) / 2.0
    ua = math.exp(e * math.log1p(-a * a))
    ub = 0.0 if b >= 1.0 else math.exp(e * math.log1p(-b * b))
    return math.exp(_log_cd(d)) * (ua - ub) / (d - 1)


class Codebook:
    """c[0..L-1] ascending centroids, t[1..L-1] boundaries (t[k] between c[k-1] and c[k])."""

    def __init__(self, d: int, bits: int, c: np.ndarray, t: np.ndarray, iterations: int):
        self.d, self.bits = d, bits
        self.c = c            # fp64, length L
        self.t = t            # fp64, length L-1 (t[k-1] is the boundary between c[k-1] and c[k])
        self.iterations = iterations

    @property
    def c32(self) -> np.ndarray:
        return self.c.astype(np.float32)

    @property
    def t32(self) -> np.ndarray:
        return self.t.astype(np.float32)


def lloyd_max(d: int, bits: int, tol: float = 1e-14, max_iter: int = 200000) -> Codebook:
    """Lloyd-Max quantiser with L = 2^bits levels for f_d.

    Runs until no centroid moves by more than ``tol`` times the largest one, then keeps
    iterating while the step still shrinks (the fp64 iteration ends in a roundoff-level
    cycle of a few ulps), so the linear convergence does not leave a tol/(1-rate) error.
    """
    if d < 3 or not (1 <= bits <= 8):
        raise ValueError("need d >= 3 and 1 <= bits <= 8")
    L = 1 << bits
    H = L // 2
    # start: positive-half quantiles of the density
    sd = 1.0 / math.sqrt(d)
    cpos = np.array([sd * special.ndtri(0.5 + 0.5 * (k + 0.5) / H) for k in range(H)], dtype=np.float64)
    cpos = np.minimum(cpos, 0.999)
    it, converged, best, stale = 0, False, np.inf, 0
    for it in range(1, max_iter + 1):
        edges = np.concatenate([[0.0], 0.5 * (cpos[:-1] + cpos[1:]), [1.0]])
        new = np.empty_like(cpos)
        for k in range(H):
            m = mass(edges[k], edges[k + 1], d)
            new[k] = first_moment(edges[k], edges[k + 1], d) / m
        delta = np.max(np.abs(new - cpos))
        cpos = new
        converged = converged or delta <= tol * cpos[-1]
        if delta < best:
            best, stale = delta, 0
        else:
            stale += 1
        if converged and (stale >= 50 or delta == 0.0):
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    c = np.concatenate([-cpos[::-1], cpos])
    t = 0.5 * (c[:-1] + c[1:])
    t[H - 1] = 0.0
    return Codebook(d, bits, c, t, it)


def distortion_per_vector(cb: Codebook) -> float:
    """E||u - u_hat||^2 for the Lloyd-Max quantiser applied coordinate-wise to a rotated unit u.

    With centroids at the conditional means, E[(X - Q(X))^2] = E[X^2] - sum_k c_k^2 P_k and
    E[X^2] = 1/d, so the per-vector distortion is 1 - d * sum_k c_k^2 P_k.
    """
    d = cb.d
    edges = np.concatenate([[-1.0], cb.t, [1.0]])
    acc = 0.0
    for k in range(len(cb.c)):
        a, b = edges[k], edges[k + 1]
        if a >= 0:
            p = mass(a, b, d)
        elif b <= 0:
            p = mass(-b, -a, d)
        else:
            p = mass(0.0, -a, d) + mass(0.0, b, d)
        acc += cb.c[k] ** 2 * p
    return 1.0 - d * acc
