"""Pins for the oracle's Lloyd-Max codebook (CPU only).

Each check compares the oracle with something other than itself: a closed
form, an independent quadrature, a textbook table, the pages' printed bounds.
"""
import math
import os

import mpmath
import numpy as np
import pytest
from scipy import integrate, special

from oracle.codebook import density, distortion_per_vector, lloyd_max

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _figures():
    out = {}
    for line in open(os.path.join(GOLDEN, "pages_figures.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = float(v)
    return out


def _max_table():
    out = {}
    for line in open(os.path.join(GOLDEN, "max1960_gaussian_lloyd_max.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            b, vals = line.split(":")
            out[int(b)] = [float(v) for v in vals.split()]
    return out


@pytest.mark.parametrize("d", [3, 4, 64, 128, 1536])
def test_one_bit_is_mean_absolute_coordinate(d):
    # b = 1: the only positive cell is (0, 1], so c = E|X| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).
    cb = lloyd_max(d, 1)
    with mpmath.workdps(40):
        exact = float(mpmath.gamma(mpmath.mpf(d) / 2)
                      / (mpmath.sqrt(mpmath.pi) * mpmath.gamma(mpmath.mpf(d + 1) / 2)))
    assert abs(cb.c[1] - exact) <= 1e-13 * exact
    assert cb.c[0] == -cb.c[1] and cb.t[0] == 0.0


def test_one_bit_large_d_limit():
    # c_1 -> sqrt(2/(pi d)); Gamma(z)/Gamma(z+1/2) = z^(-1/2) (1 + 1/(8z) + O(z^-2)) gives the
    # ratio 1 + 1/(4d) + O(1/d^2).
    for d in (128, 1536, 100000):
        r = lloyd_max(d, 1).c[1] / math.sqrt(2 / (math.pi * d))
        assert abs(r - (1 + 1 / (4 * d))) < 2.0 / d ** 2


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_is_uniform_quantiser(bits):
    # d = 3: f_3 is uniform on [-1, 1] (Archimedes), whose Lloyd-Max quantiser is the uniform one.
    cb = lloyd_max(3, bits)
    L = 1 << bits
    want = -1 + (2 * np.arange(L) + 1) / L
    assert np.max(np.abs(cb.c - want)) < 1e-13
    # and its distortion meets the lower bound exactly: 4^-b
    assert abs(distortion_per_vector(cb) - 4.0 ** -bits) < 1e-13


@pytest.mark.parametrize("d", [64, 128, 1536])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_and_midpoint_conditions(d, bits):
    cb = lloyd_max(d, bits)
    L = 1 << bits
    # midpoint condition and symmetry
    assert np.allclose(cb.t, 0.5 * (cb.c[:-1] + cb.c[1:]), rtol=0, atol=1e-17)
    assert np.array_equal(cb.c[::-1], -cb.c)
    assert np.all(np.diff(cb.c) > 0)
    # centroid condition by adaptive quadrature of the density itself (not the closed forms)
    edges = np.concatenate([[-1.0], cb.t, [1.0]])
    cut = min(1.0, 60.0 / math.sqrt(d))        # density below 1e-300 beyond 60 sigma
    for k in range(L // 2, L):
        a, b = edges[k], min(edges[k + 1], cut)
        pts = np.linspace(a, b, 9)[1:-1]
        num = integrate.quad(lambda x: x * density(x, d), a, b, epsabs=0, epsrel=2e-14, limit=400,
                             points=pts)[0]
        den = integrate.quad(lambda x: density(x, d), a, b, epsabs=0, epsrel=2e-14, limit=400,
                             points=pts)[0]
        assert abs(num / den - cb.c[k]) <= 1e-12 * abs(cb.c[k]), (d, bits, k)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_large_d_limit_matches_max_gaussian_table(bits):
    levels = _max_table()[bits]
    d = 1_000_000
    cb = lloyd_max(d, bits)
    got = cb.c[len(cb.c) // 2:] * math.sqrt(d)
    for g, w in zip(got, levels):
        assert abs(g - w) <= 6e-4 * max(1.0, abs(w)), (bits, got, levels)


@pytest.mark.parametrize("d", [64, 128, 1536])
def test_distortion_within_pages_band(d):
    fig = _figures()
    for bits in (1, 2, 3, 4):
        ratio = distortion_per_vector(lloyd_max(d, bits)) * 4.0 ** bits
        assert 1.0 <= ratio <= fig["distortion_factor_max"], (d, bits, ratio)
    # 1 bit: 1.45x the lower bound (to the page's two decimals); limit is 4 (1 - 2/pi)
    r1 = distortion_per_vector(lloyd_max(d, 1)) * 4.0
    assert abs(r1 - fig["distortion_factor_1bit"]) < 0.02
    assert abs(4 * (1 - 2 / math.pi) - fig["distortion_factor_1bit"]) < 0.005


def test_distortion_values_d128():
    # exact distortion 1 - d sum c_k^2 P_k cross-checked against a direct quadrature of
    # d * E[(X - Q(X))^2] (no use of the centroid condition)
    d = 128
    for bits in (1, 2, 3, 4):
        cb = lloyd_max(d, bits)
        edges = np.concatenate([[-1.0], cb.t, [1.0]])
        tot = 0.0
        for k in range(len(cb.c)):
            a, b = max(edges[k], -0.8), min(edges[k + 1], 0.8)
            tot += integrate.quad(lambda x: (x - cb.c[k]) ** 2 * density(x, d), a, b,
                                  epsabs=0, epsrel=1e-13, limit=200)[0]
        assert abs(d * tot - distortion_per_vector(cb)) < 1e-11
