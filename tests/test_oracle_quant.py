"""Pins for the oracle's rotation inputs, packing, Algorithm 1/2 encode and decode (CPU only)."""
import math
import os

import numpy as np
import pytest

import workloads as W
from oracle import quant as Q
from oracle.codebook import distortion_per_vector, lloyd_max

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _figures():
    out = {}
    for line in open(os.path.join(GOLDEN, "pages_figures.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = float(v)
    return out


# ---- rotation (an input, but the method needs it orthogonal) ------------------------------------

@pytest.mark.parametrize("d", [32, 64, 128, 1536])
def test_rotation_is_orthogonal(d):
    Pi = W.rotation(d).astype(np.float64)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) < 1e-6
    x = W.gaussian(256, d).astype(np.float64)
    n0 = np.linalg.norm(x, axis=1)
    n1 = np.linalg.norm(x @ Pi.T, axis=1)
    assert np.max(np.abs(n1 / n0 - 1)) < 1e-6


def test_rotation_spreads_outliers():
    # the reason for the rotation (techblog-plum page, outlier example): energy concentrated in a
    # few channels is spread over all coordinates after Pi
    d = 128
    x = W.kv_slice(2048, d, 3, 20.0, 0.0, 0, W.TAG_K, 0, 0).astype(np.float64)
    peak_before = np.max(np.mean(x * x, axis=0)) / np.mean(x * x)
    y = x @ W.rotation(d).astype(np.float64).T
    peak_after = np.max(np.mean(y * y, axis=0)) / np.mean(y * y)
    assert peak_before > 30 and peak_after < 5


# ---- packing: brute force at d = 32 ------------------------------------------------------------

def _read_bit(buf: bytes, word_index: int, bit: int) -> int:
    # independent little-endian reader: word w occupies bytes 4w..4w+3
    return (buf[4 * word_index + bit // 8] >> (bit % 8)) & 1


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_every_coordinate_every_value(bits):
    d = 32
    for lane in range(d):
        for v in range(1 << bits):
            idx = np.zeros((1, d), dtype=np.int64)
            idx[0, lane] = v
            words = Q.pack_planes(idx, bits)
            assert words.shape == (1, 1, bits) and words.dtype == np.uint32
            buf = words.tobytes()
            for p in range(bits):
                for l in range(32):
                    want = (v >> p) & 1 if l == lane else 0
                    assert _read_bit(buf, p, l) == want
            assert np.array_equal(Q.unpack_planes(words, bits), idx)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_random_round_trip(bits):
    g = np.random.default_rng(5)
    idx = g.integers(0, 1 << bits, size=(64, 128))
    words = Q.pack_planes(idx, bits)
    assert np.array_equal(Q.unpack_planes(words, bits), idx)
    buf = words.tobytes()
    G = 128 // 32
    for v in range(0, 64, 7):
        for j in range(128):
            gidx, l = divmod(j, 32)
            val = sum(_read_bit(buf, (v * G + gidx) * bits + p, l) << p for p in range(bits))
            assert val == idx[v, j]


def test_sign_pack_round_trip():
    g = np.random.default_rng(6)
    z = g.random((17, 64)) < 0.5
    w = Q.pack_signs(z)
    assert np.array_equal(Q.unpack_signs(w), z)
    buf = w.tobytes()
    for v in range(17):
        for j in range(64):
            assert _read_bit(buf, v * 2 + j // 32, j % 32) == int(z[v, j])


def test_packed_size_accounting_matches_pages():
    # b bits per coordinate: the traeai page's 16-bit -> 3-bit cache figures and the
    # techblog-plum page's 5.3x / 8x ratios are exactly 16/b
    fig = _figures()
    d, bits = 64, 3
    assert Q.pack_planes(np.zeros((1, d), dtype=np.int64), bits).nbytes == bits * d // 8
    assert abs(fig["cache_mb_fp16"] * bits / 16 - fig["cache_mb_3bit"]) < 0.005
    assert round(16 / 3, 1) == fig["ratio_keys_3bit"] and 16 / 2 == fig["ratio_values_2bit"]


# ---- quantiser --------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_boundary_count_is_nearest_centroid(bits):
    cb = lloyd_max(128, bits)
    c = cb.c32.astype(np.float64)
    y = np.random.default_rng(1).standard_normal((4000,)) * 0.12
    idx = Q.quantise(y[None, :], cb)[0]
    near = np.argmin(np.abs(y[:, None] - c[None, :]), axis=1)
    assert np.array_equal(idx, near)
    # an exact tie at a boundary goes to the lower index
    t = cb.t32.astype(np.float64)
    assert np.array_equal(Q.quantise(t[None, :], cb)[0], np.arange(len(t)))


def test_zero_vector_convention():
    d, bits = 64, 3
    Pi, S = W.rotation(d), W.jl_matrix(d)
    cb = lloyd_max(d, bits - 1)
    x = np.zeros((2, d), dtype=np.float32)
    x[1] = W.gaussian(1, d)[0]
    e = Q.encode_prod(x, Pi, S, cb)
    L = 1 << (bits - 1)
    assert np.all(e["idx"][0] == L // 2 - 1)
    assert e["norms"][0] == 0 and e["gammas"][0] == 0
    assert np.all(e["signs"][0] == 0xFFFFFFFF)
    xh = Q.decode(e["codes"], e["norms"], Pi, cb, e["signs"], e["gammas"], S)
    assert np.all(xh[0] == 0)


def test_nonfinite_rows_policy():
    """A row with a NaN entry stores n = NaN, one with an infinite entry (no NaN) n = +Inf; both are
    otherwise the zero vector's record. Finite rows beside them are unaffected, and a finite row whose
    norm overflows fp16 keeps its codes with n = +Inf."""
    d, bits = 64, 3
    Pi, S = W.rotation(d), W.jl_matrix(d)
    cb = lloyd_max(d, bits - 1)
    x = W.gaussian(6, d)
    x[1, 5] = np.nan
    x[2, 7] = np.inf
    x[3, 0] = -np.inf
    x[3, 9] = np.nan                              # NaN wins over Inf
    x[4] *= np.float32(1e4)                       # |x| about 8e4 > 65504
    e = Q.encode_prod(x, Pi, S, cb)
    ref = Q.encode_prod(x[[0, 5]], Pi, S, cb)
    L = 1 << (bits - 1)
    assert np.isnan(e["norms"][1]) and np.isnan(e["norms"][3])
    assert e["norms"][2] == np.inf and e["norms"][4] == np.inf
    for r in (1, 2, 3):
        assert np.all(e["idx"][r] == L // 2 - 1)
        assert e["gammas"][r] == 0 and np.all(e["signs"][r] == 0xFFFFFFFF)
    fin = Q.encode_prod(x[4:5] / np.float32(1e4), Pi, S, cb)
    assert np.array_equal(e["codes"][4], fin["codes"][0])
    for k in ("codes", "signs", "norms", "gammas"):
        assert np.array_equal(e[k][[0, 5]], ref[k])
    xh = Q.decode(e["codes"], e["norms"], Pi, cb, e["signs"], e["gammas"], S)
    assert np.all(np.isnan(xh[1])) and np.all(~np.isfinite(xh[2])) and np.all(np.isfinite(xh[[0, 5]]))


def test_scale_invariance_of_codes():
    d = 128
    Pi = W.rotation(d)
    cb = lloyd_max(d, 3)
    x = W.gaussian(512, d)
    a = Q.encode_mse(x, Pi, cb)
    b = Q.encode_mse(x * np.float32(8.0), Pi, cb)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(b["norms"].astype(np.float64), a["norms"].astype(np.float64) * 8)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_empirical_mse_matches_exact_distortion(bits):
    # the tiny workload: 4096 N(0,1) vectors, d = 128, Algorithm 1 quantise + dequantise
    d = 128
    x = W.gaussian(4096, d)
    Pi = W.rotation(d)
    cb = lloyd_max(d, bits)
    e = Q.encode_mse(x, Pi, cb)
    # error of the unit vector, with the exact norm (the fp16 norm is a separate rounding)
    uh = Q.decode(e["codes"], np.ones(len(x), dtype=np.float16), Pi, cb)
    err = np.sum((e["u"] - uh) ** 2, axis=1)
    D = distortion_per_vector(cb)
    se = err.std(ddof=1) / math.sqrt(len(err))
    assert abs(err.mean() - D) < 3 * se + 1e-4 * D, (err.mean(), D, se)
    # and within the pages' factor of the 4^-b lower bound
    assert 4.0 ** -bits <= err.mean() * (1 + 3 * se / D) and err.mean() <= 2.7 * 4.0 ** -bits


def test_decode_is_inverse_rotation_of_centroids():
    d = 64
    Pi = W.rotation(d).astype(np.float64)
    cb = lloyd_max(d, 2)
    idx = np.random.default_rng(3).integers(0, 4, size=(5, d))
    codes = Q.pack_planes(idx, 2)
    n16 = np.array([1, 2, 0.5, 3, 7], dtype=np.float16)
    xh = Q.decode(codes, n16, Pi.astype(np.float32), cb)
    for v in range(5):
        want = np.zeros(d)
        for i in range(d):                    # Pi^T c = sum_i c_i * row i of Pi, as loops
            for j in range(d):
                want[j] += Pi[i, j] * float(cb.c32[idx[v, i]])
        assert np.allclose(xh[v], float(n16[v]) * want, rtol=1e-12, atol=1e-14)


# ---- QJL: unbiasedness of the inner-product estimate over draws of S -------------------------

def _qjl_bias(alpha_fn, M=20000, d=32, seed=9, p3_sketch=False):
    g = np.random.default_rng(seed)
    Pi = W.rotation(d, seed=4)
    cb = lloyd_max(d, 1)
    x = g.standard_normal((1, d)).astype(np.float32)
    e1 = Q.encode_mse(x, Pi, cb)
    chat = cb.c32.astype(np.float64)[e1["idx"]][0]
    r = e1["u"][0] - chat @ Pi.astype(np.float64)
    gam = np.linalg.norm(r)
    yv = r / gam                                         # probe along r: most sensitive to alpha
    base = chat @ Pi.astype(np.float64)
    vals = np.empty(M)
    for m in range(M):
        S = g.standard_normal((d, d))
        if p3_sketch:
            # the techblog-plum sketch: rotated-domain residual sign, fixed 0.5, no S
            rho = e1["y"][0] - chat
            xh = (chat + 0.5 * np.sign(rho)) @ Pi.astype(np.float64)
        else:
            sgn = np.where(S @ r >= 0, 1.0, -1.0)
            xh = base + alpha_fn(d) * gam * (sgn @ S)
        vals[m] = yv @ xh - yv @ e1["u"][0]
    return vals.mean(), vals.std(ddof=1) / math.sqrt(M)


def test_qjl_estimate_is_unbiased():
    # the oracle's own Algorithm 2 encode+decode, averaged over independent draws of S
    g = np.random.default_rng(11)
    d, M = 32, 4000
    Pi = W.rotation(d, seed=4)
    cb = lloyd_max(d, 1)
    x = g.standard_normal((1, d)).astype(np.float32)
    q = g.standard_normal(d)
    est = np.empty(M)
    for m in range(M):
        S = g.standard_normal((d, d)).astype(np.float32)
        e = Q.encode_prod(x, Pi, S, cb)
        xh = Q.decode(e["codes"], np.array([1.0], np.float16), Pi, cb, e["signs"],
                      e["gamma"].astype(np.float16), S)
        est[m] = q @ xh[0]
    truth = q @ e["u"][0]
    se = est.std(ddof=1) / math.sqrt(M)
    # gamma is stored in fp16: allow its relative rounding on top of 4 standard errors
    assert abs(est.mean() - truth) < 4 * se + 1e-3 * abs(truth) + 1e-12


def test_qjl_alpha_unbiased_and_alternatives_are_not():
    mean, se = _qjl_bias(Q.qjl_alpha)
    assert abs(mean) < 4 * se
    mean2, se2 = _qjl_bias(lambda d: 2 * Q.qjl_alpha(d))
    assert abs(mean2) > 8 * se2
    mean3, se3 = _qjl_bias(None, M=200, p3_sketch=True)
    assert abs(mean3) > 8 * max(se3, 1e-12)


def test_planted_alpha_mistake_is_caught(monkeypatch):
    # plant a wrong constant in the oracle itself; the unbiasedness check must notice
    monkeypatch.setattr(Q, "qjl_alpha", lambda d: math.sqrt(2 / math.pi) / d)
    mean, se = _qjl_bias(Q.qjl_alpha)
    assert abs(mean) > 8 * se


# ---- mixed widths per channel group ------------------------------------------------------------

def test_mixed_uniform_map_is_algorithm_1():
    """A map with one width everywhere is plain Algorithm 1: the same words, the same decode."""
    d = 128
    Pi = W.rotation(d)
    x = W.gaussian(300, d, seed=5)
    for b in (1, 2, 3, 4):
        cb = lloyd_max(d, b)
        e = Q.encode_mse(x, Pi, cb)
        m = Q.encode_mse_mixed(x, Pi, {b: cb}, [b] * (d // 32))
        assert np.array_equal(m["codes"], e["codes"].reshape(len(x), -1))
        assert np.array_equal(Q.decode_mixed(m["codes"], m["norms"], Pi, {b: cb}, [b] * (d // 32)),
                              Q.decode(e["codes"], e["norms"], Pi, cb))


def test_mixed_packing_bit_by_bit():
    """Brute force at d = 64 with widths (1, 4) and (4, 2): every index value at every coordinate
    round-trips, and an independent reader finds bit p of idx[32 g + l] at bit l of word
    sum_{g' < g} b_g' + p."""
    g = np.random.default_rng(8)
    for gb in ([1, 4], [4, 2], [3, 3]):
        idx = np.concatenate([g.integers(0, 1 << b, size=(40, 32)) for b in gb], axis=1)
        words = Q.pack_mixed(idx, gb)
        assert words.shape == (40, sum(gb))
        assert np.array_equal(Q.unpack_mixed(words, gb), idx)
        off = np.concatenate([[0], np.cumsum(gb)[:-1]])
        for v in range(0, 40, 7):
            for j in range(64):
                gg, lane = divmod(j, 32)
                for p in range(gb[gg]):
                    assert (int(words[v, off[gg] + p]) >> lane) & 1 == (int(idx[v, j]) >> p) & 1


@pytest.mark.parametrize("gb", [[3, 3, 2, 2], [4, 2, 2, 2], [1, 2, 3, 4]])
def test_mixed_distortion_is_the_group_average(gb):
    """After the rotation every coordinate has the law f_d, so the per-vector distortion of a mixed
    map is the group-weighted average sum_g (32/d) D_{b_g} of the uniform distortions; the empirical
    MSE on 4096 vectors matches it within 3 standard errors. A (3,3,2,2) map is a 2.5-bit code
    between the 2- and 3-bit ones."""
    d = 128
    x = W.gaussian(4096, d)
    Pi = W.rotation(d)
    cbs = {b: lloyd_max(d, b) for b in set(gb)}
    m = Q.encode_mse_mixed(x, Pi, cbs, gb)
    uh = Q.decode_mixed(m["codes"], np.ones(len(x), dtype=np.float16), Pi, cbs, gb)
    err = np.sum((m["u"] - uh) ** 2, axis=1)
    D = sum(32.0 / d * distortion_per_vector(cbs[b]) for b in gb)
    se = err.std(ddof=1) / math.sqrt(len(err))
    assert abs(err.mean() - D) < 3 * se + 1e-4 * D, (err.mean(), D, se)
    lo, hi = min(gb), max(gb)
    assert distortion_per_vector(lloyd_max(d, hi)) <= D <= distortion_per_vector(lloyd_max(d, lo))
    # record size: the planes of every group plus the fp16 norm
    assert m["codes"].shape[1] * 4 + 2 == 4 * sum(gb) + 2
