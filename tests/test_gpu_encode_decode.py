"""GPU parity of tq_encode_mse / tq_encode_prod / tq_decode against the oracle (B200).

Workloads: the tiny correctness set (4096 x 128 fp32, b = 1..4), the TinyLlama-shaped KV block
(32 heads x 4096 tokens x d = 64 bf16 with 4 outlier channels per head), the Llama-8B-shaped cache
(8 x 32768 x 128 bf16, 2% outlier channels, log-normal token norms), and ragged / edge cases.
All at full size: the oracle encodes a few hundred thousand vectors in seconds.
"""
import numpy as np
import pytest

import workloads as W
from oracle import quant as Q
from oracle.codebook import lloyd_max
from parity import check_codes, check_fp16, check_signs, normwise_rel, np_f16, np_u32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
tq = pytest.importorskip("kv_cache_vector_encode_b200")


@pytest.fixture(scope="module")
def dev(gpu_required):
    tq.lib()
    return torch.device("cuda")


_rot_cache = {}


def rotation(d, dev):
    if d not in _rot_cache:
        Pi, S = W.rotation(d), W.jl_matrix(d)
        rot = tq.tq_rotation_prepare(torch.from_numpy(Pi).to(dev), torch.from_numpy(S).to(dev))
        _rot_cache[d] = (Pi, S, rot)
    return _rot_cache[d]


def to_dev(x, dtype, dev):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(dtype)


def run_mse(x, d, bits, dtype, dev):
    Pi, S, rot = rotation(d, dev)
    cb = tq.tq_codebook_init(d, bits)
    xd = to_dev(x, dtype, dev)
    codes, norms = tq.empty_mse(len(x), d, bits)
    tq.tq_encode_mse(cb, xd, rot, codes, norms)
    tq.tq_sync_check()
    return cb, codes, norms


def run_prod(x, d, bits, dtype, dev):
    Pi, S, rot = rotation(d, dev)
    cb = tq.tq_codebook_init(d, bits - 1)
    xd = to_dev(x, dtype, dev)
    codes, signs, norms, gammas = tq.empty_prod(len(x), d, bits)
    tq.tq_encode_prod(cb, xd, rot, codes, signs, norms, gammas)
    tq.tq_sync_check()
    return cb, codes, signs, norms, gammas


def check_mse(x, d, bits, dtype, dev, decode=True):
    Pi, S, rot = rotation(d, dev)
    cb, codes, norms = run_mse(x, d, bits, dtype, dev)
    ora_cb = lloyd_max(d, bits)
    ora = Q.encode_mse(x, Pi, ora_cb)
    st = check_codes(np_u32(codes), ora["idx"], ora["y"], ora_cb.t32, bits, d)
    check_fp16(np_f16(norms), ora["n"], "norms")
    if decode:
        out = torch.empty((len(x), d), dtype=torch.float32, device=dev)
        tq.tq_decode(cb, rot, codes, norms, out)
        tq.tq_sync_check()
        want = Q.decode(np_u32(codes).reshape(len(x), d // 32, bits), np_f16(norms), Pi, ora_cb)
        rel = normwise_rel(out.cpu().numpy(), want)
        assert rel.max() <= 1e-3, rel.max()
        st["decode_max_rel"] = float(rel.max())
    return st


def check_prod(x, d, bits, dtype, dev, decode=True):
    Pi, S, rot = rotation(d, dev)
    cb, codes, signs, norms, gammas = run_prod(x, d, bits, dtype, dev)
    ora_cb = lloyd_max(d, bits - 1)
    ora = Q.encode_prod(x, Pi, S, ora_cb)
    st = check_codes(np_u32(codes), ora["idx"], ora["y"], ora_cb.t32, bits - 1, d)
    # An index within the band may legitimately land on the other side of its boundary; the
    # second stage then sees a residual coordinate of the same size and opposite sign, so the
    # signs are compared with the oracle's second stage run on the GPU's (checked) indices.
    gidx = Q.unpack_planes(np_u32(codes).reshape(len(x), d // 32, bits - 1), bits - 1)
    st["vectors_with_band_flips"] = int(np.any(gidx != ora["idx"], axis=1).sum())
    ora2 = Q.residual_signs(ora["u"], gidx, ora["n"], Pi, S, ora_cb)
    st["signs"] = check_signs(np_u32(signs), ora2["z"], ora2["s"], ora2["gamma"], d)
    check_fp16(np_f16(norms), ora["n"], "norms")
    check_fp16(np_f16(gammas), ora2["gamma"], "gammas")
    if decode:
        out = torch.empty((len(x), d), dtype=torch.float32, device=dev)
        tq.tq_decode(cb, rot, codes, norms, out, signs=signs, gammas=gammas)
        tq.tq_sync_check()
        want = Q.decode(np_u32(codes).reshape(len(x), d // 32, bits - 1), np_f16(norms), Pi, ora_cb,
                        np_u32(signs).reshape(len(x), d // 32), np_f16(gammas), S)
        rel = normwise_rel(out.cpu().numpy(), want)
        assert rel.max() <= 1e-3, rel.max()
        st["decode_max_rel"] = float(rel.max())
    return st


# ---- the workloads ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_tiny_fp32_mse(dev, bits):
    x = W.gaussian(4096, 128)
    st = check_mse(x, 128, bits, torch.float32, dev)
    print("tiny", bits, st)


def test_tinyllama_block(dev):
    c = W.WORKLOADS["tinyllama_block"]
    K = W.kv_block(c["heads"], c["tokens"], c["d"], c["n_outlier"], c["outlier_scale"], 0.0, tag=W.TAG_K)
    V = W.kv_block(c["heads"], c["tokens"], c["d"], c["n_outlier"], c["outlier_scale"], 0.0, tag=W.TAG_V)
    d = c["d"]
    print("K", check_mse(K.reshape(-1, d), d, c["k_bits"], torch.bfloat16, dev))
    print("V", check_prod(V.reshape(-1, d), d, c["v_bits"], torch.bfloat16, dev))


def test_llama8b_cache(dev):
    c = W.WORKLOADS["llama8b_cache"]
    d = c["d"]
    K = W.kv_block(c["heads"], c["tokens"], d, c["n_outlier"], c["outlier_scale"], c["lognormal_sigma"],
                   tag=W.TAG_K).reshape(-1, d)
    V = W.kv_block(c["heads"], c["tokens"], d, c["n_outlier"], c["outlier_scale"], c["lognormal_sigma"],
                   tag=W.TAG_V).reshape(-1, d)
    print("K", check_mse(K, d, c["k_bits"], torch.bfloat16, dev))
    print("V", check_prod(V, d, c["v_bits"], torch.bfloat16, dev))


# ---- edge cases ------------------------------------------------------------------------------

@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("n", [1, 127, 129, 1000])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_sizes(dev, d, n, dtype):
    g = np.random.default_rng(d * 1000 + n)
    x = W.round_to_bf16(g.standard_normal((n, d)).astype(np.float32) * 3.0)
    if n > 5:
        x[3] = 0.0                      # a zero vector inside a tile
        x[n - 1] = 0.0                  # and at the ragged end
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for bits in (1, 3, 4):
        check_mse(x, d, bits, dt, dev)
    for bits in (2, 4):
        check_prod(x, d, bits, dt, dev)


def test_zero_vectors_follow_convention(dev):
    d = 128
    x = np.zeros((70, d), dtype=np.float32)
    cb, codes, signs, norms, gammas = run_prod(x, d, 3, torch.bfloat16, dev)
    idx = Q.unpack_planes(np_u32(codes).reshape(70, 4, 2), 2)
    assert np.all(idx == 1)                           # L/2 - 1 with L = 4
    assert np.all(np_u32(signs) == 0xFFFFFFFF)
    assert np.all(np_f16(norms) == 0) and np.all(np_f16(gammas) == 0)


def test_extreme_magnitudes(dev):
    # the per-vector power-of-two scaling keeps fp16 operands exact for tiny and huge bf16 vectors
    d = 128
    g = np.random.default_rng(7)
    x = W.round_to_bf16(g.standard_normal((256, d)).astype(np.float32))
    x[:64] *= np.float32(1e-30)
    x[64:128] *= np.float32(1e30)
    x = W.round_to_bf16(x)
    check_mse(x, d, 3, torch.bfloat16, dev, decode=False)
    check_prod(x, d, 3, torch.bfloat16, dev, decode=False)


@pytest.mark.parametrize("alg2", [False, True])
def test_bf16_decode_output(dev, alg2):
    # bf16 output against the oracle's fp64 decode of the same codes: normwise within 1e-3 + 2^-8
    # (the bf16 rounding adds up to 2^-9 per element), and element by element within one bf16
    # rounding (2^-8 relative) plus the fp32 path's 1e-5 of the row norm -- a misplaced element or a
    # wrong row stride fails the second check
    d = 128
    x = W.gaussian(2048, d)
    Pi, S, rot = rotation(d, dev)
    out16 = torch.empty((len(x), d), dtype=torch.bfloat16, device=dev)
    if alg2:
        cb, codes, signs, norms, gammas = run_prod(x, d, 3, torch.float32, dev)
        tq.tq_decode(cb, rot, codes, norms, out16, signs=signs, gammas=gammas)
        want = Q.decode(np_u32(codes).reshape(len(x), d // 32, 2), np_f16(norms), Pi, lloyd_max(d, 2),
                        np_u32(signs).reshape(len(x), d // 32), np_f16(gammas), S)
    else:
        cb, codes, norms = run_mse(x, d, 3, torch.float32, dev)
        tq.tq_decode(cb, rot, codes, norms, out16)
        want = Q.decode(np_u32(codes).reshape(len(x), d // 32, 3), np_f16(norms), Pi, lloyd_max(d, 3))
    tq.tq_sync_check()
    got = out16.float().cpu().numpy()
    rel = normwise_rel(got, want)
    assert rel.max() <= 1e-3 + 2.0 ** -8
    row = np.linalg.norm(want, axis=1, keepdims=True)
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-5 * row)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_nonfinite_rows(dev, d, dtype):
    # The library's policy for non-finite input (the pages are silent): a row with a NaN entry stores
    # n = NaN, a row with an infinite entry and no NaN stores n = +Inf, and both are otherwise the zero
    # vector's record (idx = L/2 - 1; gamma = 0, all sign bits 1). Rows beside them are unaffected;
    # a finite row whose norm overflows fp16 keeps its codes with n = +Inf. d = 128 runs the fused
    # encoder, d = 256 the tiled one.
    g = np.random.default_rng(11 + d)
    n = 300
    x = g.standard_normal((n, d)).astype(np.float32)
    big = [17, 150]
    x[big] *= np.float32(1e4)
    x = W.round_to_bf16(x)                              # the same values on both sides for bf16 input
    bad_nan, bad_inf = [3, 64, 200, 299], [5, 130, 201]
    for r in bad_nan:
        x[r, (7 * r) % d] = np.nan
    for r in bad_inf:
        x[r, (3 * r) % d] = np.inf if r % 2 else -np.inf
    x[201, 0] = np.nan                                  # NaN and Inf in one row: NaN
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Pi, S, rot = rotation(d, dev)
    bad = sorted(set(bad_nan + bad_inf))
    good = [r for r in range(n) if r not in bad]
    for alg2, bits in ((False, 3), (True, 3)):
        if alg2:
            cb, codes, signs, norms, gammas = run_prod(x, d, bits, dt, dev)
            cbits = bits - 1
            ora = Q.encode_prod(x, Pi, S, lloyd_max(d, cbits))
        else:
            cb, codes, norms = run_mse(x, d, bits, dt, dev)
            cbits = bits
            ora = Q.encode_mse(x, Pi, lloyd_max(d, cbits))
        gn = np_f16(norms)
        assert np.array_equal(np.isnan(gn), np.isnan(ora["norms"]))
        assert np.array_equal(np.isposinf(gn), np.isposinf(ora["norms"]))
        gw = np_u32(codes).reshape(n, d // 32, cbits)
        assert np.array_equal(gw[bad], ora["codes"][bad])          # the zero vector's codes, exactly
        check_codes(gw[good], ora["idx"][good], ora["y"][good], lloyd_max(d, cbits).t32, cbits, d)
        fin = [r for r in good if r not in big]
        check_fp16(gn[fin], ora["n"][fin], "norms")
        if alg2:
            assert np.all(np_u32(signs).reshape(n, d // 32)[bad] == 0xFFFFFFFF)
            assert np.all(np_f16(gammas)[bad] == 0)


def test_repeat_runs_identical(dev):
    d = 128
    x = W.gaussian(5000, d)
    a = run_prod(x, d, 3, torch.float32, dev)
    b = run_prod(x, d, 3, torch.float32, dev)
    for ta, tb in zip(a[1:], b[1:]):
        assert torch.equal(ta, tb)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("alg2,bits", [(False, 1), (False, 2), (False, 3), (False, 4), (True, 2), (True, 3),
                                       (True, 4), (True, 5)])
def test_decode_precision(dev, d, alg2, bits):
    # Decode from the codes alone, against the oracle's fp64 decode of the same codes. The fp16
    # hi/lo split of the codebook and of Pi^T / S^T carries about 22 significant bits and the
    # products accumulate in fp32, so the normwise error stays near 1e-6. A lost low part (2^-12)
    # or a misplaced level would show here.
    n = 700
    g = np.random.default_rng(100 * d + 10 * bits + alg2)
    cbits = bits - 1 if alg2 else bits
    codes_np = g.integers(0, 2 ** 32, size=(n, d // 32, cbits), dtype=np.uint64).astype(np.uint32)
    norms_np = W.round_to_bf16(np.abs(g.standard_normal(n)).astype(np.float32) + 0.1).astype(np.float16)
    Pi, S, rot = rotation(d, dev)
    cb = tq.tq_codebook_init(d, cbits)
    ocb = lloyd_max(d, cbits)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    codes = t(codes_np, np.int32)
    norms = t(norms_np, np.int16).view(torch.float16)
    out = torch.empty((n, d), dtype=torch.float32, device=dev)
    if alg2:
        signs_np = g.integers(0, 2 ** 32, size=(n, d // 32), dtype=np.uint64).astype(np.uint32)
        gam_np = (np.abs(g.standard_normal(n)) * 0.3).astype(np.float16)
        tq.tq_decode(cb, rot, codes, norms, out, signs=t(signs_np, np.int32),
                     gammas=t(gam_np, np.int16).view(torch.float16))
        want = Q.decode(codes_np, norms_np, Pi, ocb, signs_np, gam_np, S)
    else:
        tq.tq_decode(cb, rot, codes, norms, out)
        want = Q.decode(codes_np, norms_np, Pi, ocb)
    tq.tq_sync_check()
    rel = normwise_rel(out.cpu().numpy(), want)
    print("decode precision", d, alg2, bits, rel.max())
    assert rel.max() <= 1e-5, rel.max()
