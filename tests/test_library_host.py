"""libtq on the host (no GPU needed): the shared library loads, exports every symbol the header
declares, computes the same codebook as the oracle, and rejects bad arguments before touching a
device."""
import ctypes
import os
import re

import numpy as np
import pytest

import kv_cache_vector_encode_b200 as tq
from oracle.codebook import distortion_per_vector, lloyd_max

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from kv_cache_vector_encode_b200 import build
    build.build()
    return tq.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert tq.tq_version().startswith("libtq")


@pytest.mark.parametrize("d,bits", [(64, 1), (64, 2), (64, 3), (128, 1), (128, 2), (128, 3), (128, 4),
                                    (1536, 3), (1536, 4), (3, 2), (4, 3)])
def test_codebook_matches_oracle(L, d, bits):
    cb = tq.tq_codebook_init(d, bits)
    ora = lloyd_max(d, bits)
    assert cb.d == d and cb.bits == bits and cb.levels == 1 << bits
    c64 = np.array(cb.c64[: cb.levels])
    t64 = np.array(cb.t64[: cb.levels - 1])
    assert np.max(np.abs(c64 - ora.c)) <= 1e-12 * np.max(np.abs(ora.c))
    assert np.max(np.abs(t64 - ora.t)) <= 1e-12 * np.max(np.abs(ora.c))
    # the fp32 values that define the packed format are identical
    assert np.array_equal(np.array(cb.c[: cb.levels], dtype=np.float32), ora.c32)
    assert np.array_equal(np.array(cb.t[: cb.levels - 1], dtype=np.float32), ora.t32)
    assert abs(cb.distortion - distortion_per_vector(ora)) < 1e-11


def test_codebook_argument_errors(L):
    out = tq.Codebook()
    assert L.tq_codebook_init(128, 0, ctypes.byref(out)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_codebook_init(128, 5, ctypes.byref(out)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_codebook_init(2, 2, ctypes.byref(out)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_codebook_init(128, 2, None) == tq.TQ_ERR_INVALID_ARG
    assert b"NULL" in L.tq_last_error()
    assert L.tq_codebook_init(128, 2, ctypes.byref(out)) == tq.TQ_OK
    assert L.tq_last_error() == b""


def test_rotation_bytes(L):
    assert tq.tq_rotation_bytes(100) == 0          # not a multiple of 32
    assert tq.tq_rotation_bytes(128) >= 3 * 128 * 128 * 4 + 8 * 128 * 128 * 2
    assert tq.tq_rotation_bytes(1536) > tq.tq_rotation_bytes(128)


def test_device_calls_reject_bad_arguments_on_host(L):
    # validation happens before any CUDA call, so these run without a GPU
    cb = tq.tq_codebook_init(128, 3)
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert L.tq_encode_mse(ctypes.byref(cb), 10, 128, good, tq.TQ_BF16, good, None, good, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_encode_mse(ctypes.byref(cb), -1, 128, good, tq.TQ_BF16, good, good, good, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_encode_mse(ctypes.byref(cb), 10, 100, good, tq.TQ_BF16, good, good, good, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse(ctypes.byref(cb), 10, 64, good, tq.TQ_BF16, good, good, good, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_encode_mse(ctypes.byref(cb), 10, 128, P((1 << 20) + 4), tq.TQ_BF16, good, good, good, None) \
        == tq.TQ_ERR_INVALID_ARG
    assert L.tq_encode_mse(ctypes.byref(cb), 10, 128, good, tq.TQ_F16, good, good, good, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse(ctypes.byref(cb), 0, 128, good, tq.TQ_BF16, good, good, good, None) == tq.TQ_OK
    assert L.tq_encode_prod(ctypes.byref(cb), 10, 128, good, tq.TQ_BF16, good, good, None, good, good, None, 0, None) \
        == tq.TQ_ERR_INVALID_ARG
    # d > 128 must be a multiple of 128; Algorithm 2 there needs its workspace
    cb256 = tq.tq_codebook_init(256, 2)
    assert L.tq_encode_mse(ctypes.byref(tq.tq_codebook_init(160, 2)), 10, 160, good, tq.TQ_BF16, good, good, good,
                           None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_workspace_bytes(10, 128, 2) == 0 and L.tq_encode_workspace_bytes(1000, 256, 1) == 0
    assert L.tq_encode_workspace_bytes(1000, 256, 2) > 0
    assert L.tq_encode_prod(ctypes.byref(cb256), 1000, 256, good, tq.TQ_BF16, good, good, good, good, good, None, 0,
                            None) == tq.TQ_ERR_WORKSPACE
    assert L.tq_decode(ctypes.byref(cb), 10, 128, good, good, good, good, None, good, tq.TQ_F32, None) \
        == tq.TQ_ERR_INVALID_ARG
    assert L.tq_rotation_prepare(128, good, good, good, 16, None) == tq.TQ_ERR_WORKSPACE


def test_attend_append_rejects_bad_arguments_on_host(L):
    cbk, cbv = tq.tq_codebook_init(128, 3), tq.tq_codebook_init(128, 1)
    P = ctypes.c_void_p
    g = P(1 << 20)
    args = lambda T_cur, T_max, ws_bytes, vs=g: (ctypes.byref(cbk), ctypes.byref(cbv), 2, 8, 2, T_cur, T_max, 128, g,
                                                tq.TQ_BF16, g, g, tq.TQ_BF16, g, g, g, g, vs, g, g, ctypes.c_float(0.1), g,
                                                g, ws_bytes, None)
    need = L.tq_attend_append_workspace_bytes(2, 8, 2, 10, 128, 3, 1)
    assert need == L.tq_attend_workspace_bytes(2, 8, 2, 11, 128)      # the attention's own workspace
    assert L.tq_attend_append_workspace_bytes(2, 8, 2, -1, 128, 3, 1) == 0
    assert L.tq_attend_append(*args(10, 10, need)) == tq.TQ_ERR_INVALID_ARG        # no free slot
    assert L.tq_attend_append(*args(-1, 10, need)) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_attend_append(*args(10, 20, need, vs=None)) == tq.TQ_ERR_INVALID_ARG   # values are Algorithm 2
    assert L.tq_attend_append(*args(10, 20, need - 1)) == tq.TQ_ERR_WORKSPACE
    # the attention's limits are checked before anything touches the cache
    cb64 = tq.tq_codebook_init(64, 3)
    bad_d = (ctypes.byref(cb64), ctypes.byref(tq.tq_codebook_init(64, 1)), 2, 8, 2, 10, 20, 64, g, tq.TQ_BF16, g, g,
             tq.TQ_BF16, g, g, g, g, g, g, g, ctypes.c_float(0.1), g, g, need, None)
    assert L.tq_attend_append(*bad_d) == tq.TQ_ERR_UNSUPPORTED
    bad_q = list(args(10, 20, need))
    bad_q[9] = tq.TQ_F16
    assert L.tq_attend_append(*bad_q) == tq.TQ_ERR_UNSUPPORTED


def test_binding_signatures_match_the_header(L):
    # every function the binding declares has as many arguments as its prototype in tq.h
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    protos = {}
    for m in re.finditer(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(([^;]*?)\)\s*;", src, flags=re.S):
        params = m.group(2).strip()
        protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    for name, (_res, args) in tq._SIGNATURES.items():
        assert name in protos, name
        assert len(args) == protos[name], (name, len(args), protos[name])


def test_selftest_wait_rejects_bad_limits_on_host(L):
    for lim in (0, 999, 2_000_000_000):
        assert L.tq_selftest_wait(lim, None) == tq.TQ_ERR_INVALID_ARG


def test_attend_prefill_rejects_bad_arguments_on_host(L):
    cbk, cbv = tq.tq_codebook_init(128, 3), tq.tq_codebook_init(128, 1)
    P = ctypes.c_void_p
    g = P(1 << 20)
    need = L.tq_attend_prefill_workspace_bytes(2, 8, 2, 5, 700, 128)
    assert need >= L.tq_attend_workspace_bytes(2, 8, 2, 700, 128) > 0
    assert L.tq_attend_prefill_workspace_bytes(2, 8, 2, 0, 700, 128) == 0
    assert L.tq_attend_prefill_workspace_bytes(2, 8, 2, 701, 700, 128) == 0
    args = lambda Qn, T, ws_bytes: (ctypes.byref(cbk), ctypes.byref(cbv), 2, 8, 2, Qn, T, 128, g, tq.TQ_BF16, g, g, g,
                                    None, None, g, g, g, g, ctypes.c_float(0.0), g, g, ws_bytes, None)
    assert L.tq_attend_prefill(*args(0, 700, need)) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_attend_prefill(*args(701, 700, need)) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_attend_prefill(*args(5, 700, need - 1)) == tq.TQ_ERR_WORKSPACE


def test_mixed_width_calls_reject_bad_arguments_on_host(L):
    d = 128
    cbs = (tq.Codebook * 4)()
    for b in (1, 2, 3, 4):
        cbs[b - 1] = tq.tq_codebook_init(d, b)
    P = ctypes.c_void_p
    g = P(1 << 20)
    gb = lambda *w: (ctypes.c_int32 * len(w))(*w)
    ok = gb(3, 3, 2, 2)
    assert L.tq_encode_mse_mixed(cbs, gb(3, 3, 2, 5), 10, d, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse_mixed(cbs, gb(3, 3, 0, 2), 10, d, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse_mixed(cbs, ok, 10, 256, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse_mixed(cbs, ok, -1, d, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_encode_mse_mixed(cbs, ok, 10, d, P((1 << 20) + 4), tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_INVALID_ARG
    wrong = (tq.Codebook * 4)()
    wrong[2] = tq.tq_codebook_init(d, 2)                  # a 2-bit codebook where the 3-bit one belongs
    wrong[1] = tq.tq_codebook_init(d, 2)
    assert L.tq_encode_mse_mixed(wrong, ok, 10, d, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_decode_mixed(cbs, gb(3, 3, 2, 9), 10, d, g, g, g, g, tq.TQ_F32, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_decode_mixed(cbs, ok, 10, d, g, g, g, g, tq.TQ_F16, None) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_encode_mse_mixed(cbs, ok, 0, d, g, tq.TQ_BF16, g, g, g, None) == tq.TQ_OK      # n = 0: no work
