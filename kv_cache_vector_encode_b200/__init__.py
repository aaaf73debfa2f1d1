"""Python binding of libtq, the B200 (sm_100a) TurboQuant KV-cache quantisation library.

Argument marshalling only: every function below checks tensor placement / dtype / contiguity,
passes raw device pointers and the current CUDA stream to the C ABI declared in include/tq.h,
and raises TQError on a non-zero status. All computation happens in libtq's CUDA kernels
(and, for tq_codebook_init, in its host C++). There is no fallback: if libtq.so is missing or a
tensor is not on a CUDA device, the call fails.

Names follow the C ABI. Tensors:
  x        [n, d]  float32 / bfloat16 (CUDA)
  codes    [n, d/32, b] int32 (bit planes, uint32 bit patterns)
  signs    [n, d/32] int32
  norms    [n] float16,  gammas [n] float16
  rot      uint8 buffer of tq_rotation_bytes(d) bytes (prepared by tq_rotation_prepare)
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA = 0, 1, 2, 3
TQ_ERR_NOT_CONVERGED, TQ_ERR_DEVICE_TIMEOUT, TQ_ERR_WORKSPACE = 4, 5, 6
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2


class TQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libtq status {status}: {message}")
        self.status = status


class Codebook(ctypes.Structure):
    """Mirror of tq_codebook (host POD)."""
    _fields_ = [
        ("d", ctypes.c_int32), ("bits", ctypes.c_int32), ("levels", ctypes.c_int32),
        ("iterations", ctypes.c_int32),
        ("c", ctypes.c_float * 16), ("t", ctypes.c_float * 16),
        ("c64", ctypes.c_double * 16), ("t64", ctypes.c_double * 16),
        ("distortion", ctypes.c_double),
    ]

    @property
    def centroids(self):
        return list(self.c)[: self.levels]

    @property
    def boundaries(self):
        return list(self.t)[: self.levels - 1]


_lib = None

_P = ctypes.c_void_p
_I32, _I64, _SZ, _F = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_CB = ctypes.POINTER(Codebook)

_SIGNATURES = {
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_version": (ctypes.c_char_p, []),
    "tq_codebook_init": (_I32, [_I32, _I32, _CB]),
    "tq_rotation_bytes": (_SZ, [_I32]),
    "tq_rotation_prepare": (_I32, [_I32, _P, _P, _P, _SZ, _P]),
    "tq_encode_mse": (_I32, [_CB, _I64, _I32, _P, _I32, _P, _P, _P, _P]),
    "tq_encode_prod": (_I32, [_CB, _I64, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tq_encode_workspace_bytes": (_SZ, [_I64, _I32, _I32]),
    "tq_decode": (_I32, [_CB, _I64, _I32, _P, _P, _P, _P, _P, _P, _I32, _P]),
    "tq_encode_mse_mixed": (_I32, [_CB, _P, _I64, _I32, _P, _I32, _P, _P, _P, _P]),
    "tq_decode_mixed": (_I32, [_CB, _P, _I64, _I32, _P, _P, _P, _P, _I32, _P]),
    "tq_scores_workspace_bytes": (_SZ, [_I64, _I64, _I32, _I32]),
    "tq_scores": (_I32, [_CB, _I64, _I64, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tq_attend_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I64, _I32]),
    "tq_attend_decode": (_I32, [_CB, _CB, _I32, _I32, _I32, _I64, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P,
                                _P, _F, _P, _P, _SZ, _P]),
    "tq_attend_decode_noalloc": (_I32, [_CB, _CB, _I32, _I32, _I32, _I64, _I32, _P, _I32, _P, _P, _P, _P, _P, _P,
                                        _P, _P, _P, _F, _P, _P]),
    "tq_attend_prefill_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I64, _I32]),
    "tq_attend_prefill": (_I32, [_CB, _CB, _I32, _I32, _I32, _I32, _I64, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _P,
                                 _P, _P, _F, _P, _P, _SZ, _P]),
    "tq_attend_append_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I64, _I32, _I32, _I32]),
    "tq_attend_append": (_I32, [_CB, _CB, _I32, _I32, _I32, _I64, _I64, _I32, _P, _I32, _P, _P, _I32, _P, _P, _P,
                                _P, _P, _P, _P, _F, _P, _P, _SZ, _P]),
    "tq_selftest_wait": (_I32, [ctypes.c_uint64, _P]),
    "tq_sync_check": (_I32, [_P]),
}


def lib() -> ctypes.CDLL:
    """The loaded libtq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtq.so not found at {LIB_PATH}; build it with "
                               "`python -m kv_cache_vector_encode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name, None)
            if fn is None:
                continue
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != TQ_OK:
        raise TQError(status, lib().tq_last_error().decode())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t, name, dtypes=None, allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    return ctypes.c_void_p(t.data_ptr())


def _xdtype(t):
    import torch
    return {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}[t.dtype]


# ---- entry points ------------------------------------------------------------------------------

def tq_version() -> str:
    return lib().tq_version().decode()


def tq_codebook_init(d: int, bits: int) -> Codebook:
    cb = Codebook()
    _check(lib().tq_codebook_init(d, bits, ctypes.byref(cb)))
    return cb


def tq_rotation_bytes(d: int) -> int:
    return int(lib().tq_rotation_bytes(d))


def tq_rotation_prepare(Pi, S, rot=None, stream=None):
    """Prepare the rotation buffer from device fp32 Pi, S (d x d); returns it."""
    import torch
    d = Pi.shape[0]
    nbytes = tq_rotation_bytes(d)
    if rot is None:
        rot = torch.empty(nbytes, dtype=torch.uint8, device=Pi.device)
    _check(lib().tq_rotation_prepare(d, _ptr(Pi, "Pi", [torch.float32]), _ptr(S, "S", [torch.float32]),
                                     _ptr(rot, "rot"), rot.numel(), _stream(stream)))
    return rot


def tq_encode_mse(cb: Codebook, x, rot, codes, norms, stream=None):
    import torch
    n, d = x.shape
    _check(lib().tq_encode_mse(ctypes.byref(cb), n, d, _ptr(x, "x", [torch.float32, torch.bfloat16]), _xdtype(x),
                               _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                               _ptr(norms, "norms", [torch.float16]), _stream(stream)))


def tq_encode_workspace_bytes(n: int, d: int, alg: int) -> int:
    return int(lib().tq_encode_workspace_bytes(n, d, alg))


def tq_encode_prod(cb_bm1: Codebook, x, rot, codes, signs, norms, gammas, ws=None, stream=None):
    import torch
    n, d = x.shape
    wsb = tq_encode_workspace_bytes(n, d, 2)
    if ws is None and wsb > 0:
        ws = torch.empty(wsb, dtype=torch.uint8, device=x.device)
    _check(lib().tq_encode_prod(ctypes.byref(cb_bm1), n, d, _ptr(x, "x", [torch.float32, torch.bfloat16]),
                                _xdtype(x), _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                                _ptr(signs, "signs", [torch.int32]), _ptr(norms, "norms", [torch.float16]),
                                _ptr(gammas, "gammas", [torch.float16]), _ptr(ws, "ws", None, True),
                                ws.numel() if ws is not None else 0, _stream(stream)))


def tq_decode(cb: Codebook, rot, codes, norms, out, signs=None, gammas=None, stream=None):
    import torch
    n, d = out.shape
    _check(lib().tq_decode(ctypes.byref(cb), n, d, _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                           _ptr(signs, "signs", [torch.int32], True), _ptr(norms, "norms", [torch.float16]),
                           _ptr(gammas, "gammas", [torch.float16], True),
                           _ptr(out, "out", [torch.float32, torch.bfloat16]), _xdtype(out), _stream(stream)))


_mixed_cache = {}


def _mixed_args(d: int, group_bits):
    """Host arrays of the mixed-width calls: the 4 codebooks of d (1..4 bits) and the group widths
    (made once per (d, widths); the codebooks come from the library's host solver)."""
    key = (int(d), tuple(int(x) for x in group_bits))
    if key not in _mixed_cache:
        G = d // 32
        if len(key[1]) != G:
            raise ValueError(f"group_bits needs {G} entries for d = {d}")
        cbs = (Codebook * 4)()
        for b in sorted(set(key[1])):
            if 1 <= b <= 4:
                cbs[b - 1] = tq_codebook_init(d, b)
        _mixed_cache[key] = (cbs, (ctypes.c_int32 * G)(*key[1]))
    return _mixed_cache[key]


def tq_encode_mse_mixed(group_bits, x, rot, codes, norms, stream=None):
    """Algorithm 1 with a width per group of 32 rotated coordinates; codes [n, sum(group_bits)] int32."""
    import torch
    n, d = x.shape
    cbs, gb = _mixed_args(d, group_bits)
    _check(lib().tq_encode_mse_mixed(cbs, gb, n, d, _ptr(x, "x", [torch.float32, torch.bfloat16]), _xdtype(x),
                                     _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                                     _ptr(norms, "norms", [torch.float16]), _stream(stream)))


def tq_decode_mixed(group_bits, rot, codes, norms, out, stream=None):
    import torch
    n, d = out.shape
    cbs, gb = _mixed_args(d, group_bits)
    _check(lib().tq_decode_mixed(cbs, gb, n, d, _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                                 _ptr(norms, "norms", [torch.float16]),
                                 _ptr(out, "out", [torch.float32, torch.bfloat16]), _xdtype(out), _stream(stream)))


def tq_scores_workspace_bytes(nq: int, n: int, d: int, k: int) -> int:
    return int(lib().tq_scores_workspace_bytes(nq, n, d, k))


def tq_scores(cb: Codebook, q, rot, codes, norms, signs=None, gammas=None, scores=None, k=0, topk_ids=None,
              topk_scores=None, ws=None, stream=None):
    import torch
    nq, d = q.shape
    n = norms.shape[0]
    wsb = tq_scores_workspace_bytes(nq, n, d, k)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    _check(lib().tq_scores(ctypes.byref(cb), nq, n, d, _ptr(q, "q", [torch.float32, torch.bfloat16]), _xdtype(q),
                           _ptr(rot, "rot"), _ptr(codes, "codes", [torch.int32]),
                           _ptr(signs, "signs", [torch.int32], True), _ptr(norms, "norms", [torch.float16]),
                           _ptr(gammas, "gammas", [torch.float16], True),
                           _ptr(scores, "scores", [torch.float32], True), k,
                           _ptr(topk_ids, "topk_ids", [torch.int32], True),
                           _ptr(topk_scores, "topk_scores", [torch.float32], True),
                           _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def tq_attend_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, d: int) -> int:
    return int(lib().tq_attend_workspace_bytes(B, Hq, Hkv, T, d))


def tq_attend_decode(cb_k: Codebook, cb_v: Codebook, q, rot, k_codes, k_norms, v_codes, v_norms, out,
                     v_signs=None, v_gammas=None, scale=None, ws=None, stream=None, k_signs=None, k_gammas=None):
    import torch
    B, Hq, d = q.shape
    Hkv, T = k_norms.shape[1], k_norms.shape[2]
    if scale is None:
        scale = 0.0                   # the library's default, 1/sqrt(d)
    wsb = tq_attend_workspace_bytes(B, Hq, Hkv, T, d)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    _check(lib().tq_attend_decode(ctypes.byref(cb_k), ctypes.byref(cb_v), B, Hq, Hkv, T, d,
                                  _ptr(q, "q", [torch.float32, torch.bfloat16]), _xdtype(q), _ptr(rot, "rot"),
                                  _ptr(k_codes, "k_codes", [torch.int32]), _ptr(k_norms, "k_norms", [torch.float16]),
                                  _ptr(k_signs, "k_signs", [torch.int32], True),
                                  _ptr(k_gammas, "k_gammas", [torch.float16], True),
                                  _ptr(v_codes, "v_codes", [torch.int32]),
                                  _ptr(v_signs, "v_signs", [torch.int32], True),
                                  _ptr(v_norms, "v_norms", [torch.float16]),
                                  _ptr(v_gammas, "v_gammas", [torch.float16], True), float(scale),
                                  _ptr(out, "out", [torch.float32]), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def tq_attend_decode_noalloc(cb_k: Codebook, cb_v: Codebook, q, rot, k_codes, k_norms, v_codes, v_norms, out,
                             v_signs=None, v_gammas=None, scale=None, stream=None, k_signs=None, k_gammas=None):
    """tq_attend_decode with the library's fixed scratch array (no workspace, no allocation)."""
    import torch
    B, Hq, d = q.shape
    Hkv, T = k_norms.shape[1], k_norms.shape[2]
    if scale is None:
        scale = 0.0                   # the library's default, 1/sqrt(d)
    _check(lib().tq_attend_decode_noalloc(ctypes.byref(cb_k), ctypes.byref(cb_v), B, Hq, Hkv, T, d,
                                          _ptr(q, "q", [torch.float32, torch.bfloat16]), _xdtype(q), _ptr(rot, "rot"),
                                          _ptr(k_codes, "k_codes", [torch.int32]),
                                          _ptr(k_norms, "k_norms", [torch.float16]),
                                          _ptr(k_signs, "k_signs", [torch.int32], True),
                                          _ptr(k_gammas, "k_gammas", [torch.float16], True),
                                          _ptr(v_codes, "v_codes", [torch.int32]),
                                          _ptr(v_signs, "v_signs", [torch.int32], True),
                                          _ptr(v_norms, "v_norms", [torch.float16]),
                                          _ptr(v_gammas, "v_gammas", [torch.float16], True), float(scale),
                                          _ptr(out, "out", [torch.float32]), _stream(stream)))


def tq_attend_prefill_workspace_bytes(B: int, Hq: int, Hkv: int, Qn: int, T: int, d: int) -> int:
    return int(lib().tq_attend_prefill_workspace_bytes(B, Hq, Hkv, Qn, T, d))


def tq_attend_prefill(cb_k: Codebook, cb_v: Codebook, q, rot, k_codes, k_norms, v_codes, v_norms, out,
                      v_signs=None, v_gammas=None, scale=None, ws=None, stream=None, k_signs=None, k_gammas=None):
    """Causal multi-query attention: q, out [B, Qn, Hq, d]; the cache [B][Hkv][T] holds the Qn new
    tokens in its last Qn slots (query j attends slots t <= T - Qn + j)."""
    import torch
    B, Qn, Hq, d = q.shape
    Hkv, T = k_norms.shape[1], k_norms.shape[2]
    if scale is None:
        scale = 0.0                   # the library's default, 1/sqrt(d)
    wsb = tq_attend_prefill_workspace_bytes(B, Hq, Hkv, Qn, T, d)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    _check(lib().tq_attend_prefill(ctypes.byref(cb_k), ctypes.byref(cb_v), B, Hq, Hkv, Qn, T, d,
                                   _ptr(q, "q", [torch.float32, torch.bfloat16]), _xdtype(q), _ptr(rot, "rot"),
                                   _ptr(k_codes, "k_codes", [torch.int32]), _ptr(k_norms, "k_norms", [torch.float16]),
                                   _ptr(k_signs, "k_signs", [torch.int32], True),
                                   _ptr(k_gammas, "k_gammas", [torch.float16], True),
                                   _ptr(v_codes, "v_codes", [torch.int32]),
                                   _ptr(v_signs, "v_signs", [torch.int32], True),
                                   _ptr(v_norms, "v_norms", [torch.float16]),
                                   _ptr(v_gammas, "v_gammas", [torch.float16], True), float(scale),
                                   _ptr(out, "out", [torch.float32]), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


TQ_ATTEND_NOALLOC_MAX_BYTES = 8 << 20


def tq_attend_append_workspace_bytes(B: int, Hq: int, Hkv: int, T_cur: int, d: int, k_bits: int,
                                     v_codebook_bits: int) -> int:
    return int(lib().tq_attend_append_workspace_bytes(B, Hq, Hkv, T_cur, d, k_bits, v_codebook_bits))


def tq_attend_append(cb_k: Codebook, cb_v: Codebook, q, rot, k_new, v_new, T_cur: int, k_codes, k_norms, v_codes,
                     v_signs, v_norms, v_gammas, out, scale=None, ws=None, stream=None):
    """Encode the new token's K / V of every slice into slot T_cur of the cache, then attend over slots
    [0, T_cur]. The cache tensors are [B][Hkv][T_max]... as for tq_attend_decode; k_new, v_new [B][Hkv][d]."""
    import torch
    B, Hq, d = q.shape
    Hkv, T_max = k_norms.shape[1], k_norms.shape[2]
    if k_new.dtype != v_new.dtype:
        raise TypeError("tq_attend_append: k_new and v_new must have the same dtype (one x_dtype for both)")
    if tuple(k_new.shape) != (B, Hkv, d) or tuple(v_new.shape) != (B, Hkv, d):
        raise ValueError(f"tq_attend_append: k_new / v_new must be [B, Hkv, d] = {(B, Hkv, d)}")
    if scale is None:
        scale = 0.0                   # the library's default, 1/sqrt(d)
    wsb = tq_attend_append_workspace_bytes(B, Hq, Hkv, T_cur, d, cb_k.bits, cb_v.bits)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    _check(lib().tq_attend_append(ctypes.byref(cb_k), ctypes.byref(cb_v), B, Hq, Hkv, T_cur, T_max, d,
                                  _ptr(q, "q", [torch.float32, torch.bfloat16]), _xdtype(q),
                                  _ptr(k_new, "k_new", [torch.float32, torch.bfloat16]),
                                  _ptr(v_new, "v_new", [torch.float32, torch.bfloat16]), _xdtype(k_new),
                                  _ptr(rot, "rot"), _ptr(k_codes, "k_codes", [torch.int32]),
                                  _ptr(k_norms, "k_norms", [torch.float16]), _ptr(v_codes, "v_codes", [torch.int32]),
                                  _ptr(v_signs, "v_signs", [torch.int32]), _ptr(v_norms, "v_norms", [torch.float16]),
                                  _ptr(v_gammas, "v_gammas", [torch.float16]), float(scale),
                                  _ptr(out, "out", [torch.float32]), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def tq_sync_check(stream=None):
    _check(lib().tq_sync_check(_stream(stream)))


def tq_selftest_wait(limit_ns: int = 1_000_000, stream=None):
    """Enqueue the failure-detection self-test: a bounded device wait that runs out on purpose; the
    next tq_sync_check raises TQError with status TQ_ERR_DEVICE_TIMEOUT once."""
    _check(lib().tq_selftest_wait(int(limit_ns), _stream(stream)))


# ---- allocation helpers (torch device memory) --------------------------------------------------

def empty_mse(n: int, d: int, bits: int, device="cuda"):
    """Output tensors of an Algorithm 1 encode: codes [n, d/32, bits], norms [n]."""
    import torch
    return (torch.empty((n, d // 32, bits), dtype=torch.int32, device=device),
            torch.empty((n,), dtype=torch.float16, device=device))


def empty_prod(n: int, d: int, bits: int, device="cuda"):
    """Outputs of an Algorithm 2 encode at `bits`: codes [n, d/32, bits-1], signs, norms, gammas."""
    import torch
    return (torch.empty((n, d // 32, bits - 1), dtype=torch.int32, device=device),
            torch.empty((n, d // 32), dtype=torch.int32, device=device),
            torch.empty((n,), dtype=torch.float16, device=device),
            torch.empty((n,), dtype=torch.float16, device=device))
