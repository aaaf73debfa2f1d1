"""Seeded synthetic inputs for the TurboQuant KV-cache encode / packed-attention path.

This module is the only code shared by the oracle and the CUDA path. It draws
random inputs (vectors, the rotation Pi, the JL matrix S, queries) and holds none
of the method's arithmetic: no norms, no quantisation, no packing, no scoring.

Random numbers the method itself draws (Pi and S) are produced here and handed
to both sides as inputs, so neither side has to reproduce the other's RNG.

Recipes (all numpy ``default_rng`` / ``SeedSequence``; seeds: data 0, Pi 0,
S 1, queries 2):

* ``gaussian``: i.i.d. N(0,1) rows.
* ``kv_block``: per head, N(0,1) entries; ``n_outlier`` channels chosen per head
  without replacement are multiplied by ``outlier_scale`` (the "energy
  concentrated in a few dimensions" example in the techblog-plum page's outlier
  section); optionally each token row is multiplied by exp(sigma * N(0,1))
  (log-normal per-token norms). Values are rounded to bf16 (RNE).
* ``unit_rows``: normalised Gaussian rows (uniform on the sphere).
* ``rotation``: Pi = Q diag(sign(diag R)) from the QR of a d x d standard-normal
  matrix (the sign fix makes the factorisation unique), rounded to fp32.
* ``jl_matrix``: S with i.i.d. N(0,1) entries, fp32.

Large arrays are drawn in independent blocks keyed by (seed, tag, block), so a
checker can regenerate any block alone.
"""
from __future__ import annotations

import numpy as np

# Tags keep the K, V, query and database streams independent under one seed.
TAG_K, TAG_V, TAG_Q, TAG_DB, TAG_X = 11, 12, 13, 14, 15

SEED_DATA, SEED_PI, SEED_S, SEED_QUERY = 0, 0, 1, 2


def rng_for(seed: int, *keys: int) -> np.random.Generator:
    """Generator for the stream (seed, *keys); distinct keys give independent streams."""
    return np.random.default_rng(np.random.SeedSequence([int(seed), *[int(k) for k in keys]]))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 array rounded to the nearest bf16 value (ties to even), returned as fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of an fp32 array that already holds bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def gaussian(n: int, d: int, seed: int = SEED_DATA, tag: int = TAG_X) -> np.ndarray:
    """[n, d] fp32 i.i.d. N(0,1)."""
    return rng_for(seed, tag, n, d).standard_normal((n, d), dtype=np.float64).astype(np.float32)


def rotation(d: int, seed: int = SEED_PI) -> np.ndarray:
    """Random orthogonal d x d matrix (fp32, row-major); y = Pi @ x rotates x."""
    g = np.random.default_rng(seed).standard_normal((d, d))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.astype(np.float32))


def jl_matrix(d: int, seed: int = SEED_S) -> np.ndarray:
    """d x d matrix with i.i.d. N(0,1) entries (fp32, row-major)."""
    return np.ascontiguousarray(np.random.default_rng(seed).standard_normal((d, d)).astype(np.float32))


def kv_slice(tokens: int, d: int, n_outlier: int, outlier_scale: float,
             lognormal_sigma: float, seed: int, tag: int, *keys: int) -> np.ndarray:
    """One head's [tokens, d] bf16-valued block (returned as fp32)."""
    g = rng_for(seed, tag, *keys)
    x = g.standard_normal((tokens, d), dtype=np.float64)
    if n_outlier > 0:
        ch = g.choice(d, n_outlier, replace=False)
        x[:, ch] *= outlier_scale
    if lognormal_sigma > 0:
        x *= np.exp(lognormal_sigma * g.standard_normal((tokens, 1)))
    return round_to_bf16(x.astype(np.float32))


def kv_block(heads: int, tokens: int, d: int, n_outlier: int, outlier_scale: float = 20.0,
             lognormal_sigma: float = 0.0, seed: int = SEED_DATA, tag: int = TAG_K,
             batch_index: int = 0) -> np.ndarray:
    """[heads, tokens, d] bf16-valued KV block (fp32 container); heads drawn independently."""
    out = np.empty((heads, tokens, d), dtype=np.float32)
    for h in range(heads):
        out[h] = kv_slice(tokens, d, n_outlier, outlier_scale, lognormal_sigma, seed, tag,
                          batch_index, h)
    return out


def unit_rows_block(block: int, rows: int, d: int, seed: int = SEED_DATA, tag: int = TAG_DB) -> np.ndarray:
    """Block ``block`` of a row-blocked array of unit-norm rows, [rows, d] fp32."""
    g = rng_for(seed, tag, block, rows, d)
    x = g.standard_normal((rows, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)


def unit_rows(n: int, d: int, seed: int = SEED_DATA, tag: int = TAG_DB, block_rows: int = 4096) -> np.ndarray:
    """[n, d] fp32 unit-norm rows, drawn in independent blocks of ``block_rows``."""
    out = np.empty((n, d), dtype=np.float32)
    for b0 in range(0, n, block_rows):
        r = min(block_rows, n - b0)
        out[b0:b0 + r] = unit_rows_block(b0 // block_rows, block_rows, d, seed, tag)[:r]
    return out


def queries_bf16(shape: tuple, seed: int = SEED_QUERY) -> np.ndarray:
    """bf16-valued N(0,1) query tensor (fp32 container)."""
    return round_to_bf16(rng_for(seed, TAG_Q, *shape).standard_normal(shape).astype(np.float32))


# ---- named workloads -------------------------------------------------------------------------
# Each entry states the recipe; the sizes follow the pages' workloads (TinyLlama KV shape of
# 22 layers x 32 heads x d=64 on the traeai page's benchmark script; Llama-8B-like 8 KV heads x
# d=128; a decode-attention batch; a 1e6 x 1536 vector-search database).

WORKLOADS = {
    "tiny": dict(n=4096, d=128, bits=(1, 2, 3, 4), dtype="f32"),
    "tinyllama_block": dict(heads=32, tokens=4096, d=64, n_outlier=4, outlier_scale=20.0,
                            lognormal_sigma=0.0, k_bits=3, v_bits=2),
    "llama8b_cache": dict(heads=8, tokens=32768, d=128, n_outlier=3, outlier_scale=20.0,
                          lognormal_sigma=0.5, k_bits=3, v_bits=3),
    "decode_attention": dict(batch=16, hq=32, hkv=8, d=128, tokens=131072, n_outlier=3,
                             outlier_scale=20.0, lognormal_sigma=0.5, k_bits=3, v_bits=2),
    "vector_search": dict(n=1_000_000, d=1536, queries=1024, bits=4, topk=10),
}


def kv_slices_device(slices: int, tokens: int, d: int, n_outlier: int, outlier_scale: float,
                     lognormal_sigma: float, seed: int, device):
    """The ``kv_block`` recipe drawn on a CUDA device with a torch generator, for caches too large to
    draw on the host in a test: [slices * tokens, d] bf16, each slice of ``tokens`` rows N(0,1) with
    ``n_outlier`` channels x ``outlier_scale`` and optional log-normal token norms. Not bit-identical
    to ``kv_block`` (a different generator); same distribution."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = torch.empty((slices, tokens, d), dtype=torch.bfloat16, device=device)
    for s in range(slices):
        x = torch.randn((tokens, d), generator=g, device=device)
        if n_outlier > 0:
            ch = torch.randperm(d, generator=g, device=device)[:n_outlier]
            x[:, ch] *= outlier_scale
        if lognormal_sigma > 0:
            x *= torch.exp(lognormal_sigma * torch.randn((tokens, 1), generator=g, device=device))
        out[s] = x.to(torch.bfloat16)
    return out.view(-1, d)
