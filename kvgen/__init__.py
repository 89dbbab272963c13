"""Seeded synthetic BF16 KV-cache inputs.

This module only draws inputs; it holds none of the codec's arithmetic.  Both
the CPU oracle and the CUDA library are fed from it, so the same bytes reach
both sides.  Values are drawn in float32 and rounded to BF16 with
round-to-nearest-even; the result is returned as uint16 bit patterns.

No dataset or model weights are available, so these tensors stand in for the
KV caches of the SplitZip explainer's SGLang runs ("Les Resultats").  They are
shaped like Llama-3-8B / Llama-3-70B KV caches and follow the explainer's one
observation about the data (section 2): exponents repeat, mantissas do not.

Workloads (seed = 0x5EED0000 + workload id):
  0  tiny K tensor   [8 h][1024 t][128 d]; N(0,1) x per-(h,d) scale
                     log-uniform in [2^-4, 2^4]; 0.1% of positions x 2^(+-20..40)
  1  Llama-3-8B 4K   [32 L][K,V][8 h][4096 t][128 d]
  2  Llama-3-8B 32K  same with 32768 tokens (4 GiB)
  3  Llama-3-70B 8K  [80 L][K,V][8 h][8192 t][128 d], Student-t(2) heavy tails
  4  paged batch     256 requests, 16-token pages [8 h][16 t][128 d] scattered
                     in a 6 GiB pool by a seeded page table
K tensors: N(0,1) x per-(h,d) scale log-uniform in [2^-4, 2^4], and 4 seeded
outlier channels per head x 2^6.  V tensors: N(0,1) x per-head scale
log-uniform in [0.25, 4].
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SEED_BASE = 0x5EED0000
HEADS = 8
HEAD_DIM = 128
PAGE_TOKENS = 16
PAGE_ELEMS = HEADS * PAGE_TOKENS * HEAD_DIM  # 16384
POOL_BYTES = 6 << 30
POOL_PAGES = POOL_BYTES // (PAGE_ELEMS * 2)  # 196608

# workload id -> (layers, tokens) for the contiguous [L][2][H][T][D] caches
CONTIGUOUS = {1: (32, 4096), 2: (32, 32768), 3: (80, 8192)}
# Student-t scale exponent range for workload 3: per-channel scale is
# log-uniform in [2^-T3, 2^T3]; chosen so that 3-5% of exponents fall outside
# the per-tensor top 16 (measured value recorded in the design notes).
T3_SCALE_LOG2 = 7.0


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (nearest, ties to even); returns uint16 bits.

    For finite values and infinities (a NaN whose payload sits in the low 16
    bits would round to infinity); the generators here draw no NaN."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _log_uniform(rng, lo_log2: float, hi_log2: float, size):
    return np.exp2(rng.uniform(lo_log2, hi_log2, size=size)).astype(np.float32)


def k_scales(rng, heads: int = HEADS, dim: int = HEAD_DIM) -> np.ndarray:
    """Per-(head, channel) K scale with 4 outlier channels per head (x 2^6)."""
    s = _log_uniform(rng, -4.0, 4.0, (heads, dim))
    for h in range(heads):
        ch = rng.choice(dim, size=4, replace=False)
        s[h, ch] *= np.float32(64.0)
    return s


def v_scales(rng, heads: int = HEADS) -> np.ndarray:
    """Per-head V scale, log-uniform in [0.25, 4]."""
    return _log_uniform(rng, -2.0, 2.0, (heads,))


def k_tensor(rng, heads: int, tokens: int, dim: int) -> np.ndarray:
    s = k_scales(rng, heads, dim)
    z = rng.standard_normal((heads, tokens, dim), dtype=np.float32)
    z *= s[:, None, :]
    return f32_to_bf16_bits(z).reshape(-1)


def v_tensor(rng, heads: int, tokens: int, dim: int) -> np.ndarray:
    s = v_scales(rng, heads)
    z = rng.standard_normal((heads, tokens, dim), dtype=np.float32)
    z *= s[:, None, None]
    return f32_to_bf16_bits(z).reshape(-1)


def heavy_tail_tensor(rng, heads: int, tokens: int, dim: int,
                      scale_log2: float = T3_SCALE_LOG2) -> np.ndarray:
    """Student-t with 2 degrees of freedom, Z / sqrt(-ln U), times a
    per-channel scale log-uniform in [2^-scale_log2, 2^scale_log2]."""
    s = _log_uniform(rng, -scale_log2, scale_log2, (heads, dim))
    z = rng.standard_normal((heads, tokens, dim), dtype=np.float32)
    u = np.float32(1.0) - rng.random((heads, tokens, dim), dtype=np.float32)  # (0, 1]
    chi = np.sqrt(-np.log(u))
    chi = np.maximum(chi, np.float32(1e-30))
    z /= chi
    z *= s[:, None, :]
    return f32_to_bf16_bits(z).reshape(-1)


def tiny_k_tensor(seed: int = SEED_BASE + 0, heads: int = HEADS, tokens: int = 1024,
                  dim: int = HEAD_DIM, outlier_frac: float = 0.001) -> np.ndarray:
    """Workload 0: one K tensor with 0.1% forced escapes."""
    rng = np.random.default_rng([seed, 0])
    s = _log_uniform(rng, -4.0, 4.0, (heads, dim))
    z = rng.standard_normal((heads, tokens, dim), dtype=np.float32)
    z *= s[:, None, :]
    z = z.reshape(-1)
    n_out = int(round(outlier_frac * z.size))
    if n_out:
        pos = rng.choice(z.size, size=n_out, replace=False)
        k = rng.integers(20, 41, size=n_out)
        sign = np.where(rng.random(n_out) < 0.5, -1.0, 1.0)
        z[pos] *= np.exp2(sign * k).astype(np.float32)
    return f32_to_bf16_bits(z)


def contiguous_tensor(workload: int, layer: int, kv: int, tokens: int | None = None) -> np.ndarray:
    """One (layer, K/V) tensor [8 h][tokens][128 d] of workloads 1-3."""
    layers, t_full = CONTIGUOUS[workload]
    t = t_full if tokens is None else tokens
    rng = np.random.default_rng([SEED_BASE + workload, layer, kv])
    if workload == 3:
        return heavy_tail_tensor(rng, HEADS, t, HEAD_DIM)
    if kv == 0:
        return k_tensor(rng, HEADS, t, HEAD_DIM)
    return v_tensor(rng, HEADS, t, HEAD_DIM)


def contiguous_cache(workload: int, layers: int | None = None, tokens: int | None = None,
                     out: np.ndarray | None = None) -> np.ndarray:
    """The whole cache [L][2][8][T][128] as a [2L, 8*T*128] uint16 array, one
    row per (layer, K/V) tensor; rows are generated in parallel threads."""
    l_full, t_full = CONTIGUOUS[workload]
    L = l_full if layers is None else layers
    T = t_full if tokens is None else tokens
    n_t = HEADS * T * HEAD_DIM
    if out is None:
        out = np.empty((2 * L, n_t), np.uint16)

    def job(i):
        out[i] = contiguous_tensor(workload, i // 2, i % 2, T)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(job, range(2 * L)))
    return out


class PagedBatch:
    """Workload 4: requests stored in 16-token pages scattered in a pool.

    lengths[r]     tokens of request r (multiple of 16)
    page_table[r]  pool slot of each of request r's pages, in stream order
    pages[r]       uint16 [n_pages_r, 8*16*128]: the page contents
    """

    def __init__(self, lengths, page_table, pages, pool_pages):
        self.lengths = lengths
        self.page_table = page_table
        self.pages = pages
        self.pool_pages = pool_pages

    @property
    def n_requests(self):
        return len(self.lengths)

    def request_stream(self, r) -> np.ndarray:
        return self.pages[r].reshape(-1)


def paged_layout(n_requests: int = 256, min_tokens: int = 128, max_tokens: int = 16384,
                 pool_pages: int = POOL_PAGES, seed: int = SEED_BASE + 4):
    rng = np.random.default_rng([seed, 0xFFFF])
    raw = np.exp(rng.uniform(np.log(min_tokens), np.log(max_tokens), size=n_requests))
    lengths = (np.ceil(raw / PAGE_TOKENS) * PAGE_TOKENS).astype(np.int64)
    n_pages = lengths // PAGE_TOKENS
    total = int(n_pages.sum())
    if total > pool_pages:
        raise ValueError("pool too small: %d pages needed, %d available" % (total, pool_pages))
    perm = rng.permutation(pool_pages)[:total]
    starts = np.concatenate([[0], np.cumsum(n_pages)])
    table = [perm[starts[r]:starts[r + 1]].astype(np.int64) for r in range(n_requests)]
    return lengths, table


def paged_batch(n_requests: int = 256, min_tokens: int = 128, max_tokens: int = 16384,
                pool_pages: int = POOL_PAGES, adversarial: bool = False,
                seed: int = SEED_BASE + 4) -> PagedBatch:
    """Even requests are K-like, odd requests V-like; adversarial fills every
    page with uniform random 16-bit patterns instead."""
    lengths, table = paged_layout(n_requests, min_tokens, max_tokens, pool_pages, seed)
    pages = [None] * n_requests

    def job(r):
        rng = np.random.default_rng([seed, 1 + int(adversarial), r])
        n_p = int(lengths[r]) // PAGE_TOKENS
        if adversarial:
            pages[r] = rng.integers(0, 1 << 16, size=(n_p, PAGE_ELEMS), dtype=np.uint16)
            return
        if r % 2 == 0:
            s = k_scales(rng)[None, :, None, :]
        else:
            s = v_scales(rng)[None, :, None, None]
        z = rng.standard_normal((n_p, HEADS, PAGE_TOKENS, HEAD_DIM), dtype=np.float32)
        z *= s
        pages[r] = f32_to_bf16_bits(z).reshape(n_p, PAGE_ELEMS)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(job, range(n_requests)))
    return PagedBatch(lengths, table, pages, pool_pages)


def uniform_u16(n: int, seed: int) -> np.ndarray:
    """Uniform random 16-bit patterns (incompressible input)."""
    return np.random.default_rng([seed, 0xADAD]).integers(0, 1 << 16, size=n, dtype=np.uint16)


def mixed_small(n: int, seed: int) -> np.ndarray:
    """A small K-like stream of arbitrary length n (for ragged parity cases):
    N(0,1) x a per-channel scale over a 128-wide channel axis, with ~0.5% of
    elements pushed far out to force escapes."""
    rng = np.random.default_rng([seed, 0x5A11])
    s = _log_uniform(rng, -4.0, 4.0, (HEAD_DIM,))
    z = rng.standard_normal(n, dtype=np.float32)
    z *= np.resize(s, n)
    m = rng.random(n) < 0.005
    z[m] *= np.exp2(rng.integers(-40, 41, size=int(m.sum()))).astype(np.float32)
    return f32_to_bf16_bits(z)
