"""Seeded synthetic inputs for the head-split attention workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it.  Every array is drawn from its own NumPy generator, seeded by
``(seed, stream id)``, so any array can be regenerated alone.

Floating-point data are returned either as float32 or as bfloat16 bit
patterns in ``uint16`` arrays (round-to-nearest-even from float32), so that the
device and the host see identical bytes.

Workload shapes follow the pages' models: a Llama-2-7B-like MHA layer (32
heads, head_dim 128, 25% retrieval heads) and a Llama-3-8B-like GQA layer (32
query / 8 KV heads, 50% retrieval heads), sink 16 and recent 64.  No weights
or datasets are used.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

SINK = 16
RECENT = 64

# stream ids for the per-array generators
_S_Q, _S_K, _S_V, _S_KNEW, _S_VNEW, _S_QSTEP, _S_ALPHA, _S_SIGMA, _S_LEN, _S_PAGES, _S_HEADS = range(11)
_S_KSTREAM, _S_VSTREAM = 11, 12


def rng_for(seed: int, stream: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), *[int(e) for e in extra]])


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.
    For finite values and infinities (the generators draw no NaN) the
    rounding increment never carries out of 32 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + (np.uint32(0x7FFF) + r)) >> np.uint32(16)).astype(np.uint16)


_BLOCK = 1 << 22      # values per generator block
_pool = None


def _threads():
    global _pool
    if _pool is None:
        _pool = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _pool


def _fill_normal(rng: np.random.Generator, n: int, dtype: str, sigma=None) -> np.ndarray:
    """n samples of N(0, sigma^2) (sigma = 1 when None), as float32 or bf16
    bits.  The caller's generator gives one seed; block i of _BLOCK values
    comes from its own generator seeded (that seed, i), so the blocks are
    drawn in parallel threads and the result does not depend on how many."""
    base = int(rng.integers(0, 2 ** 63 - 1))
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)

    def fill(i):
        s, e = i * _BLOCK, min(n, (i + 1) * _BLOCK)
        x = np.random.default_rng([base, i]).standard_normal(e - s, dtype=np.float32)
        if sigma is not None:
            x *= np.float32(sigma)
        out[s:e] = to_bf16_bits(x) if dtype == "bf16" else x

    nb = (n + _BLOCK - 1) // _BLOCK
    if nb == 1:
        fill(0)
    elif nb > 1:
        list(_threads().map(fill, range(nb)))
    return out


def normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0, 1) samples of the given shape as float32 or bf16 bits."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    return _fill_normal(rng, n, dtype).reshape(shape)


def normal_scaled(rng: np.random.Generator, shape, dtype: str, sigma_per_head: np.ndarray,
                  head_axis: int) -> np.ndarray:
    """N(0, sigma_h^2) samples where sigma depends on the index along ``head_axis``."""
    shape = tuple(int(s) for s in shape)
    rest = tuple(s for i, s in enumerate(shape) if i != head_axis)
    per = int(np.prod(rest)) if rest else 1
    x = np.empty(shape, dtype=np.uint16 if dtype == "bf16" else np.float32)
    xm = np.moveaxis(x, head_axis, 0)
    for h in range(shape[head_axis]):
        xm[h] = _fill_normal(rng, per, dtype, float(sigma_per_head[h])).reshape(rest)
    return x


def retrieval_heads_by_seed(n_kv_heads: int, n_retrieval: int, seed: int = 1) -> np.ndarray:
    """The retrieval KV heads, chosen by seed (sorted)."""
    rng = rng_for(seed, _S_HEADS)
    return np.sort(rng.choice(n_kv_heads, n_retrieval, replace=False)).astype(np.int64)


def binary_alpha(n_kv_heads: int, heads) -> np.ndarray:
    a = np.zeros(n_kv_heads, dtype=np.float32)
    a[np.asarray(heads, dtype=np.int64)] = 1.0
    return a


@dataclass
class LayerShape:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str = "bf16"
    sink: int = SINK
    recent: int = RECENT

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# ---------------------------------------------------------------------------
# Workload generators
# ---------------------------------------------------------------------------

def tiny_prompt(seed: int = 0, n: int = 512, heads: int = 8, d: int = 64, steps: int = 16):
    """Tiny single-layer MHA case: fp32 prompt Q/K/V ~ N(0,1) [n, heads, d],
    ``steps`` decode tokens, heads {1, 5} retrieval, and a continuous alpha
    ~ U(0, 1) per head for the gated mix."""
    return dict(
        shape=LayerShape(heads, heads, d, "fp32"),
        q=normal(rng_for(seed, _S_Q), (n, heads, d), "fp32"),
        k=normal(rng_for(seed, _S_K), (n, heads, d), "fp32"),
        v=normal(rng_for(seed, _S_V), (n, heads, d), "fp32"),
        q_step=normal(rng_for(seed, _S_QSTEP), (steps, 1, heads, d), "fp32"),
        k_step=normal(rng_for(seed, _S_KNEW), (steps, 1, heads, d), "fp32"),
        v_step=normal(rng_for(seed, _S_VNEW), (steps, 1, heads, d), "fp32"),
        alpha_mix=rng_for(seed, _S_ALPHA).uniform(0.0, 1.0, heads).astype(np.float32),
        retrieval=np.array([1, 5], dtype=np.int64),
    )


def prompt(shape: LayerShape, n: int, seed: int = 0, batch: int = 1, sigma=None):
    """A whole prompt's Q/K/V: q [B, n, Hq, d], k/v [B, n, Hkv, d]."""
    if sigma is None:
        k = normal(rng_for(seed, _S_K), (batch, n, shape.n_kv_heads, shape.head_dim), shape.dtype)
        v = normal(rng_for(seed, _S_V), (batch, n, shape.n_kv_heads, shape.head_dim), shape.dtype)
    else:
        k = normal_scaled(rng_for(seed, _S_K), (batch, n, shape.n_kv_heads, shape.head_dim), shape.dtype, sigma, 2)
        v = normal_scaled(rng_for(seed, _S_V), (batch, n, shape.n_kv_heads, shape.head_dim), shape.dtype, sigma, 2)
    q = normal(rng_for(seed, _S_Q), (batch, n, shape.n_q_heads, shape.head_dim), shape.dtype)
    return q, k, v


def head_sigma(n_kv_heads: int, seed: int = 0) -> np.ndarray:
    """Per-KV-head scale sigma ~ U(0.5, 2)."""
    return rng_for(seed, _S_SIGMA).uniform(0.5, 2.0, n_kv_heads).astype(np.float32)


def context_lengths(batch: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Per-sequence context lengths drawn uniformly from [lo, hi]."""
    return rng_for(seed, _S_LEN).integers(lo, hi + 1, batch).astype(np.int64)


STREAM_BLOCK = 1024   # positions per generator block of a streaming head's rows


class DecodeState:
    """Seeded rows of a cache state after a prompt of ``lengths[b]`` tokens.

    ``full[(b, h)] = (k [L_b, d], v [L_b, d])`` for every retrieval KV head h:
    the rows of positions 0..L_b-1.  A streaming KV head's rows are drawn on
    demand by ``stream_rows(b, h, positions)``: the row of position p comes
    from the generator of its block of ``STREAM_BLOCK`` positions, so any set
    of positions gets the same row for p whichever other positions are asked
    for.  Which positions a streaming cache still holds is not decided here:
    that is the method's eviction rule, which each side applies itself.
    """

    def __init__(self, shape: LayerShape, retrieval, lengths, seed: int = 0, sigma=None):
        self.shape = shape
        self.retrieval = sorted(int(h) for h in retrieval)
        self.lengths = np.asarray(lengths, dtype=np.int64)
        self.seed = int(seed)
        self.sigma = None if sigma is None else np.asarray(sigma, dtype=np.float32)
        self.full = {}
        for b, L in enumerate(self.lengths):
            L = int(L)
            for h in self.retrieval:
                rk, rv = rng_for(seed, _S_K, b, h), rng_for(seed, _S_V, b, h)
                self.full[(b, h)] = (self._draw(rk, L, h), self._draw(rv, L, h))

    def _draw(self, rng, n: int, h: int) -> np.ndarray:
        d = self.shape.head_dim
        if self.sigma is None:
            return normal(rng, (n, d), self.shape.dtype)
        return normal_scaled(rng, (1, n, d), self.shape.dtype, self.sigma[h:h + 1], 0)[0]

    def stream_rows(self, b: int, h: int, positions):
        """(k [n, d], v [n, d]) of a streaming KV head at the given positions."""
        pos = np.asarray(positions, dtype=np.int64)
        d = self.shape.head_dim
        dt = np.uint16 if self.shape.dtype == "bf16" else np.float32
        k = np.empty((len(pos), d), dtype=dt)
        v = np.empty_like(k)
        for blk in np.unique(pos // STREAM_BLOCK):
            sel = np.flatnonzero(pos // STREAM_BLOCK == blk)
            kb = self._draw(rng_for(self.seed, _S_KSTREAM, b, h, int(blk)), STREAM_BLOCK, h)
            vb = self._draw(rng_for(self.seed, _S_VSTREAM, b, h, int(blk)), STREAM_BLOCK, h)
            k[sel] = kb[pos[sel] % STREAM_BLOCK]
            v[sel] = vb[pos[sel] % STREAM_BLOCK]
        return k, v

    def token_rows(self, b: int, positions):
        """k, v [n, Hkv, d] of every KV head at the given positions of sequence
        b (model head order): a retrieval head's cached rows, a streaming
        head's drawn rows."""
        pos = np.asarray(positions, dtype=np.int64)
        sh = self.shape
        dt = np.uint16 if sh.dtype == "bf16" else np.float32
        k = np.empty((len(pos), sh.n_kv_heads, sh.head_dim), dtype=dt)
        v = np.empty_like(k)
        for h in range(sh.n_kv_heads):
            if (b, h) in self.full:
                k[:, h] = self.full[(b, h)][0][pos]
                v[:, h] = self.full[(b, h)][1][pos]
            else:
                k[:, h], v[:, h] = self.stream_rows(b, h, pos)
        return k, v


def decode_state(shape: LayerShape, retrieval, lengths, seed: int = 0, sigma=None) -> DecodeState:
    """Rows of a cache state after a prompt of ``lengths[b]`` tokens per
    sequence (see DecodeState)."""
    return DecodeState(shape, retrieval, lengths, seed=seed, sigma=sigma)


def decode_steps(shape: LayerShape, batch: int, steps: int, seed: int = 0, sigma=None, first: int = 0):
    """Per-step new-token tensors: q [steps, B, Hq, d], k/v [steps, B, Hkv, d].
    Step i is drawn from its own generator, so a window of steps starting at
    ``first`` can be made without the earlier ones."""
    d = shape.head_dim
    qs, ks, vs = [], [], []
    for i in range(first, first + steps):
        qs.append(normal(rng_for(seed, _S_QSTEP, i), (batch, shape.n_q_heads, d), shape.dtype))
        if sigma is None:
            ks.append(normal(rng_for(seed, _S_KNEW, i), (batch, shape.n_kv_heads, d), shape.dtype))
            vs.append(normal(rng_for(seed, _S_VNEW, i), (batch, shape.n_kv_heads, d), shape.dtype))
        else:
            ks.append(normal_scaled(rng_for(seed, _S_KNEW, i), (batch, shape.n_kv_heads, d), shape.dtype, sigma, 1))
            vs.append(normal_scaled(rng_for(seed, _S_VNEW, i), (batch, shape.n_kv_heads, d), shape.dtype, sigma, 1))
    return np.stack(qs), np.stack(ks), np.stack(vs)


def page_assignment(lengths, extra_tokens: int, page_size: int, seed: int = 0):
    """A shuffled page pool: page_table [B, max_pages] (int32, -1 = unused) that
    gives every sequence enough pages for lengths[b] + extra_tokens tokens,
    with physical page ids drawn as a seeded permutation of the pool."""
    lengths = np.asarray(lengths, dtype=np.int64)
    need = (lengths + extra_tokens + page_size - 1) // page_size
    total = int(need.sum())
    ids = rng_for(seed, _S_PAGES).permutation(total).astype(np.int32)
    max_pages = int(need.max())
    table = np.full((len(lengths), max_pages), -1, dtype=np.int32)
    o = 0
    for b, n in enumerate(need):
        table[b, :n] = ids[o:o + n]
        o += int(n)
    return table, total
