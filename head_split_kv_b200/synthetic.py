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
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def normal(rng: np.random.Generator, shape, dtype: str, block: int = 1 << 24) -> np.ndarray:
    """N(0, 1) samples as float32 or bf16 bits, generated in blocks to bound
    host memory."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    for s in range(0, n, block):
        e = min(n, s + block)
        x = rng.standard_normal(e - s, dtype=np.float32)
        out[s:e] = to_bf16_bits(x) if dtype == "bf16" else x
    return out.reshape(shape)


def normal_scaled(rng: np.random.Generator, shape, dtype: str, sigma_per_head: np.ndarray,
                  head_axis: int, block_rows: int = 1 << 16) -> np.ndarray:
    """N(0, sigma_h^2) samples where sigma depends on the index along ``head_axis``."""
    shape = tuple(int(s) for s in shape)
    x = np.empty(shape, dtype=np.uint16 if dtype == "bf16" else np.float32)
    xm = np.moveaxis(x, head_axis, 0)
    for h in range(shape[head_axis]):
        sub = xm[h]
        flat = sub.reshape(-1)
        n = flat.shape[0]
        blk = block_rows * shape[-1]
        for s in range(0, n, blk):
            e = min(n, s + blk)
            v = rng.standard_normal(e - s, dtype=np.float32) * np.float32(sigma_per_head[h])
            flat[s:e] = to_bf16_bits(v) if dtype == "bf16" else v
        xm[h] = flat.reshape(sub.shape)
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


def decode_state(shape: LayerShape, retrieval, lengths, seed: int = 0, sigma=None):
    """Cache contents after a prompt of ``lengths[b]`` tokens, per model KV head.

    Returns a dict with, for each sequence b and KV head h:
      full[(b, h)]   = (k [L_b, d], v [L_b, d]) for a retrieval head, positions 0..L_b-1
      stream[(b, h)] = (pos [n], k [n, d], v [n, d]) for a streaming head, the
                       surviving positions: 0..min(L, sink)-1 and the last
                       ``recent`` positions
    A streaming head never keeps the other tokens, so they are not drawn.
    """
    retrieval = set(int(h) for h in retrieval)
    d = shape.head_dim
    full, stream = {}, {}
    for b, L in enumerate(np.asarray(lengths, dtype=np.int64)):
        L = int(L)
        for h in range(shape.n_kv_heads):
            sig = None if sigma is None else np.asarray([sigma[h]], dtype=np.float32)
            if h in retrieval:
                rk, rv = rng_for(seed, _S_K, b, h), rng_for(seed, _S_V, b, h)
                if sig is None:
                    full[(b, h)] = (normal(rk, (L, d), shape.dtype), normal(rv, (L, d), shape.dtype))
                else:
                    full[(b, h)] = (normal_scaled(rk, (1, L, d), shape.dtype, sig, 0)[0],
                                    normal_scaled(rv, (1, L, d), shape.dtype, sig, 0)[0])
            else:
                keep = sorted(set(range(min(L, shape.sink))) | set(range(max(0, L - shape.recent), L)))
                pos = np.asarray(keep, dtype=np.int64)
                rk, rv = rng_for(seed, _S_KSTREAM, b, h), rng_for(seed, _S_VSTREAM, b, h)
                n = len(pos)
                if sig is None:
                    stream[(b, h)] = (pos, normal(rk, (n, d), shape.dtype), normal(rv, (n, d), shape.dtype))
                else:
                    stream[(b, h)] = (pos, normal_scaled(rk, (1, n, d), shape.dtype, sig, 0)[0],
                                      normal_scaled(rv, (1, n, d), shape.dtype, sig, 0)[0])
    return dict(full=full, stream=stream, lengths=np.asarray(lengths, dtype=np.int64))


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
