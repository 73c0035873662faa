"""Plain CPU oracle for DuoAttention's head-split attention.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
product package (``head_split_kv_b200``) never imports it and shares no code
with it: no kernels, headers, helpers, tables or constants.

Everything is NumPy in float64.  Inputs arrive either as float32 arrays or as
bfloat16 bit patterns held in ``uint16`` arrays; both are widened to float64
exactly before any arithmetic.  Masks are explicit boolean matrices over
absolute token positions, the softmax is the textbook one, and the two KV
caches are explicit Python lists per (sequence, KV head).

Sources (page title, then section):

[Review]   "DuoAttention: Efficient Long-Context LLM Inference with Retrieval
           and Streaming Heads" -- paper review on xllm-io.github.io.
           S3 "Core formula" (the mixing equation and the two masks),
           S3 "Retrieval-head identification" (gate per KV head, binarisation
           with >= tau), S3 "Inference flow" (two caches per layer; decode
           splits Q/K/V by head and concatenates; chunked pre-fill),
           S3 "Deployment optimisation" (reordering heads into contiguous
           blocks), S5 "Ablations" item 3 (16 sink / 64 recent tokens).
[Summary]  "DuoAttention: Efficient Long-Context LLM Inference with Retrieval
           and Streaming Heads" -- paperlayer.ai summary of arXiv:2410.10819v1.
           S2 bullets "Optimization-based Identification" (one gate per KV
           head, GQA groups), "Binarizing Attention Implementations"
           (sparsity-quantile threshold), "Chunked Pre-filling" (both caches
           are filled chunk by chunk).

Readings where the pages are silent (each is listed with its reason in the
repository's design notes):

* The recent window includes the query itself: key j is "recent" for query i
  when ``i - j < recent``.
* The Lambda mask is causal as well: ``j <= i and (j < sink or i - j < recent)``.
* "QK^T (.) M" in the core formula is read as additive -inf masking before the
  softmax.
* Query head ``h`` uses KV head ``h // G`` with ``G = n_q_heads / n_kv_heads``.
* Softmax scale is ``1 / sqrt(head_dim)`` unless given.
* Decode appends the new token before attending, so a token sees itself.
* Streaming cache: keep every token with position < sink, plus the most recent
  ``recent`` tokens; when the list grows past ``sink + recent``, the oldest
  entry with position >= sink is evicted.
* Ring layout of the streaming cache: position p lives in slot p when
  p < sink, else in slot ``sink + (p - sink) % recent``; ``pos[slot]`` holds the
  position, -1 when the slot is empty.
* Top-k selection of retrieval heads breaks ties by the lower head index.
* Whole-chunk streaming pre-fill (a second pre-fill mode; the pages note
  that pre-fill gains grow as the chunk shrinks, which is what happens when a
  streaming head attends to its whole chunk): a streaming query at position
  i of the chunk starting at c0 sees the streaming cache as it stood before
  the chunk -- its sinks and the last ``recent`` tokens before c0 -- and every
  chunk token up to itself: ``j <= i and (j < sink or j >= c0 - recent)``.
  Decode is unchanged.
* 8-bit retrieval cache (the pages pair the method with a quantized KV cache
  but give no scheme): each cached K or V row of a head is stored as int8
  codes with one float32 scale, symmetric, amax = max |x|,
  code = rint(x * (127 / amax)) (round half to even), scale = amax / 127,
  all in float32 as written; a zero row has scale 0 and codes 0.  Attention
  reads code * scale.
* 4-bit retrieval cache (the paper review's "Quantization combination"
  pairs 8-bit weights with a 4-bit KV cache, again without a scheme): the
  same per-row symmetric steps with 7 levels a side, codes -7..7,
  scale = amax / 7.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "as_f64",
    "bf16_bits_to_f64",
    "causal_mask",
    "streaming_mask",
    "chunk_streaming_mask",
    "masked_softmax",
    "masked_attention",
    "full_attn",
    "streaming_attn",
    "gated_mix",
    "gated_mix_grad_alpha",
    "binarize_gates",
    "partition_heads",
    "ring_slot",
    "streaming_positions",
    "HeadSplitCache",
    "prefill_direct",
    "decode_direct",
    "quantize_int8_rows",
    "dequantize_int8_rows",
    "quantize_int4_rows",
]


# ---------------------------------------------------------------------------
# Exact widening of the input formats
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64, exactly.

    A bfloat16 value is the upper 16 bits of an IEEE float32, so shifting the
    pattern into the top half of a 32-bit word gives the same number as a
    float32, which float64 holds exactly.
    """
    b = np.asarray(bits)
    if b.dtype != np.uint16:
        raise TypeError("bfloat16 data must be passed as uint16 bit patterns")
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def as_f64(x: np.ndarray) -> np.ndarray:
    """Widen an input array (bf16 bits in uint16, float32 or float64) to float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_bits_to_f64(x)
    if x.dtype in (np.float32, np.float64):
        return x.astype(np.float64)
    raise TypeError(f"unsupported input dtype {x.dtype}")


# ---------------------------------------------------------------------------
# Masks [Review S3 "Core formula"]
# ---------------------------------------------------------------------------

def causal_mask(q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """M_causal[i, j] = (k_pos[j] <= q_pos[i]): the standard lower-triangular mask."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    return k_pos[None, :] <= q_pos[:, None]


def streaming_mask(q_pos: np.ndarray, k_pos: np.ndarray, sink: int, recent: int) -> np.ndarray:
    """M_streaming, the Lambda-shaped mask: a query sees only the first ``sink``
    tokens (attention sinks) and the ``recent`` most recent tokens, itself
    included, and never a future token."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    qi = q_pos[:, None]
    kj = k_pos[None, :]
    return (kj <= qi) & ((kj < sink) | (qi - kj < recent))


def chunk_streaming_mask(q_pos: np.ndarray, k_pos: np.ndarray, c0: int, sink: int, recent: int) -> np.ndarray:
    """A streaming head's mask in whole-chunk pre-fill: queries of the chunk
    that starts at ``c0`` see the sinks, the ``recent`` tokens before the
    chunk, and every chunk token up to themselves [Summary S2 "Chunked
    Pre-filling"; Review S5 "Pre-filling performance"]."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    qi = q_pos[:, None]
    kj = k_pos[None, :]
    return (kj <= qi) & ((kj < sink) | (kj >= c0 - recent))


# ---------------------------------------------------------------------------
# Attention with an explicit mask [Review S3 "Core formula"]
# ---------------------------------------------------------------------------

def masked_softmax(scores: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Row softmax of ``scores`` with -inf wherever ``mask`` is False.

    Every row must have at least one visible key.  Masked entries get
    probability exactly 0.
    """
    s = np.where(mask, scores, -np.inf)
    if not np.all(mask.any(axis=-1)):
        raise ValueError("a query row has no visible key")
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def masked_attention(q, k, v, mask, scale: float) -> np.ndarray:
    """softmax(scale * q k^T, masked) v for one head.

    q: [n, d], k: [m, d], v: [m, dv], mask: bool [n, m]; returns float64 [n, dv].
    """
    q = as_f64(q)
    k = as_f64(k)
    v = as_f64(v)
    p = masked_softmax(scale * (q @ k.T), np.asarray(mask, dtype=bool))
    return p @ v


def _default_scale(d: int, scale) -> float:
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def full_attn(q, k, v, scale=None) -> np.ndarray:
    """full_attn = softmax(Q K^T (.) M_causal) V over one head's whole sequence
    (positions 0..N-1 for both queries and keys)."""
    n = np.asarray(q).shape[0]
    pos = np.arange(n)
    return masked_attention(q, k, v, causal_mask(pos, pos), _default_scale(np.asarray(q).shape[1], scale))


def streaming_attn(q, k, v, sink: int, recent: int, scale=None) -> np.ndarray:
    """streaming_attn = softmax(Q K^T (.) M_streaming) V over one head's whole sequence."""
    n = np.asarray(q).shape[0]
    pos = np.arange(n)
    return masked_attention(q, k, v, streaming_mask(pos, pos, sink, recent),
                            _default_scale(np.asarray(q).shape[1], scale))


def gated_mix(q, k, v, alpha, sink: int, recent: int, scale=None) -> np.ndarray:
    """attn = alpha * full_attn + (1 - alpha) * streaming_attn, per head.

    q: [N, Hq, d]; k, v: [N, Hkv, d]; alpha: [Hkv] (one gate per KV head, shared
    by the G = Hq / Hkv query heads of its group [Summary S2
    "Optimization-based Identification"]).  Returns float64 [N, Hq, d].
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    alpha = np.asarray(alpha, dtype=np.float64)
    n, hq, d = q.shape
    hkv = k.shape[1]
    if hq % hkv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    g = hq // hkv
    out = np.empty((n, hq, v.shape[2]), dtype=np.float64)
    for h in range(hq):
        kv = h // g
        a = alpha[kv]
        fa = full_attn(q[:, h], k[:, kv], v[:, kv], scale)
        sa = streaming_attn(q[:, h], k[:, kv], v[:, kv], sink, recent, scale)
        out[:, h] = a * fa + (1.0 - a) * sa
    return out


def gated_mix_grad_alpha(q, k, v, dout, sink: int, recent: int, scale=None) -> np.ndarray:
    """Gradient of a loss with respect to the gates, given the gradient dout
    [N, Hq, d] of the gated-mix output.  The mix is linear in alpha, with
    d attn / d alpha = full_attn - streaming_attn for every query head of the
    gate's KV head [Review S3 "Core formula"; S3 "Retrieval-head
    identification": the gates are the only trained parameters], so

        dalpha[kv] = sum over the group's query heads h, rows i and features
                     of dout[i, h] * (full_attn[i, h] - streaming_attn[i, h]).

    Returns float64 [Hkv]."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    dout = as_f64(dout)
    n, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    grad = np.zeros(hkv, dtype=np.float64)
    for h in range(hq):
        kv = h // g
        fa = full_attn(q[:, h], k[:, kv], v[:, kv], scale)
        sa = streaming_attn(q[:, h], k[:, kv], v[:, kv], sink, recent, scale)
        grad[kv] += float(np.sum(dout[:, h] * (fa - sa)))
    return grad


# ---------------------------------------------------------------------------
# Gate binarisation and head partition
# [Review S3 "Retrieval-head identification", "Deployment optimisation";
#  Summary S2 "Binarizing Attention Implementations"]
# ---------------------------------------------------------------------------

def binarize_gates(alpha, tau: float) -> np.ndarray:
    """alpha_bin = 1[alpha >= tau] per KV head (uint8)."""
    return (np.asarray(alpha, dtype=np.float64) >= float(tau)).astype(np.uint8)


def partition_heads(alpha, tau: float, target_n_retrieval: int = -1):
    """Binary gates plus the reorder of KV heads into [retrieval | streaming].

    With ``target_n_retrieval < 0`` the gate is ``alpha >= tau``.  Otherwise the
    threshold is the quantile that keeps exactly ``target_n_retrieval`` heads:
    the heads with the largest alpha, ties going to the lower head index.

    Returns (gate uint8[Hkv], perm int32[Hkv], inv_perm int32[Hkv], n_retrieval)
    where ``perm[i]`` is the model KV head stored at block slot i (retrieval
    heads ascending, then streaming heads ascending) and ``inv_perm[perm[i]] = i``.
    """
    alpha = np.asarray(alpha, dtype=np.float64)
    hkv = alpha.shape[0]
    if target_n_retrieval is None or target_n_retrieval < 0:
        gate = binarize_gates(alpha, tau)
    else:
        if target_n_retrieval > hkv:
            raise ValueError("target_n_retrieval exceeds the number of KV heads")
        order = sorted(range(hkv), key=lambda h: (-alpha[h], h))
        gate = np.zeros(hkv, dtype=np.uint8)
        for h in order[:target_n_retrieval]:
            gate[h] = 1
    retrieval = [h for h in range(hkv) if gate[h]]
    streaming = [h for h in range(hkv) if not gate[h]]
    perm = np.array(retrieval + streaming, dtype=np.int32)
    inv_perm = np.empty(hkv, dtype=np.int32)
    for i, h in enumerate(perm):
        inv_perm[h] = i
    return gate, perm, inv_perm, len(retrieval)


# ---------------------------------------------------------------------------
# The two KV caches as explicit lists [Review S3 "Inference flow"]
# ---------------------------------------------------------------------------

def ring_slot(p: int, sink: int, recent: int) -> int:
    """Slot of absolute position p in a streaming head's sink+recent ring."""
    return p if p < sink else sink + (p - sink) % recent


# ---------------------------------------------------------------------------
# 8-bit retrieval cache [Review S5 "Decoding performance": combined with a
# quantized KV cache; Summary S3 results] -- scheme: see the module notes
# ---------------------------------------------------------------------------

def quantize_int8_rows(x) -> tuple:
    """Per-row symmetric int8 codes of x [n, d] (bf16 bits, float32 or
    float64 holding float32 values): returns (codes int8 [n, d], scales
    float32 [n]).  Every step is one float32 operation as written, so the
    codes are those any IEEE float32 implementation of the same steps gets."""
    x32 = as_f64(x).astype(np.float32)
    amax = np.abs(x32).max(axis=-1) if x32.shape[-1] else np.zeros(x32.shape[:-1], np.float32)
    nz = amax > 0
    inv = np.zeros_like(amax)
    inv[nz] = np.float32(127.0) / amax[nz]                      # float32 division
    q = np.rint(x32 * inv[..., None])                           # float32 product, round half to even
    codes = np.clip(q, -127, 127).astype(np.int8)
    scales = np.where(nz, amax / np.float32(127.0), np.float32(0)).astype(np.float32)
    return codes, scales


def dequantize_int8_rows(codes, scales) -> np.ndarray:
    """code * scale, exactly, in float64 [n, d]."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[:, None]


def quantize_int4_rows(x) -> tuple:
    """Per-row symmetric 4-bit codes of x [n, d] (bf16 bits, float32 or
    float64 holding float32 values): the 8-bit scheme's steps with 7 levels
    a side in place of 127 -- amax = max |x|, code = rint(x * (7 / amax)),
    scale = amax / 7, each one float32 operation as written; a zero row has
    scale 0 and codes 0.  Returns (codes int8 [n, d] in -7..7, scales
    float32 [n])."""
    x32 = as_f64(x).astype(np.float32)
    amax = np.abs(x32).max(axis=-1) if x32.shape[-1] else np.zeros(x32.shape[:-1], np.float32)
    nz = amax > 0
    inv = np.zeros_like(amax)
    inv[nz] = np.float32(7.0) / amax[nz]                        # float32 division
    q = np.rint(x32 * inv[..., None])                           # float32 product, round half to even
    codes = np.clip(q, -7, 7).astype(np.int8)
    scales = np.where(nz, amax / np.float32(7.0), np.float32(0)).astype(np.float32)
    return codes, scales


def _streaming_push(lst: list, entry: tuple, sink: int, recent: int) -> None:
    """Append one (position, ...) entry to a streaming head's list; when the
    list grows past sink + recent, evict the oldest token that is not an
    attention sink [Review S3 "Inference flow": a streaming head keeps only
    the sink tokens and the recent tokens]."""
    lst.append(entry)
    if len(lst) > sink + recent:
        for e in range(len(lst)):
            if lst[e][0] >= sink:
                del lst[e]
                break


def streaming_positions(length: int, sink: int, recent: int) -> np.ndarray:
    """Positions a streaming head's list holds after tokens 0..length-1 were
    appended one by one: the same pushes and evictions as
    ``HeadSplitCache.append``, on positions alone."""
    lst = []
    for p in range(int(length)):
        _streaming_push(lst, (p,), sink, recent)
    return np.array([e[0] for e in lst], dtype=np.int64)


@dataclass
class HeadSplitCache:
    """Per-layer caches for a batch: full lists for retrieval heads, a
    sink + recent list for streaming heads.

    Entries keep the caller's exact input rows (bf16 bit patterns or float32),
    so that layouts derived from the lists can be compared byte for byte.
    Heads are in model order; ``gate[h]`` is 1 for a retrieval KV head.
    """

    batch: int
    n_kv_heads: int
    head_dim: int
    gate: np.ndarray
    sink: int = 16
    recent: int = 64
    kv_int8: bool = False                # retrieval heads keep int8 codes + a scale per row
    kv_int4: bool = False                # retrieval heads keep 4-bit codes + a scale per row
    length: list = field(default=None)
    full: list = field(default=None)     # full[b][h] -> list of (pos int64[n], k[n, d], v[n, d]
                                         #   [, k codes, k scales, v codes, v scales] when kv_int8)
    stream: list = field(default=None)   # stream[b][h] -> list of (pos, k[d], v[d]) per token

    def __post_init__(self):
        self.gate = np.asarray(self.gate, dtype=np.uint8)
        assert self.gate.shape == (self.n_kv_heads,)
        self.length = [0] * self.batch
        self.full = [[[] for _ in range(self.n_kv_heads)] for _ in range(self.batch)]
        self.stream = [[[] for _ in range(self.n_kv_heads)] for _ in range(self.batch)]

    # -- updates ----------------------------------------------------------

    def append(self, k_new, v_new) -> None:
        """Append T tokens per sequence.  k_new, v_new: [B, T, Hkv, d] (model head order)."""
        k_new = np.asarray(k_new)
        v_new = np.asarray(v_new)
        b_, t, hkv, d = k_new.shape
        assert (b_, hkv, d) == (self.batch, self.n_kv_heads, self.head_dim)
        for b in range(self.batch):
            p0 = self.length[b]
            pos = np.arange(p0, p0 + t, dtype=np.int64)
            for h in range(hkv):
                if self.gate[h]:
                    if t:
                        self.full[b][h].append(self._full_entry(pos, k_new[b, :, h], v_new[b, :, h]))
                else:
                    lst = self.stream[b][h]
                    for i in range(t):
                        _streaming_push(lst, (int(pos[i]), k_new[b, i, h].copy(), v_new[b, i, h].copy()),
                                        self.sink, self.recent)
            self.length[b] = p0 + t

    def load_state(self, b: int, h: int, pos, k, v) -> None:
        """Install a cache state directly: the rows of positions ``pos`` for head h
        (all positions < length for a retrieval head; the surviving sink + recent
        positions for a streaming head).  Used to start decode from a long
        context without replaying the prompt token by token."""
        pos = np.asarray(pos, dtype=np.int64)
        if self.gate[h]:
            self.full[b][h] = [self._full_entry(pos, np.asarray(k), np.asarray(v))] if len(pos) else []
        else:
            self.stream[b][h] = [(int(p), np.asarray(k)[i].copy(), np.asarray(v)[i].copy())
                                 for i, p in enumerate(pos)]

    def set_length(self, b: int, n: int) -> None:
        self.length[b] = int(n)

    def _full_entry(self, pos, k, v):
        """A retrieval-head list entry: the rows as given, or (kv_int8,
        kv_int4) their dequantized values followed by the codes and scales."""
        if not (self.kv_int8 or self.kv_int4):
            return (pos.copy(), k.copy(), v.copy())
        quantize = quantize_int8_rows if self.kv_int8 else quantize_int4_rows
        kc, ks = quantize(k)
        vc, vs = quantize(v)
        return (pos.copy(), dequantize_int8_rows(kc, ks), dequantize_int8_rows(vc, vs), kc, ks, vc, vs)

    def quantized(self, b: int, h: int):
        """A kv_int8 / kv_int4 retrieval head's (positions, K codes, K scales,
        V codes, V scales)."""
        assert (self.kv_int8 or self.kv_int4) and self.gate[h]
        ent = self.full[b][h]
        if not ent:
            z8, z32 = np.zeros((0, self.head_dim), np.int8), np.zeros(0, np.float32)
            return np.zeros(0, dtype=np.int64), z8, z32, z8, z32
        return tuple(np.concatenate([e[i] for e in ent]) for i in (0, 3, 4, 5, 6))

    # -- views ------------------------------------------------------------

    def rows(self, b: int, h: int):
        """(positions, K rows, V rows) that head h of sequence b holds, in list order."""
        if self.gate[h]:
            ent = self.full[b][h]
            if not ent:
                z = np.zeros((0, self.head_dim))
                return np.zeros(0, dtype=np.int64), z, z
            return (np.concatenate([e[0] for e in ent]),
                    np.concatenate([e[1] for e in ent]),
                    np.concatenate([e[2] for e in ent]))
        ent = self.stream[b][h]
        if not ent:
            z = np.zeros((0, self.head_dim))
            return np.zeros(0, dtype=np.int64), z, z
        return (np.array([e[0] for e in ent], dtype=np.int64),
                np.stack([e[1] for e in ent]), np.stack([e[2] for e in ent]))

    def ring_layout(self, b: int, h: int, dtype):
        """A streaming head's list laid out as the sink+recent ring:
        (K[W, d], V[W, d], pos int32[W]); empty slots are zero rows with pos -1."""
        assert not self.gate[h]
        w = self.sink + self.recent
        kr = np.zeros((w, self.head_dim), dtype=dtype)
        vr = np.zeros((w, self.head_dim), dtype=dtype)
        pos = np.full(w, -1, dtype=np.int32)
        for p, k, v in self.stream[b][h]:
            s = ring_slot(p, self.sink, self.recent)
            kr[s] = k
            vr[s] = v
            pos[s] = p
        return kr, vr, pos

    def full_layout(self, b: int, h: int, capacity: int, dtype):
        """A retrieval head's list laid out as rows 0..capacity-1 by position."""
        assert self.gate[h]
        out = np.zeros((capacity, self.head_dim), dtype=dtype)
        pos, k, _ = self.rows(b, h)
        out[pos] = k
        outv = np.zeros((capacity, self.head_dim), dtype=dtype)
        _, _, v = self.rows(b, h)
        outv[pos] = v
        return out, outv

    # -- attention ----------------------------------------------------------

    def _head_attention(self, b, h_kv, q_rows, q_pos, extra=None, scale=1.0, whole_chunk=False):
        """Attention of query rows (positions q_pos) against what head h_kv of
        sequence b holds, plus optional extra (pos, k, v) rows, under the head's
        mask (causal for retrieval heads, Lambda for streaming heads).  With
        ``whole_chunk`` a streaming head sees all it holds and the extra rows
        causally: its list is the cache as it stood before the chunk."""
        pos, k, v = self.rows(b, h_kv)
        k = as_f64(k) if len(pos) else np.zeros((0, self.head_dim))
        v = as_f64(v) if len(pos) else np.zeros((0, self.head_dim))
        if extra is not None:
            pos = np.concatenate([pos, extra[0]])
            k = np.concatenate([k, as_f64(extra[1])])
            v = np.concatenate([v, as_f64(extra[2])])
        if self.gate[h_kv] or whole_chunk:
            mask = causal_mask(q_pos, pos)
        else:
            mask = streaming_mask(q_pos, pos, self.sink, self.recent)
        return masked_attention(q_rows, k, v, mask, scale)

    def decode(self, q, k_new, v_new, scale=None) -> np.ndarray:
        """One decode step: append the new token's K/V, then every query head
        attends over its KV head's cache [Review S3 "Inference flow"].

        q: [B, Hq, d]; k_new, v_new: [B, Hkv, d].  Returns float64 [B, Hq, d]
        in model head order (the per-head results concatenated).
        """
        q = np.asarray(q)
        k_new = np.asarray(k_new)
        v_new = np.asarray(v_new)
        self.append(k_new[:, None], v_new[:, None])
        bsz, hq, d = q.shape
        g = hq // self.n_kv_heads
        sc = _default_scale(d, scale)
        out = np.empty((bsz, hq, d), dtype=np.float64)
        for b in range(bsz):
            p = self.length[b] - 1
            for kv in range(self.n_kv_heads):
                # the G query heads of this KV head as G independent query rows at position p
                rows = q[b, kv * g:(kv + 1) * g]
                out[b, kv * g:(kv + 1) * g] = self._head_attention(b, kv, rows, np.full(g, p), scale=sc)
        return out

    def prefill_chunk(self, q, k_chunk, v_chunk, scale=None, stream_mode: str = "lambda") -> np.ndarray:
        """Chunked pre-fill from the caches [Summary S2 "Chunked Pre-filling"].

        Each query of the chunk attends to what its head's cache held before the
        chunk plus the chunk's own tokens, under the head's mask; afterwards the
        chunk is appended to both caches.  q: [B, C, Hq, d]; k_chunk, v_chunk:
        [B, C, Hkv, d].  Returns float64 [B, C, Hq, d].  ``stream_mode="chunk"``:
        a streaming head attends to its whole list and the chunk causally.
        """
        q = np.asarray(q)
        k_chunk = np.asarray(k_chunk)
        v_chunk = np.asarray(v_chunk)
        bsz, c, hq, d = q.shape
        g = hq // self.n_kv_heads
        sc = _default_scale(d, scale)
        out = np.empty((bsz, c, hq, d), dtype=np.float64)
        for b in range(bsz):
            p0 = self.length[b]
            qpos = np.arange(p0, p0 + c, dtype=np.int64)
            for h in range(hq):
                kv = h // g
                extra = (qpos, k_chunk[b, :, kv], v_chunk[b, :, kv])
                out[b, :, h] = self._head_attention(b, kv, q[b, :, h], qpos, extra, sc,
                                                    whole_chunk=stream_mode == "chunk")
        self.append(k_chunk, v_chunk)
        return out


# ---------------------------------------------------------------------------
# Direct definitions (no cache): used to check the cache-driven paths
# ---------------------------------------------------------------------------

def prefill_direct(q_chunk, k_all, v_all, c0: int, gate, sink: int, recent: int,
                   scale=None, rows=None, row_block: int = 64, stream_mode: str = "lambda") -> np.ndarray:
    """Chunk queries at positions c0 .. c0+C-1 attend to the whole token history
    k_all/v_all [N, Hkv, d] (N >= c0 + C) through the head's mask: causal for a
    retrieval head, Lambda for a streaming head.

    q_chunk: [C, Hq, d].  ``rows`` optionally selects chunk rows (sampling).
    ``stream_mode="chunk"`` gives streaming heads the whole-chunk mask.
    Rows are independent, so they are processed ``row_block`` at a time to bound
    memory; each row's arithmetic is the plain masked softmax above.
    Returns float64 [len(rows), Hq, d].
    """
    q_chunk = np.asarray(q_chunk)
    c, hq, d = q_chunk.shape
    gate = np.asarray(gate)
    hkv = gate.shape[0]
    g = hq // hkv
    sc = _default_scale(d, scale)
    rows = np.arange(c) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), hq, d), dtype=np.float64)
    for r0 in range(0, len(rows), row_block):
        rr = rows[r0:r0 + row_block]
        qpos = c0 + rr
        last = int(qpos.max()) + 1          # keys beyond the last query are masked anyway
        kpos = np.arange(last, dtype=np.int64)
        for kv in range(hkv):
            if gate[kv]:
                mask = causal_mask(qpos, kpos)
            elif stream_mode == "chunk":
                mask = chunk_streaming_mask(qpos, kpos, c0, sink, recent)
            else:
                mask = streaming_mask(qpos, kpos, sink, recent)
            kk = as_f64(k_all[:last, kv])
            vv = as_f64(v_all[:last, kv])
            for gi in range(g):
                h = kv * g + gi
                out[r0:r0 + len(rr), h] = masked_attention(q_chunk[rr, h], kk, vv, mask, sc)
    return out


def decode_direct(q, k_all, v_all, gate, sink: int, recent: int, scale=None) -> np.ndarray:
    """The decode output at position p = N-1 computed directly from the whole
    history k_all/v_all [N, Hkv, d]: row p of the head's mask.  q: [Hq, d]."""
    q = np.asarray(q)
    n = np.asarray(k_all).shape[0]
    return prefill_direct(q[None], k_all, v_all, n - 1, gate, sink, recent, scale)[0]
