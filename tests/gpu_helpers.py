"""Shared plumbing for the GPU parity tests: moving seeded inputs to the device
in the layouts include/duo.h documents, reading results back, and the
tolerances (bf16 inputs with fp32 accumulation: max-abs 2e-2 and mean-abs
2e-3; fp32 inputs: max-abs 1e-4)."""

from __future__ import annotations

import numpy as np

import oracle as O
from head_split_kv_b200 import synthetic as S

BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS = 2e-2, 2e-3, 1e-4


def torch():
    import torch as t
    return t


def to_dev(a: np.ndarray):
    """uint16 bf16 bits -> torch.bfloat16; float32 -> torch.float32; on cuda."""
    t = torch()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return t.from_numpy(a.view(np.int16)).view(t.bfloat16).cuda()
    return t.from_numpy(a).cuda()


def bits(x) -> np.ndarray:
    """Device tensor -> numpy with the exact bytes (bf16 as uint16 bits)."""
    t = torch()
    x = x.detach().contiguous().cpu()
    if x.dtype == t.bfloat16:
        return x.view(t.int16).numpy().view(np.uint16)
    return x.numpy()


def f64(x) -> np.ndarray:
    return O.as_f64(bits(x))


def assert_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str = "") -> dict:
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(want, dtype=np.float64))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    if dtype == "bf16":
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    else:
        assert mx <= FP32_MAX_ABS, f"{what}: max {mx:.3e}"
    return dict(max_abs=mx, mean_abs=mean)


# The 4-bit cache's byte layouts, as include/duo.h states them (codes -7..7
# stored as the nibble code + 8, the first of a byte's pair in its low half).

def q4_k_rows(codes: np.ndarray) -> np.ndarray:
    """K codes [n, 128] -> the cache's rows [n, 64] bytes: byte 16q + 4j + c
    holds, with e = 32q + 8j, features (e, e+2), (e+4, e+6), (e+1, e+3),
    (e+5, e+7) for c = 0..3."""
    nib = (codes.astype(np.int16) + 8).astype(np.uint8)
    out = np.zeros((codes.shape[0], 64), dtype=np.uint8)
    for q in range(4):
        for j in range(4):
            e, o = 32 * q + 8 * j, 16 * q + 4 * j
            for c, (lo, hi) in enumerate([(0, 2), (4, 6), (1, 3), (5, 7)]):
                out[:, o + c] = nib[:, e + lo] | (nib[:, e + hi] << 4)
    return out


def q4_v_gather(tiles: np.ndarray, n: int) -> np.ndarray:
    """The V cache's tiles [n_tiles, 4096] bytes -> codes [n, 128] of tokens
    0..n-1: token t of 16-token group g, key quad k = (t % 8) / 2, byte
    (t % 2) * 2 + t / 8 of the word at 1024g + 128m + 16r + 4k holds features
    16m + r (low nibble) and 16m + 8 + r (high nibble)."""
    p = np.arange(n)
    t = p % 64
    g, tt = t // 16, t % 16
    k, bw = (tt % 8) // 2, (tt % 2) * 2 + tt // 8
    m, r = np.arange(8)[None, :, None], np.arange(8)[None, None, :]
    off = 1024 * g[:, None, None] + 128 * m + 16 * r + 4 * k[:, None, None] + bw[:, None, None]   # [n, 8, 8]
    byte = tiles[(p // 64)[:, None, None], off].astype(np.int16)
    out = np.zeros((n, 128), dtype=np.int8)
    out[:, (16 * m + r).reshape(-1)] = ((byte & 15) - 8).reshape(n, -1)
    out[:, (16 * m + 8 + r).reshape(-1)] = ((byte >> 4) - 8).reshape(n, -1)
    return out


class Layer:
    """One attention layer on the device plus its oracle twin."""

    def __init__(self, duo, shape: S.LayerShape, retrieval, batch: int, capacity: int = 0, page_size: int = 0,
                 page_table=None, n_pages: int = 0, io_order=None, stream_prefill: int = 0, kv_quant: int = 0):
        self.duo = duo
        self.shape = shape
        self.B = batch
        hkv = shape.n_kv_heads
        alpha = S.binary_alpha(hkv, retrieval)
        self.gate, self.perm, self.inv, self.R = duo.partition_heads(alpha, 0.5)
        og, op, oi, on = O.partition_heads(alpha.astype(np.float64), 0.5)
        assert self.gate == list(og) and self.perm == list(op) and self.R == on
        self.io_order = duo.ORDER_MODEL if io_order is None else io_order
        self.stream_prefill = stream_prefill
        self.desc = duo.desc_init(batch, shape.n_q_heads, hkv, shape.head_dim,
                                  duo.BF16 if shape.dtype == "bf16" else duo.FP32, self.perm, self.R,
                                  sink=shape.sink, recent=shape.recent, page_size=page_size,
                                  io_order=self.io_order, stream_prefill=stream_prefill, kv_quant=kv_quant)
        self.kv_int8 = kv_quant == duo.KV_INT8
        self.kv_int4 = kv_quant == duo.KV_INT4
        self.page_table = None if page_table is None else np.asarray(page_table, dtype=np.int32)
        self.caches = duo.LayerCaches(self.desc, capacity, self.page_table, n_pages)
        self.oracle = O.HeadSplitCache(batch, hkv, shape.head_dim, gate=self.gate, sink=shape.sink,
                                       recent=shape.recent, kv_int8=self.kv_int8, kv_int4=self.kv_int4)
        self.ws = duo.Workspace(self.desc, duo.OP_DECODE, self.caches.capacity)

    # -- head order ----------------------------------------------------------
    def to_io(self, x: np.ndarray, axis: int, per_kv: int) -> np.ndarray:
        """Model head order -> the layer's io order along `axis` (blocks of per_kv heads)."""
        if self.io_order == self.duo.ORDER_MODEL:
            return x
        idx = np.concatenate([np.arange(h * per_kv, (h + 1) * per_kv) for h in self.perm])
        return np.take(x, idx, axis=axis)

    def from_io(self, x: np.ndarray, axis: int, per_kv: int) -> np.ndarray:
        if self.io_order == self.duo.ORDER_MODEL:
            return x
        idx = np.concatenate([np.arange(self.inv[h] * per_kv, (self.inv[h] + 1) * per_kv)
                              for h in range(self.shape.n_kv_heads)])
        return np.take(x, idx, axis=axis)

    # -- state ----------------------------------------------------------------
    def load_state(self, st) -> None:
        """Install a synthetic.DecodeState on the device and in the oracle.
        Retrieval heads hold every row of the prompt; a streaming head holds
        the positions the oracle's eviction rule keeps after the prompt
        (replayed on positions alone), with their seeded rows, placed in the
        ring slots by the oracle's slot function."""
        t = torch()
        c = self.caches
        sh = self.shape
        ring_pos = np.full((self.B, sh.sink + sh.recent), -1, dtype=np.int32)
        for (b, h), (k, v) in st.full.items():
            r = self.inv[h]
            L = k.shape[0]
            if self.page_table is None:
                c.k_full[b, r, :L] = to_dev(k)
                c.v_full[b, r, :L] = to_dev(v)
            else:
                pos = np.arange(L)
                pages = t.from_numpy(self.page_table[b, pos // 64].astype(np.int64)).cuda()
                rows = t.from_numpy(pos % 64).cuda()
                c.k_full[pages, r, rows] = to_dev(k)
                c.v_full[pages, r, rows] = to_dev(v)
            self.oracle.load_state(b, h, np.arange(L), k, v)
        kept = {}
        for b, L in enumerate(st.lengths):
            L = int(L)
            if L not in kept:
                kept[L] = O.streaming_positions(L, sh.sink, sh.recent)
            pos = kept[L]
            slots = np.array([O.ring_slot(int(p), sh.sink, sh.recent) for p in pos], dtype=np.int64)
            for h in range(sh.n_kv_heads):
                if self.gate[h]:
                    continue
                k, v = st.stream_rows(b, h, pos)
                s = self.inv[h] - self.R
                if len(slots):
                    idx = t.from_numpy(slots).cuda()
                    c.k_ring[b, s, idx] = to_dev(k)
                    c.v_ring[b, s, idx] = to_dev(v)
                    ring_pos[b, slots] = pos
                self.oracle.load_state(b, h, pos, k, v)
        c.ring_pos.copy_(t.from_numpy(ring_pos))
        c.seq_len.copy_(t.from_numpy(st.lengths.astype(np.int32)))
        for b, L in enumerate(st.lengths):
            self.oracle.set_length(b, int(L))

    # -- calls ------------------------------------------------------------------
    def append(self, k: np.ndarray, v: np.ndarray) -> None:
        """k, v [B, T, Hkv, d] in model order."""
        T = k.shape[1]
        kd = to_dev(self.to_io(k, 2, 1))
        vd = to_dev(self.to_io(v, 2, 1))
        self.duo.append_kv(self.desc, self.caches.state, kd, vd, T)
        self.oracle.append(k, v)

    def decode(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, check_oracle: bool = True, fused: bool = False):
        """One step: q [B, Hq, d], k/v [B, Hkv, d] (model order).  Returns (gpu, oracle).
        fused: duo_decode_step instead of duo_append_kv + duo_decode_attn."""
        t = torch()
        g = self.shape.group
        kd = to_dev(self.to_io(k[:, None], 2, 1))
        vd = to_dev(self.to_io(v[:, None], 2, 1))
        qd = to_dev(self.to_io(q, 1, g))
        out = t.empty_like(qd)
        if fused:
            self.duo.decode_step(self.desc, self.caches.state, qd, kd, vd, out, self.ws.ptr, self.ws.nbytes)
        else:
            self.duo.append_kv(self.desc, self.caches.state, kd, vd, 1)
            self.duo.decode_attn(self.desc, self.caches.state, qd, out, self.ws.ptr, self.ws.nbytes)
        got = self.from_io(f64(out), 1, g)
        if check_oracle:
            want = self.oracle.decode(q, k, v)
        else:
            self.oracle.append(k[:, None], v[:, None])
            want = None
        return got, want

    def status(self) -> int:
        return self.duo.check_status(self.caches.state)

    # -- bit-exact cache comparison --------------------------------------------
    def assert_caches_match(self, upto=None) -> None:
        sh = self.shape
        dt = np.uint16 if sh.dtype == "bf16" else np.float32
        c = self.caches
        seq = bits(c.seq_len)
        assert list(seq) == list(self.oracle.length), (list(seq), self.oracle.length)
        kf, vf = (bits(c.k_full), bits(c.v_full)) if self.R else (None, None)
        kr, vr, rp = bits(c.k_ring), bits(c.v_ring), bits(c.ring_pos)
        for b in range(self.B):
            L = self.oracle.length[b]
            for h in range(sh.n_kv_heads):
                slot = self.inv[h]
                if self.gate[h] and self.kv_int4:
                    pos, kc, ks, vc, vs = self.oracle.quantized(b, h)
                    assert np.array_equal(pos, np.arange(L))
                    assert np.array_equal(bits(c.k_full)[b, slot, :L], q4_k_rows(kc)), f"4-bit K codes b={b} h={h}"
                    tiles = bits(c.v_full)[b, slot]
                    assert np.array_equal(q4_v_gather(tiles, L), vc), f"4-bit V codes b={b} h={h}"
                    assert np.array_equal(bits(c.k_scale)[b, slot, :L], ks), f"K scales b={b} h={h}"
                    assert np.array_equal(bits(c.v_scale)[b, slot, :L], vs), f"V scales b={b} h={h}"
                elif self.gate[h] and self.kv_int8:
                    # 8-bit layout: K codes a row per token; V codes per 64-token
                    # tile, transposed, tokens of a 16-group in the order
                    # 0 1 8 9 2 3 10 11 4 5 12 13 6 7 14 15
                    pos, kc, ks, vc, vs = self.oracle.quantized(b, h)
                    assert np.array_equal(pos, np.arange(L))
                    k8 = bits(c.k_full)[b, slot, :L]
                    v8 = bits(c.v_full)[b, slot]
                    order = [0, 1, 8, 9, 2, 3, 10, 11, 4, 5, 12, 13, 6, 7, 14, 15]
                    where = np.argsort(order)                          # token -> position in its group
                    col = (pos % 64) // 16 * 16 + where[pos % 16]
                    got_v = v8[pos // 64, :, col]                      # [L, d]
                    assert np.array_equal(k8, kc), f"8-bit K codes b={b} h={h}"
                    assert np.array_equal(got_v, vc), f"8-bit V codes b={b} h={h}"
                    assert np.array_equal(bits(c.k_scale)[b, slot, :L], ks), f"K scales b={b} h={h}"
                    assert np.array_equal(bits(c.v_scale)[b, slot, :L], vs), f"V scales b={b} h={h}"
                elif self.gate[h]:
                    pos, ko, vo = self.oracle.rows(b, h)
                    if self.page_table is None:
                        gk, gv = kf[b, slot, pos], vf[b, slot, pos]
                    else:
                        pages = self.page_table[b, pos // 64]
                        gk, gv = kf[pages, slot, pos % 64], vf[pages, slot, pos % 64]
                    assert np.array_equal(gk, ko) and np.array_equal(gv, vo), f"full cache b={b} h={h}"
                    assert np.array_equal(pos, np.arange(L))
                else:
                    ko, vo, po = self.oracle.ring_layout(b, h, dt)
                    s = slot - self.R
                    assert np.array_equal(rp[b], po), f"ring_pos b={b}: {rp[b]} vs {po}"
                    valid = po >= 0
                    assert np.array_equal(kr[b, s][valid], ko[valid]), f"ring K b={b} h={h}"
                    assert np.array_equal(vr[b, s][valid], vo[valid]), f"ring V b={b} h={h}"


def prefill_run(lay, chunks, seed, sigma=None, rows_per_chunk=None):
    """Pre-fill a prompt chunk by chunk through duo_prefill_chunk (with the
    layer's pre-fill workspace) and duo_append_kv.  Each chunk's output rows
    (all, or rows_per_chunk seeded ones) are compared with the oracle's
    direct definition over the history its caches hold before the chunk
    (for an 8- or 4-bit layer the retrieval rows as code * scale; a
    streaming head's evicted positions as zeros, which no query of the chunk
    sees) followed by the chunk's rows as given, through the layer's
    streaming pre-fill mode; tensors go to the device in the layer's head
    order.  The oracle's caches then take the chunk."""
    t = torch()
    duo, sh, B = lay.duo, lay.shape, lay.B
    n = sum(chunks)
    q, k, v = S.prompt(sh, n, seed=seed, batch=B, sigma=sigma)
    ws = duo.Workspace(lay.desc, duo.OP_PREFILL, max(chunks), state=lay.caches.state)
    rng = S.rng_for(seed, 79)
    c0 = 0
    g = sh.group
    mode = "chunk" if lay.stream_prefill == duo.STREAM_CHUNK else "lambda"
    for ci, C in enumerate(chunks):
        sl = slice(c0, c0 + C)
        qd = to_dev(np.ascontiguousarray(lay.to_io(q[:, sl], 2, g)))
        kd, vd = (to_dev(np.ascontiguousarray(lay.to_io(x[:, sl], 2, 1))) for x in (k, v))
        out = t.empty_like(qd)
        duo.prefill_chunk(lay.desc, lay.caches.state, qd, kd, vd, C, out, ws.ptr, ws.nbytes)
        duo.append_kv(lay.desc, lay.caches.state, kd, vd, C)
        rows = np.arange(C) if rows_per_chunk is None or C <= rows_per_chunk else \
            np.unique(rng.choice(C, rows_per_chunk, replace=False))
        got = lay.from_io(f64(out), 2, g)
        for b in range(B):
            k_all = np.zeros((c0 + C, sh.n_kv_heads, sh.head_dim))
            v_all = np.zeros_like(k_all)
            for h in range(sh.n_kv_heads):
                pos, kh, vh = lay.oracle.rows(b, h)
                if len(pos):
                    k_all[pos, h], v_all[pos, h] = O.as_f64(kh), O.as_f64(vh)
            k_all[c0:], v_all[c0:] = O.as_f64(k[b, sl]), O.as_f64(v[b, sl])
            want = O.prefill_direct(q[b, sl], k_all, v_all, c0, np.array(lay.gate), sh.sink, sh.recent, rows=rows,
                                    stream_mode=mode)
            assert_close(got[b, rows], want, sh.dtype, f"chunk {ci} (c0={c0}) b={b}")
        lay.oracle.append(k[:, sl], v[:, sl])
        c0 += C
    assert lay.status() == 0
