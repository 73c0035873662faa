"""The algorithmic work counts behind bench.py's roofline numbers, pinned to
brute-force counts over the oracle's own masks and caches (CPU only).

bench.py reports achieved GB/s and TFLOP/s as algorithmic bytes or FLOPs
divided by measured time; a wrong count would misstate every fraction of
peak.  Each closed-form count here is checked against an explicit
enumeration: visible (query, key) pairs from the boolean masks of the
oracle, and cache rows from the oracle's per-head cache lists."""

import numpy as np
import pytest

import bench
import oracle as O
from head_split_kv_b200 import synthetic as S


def _pairs(mask_fn, q_pos, n_keys, *args):
    return int(mask_fn(q_pos, np.arange(n_keys), *args).sum())


@pytest.mark.parametrize("p0,n,sink,recent", [(0, 1, 16, 64), (0, 100, 16, 64), (5, 40, 16, 64), (300, 257, 16, 64),
                                              (0, 70, 4, 8), (17, 3, 2, 3), (1000, 1, 16, 64)])
def test_lambda_pairs_count_the_streaming_mask(p0, n, sink, recent):
    q = np.arange(p0, p0 + n)
    assert bench._lambda_pairs(p0, n, sink, recent) == _pairs(O.streaming_mask, q, p0 + n, sink, recent)


@pytest.mark.parametrize("chunk_mode", [False, True])
@pytest.mark.parametrize("c0,C", [(0, 256), (0, 1), (50, 70), (4096, 300), (128, 4096)])
def test_prefill_flops_count_the_visible_pairs(c0, C, chunk_mode):
    d, n_ret_q, n_str_q, sink, recent = 128, 12, 20, 16, 64
    q = np.arange(c0, c0 + C)
    causal = _pairs(O.causal_mask, q, c0 + C)
    if chunk_mode:
        stream = _pairs(O.chunk_streaming_mask, q, c0 + C, c0, sink, recent)
    else:
        stream = _pairs(O.streaming_mask, q, c0 + C, sink, recent)
    want = 4 * d * (n_ret_q * causal + n_str_q * stream)
    assert bench._prefill_flops(n_ret_q, n_str_q, d, c0, C, sink, recent, chunk_mode) == want


@pytest.mark.parametrize("n,B", [(512, 1), (97, 3), (4096, 1)])
def test_mix_flops_count_both_masks(n, B):
    hq, d, sink, recent = 8, 64, 16, 64
    q = np.arange(n)
    causal = _pairs(O.causal_mask, q, n)
    lam = _pairs(O.streaming_mask, q, n, sink, recent)
    assert bench._mix_flops(hq, d, n, sink, recent, B) == B * hq * (4 * d * causal + 2 * d * lam)


def _rows(cache, b, h):
    """Cached rows of one (sequence, KV head) in the oracle's lists."""
    if cache.gate[h]:
        return sum(len(e[0]) for e in cache.full[b][h])
    return len(cache.stream[b][h])


@pytest.mark.parametrize("kv_bits", [0, 8, 4])
def test_decode_bytes_count_the_cached_rows(kv_bits):
    """One fused decode step (append, then attend) after prompts of several
    lengths: every row the oracle's caches hold after the append except the
    new one is read once (a retrieval row as bf16 K and V, or d codes + a
    4-byte scale each), the new token's K/V rows are read from the inputs and
    written into the caches, q is read and out written."""
    sh = S.LayerShape(8, 4, 16, "bf16", sink=2, recent=3)
    gate = np.array([1, 0, 1, 0])
    R = int(gate.sum())
    lengths = [0, 1, 4, 5, 6, 30]
    B = len(lengths)
    cache = O.HeadSplitCache(B, sh.n_kv_heads, sh.head_dim, gate=gate, sink=sh.sink, recent=sh.recent)
    rng = np.random.default_rng(3)
    # each sequence's lists come from a one-sequence oracle cache filled token
    # by token: its prompt, then the decode step's token
    for b, L in enumerate(lengths):
        one = O.HeadSplitCache(1, sh.n_kv_heads, sh.head_dim, gate=gate, sink=sh.sink, recent=sh.recent)
        for _ in range(L + 1):
            kv = rng.standard_normal((1, 1, sh.n_kv_heads, sh.head_dim)).astype(np.float32)
            one.append(kv, kv)
        for h in range(sh.n_kv_heads):
            cache.full[b][h], cache.stream[b][h] = one.full[0][h], one.stream[0][h]
        cache.set_length(b, L + 1)
    row = sh.head_dim * 2
    full_row = {0: row, 8: sh.head_dim + 4, 4: sh.head_dim // 2 + 4}[kv_bits]
    want = 0
    for b in range(B):
        for h in range(sh.n_kv_heads):
            want += (_rows(cache, b, h) - 1) * (full_row if gate[h] else row) * 2
        want += sh.n_kv_heads * row * 2 * 2
        want += sh.n_q_heads * sh.head_dim * 2 * 2
    assert bench._decode_bytes(sh, R, [L + 1 for L in lengths], kv_bits) == want


def test_traffic_record_is_used_only_while_its_sources_are_unchanged(tmp_path, monkeypatch):
    """roofline.traffic comes from profiles/traffic.json ({kernel: {workload:
    record}}) only while every source file the record lists still has the
    recorded SHA-256; a changed kernel reports null until it is captured
    again."""
    import hashlib
    import json
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"dram_bytes_read": 1000, "dram_bytes_write": 24,
           "source_sha256": {"k.cu": hashlib.sha256(src.read_bytes()).hexdigest()}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"kern": {"wl": rec}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("kern", "wl") == 1024
    assert bench._traffic("kern", "other workload") is None
    assert bench._traffic("other kernel", "wl") is None
    src.write_text("kernel v2\n")
    assert bench._traffic("kern", "wl") is None
