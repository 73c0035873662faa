"""Pins for the CPU oracle: facts the pages and the mathematics fix.

Every check here is independent of the oracle's own code path: hand-drawn
fixtures (tests/golden), closed forms, brute-force loops, a library special
case (torch SDPA on CPU), and invariants the pages state.  Sources are cited
by page and section:

[Review]  DuoAttention paper review (xllm-io.github.io): S3 "Core formula",
          "Retrieval-head identification", "Inference flow", "Deployment
          optimisation"; S5 "Ablations" item 3.
[Summary] paperlayer.ai summary of arXiv:2410.10819v1, S2 bullets.
"""

import math

import numpy as np
import pytest

import oracle as O
from head_split_kv_b200 import synthetic as S


def _mask_from_lines(lines):
    return np.array([[c == "1" for c in ln] for ln in lines], dtype=bool)


# ---------------------------------------------------------------------------
# Masks against hand-drawn fixtures [Review S3 "Core formula"]
# ---------------------------------------------------------------------------

def test_lambda_mask_matches_hand_drawn(golden):
    params, lines = golden("lambda_mask_n10_s2_r3.txt")
    want = _mask_from_lines(lines)
    pos = np.arange(want.shape[0])
    got = O.streaming_mask(pos, pos, int(params["sink"]), int(params["recent"]))
    assert got.shape == want.shape
    assert np.array_equal(got, want)


def test_causal_mask_matches_hand_drawn(golden):
    _, lines = golden("causal_mask_n5.txt")
    want = _mask_from_lines(lines)
    pos = np.arange(want.shape[0])
    assert np.array_equal(O.causal_mask(pos, pos), want)


def test_lambda_mask_reduces_to_causal_when_window_covers_sequence():
    # [Review S3 "Core formula"]: with sink + recent >= N nothing is dropped
    for n, s, r in [(8, 2, 6), (12, 0, 12), (80, 16, 64), (30, 16, 64)]:
        pos = np.arange(n)
        assert np.array_equal(O.streaming_mask(pos, pos, s, r), O.causal_mask(pos, pos))


# ---------------------------------------------------------------------------
# Worked example by hand [Review S3 "Core formula"]
# ---------------------------------------------------------------------------

def test_worked_example_d1(golden):
    params, _ = golden("tiny_attention_d1.txt")
    q = np.ones((3, 1))
    k = np.array([[0.0], [math.log(2.0)], [math.log(3.0)]])
    v = np.array([[6.0], [0.0], [12.0]])
    full = O.full_attn(q, k, v, scale=1.0)[:, 0]
    stream = O.streaming_attn(q, k, v, sink=1, recent=1, scale=1.0)[:, 0]
    np.testing.assert_allclose(full, params["full"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(stream, params["streaming"], rtol=0, atol=1e-12)
    a = float(params["mix_alpha"])
    mix = O.gated_mix(q[:, None], k[:, None], v[:, None], [a], sink=1, recent=1, scale=1.0)[:, 0, 0]
    np.testing.assert_allclose(mix, params["mix"], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Brute force on tiny inputs: explicit loops, math.exp and math.fsum
# ---------------------------------------------------------------------------

def _brute_attention(q, k, v, visible, scale):
    n, d = q.shape
    m = k.shape[0]
    out = np.zeros((n, v.shape[1]))
    for i in range(n):
        js = [j for j in range(m) if visible(i, j)]
        sc = [scale * math.fsum(q[i, t] * k[j, t] for t in range(d)) for j in js]
        mx = max(sc)
        w = [math.exp(s - mx) for s in sc]
        z = math.fsum(w)
        for t in range(v.shape[1]):
            out[i, t] = math.fsum(w[a] * v[js[a], t] for a in range(len(js))) / z
    return out


@pytest.mark.parametrize("n,d,sink,recent,hq,hkv", [
    (12, 4, 2, 3, 2, 2), (11, 3, 1, 4, 4, 2), (9, 2, 3, 2, 3, 1), (12, 4, 0, 5, 1, 1)])
def test_brute_force_tiny(n, d, sink, recent, hq, hkv):
    rng = np.random.default_rng(n * 100 + d)
    q = rng.standard_normal((n, hq, d))
    k = rng.standard_normal((n, hkv, d))
    v = rng.standard_normal((n, hkv, d))
    alpha = rng.uniform(0, 1, hkv)
    scale = 1.0 / math.sqrt(d)
    g = hq // hkv
    got = O.gated_mix(q, k, v, alpha, sink, recent)
    for h in range(hq):
        kv = h // g
        f = _brute_attention(q[:, h], k[:, kv], v[:, kv], lambda i, j: j <= i, scale)
        s = _brute_attention(q[:, h], k[:, kv], v[:, kv],
                             lambda i, j: j <= i and (j < sink or i - j < recent), scale)
        np.testing.assert_allclose(got[:, h], alpha[kv] * f + (1 - alpha[kv]) * s, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Library special case: torch SDPA on CPU in float64 with a boolean mask
# ---------------------------------------------------------------------------

def test_matches_torch_sdpa_cpu_float64():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    n, d, sink, recent = 150, 16, 4, 20
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    pos = np.arange(n)
    for mask in (O.causal_mask(pos, pos), O.streaming_mask(pos, pos, sink, recent)):
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
            torch.from_numpy(v)[None, None], attn_mask=torch.from_numpy(mask)[None, None],
            scale=1.0 / math.sqrt(d))[0, 0].numpy()
        got = O.masked_attention(q, k, v, mask, 1.0 / math.sqrt(d))
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)


# ---------------------------------------------------------------------------
# Gated mix facts [Review S3 "Core formula", "Retrieval-head identification"]
# ---------------------------------------------------------------------------

def _rand_qkv(rng, n, hq, hkv, d):
    return rng.standard_normal((n, hq, d)), rng.standard_normal((n, hkv, d)), rng.standard_normal((n, hkv, d))


def test_alpha_one_is_full_causal_attention():
    rng = np.random.default_rng(1)
    q, k, v = _rand_qkv(rng, 100, 4, 2, 8)
    mix = O.gated_mix(q, k, v, [1.0, 1.0], 16, 64)
    for h in range(4):
        np.testing.assert_allclose(mix[:, h], O.full_attn(q[:, h], k[:, h // 2], v[:, h // 2]), atol=1e-12, rtol=0)


def test_alpha_zero_with_window_covering_sequence_is_full_attention():
    rng = np.random.default_rng(2)
    q, k, v = _rand_qkv(rng, 80, 2, 2, 8)
    mix = O.gated_mix(q, k, v, [0.0, 0.0], 16, 64)
    for h in range(2):
        np.testing.assert_allclose(mix[:, h], O.full_attn(q[:, h], k[:, h], v[:, h]), atol=1e-12, rtol=0)


def test_alpha_zero_long_sequence_differs_from_full():
    # beyond sink + recent the streaming arm really drops tokens
    rng = np.random.default_rng(3)
    q, k, v = _rand_qkv(rng, 120, 1, 1, 8)
    mix = O.gated_mix(q, k, v, [0.0], 16, 64)
    full = O.full_attn(q[:, 0], k[:, 0], v[:, 0])
    assert np.allclose(mix[:80, 0], full[:80], atol=1e-12)
    assert np.abs(mix[80:, 0] - full[80:]).max() > 1e-3


def test_mix_is_linear_in_alpha():
    rng = np.random.default_rng(4)
    q, k, v = _rand_qkv(rng, 130, 2, 1, 8)
    m1 = O.gated_mix(q, k, v, [1.0], 5, 17)
    m0 = O.gated_mix(q, k, v, [0.0], 5, 17)
    for a in (0.1, 0.5, 0.77):
        np.testing.assert_allclose(O.gated_mix(q, k, v, [a], 5, 17), a * m1 + (1 - a) * m0, atol=1e-12, rtol=0)


def test_softmax_rows_sum_to_one_and_masked_mass_is_zero():
    rng = np.random.default_rng(5)
    n = 90
    s = rng.standard_normal((n, n)) * 4
    pos = np.arange(n)
    for mask in (O.causal_mask(pos, pos), O.streaming_mask(pos, pos, 3, 10)):
        p = O.masked_softmax(s, mask)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12, rtol=0)
        assert np.all(p[~mask] == 0.0)
        assert np.all(p[mask] > 0.0)


# ---------------------------------------------------------------------------
# Textbook special cases
# ---------------------------------------------------------------------------

def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(6)
    q, k, v = _rand_qkv(rng, 5, 1, 1, 4)
    out = O.full_attn(q[:, 0], k[:, 0], v[:, 0])
    np.testing.assert_allclose(out[0], v[0, 0], atol=1e-15, rtol=0)
    # streaming with sink 0, recent 1: every query sees only itself
    out = O.streaming_attn(q[:, 0], k[:, 0], v[:, 0], 0, 1)
    np.testing.assert_allclose(out, v[:, 0], atol=1e-15, rtol=0)


def test_zero_query_gives_mean_of_visible_values():
    rng = np.random.default_rng(7)
    n, s, r = 40, 3, 7
    k = rng.standard_normal((n, 6))
    v = rng.standard_normal((n, 6))
    q = np.zeros((n, 6))
    out = O.streaming_attn(q, k, v, s, r)
    for i in range(n):
        vis = [j for j in range(i + 1) if j < s or i - j < r]
        np.testing.assert_allclose(out[i], v[vis].mean(axis=0), atol=1e-13, rtol=0)


def test_gqa_with_group_one_is_mha_and_groups_share_kv():
    rng = np.random.default_rng(8)
    q, k, v = _rand_qkv(rng, 50, 4, 4, 8)
    alpha = rng.uniform(0, 1, 4)
    mha = O.gated_mix(q, k, v, alpha, 3, 9)
    for h in range(4):
        one = O.gated_mix(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], alpha[h:h + 1], 3, 9)
        np.testing.assert_allclose(mha[:, h], one[:, 0], atol=1e-14, rtol=0)
    # G = 2: query heads 2, 3 use KV head 1 and its gate
    q2, k2, v2 = _rand_qkv(rng, 50, 4, 2, 8)
    a2 = np.array([0.3, 0.9])
    g2 = O.gated_mix(q2, k2, v2, a2, 3, 9)
    kx = np.repeat(k2, 2, axis=1)
    vx = np.repeat(v2, 2, axis=1)
    ax = np.repeat(a2, 2)
    np.testing.assert_allclose(g2, O.gated_mix(q2, kx, vx, ax, 3, 9), atol=1e-14, rtol=0)


def test_permute_attend_unpermute_is_attend():
    # [Review S3 "Deployment optimisation"]: reordering heads into contiguous
    # retrieval / streaming blocks does not change what each head computes
    rng = np.random.default_rng(9)
    hkv, g = 6, 2
    q, k, v = _rand_qkv(rng, 40, hkv * g, hkv, 8)
    alpha = np.array([0.9, 0.1, 0.95, 0.2, 0.3, 0.99])
    gate, perm, inv_perm, nret = O.partition_heads(alpha, 0.5)
    ref = O.gated_mix(q, k, v, gate.astype(float), 3, 9)
    qperm = np.concatenate([q[:, perm[i] * g:(perm[i] + 1) * g] for i in range(hkv)], axis=1)
    outp = O.gated_mix(qperm, k[:, perm], v[:, perm], gate[perm].astype(float), 3, 9)
    back = np.concatenate([outp[:, inv_perm[h] * g:(inv_perm[h] + 1) * g] for h in range(hkv)], axis=1)
    np.testing.assert_allclose(back, ref, atol=1e-14, rtol=0)


# ---------------------------------------------------------------------------
# Binarisation and partition [Review S3 "Retrieval-head identification";
# Summary S2 "Binarizing Attention Implementations"]
# ---------------------------------------------------------------------------

def test_binarize_uses_greater_or_equal():
    assert list(O.binarize_gates([0.5, 0.49999, 0.50001, 1.0, 0.0], 0.5)) == [1, 0, 1, 1, 0]


def test_partition_by_threshold():
    gate, perm, inv, n = O.partition_heads([0.1, 0.8, 0.5, 0.2, 0.9, 0.5], 0.5)
    assert list(gate) == [0, 1, 1, 0, 1, 1]
    assert list(perm) == [1, 2, 4, 5, 0, 3] and n == 4
    assert list(inv) == [4, 0, 1, 5, 2, 3]
    assert all(perm[inv[h]] == h for h in range(6))


def test_partition_top_k_ties_go_to_lower_index():
    gate, perm, inv, n = O.partition_heads([0.3, 0.7, 0.7, 0.1, 0.7], 0.0, target_n_retrieval=2)
    assert list(gate) == [0, 1, 1, 0, 0] and n == 2
    assert list(perm) == [1, 2, 0, 3, 4]
    gate, perm, _, n = O.partition_heads([0.3, 0.7, 0.7, 0.1, 0.7], 0.0, target_n_retrieval=0)
    assert n == 0 and list(perm) == [0, 1, 2, 3, 4]
    gate, perm, _, n = O.partition_heads([0.3, 0.7, 0.7, 0.1, 0.7], 0.0, target_n_retrieval=5)
    assert n == 5 and list(perm) == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------------------
# Caches [Review S3 "Inference flow"; Summary S2]
# ---------------------------------------------------------------------------

def test_ring_positions_match_hand_table(golden):
    params, lines = golden("ring_pos_s2_r3.txt")
    s, r = int(params["sink"]), int(params["recent"])
    c = O.HeadSplitCache(1, 1, 2, gate=[0], sink=s, recent=r)
    for ln in lines:
        vals = [int(x) for x in ln.split()]
        p, want = vals[0], vals[1:]
        x = np.full((1, 1, 1, 2), p, dtype=np.float32)
        c.append(x, x)
        assert c.length[0] == p + 1
        _, _, pos = c.ring_layout(0, 0, np.float32)
        assert list(pos) == want, (p, list(pos), want)


def test_ring_after_block_append_equals_token_by_token(golden):
    params, lines = golden("ring_pos_s2_r3.txt")
    s, r = int(params["sink"]), int(params["recent"])
    final = [int(x) for x in lines[-1].split()][1:]
    c = O.HeadSplitCache(1, 1, 2, gate=[0], sink=s, recent=r)
    for t0, t1 in [(0, 3), (3, 7), (7, 10)]:
        x = np.arange(t0, t1, dtype=np.float32).repeat(2).reshape(1, t1 - t0, 1, 2)
        c.append(x, x)
    kr, _, pos = c.ring_layout(0, 0, np.float32)
    assert list(pos) == final
    assert all(kr[i, 0] == pos[i] for i in range(len(pos)) if pos[i] >= 0)


@pytest.mark.parametrize("seed", range(4))
def test_streaming_cache_stays_constant_size(seed):
    rng = np.random.default_rng(seed)
    s, r = 16, 64
    c = O.HeadSplitCache(1, 2, 4, gate=[1, 0], sink=s, recent=r)
    L = 0
    for _ in range(25):
        t = int(rng.integers(0, 40))
        x = rng.standard_normal((1, t, 2, 4)).astype(np.float32)
        c.append(x, x)
        L += t
        pos, _, _ = c.rows(0, 1)
        assert len(pos) == min(L, s + r)
        assert set(pos.tolist()) == set(range(min(L, s))) | set(range(max(0, L - r), L))
        fpos, _, _ = c.rows(0, 0)
        assert fpos.tolist() == list(range(L))


def test_cache_rows_are_exact_copies():
    rng = np.random.default_rng(11)
    k = S.normal(rng, (1, 200, 3, 8), "bf16")
    v = S.normal(rng, (1, 200, 3, 8), "bf16")
    c = O.HeadSplitCache(1, 3, 8, gate=[1, 0, 1], sink=4, recent=10)
    c.append(k[:, :77], v[:, :77])
    c.append(k[:, 77:], v[:, 77:])
    fk, fv = c.full_layout(0, 2, 256, np.uint16)
    assert np.array_equal(fk[:200], k[0, :, 2]) and np.array_equal(fv[:200], v[0, :, 2])
    kr, vr, pos = c.ring_layout(0, 1, np.uint16)
    for slot, p in enumerate(pos):
        assert np.array_equal(kr[slot], k[0, p, 1]) and np.array_equal(vr[slot], v[0, p, 1])


# ---------------------------------------------------------------------------
# Cache-driven paths equal the direct mask definition (chunk invariance,
# decode == pre-fill row) [Summary S2 "Chunked Pre-filling"; Review S3
# "Inference flow"]
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [1, 7, 128, 300])
def test_chunked_prefill_from_caches_equals_direct(chunk):
    rng = np.random.default_rng(12)
    n, hq, hkv, d, s, r = 300, 4, 2, 8, 16, 64
    q, k, v = _rand_qkv(rng, n, hq, hkv, d)
    gate = np.array([1, 0], dtype=np.uint8)
    c = O.HeadSplitCache(1, hkv, d, gate=gate, sink=s, recent=r)
    outs = []
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        outs.append(c.prefill_chunk(q[None, c0:c1], k[None, c0:c1], v[None, c0:c1])[0])
    got = np.concatenate(outs)
    want = O.prefill_direct(q, k, v, 0, gate, s, r)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)
    # and the direct path equals the gated mix with binary alpha
    np.testing.assert_allclose(want, O.gated_mix(q, k, v, gate.astype(float), s, r), atol=1e-12, rtol=0)


def test_decode_after_prefill_equals_direct_row():
    rng = np.random.default_rng(13)
    n0, steps, hq, hkv, d, s, r = 100, 30, 4, 2, 8, 4, 12
    q, k, v = _rand_qkv(rng, n0 + steps, hq, hkv, d)
    gate = np.array([0, 1], dtype=np.uint8)
    c = O.HeadSplitCache(1, hkv, d, gate=gate, sink=s, recent=r)
    c.prefill_chunk(q[None, :n0], k[None, :n0], v[None, :n0])
    for i in range(steps):
        p = n0 + i
        got = c.decode(q[None, p], k[None, p], v[None, p])[0]
        want = O.decode_direct(q[p], k[:p + 1], v[:p + 1], gate, s, r)
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


def test_load_state_equals_replayed_prompt():
    """A state installed from the replayed positions equals the state the
    appends build, for a retrieval and a streaming head."""
    rng = np.random.default_rng(14)
    n0, hkv, d, s, r = 150, 2, 4, 3, 9
    k = rng.standard_normal((1, n0, hkv, d)).astype(np.float32)
    v = rng.standard_normal((1, n0, hkv, d)).astype(np.float32)
    gate = np.array([1, 0], dtype=np.uint8)
    a = O.HeadSplitCache(1, hkv, d, gate=gate, sink=s, recent=r)
    a.append(k, v)
    b = O.HeadSplitCache(1, hkv, d, gate=gate, sink=s, recent=r)
    b.load_state(0, 0, np.arange(n0), k[0, :, 0], v[0, :, 0])
    keep = O.streaming_positions(n0, s, r)
    b.load_state(0, 1, keep, k[0, keep, 1], v[0, keep, 1])
    b.set_length(0, n0)
    for h in range(hkv):
        pa, ka, va = a.rows(0, h)
        pb, kb, vb = b.rows(0, h)
        assert np.array_equal(pa, pb) and np.array_equal(ka, kb) and np.array_equal(va, vb)


@pytest.mark.parametrize("s,r", [(16, 64), (3, 9), (0, 5), (4, 1)])
def test_streaming_positions_are_the_sinks_and_the_recent_tokens(s, r):
    """After L single-token appends a streaming head holds exactly the first
    min(L, sink) positions and the last `recent` ones (the pages: sink and
    recent tokens only), for every L across the boundaries, and the list the
    appends build holds the same positions."""
    c = O.HeadSplitCache(1, 1, 1, gate=np.array([0], dtype=np.uint8), sink=s, recent=r)
    one = np.zeros((1, 1, 1, 1), dtype=np.float32)
    for L in range(0, 3 * (s + r) + 5):
        want = sorted(set(range(min(L, s))) | set(range(max(0, L - r), L)))
        got = O.streaming_positions(L, s, r)
        assert list(got) == want, (L, list(got), want)
        assert list(c.rows(0, 0)[0]) == want
        c.append(one, one)
    assert len(O.streaming_positions(1 << 16, s, r)) == s + r


def test_bf16_widening_is_exact():
    x = np.array([1.0, -2.5, 3.140625, 2.0 ** -100, 65280.0], dtype=np.float32)
    bits = S.to_bf16_bits(x)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), x.astype(np.float64))


# ---------------------------------------------------------------------------
# 8-bit retrieval cache (the build's reading of the pages' quantized KV cache)
# ---------------------------------------------------------------------------

def test_int8_codes_match_hand_worked_rows(golden):
    params, _ = golden("int8_rows.txt")
    for i in range(3):
        x = np.array([params[f"x{i}"]], dtype=np.float32)
        codes, scales = O.quantize_int8_rows(x)
        assert codes.dtype == np.int8 and scales.dtype == np.float32
        assert codes[0].tolist() == [int(c) for c in params[f"codes{i}"]], i
        assert scales[0] == np.float32(float(params[f"scale{i}"])), i


@pytest.mark.parametrize("seed", [0, 1])
def test_int8_round_trip_is_within_half_a_step(seed):
    rng = np.random.default_rng([seed, 91])
    d = 128
    # bf16-representable rows of very different magnitudes, some with a zero
    x = (rng.standard_normal((64, d)) * np.exp(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    x = (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    x[5] = 0.0
    x[7, :10] = 0.0
    codes, scales = O.quantize_int8_rows(x)
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    # the largest element of every nonzero row gets code +-127
    assert np.all(np.abs(codes[nz]).max(axis=1) == 127)
    assert np.all(scales[~nz] == 0) and np.all(codes[~nz] == 0)
    # each value is within half a step of its code
    err = np.abs(x.astype(np.float64) - O.dequantize_int8_rows(codes, scales))
    assert np.all(err <= scales.astype(np.float64)[:, None] * (0.5 + 1e-5))
    # signs are kept, and zeros stay zero
    assert np.all((codes == 0) | (np.sign(codes) == np.sign(x)))
    assert np.all(codes[x == 0] == 0)
    # codes of the reconstructed rows are the codes again
    again, _ = O.quantize_int8_rows(O.dequantize_int8_rows(codes, scales).astype(np.float32))
    assert np.array_equal(again, codes)


def test_int8_cache_decode_equals_direct_on_reconstructed_rows():
    """The 8-bit cache only changes what the retrieval heads' lists hold: a
    decode from it equals the direct mask definition over the history whose
    retrieval rows are replaced by code * scale."""
    sh = S.LayerShape(8, 4, 16, "bf16")
    gate = np.array([1, 0, 1, 0], dtype=np.uint8)
    n = 150
    q, k, v = S.prompt(sh, n, seed=4)
    c = O.HeadSplitCache(1, 4, 16, gate=gate, kv_int8=True)
    c.append(k[:, :n - 1], v[:, :n - 1])
    got = c.decode(q[:, n - 1], k[:, n - 1], v[:, n - 1])[0]
    k_hat, v_hat = O.as_f64(k[0]), O.as_f64(v[0])
    for h in (0, 2):
        kc, ks = O.quantize_int8_rows(k[0, :, h])
        vc, vs = O.quantize_int8_rows(v[0, :, h])
        k_hat[:, h] = O.dequantize_int8_rows(kc, ks)
        v_hat[:, h] = O.dequantize_int8_rows(vc, vs)
    want = O.decode_direct(q[0, n - 1], k_hat, v_hat, gate, 16, 64)
    assert np.max(np.abs(got - want)) < 1e-12
    pos, kc, ks, vc, vs = c.quantized(0, 2)
    assert np.array_equal(pos, np.arange(n)) and kc.shape == (n, 16) and ks.shape == (n,)


def test_int4_codes_match_hand_worked_rows(golden):
    params, _ = golden("int4_rows.txt")
    for i in range(4):
        x = np.array([params[f"x{i}"]], dtype=np.float32)
        codes, scales = O.quantize_int4_rows(x)
        assert codes.dtype == np.int8 and scales.dtype == np.float32
        assert codes[0].tolist() == [int(c) for c in params[f"codes{i}"]], i
        assert scales[0] == np.float32(float(params[f"scale{i}"])), i


@pytest.mark.parametrize("seed", [0, 1])
def test_int4_round_trip_is_within_half_a_step(seed):
    rng = np.random.default_rng([seed, 92])
    d = 128
    x = (rng.standard_normal((64, d)) * np.exp(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    x = (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    x[5] = 0.0
    x[7, :10] = 0.0
    codes, scales = O.quantize_int4_rows(x)
    assert np.all(np.abs(codes.astype(np.int32)) <= 7)
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    assert np.all(np.abs(codes[nz]).max(axis=1) == 7)
    assert np.all(scales[~nz] == 0) and np.all(codes[~nz] == 0)
    err = np.abs(x.astype(np.float64) - O.dequantize_int8_rows(codes, scales))
    assert np.all(err <= scales.astype(np.float64)[:, None] * (0.5 + 1e-5))
    assert np.all((codes == 0) | (np.sign(codes) == np.sign(x)))
    again, _ = O.quantize_int4_rows(O.dequantize_int8_rows(codes, scales).astype(np.float32))
    assert np.array_equal(again, codes)


def test_int4_cache_decode_equals_direct_on_reconstructed_rows():
    """The 4-bit cache, like the 8-bit one, only changes what the retrieval
    heads' lists hold: a decode from it equals the direct mask definition
    over the history whose retrieval rows are replaced by code * scale."""
    sh = S.LayerShape(8, 4, 16, "bf16")
    gate = np.array([0, 1, 1, 0], dtype=np.uint8)
    n = 140
    q, k, v = S.prompt(sh, n, seed=5)
    c = O.HeadSplitCache(1, 4, 16, gate=gate, kv_int4=True)
    c.append(k[:, :n - 1], v[:, :n - 1])
    got = c.decode(q[:, n - 1], k[:, n - 1], v[:, n - 1])[0]
    k_hat, v_hat = O.as_f64(k[0]), O.as_f64(v[0])
    for h in (1, 2):
        kc, ks = O.quantize_int4_rows(k[0, :, h])
        vc, vs = O.quantize_int4_rows(v[0, :, h])
        k_hat[:, h] = O.dequantize_int8_rows(kc, ks)
        v_hat[:, h] = O.dequantize_int8_rows(vc, vs)
    want = O.decode_direct(q[0, n - 1], k_hat, v_hat, gate, 16, 64)
    assert np.max(np.abs(got - want)) < 1e-12
    pos, kc, ks, vc, vs = c.quantized(0, 1)
    assert np.array_equal(pos, np.arange(n)) and kc.shape == (n, 16) and np.abs(kc).max() <= 7


# ---------------------------------------------------------------------------
# Whole-chunk streaming pre-fill (the second pre-fill mode)
# ---------------------------------------------------------------------------

def test_chunk_streaming_mask_matches_hand_drawn(golden):
    params, lines = golden("chunk_stream_mask_n10_c5_s1_r2.txt")
    want = _mask_from_lines(lines)
    c0 = int(params["c0"])
    got = O.chunk_streaming_mask(np.arange(c0, c0 + want.shape[0]), np.arange(want.shape[1]), c0,
                                 int(params["sink"]), int(params["recent"]))
    assert np.array_equal(got, want)
    # and it differs from the Lambda rows of the same queries
    lam = O.streaming_mask(np.arange(c0, c0 + want.shape[0]), np.arange(want.shape[1]), 1, 2)
    assert not np.array_equal(got, lam)


def test_whole_chunk_streaming_first_chunk_is_causal():
    """The first chunk has nothing cached before it, so a streaming head sees
    its whole causal prefix: the chunk-mode pre-fill of a prompt in one chunk
    is full causal attention for every head."""
    rng = np.random.default_rng(21)
    n, hq, hkv, d = 90, 4, 2, 8
    q, k, v = _rand_qkv(rng, n, hq, hkv, d)
    gate = np.array([0, 0], dtype=np.uint8)
    got = O.prefill_direct(q, k, v, 0, gate, 4, 8, stream_mode="chunk")
    want = O.prefill_direct(q, k, v, 0, np.array([1, 1], dtype=np.uint8), 4, 8)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


@pytest.mark.parametrize("chunk", [1, 7, 64, 200])
def test_whole_chunk_streaming_from_caches_equals_direct(chunk):
    """Cache lists (sinks + recent tokens before the chunk, then the chunk
    causally) against the direct mask over the whole history, chunk by chunk."""
    rng = np.random.default_rng(22)
    n, hq, hkv, d, s, r = 200, 4, 2, 8, 4, 16
    q, k, v = _rand_qkv(rng, n, hq, hkv, d)
    gate = np.array([1, 0], dtype=np.uint8)
    c = O.HeadSplitCache(1, hkv, d, gate=gate, sink=s, recent=r)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        got = c.prefill_chunk(q[None, c0:c1], k[None, c0:c1], v[None, c0:c1], stream_mode="chunk")[0]
        want = O.prefill_direct(q[c0:c1], k[:c1], v[:c1], c0, gate, s, r, stream_mode="chunk")
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)
    # the retrieval head's rows are those of the Lambda-mode pre-fill
    lam = O.prefill_direct(q[n - chunk:], k, v, n - chunk, gate, s, r)
    np.testing.assert_allclose(got[:, :2], lam[-got.shape[0]:, :2], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# Gate gradient of the gated mix [Review S3 "Core formula",
# "Retrieval-head identification"]
# ---------------------------------------------------------------------------

def test_grad_alpha_worked_example_d1(golden):
    """d = 1 example: full = (6, 2, 7), streaming = (6, 2, 10.5); with
    dout = (1, 1, 1) the gate gradient is 0 + 0 + (7 - 10.5) = -3.5, and with
    dout = (0, 0, 2) it is -7."""
    params, _ = golden("tiny_attention_d1.txt")
    q = np.ones((3, 1, 1))
    k = np.array([0.0, math.log(2), math.log(3)]).reshape(3, 1, 1)
    v = np.array([6.0, 0.0, 12.0]).reshape(3, 1, 1)
    fa, sa = np.array(params["full"]), np.array(params["streaming"])
    for dout, want in ((np.ones(3), -3.5), (np.array([0.0, 0.0, 2.0]), -7.0)):
        got = O.gated_mix_grad_alpha(q, k, v, dout.reshape(3, 1, 1), 1, 1, scale=1.0)
        assert abs(got[0] - want) < 1e-12
        assert abs(got[0] - float(np.dot(dout, fa - sa))) < 1e-12


def test_grad_alpha_equals_central_difference():
    """The mix is linear in alpha, so a central difference of <dout, mix>
    equals the gradient up to rounding."""
    rng = np.random.default_rng(31)
    n, hq, hkv, d, s, r = 60, 8, 4, 8, 2, 9
    q, k, v = _rand_qkv(rng, n, hq, hkv, d)
    dout = rng.standard_normal((n, hq, d))
    alpha = rng.uniform(0, 1, hkv)
    got = O.gated_mix_grad_alpha(q, k, v, dout, s, r)
    for kv in range(hkv):
        e = np.zeros(hkv)
        e[kv] = 1e-3
        fd = (np.sum(dout * O.gated_mix(q, k, v, alpha + e, s, r)) -
              np.sum(dout * O.gated_mix(q, k, v, alpha - e, s, r))) / 2e-3
        assert abs(fd - got[kv]) < 1e-8 * max(1.0, abs(got[kv]))


def test_grad_alpha_vanishes_when_the_window_covers_the_sequence():
    rng = np.random.default_rng(32)
    n, hq, hkv, d = 40, 4, 2, 8
    q, k, v = _rand_qkv(rng, n, hq, hkv, d)
    dout = rng.standard_normal((n, hq, d))
    assert np.all(np.abs(O.gated_mix_grad_alpha(q, k, v, dout, 8, 32)) < 1e-12)
    assert np.any(np.abs(O.gated_mix_grad_alpha(q, k, v, dout, 2, 5)) > 1e-3)


def test_oracle_pool_rows_equal_direct_rows(tmp_path):
    """The spawned workers the full-size parity test uses return the rows the
    oracle computes in this process, per chunk and in order (equal up to the
    fp64 summation order of their single-threaded BLAS)."""
    from tests.oracle_pool import PrefillOracle
    sh = S.LayerShape(8, 4, 16, "bf16", sink=3, recent=5)
    n, C = 96, 32
    q, k, v = S.prompt(sh, n, seed=2)
    gate = np.array([1, 0, 0, 1], dtype=np.uint8)
    ora = PrefillOracle(tmp_path, q[0], k[0], v[0], gate, sh.sink, sh.recent, workers=2)
    rows = {0: np.arange(C), 32: np.array([0, 5, 31]), 64: np.arange(0, C, 3)}
    for c0, r in rows.items():
        ora.submit(c0, C, r, block=4)
    got = ora.results()
    for c0, r in rows.items():
        want = O.prefill_direct(q[0, c0:c0 + C], k[0, :c0 + C], v[0, :c0 + C], c0, gate, sh.sink, sh.recent, rows=r)
        assert np.array_equal(got[c0][0], r)
        np.testing.assert_allclose(got[c0][1], want, atol=1e-12, rtol=0)
