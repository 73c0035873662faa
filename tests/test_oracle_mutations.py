"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of an oracle function (on the CPU,
through monkeypatch) and checks that at least one pin from
test_oracle_pins.py fails.  Nothing here touches a GPU.
"""

import numpy as np
import pytest

import oracle
import oracle.duo_oracle as D
import tests.test_oracle_pins as P
from tests.conftest import read_golden


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(D, name, fn)
    monkeypatch.setattr(oracle, name, fn)
    monkeypatch.setattr(P.O, name, fn, raising=False)


def _fails(*tests):
    """True if any of the pin functions raises."""
    for t in tests:
        try:
            t()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


def _pins():
    g = read_golden
    return [
        lambda: P.test_lambda_mask_matches_hand_drawn(g),
        lambda: P.test_causal_mask_matches_hand_drawn(g),
        lambda: P.test_worked_example_d1(g),
        lambda: P.test_brute_force_tiny(12, 4, 2, 3, 2, 2),
        lambda: P.test_brute_force_tiny(11, 3, 1, 4, 4, 2),
        P.test_matches_torch_sdpa_cpu_float64,
        P.test_alpha_one_is_full_causal_attention,
        P.test_mix_is_linear_in_alpha,
        P.test_gqa_with_group_one_is_mha_and_groups_share_kv,
        lambda: P.test_ring_positions_match_hand_table(g),
        lambda: P.test_ring_after_block_append_equals_token_by_token(g),
        lambda: P.test_streaming_cache_stays_constant_size(0),
        lambda: P.test_streaming_positions_are_the_sinks_and_the_recent_tokens(3, 9),
        P.test_decode_after_prefill_equals_direct_row,
        lambda: P.test_chunked_prefill_from_caches_equals_direct(7),
        P.test_partition_by_threshold,
        P.test_partition_top_k_ties_go_to_lower_index,
        P.test_binarize_uses_greater_or_equal,
        lambda: P.test_int8_codes_match_hand_worked_rows(g),
        lambda: P.test_int4_codes_match_hand_worked_rows(g),
        lambda: P.test_int4_round_trip_is_within_half_a_step(0),
        P.test_int4_cache_decode_equals_direct_on_reconstructed_rows,
        lambda: P.test_int8_round_trip_is_within_half_a_step(0),
        P.test_int8_cache_decode_equals_direct_on_reconstructed_rows,
        lambda: P.test_chunk_streaming_mask_matches_hand_drawn(g),
        P.test_whole_chunk_streaming_first_chunk_is_causal,
        lambda: P.test_whole_chunk_streaming_from_caches_equals_direct(7),
        lambda: P.test_grad_alpha_worked_example_d1(g),
        P.test_grad_alpha_equals_central_difference,
        P.test_grad_alpha_vanishes_when_the_window_covers_the_sequence,
    ]


def test_unmutated_oracle_passes_all_pins():
    assert not _fails(*_pins())


def _mask_no_sink(q_pos, k_pos, sink, recent):
    qi, kj = np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :]
    return (kj <= qi) & (qi - kj < recent)


def _mask_window_off_by_one(q_pos, k_pos, sink, recent):
    qi, kj = np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :]
    return (kj <= qi) & ((kj < sink) | (qi - kj <= recent))


def _mask_not_causal(q_pos, k_pos, sink, recent):
    qi, kj = np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :]
    return (kj < sink) | (np.abs(qi - kj) < recent)


def _causal_strict(q_pos, k_pos):
    # the mistake: the diagonal is masked, so a token never sees itself
    return np.asarray(k_pos)[None, :] < np.asarray(q_pos)[:, None]


def _attention_transposed(q, k, v, mask, scale):
    # the mistake: scores taken as K Q^T instead of Q K^T
    q, k, v = D.as_f64(q), D.as_f64(k), D.as_f64(v)
    s = scale * (k @ q.T)
    if s.shape != np.shape(mask):
        raise ValueError("shape mismatch from the transposed operand")
    return D.masked_softmax(s, np.asarray(mask, dtype=bool)) @ v


def _attention_no_scale(q, k, v, mask, scale):
    q, k, v = D.as_f64(q), D.as_f64(k), D.as_f64(v)
    return D.masked_softmax(q @ k.T, np.asarray(mask, dtype=bool)) @ v


def _slot_no_sink_offset(p, sink, recent):
    return p if p < sink else (p - sink) % recent


def _binarize_strict(alpha, tau):
    return (np.asarray(alpha, dtype=np.float64) > float(tau)).astype(np.uint8)


_orig_mix = D.gated_mix


def _mix_swapped(q, k, v, alpha, sink, recent, scale=None):
    return _orig_mix(q, k, v, 1.0 - np.asarray(alpha, dtype=np.float64), sink, recent, scale)



def _append_evicts_sinks(self, k_new, v_new):
    k_new, v_new = np.asarray(k_new), np.asarray(v_new)
    b_, t, hkv, d = k_new.shape
    for b in range(self.batch):
        p0 = self.length[b]
        for h in range(hkv):
            if self.gate[h]:
                if t:
                    self.full[b][h].append((np.arange(p0, p0 + t), k_new[b, :, h].copy(), v_new[b, :, h].copy()))
            else:
                lst = self.stream[b][h]
                for i in range(t):
                    lst.append((p0 + i, k_new[b, i, h].copy(), v_new[b, i, h].copy()))
                    if len(lst) > self.sink + self.recent:
                        del lst[0]              # the mistake: sinks are evicted too
        self.length[b] = p0 + t


@pytest.mark.parametrize("name,fn", [
    ("streaming_mask", _mask_no_sink),
    ("streaming_mask", _mask_window_off_by_one),
    ("streaming_mask", _mask_not_causal),
    ("causal_mask", _causal_strict),
    ("masked_attention", _attention_transposed),
    ("masked_attention", _attention_no_scale),
    ("ring_slot", _slot_no_sink_offset),
    ("binarize_gates", _binarize_strict),
    ("gated_mix", _mix_swapped),
])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    _patch(monkeypatch, name, fn)
    assert _fails(*_pins()), f"no pin caught the planted mistake in {name} ({fn.__name__})"


def test_planted_eviction_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(D.HeadSplitCache, "append", _append_evicts_sinks)
    assert _fails(*_pins())


def _push_evicts_sinks(lst, entry, sink, recent):
    lst.append(entry)
    if len(lst) > sink + recent:
        del lst[0]                              # the mistake: sinks are evicted too


def _push_keeps_one_too_many(lst, entry, sink, recent):
    lst.append(entry)
    if len(lst) > sink + recent + 1:            # the mistake: the window is one token long
        for e in range(len(lst)):
            if lst[e][0] >= sink:
                del lst[e]
                break


@pytest.mark.parametrize("fn", [_push_evicts_sinks, _push_keeps_one_too_many])
def test_planted_push_mistake_is_caught(monkeypatch, fn):
    """A mistake in the shared eviction step shows in the appends and in the
    replayed positions alike."""
    monkeypatch.setattr(D, "_streaming_push", fn)
    assert _fails(*_pins())


def test_planted_gqa_mapping_mistake_is_caught(monkeypatch):
    def mix_mod_mapping(q, k, v, alpha, sink, recent, scale=None):
        q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
        hq, hkv = q.shape[1], k.shape[1]
        out = np.empty(q.shape[:2] + (v.shape[2],))
        for h in range(hq):
            kv = h % hkv                      # the mistake: interleaved groups
            a = float(np.asarray(alpha)[kv])
            out[:, h] = a * D.full_attn(q[:, h], k[:, kv], v[:, kv], scale) + \
                (1 - a) * D.streaming_attn(q[:, h], k[:, kv], v[:, kv], sink, recent, scale)
        return out
    _patch(monkeypatch, "gated_mix", mix_mod_mapping)
    assert _fails(*_pins())


def _q8(x, factor_num=127.0, scale_den=127.0, rnd=np.rint, per_tensor=False):
    x32 = D.as_f64(x).astype(np.float32)
    codes = np.zeros(x32.shape, dtype=np.int8)
    scales = np.zeros(x32.shape[:-1], dtype=np.float32)
    amax_all = np.float32(np.abs(x32).max()) if x32.size else np.float32(0)
    for i in range(x32.shape[0]):
        amax = amax_all if per_tensor else np.float32(np.abs(x32[i]).max())
        if amax == 0:
            continue
        codes[i] = np.clip(rnd(x32[i] * (np.float32(factor_num) / amax)), -128, 127).astype(np.int8)
        scales[i] = amax / np.float32(scale_den)
    return codes, scales


@pytest.mark.parametrize("mistake", [
    dict(rnd=np.floor),                     # rounds down instead of to nearest
    dict(rnd=np.trunc),                     # rounds toward zero
    dict(rnd=lambda v: np.floor(v + np.float32(0.5))),   # ties away from even
    dict(factor_num=128.0, scale_den=128.0),             # 128 steps: the extreme code overflows
    dict(scale_den=128.0),                  # scale from a different step than the codes
    dict(per_tensor=True),                  # one scale for all rows
])
def test_planted_int8_mistake_is_caught(monkeypatch, mistake):
    _patch(monkeypatch, "quantize_int8_rows", lambda x: _q8(x, **mistake))
    assert _fails(*_pins()), f"no pin caught the planted quantizer mistake {mistake}"


@pytest.mark.parametrize("mistake", [
    dict(factor_num=7.0, scale_den=7.0, rnd=np.floor),                         # rounds down
    dict(factor_num=7.0, scale_den=7.0, rnd=lambda v: np.floor(v + np.float32(0.5))),   # ties away from even
    dict(factor_num=8.0, scale_den=8.0),                                       # 8 levels: +8 does not fit
    dict(factor_num=7.0, scale_den=8.0),                                       # scale from another step
    dict(factor_num=7.5, scale_den=7.5),                                       # 15 levels over 16 codes
    dict(factor_num=7.0, scale_den=7.0, per_tensor=True),                      # one scale for all rows
])
def test_planted_int4_mistake_is_caught(monkeypatch, mistake):
    _patch(monkeypatch, "quantize_int4_rows", lambda x: _q8(x, **mistake))
    assert _fails(*_pins()), f"no pin caught the planted 4-bit quantizer mistake {mistake}"


def _chunk_mask_window_short(q_pos, k_pos, c0, sink, recent):
    qi, kj = np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :]
    return (kj <= qi) & ((kj < sink) | (kj >= c0 - recent + 1))   # one recent token too few


def _chunk_mask_is_lambda(q_pos, k_pos, c0, sink, recent):
    return D.streaming_mask(q_pos, k_pos, sink, recent)


def _chunk_mask_no_sink(q_pos, k_pos, c0, sink, recent):
    qi, kj = np.asarray(q_pos)[:, None], np.asarray(k_pos)[None, :]
    return (kj <= qi) & (kj >= c0 - recent)


@pytest.mark.parametrize("fn", [_chunk_mask_window_short, _chunk_mask_is_lambda, _chunk_mask_no_sink])
def test_planted_chunk_mask_mistake_is_caught(monkeypatch, fn):
    _patch(monkeypatch, "chunk_streaming_mask", fn)
    assert _fails(*_pins()), f"no pin caught {fn.__name__}"


def _grad(q, k, v, dout, sink, recent, scale=None, sign=1.0, mapping="group", first_only=False, mean=False):
    q, k, v, dout = np.asarray(q), np.asarray(k), np.asarray(v), D.as_f64(dout)
    n, hq, _ = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    grad = np.zeros(hkv)
    for h in range(hq):
        kv = h // g if mapping == "group" else h % hkv
        if first_only and h % g:
            continue
        fa = D.full_attn(q[:, h], k[:, kv], v[:, kv], scale)
        sa = D.streaming_attn(q[:, h], k[:, kv], v[:, kv], sink, recent, scale)
        t = float(np.sum(dout[:, h] * (fa - sa))) * sign
        grad[kv] += t / n if mean else t
    return grad


@pytest.mark.parametrize("mistake", [dict(sign=-1.0), dict(mapping="interleaved"), dict(first_only=True),
                                     dict(mean=True)])
def test_planted_grad_alpha_mistake_is_caught(monkeypatch, mistake):
    _patch(monkeypatch, "gated_mix_grad_alpha", lambda *a, **kw: _grad(*a, **kw, **mistake))
    assert _fails(*_pins()), f"no pin caught {mistake}"
