"""duo_decode_attn_noalloc: the decode entry point for callers that cannot
allocate device memory (its scratch is an array inside the library).

The GPU test runs two decode steps in a row through the C ABI on two
identical layers -- one with duo_decode_attn and a caller workspace, one with
duo_decode_attn_noalloc -- and compares the outputs within the bf16 tolerance
used everywhere else (max-abs 2e-2, mean-abs 2e-3).  This file is collected
last, so a run that stops at the first failure has run every other test."""

import numpy as np
import pytest

from head_split_kv_b200 import synthetic as S
from tests.gpu_helpers import Layer, assert_close, f64, to_dev, torch


def _pair(duo, sh, retrieval, L0, seed):
    lays = []
    for _ in range(2):
        lay = Layer(duo, sh, retrieval, 1, capacity=L0 + 8)
        lay.load_state(S.decode_state(sh, retrieval, [L0], seed=seed))
        lays.append(lay)
    return lays


@pytest.mark.gpu
@pytest.mark.parametrize("hq,hkv,n_ret,L0", [(32, 32, 8, 5000), (32, 8, 4, 20011)])
def test_noalloc_decode_matches_workspace_decode_twice(duo, hq, hkv, n_ret, L0):
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sh = S.LayerShape(hq, hkv, 128, "bf16")
    retrieval = S.retrieval_heads_by_seed(hkv, n_ret)
    ref, noalloc = _pair(duo, sh, retrieval, L0, seed=11)
    qs, ks, vs = S.decode_steps(sh, 1, 2, seed=11)
    for i in range(2):                        # two calls in a row
        q, k, v = to_dev(qs[i]), to_dev(ks[i][:, None]), to_dev(vs[i][:, None])
        out_ref, out_na = t.empty_like(q), t.empty_like(q)
        duo.append_kv(ref.desc, ref.caches.state, k, v, 1)
        duo.decode_attn(ref.desc, ref.caches.state, q, out_ref, ref.ws.ptr, ref.ws.nbytes)
        duo.append_kv(noalloc.desc, noalloc.caches.state, k, v, 1)
        duo.decode_attn_noalloc(noalloc.desc, noalloc.caches.state, q, out_na)
        assert_close(f64(out_na), f64(out_ref), "bf16", f"call {i}")
        assert np.all(np.isfinite(f64(out_na)))
    assert ref.status() == 0 and noalloc.status() == 0


@pytest.mark.gpu
def test_noalloc_alternating_plans_on_one_stream(duo):
    """Two layers whose split plans differ (an MHA layer at 5,000 tokens: 8
    heads x 34 splits of one query head; a GQA layer at 20,011 tokens: 4
    heads x 73 splits of four query heads) take turns on one stream, so each
    call finds the other plan's partial records and ticket words in the
    shared array.  Each output matches duo_decode_attn with a caller
    workspace on an identical layer."""
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cases = []
    for hq, hkv, n_ret, L0, seed in [(32, 32, 8, 5000, 21), (32, 8, 4, 20011, 22)]:
        sh = S.LayerShape(hq, hkv, 128, "bf16")
        retrieval = S.retrieval_heads_by_seed(hkv, n_ret)
        ref, noalloc = _pair(duo, sh, retrieval, L0, seed=seed)
        cases.append((sh, ref, noalloc, S.decode_steps(sh, 1, 3, seed=seed)))
    plans = {duo.workspace_bytes(c[2].desc, duo.OP_DECODE, c[2].caches.capacity) for c in cases}
    assert len(plans) == 2 and max(plans) <= duo.NOALLOC_SCRATCH_BYTES
    for i in range(3):
        for sh, ref, noalloc, (qs, ks, vs) in cases:
            q, k, v = to_dev(qs[i]), to_dev(ks[i][:, None]), to_dev(vs[i][:, None])
            out_ref, out_na = t.empty_like(q), t.empty_like(q)
            duo.append_kv(ref.desc, ref.caches.state, k, v, 1)
            duo.decode_attn(ref.desc, ref.caches.state, q, out_ref, ref.ws.ptr, ref.ws.nbytes)
            duo.append_kv(noalloc.desc, noalloc.caches.state, k, v, 1)
            duo.decode_attn_noalloc(noalloc.desc, noalloc.caches.state, q, out_na)
            assert_close(f64(out_na), f64(out_ref), "bf16", f"step {i}, {sh.n_kv_heads} KV heads")
    for _, ref, noalloc, _ in cases:
        assert ref.status() == 0 and noalloc.status() == 0


def test_noalloc_rejects_a_layer_beyond_the_array(duo):
    # 64 sequences x 32 retrieval heads of a 1M-token cache need far more than
    # the built-in 2 MiB; the size check runs on the host before any GPU work
    d = duo.desc_init(64, 32, 32, 128, duo.BF16, list(range(32)), 32)
    need = duo.workspace_bytes(d, duo.OP_DECODE, 1 << 20)
    assert need > duo.NOALLOC_SCRATCH_BYTES
    st = duo.KVState(k_full=16, v_full=32, capacity=1 << 20, k_ring=48, v_ring=64, ring_pos=80, seq_len=96,
                     counters=112, status=128)
    with pytest.raises(duo.DuoError) as e:
        duo.decode_attn_noalloc(d, st, 256, 512, stream=0)
    assert e.value.status == duo.ERR_CAPACITY
    assert str(duo.NOALLOC_SCRATCH_BYTES) in duo.last_error()
