"""Device status bits: each condition only the device can see is made to
happen through the C ABI -- from the host, with a bad page-table entry, a
length set past the cache, or a wait on a barrier nothing completes -- and
the test checks that its DUO_DEV_* bit reaches the status word, that the
access it guards was skipped (the caches are byte-for-byte what they were),
and that the context stays usable (a normal call afterwards matches the
oracle).  No case faults, traps or hangs the GPU: every guard runs before the
access it protects, and the wait is bounded in wall time."""

import numpy as np
import pytest

from head_split_kv_b200 import synthetic as S
from tests.gpu_helpers import Layer, assert_close, bits, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    t.cuda.synchronize()


def _snapshot(lay):
    c = lay.caches
    return {n: bits(getattr(c, n)).copy() for n in ("k_full", "v_full", "k_ring", "v_ring", "ring_pos")}


def _same(a, b):
    return all(np.array_equal(a[n], b[n]) for n in a)


def _paged_layer(duo, lengths, hole_page_of=None):
    """MHA layer, 4 retrieval heads, paged; optionally the page table entry
    of sequence 0 at page index hole_page_of is -1 (missing)."""
    sh = S.LayerShape(8, 8, 128, "bf16")
    table, n_pages = S.page_assignment(lengths, 64, 64, seed=9)
    if hole_page_of is not None:
        table[0, hole_page_of] = -1
    lay = Layer(duo, sh, [0, 2, 5, 7], len(lengths), page_size=64, page_table=table, n_pages=n_pages)
    return sh, lay, table


def test_bad_page_on_append_is_reported_and_skipped(duo):
    # sequence 0 holds 100 tokens; its page 2 (positions 128..191) is missing
    sh, lay, table = _paged_layer(duo, [100, 40], hole_page_of=2)
    t = torch()
    lay.caches.seq_len.copy_(t.tensor([100, 40], dtype=t.int32))
    before = _snapshot(lay)
    k = S.normal(S.rng_for(9, 1), (2, 60, 8, 128), "bf16")       # sequence 0: positions 100..159
    duo.append_kv(lay.desc, lay.caches.state, to_dev(k), to_dev(k), 60)
    st = lay.status()
    assert st & duo.DEV_BAD_PAGE and not st & ~duo.DEV_BAD_PAGE
    after = _snapshot(lay)
    # rows 100..127 of sequence 0 and all of sequence 1 landed; nothing went
    # anywhere for positions 128..159 (every other byte of the pool is as before)
    kf = after["k_full"].copy()
    for b, (p0, n) in enumerate([(100, 28), (40, 60)]):
        for i in range(n):
            p = p0 + i
            pg = table[b, p // 64]
            for r, h in enumerate([0, 2, 5, 7]):
                assert np.array_equal(kf[pg, r, p % 64], k[b, i, h])
                kf[pg, r, p % 64] = before["k_full"][pg, r, p % 64]
    assert np.array_equal(kf, before["k_full"])
    assert list(bits(lay.caches.seq_len)) == [160, 100]


def test_bad_page_on_decode_is_reported(duo):
    # a 300-token sequence whose page 1 is missing: the decode tile of rows
    # 64..127 is skipped as empty and the bit is set; the caches stay as they were
    sh, lay, table = _paged_layer(duo, [300], hole_page_of=1)
    t = torch()
    lay.caches.seq_len.copy_(t.tensor([300], dtype=t.int32))
    before = _snapshot(lay)
    q = to_dev(S.normal(S.rng_for(9, 2), (1, 8, 128), "bf16"))
    out = t.empty_like(q)
    duo.decode_attn(lay.desc, lay.caches.state, q, out, lay.ws.ptr, lay.ws.nbytes)
    assert lay.status() & duo.DEV_BAD_PAGE
    assert _same(before, _snapshot(lay))
    assert bool(t.isfinite(out.float()).all())


def test_length_past_capacity_is_reported_and_clamped(duo):
    sh = S.LayerShape(16, 4, 128, "bf16")
    retrieval = [1, 3]
    lay = Layer(duo, sh, retrieval, 1, capacity=500)
    lay.load_state(S.decode_state(sh, retrieval, [400], seed=12))
    t = torch()
    lay.caches.seq_len.copy_(t.tensor([512], dtype=t.int32))     # 12 rows past the cache
    before = _snapshot(lay)
    q = to_dev(S.normal(S.rng_for(12, 3), (1, 16, 128), "bf16"))
    out = t.empty_like(q)
    duo.decode_attn(lay.desc, lay.caches.state, q, out, lay.ws.ptr, lay.ws.nbytes)
    assert lay.status() & duo.DEV_BAD_LENGTH
    assert _same(before, _snapshot(lay))
    assert bool(t.isfinite(out.float()).all())
    # a negative length: the append skips every row and reports it
    lay2 = Layer(duo, sh, retrieval, 1, capacity=500)
    lay2.caches.seq_len.copy_(t.tensor([-5], dtype=t.int32))
    before = _snapshot(lay2)
    k = to_dev(S.normal(S.rng_for(12, 4), (1, 3, 4, 128), "bf16"))
    duo.append_kv(lay2.desc, lay2.caches.state, k, k, 3)
    assert lay2.status() & duo.DEV_BAD_LENGTH
    assert _same(before, _snapshot(lay2))


@pytest.mark.parametrize("limit_us", [2000, 50000])
def test_wait_timeout_is_reported_and_the_context_stays_usable(duo, limit_us):
    t = torch()
    status = t.zeros(1, dtype=t.int32, device="cuda")
    e0, e1 = t.cuda.Event(enable_timing=True), t.cuda.Event(enable_timing=True)
    e0.record()
    duo.wait_probe(status, limit_us)
    e1.record()
    t.cuda.synchronize()
    assert status.item() == duo.DEV_WAIT_TIMEOUT
    ms = e0.elapsed_time(e1)
    assert limit_us / 1e3 <= ms < limit_us / 1e3 + 500, ms          # it waited its limit, then returned
    # the same context runs a decode step against the oracle afterwards
    sh = S.LayerShape(8, 4, 128, "bf16")
    lay = Layer(duo, sh, [0, 3], 1, capacity=300)
    lay.load_state(S.decode_state(sh, [0, 3], [200], seed=13))
    qs, ks, vs = S.decode_steps(sh, 1, 1, seed=13)
    got, want = lay.decode(qs[0], ks[0], vs[0], fused=True)
    assert_close(got, want, "bf16", "decode after the timeout")
    assert lay.status() == 0
