"""GPU parity of the tensor-core chunked pre-fill (bf16, head_dim 128) against
the oracle's direct mask definition: every query row of chunk k attends to the
whole token history 0..P through its head's mask.  Also checks that the caches
filled chunk by chunk stay bit-exact."""

import numpy as np
import pytest

import oracle as O
from head_split_kv_b200 import synthetic as S
from tests.gpu_helpers import Layer, assert_close, f64, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    t.cuda.synchronize()


def _run(duo, sh, retrieval, n, chunks, B=1, seed=0, sample_rows=None, check_cache=True, sigma=None,
         stream_mode="lambda", workspace=True):
    """Pre-fill n tokens in the given chunk lengths; compare every output row
    (or `sample_rows` seeded rows per chunk) with the oracle.  With a
    workspace, long retrieval units split their key tiles across CTAs."""
    t = torch()
    lay = Layer(duo, sh, retrieval, B, capacity=n + 16,
                stream_prefill=duo.STREAM_CHUNK if stream_mode == "chunk" else duo.STREAM_LAMBDA)
    ws = duo.Workspace(lay.desc, duo.OP_PREFILL, max(chunks)) if workspace else None
    q, k, v = S.prompt(sh, n, seed=seed, batch=B, sigma=sigma)
    c0 = 0
    rng = S.rng_for(seed, 77)
    errs = []
    for ci, C in enumerate(chunks):
        c1 = c0 + C
        qd = to_dev(np.ascontiguousarray(q[:, c0:c1]))
        kd = to_dev(np.ascontiguousarray(k[:, c0:c1]))
        vd = to_dev(np.ascontiguousarray(v[:, c0:c1]))
        out = t.empty_like(qd)
        duo.prefill_chunk(lay.desc, lay.caches.state, qd, kd, vd, C, out, ws and ws.ptr, ws.nbytes if ws else 0)
        duo.append_kv(lay.desc, lay.caches.state, kd, vd, C)
        lay.oracle.append(k[:, c0:c1], v[:, c0:c1])
        got = f64(out)
        if sample_rows is None or C <= sample_rows:
            rows = np.arange(C)
        else:
            rows = np.unique(np.concatenate([[0, C - 1], rng.choice(C, sample_rows, replace=False)]))
        for b in range(B):
            want = O.prefill_direct(q[b, c0:c1], k[b, :c1], v[b, :c1], c0, np.array(lay.gate), sh.sink, sh.recent,
                                    rows=rows, stream_mode=stream_mode)
            errs.append(assert_close(got[b, rows], want, "bf16", f"chunk {ci} (c0={c0}) b={b}"))
        c0 = c1
    if check_cache:
        lay.assert_caches_match()
    assert lay.status() == 0
    return errs


@pytest.mark.parametrize("chunks", [[700], [128] * 5 + [60], [300, 300, 100], [7, 9, 64, 1, 200, 419]])
def test_prefill_tc_gqa_chunkings(duo, chunks):
    sh = S.LayerShape(16, 4, 128, "bf16")
    _run(duo, sh, [1, 2], sum(chunks), chunks)


def _history(sh, st, b, L, k_new, v_new):
    """Token history [L + C, Hkv, d] of sequence b: the decode state's rows
    (a streaming head: the positions the oracle's eviction rule keeps, zeros
    elsewhere -- the Lambda mask never reads those positions from a later
    query) followed by the chunk's rows."""
    C = k_new.shape[0]
    k_all = np.zeros((L + C, sh.n_kv_heads, sh.head_dim), dtype=np.float64)
    v_all = np.zeros_like(k_all)
    kept = O.streaming_positions(L, sh.sink, sh.recent)
    for h in range(sh.n_kv_heads):
        if (b, h) in st.full:
            k, v = st.full[(b, h)]
            k_all[:L, h], v_all[:L, h] = O.as_f64(k), O.as_f64(v)
        else:
            k, v = st.stream_rows(b, h, kept)
            k_all[kept, h], v_all[kept, h] = O.as_f64(k), O.as_f64(v)
    k_all[L:], v_all[L:] = O.as_f64(k_new), O.as_f64(v_new)
    return k_all, v_all


@pytest.mark.parametrize("chunk,lengths", [(1000, [0, 1100, 2300]), (256, [0, 1100, 2300]),
                                          (4096, [0, 5000, 9001])])
def test_prefill_tc_uneven_batch(duo, chunk, lengths):
    """Sequences of one batch at different lengths take one chunk together:
    each sequence's query tiles see their own prior tiles, the first of them
    partly before position 0 when the length is not a multiple of the tile.
    With 4,096-token chunks the three sequences split their key tiles 2, 4
    and 4 ways in the same launch."""
    t = torch()
    sh = S.LayerShape(16, 4, 128, "bf16")
    retrieval = [0, 3]
    B = len(lengths)
    lay = Layer(duo, sh, retrieval, B, capacity=max(lengths) + chunk + 16)
    st = S.decode_state(sh, retrieval, lengths, seed=5)
    lay.load_state(st)
    q, k, v = S.prompt(sh, chunk, seed=6, batch=B)
    rows = np.unique(np.concatenate([[0, chunk - 1], S.rng_for(6, 78).choice(chunk, 96, replace=False)]))
    want = [O.prefill_direct(q[b], *_history(sh, st, b, L, k[b], v[b]), L, np.array(lay.gate), sh.sink, sh.recent,
                             rows=rows) for b, L in enumerate(lengths)]
    out = t.empty((B, chunk, sh.n_q_heads, sh.head_dim), dtype=t.bfloat16, device="cuda")
    ws = duo.Workspace(lay.desc, duo.OP_PREFILL, chunk)
    for call in range(2):   # the second call reuses the workspace the first left
        out.zero_()
        duo.prefill_chunk(lay.desc, lay.caches.state, to_dev(q), to_dev(k), to_dev(v), chunk, out, ws.ptr, ws.nbytes)
        got = f64(out)
        for b, L in enumerate(lengths):
            assert_close(got[b, rows], want[b], "bf16", f"call {call} b={b} (cached {L})")
    assert lay.status() == 0


@pytest.mark.parametrize("chunks", [[700], [128] * 5 + [60], [300, 300, 100], [7, 9, 64, 1, 200, 419]])
def test_prefill_tc_whole_chunk_streaming(duo, chunks):
    """Streaming heads in whole-chunk mode on the tensor cores: the ring as it
    stood before the chunk, then the chunk causally."""
    sh = S.LayerShape(16, 4, 128, "bf16")
    _run(duo, sh, [1, 2], sum(chunks), chunks, stream_mode="chunk")


def test_prefill_tc_whole_chunk_streaming_long_prefix(duo):
    sh = S.LayerShape(32, 8, 128, "bf16")
    _run(duo, sh, S.retrieval_heads_by_seed(8, 4), 12288, [8192, 4096], sample_rows=96, check_cache=False,
         stream_mode="chunk")


def test_prefill_tc_mha_25pct(duo):
    sh = S.LayerShape(32, 32, 128, "bf16")
    _run(duo, sh, S.retrieval_heads_by_seed(32, 8), 2048, [512] * 4, sample_rows=64)


def test_prefill_tc_batch_and_scaled_heads(duo):
    sh = S.LayerShape(8, 2, 128, "bf16")
    _run(duo, sh, [0], 900, [256, 644], B=3, sigma=S.head_sigma(2))


def test_prefill_tc_all_retrieval_and_all_streaming(duo):
    sh = S.LayerShape(8, 4, 128, "bf16")
    _run(duo, sh, [0, 1, 2, 3], 500, [200, 300])
    _run(duo, sh, [], 500, [200, 300])


@pytest.mark.parametrize("workspace", [True, False])
def test_prefill_tc_long_prefix(duo, workspace):
    # a 20K-token history, then a 4096 chunk: many prior tiles per query tile,
    # split 4 ways across CTAs with a workspace, whole without
    sh = S.LayerShape(32, 8, 128, "bf16")
    _run(duo, sh, S.retrieval_heads_by_seed(8, 4), 24576, [20480, 4096], sample_rows=96, check_cache=False,
         workspace=workspace)


def test_prefill_tc_mha_split(duo):
    # MHA with 8 retrieval heads: 128 retrieval units per 4,096 chunk, planned
    # at 8 splits; over a 16K history a unit has 160 key tiles and takes 3
    # (no split under 48 tiles)
    sh = S.LayerShape(32, 32, 128, "bf16")
    _run(duo, sh, S.retrieval_heads_by_seed(32, 8), 20480, [16384, 4096], sample_rows=64, check_cache=False)


def test_prefill_tc_gqa_eight_way_split(duo):
    # GQA with 2 of 8 KV heads retrieval: 128 retrieval units per 4,096 chunk,
    # planned at 8 splits; over a 48K history a unit has 416 key tiles and
    # takes all 8.  The 49,152-token first chunk runs 2-way splits.
    sh = S.LayerShape(32, 8, 128, "bf16")
    _run(duo, sh, [2, 5], 53248, [49152, 4096], sample_rows=48, check_cache=False)


@pytest.mark.slow
def test_prefill_gqa_131k_full(duo, tmp_path):
    """The full workload the bench times, in its launch configuration: a
    131,072-token prompt in 32 chunks of 4,096 with the bench's workspace.
    Every row of chunks 0, 1 and 31 and 512 seeded rows of every other chunk
    (plus each chunk's first and last row) are compared with the oracle,
    whose rows a spawned process pool computes while the GPU runs; the caches
    are compared byte for byte at the end."""
    from tests.oracle_pool import PrefillOracle
    t = torch()
    sh = S.LayerShape(32, 8, 128, "bf16")
    n, C = 131072, 4096
    n_chunks = n // C
    lay = Layer(duo, sh, S.retrieval_heads_by_seed(8, 4), 1, capacity=n + 16)
    ws = duo.Workspace(lay.desc, duo.OP_PREFILL, C)
    q, k, v = S.prompt(sh, n, seed=0)
    rng = S.rng_for(0, 77)
    rows = {}
    for ci in range(n_chunks):
        if ci in (0, 1, n_chunks - 1):
            rows[ci] = np.arange(C)
        else:
            rows[ci] = np.unique(np.concatenate([[0, C - 1], rng.choice(C, 512, replace=False)]))
    ora = PrefillOracle(tmp_path, q[0], k[0], v[0], lay.gate, sh.sink, sh.recent)
    for ci in sorted(rows, key=lambda c: -(c + 1) * len(rows[c])):     # the longest jobs first
        ora.submit(ci * C, C, rows[ci])
    got = {}
    for ci in range(n_chunks):
        c0 = ci * C
        qd, kd, vd = (to_dev(np.ascontiguousarray(x[:, c0:c0 + C])) for x in (q, k, v))
        out = t.empty_like(qd)
        duo.prefill_chunk(lay.desc, lay.caches.state, qd, kd, vd, C, out, ws.ptr, ws.nbytes)
        duo.append_kv(lay.desc, lay.caches.state, kd, vd, C)
        lay.oracle.append(k[:, c0:c0 + C], v[:, c0:c0 + C])
        got[c0] = f64(out[0].index_select(0, t.from_numpy(rows[ci]).cuda()))
    assert lay.status() == 0
    lay.assert_caches_match()
    want = ora.results()
    for ci in range(n_chunks):
        r, w = want[ci * C]
        assert np.array_equal(r, rows[ci])
        assert_close(got[ci * C], w, "bf16", f"chunk {ci} ({len(r)} rows)")


def test_exp2_fma_probe_error_bound(duo):
    """The FMA-pipe exponential that the pre-fill softmax uses for one pair in
    four, against 2^x in float64 over the range the softmax feeds it
    (x <= 8: the lazily raised row maximum lags the true one by at most 2^8):
    relative error below 1e-4, far inside the 2^-9 half-step of the bf16
    probabilities it produces; inputs below -125 (masked keys: -inf) give the
    value at -125.  An odd count exercises the unpaired last element."""
    t = torch()
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-125.0, 8.0, 266001), rng.uniform(-125.0, 8.0, 100000),
                        [-0.5, 0.5, -1.5, 0.0, 8.0, -125.0, -125.5, -126.0, -1000.0, -np.inf]]).astype(np.float32)
    assert x.size % 2 == 1
    xd = t.from_numpy(x).cuda()
    yd = t.full_like(xd, float("nan"))
    duo.exp2_fma_probe(xd, yd, x.size)
    y = yd.cpu().numpy().astype(np.float64)
    inside = x >= -125.0
    rel = np.abs(y[inside] / np.exp2(x[inside].astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4, f"max relative error {rel.max():.3e} at x = {x[inside][rel.argmax()]}"
    # below the clamp every input gives the value at -125: 2^-125 within the same bound
    assert np.all(y[~inside] == y[x == -125.0][0])
    assert abs(y[~inside][0] / 2.0 ** -125 - 1.0) < 1e-4
