"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Caches, ring positions and lengths are compared bit for
bit; attention outputs within max-abs 2e-2 / mean-abs 2e-3 (bf16 inputs,
fp32 accumulation) or max-abs 1e-4 (fp32 inputs)."""

import numpy as np
import pytest

import oracle as O
from head_split_kv_b200 import synthetic as S
from tests.gpu_helpers import Layer, assert_close, bits, f64, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    t.cuda.synchronize()


# ---------------------------------------------------------------------------
# duo_append_kv: bit-exact caches
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,io_order", [("bf16", 0), ("fp32", 0), ("bf16", 1)])
def test_append_bit_exact(duo, dtype, io_order):
    sh = S.LayerShape(8, 4, 64, dtype, sink=4, recent=8)
    lay = Layer(duo, sh, retrieval=[1, 2], batch=2, capacity=400, io_order=io_order)
    rng = S.rng_for(3, 99)
    for T in [1, 3, 1, 13, 2, 40, 1, 1, 7, 100, 0, 5]:
        k = S.normal(rng, (2, T, 4, 64), dtype)
        v = S.normal(rng, (2, T, 4, 64), dtype)
        if T:
            lay.append(k, v)
        lay.assert_caches_match()
    assert lay.status() == 0


def test_append_paged_bit_exact(duo):
    sh = S.LayerShape(32, 32, 128, "bf16")
    # 493 tokens are appended per sequence: give each 10 pages (640 tokens)
    table, n_pages = S.page_assignment([600, 600, 600], 0, 64, seed=5)
    lay = Layer(duo, sh, retrieval=S.retrieval_heads_by_seed(32, 8), batch=3, page_size=64, page_table=table,
                n_pages=n_pages)
    rng = S.rng_for(4, 99)
    for T in [64, 1, 100, 63, 1, 64, 200]:
        k = S.normal(rng, (3, T, 32, 128), "bf16")
        v = S.normal(rng, (3, T, 32, 128), "bf16")
        lay.append(k, v)
    lay.assert_caches_match()
    assert lay.status() == 0


def test_append_overflow_sets_status_and_skips(duo):
    sh = S.LayerShape(4, 4, 64, "bf16", sink=2, recent=4)
    lay = Layer(duo, sh, retrieval=[0], batch=1, capacity=10)
    rng = S.rng_for(5, 99)
    k = S.normal(rng, (1, 12, 4, 64), "bf16")
    lay.duo.append_kv(lay.desc, lay.caches.state, to_dev(k), to_dev(k), 12)
    st = lay.status()
    assert st & duo.DEV_FULL_CACHE_OVERFLOW
    got = bits(lay.caches.k_full)[0, 0]
    assert np.array_equal(got[:10], k[0, :10, 0])


# ---------------------------------------------------------------------------
# duo_decode_attn
# ---------------------------------------------------------------------------

def _decode_run(duo, sh, retrieval, lengths, steps, check_steps, capacity=None, paged=False, io_order=None,
                sigma=None, seed=0, fused=False):
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    cap = int(lengths.max()) + steps if capacity is None else capacity
    if paged:
        table, n_pages = S.page_assignment(lengths, steps, 64, seed=seed)
        lay = Layer(duo, sh, retrieval, B, page_size=64, page_table=table, n_pages=n_pages, io_order=io_order)
    else:
        lay = Layer(duo, sh, retrieval, B, capacity=cap, io_order=io_order)
    lay.load_state(S.decode_state(sh, retrieval, lengths, seed=seed, sigma=sigma))
    qs, ks, vs = S.decode_steps(sh, B, steps, seed=seed, sigma=sigma)
    errs = []
    for i in range(steps):
        check = i in check_steps
        got, want = lay.decode(qs[i], ks[i], vs[i], check_oracle=check, fused=fused)
        if check:
            errs.append(assert_close(got, want, sh.dtype, f"step {i}"))
    assert lay.status() == 0
    return lay, errs


def test_decode_tiny_fp32(duo):
    sh = S.LayerShape(8, 8, 64, "fp32")
    _decode_run(duo, sh, [1, 5], [512], 16, set(range(16)))


@pytest.mark.parametrize("L0", [0, 1, 15, 16, 17, 79, 80, 81, 200, 4097])
def test_decode_lengths_around_boundaries(duo, L0):
    sh = S.LayerShape(8, 4, 128, "bf16")
    lay, _ = _decode_run(duo, sh, [0, 3], [L0], 3, {0, 1, 2})
    lay.assert_caches_match()


@pytest.mark.parametrize("io_order", [0, 1])
def test_decode_mha_bf16(duo, io_order):
    sh = S.LayerShape(32, 32, 128, "bf16")
    _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), [5000], 6, {0, 3, 5}, io_order=io_order)


@pytest.mark.parametrize("G", [2, 4, 8])
def test_decode_gqa_bf16(duo, G):
    sh = S.LayerShape(8 * G, 8, 128, "bf16")
    _decode_run(duo, sh, S.retrieval_heads_by_seed(8, 4), [20011], 4, {0, 3}, sigma=S.head_sigma(8))


def test_decode_all_streaming_and_all_retrieval(duo):
    sh = S.LayerShape(16, 4, 64, "bf16")
    _decode_run(duo, sh, [], [300], 3, {0, 2})
    _decode_run(duo, sh, [0, 1, 2, 3], [300], 3, {0, 2})


def test_decode_batch_paged(duo):
    sh = S.LayerShape(32, 32, 128, "bf16")
    lengths = S.context_lengths(6, 1, 3000, seed=2)
    lengths[0] = 0
    _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), lengths, 3, {0, 2}, paged=True)


def test_decode_batch_contiguous_fp32_d128(duo):
    sh = S.LayerShape(8, 2, 128, "fp32")
    _decode_run(duo, sh, [1], [100, 1000, 37], 2, {0, 1})


def test_decode_workspace_reuse_leaves_tickets_zero(duo):
    sh = S.LayerShape(32, 8, 128, "bf16")
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(8, 4), [3000], 5, {4})
    ws = bits(lay.ws.buf)
    plan_bytes = lay.ws.nbytes
    # the ticket words sit at the end of the workspace; all must be zero again
    assert np.all(ws[plan_bytes - 256:plan_bytes] == 0)


# ---------------------------------------------------------------------------
# duo_decode_step: append + decode in one launch
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L0", [0, 1, 15, 16, 17, 63, 64, 79, 80, 81, 4097])
def test_decode_step_boundaries(duo, L0):
    sh = S.LayerShape(8, 4, 128, "bf16")
    lay, _ = _decode_run(duo, sh, [0, 3], [L0], 4, {0, 1, 2, 3}, fused=True)
    lay.assert_caches_match()


@pytest.mark.parametrize("io_order", [0, 1])
def test_decode_step_mha(duo, io_order):
    sh = S.LayerShape(32, 32, 128, "bf16")
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), [5000], 6, {0, 5}, io_order=io_order,
                         fused=True)
    lay.assert_caches_match()


def test_decode_step_gqa_and_fp32(duo):
    sh = S.LayerShape(32, 8, 128, "bf16")
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(8, 4), [20011], 3, {2}, sigma=S.head_sigma(8),
                         fused=True)
    lay.assert_caches_match()
    sh = S.LayerShape(8, 8, 64, "fp32")
    lay, _ = _decode_run(duo, sh, [1, 5], [512], 16, set(range(16)), fused=True)
    lay.assert_caches_match()


def test_decode_step_paged_batch(duo):
    sh = S.LayerShape(32, 32, 128, "bf16")
    lengths = S.context_lengths(6, 1, 3000, seed=3)
    lengths[0] = 0
    lengths[1] = 63
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), lengths, 3, {0, 2}, paged=True, fused=True)
    lay.assert_caches_match()


def test_decode_step_mixed_with_separate_calls(duo):
    sh = S.LayerShape(16, 4, 128, "bf16")
    retrieval = [1, 2]
    lay = Layer(duo, sh, retrieval, 2, capacity=700)
    lay.load_state(S.decode_state(sh, retrieval, [300, 555], seed=4))
    qs, ks, vs = S.decode_steps(sh, 2, 6, seed=4)
    for i in range(6):
        got, want = lay.decode(qs[i], ks[i], vs[i], fused=(i % 2 == 0))
        assert_close(got, want, "bf16", f"step {i}")
    lay.assert_caches_match()
    assert lay.status() == 0


def test_decode_step_full_cache_overflow(duo):
    sh = S.LayerShape(4, 4, 64, "bf16")
    lay = Layer(duo, sh, [0], 1, capacity=40)
    lay.load_state(S.decode_state(sh, [0], [40], seed=6))
    qs, ks, vs = S.decode_steps(sh, 1, 1, seed=6)
    lay.decode(qs[0], ks[0], vs[0], check_oracle=False, fused=True)
    assert lay.status() & duo.DEV_FULL_CACHE_OVERFLOW


# ---------------------------------------------------------------------------
# Full-size decode workloads in the launch configuration the bench times
# ---------------------------------------------------------------------------

@pytest.mark.slow
@pytest.mark.parametrize("fused", [False, True])
def test_decode_mha_32k_full(duo, fused):
    sh = S.LayerShape(32, 32, 128, "bf16")
    lay, errs = _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), [32768], 256, {0, 1, 127, 255}, fused=fused)
    lay.assert_caches_match()


@pytest.mark.slow
@pytest.mark.parametrize("L0", [131072, 1048576])
def test_decode_gqa_long_full(duo, L0):
    """The 128K and 1M GQA decode workloads: outputs against the oracle on
    sampled steps, then every cache byte (the full caches past 2^20 rows
    included), the rings, ring positions and lengths against its lists."""
    sh = S.LayerShape(32, 8, 128, "bf16")
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(8, 4), [L0], 64, {0, 31, 63}, sigma=S.head_sigma(8),
                         fused=True)
    lay.assert_caches_match()


@pytest.mark.slow
def test_decode_batch64_paged_full(duo):
    """64 sequences of 4K..32K tokens in 64-token pages scattered over the
    pool: outputs on sampled steps, then every page against the oracle."""
    sh = S.LayerShape(32, 32, 128, "bf16")
    lengths = S.context_lengths(64, 4096, 32768, seed=0)
    lay, _ = _decode_run(duo, sh, S.retrieval_heads_by_seed(32, 8), lengths, 32, {0, 31}, paged=True, fused=True)
    lay.assert_caches_match()


# ---------------------------------------------------------------------------
# duo_prefill_chunk on the CUDA cores (fp32, d = 64) and duo_gated_mix
# ---------------------------------------------------------------------------

def _prefill_run(duo, sh, retrieval, n, chunk, B=1, seed=0, check_cache=True, stream_mode="lambda"):
    lay = Layer(duo, sh, retrieval, B, capacity=n + 8,
                stream_prefill=duo.STREAM_CHUNK if stream_mode == "chunk" else duo.STREAM_LAMBDA)
    q, k, v = S.prompt(sh, n, seed=seed, batch=B)
    t = torch()
    outs = []
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        C = c1 - c0
        qd = to_dev(np.ascontiguousarray(q[:, c0:c1]))
        kd = to_dev(np.ascontiguousarray(k[:, c0:c1]))
        vd = to_dev(np.ascontiguousarray(v[:, c0:c1]))
        out = t.empty_like(qd)
        duo.prefill_chunk(lay.desc, lay.caches.state, qd, kd, vd, C, out)
        duo.append_kv(lay.desc, lay.caches.state, kd, vd, C)
        lay.oracle.append(k[:, c0:c1], v[:, c0:c1])
        outs.append(f64(out))
        if check_cache:
            lay.assert_caches_match()
    got = np.concatenate(outs, axis=1)
    for b in range(B):
        if stream_mode == "chunk":      # the direct definition depends on where each chunk starts
            want = np.concatenate([O.prefill_direct(q[b, c0:c0 + chunk], k[b, :c0 + chunk], v[b, :c0 + chunk], c0,
                                                    np.array(lay.gate), sh.sink, sh.recent, stream_mode="chunk")
                                   for c0 in range(0, n, chunk)])
        else:
            want = O.prefill_direct(q[b], k[b], v[b], 0, np.array(lay.gate), sh.sink, sh.recent)
        assert_close(got[b], want, sh.dtype, f"prefill b={b}")
    assert lay.status() == 0
    return lay


def test_prefill_tiny_fp32(duo):
    sh = S.LayerShape(8, 8, 64, "fp32")
    _prefill_run(duo, sh, [1, 5], 512, 128)


@pytest.mark.parametrize("chunk", [1, 7, 64, 128])
def test_prefill_whole_chunk_streaming_fp32(duo, chunk):
    """The tiny fp32 layer with streaming heads in whole-chunk mode (CUDA-core path)."""
    sh = S.LayerShape(8, 8, 64, "fp32")
    _prefill_run(duo, sh, [1, 5], 512, chunk, check_cache=(chunk >= 64), stream_mode="chunk")


@pytest.mark.parametrize("chunk", [1, 7, 64, 300])
def test_prefill_simt_chunk_invariance(duo, chunk):
    sh = S.LayerShape(8, 4, 64, "bf16", sink=4, recent=16)
    _prefill_run(duo, sh, [0, 2], 300, chunk, check_cache=(chunk != 1))


def test_prefill_fp32_d128_gqa_batch(duo):
    sh = S.LayerShape(8, 2, 128, "fp32")
    _prefill_run(duo, sh, [1], 200, 96, B=2)


def test_gated_mix_tiny_fp32(duo):
    t = torch()
    w = S.tiny_prompt()
    sh = w["shape"]
    desc = duo.desc_init(1, 8, 8, 64, duo.FP32, list(range(8)), 0)
    q, k, v = (to_dev(w[x][None]) for x in ("q", "k", "v"))
    out = t.empty_like(q)
    alpha = t.from_numpy(w["alpha_mix"]).cuda()
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix(desc, alpha, q, k, v, 512, out, status)
    assert status.item() == 0
    want = O.gated_mix(w["q"], w["k"], w["v"], w["alpha_mix"].astype(np.float64), sh.sink, sh.recent)
    assert_close(f64(out)[0], want, "fp32", "gated mix")


@pytest.mark.parametrize("alpha_kind", ["uniform", "ones", "zeros"])
def test_gated_mix_bf16_gqa(duo, alpha_kind):
    t = torch()
    sh = S.LayerShape(16, 4, 128, "bf16")
    q, k, v = S.prompt(sh, 333, seed=4, batch=2)
    alpha = {"uniform": S.rng_for(4, 50).uniform(0, 1, 4), "ones": np.ones(4), "zeros": np.zeros(4)}[alpha_kind]
    alpha = alpha.astype(np.float32)
    desc = duo.desc_init(2, 16, 4, 128, duo.BF16, [0, 1, 2, 3], 0)
    out = t.empty_like(to_dev(q))
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix(desc, t.from_numpy(alpha).cuda(), to_dev(q), to_dev(k), to_dev(v), 333, out, status)
    assert status.item() == 0
    got = f64(out)
    for b in range(2):
        want = O.gated_mix(q[b], k[b], v[b], alpha.astype(np.float64), sh.sink, sh.recent)
        assert_close(got[b], want, "bf16", f"mix b={b}")


@pytest.mark.parametrize("hq,hkv,n,B", [(8, 8, 700, 1), (32, 4, 513, 2), (16, 8, 1031, 1)])
def test_gated_mix_bf16_tensor_core_path(duo, hq, hkv, n, B):
    """bf16, d 128: the causal half on the tensor cores, the streaming half and
    the mix in a second pass; several 256-row query-tile pairs with a ragged
    tail, MHA, G = 8 and G = 2, alpha ~ U(0, 1) with one gate at each end."""
    t = torch()
    sh = S.LayerShape(hq, hkv, 128, "bf16")
    q, k, v = S.prompt(sh, n, seed=8, batch=B)
    alpha = S.rng_for(8, 51).uniform(0, 1, hkv).astype(np.float32)
    alpha[0], alpha[-1] = 1.0, 0.0
    desc = duo.desc_init(B, hq, hkv, 128, duo.BF16, list(range(hkv)), 0)
    out = t.empty_like(to_dev(q))
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix(desc, t.from_numpy(alpha).cuda(), to_dev(q), to_dev(k), to_dev(v), n, out, status)
    assert status.item() == 0
    got = f64(out)
    for b in range(B):
        want = O.gated_mix(q[b], k[b], v[b], alpha.astype(np.float64), sh.sink, sh.recent)
        assert_close(got[b], want, "bf16", f"mix b={b}")


# duo_gated_mix_grad_alpha: each dalpha[kv] sums dout * (full - streaming)
# over its heads, rows and features, so its error is at most the attention
# error bound times sum |dout| of those terms: 1e-4 for fp32; for bf16 the
# mean-abs bound 2e-3 (dout is drawn independently of the rounding errors).

def _grad_check(got, want, dout64, g, tol):
    hkv = got.shape[0]
    w = np.abs(dout64).reshape(-1, hkv, g, dout64.shape[-1]).sum(axis=(0, 2, 3))
    err = np.abs(got - want)
    assert np.all(err <= tol * w), f"dalpha error {err} vs bound {tol * w}"


def test_gated_mix_grad_alpha_tiny_fp32(duo):
    t = torch()
    w = S.tiny_prompt()
    sh = w["shape"]
    desc = duo.desc_init(1, 8, 8, 64, duo.FP32, list(range(8)), 0)
    q, k, v = (to_dev(w[x][None]) for x in ("q", "k", "v"))
    dout = S.rng_for(9, 60).standard_normal((1, 512, 8, 64)).astype(np.float32)
    dalpha = t.full((8,), 7.0, dtype=t.float32, device="cuda")      # overwritten by the call
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix_grad_alpha(desc, q, k, v, 512, to_dev(dout), dalpha, status)
    assert status.item() == 0
    want = O.gated_mix_grad_alpha(w["q"], w["k"], w["v"], dout[0], sh.sink, sh.recent)
    _grad_check(dalpha.cpu().numpy().astype(np.float64), want, dout.astype(np.float64), 1, 1e-4)


def test_gated_mix_grad_alpha_bf16_gqa_batch(duo):
    t = torch()
    sh = S.LayerShape(16, 4, 128, "bf16")
    q, k, v = S.prompt(sh, 333, seed=4, batch=2)
    dout = S.normal(S.rng_for(4, 61), (2, 333, 16, 128), "bf16")
    desc = duo.desc_init(2, 16, 4, 128, duo.BF16, [0, 1, 2, 3], 0)
    dalpha = t.empty((4,), dtype=t.float32, device="cuda")
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix_grad_alpha(desc, to_dev(q), to_dev(k), to_dev(v), 333, to_dev(dout), dalpha, status)
    assert status.item() == 0
    want = sum(O.gated_mix_grad_alpha(q[b], k[b], v[b], dout[b], sh.sink, sh.recent) for b in range(2))
    _grad_check(dalpha.cpu().numpy().astype(np.float64), want, O.as_f64(dout), 4, 2e-3)


@pytest.mark.parametrize("hq,hkv,n,B", [(8, 8, 700, 1), (32, 4, 513, 2), (16, 8, 1031, 1)])
def test_gated_mix_grad_alpha_bf16_tensor_core_path(duo, hq, hkv, n, B):
    """bf16, d 128: the gate gradient from the two tensor-core launches (the
    streaming and the causal attention's dot products with dout); several
    256-row query-tile pairs with a ragged tail, MHA, G = 8 and G = 2."""
    t = torch()
    sh = S.LayerShape(hq, hkv, 128, "bf16")
    q, k, v = S.prompt(sh, n, seed=10, batch=B)
    dout = S.normal(S.rng_for(10, 63), (B, n, hq, 128), "bf16")
    desc = duo.desc_init(B, hq, hkv, 128, duo.BF16, list(range(hkv)), 0)
    dalpha = t.empty((hkv,), dtype=t.float32, device="cuda")
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix_grad_alpha(desc, to_dev(q), to_dev(k), to_dev(v), n, to_dev(dout), dalpha, status)
    assert status.item() == 0
    want = sum(O.gated_mix_grad_alpha(q[b], k[b], v[b], dout[b], sh.sink, sh.recent) for b in range(B))
    _grad_check(dalpha.cpu().numpy().astype(np.float64), want, O.as_f64(dout), hq // hkv, 2e-3)


def test_gated_mix_grad_alpha_zero_when_window_covers_sequence(duo):
    """Both attentions see every key, in the same order: the difference, and
    with it the gradient, is exactly zero."""
    t = torch()
    sh = S.LayerShape(8, 4, 64, "bf16", sink=16, recent=64)
    q, k, v = S.prompt(sh, 80, seed=5)
    dout = S.normal(S.rng_for(5, 62), (1, 80, 8, 64), "bf16")
    desc = duo.desc_init(1, 8, 4, 64, duo.BF16, [0, 1, 2, 3], 0)
    dalpha = t.empty((4,), dtype=t.float32, device="cuda")
    status = t.zeros(1, dtype=t.int32, device="cuda")
    duo.gated_mix_grad_alpha(desc, to_dev(q), to_dev(k), to_dev(v), 80, to_dev(dout), dalpha, status)
    assert status.item() == 0
    assert t.count_nonzero(dalpha).item() == 0


# ---------------------------------------------------------------------------
# duo_permute_heads
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("head_elems,elem_bytes", [(128, 2), (64, 4), (3, 2), (4096, 2)])
def test_permute_heads_roundtrip(duo, head_elems, elem_bytes):
    t = torch()
    hkv, hpk, rows = 8, 4, 5
    alpha = S.rng_for(7, 1).uniform(0, 1, hkv)
    _, perm, inv, n = duo.partition_heads(alpha, 0.5)
    desc = duo.desc_init(1, hkv * hpk, hkv, 128, duo.BF16, perm, n)
    nbytes = rows * hkv * hpk * head_elems * elem_bytes
    x = t.randint(0, 255, (nbytes,), dtype=t.uint8, device="cuda")
    y = t.empty_like(x)
    z = t.empty_like(x)
    duo.permute_heads(desc, x, y, rows, hpk, head_elems, elem_bytes, duo.MODEL_TO_BLOCK)
    duo.permute_heads(desc, y, z, rows, hpk, head_elems, elem_bytes, duo.BLOCK_TO_MODEL)
    xs = x.cpu().numpy().reshape(rows, hkv, hpk, head_elems * elem_bytes)
    ys = y.cpu().numpy().reshape(rows, hkv, hpk, head_elems * elem_bytes)
    assert np.array_equal(ys, xs[:, perm])
    assert np.array_equal(z.cpu().numpy(), x.cpu().numpy())
