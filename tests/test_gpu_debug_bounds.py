"""The debug build (libduo_debug.so, compiled with DUO_DEBUG_BOUNDS): the
same kernels with device index checks at every computed-address write and
every untiled bulk read, which on failure set DUO_DEV_BOUNDS and skip the
access instead of faulting.

Run side by side with the release library in one process (a second copy of
the binding bound to the debug library) over small cases that reach every
kernel -- tensor-core and CUDA-core pre-fill, the pre-fill key-range splits,
appends to contiguous and paged caches, the fused decode step over bf16, 8-
and 4-bit caches, the gated mix and its gradient -- no check fires (the
status words stay 0), the caches match the oracle byte for byte, the pre-fill and
gated-mix outputs are bit-identical to the release build's (their reduction
order is fixed), the decode outputs of both builds are within the parity
bound of the oracle (the decode's drawn tiles change which split holds which
keys from run to run, and with it each p's bf16 rounding), and the gate
gradients agree to 1e-5 (float atomics).

Making a check fire on purpose would need an out-of-range index on the GPU,
and a check that failed to catch it would fault; the checks are therefore
shown not to fire and not to change results, and their placement is
reviewed in the source."""

import importlib.util
import os

import numpy as np
import pytest

from head_split_kv_b200 import synthetic as S
from gpu_helpers import Layer, assert_close, bits, f64, to_dev, torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def duo_debug():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    path = os.path.join(ROOT, "head_split_kv_b200", "duo.py")
    old = os.environ.get("DUO_DEBUG_BOUNDS")
    os.environ["DUO_DEBUG_BOUNDS"] = "1"
    try:
        spec = importlib.util.spec_from_file_location("duo_debug_binding", path)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        if old is None:
            del os.environ["DUO_DEBUG_BOUNDS"]
        else:
            os.environ["DUO_DEBUG_BOUNDS"] = old
    assert mod.LIB_PATH.endswith("libduo_debug.so")
    yield mod
    t.cuda.synchronize()


# (name, shape, retrieval KV heads, batch, pre-fill chunks, decode steps,
#  paged, 8/4-bit cache)
CASES = [
    # 128 retrieval units per 4,096-token chunk, planned at 8 splits; over
    # the 16K history a unit has 160 key tiles and takes 3
    ("bf16 GQA, tensor-core pre-fill with key splits", S.LayerShape(32, 8, 128, "bf16"), [2, 5], 1,
     [16384, 4096], 3, False, 0),
    ("bf16 MHA, paged cache", S.LayerShape(8, 8, 128, "bf16"), [0, 3, 5], 2, [150, 90], 3, True, 0),
    ("8-bit cache", S.LayerShape(16, 4, 128, "bf16"), [1, 2], 1, [200, 130], 3, False, 8),
    ("4-bit cache", S.LayerShape(16, 4, 128, "bf16"), [0, 3], 2, [256, 70], 3, False, 4),
    ("fp32, head_dim 64 (CUDA cores)", S.LayerShape(8, 4, 64, "fp32"), [2], 1, [100, 60], 2, False, 0),
]


def _run_case(duo, case, seed):
    """Pre-fill and append the chunks, then fused decode steps, each checked
    against the oracle; returns the pre-fill outputs (float64) and the status
    word after checking the caches against the oracle twin."""
    t = torch()
    name, sh, retrieval, B, chunks, steps, paged, bits_ = case
    n = sum(chunks)
    kv_quant = {0: duo.KV_PLAIN, 8: duo.KV_INT8, 4: duo.KV_INT4}[bits_]
    if paged:
        table, n_pages = S.page_assignment([n] * B, steps, 64, seed=seed)
        lay = Layer(duo, sh, retrieval, B, page_size=64, page_table=table, n_pages=n_pages)
    else:
        lay = Layer(duo, sh, retrieval, B, capacity=(n + steps + 63) // 64 * 64, kv_quant=kv_quant)
    q, k, v = S.prompt(sh, n + steps, seed=seed, batch=B)
    outs = []
    if not paged:
        # the pre-fill reads contiguous caches only; a paged layer is filled by appends
        ws = duo.Workspace(lay.desc, duo.OP_PREFILL, max(chunks), state=lay.caches.state)
        c0 = 0
        for C in chunks:
            sl = slice(c0, c0 + C)
            qd, kd, vd = (to_dev(np.ascontiguousarray(x[:, sl])) for x in (q, k, v))
            out = t.empty_like(qd)
            duo.prefill_chunk(lay.desc, lay.caches.state, qd, kd, vd, C, out, ws.ptr, ws.nbytes)
            outs.append(f64(out))
            lay.append(k[:, sl], v[:, sl])
            c0 += C
    else:
        lay.append(k[:, :n], v[:, :n])
    for i in range(steps):
        got, want = lay.decode(q[:, n + i], k[:, n + i], v[:, n + i], fused=True)
        assert_close(got, want, sh.dtype, f"{name}: decode step {i} ({os.path.basename(duo.LIB_PATH)})")
    t.cuda.synchronize()
    status = lay.status()
    lay.assert_caches_match()
    return outs, status


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_debug_build_checks_do_not_fire_and_change_nothing(duo, duo_debug, case):
    rel, st_rel = _run_case(duo, case, seed=61)
    dbg, st_dbg = _run_case(duo_debug, case, seed=61)
    assert st_rel == 0
    assert st_dbg == 0, f"debug build status 0x{st_dbg:x} (DUO_DEV_BOUNDS = {duo.DEV_BOUNDS})"
    assert len(rel) == len(dbg)
    for i, (a, b) in enumerate(zip(rel, dbg)):
        assert np.array_equal(a, b), f"{case[0]}: pre-fill chunk {i} differs between the builds"


@pytest.mark.parametrize("dtype,hq,hkv,d,n", [("bf16", 16, 4, 128, 700), ("fp32", 8, 8, 64, 300)])
def test_debug_build_gated_mix_and_gradient(duo, duo_debug, dtype, hq, hkv, d, n):
    t = torch()
    sh = S.LayerShape(hq, hkv, d, dtype)
    q, k, v = S.prompt(sh, n, seed=62, batch=1)
    dout, _, _ = S.prompt(sh, n, seed=63, batch=1)
    alpha = S.rng_for(62, 5).uniform(0, 1, hkv).astype(np.float32)
    res = []
    for mod in (duo, duo_debug):
        desc = mod.desc_init(1, hq, hkv, d, mod.BF16 if dtype == "bf16" else mod.FP32, list(range(hkv)), 0)
        qd, kd, vd, dd = to_dev(q), to_dev(k), to_dev(v), to_dev(dout)
        out = t.empty_like(qd)
        dalpha = t.zeros(hkv, dtype=t.float32, device="cuda")
        status = t.zeros(1, dtype=t.int32, device="cuda")
        mod.gated_mix(desc, t.from_numpy(alpha).cuda(), qd, kd, vd, n, out, status)
        mod.gated_mix_grad_alpha(desc, qd, kd, vd, n, dd, dalpha, status)
        t.cuda.synchronize()
        assert status.item() == 0, f"{mod.LIB_PATH}: status 0x{status.item():x}"
        res.append((f64(out), bits(dalpha).astype(np.float64)))
    (o_rel, g_rel), (o_dbg, g_dbg) = res
    assert np.array_equal(o_rel, o_dbg), "gated mix differs between the builds"
    assert np.allclose(g_rel, g_dbg, rtol=1e-5, atol=1e-5 * np.abs(g_rel).max()), (g_rel, g_dbg)
