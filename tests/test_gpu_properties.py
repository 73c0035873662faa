"""Property tests on seeded random small layers: the whole path -- chunked
pre-fill (or, for a paged cache, the prompt appended in chunks), then decode
steps, separate or fused -- against the oracle, on shapes drawn across what
the library builds:

* head_dim 64 or 128, bf16 or fp32; query groups of 1, 2, 4 or 8;
* any subset of retrieval KV heads (none and all included);
* sink / recent pairs other than 16 / 64 (a zero sink among them);
* prompt lengths that straddle sink, sink + recent, the 64-token tile and
  page sizes, and the 128-row pre-fill tiles, cut into random chunks;
* contiguous and 64-token paged caches, 8- and 4-bit retrieval caches;
* model and block head order; per-query and whole-chunk streaming pre-fill.

Every case checks each pre-fill chunk's rows and each decode output against
the oracle within the stated tolerances, and the caches byte for byte at the
end.  The cases are drawn once from a fixed seed, so the set is the same on
every run."""

import numpy as np
import pytest

from head_split_kv_b200 import synthetic as S
from gpu_helpers import Layer, assert_close, prefill_run, torch

pytestmark = pytest.mark.gpu

N_CASES = 36


def _boundary_lengths(sink, recent):
    w = sink + recent
    base = [1, 2, sink - 1, sink, sink + 1, w - 1, w, w + 1, 63, 64, 65, 127, 128, 129, 255, 257]
    return sorted({n for n in base if n >= 1})


def _cases():
    rng = np.random.default_rng(20240611)
    out = []
    while len(out) < N_CASES:
        d = int(rng.choice([64, 128]))
        dtype = str(rng.choice(["bf16", "fp32"]))
        g = int(rng.choice([1, 2, 4, 8]))
        hkv = int(rng.choice([1, 2, 4, 8]))
        if hkv * g > 32:
            continue
        sink, recent = [(16, 64), (2, 3), (0, 5), (4, 8), (20, 100), (1, 127)][int(rng.integers(6))]
        quant = 0
        if dtype == "bf16" and d == 128 and rng.random() < 0.35:
            quant = int(rng.choice([8, 4]))
        paged = quant == 0 and rng.random() < 0.25
        n_ret = int(rng.integers(0, hkv + 1))
        retrieval = sorted(rng.choice(hkv, n_ret, replace=False).tolist())
        if rng.random() < 0.6:
            n = int(rng.choice(_boundary_lengths(sink, recent)))
        else:
            n = int(rng.integers(100, 700))
        n_chunks = int(rng.integers(1, 5))
        cuts = sorted(set(rng.integers(1, n, size=n_chunks - 1).tolist())) if n > 1 else []
        chunks = [b - a for a, b in zip([0] + cuts, cuts + [n])]
        out.append(dict(
            d=d, dtype=dtype, g=g, hkv=hkv, sink=sink, recent=recent, quant=quant, paged=paged,
            retrieval=retrieval, B=int(rng.integers(1, 3)), chunks=chunks, steps=int(rng.integers(1, 4)),
            fused=bool(rng.random() < 0.5), block_order=bool(rng.random() < 0.3),
            chunk_mode=bool(rng.random() < 0.25), seed=int(rng.integers(1 << 30))))
    return out


CASES = _cases()


def _case_id(c):
    return (f"{c['dtype']}-d{c['d']}-G{c['g']}-R{len(c['retrieval'])}of{c['hkv']}-s{c['sink']}r{c['recent']}"
            f"-B{c['B']}-n{sum(c['chunks'])}x{len(c['chunks'])}"
            + (f"-q{c['quant']}" if c["quant"] else "") + ("-paged" if c["paged"] else "")
            + ("-block" if c["block_order"] else "") + ("-wholechunk" if c["chunk_mode"] else "")
            + ("-fused" if c["fused"] else ""))


@pytest.mark.parametrize("case", CASES, ids=[_case_id(c) for c in CASES])
def test_random_layer_prefill_then_decode(duo, case):
    c = case
    sh = S.LayerShape(c["hkv"] * c["g"], c["hkv"], c["d"], c["dtype"], sink=c["sink"], recent=c["recent"])
    n, steps, B = sum(c["chunks"]), c["steps"], c["B"]
    io_order = duo.ORDER_BLOCK if c["block_order"] else duo.ORDER_MODEL
    stream_prefill = duo.STREAM_CHUNK if c["chunk_mode"] else duo.STREAM_LAMBDA
    if c["paged"]:
        table, n_pages = S.page_assignment([n] * B, steps, 64, seed=c["seed"] % 1000)
        lay = Layer(duo, sh, c["retrieval"], B, page_size=64, page_table=table, n_pages=n_pages,
                    io_order=io_order, stream_prefill=stream_prefill)
        _, k, v = S.prompt(sh, n, seed=c["seed"], batch=B)
        c0 = 0
        for C in c["chunks"]:
            lay.append(k[:, c0:c0 + C], v[:, c0:c0 + C])
            c0 += C
    else:
        kv_quant = {0: duo.KV_PLAIN, 8: duo.KV_INT8, 4: duo.KV_INT4}[c["quant"]]
        cap = (n + steps + 63) // 64 * 64
        lay = Layer(duo, sh, c["retrieval"], B, capacity=cap, io_order=io_order, stream_prefill=stream_prefill,
                    kv_quant=kv_quant)
        prefill_run(lay, c["chunks"], seed=c["seed"])
    qs, ks, vs = S.prompt(sh, steps, seed=c["seed"] + 1, batch=B)
    for i in range(steps):
        got, want = lay.decode(qs[:, i], ks[:, i], vs[:, i], fused=c["fused"])
        assert_close(got, want, c["dtype"], f"{_case_id(c)}: decode step {i}")
    torch().cuda.synchronize()
    assert lay.status() == 0
    lay.assert_caches_match()
