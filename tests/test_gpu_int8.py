"""GPU parity of the 8-bit retrieval cache: duo_append_kv quantizes the
retrieval heads' rows into codes and scales bit-exactly as the oracle does
(per-row symmetric, round half to even, every step one fp32 operation), and
decode over the 8-bit cache matches the oracle's decode over code * scale
within the bf16 tolerances (max-abs 2e-2, mean-abs 2e-3)."""

import numpy as np
import pytest

from head_split_kv_b200 import synthetic as S
from tests.gpu_helpers import Layer, assert_close, prefill_run, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    t.cuda.synchronize()


def _layer(duo, sh, retrieval, B, capacity):
    return Layer(duo, sh, retrieval, B, capacity=capacity, kv_quant=duo.KV_INT8)


def _append_prompt(lay, sh, n, chunks, B, seed, sigma=None):
    _, k, v = S.prompt(sh, n, seed=seed, batch=B, sigma=sigma)
    c0 = 0
    for C in chunks:
        lay.append(k[:, c0:c0 + C], v[:, c0:c0 + C])
        c0 += C
    assert c0 == n


@pytest.mark.parametrize("chunks", [[700], [256, 300, 1, 143], [64] * 11])
def test_int8_append_is_bit_exact(duo, chunks):
    sh = S.LayerShape(16, 4, 128, "bf16")
    n = sum(chunks)
    lay = _layer(duo, sh, [0, 2], 2, n + 64)
    _append_prompt(lay, sh, n, chunks, 2, seed=11, sigma=S.head_sigma(4))
    lay.assert_caches_match()
    assert lay.status() == 0


@pytest.mark.parametrize("hq,hkv,retrieval", [(8, 8, [1, 5]), (8, 4, [0, 3]), (16, 4, [1, 2]), (16, 2, [1])])
@pytest.mark.parametrize("fused", [False, True])
def test_int8_decode_matches_oracle(duo, hq, hkv, retrieval, fused):
    sh = S.LayerShape(hq, hkv, 128, "bf16")
    B, n, steps = 2, 1000, 6
    lay = _layer(duo, sh, retrieval, B, n + steps + 64)
    _append_prompt(lay, sh, n, [512, 488], B, seed=12)
    qs, ks, vs = S.decode_steps(sh, B, steps, seed=12)
    for i in range(steps):
        got, want = lay.decode(qs[i], ks[i], vs[i], fused=fused)
        assert_close(got, want, "bf16", f"step {i}")
    lay.assert_caches_match()
    assert lay.status() == 0


def test_int8_decode_long_context(duo):
    """A 20K-token history on the Llama-3-8B-shaped GQA layer: many tiles per
    split, splits whose last tile is partial."""
    sh = S.LayerShape(32, 8, 128, "bf16")
    B, n = 1, 20000
    retrieval = S.retrieval_heads_by_seed(8, 4)
    lay = _layer(duo, sh, retrieval, B, n + 64)
    _append_prompt(lay, sh, n, [4096] * 4 + [3616], B, seed=13, sigma=S.head_sigma(8))
    qs, ks, vs = S.decode_steps(sh, B, 3, seed=13, sigma=S.head_sigma(8))
    for i in range(3):
        got, want = lay.decode(qs[i], ks[i], vs[i], fused=True)
        assert_close(got, want, "bf16", f"step {i}")
    assert lay.status() == 0


@pytest.mark.parametrize("chunks", [[300, 300, 100], [128] * 5 + [60], [4096, 4096], [301, 250, 99, 130]])
def test_int8_prefill_reads_the_quantized_cache(duo, chunks):
    """duo_prefill_chunk on a layer with a 8-bit full cache: the prior
    rows widened to bf16 code * scale in the workspace's staging area, the
    chunk's own rows as given -- against the oracle's pre-fill from its
    8-bit caches; the caches filled by the appends stay byte-exact."""
    sh = S.LayerShape(32, 8, 128, "bf16")
    retrieval = S.retrieval_heads_by_seed(8, 4)
    n = sum(chunks)
    lay = _layer(duo, sh, retrieval, 1, n + 64)
    prefill_run(lay, chunks, seed=38, sigma=S.head_sigma(8), rows_per_chunk=256)
    lay.assert_caches_match()
