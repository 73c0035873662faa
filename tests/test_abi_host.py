"""The C-ABI library on the host: it loads, exports every symbol include/duo.h
declares, its struct layouts match the C compiler's, and its host-side logic
(gate binarisation, head partition, argument checks) behaves -- all without a
GPU: every call here returns before anything is queued on a device."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "duo.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(duo_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ["duo_partition_heads", "duo_permute_heads", "duo_append_kv", "duo_decode_attn",
                 "duo_prefill_chunk", "duo_gated_mix", "duo_workspace_bytes", "duo_last_error"]:
        assert want in names


def test_library_exports_every_declared_symbol(duo):
    out = subprocess.run(["nm", "-D", "--defined-only", duo.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\s[TW]\s(duo_\w+)", out.stdout))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, f"declared in duo.h but not exported: {missing}"
    lib = ctypes.CDLL(duo.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n)


def test_debug_bounds_library_exports_the_same_symbols(duo):
    """libduo_debug.so (the build with device index checks, built beside
    libduo.so) exports every declared entry point too, and the binding loads
    it in a process whose environment asks for it."""
    debug = os.path.join(os.path.dirname(duo.LIB_PATH), "libduo_debug.so")
    assert os.path.exists(debug), "build both libraries: python -m head_split_kv_b200.build [--debug-bounds]"
    out = subprocess.run(["nm", "-D", "--defined-only", debug], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\s[TW]\s(duo_\w+)", out.stdout))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, f"declared in duo.h but not exported by the debug build: {missing}"
    probe = ("import head_split_kv_b200.duo as d; "
             "print(d.LIB_PATH.endswith('libduo_debug.so'), d.abi_version(), d.DEV_BOUNDS)")
    r = subprocess.run([os.sys.executable, "-c", probe], cwd=ROOT, capture_output=True, text=True, check=True,
                       env={**os.environ, "DUO_DEBUG_BOUNDS": "1"})
    assert r.stdout.split() == ["True", str(duo.ABI_VERSION), "16"]


def test_struct_layouts_match_the_c_compiler(duo, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "duo.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\\n", sizeof(duo_layer_desc), offsetof(duo_layer_desc, scale),
         offsetof(duo_layer_desc, kv_perm), sizeof(duo_kv_state), offsetof(duo_kv_state, k_ring));
  printf("%zu %zu %zu\\n", offsetof(duo_kv_state, seq_len), offsetof(duo_kv_state, counters),
         offsetof(duo_kv_state, status));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    a, b = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")[:2]
    L, K = duo.LayerDesc, duo.KVState
    assert [int(x) for x in a.split()] == [ctypes.sizeof(L), L.scale.offset, L.kv_perm.offset,
                                           ctypes.sizeof(K), K.k_ring.offset]
    assert [int(x) for x in b.split()] == [K.seq_len.offset, K.counters.offset, K.status.offset]


def test_abi_version_and_status_strings(duo):
    assert duo.abi_version() == duo.ABI_VERSION == 4
    assert duo.status_string(duo.OK) == "DUO_OK"
    assert duo.status_string(duo.ERR_CAPACITY) == "DUO_ERR_CAPACITY"


# ---------------------------------------------------------------------------
# Gate binarisation + partition: bit-exact against the oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(20))
def test_partition_matches_oracle(duo, seed):
    rng = np.random.default_rng(seed)
    hkv = int(rng.integers(1, 65))
    alpha = rng.uniform(0, 1, hkv).astype(np.float32)
    if seed % 3 == 0:  # ties and values exactly at tau
        alpha = rng.choice(np.array([0.0, 0.25, 0.5, 0.75, 1.0], dtype=np.float32), hkv)
    tau = float(np.float32(0.5))
    for target in (-1, 0, hkv // 4, hkv // 2, hkv):
        g, p, ip, n = duo.partition_heads(alpha, tau, target)
        og, op, oip, on = O.partition_heads(alpha.astype(np.float64), tau, target)
        assert g == list(og) and p == list(op) and ip == list(oip) and n == on


def test_partition_rejects_bad_arguments(duo):
    with pytest.raises(duo.DuoError) as e:
        duo.partition_heads([0.1] * 65, 0.5)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.partition_heads([0.1, float("nan")], 0.5)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.partition_heads([0.1, 0.2], 0.5, target_n_retrieval=3)
    assert e.value.status == duo.ERR_SHAPE


# ---------------------------------------------------------------------------
# Descriptor checks
# ---------------------------------------------------------------------------

def _desc(duo, **kw):
    args = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, dtype=duo.BF16,
                kv_perm=list(range(8)), n_retrieval=4)
    args.update(kw)
    return duo.desc_init(**args)


def test_desc_defaults(duo):
    d = _desc(duo)
    assert (d.sink, d.recent, d.page_size, d.io_order) == (16, 64, 0, duo.ORDER_MODEL)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), "ERR_SHAPE"),
    (dict(n_q_heads=30), "ERR_SHAPE"),
    (dict(n_q_heads=24), "ERR_UNSUPPORTED"),         # group of 3
    (dict(head_dim=96), "ERR_UNSUPPORTED"),
    (dict(head_dim=0), "ERR_SHAPE"),
    (dict(dtype=7), "ERR_DTYPE"),
    (dict(n_retrieval=9), "ERR_SHAPE"),
    (dict(kv_perm=[0, 1, 2, 3, 4, 5, 6, 6]), "ERR_INVALID_ARG"),
    (dict(kv_perm=[0, 1, 2, 3, 4, 5, 6, 8]), "ERR_INVALID_ARG"),
    (dict(page_size=32), "ERR_UNSUPPORTED"),
    (dict(sink=-1), "ERR_SHAPE"),
    (dict(recent=0), "ERR_SHAPE"),
])
def test_desc_rejections(duo, kw, status):
    with pytest.raises(duo.DuoError) as e:
        _desc(duo, **kw)
    assert e.value.status == getattr(duo, status)
    assert duo.last_error()


def test_workspace_bytes(duo):
    d = _desc(duo)
    n = duo.workspace_bytes(d, duo.OP_DECODE, 131072 + 64)
    assert n >= 4 * 4 * 130 * 4 and n % 256 == 0
    assert duo.workspace_bytes(d, 99, 0) == 0


def _prefill_plan_bytes(units, n_sms=148, max_split=8, part_floats=2 * 128 + 128 * 128):
    """The pre-fill key-split plan restated: the smallest split count whose
    units * ns CTAs fill their waves of n_sms to 95 % (else the fullest), and
    the workspace it needs -- per split and query tile a partial record, then
    a ticket word per unit, each region rounded up to 256 bytes."""
    best, ns = 0.0, 1
    for k in range(1, max_split + 1):
        items = units * k
        fill = items / (-(-items // n_sms) * n_sms)
        if fill > best + 1e-9:
            best, ns = fill, k
        if fill >= 0.95:
            break
    if ns == 1:
        return 256
    part = units * ns * 2 * part_floats * 4
    return -(-part // 256) * 256 + -(-(units * 4) // 256) * 256


@pytest.mark.parametrize("hq,hkv,R,B,chunk", [(32, 8, 4, 1, 4096), (32, 32, 8, 1, 4096), (32, 8, 2, 1, 49152),
                                              (16, 4, 2, 3, 1000), (8, 8, 8, 64, 4096)])
def test_prefill_workspace_follows_the_split_plan(duo, hq, hkv, R, B, chunk):
    # a workspace sized for `chunk` serves every shorter chunk, so it is the
    # largest plan over 1 .. ceil(chunk / 256) query-tile pairs
    d = duo.desc_init(B, hq, hkv, 128, duo.BF16, list(range(hkv)), R)
    want = max(_prefill_plan_bytes(B * R * (hq // hkv) * mp) for mp in range(1, -(-chunk // 256) + 1))
    assert duo.workspace_bytes(d, duo.OP_PREFILL, chunk) == max(want, 256)


def test_prefill_workspace_plans_at_the_bench_shape(duo):
    # 4,096-token chunks of the GQA layer with 4 of 8 KV heads retrieval: 256
    # units, 4 splits each (1,024 CTAs in 6.92 waves of 148)
    assert _prefill_plan_bytes(4 * 4 * 16) == 256 * 4 * 2 * 16640 * 4 + 1024
    d32 = duo.desc_init(1, 8, 8, 64, duo.FP32, list(range(8)), 2)
    assert duo.workspace_bytes(d32, duo.OP_PREFILL, 4096) == 256   # the CUDA-core path splits nothing


def test_exp2_probe_rejects_bad_arguments(duo):
    with pytest.raises(duo.DuoError) as e:
        duo.exp2_fma_probe(0, 0, -1, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.exp2_fma_probe(0, 256, 8, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    duo.exp2_fma_probe(0, 0, 0, stream=0)   # nothing to do: no launch


# ---------------------------------------------------------------------------
# Device entry points reject bad arguments on the host, before any launch
# ---------------------------------------------------------------------------

def _state(duo, **kw):
    st = duo.KVState()
    for k, v in dict(k_full=16, v_full=32, capacity=1024, k_ring=48, v_ring=64, ring_pos=80,
                     seq_len=96, counters=112, status=128).items():
        setattr(st, k, v)
    for k, v in kw.items():
        setattr(st, k, v)
    return st


def test_append_rejects(duo):
    d = _desc(duo)
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo, seq_len=None), 256, 512, 1, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo), 256, 512, -1, stream=0)
    assert e.value.status == duo.ERR_SHAPE
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo), 255, 512, 1, stream=0)     # misaligned
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo, capacity=0), 256, 512, 1, stream=0)
    assert e.value.status == duo.ERR_SHAPE
    duo.append_kv(d, _state(duo), 256, 512, 0, stream=0)         # T = 0: nothing to do


def test_decode_rejects_small_workspace(duo):
    d = _desc(duo)
    need = duo.workspace_bytes(d, duo.OP_DECODE, 1024)
    with pytest.raises(duo.DuoError) as e:
        duo.decode_attn(d, _state(duo), 256, 512, 1024, need - 16, stream=0)
    assert e.value.status == duo.ERR_CAPACITY
    with pytest.raises(duo.DuoError) as e:
        duo.decode_attn(d, _state(duo), 256, 512, None, need, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG


def test_paged_state_checks(duo):
    d = _desc(duo, page_size=64)
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo), 256, 512, 1, stream=0)      # no page table
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, _state(duo, page_table=144, max_pages=4, n_pages=8, capacity=300), 256, 512, 1, stream=0)
    assert e.value.status == duo.ERR_SHAPE


def test_prefill_rejects(duo):
    d = _desc(duo)
    with pytest.raises(duo.DuoError) as e:
        duo.prefill_chunk(d, _state(duo), 256, 512, 768, 0, 1024, stream=0)
    assert e.value.status == duo.ERR_SHAPE
    with pytest.raises(duo.DuoError) as e:
        duo.prefill_chunk(_desc(duo, page_size=64), _state(duo, page_table=144, max_pages=16, n_pages=16),
                          256, 512, 768, 64, 1024, stream=0)
    assert e.value.status == duo.ERR_UNSUPPORTED


def test_gated_mix_rejects(duo):
    d = _desc(duo)
    with pytest.raises(duo.DuoError) as e:
        duo.gated_mix(d, None, 256, 512, 768, 10, 1024, 2048, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:                          # the status word is required
        duo.gated_mix(d, 16, 256, 512, 768, 10, 1024, None, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    with pytest.raises(duo.DuoError) as e:
        duo.gated_mix_grad_alpha(d, 256, 512, 768, 10, 1024, 2048, None, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
    duo.gated_mix(d, 16, 256, 512, 768, 0, 1024, 2048, stream=0)       # N = 0: nothing to do


def test_gated_mix_rejects_out_overlapping_an_input(duo):
    # 32 query / 8 KV heads, d 128, bf16, 10 tokens: q and out are 80 KB, k
    # and v 20 KB; the check runs on the host, before any launch
    d = _desc(duo)
    q, k, v = 1 << 20, 2 << 20, 3 << 20
    for out in (q, q + 4096, k - 4096, v + 16):
        with pytest.raises(duo.DuoError) as e:
            duo.gated_mix(d, 16, q, k, v, 10, out, 64, stream=0)
        assert e.value.status == duo.ERR_INVALID_ARG
        assert "overlaps" in duo.last_error()


def test_wait_probe_rejects(duo):
    for status, limit in ((None, 10), (64, 0), (64, 1000001)):
        with pytest.raises(duo.DuoError) as e:
            duo.wait_probe(status, limit, stream=0)
        assert e.value.status == duo.ERR_INVALID_ARG


def test_permute_rejects_overlap(duo):
    d = _desc(duo)
    with pytest.raises(duo.DuoError) as e:
        duo.permute_heads(d, 4096, 4096 + 64, 4, 4, 128, 2, duo.MODEL_TO_BLOCK, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG


def test_stream_prefill_mode_is_validated(duo):
    d = duo.desc_init(1, 8, 4, 128, duo.BF16, [0, 1, 2, 3], 2, stream_prefill=duo.STREAM_CHUNK)
    assert d.stream_prefill == duo.STREAM_CHUNK and duo.desc_validate(d) == duo.OK
    assert duo.desc_init(1, 8, 4, 128, duo.BF16, [0, 1, 2, 3], 2).stream_prefill == duo.STREAM_LAMBDA
    d.stream_prefill = 2
    assert duo.desc_validate(d) == duo.ERR_INVALID_ARG


def test_int8_cache_is_validated(duo):
    perm = [0, 1, 2, 3]
    d = duo.desc_init(1, 8, 4, 128, duo.BF16, perm, 2, kv_quant=duo.KV_INT8)
    assert d.kv_quant == duo.KV_INT8
    with pytest.raises(duo.DuoError) as e:
        duo.desc_init(1, 8, 4, 64, duo.BF16, perm, 2, kv_quant=duo.KV_INT8)
    assert e.value.status == duo.ERR_UNSUPPORTED
    with pytest.raises(duo.DuoError) as e:
        duo.desc_init(1, 8, 4, 128, duo.FP32, perm, 2, kv_quant=duo.KV_INT8)
    assert e.value.status == duo.ERR_UNSUPPORTED
    d.kv_quant = duo.KV_INT4
    assert duo.desc_validate(d) == duo.OK
    with pytest.raises(duo.DuoError) as e:
        duo.desc_init(1, 8, 4, 64, duo.BF16, perm, 2, kv_quant=duo.KV_INT4)
    assert e.value.status == duo.ERR_UNSUPPORTED
    d.kv_quant = 3
    assert duo.desc_validate(d) == duo.ERR_INVALID_ARG


def test_quantized_prefill_needs_its_staging_workspace(duo):
    """An 8- or 4-bit layer's pre-fill reads its prior rows from a staging
    area in the workspace: without one, or with one smaller than the staging
    area, the call is refused before anything is queued; the size query
    counts, on top of the plain layer's workspace, 512 bytes of codes per
    token of the capacity and retrieval head and two rows of capacity + 4
    fp32 scales per retrieval head, rounded up to 256 bytes."""
    for quant in (duo.KV_INT8, duo.KV_INT4):
        d = duo.desc_init(1, 8, 4, 128, duo.BF16, [0, 1, 2, 3], 2, kv_quant=quant)
        st = _state(duo)
        st.k_scale, st.v_scale = 4096, 8192
        st.capacity = 1024
        plain = duo.workspace_bytes(d, duo.OP_PREFILL, 16)
        staging = 1 * 2 * 1024 * (2 * 128 * 2) + 1 * 2 * 2 * (1024 + 4) * 4
        assert duo.prefill_workspace_bytes(d, st, 16) == plain + (staging + 255) // 256 * 256
        for ws, nbytes in ((None, 0), (1 << 20, 1 << 19)):
            with pytest.raises(duo.DuoError) as e:
                duo.prefill_chunk(d, st, 256, 512, 768, 16, 1024, ws, nbytes, stream=0)
            assert e.value.status == duo.ERR_CAPACITY
    st = _state(duo)
    st.k_scale, st.v_scale = 4096, 8192
    st.capacity = 1024
    # the state must carry the scales and a capacity in whole 64-token tiles
    st.capacity = 1000
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, st, 256, 512, 1, stream=0)
    assert e.value.status == duo.ERR_SHAPE
    st.capacity, st.k_scale = 1024, None
    with pytest.raises(duo.DuoError) as e:
        duo.append_kv(d, st, 256, 512, 1, stream=0)
    assert e.value.status == duo.ERR_INVALID_ARG
