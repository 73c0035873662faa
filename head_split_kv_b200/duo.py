"""Thin ctypes binding over libduo.so (include/duo.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  Tensor arguments are raw device pointers (ints) or
objects with ``data_ptr()`` (torch tensors); streams are raw ``cudaStream_t``
values, torch streams, or None for torch's current stream.

Importing this module fails with ImportError when libduo.so has not been
built; there is no other implementation to fall back to.  With
``DUO_DEBUG_BOUNDS=1`` in the environment it loads libduo_debug.so instead:
the same kernels built with device index checks, which set DEV_BOUNDS in the
status word and skip the access rather than fault
(``python -m head_split_kv_b200.build --debug-bounds``).
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_BOUNDS = os.environ.get("DUO_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libduo_debug.so" if DEBUG_BOUNDS else "libduo.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m head_split_kv_b200.build"
                      f"{' --debug-bounds' if DEBUG_BOUNDS else ''}`")

_lib = ctypes.CDLL(LIB_PATH)

# --------------------------------------------------------------- constants
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_DTYPE, ERR_CAPACITY, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE = range(8)
BF16, FP32 = 0, 1
ORDER_MODEL, ORDER_BLOCK = 0, 1
STREAM_LAMBDA, STREAM_CHUNK = 0, 1
KV_PLAIN, KV_INT8, KV_INT4 = 0, 1, 2
MODEL_TO_BLOCK, BLOCK_TO_MODEL = 0, 1
OP_DECODE, OP_PREFILL = 0, 1
DEV_FULL_CACHE_OVERFLOW, DEV_BAD_PAGE, DEV_WAIT_TIMEOUT, DEV_BAD_LENGTH, DEV_BOUNDS = 1, 2, 4, 8, 16
MAX_KV_HEADS = 64
STATE_COUNTER_WORDS = 4


class LayerDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("sink", ctypes.c_int32), ("recent", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("page_size", ctypes.c_int32), ("scale", ctypes.c_float),
        ("n_retrieval", ctypes.c_int32), ("io_order", ctypes.c_int32), ("stream_prefill", ctypes.c_int32),
        ("kv_quant", ctypes.c_int32), ("kv_perm", ctypes.c_int32 * MAX_KV_HEADS),
    ]


class KVState(ctypes.Structure):
    _fields_ = [
        ("k_full", ctypes.c_void_p), ("v_full", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
        ("capacity", ctypes.c_int32), ("max_pages", ctypes.c_int32), ("n_pages", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
        ("k_ring", ctypes.c_void_p), ("v_ring", ctypes.c_void_p), ("ring_pos", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p), ("counters", ctypes.c_void_p), ("status", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_DESC = ctypes.POINTER(LayerDesc)
_STATE = ctypes.POINTER(KVState)


def _fn(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_lib_last_error = _fn("duo_last_error", ctypes.c_char_p)
_lib_status_string = _fn("duo_status_string", ctypes.c_char_p, ctypes.c_int)
_lib_abi_version = _fn("duo_abi_version", _I32)
ABI_VERSION = 4           # the layout of LayerDesc / KVState and the signatures below
if _lib_abi_version() != ABI_VERSION:
    raise ImportError(f"{LIB_PATH} has ABI version {_lib_abi_version()}, this binding needs {ABI_VERSION}; rebuild it")
_lib_partition = _fn("duo_partition_heads", ctypes.c_int, ctypes.POINTER(ctypes.c_float), _I32, ctypes.c_float,
                     _I32, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(_I32), ctypes.POINTER(_I32),
                     ctypes.POINTER(_I32))
_lib_desc_init = _fn("duo_desc_init", ctypes.c_int, _DESC, _I32, _I32, _I32, _I32, _I32, ctypes.POINTER(_I32), _I32)
_lib_desc_validate = _fn("duo_desc_validate", ctypes.c_int, _DESC)
_lib_ws_bytes = _fn("duo_workspace_bytes", ctypes.c_size_t, _DESC, _I32, _I32)
_lib_pf_ws_bytes = _fn("duo_prefill_workspace_bytes", ctypes.c_size_t, _DESC, _STATE, _I32)
_lib_permute = _fn("duo_permute_heads", ctypes.c_int, _DESC, _P, _P, ctypes.c_int64, _I32, ctypes.c_int64, _I32,
                   _I32, _P)
_lib_append = _fn("duo_append_kv", ctypes.c_int, _DESC, _STATE, _P, _P, _I32, _P)
_lib_decode = _fn("duo_decode_attn", ctypes.c_int, _DESC, _STATE, _P, _P, _P, ctypes.c_size_t, _P)
_lib_prefill = _fn("duo_prefill_chunk", ctypes.c_int, _DESC, _STATE, _P, _P, _P, _I32, _P, _P, ctypes.c_size_t, _P)
_lib_mix = _fn("duo_gated_mix", ctypes.c_int, _DESC, _P, _P, _P, _P, _I32, _P, _P, _P)
_lib_mix_grad = _fn("duo_gated_mix_grad_alpha", ctypes.c_int, _DESC, _P, _P, _P, _I32, _P, _P, _P, _P)
_lib_wait_probe = _fn("duo_wait_probe", ctypes.c_int, _P, ctypes.c_uint32, _P)
_lib_check = _fn("duo_check_status", ctypes.c_int, _STATE, ctypes.POINTER(_I32), _P)
_lib_decode_step = _fn("duo_decode_step", ctypes.c_int, _DESC, _STATE, _P, _P, _P, _P, _P, ctypes.c_size_t, _P)
_lib_decode_noalloc = _fn("duo_decode_attn_noalloc", ctypes.c_int, _DESC, _STATE, _P, _P, _P)
_lib_exp2_probe = _fn("duo_exp2_fma_probe", ctypes.c_int, _P, _P, ctypes.c_int64, _P)
NOALLOC_SCRATCH_BYTES = 2 << 20


class DuoError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib_last_error().decode()
        super().__init__(f"{where}: {_lib_status_string(status).decode()}: {msg}")


def _check(st: int, where: str) -> None:
    if st != OK:
        raise DuoError(st, where)


def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def last_error() -> str:
    return _lib_last_error().decode()


def status_string(s: int) -> str:
    return _lib_status_string(s).decode()


def abi_version() -> int:
    return int(_lib_abi_version())


# ------------------------------------------------------------------- set-up

def partition_heads(alpha, tau: float, target_n_retrieval: int = -1):
    """Host call: (gate list[int], kv_perm list[int], kv_inv_perm list[int], n_retrieval)."""
    alpha = [float(a) for a in alpha]
    n = len(alpha)
    a = (ctypes.c_float * max(n, 1))(*alpha)
    gate = (ctypes.c_uint8 * max(n, 1))()
    perm = (_I32 * max(n, 1))()
    inv = (_I32 * max(n, 1))()
    nret = _I32()
    _check(_lib_partition(a, n, tau, target_n_retrieval, gate, perm, inv, ctypes.byref(nret)),
           "duo_partition_heads")
    return list(gate[:n]), list(perm[:n]), list(inv[:n]), int(nret.value)


def desc_init(batch, n_q_heads, n_kv_heads, head_dim, dtype, kv_perm, n_retrieval, *, sink=None, recent=None,
              page_size=0, io_order=ORDER_MODEL, scale=0.0, stream_prefill=STREAM_LAMBDA,
              kv_quant=KV_PLAIN) -> LayerDesc:
    d = LayerDesc()
    perm = (_I32 * max(len(kv_perm), 1))(*[int(p) for p in kv_perm])
    _check(_lib_desc_init(ctypes.byref(d), batch, n_q_heads, n_kv_heads, head_dim, dtype, perm, n_retrieval),
           "duo_desc_init")
    if sink is not None:
        d.sink = sink
    if recent is not None:
        d.recent = recent
    d.page_size = page_size
    d.io_order = io_order
    d.scale = scale
    d.stream_prefill = stream_prefill
    d.kv_quant = kv_quant
    _check(_lib_desc_validate(ctypes.byref(d)), "duo_desc_validate")
    return d


def desc_validate(desc: LayerDesc) -> int:
    return int(_lib_desc_validate(ctypes.byref(desc)))


def workspace_bytes(desc: LayerDesc, op: int, max_tokens: int) -> int:
    return int(_lib_ws_bytes(ctypes.byref(desc), op, max_tokens))


def prefill_workspace_bytes(desc: LayerDesc, state: KVState, max_chunk: int) -> int:
    return int(_lib_pf_ws_bytes(ctypes.byref(desc), ctypes.byref(state), max_chunk))


# ------------------------------------------------------------ device calls

def permute_heads(desc, x, y, rows, heads_per_kv, head_elems, elem_bytes, direction, stream=None) -> None:
    _check(_lib_permute(ctypes.byref(desc), _ptr(x), _ptr(y), rows, heads_per_kv, head_elems, elem_bytes,
                        direction, _stream(stream)), "duo_permute_heads")


def append_kv(desc, state: KVState, k_new, v_new, T: int, stream=None) -> None:
    _check(_lib_append(ctypes.byref(desc), ctypes.byref(state), _ptr(k_new), _ptr(v_new), T, _stream(stream)),
           "duo_append_kv")


def decode_attn(desc, state: KVState, q, out, workspace, ws_bytes: int, stream=None) -> None:
    _check(_lib_decode(ctypes.byref(desc), ctypes.byref(state), _ptr(q), _ptr(out), _ptr(workspace), ws_bytes,
                       _stream(stream)), "duo_decode_attn")


def decode_step(desc, state: KVState, q, k_new, v_new, out, workspace, ws_bytes: int, stream=None) -> None:
    """Append one token per sequence and attend, in one launch."""
    _check(_lib_decode_step(ctypes.byref(desc), ctypes.byref(state), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                            _ptr(workspace), ws_bytes, _stream(stream)), "duo_decode_step")


def decode_attn_noalloc(desc, state: KVState, q, out, stream=None) -> None:
    """duo_decode_attn with the library's built-in scratch array instead of a
    caller workspace, for callers that cannot allocate device memory (a host
    engine owning all of HBM, a binding without memory management, a loop that
    must not call cudaMalloc).  Calls sharing a device must not overlap."""
    _check(_lib_decode_noalloc(ctypes.byref(desc), ctypes.byref(state), _ptr(q), _ptr(out), _stream(stream)),
           "duo_decode_attn_noalloc")


def prefill_chunk(desc, state: KVState, q, k_chunk, v_chunk, C: int, out, workspace=None, ws_bytes: int = 0,
                  stream=None) -> None:
    _check(_lib_prefill(ctypes.byref(desc), ctypes.byref(state), _ptr(q), _ptr(k_chunk), _ptr(v_chunk), C,
                        _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)), "duo_prefill_chunk")


def gated_mix(desc, alpha, q, k, v, N: int, out, status, stream=None) -> None:
    """status: an int32 device word; DUO_DEV_* bits are ORed into it."""
    _check(_lib_mix(ctypes.byref(desc), _ptr(alpha), _ptr(q), _ptr(k), _ptr(v), N, _ptr(out), _ptr(status),
                    _stream(stream)), "duo_gated_mix")


def gated_mix_grad_alpha(desc, q, k, v, N: int, dout, dalpha, status, stream=None) -> None:
    _check(_lib_mix_grad(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), N, _ptr(dout), _ptr(dalpha), _ptr(status),
                         _stream(stream)), "duo_gated_mix_grad_alpha")


def wait_probe(status, limit_us: int, stream=None) -> None:
    """One warp runs the library's bounded device wait on a barrier nothing
    completes; DUO_DEV_WAIT_TIMEOUT is ORed into the int32 device word `status`."""
    _check(_lib_wait_probe(_ptr(status), limit_us, _stream(stream)), "duo_wait_probe")


def exp2_fma_probe(x, y, n: int, stream=None) -> None:
    """y[:n] = the pre-fill softmax's FMA-pipe 2^x of x[:n] (fp32 device buffers)."""
    _check(_lib_exp2_probe(_ptr(x), _ptr(y), n, _stream(stream)), "duo_exp2_fma_probe")


def check_status(state: KVState, stream=None, raise_on_error: bool = False) -> int:
    v = _I32()
    st = _lib_check(ctypes.byref(state), ctypes.byref(v), _stream(stream))
    if st not in (OK, ERR_DEVICE) or (raise_on_error and st != OK):
        raise DuoError(st, "duo_check_status")
    return int(v.value)


# ----------------------------------------------------- torch-owned buffers

class LayerCaches:
    """Device buffers of one layer's two caches, allocated through torch in
    the layout include/duo.h documents, plus the KVState that points at them.

    Contiguous full cache: k_full/v_full [B, R, capacity, d].
    Paged full cache: k_full/v_full [n_pages, R, page_size, d] and page_table
    [B, max_pages] int32 (copied from the given host table).
    8-bit full cache: k_full int8 [B, R, capacity, d], v_full int8
    [B, R, capacity / 64, d, 64], k_scale/v_scale fp32 [B, R, capacity]
    (capacity rounded up to a multiple of 64).
    4-bit full cache: k_full uint8 [B, R, capacity, d / 2], v_full uint8
    [B, R, capacity / 64, 32 d], scales as for 8 bits.
    Rings: k_ring/v_ring [B, S, sink + recent, d]; ring_pos [B, W] (-1);
    seq_len [B] (0); counters [4] (0); status [1] (0).
    """

    def __init__(self, desc: LayerDesc, capacity: int = 0, page_table=None, n_pages: int = 0, device="cuda"):
        import torch
        dt = torch.bfloat16 if desc.dtype == BF16 else torch.float32
        B, R, S = desc.batch, desc.n_retrieval, desc.n_kv_heads - desc.n_retrieval
        d, W = desc.head_dim, desc.sink + desc.recent
        self.desc = desc
        if desc.page_size:
            pt = torch.as_tensor(page_table, dtype=torch.int32)
            max_pages = pt.shape[1]
            self.page_table = pt.to(device).contiguous()
            self.k_full = torch.zeros((n_pages, R, desc.page_size, d), dtype=dt, device=device)
            self.v_full = torch.zeros_like(self.k_full)
            capacity = max_pages * desc.page_size
        elif desc.kv_quant == KV_INT8:
            # 8-bit codes: K row per token, V per 64-token tile transposed; fp32 scale per row
            max_pages = 0
            self.page_table = None
            capacity = (max(capacity, 1) + 63) // 64 * 64
            self.k_full = torch.zeros((B, R, capacity, d), dtype=torch.int8, device=device)
            self.v_full = torch.zeros((B, R, capacity // 64, d, 64), dtype=torch.int8, device=device)
            self.k_scale = torch.zeros((B, R, capacity), dtype=torch.float32, device=device)
            self.v_scale = torch.zeros_like(self.k_scale)
        elif desc.kv_quant == KV_INT4:
            # 4-bit codes: K 64 bytes per token, V 4 KB per 64-token tile; fp32 scale per row
            max_pages = 0
            self.page_table = None
            capacity = (max(capacity, 1) + 63) // 64 * 64
            self.k_full = torch.zeros((B, R, capacity, d // 2), dtype=torch.uint8, device=device)
            self.v_full = torch.zeros((B, R, capacity // 64, 64 * d // 2), dtype=torch.uint8, device=device)
            self.k_scale = torch.zeros((B, R, capacity), dtype=torch.float32, device=device)
            self.v_scale = torch.zeros_like(self.k_scale)
        else:
            max_pages = 0
            self.page_table = None
            self.k_full = torch.zeros((B, R, max(capacity, 0), d), dtype=dt, device=device)
            self.v_full = torch.zeros_like(self.k_full)
        if desc.kv_quant not in (KV_INT8, KV_INT4):
            self.k_scale = self.v_scale = None
        self.capacity = capacity
        self.k_ring = torch.zeros((B, S, W, d), dtype=dt, device=device)
        self.v_ring = torch.zeros_like(self.k_ring)
        self.ring_pos = torch.full((B, W), -1, dtype=torch.int32, device=device)
        self.seq_len = torch.zeros((B,), dtype=torch.int32, device=device)
        self.counters = torch.zeros((STATE_COUNTER_WORDS,), dtype=torch.int32, device=device)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        self.state = KVState(
            k_full=_ptr(self.k_full), v_full=_ptr(self.v_full), page_table=_ptr(self.page_table),
            capacity=capacity, max_pages=max_pages, n_pages=n_pages, reserved0=0,
            k_ring=_ptr(self.k_ring), v_ring=_ptr(self.v_ring), ring_pos=_ptr(self.ring_pos),
            seq_len=_ptr(self.seq_len), counters=_ptr(self.counters), status=_ptr(self.status),
            k_scale=_ptr(self.k_scale), v_scale=_ptr(self.v_scale))


class Workspace:
    """A zero-filled device workspace of the size the library asks for
    (pre-fill: pass the layer's state, so that an 8- or 4-bit layer gets its
    staging area too)."""

    def __init__(self, desc: LayerDesc, op: int, max_tokens: int, device="cuda", state: KVState = None):
        import torch
        if op == OP_PREFILL and state is not None:
            self.nbytes = prefill_workspace_bytes(desc, state, max_tokens)
        else:
            self.nbytes = workspace_bytes(desc, op, max_tokens)
        self.buf = torch.zeros((max(self.nbytes, 16),), dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return _ptr(self.buf)
