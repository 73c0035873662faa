#!/usr/bin/env python3
"""Benchmark of the head-split attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload ``gqa_decode_128k``: a Llama-3-8B-shaped GQA attention
layer (32 query heads over 8 KV heads, head_dim 128, bf16, batch 1), 4 of 8
KV heads retrieval (chosen by seed), sink 16 / recent 64, context 131,072
tokens, one token appended and attended per decode step.  A step is one pass
of the path: duo_decode_step, the one-launch form of duo_append_kv +
duo_decode_attn (both caches, both head types, output concatenated in model
head order), for each of 32 layers with their own caches, back to back as in
a forward pass; the value is per layer.  Inputs are resident in HBM before
timing starts; the layers' caches (8.6 GB) exceed the 126 MB L2, so nothing
is flushed between steps.

The default line also carries ``decode_configs``: mha_decode_32k (Llama-2-7B-
shaped MHA, 8 of 32 heads retrieval, 32 layers), gqa_decode_1m (16 layers)
and batch64_paged_decode (64 sequences, lengths U[4096, 32768], 64-token
pages, 8 layers), each with its own roofline, clocks, e2e and CPU baseline
(--no-extra drops them).  Other workloads: the same decode shapes over 8- or
4-bit retrieval caches (``*_int8``, ``*_int4``), gqa_prefill_128k (one
131,072-token prompt in 32 chunks of 4,096; a step is one chunk's
duo_prefill_chunk + duo_append_kv) and the same over 8- / 4-bit caches
(``gqa_prefill_128k_int8``, ``_int4``), gqa_prefill_32k, and the gated mix
(gated_mix_pr1, gated_mix_gqa_4k: forward and gate gradient).

A decode run also measures the pre-fill workload (unless --no-prefill) and
reports it under "prefill" in the same line; its TFLOP/s count 4*d FLOPs per
visible (query, key) pair and query head.

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
replica of the workload on its own GPU (the path has no exchange step); the
time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from head_split_kv_b200 import synthetic as S  # noqa: E402

METRIC = "decode attn µs/step/layer & HBM GB/s; chunked-prefill TFLOP/s; % of roofline"

# "layers": attention layers a decode step runs through, each with its own
# caches (Llama-2-7B and Llama-3-8B have 32; fewer where 32 layers' caches
# would not leave room on one GPU)
WORKLOADS = {
    "mha_decode_32k": dict(kind="decode", hq=32, hkv=32, d=128, n_ret=8, lengths=[32768], steps=256, sigma=False,
                           layers=32),
    "gqa_decode_128k": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[131072], steps=64, sigma=True,
                            layers=32),
    "gqa_decode_1m": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[1048576], steps=64, sigma=True,
                          layers=16),
    "batch64_paged_decode": dict(kind="decode", hq=32, hkv=32, d=128, n_ret=8, batch=64, lo=4096, hi=32768,
                                 steps=32, sigma=False, paged=True, layers=8),
    # the same decode workloads over the 8-bit retrieval cache (codes + a scale per row)
    "mha_decode_32k_int8": dict(kind="decode", hq=32, hkv=32, d=128, n_ret=8, lengths=[32768], steps=256,
                                sigma=False, kv_int8=True, layers=32),
    "gqa_decode_128k_int8": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[131072], steps=64,
                                 sigma=True, kv_int8=True, layers=32),
    "gqa_decode_1m_int8": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[1048576], steps=64,
                               sigma=True, kv_int8=True, layers=16),
    # ... and over the 4-bit retrieval cache
    "mha_decode_32k_int4": dict(kind="decode", hq=32, hkv=32, d=128, n_ret=8, lengths=[32768], steps=256,
                                sigma=False, kv_int4=True, layers=32),
    "gqa_decode_128k_int4": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[131072], steps=64,
                                 sigma=True, kv_int4=True, layers=32),
    "gqa_decode_1m_int4": dict(kind="decode", hq=32, hkv=8, d=128, n_ret=4, lengths=[1048576], steps=64,
                               sigma=True, kv_int4=True, layers=16),
    "gqa_prefill_128k": dict(kind="prefill", hq=32, hkv=8, d=128, n_ret=4, n=131072, chunk=4096, sigma=False),
    # ... over 8- and 4-bit retrieval caches (each chunk stages the prior codes
    # and scales, then runs the tensor-core pre-fill over them)
    "gqa_prefill_128k_int8": dict(kind="prefill", hq=32, hkv=8, d=128, n_ret=4, n=131072, chunk=4096, sigma=False,
                                  kv_int8=True),
    "gqa_prefill_128k_int4": dict(kind="prefill", hq=32, hkv=8, d=128, n_ret=4, n=131072, chunk=4096, sigma=False,
                                  kv_int4=True),
    # the same pre-fill on a 32K prompt: a small case for profiler captures
    "gqa_prefill_32k": dict(kind="prefill", hq=32, hkv=8, d=128, n_ret=4, n=32768, chunk=4096, sigma=False),
    # the gated mix alpha * full + (1 - alpha) * streaming over whole sequences
    # and its gate gradient: the tiny single-layer MHA case (fp32, d 64, 512
    # tokens, alpha ~ U(0, 1)) and a Llama-3-8B-shaped GQA layer over 4,096 tokens
    "gated_mix_pr1": dict(kind="mix", hq=8, hkv=8, d=64, n=512, dtype="fp32", n_ret=2),
    "gated_mix_gqa_4k": dict(kind="mix", hq=32, hkv=8, d=128, n=4096, dtype="bf16", n_ret=4),
}
DEFAULT_WORKLOAD = "gqa_decode_128k"
# decode configurations timed beside the default one, each as its own record
EXTRA_DECODE = ("mha_decode_32k", "gqa_decode_1m", "batch64_paged_decode")
for _name, _wl in WORKLOADS.items():
    _wl["name"] = _name
    _wl["kv_bits"] = 8 if _wl.get("kv_int8") else 4 if _wl.get("kv_int4") else 0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def _traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu record profiles/traffic.json ({kernel: {workload: record}})
    -- only while every source file the record lists still has the recorded
    SHA-256 (a changed kernel has no measured traffic until it is captured
    again)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = (json.load(f).get(kernel) or {}).get(workload)
    except (OSError, ValueError, AttributeError):
        return None
    if not rec:
        return None
    for rel, digest in rec.get("source_sha256", {}).items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return int(rec["dram_bytes_read"] + rec["dram_bytes_write"])


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

_NVML_POLL = r"""
import sys, time
import pynvml as nv
nv.nvmlInit()
h = nv.nvmlDeviceGetHandleByPciBusId(sys.argv[1])
period = float(sys.argv[2])
print("ready", nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM), flush=True)
while True:
    t = time.monotonic()
    print(t, nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), nv.nvmlDeviceGetCurrentClocksEventReasons(h), flush=True)
    time.sleep(max(0.0, period - (time.monotonic() - t)))
"""


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this process's GPU,
    sampled while the timed region runs, from a separate process so that the
    launching thread's hold on the interpreter cannot starve the sampling.

    Through NVML every 1 ms when the bindings load (the CUDA device is
    matched to its NVML handle by PCI bus id, so CUDA_VISIBLE_DEVICES cannot
    point it at another GPU), else through `nvidia-smi -lms 100`.  Each NVML
    sample carries the poller's CLOCK_MONOTONIC time (one clock for every
    process on the host); entering waits until the first sample has arrived,
    and the summary keeps the samples taken between entering and leaving --
    the timed region, which ends with a device synchronisation.  Only reads;
    nothing about the GPU is changed."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # NVML clock-event reason bits
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int, period_s: float = 0.001):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.lines = []
        self.mode = None
        self.max_mhz = None
        self.t_enter = self.t_exit = None
        self._first = threading.Event()

    def _start_nvml(self) -> bool:
        import torch
        props = torch.cuda.get_device_properties(self.gpu)
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLL, bus, str(self.period)],
                                     stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        first = self.proc.stdout.readline().split()
        if len(first) != 2 or first[0] != "ready":
            self.proc.kill()
            self.proc = None
            return False
        self.max_mhz = float(first[1])
        return True

    def __enter__(self):
        try:
            if self._start_nvml():
                self.mode = f"nvml {self.period * 1e3:g} ms"
        except Exception:
            self.proc = None
        if self.proc is None:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.mode = "nvidia-smi 100 ms"
            except OSError:
                self.proc = None
        if self.proc is not None:
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            self._first.wait(timeout=5.0)   # the sampler is running before the region starts
        self.t_enter = time.monotonic()
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())
            self._first.set()

    def __exit__(self, *exc):
        self.t_exit = time.monotonic()
        if self.proc:
            # let the sample taken across the end of the region arrive
            time.sleep(0.25 if not self.mode.startswith("nvml") else 3 * self.period)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=5)

    def summary(self):
        mhz, mx, reasons, outside = [], self.max_mhz, set(), 0
        for ln in list(self.lines):
            if self.mode.startswith("nvml"):
                parts = ln.split()
                if len(parts) != 3:
                    continue
                try:
                    t, f, bits = float(parts[0]), float(parts[1]), int(parts[2])
                except ValueError:
                    continue
                if not (self.t_enter <= t <= self.t_exit):
                    outside += 1
                    continue
                mhz.append(f)
                reasons |= {n for n, bit in self.BITS.items() if bits & bit}
            else:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    mhz.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(self.NAMES, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        region_ms = (self.t_exit - self.t_enter) * 1e3 if self.t_exit else None
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz), "sampler": self.mode,
                "region_ms": round(region_ms, 1) if region_ms is not None else None,
                "samples_outside_region": outside}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------

def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def _max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_unit(local_total_ms: float, units_per_rank: int, world: int) -> float:
    """Whole-job time per unit for replicas: the slowest rank's time over
    every rank's units (each rank runs the same number of units)."""
    return _max_over_ranks(local_total_ms, world) * 1e3 / (units_per_rank * world)


# ---------------------------------------------------------------------------
# decode workloads
# ---------------------------------------------------------------------------

def _decode_setup(duo, wl, total_steps, seed=0):
    import torch
    sh = S.LayerShape(wl["hq"], wl["hkv"], wl["d"], "bf16")
    retrieval = S.retrieval_heads_by_seed(wl["hkv"], wl["n_ret"], seed=1)
    if "batch" in wl:
        lengths = S.context_lengths(wl["batch"], wl["lo"], wl["hi"], seed=seed)
    else:
        lengths = np.asarray(wl["lengths"], dtype=np.int64)
    B = len(lengths)
    sigma = S.head_sigma(wl["hkv"], seed=seed) if wl.get("sigma") else None
    alpha = S.binary_alpha(wl["hkv"], retrieval)
    gate, perm, inv, R = duo.partition_heads(alpha, 0.5)
    paged = wl.get("paged", False)
    if paged:
        table, n_pages = S.page_assignment(lengths, total_steps, 64, seed=seed)
        desc = duo.desc_init(B, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, duo.BF16, perm, R, page_size=64)
        caches = duo.LayerCaches(desc, 0, table, n_pages)
    else:
        table = None
        desc = duo.desc_init(B, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, duo.BF16, perm, R,
                             kv_quant={8: duo.KV_INT8, 4: duo.KV_INT4}.get(wl.get("kv_bits", 0), duo.KV_PLAIN))
        caches = duo.LayerCaches(desc, int(lengths.max()) + total_steps)
    st = S.decode_state(sh, retrieval, lengths, seed=seed, sigma=sigma)
    _fill_decode_state(duo, desc, caches, st, inv, R, sh, table, wl.get("kv_bits", 0))
    ws = duo.Workspace(desc, duo.OP_DECODE, caches.capacity)
    qs, ks, vs = S.decode_steps(sh, B, total_steps, seed=seed, sigma=sigma)
    torch.cuda.synchronize()
    return dict(sh=sh, desc=desc, caches=caches, ws=ws, qs=qs, ks=ks, vs=vs, lengths=lengths, B=B, R=R,
                kv_bits=wl.get("kv_bits", 0),
                retrieval=retrieval, gate=gate, state=st, sigma=sigma, table=table,
                n_pages=n_pages if paged else 0)


def _to_dev(a):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _fill_decode_state(duo, desc, caches, st, inv, R, sh, table, kv_bits, chunk=32768):
    """Put a seeded prompt state on the device.

    Retrieval rows: written straight into the documented cache layout (bf16),
    or appended through duo_append_kv, which quantizes them (8- or 4-bit; the
    other heads get zero rows there).  Streaming rings: built by the library's own
    append -- seq_len is set to 0 and the prompt's first W = sink + recent
    tokens are appended, then seq_len is set to L - W and its last W tokens
    are appended (every head's rows, so a retrieval head gets its own rows
    again).  A ring holds at most W tokens, so this leaves it as appending the
    whole prompt would, without drawing the streaming rows in between."""
    import torch
    lengths = st.lengths
    B = len(lengths)
    W = sh.sink + sh.recent
    assert int(lengths.min()) >= 2 * W, "bench states are built for prompts of at least 2 (sink + recent) tokens"
    if kv_bits:
        L = int(lengths.max())
        assert np.all(lengths == L), "quantized states are built for equal lengths"
        for c0 in range(0, L, chunk):
            T = min(chunk, L - c0)
            kc = torch.zeros((B, T, sh.n_kv_heads, sh.head_dim), dtype=torch.bfloat16, device="cuda")
            vc = torch.zeros_like(kc)
            for (b, h), (k, v) in st.full.items():
                kc[b, :, h] = _to_dev(k[c0:c0 + T])
                vc[b, :, h] = _to_dev(v[c0:c0 + T])
            duo.append_kv(desc, caches.state, kc, vc, T)
    else:
        for (b, h), (k, v) in st.full.items():
            r = inv[h]
            L = k.shape[0]
            if table is None:
                caches.k_full[b, r, :L] = _to_dev(k)
                caches.v_full[b, r, :L] = _to_dev(v)
            else:
                pos = np.arange(L)
                pages = torch.from_numpy(table[b, pos // 64].astype(np.int64)).cuda()
                rows = torch.from_numpy(pos % 64).cuda()
                caches.k_full[pages, r, rows] = _to_dev(k)
                caches.v_full[pages, r, rows] = _to_dev(v)
    for first in (True, False):
        start = np.zeros(B, dtype=np.int64) if first else lengths - W
        rows = [st.token_rows(b, np.arange(start[b], start[b] + W)) for b in range(B)]
        kk = np.stack([r[0] for r in rows])
        vv = np.stack([r[1] for r in rows])
        caches.seq_len.copy_(torch.from_numpy(start.astype(np.int32)))
        duo.append_kv(desc, caches.state, _to_dev(kk), _to_dev(vv), W)
    torch.cuda.synchronize()
    assert np.array_equal(caches.seq_len.cpu().numpy(), lengths.astype(np.int32))
    assert duo.check_status(caches.state) == 0


def _decode_bytes(sh, R, lengths_after, kv_bits=0):
    """Algorithmic HBM bytes of one fused decode step: every cached K/V row of
    every retrieval head once (8-bit: d code bytes + a 4-byte scale per row;
    4-bit: d / 2 + 4), the ring rows of the streaming heads, q and out, and
    the new token's K/V rows read once and written once into the caches."""
    S_ = sh.n_kv_heads - R
    row = sh.head_dim * 2
    full_row = {8: sh.head_dim + 4, 4: sh.head_dim // 2 + 4}.get(int(kv_bits), row)
    total = 0
    for L in lengths_after:
        total += R * (L - 1) * full_row * 2
        total += S_ * (min(L, sh.sink + sh.recent) - 1) * row * 2
        total += sh.n_kv_heads * row * 2 * 2
    total += len(lengths_after) * sh.n_q_heads * sh.head_dim * 2 * 2
    return total


def _replicate_layers(duo, env, n_layers):
    """n_layers independent caches of the same shape, each a device copy of the
    seeded state (the layers of one model), each with its own workspace."""
    import torch
    first = env["caches"]
    layers = [(first, env["ws"])]
    for _ in range(n_layers - 1):
        c = duo.LayerCaches(env["desc"], first.capacity, env.get("table"), env.get("n_pages", 0))
        for name in ("k_full", "v_full", "k_ring", "v_ring", "ring_pos", "seq_len", "k_scale", "v_scale"):
            if getattr(first, name, None) is not None:
                getattr(c, name).copy_(getattr(first, name))
        layers.append((c, duo.Workspace(env["desc"], duo.OP_DECODE, c.capacity)))
    torch.cuda.synchronize()
    return layers


def run_decode(args, wl, world, rank):
    """Decode steps: a step is one new token per sequence through every layer
    of the model's attention -- per layer duo_decode_step (append + attend,
    one launch), the layers back to back as in a forward pass, each with its
    own caches.  A step streams layers x (retrieval cache) bytes, far more
    than the 126 MB L2, so nothing is flushed between steps."""
    import torch
    from head_split_kv_b200 import duo
    steps, warm = args.steps, args.warmup
    nl = args.layers or wl["layers"]
    total = warm + steps
    n_e2e = 0 if getattr(args, "no_e2e", False) else min(steps, 32)
    env = _decode_setup(duo, wl, total + n_e2e + 1)
    sh, desc, B, R = env["sh"], env["desc"], env["B"], env["R"]
    layers = _replicate_layers(duo, env, nl)
    qd = [_to_dev(env["qs"][i]) for i in range(total)]
    kd = [_to_dev(env["ks"][i][:, None]) for i in range(total)]
    vd = [_to_dev(env["vs"][i][:, None]) for i in range(total)]
    out = torch.empty_like(qd[0])
    stream = torch.cuda.current_stream()
    sp = int(stream.cuda_stream)

    def step(i):
        for caches, ws in layers:
            duo.decode_step(desc, caches.state, qd[i], kd[i], vd[i], out, ws.ptr, ws.nbytes, sp)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    lengths_seen = []
    base = env["lengths"] + warm
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        for j in range(steps):
            e0, e1 = ev[j]
            e0.record(stream)
            step(warm + j)
            e1.record(stream)
            lengths_seen.append(base + j + 1)
        torch.cuda.synchronize()
    _barrier(world)
    # one launch per layer and step (append fused into the decode kernel)
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    dec_ms = [t / nl for t in step_ms]
    total_ms = _max_over_ranks(sum(step_ms), world)
    us_step = total_ms * 1e3 / (steps * nl * world)
    for caches, _ in layers:
        st_code = duo.check_status(caches.state)
        if st_code:
            raise RuntimeError(f"device status 0x{st_code:x} after the timed steps")

    # end to end through the public API with host buffers
    e2e = _decode_e2e(duo, env, layers, total, n_e2e, world) if n_e2e else None

    hbm, _, peak_kind = _peaks()
    kernel = {8: "decode_q8_kernel", 4: "decode_q4_kernel"}.get(wl.get("kv_bits", 0), "decode_mma_kernel")
    bytes_per_launch = statistics.mean(_decode_bytes(sh, R, L, wl.get("kv_bits", 0)) for L in lengths_seen)
    dec_avg_s = statistics.mean(dec_ms) * 1e-3
    achieved = bytes_per_launch / dec_avg_s / 1e9
    res = {
        "metric": METRIC, "value": round(us_step, 3), "unit": "us/step/layer", "n_gpus": world, "steps": steps,
        "warmup": warm, "ms_per_step": round(total_ms / steps, 6), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "batch": B, "n_q_heads": sh.n_q_heads, "n_kv_heads": sh.n_kv_heads,
                   "head_dim": sh.head_dim, "n_retrieval": R, "sink": sh.sink, "recent": sh.recent,
                   "context": [int(env["lengths"].min()), int(env["lengths"].max())],
                   "paged": bool(wl.get("paged", False)), "layers_per_step": nl,
                   "full_cache": {8: "int8 codes + fp32 scale per row", 4: "4-bit codes + fp32 scale per row"}.get(
                       wl.get("kv_bits", 0), "bf16"),
                   "parallelism": f"replicas{world}",
                   "l2": f"not flushed: inputs larger than L2 (each step streams {nl} layers' caches, "
                         f"{nl * bytes_per_launch / 1e6:.0f} MB > 126 MB)"},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "traffic": _traffic(kernel, wl["name"]),
                     "algorithmic_bytes_per_launch": int(bytes_per_launch),
                     "kernel_us": round(statistics.mean(dec_ms) * 1e3, 3),
                     "timing": "CUDA events on the launching stream around each step; kernel_us = step time / "
                               "layers (one launch per layer)"},
        "e2e": e2e,
        "gpu_launches": steps * nl,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = _decode_cpu_baseline(env, budget_s=args.cpu_budget)
    del layers, env
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def _decode_e2e(duo, env, layers, first, n, world):
    """The same decode steps through the binding with pinned host buffers.
    Per step, every layer's new-token q, k and v go host->device in one copy
    and every layer's output comes back device->host in one copy, inside the
    timed interval.  The copies run on their own streams, ordered by events
    against the compute stream, with two device input and output buffers:
    step i + 1's inputs arrive and step i - 1's outputs leave while step i's
    kernels run.  Every layer of a step takes the step's token (as in the
    device-resident timing)."""
    import torch
    desc = env["desc"]
    nl = len(layers)
    q_shape, kv_shape = env["qs"][0].shape, env["ks"][0][:, None].shape
    nq, nk = int(np.prod(q_shape)), int(np.prod(kv_shape))
    per = nq + 2 * nk                       # bf16 elements of one layer's q | k | v (whole d-rows each)

    def pinned(i):
        one = np.concatenate([np.ascontiguousarray(a).reshape(-1) for a in
                              (env["qs"][i], env["ks"][i], env["vs"][i])])
        flat = np.tile(one, nl)
        return torch.from_numpy(flat.view(np.int16)).view(torch.bfloat16).pin_memory()

    h_in = [pinned(first + i) for i in range(n)]
    h_out = [torch.empty((nl,) + tuple(q_shape), dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    d_in = [torch.empty(nl * per, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    d_out = [torch.empty((nl,) + tuple(q_shape), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    views = [[(x[l * per:l * per + nq].view(q_shape), x[l * per + nq:l * per + nq + nk].view(kv_shape),
               x[l * per + nq + nk:(l + 1) * per].view(kv_shape)) for l in range(nl)] for x in d_in]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    sp = int(comp.cuda_stream)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    t0.record(s_in)
    comp.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(n):
        k = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[i - 2])          # d_in[k] is free once step i - 2 ran
            d_in[k].copy_(h_in[i], non_blocking=True)
            ev_in[k].record(s_in)
        comp.wait_event(ev_in[k])
        if i >= 2:
            comp.wait_event(ev_out[k])                   # d_out[k] is free once step i - 2's outputs left
        for l, (caches, ws) in enumerate(layers):
            q, kk, vv = views[k][l]
            duo.decode_step(desc, caches.state, q, kk, vv, d_out[k][l], ws.ptr, ws.nbytes, sp)
        ev_comp[i].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[i])
            h_out[i].copy_(d_out[k], non_blocking=True)
            ev_out[k].record(s_out)
    comp.wait_event(ev_out[(n - 1) % 2])
    if n >= 2:
        comp.wait_event(ev_out[(n - 2) % 2])
    t1.record(comp)
    torch.cuda.synchronize()
    _barrier(world)
    tot = _max_over_ranks(t0.elapsed_time(t1), world)
    for caches, _ in layers:
        st_code = duo.check_status(caches.state)
        if st_code:
            raise RuntimeError(f"device status 0x{st_code:x} after the end-to-end steps")
    assert all(torch.isfinite(h.float()).all().item() for h in h_out)
    return {"value": round(tot * 1e3 / (n * nl * world), 3), "unit": "us/step/layer",
            "h2d_bytes_per_step": nl * per * 2, "d2h_bytes_per_step": nl * nq * 2, "steps": n,
            "note": "bytes per step (all layers); copies on their own streams, double-buffered"}


def _oracle_cache(O, st, gate, sh, b_list, heads, kv_bits):
    """The oracle's caches for sequences b_list and KV heads `heads` of a
    seeded state: retrieval heads hold every prompt row; a streaming head the
    positions the oracle's own eviction rule keeps, with their seeded rows."""
    g = np.array([gate[h] for h in heads], dtype=np.uint8)
    cache = O.HeadSplitCache(len(b_list), len(heads), sh.head_dim, gate=g, sink=sh.sink, recent=sh.recent,
                             kv_int8=kv_bits == 8, kv_int4=kv_bits == 4)
    for bi, b in enumerate(b_list):
        L = int(st.lengths[b])
        kept = O.streaming_positions(L, sh.sink, sh.recent)
        for hi, h in enumerate(heads):
            if gate[h]:
                k, v = st.full[(b, h)]
                cache.load_state(bi, hi, np.arange(L), k, v)
            else:
                k, v = st.stream_rows(b, h, kept)
                cache.load_state(bi, hi, kept, k, v)
        cache.set_length(bi, L)
    return cache


def _decode_cpu_baseline(env, budget_s=8.0):
    """The oracle, as it stands, on this host's cores: decode steps from the
    same seeded state until the time budget is used (at least one)."""
    import oracle as O
    sh, B = env["sh"], env["B"]
    cache = _oracle_cache(O, env["state"], env["gate"], sh, list(range(B)), list(range(sh.n_kv_heads)),
                          env.get("kv_bits", 0))
    t0 = time.perf_counter()
    n = 0
    while n < len(env["qs"]) and (time.perf_counter() - t0 < budget_s or n < 1):
        cache.decode(env["qs"][n], env["ks"][n], env["vs"][n])
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(dt * 1e6 / n, 1), "unit": "us/step/layer", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{n} decode steps of one layer of the same workload from the same seeded state "
                      f"(fp64 NumPy oracle)"}


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def _lambda_pairs(p0: int, n: int, sink: int, recent: int) -> int:
    """Visible (query, key) pairs of the Lambda mask for queries p0 .. p0+n-1."""
    P = np.arange(p0, p0 + n, dtype=np.int64)
    sinks = np.minimum(P + 1, sink)
    band = np.minimum(P + 1, recent)
    both = np.clip(np.minimum(sink, P + 1) - np.maximum(0, P - recent + 1), 0, None)
    return int((sinks + band - both).sum())


def _prefill_flops(n_ret_q, n_str_q, d, c0, C, sink, recent, stream_chunk=False):
    """Algorithmic FLOPs of one chunk: 4*d per visible (query, key) pair and
    query head (2*d for Q K^T, 2*d for P V); masked pairs are not counted.
    Whole-chunk streaming: every query sees the min(c0, sink + recent) cached
    tokens and the chunk up to itself."""
    causal = C * c0 + C * (C + 1) // 2
    stream = (C * min(c0, sink + recent) + C * (C + 1) // 2) if stream_chunk else _lambda_pairs(c0, C, sink, recent)
    return 4 * d * (n_ret_q * causal + n_str_q * stream)


def run_prefill(args, wl, world, rank, steps=None, warmup=None):
    """Chunked pre-fill of one prompt: a step is one chunk (duo_prefill_chunk
    then duo_append_kv).  The timed steps are the prompt's chunks in order from
    an empty cache; warm-up chunks run first on the same buffers, which are then
    reset (seq_len 0, ring positions -1) outside the timed region."""
    import torch
    from head_split_kv_b200 import duo
    sh = S.LayerShape(wl["hq"], wl["hkv"], wl["d"], "bf16")
    n, C = wl["n"], wl["chunk"]
    n_chunks = n // C
    steps = n_chunks if steps is None else min(steps, n_chunks)
    warmup = 3 if warmup is None else warmup
    retrieval = S.retrieval_heads_by_seed(wl["hkv"], wl["n_ret"], seed=1)
    gate, perm, inv, R = duo.partition_heads(S.binary_alpha(wl["hkv"], retrieval), 0.5)
    stream_chunk = wl.get("stream") == "chunk"
    kv_bits = wl.get("kv_bits", 0)
    desc = duo.desc_init(1, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, duo.BF16, perm, R,
                         stream_prefill=duo.STREAM_CHUNK if stream_chunk else duo.STREAM_LAMBDA,
                         kv_quant={8: duo.KV_INT8, 4: duo.KV_INT4}.get(kv_bits, duo.KV_PLAIN))
    caches = duo.LayerCaches(desc, n)
    q, k, v = S.prompt(sh, n, seed=0)
    qd, kd, vd = _to_dev(q), _to_dev(k), _to_dev(v)
    del q, k, v
    out = torch.empty((1, C, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    sp = int(stream.cuda_stream)
    G = sh.group

    def chunk(i):
        sl = slice(i * C, (i + 1) * C)
        qc, kc, vc = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        return qc, kc, vc

    chunks = [chunk(i) for i in range(n_chunks)]
    # lets long retrieval units split their key tiles; for an 8- or 4-bit
    # layer it also holds the staged codes and scales
    ws = duo.Workspace(desc, duo.OP_PREFILL, C, state=caches.state)
    for i in range(min(warmup, n_chunks)):
        qc, kc, vc = chunks[i]
        duo.prefill_chunk(desc, caches.state, qc, kc, vc, C, out, ws.ptr, ws.nbytes, sp)
        duo.append_kv(desc, caches.state, kc, vc, C, sp)
    torch.cuda.synchronize()
    caches.seq_len.zero_()
    caches.ring_pos.fill_(-1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        for i in range(steps):
            flush.zero_()
            qc, kc, vc = chunks[i]
            e0, e1, e2 = ev[i]
            e0.record(stream)
            duo.prefill_chunk(desc, caches.state, qc, kc, vc, C, out, ws.ptr, ws.nbytes, sp)
            e1.record(stream)
            duo.append_kv(desc, caches.state, kc, vc, C, sp)
            e2.record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    st_code = duo.check_status(caches.state)
    if st_code:
        raise RuntimeError(f"device status 0x{st_code:x} after the timed chunks")
    pre_ms = [a.elapsed_time(b) for a, b, _ in ev]
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    flops = [_prefill_flops(R * G, (sh.n_kv_heads - R) * G, sh.head_dim, i * C, C, sh.sink, sh.recent, stream_chunk)
             for i in range(steps)]
    total_ms = _max_over_ranks(sum(step_ms), world)
    _, tf_peak, peak_kind = _peaks()
    achieved = sum(flops) / (sum(pre_ms) * 1e-3) / 1e12
    value = sum(flops) * world / (total_ms * 1e-3) / 1e12
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(total_ms / steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "prompt": n, "chunk": C, "n_q_heads": sh.n_q_heads,
                   "n_kv_heads": sh.n_kv_heads, "head_dim": sh.head_dim, "n_retrieval": R, "sink": sh.sink,
                   "recent": sh.recent, "parallelism": f"replicas{world}", "workspace_bytes": ws.nbytes,
                   "full_cache": {8: "int8 codes + fp32 scale per row", 4: "4-bit codes + fp32 scale per row"}.get(
                       kv_bits, "bf16"),
                   "l2": "flushed (1 GiB write) before every timed chunk, outside the timed interval"},
        "roofline": {"bound": "tensor",
                     "kernel": "prefill_tc_kernel" if not kv_bits else
                               "dequant_kernel (staging) + prefill_tc_kernel (fp16 PV on the prior tiles)",
                     "achieved": round(achieved, 1),
                     "peak": tf_peak, "peak_kind": peak_kind + " (burst; sustained 1381.5)", "unit": "TFLOP/s",
                     "frac": round(achieved / tf_peak, 4), "traffic": _traffic("prefill_tc_kernel", wl["name"]),
                     "algorithmic_tflop_total": round(sum(flops) / 1e12, 3),
                     "prefill_ms_total": round(sum(pre_ms), 3), "append_ms_total": round(sum(step_ms) - sum(pre_ms), 3),
                     "per_chunk_ms": [round(x, 3) for x in pre_ms]},
        "gpu_launches": (3 if kv_bits else 2) * steps,
        "clocks": clk.summary(),
    }


# ---------------------------------------------------------------------------
# gated mix (whole sequences, no cache) and its gate gradient
# ---------------------------------------------------------------------------

# fp32 FMA pipe of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP per clock at
# the 1,965 MHz maximum SM clock
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def _mix_flops(hq, d, n, sink, recent, B):
    """Algorithmic FLOPs of one gated-mix forward: Q K^T once per causal pair
    (2*d), P V for the causal softmax over the same pairs (2*d) and for the
    Lambda softmax over its pairs (2*d), per query head."""
    return B * hq * (4 * d * (n * (n + 1) // 2) + 2 * d * _lambda_pairs(0, n, sink, recent))


def run_mix(args, wl, world, rank):
    """duo_gated_mix then duo_gated_mix_grad_alpha on one batch of whole
    sequences; a step is one forward and one gate gradient, L2 flushed (1 GiB
    write) before each, outside the timed intervals."""
    import torch
    from head_split_kv_b200 import duo
    import oracle as O
    dt = wl["dtype"]
    sh = S.LayerShape(wl["hq"], wl["hkv"], wl["d"], dt)
    n, B = wl["n"], 1
    if wl["name"] == "gated_mix_pr1":
        w = S.tiny_prompt()
        q, k, v, alpha = w["q"][None], w["k"][None], w["v"][None], w["alpha_mix"]
    else:
        q, k, v = S.prompt(sh, n, seed=0)
        alpha = S.rng_for(0, 50).uniform(0.0, 1.0, sh.n_kv_heads).astype(np.float32)
    dout = S.normal(S.rng_for(0, 61), q.shape, dt)
    desc = duo.desc_init(B, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, duo.BF16 if dt == "bf16" else duo.FP32,
                         list(range(sh.n_kv_heads)), 0)
    qd, kd, vd, dod = _to_dev(q), _to_dev(k), _to_dev(v), _to_dev(dout)
    ad = torch.from_numpy(alpha).cuda()
    out = torch.empty_like(qd)
    dalpha = torch.empty((sh.n_kv_heads,), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    flush = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    sp = int(stream.cuda_stream)
    for _ in range(args.warmup):
        duo.gated_mix(desc, ad, qd, kd, vd, n, out, status, sp)
        duo.gated_mix_grad_alpha(desc, qd, kd, vd, n, dod, dalpha, status, sp)
    steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(int(os.environ.get("LOCAL_RANK", "0"))) as clk:
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            duo.gated_mix(desc, ad, qd, kd, vd, n, out, status, sp)
            ev[i][1].record(stream)
            flush.zero_()
            ev[i][2].record(stream)
            duo.gated_mix_grad_alpha(desc, qd, kd, vd, n, dod, dalpha, status, sp)
            ev[i][3].record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    if int(status.item()):
        raise RuntimeError(f"device status 0x{int(status.item()):x} after the gated-mix calls")
    mix_ms = sorted(e[0].elapsed_time(e[1]) for e in ev)
    grad_ms = sorted(e[2].elapsed_time(e[3]) for e in ev)
    mix_med = _max_over_ranks(mix_ms[len(mix_ms) // 2], world)
    grad_med = _max_over_ranks(grad_ms[len(grad_ms) // 2], world)
    flops = _mix_flops(sh.n_q_heads, sh.head_dim, n, sh.sink, sh.recent, B)
    tf = flops / (mix_med * 1e-3) / 1e12
    if dt == "bf16" and sh.head_dim == 128:
        # both attentions on the tensor cores: two launches of the pre-fill
        # kernel (streaming, then causal with the mix in its epilogue)
        _, tf_peak, peak_kind = _peaks()
        bound = {"bound": "tensor", "kernel": "prefill_tc_kernel (streaming launch + causal launch with the mix)",
                 "peak": tf_peak,
                 "peak_kind": peak_kind + " bf16 (burst)"}
    else:
        bound = {"bound": "alu", "kernel": "simt_attention_kernel (gated mix)", "peak": round(ALU_FP32_TFLOPS, 1),
                 "peak_kind": "derived: fp32 FMA lanes x max SM clock"}
    res = {
        "metric": METRIC, "value": round(mix_med * 1e3, 2), "unit": "us/call", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(mix_med + grad_med, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if dt == "fp32" else "bf16", "data": "synthetic",
        "config": {"workload": wl["name"], "tokens": n, "batch": B, "n_q_heads": sh.n_q_heads,
                   "n_kv_heads": sh.n_kv_heads, "head_dim": sh.head_dim, "sink": sh.sink, "recent": sh.recent,
                   "alpha": "U(0, 1) per KV head", "parallelism": f"replicas{world}",
                   "l2": "flushed (1 GiB write) before every timed call, outside the timed interval"},
        "roofline": dict(bound, achieved=round(tf, 3), unit="TFLOP/s", frac=round(tf / bound["peak"], 4),
                         traffic=None, algorithmic_gflop=round(flops / 1e9, 3)),
        "grad_alpha": {"value": round(grad_med * 1e3, 2), "unit": "us/call",
                       "kernel": ("prefill_tc_kernel<EPI_DOT> (streaming launch + causal launch)"
                                  if bound["bound"] == "tensor" else "simt_attention_kernel"),
                       "achieved_frac_of_bf16_peak": (round(flops / (grad_med * 1e-3) / 1e12 / bound["peak"], 4)
                                                      if bound["bound"] == "tensor" else None),
                       "achieved_tflops": round(flops / (grad_med * 1e-3) / 1e12, 3),
                       "frac_of_alu": (None if bound["bound"] == "tensor"
                                       else round(flops / (grad_med * 1e-3) / 1e12 / ALU_FP32_TFLOPS, 4))},
        "gpu_launches": (4 if bound["bound"] == "tensor" else 2) * steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        # the oracle as it stands on the query heads of KV head 0, scaled to all
        # KV heads (the heads are independent and cost the same)
        G = sh.group
        t0 = time.perf_counter()
        O.gated_mix(q[0][:, :G], k[0][:, :1], v[0][:, :1], alpha[:1].astype(np.float64), sh.sink, sh.recent)
        dt_s = (time.perf_counter() - t0) * sh.n_kv_heads
        res["cpu_baseline"] = {"value": round(dt_s * 1e6, 1), "unit": "us/call", "cores": _blas_threads(),
                               "kind": "oracle",
                               "sample": f"the gated mix of KV head 0's {G} query heads (fp64 NumPy oracle), "
                                         f"scaled by the {sh.n_kv_heads} KV heads"}
    return res


# ---------------------------------------------------------------------------
# reference arm: the oracle, timed on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, wl, budget_s: float = 120.0):
    """The oracle, as it stands, timed on this host's cores on the same
    workload.  When K + W full steps would exceed `budget_s`, each step is a
    bounded sample -- sequence 0, one retrieval and one streaming KV head with
    their query heads -- and its time is scaled to the whole step by the ratio
    of algorithmic bytes; the line says which."""
    import oracle as O
    sh = S.LayerShape(wl["hq"], wl["hkv"], wl["d"], "bf16")
    if wl["kind"] != "decode":
        return {"impl": "reference", "unavailable": "the reference arm is timed on decode workloads only"}
    retrieval = S.retrieval_heads_by_seed(wl["hkv"], wl["n_ret"], seed=1)
    lengths = (S.context_lengths(wl["batch"], wl["lo"], wl["hi"]) if "batch" in wl
               else np.asarray(wl["lengths"], dtype=np.int64))
    B = len(lengths)
    sigma = S.head_sigma(wl["hkv"]) if wl.get("sigma") else None
    gate, _, _, R = O.partition_heads(S.binary_alpha(wl["hkv"], retrieval).astype(np.float64), 0.5)
    st = S.decode_state(sh, retrieval, lengths, sigma=sigma)
    total = args.warmup + args.steps
    qs, ks, vs = S.decode_steps(sh, B, total, sigma=sigma)

    def build(b_list, heads):
        return _oracle_cache(O, st, gate, sh, b_list, heads, wl.get("kv_bits", 0))

    def sl(i, b_list, heads):
        G = sh.group
        qh = [h * G + g for h in heads for g in range(G)]
        return qs[i][b_list][:, qh], ks[i][b_list][:, heads], vs[i][b_list][:, heads]

    full_heads = list(range(sh.n_kv_heads))
    full_b = list(range(B))
    cache = build(full_b, full_heads)
    t0 = time.perf_counter()
    cache.decode(*sl(0, full_b, full_heads))
    t_full = time.perf_counter() - t0
    bytes_full = _decode_bytes(sh, R, lengths + 1, wl.get("kv_bits", 0))
    if total * t_full <= budget_s:
        b_list, heads, scale, sample = full_b, full_heads, 1.0, "full decode steps"
        first = 1
    else:
        ret0 = int(np.flatnonzero(gate)[0]) if R else None
        str0 = int(np.flatnonzero(gate == 0)[0]) if R < sh.n_kv_heads else None
        heads = [h for h in (ret0, str0) if h is not None]
        b_list = [0]
        sub = S.LayerShape(sh.group * len(heads), len(heads), sh.head_dim, "bf16", sh.sink, sh.recent)
        n_ret = 1 if ret0 is not None else 0
        bytes_sample = _decode_bytes(sub, n_ret, lengths[:1] + 1, wl.get("kv_bits", 0))
        scale = bytes_full / bytes_sample
        sample = (f"sequence 0, KV heads {heads} (one retrieval, one streaming) with their query heads; "
                  f"time scaled x{scale:.1f} to the whole step by algorithmic bytes")
        cache = build(b_list, heads)
        first = 0
    for i in range(first, args.warmup):
        cache.decode(*sl(i, b_list, heads))
    t0 = time.perf_counter()
    for i in range(args.warmup, total):
        cache.decode(*sl(i, b_list, heads))
    dt = (time.perf_counter() - t0) * scale
    v = round(dt * 1e6 / args.steps, 1)
    cores = _blas_threads()
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "us/step/layer", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": B, "n_q_heads": sh.n_q_heads,
                       "n_kv_heads": sh.n_kv_heads, "head_dim": sh.head_dim, "n_retrieval": R,
                       "context": [int(lengths.min()), int(lengths.max())]},
            "cpu_baseline": {"value": v, "unit": "us/step/layer", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} timed steps after {args.warmup} warm-up steps: {sample}"},
            "e2e": {"value": v, "unit": "us/step/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

def _linear_fit(xs, ys):
    """Least-squares line y = a + b x and its coefficient of determination."""
    x = np.asarray(xs, dtype=np.float64)
    y = np.asarray(ys, dtype=np.float64)
    b, a = np.polyfit(x, y, 1)
    resid = y - (a + b * x)
    ss = float(((y - y.mean()) ** 2).sum())
    return {"intercept": round(float(a), 4), "slope": round(float(b), 4),
            "r2": round(1.0 - float((resid ** 2).sum()) / ss, 5) if ss > 0 else 1.0}


def run_ratio_sweep(args, world, rank):
    """Decode and pre-fill time against the share of retrieval heads (the
    pages report both as linear in it).  Decode: the 32K MHA layer with 0, 4,
    ..., 32 of its 32 heads retrieval; pre-fill: the 32K-token GQA prompt in
    4,096-token chunks with 0 .. 8 of its 8 KV heads retrieval.  Heads chosen
    by the same seeded draw as the workloads."""
    import copy
    dec, pre = [], []
    a2 = copy.copy(args)
    a2.steps, a2.warmup, a2.no_e2e, a2.no_cpu_baseline = 64, 3, True, True
    for r in range(0, 33, 4):
        wl = dict(WORKLOADS["mha_decode_32k"], n_ret=r, name="mha_decode_32k")
        res = run_decode(a2, wl, world, rank)
        dec.append({"n_retrieval": r, "ratio": r / 32, "us_per_step_layer": res["value"],
                    "achieved_gbs": res["roofline"]["achieved"],
                    "bytes_per_launch": res["roofline"]["algorithmic_bytes_per_launch"]})
    for r in range(0, 9):
        wl = dict(WORKLOADS["gqa_prefill_32k"], n_ret=r, name="gqa_prefill_32k")
        res = run_prefill(a2, wl, world, rank, steps=8, warmup=3)
        pre.append({"n_retrieval": r, "ratio": r / 8, "ms_total": res["roofline"]["prefill_ms_total"],
                    "tflops": res["roofline"]["achieved"]})
    return {"metric": "decode us/step/layer and pre-fill ms vs retrieval-head ratio", "n_gpus": world,
            "data": "synthetic",
            "decode": {"workload": f"mha_decode_32k (32 heads, context 32,768, "
                                   f"{args.layers or WORKLOADS['mha_decode_32k']['layers']} layers/step, 64 steps)",
                       "points": dec,
                       "fit_us_vs_ratio": _linear_fit([d["ratio"] for d in dec],
                                                      [d["us_per_step_layer"] for d in dec])},
            "prefill": {"workload": "gqa_prefill_32k (8 KV heads, 32,768 tokens in 8 chunks of 4,096)",
                        "points": pre,
                        "fit_ms_vs_ratio": _linear_fit([d["ratio"] for d in pre], [d["ms_total"] for d in pre])}}


def run_chunk_sweep(args, world, rank):
    """Pre-fill time of the 32K-token GQA prompt against the chunk length,
    with streaming heads in Lambda mode and in whole-chunk mode, next to the
    same prompt with every KV head retrieval (full attention).  The pages
    report the pre-fill speed-up over full attention growing as the chunk
    shrinks ([Review] S5 "Pre-filling performance")."""
    import copy
    a2 = copy.copy(args)
    a2.no_cpu_baseline = True
    base = WORKLOADS["gqa_prefill_32k"]
    rows = []
    for C in (512, 1024, 2048, 4096, 8192):
        point = {"chunk": C}
        for tag, extra in (("full", dict(n_ret=base["hkv"])), ("lambda", {}), ("chunk", dict(stream="chunk"))):
            wl = dict(base, chunk=C, name="gqa_prefill_32k", **extra)
            res = run_prefill(a2, wl, world, rank, warmup=3)
            point[tag + "_ms"] = res["roofline"]["prefill_ms_total"]
            point[tag + "_tflops"] = res["roofline"]["achieved"]
        point["speedup_lambda"] = round(point["full_ms"] / point["lambda_ms"], 3)
        point["speedup_chunk"] = round(point["full_ms"] / point["chunk_ms"], 3)
        rows.append(point)
    return {"metric": "pre-fill ms vs chunk length; speed-up over full attention", "n_gpus": world,
            "data": "synthetic",
            "workload": "gqa_prefill_32k (32 query / 8 KV heads, 4 retrieval, 32,768 tokens); full = 8 retrieval",
            "points": rows}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=8.0, help="seconds of oracle time per cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the pre-fill measurement of a decode run")
    ap.add_argument("--no-extra", action="store_true",
                    help="default run: skip the other decode configurations' records")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end decode measurement")
    ap.add_argument("--layers", type=int, default=0,
                    help="decode: layers per step, each with its own caches (default: the workload's)")
    ap.add_argument("--retrieval-ratio-sweep", action="store_true",
                    help="time decode and pre-fill against the share of retrieval heads (one JSON line)")
    ap.add_argument("--chunk-sweep", action="store_true",
                    help="time the pre-fill against the chunk length, both streaming modes (one JSON line)")
    ap.add_argument("--n-retrieval", type=int, default=None,
                    help="override the workload's number of retrieval KV heads (profiling)")
    ap.add_argument("--stream-prefill", choices=["lambda", "chunk"], default="lambda",
                    help="pre-fill workloads: what streaming heads see inside a chunk")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = dict(WORKLOADS[args.workload])
    if args.n_retrieval is not None:
        wl["n_ret"] = args.n_retrieval
    if args.stream_prefill == "chunk":
        wl["stream"] = "chunk"

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, wl)), flush=True)
        return 0

    import torch
    world, rank, local = _dist_init()
    torch.cuda.set_device(local)
    from head_split_kv_b200 import duo  # noqa: F401  (fails loudly without libduo.so)
    try:
        if args.retrieval_ratio_sweep:
            res = run_ratio_sweep(args, world, rank)
        elif args.chunk_sweep:
            res = run_chunk_sweep(args, world, rank)
        elif wl["kind"] == "mix":
            res = run_mix(args, wl, world, rank)
        elif wl["kind"] == "decode":
            res = run_decode(args, wl, world, rank)
            if args.workload == DEFAULT_WORKLOAD and not args.no_extra and args.n_retrieval is None:
                res["decode_configs"] = {}
                for name in EXTRA_DECODE:
                    sub = run_decode(args, WORKLOADS[name], world, rank)
                    res["decode_configs"][name] = {k: sub[k] for k in (
                        "value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline", "e2e",
                        "gpu_launches", "clocks", "cpu_baseline") if k in sub}
            if not args.no_prefill:
                pre = run_prefill(args, WORKLOADS["gqa_prefill_128k"], world, rank)
                res["prefill"] = {k: pre[k] for k in ("value", "unit", "steps", "ms_per_step", "config",
                                                      "roofline", "gpu_launches", "clocks")}
        else:
            res = run_prefill(args, wl, world, rank, steps=args.steps, warmup=args.warmup)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
