"""Benchmark of the Beam 1.0 attention core on B200.

One step = the prefill of one local and one global attention layer of the
batched-prefill workload (4 sequences x 8192 tokens, 48 query / 8 KV heads,
head_dim 128), including the fused KV-cache append, through the C ABI.  The
headline value is algorithmic TFLOP/s (visible (query, key) pairs x 4 x 128 x 48).
More measurements ride along on the same line: the 1M-context decode step across the
52-layer schedule over BF16 and over FP8 caches (KV-read GB/s, tokens/s), the
52-layer step verifying 8 new tokens at 1M context, the batched decode step (64
sequences, contexts in [1024, 32768]) and the chunked prefill (8192 new tokens after
57,344 cached ones, one local and one global layer; TFLOP/s).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl beam|reference]
N > 1 runs under torch.distributed.run, one process per GPU; every rank processes
its own batch (weak scaling, no collective on the data path); the time is the
max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "prefill TFLOP/s (% bf16 peak); decode KV-read GB/s and tokens/s at 1M ctx"
HEAD_FLOPS_PER_PAIR = 4 * wl.HEAD_DIM * wl.N_Q_HEADS   # QK^T and PV, all query heads
HBM_SPEC_GBPS = 8000.0   # B200 datasheet HBM3e bandwidth


def prefill_flops(B: int, T: int, kind: int, window: int = wl.WINDOW) -> int:
    pairs = wl.visible_pairs(T, window if kind == wl.LOCAL else None)
    return B * pairs * HEAD_FLOPS_PER_PAIR


def decode_kv_bytes(ctx, kind: int, window: int = wl.WINDOW, elem_bytes: int = 2) -> int:
    """Algorithmic bytes of one decode layer: the visible K and V rows (4 KiB per
    token per layer in bf16, 2 KiB in FP8) plus the new token's q, k, v, gate and output."""
    vis = sum(min(c, window) if kind == wl.LOCAL else c for c in ctx)
    per_token = 2 * wl.N_KV_HEADS * wl.HEAD_DIM * elem_bytes
    io = len(ctx) * 2 * (3 * wl.N_Q_HEADS * wl.HEAD_DIM + 2 * wl.N_KV_HEADS * wl.HEAD_DIM)
    return vis * per_token + io


def _jsonable(o):
    if isinstance(o, (np.integer,)):
        return int(o)
    if isinstance(o, (np.floating,)):
        return float(o)
    raise TypeError(type(o))


def measured_traffic():
    """DRAM traffic (read + write bytes) of one global-layer attention launch of the batched
    prefill, from the committed ncu figure in profiles/traffic.json -- only while the kernel
    source it was taken on is unchanged (its hash is recorded beside the figure)."""
    import hashlib
    try:
        src = os.path.join(ROOT, "global_nope_gqa_b200", "csrc", "prefill_tc.cuh")
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)["prefill_tc_kernel_global_batched_prefill"]
        if rec.get("kernel_source_sha256_16") == sha:
            return int(rec["bytes_per_launch"])
    except Exception:
        pass
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------ distributed helpers
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return per_rank_units * world / seconds_max


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML (read-only queries)
    every 5 ms while the timed region runs (the timed prefill region lasts ~0.1 s)."""
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}

    def __init__(self, cuda_index: int):
        self.rows = []
        self._stop = threading.Event()
        self._th = None
        self._handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                cand = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(cand)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = cand
            if h is None and pynvml.nvmlDeviceGetCount() == 1:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self._nvml, self._handle = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM) if h else None
        except Exception:
            self._handle = None
            self.max_mhz = None

    def _sample(self):
        n = self._nvml
        sm = n.nvmlDeviceGetClockInfo(self._handle, n.NVML_CLOCK_SM)
        try:
            reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
        except AttributeError:
            reasons = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._handle)
        self.rows.append((sm, reasons))

    def _run(self):
        while not self._stop.wait(0.005):
            try:
                self._sample()
            except Exception:
                pass

    def __enter__(self):
        if self._handle is not None:
            self._sample()   # first query outside the timed region
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._th:
            self._th.join(timeout=10)

    def summary(self):
        rows = self.rows[1:] or self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = sorted({name for _, r in rows for name, bit in self.BITS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ GPU arm
class PrefillLayer:
    """Device buffers of one prefill layer call (inputs drawn on the device)."""

    def __init__(self, torch, beam, kind, B, T, seed, tag):
        self.torch, self.beam, self.kind, self.B, self.T = torch, beam, kind, B, T
        self.params = beam.default_params()
        dev = "cuda"
        self.x = {}
        for name, width in (("q", 6144), ("k", 1024), ("v", 1024), ("gate", 6144)):
            t = torch.empty((B, T, width), dtype=torch.bfloat16, device=dev)
            wl.device_normal_bf16_(t, seed, f"{tag}/{name}")
            self.x[name] = t
        inp = wl.prefill_inputs(1, 1, seed, layer=tag)
        self.qw = torch.from_numpy(inp.q_norm_w).to(dev)
        self.kw = torch.from_numpy(inp.k_norm_w).to(dev)
        self.bias = torch.from_numpy(inp.gate_bias).to(dev)
        self.out = torch.empty_like(self.x["q"])
        self.layout = beam.beam_kv_layout(kind, self.params, B, T)
        self.kc = torch.empty(self.layout.bytes_k // 2, dtype=torch.bfloat16, device=dev)
        self.vc = torch.empty_like(self.kc)
        self.ws = torch.empty(beam.beam_prefill_workspace_bytes(self.params, B, T),
                              dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, x=None, out=None):
        x = x or self.x
        self.beam.beam_attn_prefill(self.kind, self.params, x["q"], x["k"], x["v"], x["gate"],
                                    self.qw, self.kw, self.bias, out if out is not None else self.out,
                                    self.kc, self.vc, self.layout, workspace=self.ws,
                                    dev_status=self.status)

    launches_per_call = 2  # prologue + attention


class DecodeLayer:
    def __init__(self, torch, beam, kind, ctx, slots, seed, tag, cache=None, fp8=False):
        self.torch, self.beam, self.kind, self.fp8 = torch, beam, kind, fp8
        self.k_scale, self.v_scale = 0.5, 1.0
        self.params = beam.default_params()
        dev = "cuda"
        ctx = np.asarray(ctx, np.int64)
        self.B = len(ctx)
        di = wl.decode_inputs(kind, ctx, slots, seed, layer=tag, with_cache=False)
        self.inputs = di   # the host bits of the new token's tensors (for parity checks)

        def d(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
        self.q, self.k, self.v, self.gate = d(di.q), d(di.k), d(di.v), d(di.gate)
        self.qw = torch.from_numpy(di.q_norm_w).to(dev)
        self.kw = torch.from_numpy(di.k_norm_w).to(dev)
        self.bias = torch.from_numpy(di.gate_bias).to(dev)
        self.pos = torch.from_numpy(di.pos).to(dev)
        if fp8:
            self.layout = beam.beam_kv_layout_fp8(kind, self.params, self.B, slots)
        else:
            self.layout = beam.beam_kv_layout(kind, self.params, self.B, slots)
        if cache is None and fp8:
            self.kc = torch.empty(self.layout.bytes_k, dtype=torch.uint8, device=dev)
            self.vc = torch.empty_like(self.kc)
            wl.device_normal_e4m3_(self.kc, seed, f"{tag}/kc", self.k_scale)
            wl.device_normal_e4m3_(self.vc, seed, f"{tag}/vc", self.v_scale)
        elif cache is None:
            self.kc = torch.empty(self.layout.bytes_k // 2, dtype=torch.bfloat16, device=dev)
            self.vc = torch.empty_like(self.kc)
            wl.device_normal_bf16_(self.kc, seed, f"{tag}/kc")
            wl.device_normal_bf16_(self.vc, seed, f"{tag}/vc")
        else:
            self.kc, self.vc = cache
        self.out = torch.empty((self.B, 6144), dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(max(16, beam.beam_decode_workspace_bytes(kind, self.params, self.B,
                                                                      self.layout)),
                              dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.bytes = decode_kv_bytes(ctx, kind, elem_bytes=1 if fp8 else 2)
        # a ring layer is one launch; a global layer is split-K + combine
        self.launches_per_call = 1 if kind == wl.LOCAL else 2

    def run(self):
        if self.fp8:
            self.beam.beam_attn_decode_fp8(self.kind, self.params, self.q, self.k, self.v,
                                           self.gate, self.qw, self.kw, self.bias, self.pos,
                                           self.kc, self.vc, self.layout, self.k_scale,
                                           self.v_scale, self.out, workspace=self.ws,
                                           dev_status=self.status)
            return
        self.beam.beam_attn_decode(self.kind, self.params, self.q, self.k, self.v, self.gate,
                                   self.qw, self.kw, self.bias, self.pos, self.kc, self.vc,
                                   self.layout, self.out, workspace=self.ws, dev_status=self.status)



def time_loop(torch, fn, steps, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(steps):
        fn()
    ev[1].record()
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / 1e3 / steps


def decode_step_layers(torch, beam, context, seed, fp8=False, tag="d1m"):
    """The 52 decode calls of one step of the decoder (schedule: workloads.layer_kind),
    B=1 at `context` visible keys: a global layer's cache holds `context` slots, a local
    layer's the 512-slot ring.  The 1M-context decode bench and the 52-layer parity test
    both build their step here."""
    layers = []
    for i in range(1, wl.N_LAYERS + 1):
        kind = wl.layer_kind(i)
        slots = context if kind == wl.GLOBAL else wl.WINDOW
        layers.append(DecodeLayer(torch, beam, kind, [context], slots, seed, f"{tag}/L{i}",
                                  fp8=fp8))
    return layers


def capture_step(torch, layers):
    """Capture one call of every layer, in schedule order, as one CUDA graph."""
    def step():
        for L in layers:
            L.run()

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step()  # warm the launch path outside capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    return graph


def bench_decode_1m(torch, beam, steps, warmup, seed, fp8=False):
    """52-layer decode step at context 1,048,576: 9 global layers with 4 GiB caches
    (2 GiB in FP8), 43 local rings; the whole step is one CUDA graph replay."""
    layers = decode_step_layers(torch, beam, wl.MAX_CONTEXT, seed, fp8=fp8)
    total_bytes = sum(L.bytes for L in layers)
    glob_bytes = sum(L.bytes for L in layers if L.kind == wl.GLOBAL)
    graph = capture_step(torch, layers)
    sec = time_loop(torch, graph.replay, steps, warmup)
    # the dominant kernel: one global layer's decode call timed alone
    g0 = next(L for L in layers if L.kind == wl.GLOBAL)
    sec_g = time_loop(torch, g0.run, steps * 4, warmup)
    status = [int(L.status.item()) for L in layers]
    assert all(s == 0 for s in status), status
    res = {
        "workload": ("decode_1m_fp8: B=1, context 1048576, 52 layers, FP8 E4M3 caches (9 global "
                     "2 GiB caches, 43 x 512-slot rings)") if fp8 else
                    "decode_1m: B=1, context 1048576, 52 layers (9 global 4 GiB caches, 43 x 512-slot rings)",
        "ms_per_token": sec * 1e3,
        "tokens_per_s": 1.0 / sec,
        "kv_read_GBps": total_bytes / sec / 1e9,
        "bytes_per_step": total_bytes,
        "global_layer_GBps": g0.bytes / sec_g / 1e9,
        "global_layer_ms": sec_g * 1e3,
        "gpu_launches_per_step": sum(L.launches_per_call for L in layers),
    }
    del graph, layers
    torch.cuda.empty_cache()
    return res, glob_bytes


class ChunkLayer:
    """One chunk call (T new tokens after pos0 cached ones, B = 1) with its own caches
    (BF16, or FP8 E4M3 codes with one scale per cache tensor)."""

    def __init__(self, torch, beam, kind, T, pos0, slots, seed, tag, fp8=False):
        self.beam, self.kind, self.fp8 = beam, kind, fp8
        self.k_scale, self.v_scale = 0.0173, 3.7   # scales an amax / 448 rule gives
        self.params = beam.default_params()
        dev = "cuda"
        ci = wl.chunk_inputs(kind, T, [pos0], slots, seed, layer=tag, with_cache=False)

        def d(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
        self.q, self.k, self.v, self.gate = d(ci.q), d(ci.k), d(ci.v), d(ci.gate)
        self.qw = torch.from_numpy(ci.q_norm_w).to(dev)
        self.kw = torch.from_numpy(ci.k_norm_w).to(dev)
        self.bias = torch.from_numpy(ci.gate_bias).to(dev)
        self.pos0 = torch.from_numpy(ci.pos0).to(dev)
        if fp8:
            self.layout = beam.beam_kv_layout_fp8(kind, self.params, 1, slots)
            self.kc = torch.empty(self.layout.bytes_k, dtype=torch.uint8, device=dev)
            self.vc = torch.empty_like(self.kc)
            wl.device_normal_e4m3_(self.kc, seed, f"{tag}/kc", self.k_scale)
            wl.device_normal_e4m3_(self.vc, seed, f"{tag}/vc", self.v_scale)
            ws = beam.beam_prefill_chunk_fp8_workspace_bytes(kind, self.params, 1, T, self.layout)
        else:
            self.layout = beam.beam_kv_layout(kind, self.params, 1, slots)
            self.kc = torch.empty(self.layout.bytes_k // 2, dtype=torch.bfloat16, device=dev)
            self.vc = torch.empty_like(self.kc)
            wl.device_normal_bf16_(self.kc, seed, f"{tag}/kc")
            wl.device_normal_bf16_(self.vc, seed, f"{tag}/vc")
            ws = beam.beam_prefill_chunk_workspace_bytes(kind, self.params, 1, T, self.layout)
        self.out = torch.empty_like(self.q)
        self.ws = torch.empty(max(16, ws), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        vis = wl.chunk_visible_pairs(T, pos0, wl.WINDOW if kind == wl.LOCAL else None)
        self.flops = vis * HEAD_FLOPS_PER_PAIR
        ctx = [pos0 + T]
        self.bytes = decode_kv_bytes(ctx, kind, elem_bytes=1 if fp8 else 2) + \
            (T - 1) * 2 * 2 * (3 * 6144 + 2 * 1024)
        # prologue (with the ring copy or the value padding), split-K attention, and for a
        # global layer at 1M context (37 runs per KV head) the merge kernel; a local layer's
        # 5 runs are merged by the attention kernel's last CTA
        self.launches_per_call = 2 if kind == wl.LOCAL else 3

    def run(self):
        if self.fp8:
            self.beam.beam_attn_prefill_chunk_fp8(
                self.kind, self.params, self.q, self.k, self.v, self.gate, self.qw, self.kw,
                self.bias, self.pos0, self.out, self.kc, self.vc, self.layout, self.k_scale,
                self.v_scale, workspace=self.ws, dev_status=self.status)
            return
        self.beam.beam_attn_prefill_chunk(self.kind, self.params, self.q, self.k, self.v, self.gate,
                                          self.qw, self.kw, self.bias, self.pos0, self.out,
                                          self.kc, self.vc, self.layout, workspace=self.ws,
                                          dev_status=self.status)


def bench_decode_multi_1m(torch, beam, steps, warmup, seed, T=8, fp8=False):
    """52-layer step verifying T = 8 drafted tokens at context 1,048,576 (the last T positions
    of the 1M window): every layer is one chunk call of T new tokens; one CUDA graph.  With
    fp8, over FP8 E4M3 caches (9 global caches of 2 GiB)."""
    pos0 = wl.MAX_CONTEXT - T
    layers = []
    for i in range(1, wl.N_LAYERS + 1):
        kind = wl.layer_kind(i)
        slots = wl.MAX_CONTEXT if kind == wl.GLOBAL else wl.WINDOW
        layers.append(ChunkLayer(torch, beam, kind, T, pos0, slots, seed, f"dm/L{i}", fp8=fp8))

    def step():
        for L in layers:
            L.run()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step()
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    sec = time_loop(torch, graph.replay, steps, warmup)
    assert all(int(L.status.item()) == 0 for L in layers)
    total_bytes = sum(L.bytes for L in layers)
    res = {
        "workload": (f"decode_multi_1m_fp8: B=1, {T} new tokens per step after {pos0} cached, 52 "
                     "layers, FP8 E4M3 caches (9 global 2 GiB caches, 43 x 512-slot rings)") if fp8
        else (f"decode_multi_1m: B=1, {T} new tokens per step after {pos0} cached, 52 layers "
              "(9 global 4 GiB caches, 43 x 512-slot rings)"),
        "ms_per_step": sec * 1e3,
        "tokens_per_s": T / sec,
        "kv_read_GBps": total_bytes / sec / 1e9,
        "gpu_launches_per_step": sum(L.launches_per_call for L in layers),
    }
    del graph, layers
    torch.cuda.empty_cache()
    return res


def bench_decode_batched(torch, beam, steps, warmup, seed):
    w = wl.workload("batched_decode", seed)
    g = DecodeLayer(torch, beam, wl.GLOBAL, w.ctx, w.extra["global_slots"], seed, "bdec/g")
    l = DecodeLayer(torch, beam, wl.LOCAL, w.ctx, wl.WINDOW, seed, "bdec/l")

    def step():
        g.run()
        l.run()
    sec = time_loop(torch, step, steps * 4, warmup)
    res = {
        "workload": "batched_decode: 64 sequences, contexts U[1024,32768], one global + one local layer",
        "ms_per_step": sec * 1e3,
        "tokens_per_s": w.B / sec,
        "kv_read_GBps": (g.bytes + l.bytes) / sec / 1e9,
    }
    del g, l
    torch.cuda.empty_cache()
    return res


def bench_prefill_chunk(torch, beam, steps, warmup, seed):
    """The chunked-prefill workload: one local and one global layer call of 8192 new
    tokens after 57,344 cached ones (cache contents drawn on the device)."""
    w = wl.workload("chunked_prefill", seed)
    p0 = w.extra["pos0"]
    params = beam.default_params()
    dev = "cuda"
    x = {}
    for name, width in (("q", 6144), ("k", 1024), ("v", 1024), ("gate", 6144)):
        t = torch.empty((w.B, w.T, width), dtype=torch.bfloat16, device=dev)
        wl.device_normal_bf16_(t, seed, f"chunk/{name}")
        x[name] = t
    inp = wl.prefill_inputs(1, 1, seed, layer="chunk")
    qw = torch.from_numpy(inp.q_norm_w).to(dev)
    kw = torch.from_numpy(inp.k_norm_w).to(dev)
    bias = torch.from_numpy(inp.gate_bias).to(dev)
    out = torch.empty_like(x["q"])
    pos0 = torch.full((w.B,), p0, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    calls, res = [], {"workload": f"chunked_prefill: B={w.B}, T={w.T} new tokens after {p0} "
                                  "cached (global cache 65536 slots; local 512-slot ring)"}
    for kind in (wl.LOCAL, wl.GLOBAL):
        slots = w.extra["global_slots"] if kind == wl.GLOBAL else wl.WINDOW
        layout = beam.beam_kv_layout(kind, params, w.B, slots)
        kc = torch.empty(layout.bytes_k // 2, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        wl.device_normal_bf16_(kc, seed, f"chunk/kc{kind}")
        wl.device_normal_bf16_(vc, seed, f"chunk/vc{kind}")
        ws = torch.empty(max(16, beam.beam_prefill_chunk_workspace_bytes(kind, params, w.B, w.T,
                                                                         layout)),
                         dtype=torch.uint8, device=dev)

        def call(kind=kind, layout=layout, kc=kc, vc=vc, ws=ws):
            # the same position every step: the call appends the same rows again
            beam.beam_attn_prefill_chunk(kind, params, x["q"], x["k"], x["v"], x["gate"], qw, kw,
                                         bias, pos0, out, kc, vc, layout, workspace=ws,
                                         dev_status=status)
        sec = time_loop(torch, call, steps, warmup)
        flops = w.B * wl.chunk_visible_pairs(w.T, p0, wl.WINDOW if kind == wl.LOCAL else None) \
            * HEAD_FLOPS_PER_PAIR
        name = "local" if kind == wl.LOCAL else "global"
        res[f"{name}_ms"] = sec * 1e3
        res[f"{name}_tflops"] = flops / sec / 1e12
        calls.append((sec, flops))
    assert int(status.item()) == 0, "device status set during the chunked-prefill bench"
    res["tflops"] = sum(f for _, f in calls) / sum(s for s, _ in calls) / 1e12
    res["gpu_launches_per_step"] = 4   # per layer: prologue (with the ring copy or padding), attention
    del x, out
    torch.cuda.empty_cache()
    return res


def bench_long_global_prefill(torch, beam, steps, warmup, seed, pk):
    """The long-context global prefill: one global-layer call over B=1, T=131072 (211 TFLOP,
    a(p) up to p = 131072).  A call runs for about 0.2 s under the power cap, so it is
    set against the sustained bf16 figure as well as the burst one."""
    w = wl.workload("long_global_prefill", seed)
    L = PrefillLayer(torch, beam, wl.GLOBAL, w.B, w.T, w.seed, "bench/long")
    sec = time_loop(torch, L.run, steps, warmup)
    assert int(L.status.item()) == 0, "device status set during the long-prefill bench"
    flops = prefill_flops(w.B, w.T, wl.GLOBAL)
    tf = flops / sec / 1e12
    res = {"workload": f"long_global_prefill: B={w.B}, T={w.T}, global layer only",
           "ms": sec * 1e3, "tflop": flops / 1e12, "tflops": tf,
           "pct_of_bf16_peak": round(100 * tf / pk["bf16_tflops"], 2),
           "pct_of_sustained_bf16": round(100 * tf / pk["bf16_tflops_sustained"], 2),
           "gpu_launches_per_step": L.launches_per_call}
    del L
    torch.cuda.empty_cache()
    return res


_CPU_INPUTS = {}
L2_NOTE = "inputs larger than L2 (Q alone is 403 MB per layer)"
PREFILL_WORKLOAD = ("batched_prefill: B={B}, T={T} per GPU, layers={layers} (local: window 512, "
                    "RoPE; global: NoPE, SSMax), 48 q / 8 kv heads, d=128, fused KV append")


def cpu_baseline_prefill(seconds_target=10.0, seconds_cap=30.0, seed=1234):
    """The fp64 oracle, as it stands, on a bounded row sample of the batched-prefill
    workload (B=4, T=8192, both layers): query rows drawn uniformly from 0..8191 of the 4
    sequences, all 48 heads, alternately from the global and the local layer.  Each layer's
    rate (algorithmic FLOPs of its sampled rows / its time) is measured separately, and the
    step's rate combines them by the step's FLOPs: (F_g + F_l) / (F_g / r_g + F_l / r_l).
    Returns TFLOP/s and the sample description."""
    import oracle
    P = oracle.params()
    B, T = 4, 8192
    key = (B, T, seed)
    if key not in _CPU_INPUTS:
        _CPU_INPUTS.clear()
        _CPU_INPUTS[key] = wl.prefill_inputs(B, T, seed, layer="cpu")
    inp = _CPU_INPUTS[key]
    rng = np.random.default_rng(seed)
    threads = oracle.n_threads_default()
    kinds = ((oracle.GLOBAL, wl.GLOBAL), (oracle.LOCAL, wl.LOCAL))
    flops = {kw: 0 for _, kw in kinds}
    secs = {kw: 0.0 for _, kw in kinds}
    rows = {kw: 0 for _, kw in kinds}
    batch = max(8, threads)
    t0 = time.perf_counter()
    while True:
        for ko, kw in kinds:
            rb = rng.integers(0, B, size=batch)
            rt = rng.integers(0, T, size=batch)
            t1 = time.perf_counter()
            oracle.prefill_rows(ko, P, inp.q, inp.k, inp.v, inp.gate, inp.q_norm_w, inp.k_norm_w,
                                inp.gate_bias, rb, rt, n_threads=threads)
            secs[kw] += time.perf_counter() - t1
            vis = rt + 1 if kw == wl.GLOBAL else np.minimum(rt + 1, wl.WINDOW)
            flops[kw] += int(vis.sum()) * HEAD_FLOPS_PER_PAIR
            rows[kw] += batch
        el = time.perf_counter() - t0
        if el >= seconds_target or el >= seconds_cap:
            break
    step = {kw: prefill_flops(B, T, kw) for _, kw in kinds}
    est = sum(step[kw] / (flops[kw] / secs[kw]) for _, kw in kinds)   # oracle seconds per step
    return {"value": sum(step.values()) / est / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows[wl.GLOBAL]} global-layer and {rows[wl.LOCAL]} local-layer query rows "
                      f"x 48 heads of batched_prefill (B=4, T=8192), uniform row positions, "
                      f"{secs[wl.GLOBAL]:.1f} s + {secs[wl.LOCAL]:.1f} s; step rate = the two "
                      "layers' rates combined by the step's FLOPs"}


def e2e_prefill(torch, beam, layers, steps, warmup):
    """Same metric through the public call with pinned host buffers: every step copies the
    step's inputs host->device and reads the outputs back.  The step is streamed one
    sequence at a time (the call with B = 1, caches offset to that sequence): uploads on one
    stream into two alternating device buffers, the attention on the compute stream, the
    read-back on a third stream, so the upload of sequence b + 1 and the read-back of b - 1
    overlap the attention of b (PCIe is full duplex)."""
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    compute = torch.cuda.current_stream()
    host_in = [{k: v.cpu().pin_memory() for k, v in L.x.items()} for L in layers]
    host_out = [torch.empty(L.out.shape, dtype=L.out.dtype, pin_memory=True) for L in layers]
    B, T = layers[0].B, layers[0].T
    dev_in = [{k: torch.empty_like(v[:1]) for k, v in layers[0].x.items()} for _ in range(2)]
    params = layers[0].params
    ws = torch.empty(beam.beam_prefill_workspace_bytes(params, 1, T), dtype=torch.uint8,
                     device="cuda")
    one = {L.kind: beam.beam_kv_layout(L.kind, params, 1, T) for L in layers}
    h2d = sum(v.numel() * v.element_size() for d in host_in for v in d.values())
    d2h = sum(o.numel() * o.element_size() for o in host_out)
    free = [torch.cuda.Event() for _ in range(2)]
    loaded = [torch.cuda.Event() for _ in range(2)]
    done = torch.cuda.Event()
    for e in free:
        e.record(compute)

    def step():
        i = 0
        for L, hi, ho in zip(layers, host_in, host_out):
            kc = L.kc.view(B, -1)
            vc = L.vc.view(B, -1)
            for b in range(B):
                buf = i % 2
                with torch.cuda.stream(h2d_stream):
                    h2d_stream.wait_event(free[buf])
                    for k in hi:
                        dev_in[buf][k].copy_(hi[k][b:b + 1], non_blocking=True)
                    loaded[buf].record(h2d_stream)
                compute.wait_event(loaded[buf])
                x = dev_in[buf]
                beam.beam_attn_prefill(L.kind, params, x["q"], x["k"], x["v"], x["gate"], L.qw,
                                       L.kw, L.bias, L.out[b:b + 1], kc[b], vc[b], one[L.kind],
                                       workspace=ws, dev_status=L.status)
                free[buf].record(compute)
                done.record(compute)
                with torch.cuda.stream(d2h_stream):
                    d2h_stream.wait_event(done)
                    ho[b:b + 1].copy_(L.out[b:b + 1], non_blocking=True)
                i += 1
        compute.wait_stream(d2h_stream)
    sec = time_loop(torch, step, max(1, steps // 2), max(1, warmup // 2))
    return sec, h2d, d2h


def run_gpu(args):
    import torch
    rank, world, local_rank = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    import global_nope_gqa_b200 as beam
    beam.lib()
    pk = peaks()
    w = wl.workload("batched_prefill", args.seed + rank)
    if args.batch:
        w.B = args.batch
    kinds = {"both": (wl.LOCAL, wl.GLOBAL), "global": (wl.GLOBAL,), "local": (wl.LOCAL,)}[args.layers]
    layers = [PrefillLayer(torch, beam, kind, w.B, w.T, w.seed, f"bench/{kind}") for kind in kinds]
    flops_step = sum(prefill_flops(w.B, w.T, L.kind) for L in layers)

    # Each layer call is captured once in a CUDA graph and replayed: the timed region is
    # then a handful of host calls, so nothing on the host can starve the GPU between
    # kernels (the replays run exactly the kernels a direct call launches).
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for L in layers:
            L.run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for L in layers:
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph):
            L.run()
        graphs.append(gph)

    for _ in range(args.warmup):
        for gph in graphs:
            gph.replay()
    torch.cuda.synchronize()
    # per-call events on the launching stream for the dominant (global) layer
    stream = torch.cuda.current_stream()
    ev_step = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev_g = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        ev_step[0].record(stream)
        for i in range(args.steps):
            for L, gph in zip(layers, graphs):
                if L.kind == wl.GLOBAL:
                    ev_g[i][0].record(stream)
                gph.replay()
                if L.kind == wl.GLOBAL:
                    ev_g[i][1].record(stream)
        ev_step[1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sec = ev_step[0].elapsed_time(ev_step[1]) / 1e3 / args.steps
    has_global = any(L.kind == wl.GLOBAL for L in layers)
    sec_g = (sum(a.elapsed_time(b) for a, b in ev_g) / 1e3 / args.steps) if has_global else sec
    sec_max = max_over_ranks(sec, "cuda")
    value = aggregate(flops_step, world, sec_max) / 1e12
    for L in layers:
        assert int(L.status.item()) == 0, "device status set during the bench"

    g_flops = prefill_flops(w.B, w.T, wl.GLOBAL) if has_global else flops_step
    achieved = g_flops / sec_g / 1e12
    if args.no_e2e:
        e2e_sec, h2d, d2h = float("nan"), 0, 0
    else:
        e2e_sec, h2d, d2h = e2e_prefill(torch, beam, layers, args.steps, args.warmup)
        e2e_sec = max_over_ranks(e2e_sec, "cuda")
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(sec_max * 1e3, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: N(0,1) bf16 activations drawn on the device (seeded torch Philox)",
        "config": {"workload": PREFILL_WORKLOAD.format(B=w.B, T=w.T, layers=args.layers),
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
                   "l2": L2_NOTE},
        "pct_of_bf16_peak": round(100 * value / world / pk["bf16_tflops"], 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                     "traffic": measured_traffic() if (w.B, w.T, has_global) == (4, 8192, True)
                     else None,
                     "kernel": "global-layer prefill call: K prologue + prefill_tc_kernel "
                               "(traffic: prefill_tc_kernel, ncu)",
                     "peak_source": pk["source"] + " burst bf16"},
        "e2e": None if args.no_e2e else {
            "value": round(aggregate(flops_step, world, e2e_sec) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * sum(L.launches_per_call for L in layers),
        "clocks": clocks.summary(),
    }
    del graphs, layers
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_decode:
        def hbm_fracs(d):
            # pct_of_hbm: of the measured read+write copy bandwidth (MEASURED_PEAKS.json);
            # a read-only stream can exceed it.  pct_of_hbm_spec: of the 8 TB/s datasheet figure.
            d["pct_of_hbm"] = round(100 * d["kv_read_GBps"] / pk["hbm_gbs"], 2)
            d["pct_of_hbm_spec"] = round(100 * d["kv_read_GBps"] / HBM_SPEC_GBPS, 2)
            d["hbm_peak_note"] = (f"pct_of_hbm: of {pk['hbm_gbs']} GB/s, a measured read+write "
                                  f"copy ({pk['source']}); pct_of_hbm_spec: of {HBM_SPEC_GBPS} GB/s")
            return d
        d1m, _ = bench_decode_1m(torch, beam, args.steps, args.warmup, args.seed)
        result["decode_1m"] = hbm_fracs(d1m)
        db = bench_decode_batched(torch, beam, args.steps, args.warmup, args.seed)
        result["decode_batched"] = hbm_fracs(db)
        d8, _ = bench_decode_1m(torch, beam, args.steps, args.warmup, args.seed, fp8=True)
        result["decode_1m_fp8"] = hbm_fracs(d8)
        dm = bench_decode_multi_1m(torch, beam, args.steps, args.warmup, args.seed)
        result["decode_multi_1m"] = hbm_fracs(dm)
        dm8 = bench_decode_multi_1m(torch, beam, args.steps, args.warmup, args.seed, fp8=True)
        result["decode_multi_1m_fp8"] = hbm_fracs(dm8)
        pc = bench_prefill_chunk(torch, beam, args.steps, args.warmup, args.seed)
        pc["pct_of_bf16_peak"] = round(100 * pc["tflops"] / pk["bf16_tflops"], 2)
        result["prefill_chunk"] = pc
        result["prefill_long_global"] = bench_long_global_prefill(
            torch, beam, min(args.steps, 5), args.warmup, args.seed, pk)
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline_prefill(seed=args.seed)
    if rank == 0:
        print(json.dumps(result, default=_jsonable), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_decode_case(args):
    """Profiling case: one global-layer decode call (B=1) at --context, BF16 or FP8 cache, or
    one 8-new-token chunk call (multi8), timed alone; prints one JSON line (not the headline)."""
    import torch
    torch.cuda.set_device(0)
    import global_nope_gqa_b200 as beam
    beam.lib()
    if args.decode_case in ("multi8", "multi8_local", "multi8_fp8"):
        glob = args.decode_case != "multi8_local"
        fp8 = args.decode_case == "multi8_fp8"
        kind, slots = (wl.GLOBAL, args.context) if glob else (wl.LOCAL, wl.WINDOW)
        L = ChunkLayer(torch, beam, kind, 8, args.context - 8, slots, args.seed, "case", fp8=fp8)
        sec = time_loop(torch, L.run, args.steps, args.warmup)
        assert int(L.status.item()) == 0
        print(json.dumps({"case": f"{'global' if glob else 'local'} chunk of 8 new tokens, B=1, "
                                  f"context {args.context}{', FP8 E4M3 cache' if fp8 else ''}",
                          "ms": sec * 1e3, "GBps": L.bytes / sec / 1e9}), flush=True)
        return
    fp8 = args.decode_case == "fp8"
    L = DecodeLayer(torch, beam, wl.GLOBAL, [args.context], args.context, args.seed, "case",
                    fp8=fp8)
    sec = time_loop(torch, L.run, args.steps, args.warmup)
    assert int(L.status.item()) == 0
    print(json.dumps({"case": f"global decode, B=1, context {args.context}, "
                              f"{'FP8 E4M3' if fp8 else 'BF16'} cache",
                      "ms": sec * 1e3, "GBps": L.bytes / sec / 1e9}), flush=True)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        b = cpu_baseline_prefill(seconds_target=3.0, seconds_cap=20.0, seed=args.seed)
        if i >= args.warmup:
            per_step.append(b)
        base = b
    value = statistics.mean(x["value"] for x in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: N(0,1) bf16 activations (seeded numpy Philox)",
        "config": {"workload": PREFILL_WORKLOAD.format(B=4, T=8192, layers="both"),
                   "global_batch": 4, "seq_len": 8192, "parallelism": "none (host cores)",
                   "l2": L2_NOTE},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": base["cores"],
                         "kind": "oracle", "sample": base["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line, default=_jsonable), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="beam", choices=["beam", "reference"])
    ap.add_argument("--seed", type=int, default=1234)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", default="both", choices=["both", "global", "local"],
                    help="prefill layers per step (profiling cases; the headline step is both)")
    ap.add_argument("--batch", type=int, default=0, help="override B (profiling cases)")
    ap.add_argument("--decode-case", choices=["bf16", "fp8", "multi8", "multi8_local", "multi8_fp8"], default=None,
                    help="profiling case: time one global decode call at --context only")
    ap.add_argument("--context", type=int, default=wl.MAX_CONTEXT)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.decode_case:
        run_decode_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
