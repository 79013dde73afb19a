"""Seeded synthetic inputs for the Beam 1.0 attention core.

This module is the only code shared by the fp64 oracle's tests and the CUDA
path's tests and bench.  It holds no attention arithmetic: only random draws,
the round-to-nearest-even conversion of those draws to bf16 bit patterns, and
the shapes of the workloads.

Workload shapes follow the attention sublayer of "Beam 1.0: Local RoPE, Global
NoPE and Scalable Softmax" (section "Follow the tensors, not the parameter
label": 48 query heads over 8 KV heads, head axis 128, attention width 6,144;
section "Two attention paths in one decoder": window 512, global layers
6, 12, ..., 48, 52, maximum context 1,048,576).

Draws:
  * activations Q, K, V, gate logits and cache rows: N(0, 1), rounded to bf16;
  * RMSNorm weights: 1 + 0.1 * N(0, 1), float32;
  * per-head gate bias: N(0, 0.5) read as standard deviation 0.5, float32;
  * decode context lengths: integers uniform in [1024, 32768].

Every tensor is drawn from numpy's Philox counter-based generator keyed by
(seed, crc32(tag)), so each tensor is reproducible on its own.  Large device
tensors (the 1M-token caches) are drawn on the device with torch's seeded
Philox generator instead; both sides then read the same bits.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

N_Q_HEADS = 48
N_KV_HEADS = 8
HEAD_DIM = 128
WINDOW = 512
ROPE_THETA = 10000.0
RMS_EPS = 1e-6
SSMAX_BASE = 2048.0
SSMAX_EXP = 0.1
SOFTMAX_SCALE = 1.0 / np.sqrt(128.0)
# 1-based indices of the global (NoPE + SSMax) layers in the 52-layer decoder.
GLOBAL_LAYERS = (6, 12, 18, 24, 30, 36, 42, 48, 52)
N_LAYERS = 52
MAX_CONTEXT = 1_048_576

LOCAL, GLOBAL = 0, 1


def layer_kind(layer_1based: int) -> int:
    return GLOBAL if layer_1based in GLOBAL_LAYERS else LOCAL


def rng(seed: int, tag: str) -> np.random.Generator:
    key = (int(seed) & 0xFFFFFFFF) << 32 | zlib.crc32(tag.encode())
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, seed: int, tag: str, std: float = 1.0) -> np.ndarray:
    g = rng(seed, tag)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def norm_weight(seed: int, tag: str) -> np.ndarray:
    g = rng(seed, tag)
    return (1.0 + 0.1 * g.standard_normal(HEAD_DIM)).astype(np.float32)


def gate_bias(seed: int, tag: str = "gate_bias") -> np.ndarray:
    g = rng(seed, tag)
    return (0.5 * g.standard_normal(N_Q_HEADS)).astype(np.float32)


def normal_e4m3(shape, seed: int, tag: str, scale: float = 1.0) -> np.ndarray:
    """FP8 E4M3 codes (uint8) of seeded N(0,1) draws divided by `scale` -- synthetic
    cache contents; the draw is clamped to the finite range +-448 (a small scale pushes
    the tails past it, and the cast would make those NaN) and rounded to the nearest code
    by PyTorch's float8_e4m3fn cast."""
    import torch
    x = rng(seed, tag).standard_normal(size=shape, dtype=np.float32) / np.float32(scale)
    x = np.clip(x, -448.0, 448.0)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def device_normal_e4m3_(tensor_u8, seed: int, tag: str, scale: float = 1.0):
    """Fill a CUDA uint8 tensor in place with E4M3 codes of seeded N(0,1) / scale draws."""
    import torch
    g = torch.Generator(device=tensor_u8.device)
    g.manual_seed((int(seed) << 32) ^ zlib.crc32(tag.encode()))
    flat = tensor_u8.view(-1)
    chunk = 1 << 28
    for s in range(0, flat.numel(), chunk):
        part = flat[s:s + chunk]
        x = torch.randn(part.numel(), device=tensor_u8.device, dtype=torch.float32, generator=g)
        x = (x / scale).clamp_(-448.0, 448.0)   # the cast would turn values past 448 into NaN
        part.copy_(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return tensor_u8


@dataclass
class PrefillInputs:
    """bf16 bit patterns (uint16) of one prefill call, token-major as projected."""
    B: int
    T: int
    q: np.ndarray       # [B, T, 48*128]
    k: np.ndarray       # [B, T, 8*128]
    v: np.ndarray       # [B, T, 8*128]
    gate: np.ndarray    # [B, T, 48*128]
    q_norm_w: np.ndarray  # [128] float32
    k_norm_w: np.ndarray  # [128] float32
    gate_bias: np.ndarray  # [48] float32


def prefill_inputs(B: int, T: int, seed: int, layer: str = "L") -> PrefillInputs:
    t = f"prefill/{layer}/"
    return PrefillInputs(
        B=B, T=T,
        q=normal_bf16((B, T, N_Q_HEADS * HEAD_DIM), seed, t + "q"),
        k=normal_bf16((B, T, N_KV_HEADS * HEAD_DIM), seed, t + "k"),
        v=normal_bf16((B, T, N_KV_HEADS * HEAD_DIM), seed, t + "v"),
        gate=normal_bf16((B, T, N_Q_HEADS * HEAD_DIM), seed, t + "gate"),
        q_norm_w=norm_weight(seed, t + "qw"),
        k_norm_w=norm_weight(seed, t + "kw"),
        gate_bias=gate_bias(seed, t + "bias"),
    )


@dataclass
class DecodeInputs:
    """One decode step: the new token's projections plus the cache before the append.

    ctx[b] counts the visible keys including the new token, so the new token's
    0-based position is t = ctx - 1 and the cache holds ctx - 1 earlier rows.
    Cache rows are head-major [B][8][slots][128]; a global cache keeps position j
    at slot j, a local ring keeps it at slot j mod 512.  Cache keys are already
    normalised (and, for the local ring, already rotated).
    """
    B: int
    kind: int
    pos: np.ndarray     # [B] int64, 0-based position t of the new token
    q: np.ndarray       # [B, 48*128]
    k: np.ndarray       # [B, 8*128]
    v: np.ndarray       # [B, 8*128]
    gate: np.ndarray    # [B, 48*128]
    q_norm_w: np.ndarray
    k_norm_w: np.ndarray
    gate_bias: np.ndarray
    slots: int          # slots per sequence in the cache
    k_cache: np.ndarray | None = None  # [B, 8, slots, 128] uint16, or None when drawn on device
    v_cache: np.ndarray | None = None


def decode_contexts(n_seqs: int, seed: int, lo: int = 1024, hi: int = 32768) -> np.ndarray:
    g = rng(seed, "decode/ctx")
    return g.integers(lo, hi, size=n_seqs, endpoint=True).astype(np.int64)


def decode_inputs(kind: int, ctx: np.ndarray, slots: int, seed: int, layer: str = "L",
                  with_cache: bool = True) -> DecodeInputs:
    ctx = np.asarray(ctx, dtype=np.int64)
    B = int(ctx.shape[0])
    t = f"decode/{layer}/"
    di = DecodeInputs(
        B=B, kind=kind, pos=ctx - 1,
        q=normal_bf16((B, N_Q_HEADS * HEAD_DIM), seed, t + "q"),
        k=normal_bf16((B, N_KV_HEADS * HEAD_DIM), seed, t + "k"),
        v=normal_bf16((B, N_KV_HEADS * HEAD_DIM), seed, t + "v"),
        gate=normal_bf16((B, N_Q_HEADS * HEAD_DIM), seed, t + "gate"),
        q_norm_w=norm_weight(seed, t + "qw"),
        k_norm_w=norm_weight(seed, t + "kw"),
        gate_bias=gate_bias(seed, t + "bias"),
        slots=int(slots),
    )
    if with_cache:
        shape = (B, N_KV_HEADS, int(slots), HEAD_DIM)
        di.k_cache = normal_bf16(shape, seed, t + "kcache")
        di.v_cache = normal_bf16(shape, seed, t + "vcache")
    return di


@dataclass
class ChunkInputs:
    """One chunked-prefill call: T new tokens per sequence at positions pos0[b] ..
    pos0[b] + T - 1, plus the cache as it was before the call (rows of earlier
    positions; same layout and meaning as DecodeInputs' caches)."""
    B: int
    T: int
    kind: int
    pos0: np.ndarray    # [B] int64
    q: np.ndarray       # [B, T, 48*128]
    k: np.ndarray       # [B, T, 8*128]
    v: np.ndarray
    gate: np.ndarray
    q_norm_w: np.ndarray
    k_norm_w: np.ndarray
    gate_bias: np.ndarray
    slots: int
    k_cache: np.ndarray | None = None  # [B, 8, slots, 128] uint16
    v_cache: np.ndarray | None = None


def chunk_inputs(kind: int, T: int, pos0, slots: int, seed: int, layer: str = "L",
                 with_cache: bool = True) -> ChunkInputs:
    pos0 = np.asarray(pos0, dtype=np.int64)
    B = int(pos0.shape[0])
    p = prefill_inputs(B, T, seed, layer=f"chunk/{layer}")
    ci = ChunkInputs(B=B, T=T, kind=kind, pos0=pos0, q=p.q, k=p.k, v=p.v, gate=p.gate,
                     q_norm_w=p.q_norm_w, k_norm_w=p.k_norm_w, gate_bias=p.gate_bias,
                     slots=int(slots))
    if with_cache:
        shape = (B, N_KV_HEADS, int(slots), HEAD_DIM)
        ci.k_cache = normal_bf16(shape, seed, f"chunk/{layer}/kcache")
        ci.v_cache = normal_bf16(shape, seed, f"chunk/{layer}/vcache")
    return ci


def device_normal_bf16_(tensor, seed: int, tag: str):
    """Fill a CUDA bf16 tensor in place with seeded N(0,1) draws (torch Philox).

    Used for tensors too large to draw on the host (the 4 GiB caches of the
    1M-token decode workload).  The oracle reads the same bits back by copy.
    """
    import torch
    g = torch.Generator(device=tensor.device)
    g.manual_seed((int(seed) << 32) ^ zlib.crc32(tag.encode()))
    flat = tensor.view(-1)
    chunk = 1 << 28
    for s in range(0, flat.numel(), chunk):
        part = flat[s:s + chunk]
        part.copy_(torch.randn(part.numel(), device=tensor.device, dtype=torch.float32,
                               generator=g))
    return tensor


@dataclass
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    B: int
    T: int = 0                # prefill query tokens
    layers: tuple = ()        # layer kinds run per step
    ctx: tuple = ()           # decode contexts (visible keys incl. new token)
    seed: int = 0
    extra: dict = field(default_factory=dict)


def workload(name: str, seed: int = 1234) -> Workload:
    """The five workloads of the attention core, by name."""
    if name == "tiny_prefill":
        return Workload(name, "prefill", B=1, T=768, layers=(LOCAL, GLOBAL), seed=seed)
    if name == "batched_prefill":
        return Workload(name, "prefill", B=4, T=8192, layers=(LOCAL, GLOBAL), seed=seed)
    if name == "batched_decode":
        ctx = decode_contexts(64, seed)
        return Workload(name, "decode", B=64, layers=(LOCAL, GLOBAL), ctx=tuple(int(c) for c in ctx),
                        seed=seed, extra={"global_slots": 32768})
    if name == "long_global_prefill":
        return Workload(name, "prefill", B=1, T=131072, layers=(GLOBAL,), seed=seed)
    if name == "chunked_prefill":
        # the last 8192-token chunk of a 65,536-token prompt: 57,344 tokens already cached
        return Workload(name, "prefill", B=1, T=8192, layers=(LOCAL, GLOBAL), seed=seed,
                        extra={"pos0": 57344, "global_slots": 65536})
    if name == "decode_1m":
        kinds = tuple(layer_kind(i) for i in range(1, N_LAYERS + 1))
        return Workload(name, "decode", B=1, layers=kinds, ctx=(MAX_CONTEXT,), seed=seed,
                        extra={"global_slots": MAX_CONTEXT})
    raise KeyError(name)


def chunk_visible_pairs(T: int, pos0: int, window: int | None) -> int:
    """(query, key) pairs the mask admits for queries pos0 .. pos0+T-1 over keys 0 ..."""
    if window is None:
        return T * pos0 + T * (T + 1) // 2
    return sum(min(window, pos0 + i + 1) for i in range(T))


def visible_pairs(T: int, window: int | None) -> int:
    """Number of (query, key) pairs the mask admits for positions 0..T-1."""
    if window is None:
        return T * (T + 1) // 2
    w = min(window, T)
    return w * (w + 1) // 2 + (T - w) * window
