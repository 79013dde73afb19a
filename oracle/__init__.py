"""fp64 CPU oracle of the Beam 1.0 attention core -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
import this package.  The product path never does: it shares no code with the
oracle and fails loudly when its CUDA library is missing.

The arithmetic lives in ``beam_oracle.c`` (plain C, double precision, POSIX
threads over whole output rows).  This module only builds it with gcc, loads it
with ctypes and marshals numpy arrays.  Parity of the full attention output
against the source page is pinned only through the invariants and closed forms
in ``tests/test_oracle_pins.py``: the page prints no worked attention output.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "beam_oracle.c")
_LIB = os.path.join(_HERE, "libbeam_oracle.so")

LOCAL, GLOBAL = 0, 1


class Params(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double),
        ("ssmax_base", ctypes.c_double), ("ssmax_exp", ctypes.c_double),
        ("softmax_scale", ctypes.c_double),
    ]


def params(n_q_heads=48, n_kv_heads=8, head_dim=128, window=512, rope_theta=10000.0,
           rms_eps=1e-6, ssmax_base=2048.0, ssmax_exp=0.1, softmax_scale=None) -> Params:
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(head_dim)
    return Params(n_q_heads, n_kv_heads, head_dim, window, rope_theta, rms_eps, ssmax_base,
                  ssmax_exp, softmax_scale)


def build(force: bool = False) -> str:
    """Compile beam_oracle.c with gcc into libbeam_oracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.POINTER
        dp, fp, u16p, i64p = P(ctypes.c_double), P(ctypes.c_float), P(ctypes.c_uint16), P(ctypes.c_int64)
        pp = P(Params)
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_ssmax_factor.restype = ctypes.c_double
        L.oracle_ssmax_factor.argtypes = [ctypes.c_int64, ctypes.c_double, ctypes.c_double]
        L.oracle_sigmoid.restype = ctypes.c_double
        L.oracle_sigmoid.argtypes = [ctypes.c_double]
        L.oracle_rms_norm.restype = None
        L.oracle_rms_norm.argtypes = [dp, dp, ctypes.c_int, ctypes.c_double, dp]
        L.oracle_rope.restype = None
        L.oracle_rope.argtypes = [dp, ctypes.c_int, ctypes.c_int64, ctypes.c_double]
        L.oracle_softmax.restype = None
        L.oracle_softmax.argtypes = [dp, ctypes.c_int64, dp]
        L.oracle_visible.restype = ctypes.c_int
        L.oracle_visible.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_cache_slot.restype = ctypes.c_int64
        L.oracle_cache_slot.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64]
        L.oracle_prepare_query.restype = None
        L.oracle_prepare_query.argtypes = [ctypes.c_int, pp, u16p, fp, ctypes.c_int64, dp]
        L.oracle_prepare_key.restype = None
        L.oracle_prepare_key.argtypes = [ctypes.c_int, pp, u16p, fp, ctypes.c_int64, dp]
        L.oracle_prefill_rows.restype = ctypes.c_int
        L.oracle_prefill_rows.argtypes = [ctypes.c_int, pp, ctypes.c_int, ctypes.c_int, u16p, u16p,
                                          u16p, u16p, fp, fp, fp, ctypes.c_int64, i64p, i64p, dp,
                                          ctypes.c_int]
        L.oracle_prefill_row_heads.restype = ctypes.c_int
        L.oracle_prefill_row_heads.argtypes = [ctypes.c_int, pp, ctypes.c_int, ctypes.c_int, u16p,
                                               u16p, u16p, u16p, fp, fp, fp, ctypes.c_int64, i64p,
                                               i64p, i64p, dp, ctypes.c_int]
        L.oracle_decode.restype = ctypes.c_int
        L.oracle_decode.argtypes = [ctypes.c_int, pp, ctypes.c_int, u16p, u16p, u16p, u16p, fp, fp,
                                    fp, i64p, u16p, u16p, ctypes.c_int64, dp, ctypes.c_int]
        L.oracle_prefill_chunk_rows.restype = ctypes.c_int
        L.oracle_prefill_chunk_rows.argtypes = [
            ctypes.c_int, pp, ctypes.c_int, ctypes.c_int, u16p, u16p, u16p, u16p, fp, fp, fp,
            ctypes.POINTER(ctypes.c_int64), u16p, u16p, ctypes.c_int64, ctypes.c_int64,
            ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), dp, ctypes.c_int]
        u8p = ctypes.POINTER(ctypes.c_uint8)
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_decode_fp8.restype = ctypes.c_int
        L.oracle_decode_fp8.argtypes = [
            ctypes.c_int, pp, ctypes.c_int, u16p, u16p, u16p, u16p, fp, fp, fp,
            ctypes.POINTER(ctypes.c_int64), u8p, u8p, ctypes.c_int64, ctypes.c_double,
            ctypes.c_double, dp, ctypes.c_int]
        L.oracle_prefill_chunk_rows_fp8.restype = ctypes.c_int
        L.oracle_prefill_chunk_rows_fp8.argtypes = [
            ctypes.c_int, pp, ctypes.c_int, ctypes.c_int, u16p, u16p, u16p, u16p, fp, fp, fp,
            ctypes.POINTER(ctypes.c_int64), u8p, u8p, ctypes.c_int64, ctypes.c_double,
            ctypes.c_double, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
            ctypes.POINTER(ctypes.c_int64), dp, ctypes.c_int]
        L.oracle_kv_row_fp8.restype = None
        L.oracle_kv_row_fp8.argtypes = [ctypes.c_int, pp, u16p, u16p, fp, ctypes.c_int64,
                                        ctypes.c_double, ctypes.c_double, u8p, u8p]
        L.oracle_kv_row.restype = None
        L.oracle_kv_row.argtypes = [ctypes.c_int, pp, u16p, u16p, fp, ctypes.c_int64, u16p, u16p]
        _lib = L
    return _lib


def _scale32(x) -> float:
    """An FP8 cache scale as the library takes it: a float32 (the C ABI's `float`), so
    that both sides divide by the same number."""
    return float(np.float32(x))


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def n_threads_default() -> int:
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ scalars
def ssmax_factor(p: int, base: float = 2048.0, expo: float = 0.1) -> float:
    return lib().oracle_ssmax_factor(int(p), base, expo)


def sigmoid(x: float) -> float:
    return lib().oracle_sigmoid(float(x))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def double_to_bf16(x: float) -> int:
    return lib().oracle_double_to_bf16(float(x))


def visible(kind: int, t: int, j: int, window: int) -> bool:
    return bool(lib().oracle_visible(kind, t, j, window))


def cache_slot(kind: int, j: int, slots: int) -> int:
    return lib().oracle_cache_slot(kind, j, slots)


# ------------------------------------------------------------------ vectors
def rms_norm(x, w, eps: float = 1e-6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    y = np.empty_like(x)
    lib().oracle_rms_norm(_ptr(x, ctypes.c_double), _ptr(w, ctypes.c_double), x.size, eps,
                          _ptr(y, ctypes.c_double))
    return y


def rope(x, t: int, theta: float = 10000.0) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().oracle_rope(_ptr(y, ctypes.c_double), y.size, int(t), theta)
    return y


def softmax(s) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    p = np.empty_like(s)
    lib().oracle_softmax(_ptr(s, ctypes.c_double), s.size, _ptr(p, ctypes.c_double))
    return p


def prepare_query(kind, P: Params, q_bits, w, t) -> np.ndarray:
    q_bits, w = _u16(q_bits), _f32(w)
    out = np.empty(P.head_dim, dtype=np.float64)
    lib().oracle_prepare_query(kind, ctypes.byref(P), _ptr(q_bits, ctypes.c_uint16),
                               _ptr(w, ctypes.c_float), int(t), _ptr(out, ctypes.c_double))
    return out


def prepare_key(kind, P: Params, k_bits, w, j) -> np.ndarray:
    k_bits, w = _u16(k_bits), _f32(w)
    out = np.empty(P.head_dim, dtype=np.float64)
    lib().oracle_prepare_key(kind, ctypes.byref(P), _ptr(k_bits, ctypes.c_uint16),
                             _ptr(w, ctypes.c_float), int(j), _ptr(out, ctypes.c_double))
    return out


# ------------------------------------------------------------------ attention
def prefill_rows(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, rows_b, rows_t,
                 n_threads: int | None = None) -> np.ndarray:
    """Gated attention output for the listed (b, t) rows: [n_rows, Hq, d] float64.

    q, gate: [B, T, Hq*d] bf16 bits; k, v: [B, T, Hkv*d] bf16 bits.
    """
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    B, T = q.shape[0], q.shape[1]
    rows_b = np.ascontiguousarray(rows_b, dtype=np.int64)
    rows_t = np.ascontiguousarray(rows_t, dtype=np.int64)
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((rows_b.size, P.n_q_heads, P.head_dim), dtype=np.float64)
    rc = lib().oracle_prefill_rows(
        kind, ctypes.byref(P), B, T, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), rows_b.size,
        _ptr(rows_b, ctypes.c_int64), _ptr(rows_t, ctypes.c_int64), _ptr(out, ctypes.c_double),
        n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_prefill_rows rejected its arguments")
    return out


def prefill_row_heads(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, rows_b,
                      rows_t, rows_h, n_threads: int | None = None) -> np.ndarray:
    """Gated attention output of single query heads: item r is head rows_h[r] of row
    (rows_b[r], rows_t[r]); [n_items, d] float64.  Same arithmetic as prefill_rows."""
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    B, T = q.shape[0], q.shape[1]
    rows_b = np.ascontiguousarray(rows_b, dtype=np.int64)
    rows_t = np.ascontiguousarray(rows_t, dtype=np.int64)
    rows_h = np.ascontiguousarray(rows_h, dtype=np.int64)
    assert rows_b.size == rows_t.size == rows_h.size
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((rows_b.size, P.head_dim), dtype=np.float64)
    rc = lib().oracle_prefill_row_heads(
        kind, ctypes.byref(P), B, T, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), rows_b.size,
        _ptr(rows_b, ctypes.c_int64), _ptr(rows_t, ctypes.c_int64), _ptr(rows_h, ctypes.c_int64),
        _ptr(out, ctypes.c_double), n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_prefill_row_heads rejected its arguments")
    return out


def prefill(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias,
            n_threads: int | None = None) -> np.ndarray:
    """All rows: [B, T, Hq, d] float64."""
    B, T = q.shape[0], q.shape[1]
    bb, tt = np.meshgrid(np.arange(B), np.arange(T), indexing="ij")
    out = prefill_rows(kind, P, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, bb.ravel(),
                       tt.ravel(), n_threads)
    return out.reshape(B, T, P.n_q_heads, P.head_dim)


def decode(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache, v_cache,
           n_threads: int | None = None) -> np.ndarray:
    """One decode step: [B, Hq, d] float64.  Caches are [B, Hkv, slots, d] bf16 bits."""
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    B = q.shape[0]
    slots = k_cache.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((B, P.n_q_heads, P.head_dim), dtype=np.float64)
    rc = lib().oracle_decode(
        kind, ctypes.byref(P), B, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), _ptr(pos, ctypes.c_int64),
        _ptr(k_cache, ctypes.c_uint16), _ptr(v_cache, ctypes.c_uint16), slots,
        _ptr(out, ctypes.c_double), n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return out


def prefill_chunk_rows(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                       k_cache, v_cache, rows_b, rows_i, n_threads: int | None = None) -> np.ndarray:
    """Chunked prefill against an existing cache, for the listed (b, new token i) rows:
    [n_rows, Hq, d] float64.  q, gate: [B, T, Hq*d]; k, v: [B, T, Hkv*d] (bf16 bits);
    pos0: [B] positions of each sequence's first new token; caches [B, Hkv, slots, d]
    bf16 bits as they were before the call."""
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    B, T = q.shape[0], q.shape[1]
    slots = k_cache.shape[2]
    pos0 = np.ascontiguousarray(pos0, dtype=np.int64)
    rows_b = np.ascontiguousarray(rows_b, dtype=np.int64)
    rows_i = np.ascontiguousarray(rows_i, dtype=np.int64)
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((rows_b.size, P.n_q_heads, P.head_dim), dtype=np.float64)
    i64 = ctypes.c_int64
    rc = lib().oracle_prefill_chunk_rows(
        kind, ctypes.byref(P), B, T, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), _ptr(pos0, i64),
        _ptr(k_cache, ctypes.c_uint16), _ptr(v_cache, ctypes.c_uint16), slots, rows_b.size,
        _ptr(rows_b, i64), _ptr(rows_i, i64), _ptr(out, ctypes.c_double),
        n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_prefill_chunk_rows rejected its arguments")
    return out


def prefill_chunk(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0, k_cache,
                  v_cache, n_threads: int | None = None) -> np.ndarray:
    """All rows of a chunk: [B, T, Hq, d] float64."""
    B, T = q.shape[0], q.shape[1]
    bb, ii = np.meshgrid(np.arange(B), np.arange(T), indexing="ij")
    out = prefill_chunk_rows(kind, P, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                             k_cache, v_cache, bb.ravel(), ii.ravel(), n_threads)
    return out.reshape(B, T, P.n_q_heads, P.head_dim)


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code))


def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def decode_fp8(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_codes,
               v_codes, k_scale: float, v_scale: float, n_threads: int | None = None) -> np.ndarray:
    """One decode step over FP8 E4M3 caches ([B, Hkv, slots, d] uint8 codes, one scale per
    cache tensor): [B, Hq, d] float64."""
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    k_codes = np.ascontiguousarray(k_codes, dtype=np.uint8)
    v_codes = np.ascontiguousarray(v_codes, dtype=np.uint8)
    B = q.shape[0]
    slots = k_codes.shape[2]
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((B, P.n_q_heads, P.head_dim), dtype=np.float64)
    u8 = ctypes.c_uint8
    rc = lib().oracle_decode_fp8(
        kind, ctypes.byref(P), B, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), _ptr(pos, ctypes.c_int64),
        _ptr(k_codes, u8), _ptr(v_codes, u8), slots, _scale32(k_scale), _scale32(v_scale),
        _ptr(out, ctypes.c_double), n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_decode_fp8 rejected its arguments")
    return out


def prefill_chunk_rows_fp8(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                           k_codes, v_codes, k_scale: float, v_scale: float, rows_b, rows_i,
                           n_threads: int | None = None) -> np.ndarray:
    """Chunked prefill over FP8 E4M3 caches (uint8 codes [B, Hkv, slots, d] as they were
    before the call, one scale per tensor) for the listed (b, new token i) rows:
    [n_rows, Hq, d] float64.  The chunk's own keys and values are quantised first."""
    q, k, v, gate = _u16(q), _u16(k), _u16(v), _u16(gate)
    k_codes = np.ascontiguousarray(k_codes, dtype=np.uint8)
    v_codes = np.ascontiguousarray(v_codes, dtype=np.uint8)
    B, T = q.shape[0], q.shape[1]
    slots = k_codes.shape[2]
    pos0 = np.ascontiguousarray(pos0, dtype=np.int64)
    rows_b = np.ascontiguousarray(rows_b, dtype=np.int64)
    rows_i = np.ascontiguousarray(rows_i, dtype=np.int64)
    qw, kw, bias = _f32(q_norm_w), _f32(k_norm_w), _f32(gate_bias)
    out = np.empty((rows_b.size, P.n_q_heads, P.head_dim), dtype=np.float64)
    i64 = ctypes.c_int64
    rc = lib().oracle_prefill_chunk_rows_fp8(
        kind, ctypes.byref(P), B, T, _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
        _ptr(v, ctypes.c_uint16), _ptr(gate, ctypes.c_uint16), _ptr(qw, ctypes.c_float),
        _ptr(kw, ctypes.c_float), _ptr(bias, ctypes.c_float), _ptr(pos0, i64),
        _ptr(k_codes, ctypes.c_uint8), _ptr(v_codes, ctypes.c_uint8), slots, _scale32(k_scale),
        _scale32(v_scale), rows_b.size, _ptr(rows_b, i64), _ptr(rows_i, i64),
        _ptr(out, ctypes.c_double), n_threads or n_threads_default())
    if rc != 0:
        raise ValueError("oracle_prefill_chunk_rows_fp8 rejected its arguments")
    return out


def prefill_chunk_fp8(kind, P: Params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                      k_codes, v_codes, k_scale: float, v_scale: float,
                      n_threads: int | None = None) -> np.ndarray:
    """All rows of a chunk over FP8 caches: [B, T, Hq, d] float64."""
    B, T = q.shape[0], q.shape[1]
    bb, ii = np.meshgrid(np.arange(B), np.arange(T), indexing="ij")
    out = prefill_chunk_rows_fp8(kind, P, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                                 k_codes, v_codes, k_scale, v_scale, bb.ravel(), ii.ravel(),
                                 n_threads)
    return out.reshape(B, T, P.n_q_heads, P.head_dim)


def kv_row_fp8(kind, P: Params, k_token, v_token, k_norm_w, j, k_scale: float, v_scale: float):
    """Expected FP8 cache codes for one token at position j: (k_codes, v_codes), [Hkv, d]."""
    k_token, v_token, kw = _u16(k_token), _u16(v_token), _f32(k_norm_w)
    kr = np.empty((P.n_kv_heads, P.head_dim), dtype=np.uint8)
    vr = np.empty_like(kr)
    u8 = ctypes.c_uint8
    lib().oracle_kv_row_fp8(kind, ctypes.byref(P), _ptr(k_token, ctypes.c_uint16),
                            _ptr(v_token, ctypes.c_uint16), _ptr(kw, ctypes.c_float), int(j),
                            _scale32(k_scale), _scale32(v_scale), _ptr(kr, u8), _ptr(vr, u8))
    return kr, vr


def kv_row(kind, P: Params, k_token, v_token, k_norm_w, j):
    """Expected cache rows for one token at position j: (k_row, v_row), [Hkv, d] bf16 bits."""
    k_token, v_token, kw = _u16(k_token), _u16(v_token), _f32(k_norm_w)
    kr = np.empty((P.n_kv_heads, P.head_dim), dtype=np.uint16)
    vr = np.empty_like(kr)
    lib().oracle_kv_row(kind, ctypes.byref(P), _ptr(k_token, ctypes.c_uint16),
                        _ptr(v_token, ctypes.c_uint16), _ptr(kw, ctypes.c_float), int(j),
                        _ptr(kr, ctypes.c_uint16), _ptr(vr, ctypes.c_uint16))
    return kr, vr
