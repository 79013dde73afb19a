"""Beam 1.0 attention core on B200: thin Python binding of libbeam_attn.so.

The binding only marshals arguments: torch tensors become device pointers, the
current torch stream becomes the CUDA stream.  Every step of the path runs in
the library's CUDA kernels; there is no Python or CPU fallback, and loading fails
loudly when the library has not been built (``python -m global_nope_gqa_b200.build``
or ``__graft_entry__.build()``).

Function names follow the C ABI in ``include/beam_attn.h``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbeam_attn.so")

LOCAL, GLOBAL = 0, 1

STATUS = {
    0: "BEAM_OK", -1: "BEAM_ERR_INVALID_ARG", -2: "BEAM_ERR_UNSUPPORTED", -3: "BEAM_ERR_CUDA",
    -4: "BEAM_ERR_DEVICE_TIMEOUT", -5: "BEAM_ERR_CAPACITY", -6: "BEAM_ERR_WORKSPACE",
    -7: "BEAM_ERR_ALIGNMENT", -8: "BEAM_ERR_SCRATCH_LIMIT",
}

EXPORTS = (
    "beam_default_params", "beam_kv_layout", "beam_prefill_workspace_bytes", "beam_attn_prefill",
    "beam_kv_append", "beam_decode_workspace_bytes", "beam_attn_decode", "beam_status_string",
    "beam_attn_decode_noalloc", "beam_prefill_chunk_workspace_bytes", "beam_attn_prefill_chunk",
    "beam_kv_layout_fp8", "beam_kv_append_fp8", "beam_attn_decode_fp8",
    "beam_prefill_chunk_fp8_workspace_bytes", "beam_attn_prefill_chunk_fp8",
)


class BeamError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")


class Params(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
        ("ssmax_base", ctypes.c_float), ("ssmax_exp", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
    ]


class KVLayout(ctypes.Structure):
    _fields_ = [
        ("slots_per_seq", ctypes.c_int64), ("stride_seq", ctypes.c_int64),
        ("stride_head", ctypes.c_int64), ("stride_slot", ctypes.c_int64),
        ("bytes_k", ctypes.c_int64), ("bytes_v", ctypes.c_int64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbeam_attn.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m global_nope_gqa_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        pp, lp = ctypes.POINTER(Params), ctypes.POINTER(KVLayout)
        L.beam_default_params.restype = None
        L.beam_default_params.argtypes = [pp]
        L.beam_kv_layout.restype = ctypes.c_int
        L.beam_kv_layout.argtypes = [ctypes.c_int, pp, i32, i64, lp]
        L.beam_prefill_workspace_bytes.restype = sz
        L.beam_prefill_workspace_bytes.argtypes = [pp, i32, i32]
        L.beam_attn_prefill.restype = ctypes.c_int
        L.beam_attn_prefill.argtypes = [ctypes.c_int, pp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                        vp, vp, lp, vp, sz, vp, vp]
        L.beam_prefill_chunk_workspace_bytes.restype = sz
        L.beam_prefill_chunk_workspace_bytes.argtypes = [ctypes.c_int, pp, i32, i32, lp]
        L.beam_attn_prefill_chunk.restype = ctypes.c_int
        L.beam_attn_prefill_chunk.argtypes = [ctypes.c_int, pp, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                              vp, vp, vp, vp, lp, vp, sz, vp, vp]
        L.beam_prefill_chunk_fp8_workspace_bytes.restype = sz
        L.beam_prefill_chunk_fp8_workspace_bytes.argtypes = [ctypes.c_int, pp, i32, i32, lp]
        L.beam_attn_prefill_chunk_fp8.restype = ctypes.c_int
        L.beam_attn_prefill_chunk_fp8.argtypes = [ctypes.c_int, pp, i32, i32, vp, vp, vp, vp, vp,
                                                  vp, vp, vp, vp, vp, vp, lp, ctypes.c_float,
                                                  ctypes.c_float, vp, sz, vp, vp]
        L.beam_kv_append.restype = ctypes.c_int
        L.beam_kv_append.argtypes = [ctypes.c_int, pp, i32, i32, vp, vp, vp, vp, vp, vp, lp, vp, vp]
        L.beam_decode_workspace_bytes.restype = sz
        L.beam_decode_workspace_bytes.argtypes = [ctypes.c_int, pp, i32, lp]
        L.beam_attn_decode.restype = ctypes.c_int
        L.beam_attn_decode.argtypes = [ctypes.c_int, pp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                       vp, lp, vp, vp, sz, vp, vp]
        L.beam_attn_decode_noalloc.restype = ctypes.c_int
        L.beam_attn_decode_noalloc.argtypes = [ctypes.c_int, pp, i32, vp, vp, vp, vp, vp, vp, vp,
                                               vp, vp, vp, lp, vp, vp, vp]
        f32 = ctypes.c_float
        L.beam_kv_layout_fp8.restype = ctypes.c_int
        L.beam_kv_layout_fp8.argtypes = [ctypes.c_int, pp, i32, i64, lp]
        L.beam_kv_append_fp8.restype = ctypes.c_int
        L.beam_kv_append_fp8.argtypes = [ctypes.c_int, pp, i32, i32, vp, vp, vp, vp, vp, vp, lp,
                                         f32, f32, vp, vp]
        L.beam_attn_decode_fp8.restype = ctypes.c_int
        L.beam_attn_decode_fp8.argtypes = [ctypes.c_int, pp, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                           vp, vp, lp, f32, f32, vp, vp, sz, vp, vp]
        L.beam_status_string.restype = ctypes.c_char_p
        L.beam_status_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def default_params(**over) -> Params:
    p = Params()
    lib().beam_default_params(ctypes.byref(p))
    for k, v in over.items():
        setattr(p, k, v)
    return p


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, rc: int):
    if rc != 0:
        raise BeamError(fn, rc)


def beam_kv_layout(kind: int, params: Params, batch: int, capacity_tokens: int) -> KVLayout:
    out = KVLayout()
    _check("beam_kv_layout",
           lib().beam_kv_layout(kind, ctypes.byref(params), batch, capacity_tokens, ctypes.byref(out)))
    return out


def beam_prefill_workspace_bytes(params: Params, B: int, T: int) -> int:
    return lib().beam_prefill_workspace_bytes(ctypes.byref(params), B, T)


def beam_decode_workspace_bytes(kind: int, params: Params, B: int, layout: KVLayout) -> int:
    return lib().beam_decode_workspace_bytes(kind, ctypes.byref(params), B, ctypes.byref(layout))


def _workspace(nbytes: int, device):
    import torch
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def beam_attn_prefill(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, out,
                      k_cache=None, v_cache=None, layout: KVLayout | None = None, workspace=None,
                      dev_status=None, stream=None, B: int | None = None, T: int | None = None):
    """q, gate: [B, T, 6144] bf16; k, v: [B, T, 1024] bf16; out: [B, T, 6144] bf16."""
    B = q.shape[0] if B is None else B
    T = q.shape[1] if T is None else T
    need = beam_prefill_workspace_bytes(params, B, T)
    if workspace is None:
        workspace = _workspace(need, q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().beam_attn_prefill(
        kind, ctypes.byref(params), B, T, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(out), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout) if layout is not None else None, _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream))
    _check("beam_attn_prefill", rc)
    return out


def beam_prefill_chunk_workspace_bytes(kind: int, params: Params, B: int, T: int,
                                       layout: KVLayout | None = None) -> int:
    return lib().beam_prefill_chunk_workspace_bytes(
        kind, ctypes.byref(params), B, T, ctypes.byref(layout) if layout is not None else None)


def beam_attn_prefill_chunk(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0, out,
                            k_cache, v_cache, layout: KVLayout, workspace=None, dev_status=None,
                            stream=None):
    """Chunked prefill: q, gate [B, T, 6144]; k, v [B, T, 1024] bf16; pos0 [B] int64 on the
    device (position of each sequence's first new token); caches as for decode."""
    B, T = q.shape[0], q.shape[1]
    need = beam_prefill_chunk_workspace_bytes(kind, params, B, T, layout)
    if workspace is None and need:
        workspace = _workspace(need, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().beam_attn_prefill_chunk(
        kind, ctypes.byref(params), B, T, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(pos0), _ptr(out), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check("beam_attn_prefill_chunk", rc)
    return out


def beam_prefill_chunk_fp8_workspace_bytes(kind: int, params: Params, B: int, T: int,
                                           layout: KVLayout) -> int:
    return lib().beam_prefill_chunk_fp8_workspace_bytes(kind, ctypes.byref(params), B, T,
                                                        ctypes.byref(layout))


def beam_attn_prefill_chunk_fp8(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos0,
                                out, k_cache, v_cache, layout: KVLayout, k_scale: float,
                                v_scale: float, workspace=None, dev_status=None, stream=None):
    """Chunked prefill over FP8 E4M3 caches (uint8 code arrays, FP8 layout, one scale per
    cache tensor); otherwise as beam_attn_prefill_chunk."""
    B, T = q.shape[0], q.shape[1]
    need = beam_prefill_chunk_fp8_workspace_bytes(kind, params, B, T, layout)
    if workspace is None and need:
        workspace = _workspace(need, q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().beam_attn_prefill_chunk_fp8(
        kind, ctypes.byref(params), B, T, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(pos0), _ptr(out), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout), float(k_scale), float(v_scale), _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream))
    _check("beam_attn_prefill_chunk_fp8", rc)
    return out


def beam_kv_append(kind, params, k, v, k_norm_w, pos0, k_cache, v_cache, layout: KVLayout,
                   dev_status=None, stream=None):
    """k, v: [B, T, 1024] bf16; pos0: [B] int64 on the device."""
    B, T = k.shape[0], k.shape[1]
    rc = lib().beam_kv_append(kind, ctypes.byref(params), B, T, _ptr(k), _ptr(v), _ptr(k_norm_w),
                              _ptr(pos0), _ptr(k_cache), _ptr(v_cache), ctypes.byref(layout),
                              _ptr(dev_status), _stream(stream))
    _check("beam_kv_append", rc)


def beam_attn_decode(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache,
                     v_cache, layout: KVLayout, out, workspace=None, dev_status=None, stream=None):
    """q, gate: [B, 6144] bf16; k, v: [B, 1024] bf16; pos: [B] int64; out: [B, 6144] bf16."""
    B = q.shape[0]
    need = beam_decode_workspace_bytes(kind, params, B, layout)
    if workspace is None:
        workspace = _workspace(need, q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().beam_attn_decode(
        kind, ctypes.byref(params), B, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(pos), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout), _ptr(out), _ptr(workspace), ws_bytes, _ptr(dev_status),
        _stream(stream))
    _check("beam_attn_decode", rc)
    return out


def beam_attn_decode_noalloc(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos,
                             k_cache, v_cache, layout: KVLayout, out, dev_status=None, stream=None):
    """Same as beam_attn_decode, for callers that cannot allocate: the scratch is the
    library's fixed 8 MiB device array (shared by all calls; overlapping calls race)."""
    B = q.shape[0]
    rc = lib().beam_attn_decode_noalloc(
        kind, ctypes.byref(params), B, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(pos), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout), _ptr(out), _ptr(dev_status), _stream(stream))
    _check("beam_attn_decode_noalloc", rc)
    return out


def beam_kv_layout_fp8(kind: int, params: Params, batch: int, capacity_tokens: int) -> KVLayout:
    """Layout of an FP8 E4M3 cache (one byte per element; same element strides)."""
    out = KVLayout()
    _check("beam_kv_layout_fp8", lib().beam_kv_layout_fp8(kind, ctypes.byref(params), batch,
                                                          capacity_tokens, ctypes.byref(out)))
    return out


def beam_kv_append_fp8(kind, params, k, v, k_norm_w, pos0, k_cache, v_cache, layout: KVLayout,
                       k_scale: float, v_scale: float, dev_status=None, stream=None):
    """k, v: [B, T, 1024] bf16; caches: uint8 code arrays of the FP8 layout."""
    B, T = k.shape[0], k.shape[1]
    rc = lib().beam_kv_append_fp8(kind, ctypes.byref(params), B, T, _ptr(k), _ptr(v),
                                  _ptr(k_norm_w), _ptr(pos0), _ptr(k_cache), _ptr(v_cache),
                                  ctypes.byref(layout), float(k_scale), float(v_scale),
                                  _ptr(dev_status), _stream(stream))
    _check("beam_kv_append_fp8", rc)


def beam_attn_decode_fp8(kind, params, q, k, v, gate, q_norm_w, k_norm_w, gate_bias, pos, k_cache,
                         v_cache, layout: KVLayout, k_scale: float, v_scale: float, out,
                         workspace=None, dev_status=None, stream=None):
    """Decode over FP8 E4M3 caches (uint8 code arrays); otherwise as beam_attn_decode."""
    B = q.shape[0]
    need = beam_decode_workspace_bytes(kind, params, B, layout)
    if workspace is None:
        workspace = _workspace(need, q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().beam_attn_decode_fp8(
        kind, ctypes.byref(params), B, _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(q_norm_w),
        _ptr(k_norm_w), _ptr(gate_bias), _ptr(pos), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(layout), float(k_scale), float(v_scale), _ptr(out), _ptr(workspace),
        ws_bytes, _ptr(dev_status), _stream(stream))
    _check("beam_attn_decode_fp8", rc)
    return out


def beam_status_string(status: int) -> str:
    return lib().beam_status_string(status).decode()
