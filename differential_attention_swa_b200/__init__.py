"""B200 (sm_100a) masked attention: sliding window, local + strided,
differential, and a rolling-window decode step.

A thin ctypes binding over ``libswa_attn.so`` (the C ABI in
``include/swa_attn.h``). Every step of the computation runs in the library's
CUDA kernels; this module only checks tensor properties, allocates outputs
with PyTorch and passes raw pointers, sizes and the current CUDA stream.
There is no CPU fallback: without the built library or a CUDA device the
calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswa_attn.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libswa_attn_debug.so")  # bounds-checking build (tests)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_TOO_SMALL, ERR_BOUNDS = range(7)
MASK_WINDOW, MASK_STRIDED, MASK_CAUSAL, MASK_GLOBAL = 0, 1, 2, 3
STRIDE_TAG = 0x40000000
TILE = 128  # query rows and keys per tile in the prefill kernels

__all__ = [
    "swa_attn_fwd", "strided_attn_fwd", "global_attn_fwd", "dilated_attn_fwd", "swa_attn_bwd", "diff_attn_fwd", "swa_decode_step", "decode_workspace_bytes",
    "swa_sink_decode_step", "sink_decode_workspace_bytes", "swa_diff_decode_step", "diff_decode_workspace_bytes",
    "prefill_debug", "schedule", "count_nonmasked", "last_device_error", "SwaError", "library",
]


class SwaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {library().swa_status_string(status).decode()} (status {status})")


class _Debug(ctypes.Structure):
    _fields_ = [("cells", ctypes.c_void_p), ("tiles", ctypes.c_void_p), ("ntiles", ctypes.c_void_p),
                ("tiles_cap", ctypes.c_int32), ("inject_timeout", ctypes.c_int32)]


_lib = None


def library() -> ctypes.CDLL:
    """Loads libswa_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = load(LIB_PATH)
    return _lib


def use_library(lib: ctypes.CDLL | None) -> ctypes.CDLL | None:
    """Routes every call of this module to `lib` (for instance the
    bounds-checking build from load(DEBUG_LIB_PATH)); None restores the
    release library. Returns the previous one."""
    global _lib
    prev, _lib = _lib, lib
    return prev


def load(path: str) -> ctypes.CDLL:
    """Opens a build of the library and declares its entry points."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with differential_attention_swa_b200/build.py")
    lib = ctypes.CDLL(path)
    P, I, F, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
    lib.swa_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.strided_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.global_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.global_attn_fwd.restype = I
    lib.dilated_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.dilated_attn_fwd.restype = I
    lib.swa_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, SZ, P]
    lib.swa_attn_bwd.restype = I
    lib.swa_attn_bwd_workspace_bytes.argtypes = [I, I, I]
    lib.swa_attn_bwd_workspace_bytes.restype = SZ
    lib.strided_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, SZ, P]
    lib.strided_attn_bwd.restype = I
    lib.strided_attn_bwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.strided_attn_bwd_workspace_bytes.restype = SZ
    lib.diff_attn_fwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]
    lib.swa_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P, SZ, P]
    lib.swa_decode_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.swa_decode_workspace_bytes.restype = SZ
    lib.swa_sink_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, SZ, P]
    lib.swa_sink_decode_step.restype = I
    lib.swa_sink_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.swa_sink_decode_workspace_bytes.restype = SZ
    lib.swa_diff_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, SZ, P]
    lib.swa_diff_decode_step.restype = I
    lib.swa_diff_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.swa_diff_decode_workspace_bytes.restype = SZ
    lib.swa_prefill_debug.argtypes = [I, P, P, P, P, P, I, I, I, I, I, I, I, F, ctypes.POINTER(_Debug), P]
    lib.swa_schedule.argtypes = [I, I, I, I, I, I, P, P, I64]
    lib.swa_schedule.restype = I64
    lib.swa_count_nonmasked.argtypes = [I, I, I, I]
    lib.swa_count_nonmasked.restype = I64
    lib.swa_debug_exp2.argtypes = [P, P, I64, P]
    lib.swa_debug_exp2.restype = I
    lib.swa_last_device_error.argtypes = [P]
    lib.swa_status_string.argtypes = [I]
    lib.swa_status_string.restype = ctypes.c_char_p
    for name in ("swa_attn_fwd", "strided_attn_fwd", "diff_attn_fwd", "swa_decode_step", "swa_prefill_debug",
                 "swa_last_device_error"):
        getattr(lib, name).restype = I
    return lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype=torch.bfloat16, dim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")


def _raise(status: int, what: str):
    if status != OK:
        raise SwaError(status, what)


def _prefill_common(q, k, v, out, want_lse):
    _check(q, "q", dim=4)
    _check(k, "k", dim=4)
    _check(v, "v", dim=4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape[:3] != (B, Hkv, N):
        raise ValueError("k/v shapes must be [B, Hkv, N, d]")
    if out is None:
        out = torch.empty((B, Hq, N, v.shape[3]), dtype=torch.bfloat16, device=q.device)
    else:
        _check(out, "out", dim=4)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if want_lse else None
    return B, Hq, Hkv, N, d, out, lse


def swa_attn_fwd(q, k, v, window: int, scale: float | None = None, out=None, return_lse: bool = False,
                 stream=None):
    """Sliding-window attention: row i attends keys max(0, i-W+1) .. i."""
    B, Hq, Hkv, N, d, out, lse = _prefill_common(q, k, v, out, return_lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().swa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d, int(window),
                                float(scale), _stream(stream))
    _raise(st, "swa_attn_fwd")
    return (out, lse) if return_lse else out


def strided_attn_fwd(q, k, v, window: int, stride: int, scale: float | None = None, out=None,
                     return_lse: bool = False, stream=None):
    """Local + strided attention: the window OR keys j % stride == 0, j <= i."""
    B, Hq, Hkv, N, d, out, lse = _prefill_common(q, k, v, out, return_lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().strided_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                    int(window), int(stride), float(scale), _stream(stream))
    _raise(st, "strided_attn_fwd")
    return (out, lse) if return_lse else out


def global_attn_fwd(q, k, v, window: int, n_global: int, scale: float | None = None, out=None,
                    return_lse: bool = False, stream=None):
    """Window + global tokens: the window OR keys j < n_global (positions
    0 .. n_global-1 are the global tokens), j <= i."""
    B, Hq, Hkv, N, d, out, lse = _prefill_common(q, k, v, out, return_lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().global_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                   int(window), int(n_global), float(scale), _stream(stream))
    _raise(st, "global_attn_fwd")
    return (out, lse) if return_lse else out


def dilated_attn_fwd(q, k, v, window: int, dilation: int, scale: float | None = None, out=None,
                     return_lse: bool = False, stream=None):
    """Dilated window: row i attends keys i, i - dilation, ..., i - (window-1)*dilation."""
    B, Hq, Hkv, N, d, out, lse = _prefill_common(q, k, v, out, return_lse)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().dilated_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                                    int(window), int(dilation), float(scale), _stream(stream))
    _raise(st, "dilated_attn_fwd")
    return (out, lse) if return_lse else out


def attn_bwd_workspace_bytes(B: int, Hq: int, N: int) -> int:
    return int(library().swa_attn_bwd_workspace_bytes(B, Hq, N))


def swa_attn_bwd(q, k, v, o, d_o, lse, window: int, scale: float | None = None, workspace=None, stream=None,
                 stride: int = 0):
    """Gradients (dq, dk, dv) of the window attention forward, given its
    inputs, output o, log-sum-exp lse (swa_attn_fwd(..., return_lse=True))
    and the output's gradient d_o. With stride >= 1: the backward of the
    local + strided forward (strided_attn_fwd)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (d_o, "d_o")):
        _check(t, n, dim=4)
    _check(lse, "lse", dtype=torch.float32, dim=3)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if o.shape != q.shape or d_o.shape != q.shape or k.shape != (B, Hkv, N, d) or v.shape != k.shape \
            or lse.shape != (B, Hq, N):
        raise ValueError("backward shapes do not agree")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if stride:
        need = int(library().strided_attn_bwd_workspace_bytes(B, Hq, Hkv, N, d, int(stride)))
    else:
        need = attn_bwd_workspace_bytes(B, Hq, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    common = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv,
              N, d, int(window))
    tail = (float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if stride:
        st = library().strided_attn_bwd(*common, int(stride), *tail)
        _raise(st, "strided_attn_bwd")
    else:
        st = library().swa_attn_bwd(*common, *tail)
        _raise(st, "swa_attn_bwd")
    return dq, dk, dv


def diff_attn_fwd(q1, k1, q2, k2, v, lam, window: int | None = None, scale: float | None = None, out=None,
                  stream=None):
    """Differential attention: softmax(Q1K1^T)V - lam[h] softmax(Q2K2^T)V."""
    for t, n in ((q1, "q1"), (k1, "k1"), (q2, "q2"), (k2, "k2"), (v, "v")):
        _check(t, n, dim=4)
    _check(lam, "lam", dtype=torch.float32, dim=1)
    B, Hq, N, dqk = q1.shape
    Hkv = k1.shape[1]
    dv = v.shape[3]
    if q2.shape != q1.shape or k1.shape != (B, Hkv, N, dqk) or k2.shape != k1.shape or v.shape[:3] != (B, Hkv, N):
        raise ValueError("differential attention shapes do not agree")
    if lam.numel() != Hq:
        raise ValueError("lam must hold one value per query head")
    if out is None:
        out = torch.empty((B, Hq, N, dv), dtype=torch.bfloat16, device=q1.device)
    window = N if window is None else window
    scale = 1.0 / math.sqrt(dqk) if scale is None else scale
    st = library().diff_attn_fwd(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(v), _ptr(out), _ptr(lam), B, Hq, Hkv,
                                 N, dqk, dv, int(window), float(scale), _stream(stream))
    _raise(st, "diff_attn_fwd")
    return out


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, W: int) -> int:
    return int(library().swa_decode_workspace_bytes(B, Hq, Hkv, d, W))


def swa_decode_step(q, k_new, v_new, k_cache, v_cache, pos, out=None, workspace=None, scale: float | None = None,
                    stream=None):
    """One decode step: stores k_new/v_new into slot pos % W of each
    sequence's cache, then attends over the last W positions."""
    _check(q, "q", dim=3)
    _check(k_new, "k_new", dim=3)
    _check(v_new, "v_new", dim=3)
    _check(k_cache, "k_cache", dim=4)
    _check(v_cache, "v_cache", dim=4)
    _check(pos, "pos", dtype=torch.int32, dim=1)
    B, Hq, d = q.shape
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(B, Hq, Hkv, d, W)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().swa_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(pos),
                                   _ptr(out), B, Hq, Hkv, d, W, float(scale), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "swa_decode_step")
    return out


def sink_decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, n_sink: int, W: int) -> int:
    return int(library().swa_sink_decode_workspace_bytes(B, Hq, Hkv, d, n_sink, W))


def swa_sink_decode_step(q, k_new, v_new, k_cache, v_cache, pos, n_sink: int, out=None, workspace=None,
                         scale: float | None = None, stream=None):
    """One decode step with attention sinks: the cache holds n_sink sink
    slots (positions 0 .. n_sink-1, kept for good) then W rolling slots."""
    _check(q, "q", dim=3)
    _check(k_new, "k_new", dim=3)
    _check(v_new, "v_new", dim=3)
    _check(k_cache, "k_cache", dim=4)
    _check(v_cache, "v_cache", dim=4)
    _check(pos, "pos", dtype=torch.int32, dim=1)
    B, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    W = k_cache.shape[2] - int(n_sink)
    if W < 1:
        raise ValueError("the cache needs at least one window slot after the sinks")
    if out is None:
        out = torch.empty_like(q)
    need = sink_decode_workspace_bytes(B, Hq, Hkv, d, n_sink, W)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().swa_sink_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(pos), _ptr(out), B, Hq, Hkv, d, int(n_sink), W, float(scale),
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream))
    _raise(st, "swa_sink_decode_step")
    return out


def diff_decode_workspace_bytes(B: int, Hq: int, Hkv: int, d_qk: int, d_v: int, W: int) -> int:
    return int(library().swa_diff_decode_workspace_bytes(B, Hq, Hkv, d_qk, d_v, W))


def swa_diff_decode_step(q1, q2, k1_new, k2_new, v_new, k1_cache, k2_cache, v_cache, pos, lam, out=None,
                         workspace=None, scale: float | None = None, stream=None):
    """One differential decode step: two maps over the same rolling window,
    V cache shared. q1, q2 [B,Hq,64]; k*_new [B,Hkv,64]; v_new [B,Hkv,128];
    k*_cache [B,Hkv,W,64]; v_cache [B,Hkv,W,128]; lam fp32 [Hq]."""
    for t, n in ((q1, "q1"), (q2, "q2"), (k1_new, "k1_new"), (k2_new, "k2_new"), (v_new, "v_new")):
        _check(t, n, dim=3)
    for t, n in ((k1_cache, "k1_cache"), (k2_cache, "k2_cache"), (v_cache, "v_cache")):
        _check(t, n, dim=4)
    _check(pos, "pos", dtype=torch.int32, dim=1)
    _check(lam, "lambda", dtype=torch.float32, dim=1)
    B, Hq, dqk = q1.shape
    Hkv, W, dv = v_cache.shape[1], v_cache.shape[2], v_cache.shape[3]
    if out is None:
        out = torch.empty((B, Hq, dv), dtype=q1.dtype, device=q1.device)
    need = diff_decode_workspace_bytes(B, Hq, Hkv, dqk, dv, W)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q1.device)
    scale = 1.0 / math.sqrt(dqk) if scale is None else scale
    st = library().swa_diff_decode_step(_ptr(q1), _ptr(q2), _ptr(k1_new), _ptr(k2_new), _ptr(v_new), _ptr(k1_cache),
                                        _ptr(k2_cache), _ptr(v_cache), _ptr(pos), _ptr(lam), _ptr(out), B, Hq, Hkv,
                                        dqk, dv, W, float(scale), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "swa_diff_decode_step")
    return out


def prefill_debug(kind: int, q, k, v, window: int, stride: int = 0, scale: float | None = None,
                  tiles_cap: int = 64, inject_timeout: bool = False, stream=None):
    """Prefill that also reports, per (b, hq, query tile), the attended
    cells it processed and the key tiles it visited. Returns
    (out, cells [B,Hq,nq] int64, tiles [B,Hq,nq,cap] int32, ntiles [B,Hq,nq])."""
    B, Hq, Hkv, N, d, out, _ = _prefill_common(q, k, v, None, False)
    nq = (N + TILE - 1) // TILE
    cells = torch.zeros((B, Hq, nq), dtype=torch.int64, device=q.device)
    tiles = torch.full((B, Hq, nq, tiles_cap), -1, dtype=torch.int32, device=q.device)
    ntiles = torch.zeros((B, Hq, nq), dtype=torch.int32, device=q.device)
    dbg = _Debug(cells.data_ptr(), tiles.data_ptr(), ntiles.data_ptr(), tiles_cap, 1 if inject_timeout else 0)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    st = library().swa_prefill_debug(int(kind), _ptr(q), _ptr(k), _ptr(v), _ptr(out), None, B, Hq, Hkv, N, d,
                                     int(window), int(stride), float(scale), ctypes.byref(dbg), _stream(stream))
    _raise(st, "swa_prefill_debug")
    return out, cells, tiles, ntiles


def debug_exp2(x, out=None, stream=None):
    """2^x through the prefill kernels' FMA-pipe exponential (a debug entry:
    the differential kernel evaluates part of its exponentials this way)."""
    _check(x, "x", dtype=torch.float32)
    out = torch.empty_like(x) if out is None else out
    _check(out, "out", dtype=torch.float32)
    st = library().swa_debug_exp2(_ptr(x), _ptr(out), x.numel(), _stream(stream))
    _raise(st, "swa_debug_exp2")
    return out


def schedule(kind: int, N: int, W: int, stride: int = 0, Bq: int = TILE, Bk: int = TILE):
    """Per query tile, the key tiles the kernels visit (host computation)."""
    lib = library()
    n = lib.swa_schedule(kind, N, W, stride, Bq, Bk, None, None, 0)
    if n < 0:
        raise ValueError("bad schedule arguments")
    nq = (N + Bq - 1) // Bq
    offs = (ctypes.c_int32 * (nq + 1))()
    tiles = (ctypes.c_int32 * max(int(n), 1))()
    lib.swa_schedule(kind, N, W, stride, Bq, Bk, offs, tiles, n)
    return [list(tiles[offs[i]:offs[i + 1]]) for i in range(nq)]


def count_nonmasked(kind: int, N: int, W: int, stride: int = 0) -> int:
    n = library().swa_count_nonmasked(kind, N, W, stride)
    if n < 0:
        raise ValueError("bad arguments")
    return int(n)


def last_device_error(stream=None) -> int:
    """Synchronises the stream, then returns and clears the device error flag."""
    return int(library().swa_last_device_error(_stream(stream)))
