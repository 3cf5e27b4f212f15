"""Plain fp64 CPU oracle for masked causal attention.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers. The CUDA library never imports, links or
runs anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one thread
per block of rows); this module only marshals numpy arrays into it and adds
the pages' small closed-form helpers. Sources, by page title:

* "Attention Variants Compared" (cheatsheet): swa_mask, strided_mask,
  count_nonmasked, kv_cache_bytes(N, n_layers, n_heads_kv, d_head, dtype=2),
  tiled_softmax_dot, count_nsa(N, l, k, W); FAQ "NSA keys at 1024 tokens".
* "Learn: Sparse & Sliding-Window Attention": section 3 (masked softmax,
  band mask), section 4 (rolling window cache), section 6 (core FLOPs table).
* "Exploring Attention Variants: Flash Attention, Sliding-Window, and Sparse
  Attention Implementation": attention_row, mask OR, kv_cache_bytes usage.
* "Attention Variants -- Sliding Window, Sparse, Differential": the
  differential problem statement.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MASK_SWA = 0
MASK_STRIDED = 1
MASK_CAUSAL = 2
MASK_GLOBAL = 3  # window + global tokens 0 .. g-1; the `stride` argument carries g
MASK_DILATED = 4  # window of W keys spaced by the dilation; the `stride` argument carries it

_KIND = {"swa": MASK_SWA, "strided": MASK_STRIDED, "causal": MASK_CAUSAL, "global": MASK_GLOBAL,
         "dilated": MASK_DILATED}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        I64 = ctypes.c_int64
        lib.orc_mask_row.argtypes = [I, I, I, I, I, P]
        lib.orc_mask.argtypes = [I, I, I, I, P]
        lib.orc_count_nonmasked.argtypes = [P, I64]
        lib.orc_count_nonmasked.restype = I64
        lib.orc_attention_row_f64.argtypes = [P, P, P, P, I, I, I, D, P, P]
        lib.orc_tiled_softmax_dot.argtypes = [P, P, P, P, I, I, I, D, I, P]
        lib.orc_attention.argtypes = [I, P, P, P, I, I, I, I, I, I, I, I, D, P, I64, P, P, I]
        lib.orc_attention.restype = I
        lib.orc_diff_attention.argtypes = [I, P, P, P, P, P, P, I, I, I, I, I, I, I, I, D, P, I64, P, I]
        lib.orc_diff_attention.restype = I
        lib.orc_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, D, P]
        lib.orc_decode.restype = I
        lib.orc_sink_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, D, P]
        lib.orc_sink_decode.restype = I
        lib.orc_diff_decode.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, D, P]
        lib.orc_diff_decode.restype = I
        for fn in ("orc_attention_bwd_dq_row", "orc_attention_bwd_dkv_row"):
            getattr(lib, fn).argtypes = [I, P, P, P, P, I, I, I, I, I, I, I, I, D, I, I, I] + (
                [P] if fn.endswith("dq_row") else [P, P])
            getattr(lib, fn).restype = None
        lib.orc_schedule_qtile.argtypes = [I, I, I, I, I, I, I, P, I64, P]
        lib.orc_schedule_qtile.restype = I64
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    """Accept numpy arrays or torch tensors (any float dtype, CPU)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def default_threads() -> int:
    return os.cpu_count() or 1


# ---------------------------------------------------------------- masks ---

def mask(kind: str, n: int, window: int = 0, stride: int = 0) -> np.ndarray:
    """The explicit n x n additive mask (0.0 attends, -inf masked)."""
    M = np.empty((n, n), dtype=np.float64)
    _L().orc_mask(_KIND[kind], n, window, stride, _p(M))
    return M


def swa_mask(n: int, window: int) -> np.ndarray:
    return mask("swa", n, window)


def strided_mask(n: int, window: int, stride: int) -> np.ndarray:
    return mask("strided", n, window, stride)


def causal_mask(n: int) -> np.ndarray:
    return mask("causal", n)


def mask_row(kind: str, n: int, i: int, window: int = 0, stride: int = 0) -> np.ndarray:
    r = np.empty(n, dtype=np.float64)
    _L().orc_mask_row(_KIND[kind], n, window, stride, i, _p(r))
    return r


def count_nonmasked(M: np.ndarray) -> int:
    M = np.ascontiguousarray(M, dtype=np.float64)
    return int(_L().orc_count_nonmasked(_p(M), M.size))


# ------------------------------------------------------------ attention ---

def attention_row(q, K, V, mask_row_, scale: float):
    """(out, weights) for one query row, in fp64."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    m = np.ascontiguousarray(mask_row_, dtype=np.float64)
    n, dk = K.shape
    dv = V.shape[1]
    out = np.empty(dv, dtype=np.float64)
    w = np.empty(n, dtype=np.float64)
    _L().orc_attention_row_f64(_p(q), _p(K), _p(V), _p(m), n, dk, dv, float(scale), _p(out), _p(w))
    return out, w


def tiled_softmax_dot(q, K, V, mask_row_, scale: float, tile: int = 4) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    m = np.ascontiguousarray(mask_row_, dtype=np.float64)
    n, dk = K.shape
    dv = V.shape[1]
    out = np.empty(dv, dtype=np.float64)
    _L().orc_tiled_softmax_dot(_p(q), _p(K), _p(V), _p(m), n, dk, dv, float(scale), int(tile), _p(out))
    return out


def _rows_arg(rows, total):
    if rows is None:
        return None, total
    r = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    if r.size and (r.min() < 0 or r.max() >= total):
        raise ValueError(f"row ids must lie in [0, {total})")
    return r, r.size


def attention(kind: str, q, k, v, W: int = 0, S: int = 0, scale: float | None = None,
              rows=None, with_lse: bool = False, nthreads: int | None = None):
    """Masked attention over [B,H,N,d] tensors.

    kind: "swa" (window W; W >= N is full causal), "strided" (window W OR
    every S-th key) or "causal". rows: optional flat row ids
    (b*Hq + h)*N + i; the result then has one row per id. Returns fp64
    [B,Hq,N,dv] (or [len(rows), dv]) and optionally the natural-log LSE.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, N, dk = q.shape
    Hkv = k.shape[1]
    dv = v.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    r, nrows = _rows_arg(rows, B * Hq * N)
    out = np.empty((nrows, dv), dtype=np.float64)
    lse = np.empty(nrows, dtype=np.float64) if with_lse else None
    rc = _L().orc_attention(_KIND[kind], _p(q), _p(k), _p(v), B, Hq, Hkv, N, dk, dv, int(W), int(S),
                            float(scale), None if r is None else _p(r), nrows, _p(out),
                            None if lse is None else _p(lse), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    if rows is None:
        out = out.reshape(B, Hq, N, dv)
        if lse is not None:
            lse = lse.reshape(B, Hq, N)
    return (out, lse) if with_lse else out


def diff_attention(q1, k1, q2, k2, v, lam, W: int | None = None, scale: float | None = None,
                   rows=None, nthreads: int | None = None):
    """Differential attention: sum_j (w1_ij - lambda_h w2_ij) v_j, both maps
    under the same sliding-window mask (W >= N, or None, is full causal)."""
    q1, k1, q2, k2, v = _f32(q1), _f32(k1), _f32(q2), _f32(k2), _f32(v)
    lam = _f32(lam).reshape(-1)
    B, Hq, N, dk = q1.shape
    Hkv = k1.shape[1]
    dv = v.shape[3]
    if W is None:
        W = N
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    r, nrows = _rows_arg(rows, B * Hq * N)
    out = np.empty((nrows, dv), dtype=np.float64)
    rc = _L().orc_diff_attention(MASK_SWA, _p(q1), _p(k1), _p(q2), _p(k2), _p(v), _p(lam), B, Hq, Hkv,
                                 N, dk, dv, int(W), 0, float(scale), None if r is None else _p(r),
                                 nrows, _p(out), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out.reshape(B, Hq, N, dv) if rows is None else out


def decode(q, k_new, v_new, k_cache, v_cache, pos, scale: float | None = None):
    """T decode steps over a rolling W-slot cache.

    q: [T,B,Hq,d]; k_new, v_new: [T,B,Hkv,d]; caches: [B,Hkv,W,d] (copied,
    the caller's arrays are not changed); pos: [T,B]. Returns (out [T,B,Hq,d]
    fp64, k_cache_after, v_cache_after)."""
    q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
    kc = _f32(k_cache).copy()
    vc = _f32(v_cache).copy()
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, B, Hq, d = q.shape
    Hkv = k_new.shape[2]
    W = kc.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((T, B, Hq, d), dtype=np.float64)
    rc = _L().orc_decode(_p(q), _p(k_new), _p(v_new), _p(kc), _p(vc), _p(pos), T, B, Hq, Hkv, d, W,
                         float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, kc, vc


def sink_decode(q, k_new, v_new, k_cache, v_cache, pos, n_sink: int, scale: float | None = None):
    """T decode steps with attention sinks over an (n_sink + W)-slot cache
    (StreamingLLM): positions below n_sink stay in their own slot, later ones
    rotate through the W window slots. Shapes as decode(); caches
    [B,Hkv,n_sink+W,d]. Returns (out, k_cache_after, v_cache_after)."""
    q, k_new, v_new = _f32(q), _f32(k_new), _f32(v_new)
    kc = _f32(k_cache).copy()
    vc = _f32(v_cache).copy()
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, B, Hq, d = q.shape
    Hkv = k_new.shape[2]
    W = kc.shape[2] - n_sink
    if W < 1:
        raise ValueError("the cache needs at least one window slot")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((T, B, Hq, d), dtype=np.float64)
    rc = _L().orc_sink_decode(_p(q), _p(k_new), _p(v_new), _p(kc), _p(vc), _p(pos), T, B, Hq, Hkv, d,
                              int(n_sink), W, float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, kc, vc


def diff_decode(q1, q2, k1_new, k2_new, v_new, k1_cache, k2_cache, v_cache, lam, pos,
                scale: float | None = None):
    """T differential decode steps over a rolling W-slot cache: both maps
    attend over the window, one V cache is shared.

    q1, q2: [T,B,Hq,dk]; k1_new, k2_new: [T,B,Hkv,dk]; v_new: [T,B,Hkv,dv];
    caches [B,Hkv,W,dk] / [B,Hkv,W,dv] (copied); lam: [Hq]; pos: [T,B].
    Returns (out [T,B,Hq,dv] fp64, k1_cache, k2_cache, v_cache after)."""
    q1, q2, k1_new, k2_new, v_new = _f32(q1), _f32(q2), _f32(k1_new), _f32(k2_new), _f32(v_new)
    k1c, k2c, vc = _f32(k1_cache).copy(), _f32(k2_cache).copy(), _f32(v_cache).copy()
    lam = _f32(lam).reshape(-1)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, B, Hq, dk = q1.shape
    Hkv, W, dv = vc.shape[1], vc.shape[2], vc.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    out = np.empty((T, B, Hq, dv), dtype=np.float64)
    rc = _L().orc_diff_decode(_p(q1), _p(q2), _p(k1_new), _p(k2_new), _p(v_new), _p(k1c), _p(k2c), _p(vc),
                              _p(lam), _p(pos), T, B, Hq, Hkv, dk, dv, W, float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle: bad arguments")
    return out, k1c, k2c, vc


def attention_bwd(kind: str, q, k, v, dO, W: int = 0, S: int = 0, scale: float | None = None,
                  dq_rows=None, dkv_rows=None):
    """Gradients of sum(O * dO) for the masked attention forward, from the
    chain rule written per output row (see oracle.c). q [B,Hq,N,dk], k
    [B,Hkv,N,dk], v [B,Hkv,N,dv], dO [B,Hq,N,dv]. With no row lists, returns
    full (dq, dk, dv); else dq for the flat (b*Hq + hq)*N + i rows in dq_rows
    and (dk, dv) for the flat (b*Hkv + hk)*N + j rows in dkv_rows."""
    q, k, v, dO = _f32(q), _f32(k), _f32(v), _f32(dO)
    B, Hq, N, dk = q.shape
    Hkv, dv = k.shape[1], v.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    lib, kd = _L(), _KIND[kind]
    args = (kd, _p(q), _p(k), _p(v), _p(dO), B, Hq, Hkv, N, dk, dv, int(W), int(S), float(scale))
    full = dq_rows is None and dkv_rows is None
    qr = np.arange(B * Hq * N) if full else np.asarray(dq_rows if dq_rows is not None else [], dtype=np.int64)
    kr = np.arange(B * Hkv * N) if full else np.asarray(dkv_rows if dkv_rows is not None else [], dtype=np.int64)
    dq = np.zeros((qr.size, dk))
    dkk = np.zeros((kr.size, dk))
    dvv = np.zeros((kr.size, dv))
    for n_, r in enumerate(qr):
        r = int(r)
        if not 0 <= r < B * Hq * N:
            raise ValueError("row out of range")
        buf = np.zeros(dk)
        lib.orc_attention_bwd_dq_row(*args, r // (Hq * N), (r // N) % Hq, r % N, _p(buf))
        dq[n_] = buf
    for n_, r in enumerate(kr):
        r = int(r)
        if not 0 <= r < B * Hkv * N:
            raise ValueError("row out of range")
        a, b_ = np.zeros(dk), np.zeros(dv)
        lib.orc_attention_bwd_dkv_row(*args, r // (Hkv * N), (r // N) % Hkv, r % N, _p(a), _p(b_))
        dkk[n_], dvv[n_] = a, b_
    if full:
        return dq.reshape(B, Hq, N, dk), dkk.reshape(B, Hkv, N, dk), dvv.reshape(B, Hkv, N, dv)
    return dq, dkk, dvv


# ------------------------------------------------------------- schedule ---

STRIDE_TAG = 0x40000000


def schedule_qtile(kind: str, N: int, W: int, S: int, Bq: int, Bk: int, qt: int):
    """(tiles, cells) for one query tile, read off the explicit mask."""
    cap = 2 * ((N + Bk - 1) // Bk) + ((N + max(S, 1) - 1) // max(S, 1) + Bk - 1) // Bk + 1
    tiles = np.empty(cap, dtype=np.int32)
    cells = np.zeros(1, dtype=np.int64)
    n = _L().orc_schedule_qtile(_KIND[kind], N, W, S, Bq, Bk, qt, _p(tiles), cap, _p(cells))
    if n == -2:
        raise AssertionError("an attended cell outside the window is not a multiple of S")
    if n < 0:
        raise ValueError("schedule capacity")
    return tiles[:n].tolist(), int(cells[0])


def schedule(kind: str, N: int, W: int, S: int, Bq: int, Bk: int):
    """Per query tile: lists of touched tiles and attended-cell counts."""
    nq = (N + Bq - 1) // Bq
    lists, cells = [], []
    for qt in range(nq):
        t, c = schedule_qtile(kind, N, W, S, Bq, Bk, qt)
        lists.append(t)
        cells.append(c)
    return lists, cells


# ------------------------------------------------------ closed helpers ---

def kv_cache_bytes(N: int, n_layers: int, n_heads_kv: int, d_head: int, dtype: int = 2,
                   window: int | None = None) -> int:
    """Cheatsheet task table kv_cache_bytes(N, n_layers, n_heads_kv, d_head,
    dtype=2): K and V, per layer, per KV head, per cached token, dtype bytes
    each. With a sliding window only min(N, window) tokens are cached
    (rolling buffer, "Learn: Sparse & Sliding-Window Attention" section 6)."""
    tokens = N if window is None else min(N, window)
    return 2 * n_layers * n_heads_kv * d_head * tokens * dtype


def count_nsa(N: int, l: int, k: int, W: int) -> int:
    """Cheatsheet count_nsa(N, l, k, W): compressed keys N/l, plus k selected
    blocks of l keys, plus a window of W keys (FAQ: 32 + 128 + 128 = 288 at
    N=1024, l=32, k=4, w=128)."""
    return N // l + k * l + W


def core_flops(nnz: int, d: int, b: int = 1) -> int:
    """Core attention FLOPs ("Learn: Sparse & Sliding-Window Attention"
    section 6 table): 4 * b * allowed_entries * d (scores plus A.V, a
    multiply-add counted as 2)."""
    return 4 * b * nnz * d
