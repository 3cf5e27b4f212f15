"""The bounds-checking debug build (libswa_attn_debug.so, compiled with
-DSWA_DEBUG_BOUNDS): every TMA coordinate and computed global index of the
prefill, decode, differential decode and backward kernels checks itself
against the tensor it addresses and reports SWA_ERR_BOUNDS instead of
accessing out of range. The tiny and edge cases run through it here; each
must report SWA_OK and give the release build's outputs bit for bit (the
checks add no arithmetic)."""
import numpy as np
import pytest
import torch

import differential_attention_swa_b200 as swa
from differential_attention_swa_b200.inputs import (attn_inputs, decode_inputs, diff_decode_inputs, diff_inputs,
                                                    randn_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib():
    from differential_attention_swa_b200 import build

    build.build()
    build.build(debug_bounds=True)
    swa.library()
    return swa.load(swa.DEBUG_LIB_PATH)


def release_and_debug(debug_lib, fn):
    """Runs fn with the release library, then with the debug build; both must
    report SWA_OK and agree bit for bit."""
    got_r = fn()
    assert swa.last_device_error() == swa.OK
    prev = swa.use_library(debug_lib)
    try:
        got_d = fn()
        st = swa.last_device_error()
    finally:
        swa.use_library(prev)
    assert st == swa.OK, f"debug build reported status {st}"
    got_r = got_r if isinstance(got_r, (tuple, list)) else (got_r,)
    got_d = got_d if isinstance(got_d, (tuple, list)) else (got_d,)
    for a, b in zip(got_r, got_d):
        assert torch.equal(a, b)


PREFILL = [
    # kind, B, Hq, Hkv, N, d, W, S (stride, global tokens or dilation)
    ("swa", 1, 2, 2, 256, 64, 64, 0),
    ("strided", 1, 2, 2, 256, 64, 16, 8),
    ("swa", 1, 2, 2, 1, 64, 4, 0),
    ("swa", 1, 2, 2, 200, 64, 64, 0),
    ("swa", 1, 6, 2, 257, 128, 129, 0),
    ("swa", 2, 4, 2, 640, 128, 256, 0),
    ("swa", 2, 4, 4, 500, 64, 100, 0),
    ("strided", 1, 2, 2, 300, 64, 17, 5),
    ("strided", 1, 2, 2, 333, 64, 20, 400),
    ("strided", 2, 6, 2, 700, 64, 40, 9),
    ("global", 1, 2, 2, 900, 64, 100, 300),
    ("global", 1, 6, 2, 513, 128, 40, 7),
    ("dilated", 1, 4, 2, 777, 128, 64, 3),
    ("dilated", 1, 3, 1, 300, 64, 20, 7),
]


@pytest.mark.parametrize("kind,B,Hq,Hkv,N,d,W,S", PREFILL)
def test_prefill_in_bounds(debug_lib, kind, B, Hq, Hkv, N, d, W, S):
    q, k, v = (t.cuda() for t in attn_inputs(B, Hq, Hkv, N, d, seed=N + W))

    def run():
        if kind == "swa":
            return swa.swa_attn_fwd(q, k, v, W, return_lse=True)
        if kind == "strided":
            return swa.strided_attn_fwd(q, k, v, W, S, return_lse=True)
        if kind == "global":
            return swa.global_attn_fwd(q, k, v, W, S, return_lse=True)
        return swa.dilated_attn_fwd(q, k, v, W, S, return_lse=True)

    release_and_debug(debug_lib, run)


def test_prefill_debug_outputs_in_bounds(debug_lib):
    q, k, v = (t.cuda() for t in attn_inputs(1, 2, 2, 700, 64, seed=3))
    release_and_debug(debug_lib, lambda: swa.prefill_debug(swa.MASK_STRIDED, q, k, v, 40, 9, tiles_cap=8))


@pytest.mark.parametrize("N,W,dv,Hq,Hkv", [(256, None, 128, 2, 2), (300, 70, 128, 2, 1), (513, None, 64, 4, 2)])
def test_diff_prefill_in_bounds(debug_lib, N, W, dv, Hq, Hkv):
    ins = [t.cuda() for t in diff_inputs(1, Hq, Hkv, N, 64, dv, seed=3)]
    lam = torch.linspace(0.2, 0.8, Hq, device="cuda")
    release_and_debug(debug_lib, lambda: swa.diff_attn_fwd(*ins, lam, window=W, scale=0.125))


@pytest.mark.parametrize("B,Hq,Hkv,d,n_sink,W,pos0,T", [(2, 4, 2, 128, 0, 64, 60, 6), (5, 8, 8, 64, 0, 1500, 1400, 2),
                                                         (2, 4, 2, 128, 4, 64, 0, 8), (1, 8, 1, 64, 2, 100, 120, 2)])
def test_decode_in_bounds(debug_lib, B, Hq, Hkv, d, n_sink, W, pos0, T):
    q, kn, vn, kc0, vc0 = (t.cuda() for t in decode_inputs(T, B, Hq, Hkv, d, n_sink + W, seed=9))
    pos = torch.tensor([[pos0 + t] * B for t in range(T)], dtype=torch.int32, device="cuda")

    def run():
        kc, vc = kc0.clone(), vc0.clone()
        outs = [swa.swa_sink_decode_step(q[t], kn[t], vn[t], kc, vc, pos[t], n_sink) for t in range(T)]
        return torch.stack(outs), kc, vc

    release_and_debug(debug_lib, run)


def test_diff_decode_in_bounds(debug_lib):
    T, B, Hq, Hkv, W = 4, 2, 4, 2, 64
    q1, q2, k1n, k2n, vn, k1c, k2c, vc = (t.cuda() for t in diff_decode_inputs(T, B, Hq, Hkv, 64, 128, W, seed=31))
    pos = torch.tensor([[62 + t] * B for t in range(T)], dtype=torch.int32, device="cuda")
    lam = torch.linspace(0.2, 0.8, Hq, device="cuda")

    def run():
        caches = [c.clone() for c in (k1c, k2c, vc)]
        outs = [swa.swa_diff_decode_step(q1[t], q2[t], k1n[t], k2n[t], vn[t], *caches, pos[t], lam) for t in range(T)]
        return (torch.stack(outs), *caches)

    release_and_debug(debug_lib, run)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W,S", [(1, 4, 2, 300, 128, 100, 0), (1, 2, 2, 129, 64, 1, 0),
                                              (1, 6, 2, 257, 64, 130, 0), (1, 2, 2, 700, 64, 40, 9)])
def test_backward_in_bounds(debug_lib, B, Hq, Hkv, N, d, W, S):
    q, k, v = (t.cuda() for t in attn_inputs(B, Hq, Hkv, N, d, seed=N + W))
    d_o = randn_bf16((B, Hq, N, d), N + W + 10).cuda()
    if S:
        o, lse = swa.strided_attn_fwd(q, k, v, W, S, return_lse=True)
    else:
        o, lse = swa.swa_attn_fwd(q, k, v, W, return_lse=True)

    def run():
        dq, dk, dv = swa.swa_attn_bwd(q, k, v, o, d_o, lse, W, stride=S)
        if S:  # the stride keys' fp32 partials are summed with atomics in varying order
            return (dq,)
        return dq, dk, dv

    release_and_debug(debug_lib, run)
    if S:  # dK/dV of the strided backward: in bounds, and within rounding of the release build
        prev = swa.use_library(debug_lib)
        try:
            dq, dk, dv = swa.swa_attn_bwd(q, k, v, o, d_o, lse, W, stride=S)
            assert swa.last_device_error() == swa.OK
        finally:
            swa.use_library(prev)
        rq, rk, rv = swa.swa_attn_bwd(q, k, v, o, d_o, lse, W, stride=S)
        for a, b in ((dk, rk), (dv, rv)):
            scale = b.float().abs().max().item()
            assert (a.float() - b.float()).abs().max().item() <= 1e-2 * scale


def test_exp2_in_bounds(debug_lib):
    x = torch.from_numpy(np.linspace(-130, 8, 4097, dtype=np.float32)).cuda()
    release_and_debug(debug_lib, lambda: swa.debug_exp2(x))
