"""swa_decode_step_static: the decode step for callers that cannot allocate
device memory (for instance a plugin host that gives the library tensors but
no allocator, or a serving loop that may not allocate on its hot path). Its
scratch is a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against swa_decode_step (which takes a caller
workspace) on two calls in a row, at the tolerance the other GPU tests use.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import differential_attention_swa_b200 as swa
from differential_attention_swa_b200.inputs import decode_inputs

pytestmark = pytest.mark.gpu

MAX_TOL = 1e-2
MEAN_TOL = 2e-3
SCRATCH_TOO_SMALL = 5
STATIC_SCRATCH_BYTES = 4 << 20


@pytest.fixture(scope="module")
def lib():
    from differential_attention_swa_b200 import build

    build.build()
    lib = swa.library()
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.swa_decode_step_static.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P]
    lib.swa_decode_step_static.restype = I
    return lib


def ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_static_scratch_matches_workspace_entry_point(lib):
    B, Hq, Hkv, d, W, T = 8, 16, 8, 128, 1024, 2
    assert swa.decode_workspace_bytes(B, Hq, Hkv, d, W) <= STATIC_SCRATCH_BYTES
    q, k_new, v_new, k_cache, v_cache = (t.cuda() for t in decode_inputs(T, B, Hq, Hkv, d, W, seed=21))
    kc_a, vc_a = k_cache.clone(), v_cache.clone()
    kc_b, vc_b = k_cache.clone(), v_cache.clone()
    pos = torch.tensor([[1500 + t] * B for t in range(T)], dtype=torch.int32, device="cuda")
    ws = torch.empty(swa.decode_workspace_bytes(B, Hq, Hkv, d, W), dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    scale = ctypes.c_float(1.0 / np.sqrt(d))
    for t in range(T):  # two calls in a row: the array keeps the previous call's contents
        out_a = torch.empty_like(q[t])
        out_b = torch.full_like(q[t], float("nan"))
        st = lib.swa_decode_step(ptr(q[t]), ptr(k_new[t]), ptr(v_new[t]), ptr(kc_a), ptr(vc_a), ptr(pos[t]),
                                 ptr(out_a), B, Hq, Hkv, d, W, scale, ptr(ws), ws.numel(), stream)
        assert st == swa.OK
        st = lib.swa_decode_step_static(ptr(q[t]), ptr(k_new[t]), ptr(v_new[t]), ptr(kc_b), ptr(vc_b),
                                        ptr(pos[t]), ptr(out_b), B, Hq, Hkv, d, W, scale, stream)
        assert st == swa.OK
        torch.cuda.synchronize()
        assert swa.last_device_error() == swa.OK
        diff = (out_a.float() - out_b.float()).abs()
        assert torch.isfinite(out_b.float()).all()
        assert diff.max().item() <= MAX_TOL and diff.mean().item() <= MEAN_TOL
        # the same kernels with the same split plan: identical bits, so no
        # record of the shared array may be stale or misplaced
        assert torch.equal(out_a, out_b)
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)


def test_short_history_after_a_larger_call(lib):
    """A call whose position is still inside the first window (pos < W, so
    some splits hold no position yet) right after a call that filled every
    record of the array: the empty splits must overwrite the old records."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for (B, Hq, Hkv, d, W, pos0) in [(8, 16, 8, 128, 1024, 5000), (8, 16, 8, 128, 1024, 3)]:
        T = 2
        q, k_new, v_new, k_cache, v_cache = (t.cuda() for t in decode_inputs(T, B, Hq, Hkv, d, W, seed=pos0))
        kc_a, vc_a = k_cache.clone(), v_cache.clone()
        kc_b, vc_b = k_cache.clone(), v_cache.clone()
        pos = torch.tensor([[pos0 + t] * B for t in range(T)], dtype=torch.int32, device="cuda")
        ws = torch.empty(swa.decode_workspace_bytes(B, Hq, Hkv, d, W), dtype=torch.uint8, device="cuda")
        scale = ctypes.c_float(1.0 / np.sqrt(d))
        for t in range(T):
            out_a = torch.empty_like(q[t])
            out_b = torch.full_like(q[t], float("nan"))
            assert lib.swa_decode_step(ptr(q[t]), ptr(k_new[t]), ptr(v_new[t]), ptr(kc_a), ptr(vc_a), ptr(pos[t]),
                                       ptr(out_a), B, Hq, Hkv, d, W, scale, ptr(ws), ws.numel(), stream) == swa.OK
            assert lib.swa_decode_step_static(ptr(q[t]), ptr(k_new[t]), ptr(v_new[t]), ptr(kc_b), ptr(vc_b),
                                              ptr(pos[t]), ptr(out_b), B, Hq, Hkv, d, W, scale, stream) == swa.OK
            torch.cuda.synchronize()
            assert swa.last_device_error() == swa.OK
            assert torch.equal(out_a, out_b), (pos0, t)


def test_sizes_beyond_the_array_are_rejected(lib):
    B, Hq, Hkv, d, W = 256, 32, 8, 128, 4096
    assert swa.decode_workspace_bytes(B, Hq, Hkv, d, W) > STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    st = lib.swa_decode_step_static(fake, fake, fake, fake, fake, fake, fake, B, Hq, Hkv, d, W,
                                    ctypes.c_float(0.1), None)
    assert st == SCRATCH_TOO_SMALL
    assert lib.swa_status_string(SCRATCH_TOO_SMALL) != b"unknown status"
