"""Host-side checks of the C ABI (no GPU needed): the library loads and
exports every function include/*.h declares; the schedule export matches the
oracle's explicit-mask derivation bit for bit; the closed-form attended-cell
count matches the oracle; bad arguments are rejected before any launch."""
import ctypes
import glob
import os
import re

import pytest

from conftest import ROOT

import differential_attention_swa_b200 as swa


@pytest.fixture(scope="module")
def lib():
    from differential_attention_swa_b200 import build

    build.build()
    return swa.library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "while", "for", "sizeof", "return"):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("swa_attn_fwd", "strided_attn_fwd", "diff_attn_fwd", "swa_decode_step", "swa_schedule",
                 "swa_count_nonmasked", "swa_last_device_error", "swa_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {swa.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


@pytest.mark.parametrize("kind,okind,N,W,S", [
    (0, "swa", 256, 64, 0), (1, "strided", 256, 16, 8), (0, "swa", 1000, 130, 0), (1, "strided", 1000, 1, 1),
    (1, "strided", 777, 200, 7), (0, "swa", 129, 5000, 0), (1, "strided", 300, 17, 400), (2, "causal", 513, 0, 0),
    (0, "swa", 1, 1, 0), (1, "strided", 4000, 128, 128), (3, "global", 256, 16, 8), (3, "global", 1000, 130, 300),
    (3, "global", 777, 64, 0), (3, "global", 500, 600, 40), (3, "global", 4000, 512, 64), (3, "global", 300, 1, 1)])
def test_schedule_export_bit_exact_vs_oracle(lib, orc, kind, okind, N, W, S):
    got = swa.schedule(kind, N, W, S)
    want, _ = orc.schedule(okind, N, W, S, 128, 128)
    assert got == want


def test_schedule_sampled_at_workload_sizes(lib, orc):
    for (kind, okind, N, W, S, qts) in [(0, "swa", 8192, 4096, 0, (0, 1, 31, 32, 63)),
                                        (1, "strided", 16384, 128, 128, (0, 1, 2, 64, 127)),
                                        (0, "swa", 131072, 1024, 0, (0, 7, 8, 9, 1023))]:
        got = swa.schedule(kind, N, W, S)
        for qt in qts:
            want, _ = orc.schedule_qtile(okind, N, W, S, 128, 128, qt)
            assert got[qt] == want, (N, qt)
    assert sum(len(x) for x in swa.schedule(0, 8192, 4096)) == 1584
    assert sum(len(x) for x in swa.schedule(0, 131072, 1024)) == 9180
    assert sum(len(x) for x in swa.schedule(1, 16384, 128, 128)) == 382


@pytest.mark.parametrize("kind,okind,N,W,S", [
    (0, "swa", 256, 64, 0), (1, "strided", 256, 16, 8), (1, "strided", 300, 17, 5), (0, "swa", 50, 50, 0),
    (0, "swa", 50, 1, 0), (1, "strided", 97, 3, 1), (1, "strided", 97, 200, 3), (2, "causal", 70, 0, 0),
    (3, "global", 256, 16, 8), (3, "global", 300, 17, 200), (3, "global", 97, 3, 0), (3, "global", 97, 200, 5),
    (3, "global", 130, 9, 130)])
def test_count_nonmasked_closed_form_vs_oracle(lib, orc, kind, okind, N, W, S):
    M = orc.mask(okind, N, W, S)
    assert swa.count_nonmasked(kind, N, W, S) == orc.count_nonmasked(M)


def test_count_nonmasked_workloads(lib):
    assert swa.count_nonmasked(0, 8192, 4096) == 25167872
    assert swa.count_nonmasked(1, 16384, 128, 128) == 3129408
    assert swa.count_nonmasked(0, 131072, 1024) == 133693952
    assert swa.count_nonmasked(0, 4096, 4096) == 8390656
    assert swa.count_nonmasked(0, 256, 64) == 14368
    assert swa.count_nonmasked(1, 256, 16, 8) == 7696


def test_bad_arguments_rejected_before_launch(lib):
    P = ctypes.c_void_p
    good = P(0x10000)  # aligned, never dereferenced: validation fails first
    nullp = None
    st = lib.swa_attn_fwd(nullp, good, good, good, None, 1, 2, 2, 256, 64, 64, 0.125, None)
    assert st == swa.ERR_INVALID_ARG
    st = lib.swa_attn_fwd(P(0x10008), good, good, good, None, 1, 2, 2, 256, 64, 64, 0.125, None)
    assert st == swa.ERR_INVALID_ARG  # misaligned
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 3, 2, 256, 64, 64, 0.125, None)
    assert st == swa.ERR_INVALID_ARG  # Hq % Hkv
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 2, 2, 256, 64, 0, 0.125, None)
    assert st == swa.ERR_INVALID_ARG  # W < 1
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 2, 2, 0, 64, 4, 0.125, None)
    assert st == swa.ERR_INVALID_ARG  # N < 1
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 2, 2, 256, 64, 4, -1.0, None)
    assert st == swa.ERR_INVALID_ARG  # scale
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 2, 2, 256, 64, 4, 1e-31, None)
    assert st == swa.ERR_INVALID_ARG  # scale below 1e-30: masked weights would no longer be exactly 0
    st = lib.swa_attn_fwd(good, good, good, good, None, 1, 2, 2, 256, 96, 4, 0.1, None)
    assert st == swa.ERR_UNSUPPORTED  # head dim
    st = lib.strided_attn_fwd(good, good, good, good, None, 1, 2, 2, 256, 64, 4, 0, 0.1, None)
    assert st == swa.ERR_INVALID_ARG  # stride < 1
    st = lib.diff_attn_fwd(good, good, good, good, good, good, None, 1, 2, 2, 64, 64, 128, 64, 0.1, None)
    assert st == swa.ERR_INVALID_ARG  # lambda missing
    st = lib.diff_attn_fwd(good, good, good, good, good, good, good, 1, 2, 2, 64, 128, 128, 64, 0.1, None)
    assert st == swa.ERR_UNSUPPORTED  # d_qk 128 not built for the differential kernel
    ws = lib.swa_decode_workspace_bytes(64, 16, 8, 128, 1024)
    assert ws > 0
    st = lib.swa_decode_step(good, good, good, good, good, good, good, 64, 16, 8, 128, 1024, 0.1, good, ws - 1,
                             None)
    assert st == swa.ERR_INVALID_ARG  # workspace too small
    st = lib.swa_decode_step(good, good, good, good, good, good, good, 2, 6, 2, 128, 16, 0.1, good, 1 << 20,
                             None)
    assert st == swa.ERR_UNSUPPORTED  # group size 3
    assert lib.swa_decode_workspace_bytes(1, 3, 2, 128, 16) == 0
    assert lib.swa_schedule(0, 0, 4, 0, 128, 128, None, None, 0) == -1
    assert lib.swa_count_nonmasked(1, 10, 4, 0) == -1
    assert lib.swa_status_string(swa.ERR_TIMEOUT) == b"in-kernel wait timed out"


def test_python_binding_refuses_cpu_tensors(lib):
    import torch

    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        swa.swa_attn_fwd(q, q, q, 4)


def test_diff_decode_bad_arguments_rejected_before_launch(lib):
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    g = P(0x10000)  # aligned, never dereferenced: validation fails first
    ws = lib.swa_diff_decode_workspace_bytes(64, 16, 8, 64, 128, 4096)
    assert ws > 0
    assert lib.swa_diff_decode_workspace_bytes(64, 16, 8, 128, 128, 4096) == 0  # d_qk 128 not built
    assert lib.swa_diff_decode_workspace_bytes(64, 16, 6, 64, 128, 4096) == 0  # Hq % Hkv

    def call(B=64, Hq=16, Hkv=8, dqk=64, dv=128, W=4096, scale=0.125, wsb=ws, lam=g, q1=g):
        return lib.swa_diff_decode_step(q1, g, g, g, g, g, g, g, g, lam, g, I(B), I(Hq), I(Hkv), I(dqk), I(dv),
                                        I(W), F(scale), g, SZ(wsb), None)

    assert call(wsb=ws - 1) == swa.ERR_INVALID_ARG  # workspace too small
    assert call(lam=None) == swa.ERR_INVALID_ARG  # lambda missing
    assert call(q1=P(0x10008)) == swa.ERR_INVALID_ARG  # misaligned
    assert call(W=0) == swa.ERR_INVALID_ARG
    assert call(scale=0.0) == swa.ERR_INVALID_ARG
    assert call(dqk=128) == swa.ERR_UNSUPPORTED
    assert call(Hq=24, Hkv=8) == swa.ERR_UNSUPPORTED  # group of 3


def test_global_and_dilated_bad_arguments(lib):
    P = ctypes.c_void_p
    g = P(0x10000)
    st = lib.global_attn_fwd(g, g, g, g, None, 1, 2, 2, 256, 64, 16, -1, ctypes.c_float(0.1), None)
    assert st == swa.ERR_INVALID_ARG  # negative number of global tokens
    st = lib.dilated_attn_fwd(g, g, g, g, None, 1, 2, 2, 256, 64, 16, 0, ctypes.c_float(0.1), None)
    assert st == swa.ERR_INVALID_ARG  # dilation 0
    st = lib.dilated_attn_fwd(g, g, g, g, None, 1, 2, 2, 256, 96, 16, 2, ctypes.c_float(0.1), None)
    assert st == swa.ERR_UNSUPPORTED  # head dim
    assert lib.swa_count_nonmasked(3, 10, 4, -1) == -1


def test_decode_window_beyond_limit_rejected_before_launch(lib):
    """A window past 2^30 slots would overflow the split arithmetic: every
    decode entry rejects it (and the workspace query returns 0) up front."""
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    g = P(0x10000)  # aligned, never dereferenced: validation fails first
    big = (1 << 30) + 1
    lib.swa_decode_step_static.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P]
    lib.swa_decode_step_static.restype = I
    st = lib.swa_decode_step_static(g, g, g, g, g, g, g, 1, 2, 1, 128, big, F(0.1), None)
    assert st == swa.ERR_INVALID_ARG
    st = lib.swa_decode_step_static(g, g, g, g, g, g, g, 1, 2, 1, 128, 0x7fffffff, F(0.1), None)
    assert st == swa.ERR_INVALID_ARG
    assert lib.swa_decode_workspace_bytes(1, 2, 1, 128, big) == 0
    assert lib.swa_sink_decode_workspace_bytes(1, 2, 1, 128, 4, 1 << 30) == 0
    assert lib.swa_diff_decode_workspace_bytes(1, 2, 1, 64, 128, big) == 0
    st = lib.swa_decode_step(g, g, g, g, g, g, g, 1, 2, 1, 128, big, 0.1, g, 1 << 40, None)
    assert st == swa.ERR_INVALID_ARG


def test_debug_exp2_bad_arguments(lib):
    P = ctypes.c_void_p
    g = P(0x10000)
    assert lib.swa_debug_exp2(None, g, 4, None) == swa.ERR_INVALID_ARG
    assert lib.swa_debug_exp2(g, P(0x10002), 4, None) == swa.ERR_INVALID_ARG  # misaligned
    assert lib.swa_debug_exp2(g, g, -1, None) == swa.ERR_INVALID_ARG
    assert lib.swa_debug_exp2(g, g, 0, None) == swa.OK  # nothing to do, nothing launched
