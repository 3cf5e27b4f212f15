"""GPU parity: every C-ABI entry point against the fp64 oracle on the same
seeded bf16 inputs.

Bars: bf16 outputs (fp32 accumulate) within max|diff| <= 1e-2 and
mean|diff| <= 2e-3 of the fp64 oracle; visited key-tile lists and attended
cell counts bit-exact against the oracle's explicit-mask derivation."""
import math

import numpy as np
import pytest
import torch

import differential_attention_swa_b200 as swa
from differential_attention_swa_b200.inputs import WORKLOADS, attn_inputs, decode_inputs, diff_decode_inputs, diff_inputs

pytestmark = pytest.mark.gpu

MAX_TOL = 1e-2
MEAN_TOL = 2e-3
KIND = {"swa": swa.MASK_WINDOW, "strided": swa.MASK_STRIDED, "global": swa.MASK_GLOBAL}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from differential_attention_swa_b200 import build

    build.build()
    swa.library()
    assert swa.last_device_error() == swa.OK


def gpu(*ts):
    return [t.cuda() for t in ts]


def compare(got, want, what):
    got = got.float().cpu().numpy().astype(np.float64).reshape(want.shape)
    diff = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = diff.max(), diff.mean()
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def run_prefill(kind, q, k, v, W, S, lse=False):
    qd, kd, vd = gpu(q, k, v)
    if kind == "swa":
        r = swa.swa_attn_fwd(qd, kd, vd, W, return_lse=lse)
    elif kind == "global":  # S carries the number of global tokens
        r = swa.global_attn_fwd(qd, kd, vd, W, S, return_lse=lse)
    elif kind == "dilated":  # S carries the dilation
        r = swa.dilated_attn_fwd(qd, kd, vd, W, S, return_lse=lse)
    else:
        r = swa.strided_attn_fwd(qd, kd, vd, W, S, return_lse=lse)
    assert swa.last_device_error() == swa.OK
    return r


# ------------------------------------------------------------ tiny, full --

@pytest.mark.parametrize("name", ["tiny_swa", "tiny_strided"])
def test_tiny_workloads_full(orc, name):
    w = WORKLOADS[name]
    q, k, v = attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=0)
    out, lse = run_prefill(w.kind, q, k, v, w.W, w.S, lse=True)
    ref, ref_lse = orc.attention(w.kind, q, k, v, W=w.W, S=w.S, scale=w.scale, with_lse=True)
    compare(out, ref, name)
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 2e-3


EDGE = [
    # kind, B, Hq, Hkv, N, d, W, S
    ("swa", 1, 2, 2, 200, 64, 64, 0),       # ragged tail, odd tile count
    ("swa", 1, 2, 2, 1, 64, 4, 0),          # a single row
    ("swa", 1, 1, 1, 127, 64, 1, 0),        # window 1: out = V
    ("swa", 2, 4, 4, 300, 64, 5000, 0),     # window beyond N: full causal
    ("swa", 1, 8, 2, 384, 128, 100, 0),     # GQA group 4: head pairs
    ("swa", 1, 6, 2, 257, 128, 129, 0),     # GQA group 3: tile pairs, ragged
    ("swa", 2, 4, 2, 640, 128, 256, 0),     # group 2, several tiles
    ("swa", 1, 2, 1, 130, 64, 128, 0),      # W equal to one tile
    ("strided", 1, 2, 2, 300, 64, 17, 5),   # N not a multiple of S
    ("strided", 1, 2, 2, 256, 64, 3, 1),    # stride 1: every key (full causal)
    ("strided", 1, 2, 2, 333, 64, 20, 400), # stride beyond N: window + key 0
    ("strided", 1, 4, 2, 1000, 128, 64, 7), # group 2 with stride tiles
    ("strided", 1, 2, 2, 700, 64, 1, 3),    # window 1 + stride
    ("global", 1, 2, 2, 700, 64, 64, 50),   # global keys in a partial tile
    ("global", 1, 2, 2, 900, 64, 100, 300), # global tokens span several tiles and the window
    ("global", 1, 4, 2, 1000, 128, 64, 128),# group 2, one whole global tile
    ("global", 1, 6, 2, 513, 128, 40, 7),   # group 3 (tile pairs), ragged
    ("global", 1, 2, 2, 300, 64, 5000, 9),  # window beyond N: full causal
    ("global", 1, 2, 2, 400, 64, 16, 0),    # no global token: the window
    ("global", 1, 2, 2, 333, 64, 1, 1000),  # every token global: full causal
    ("dilated", 1, 2, 2, 1000, 64, 100, 2), # dilation 2, several tiles per class
    ("dilated", 1, 4, 2, 777, 128, 64, 3),  # N not a multiple of the dilation, group 2
    ("dilated", 1, 3, 1, 300, 64, 20, 7),   # group 3 (tile pairs), short classes
    ("dilated", 1, 2, 2, 250, 64, 30, 1),   # dilation 1: the window
    ("dilated", 1, 2, 2, 100, 64, 5, 150),  # dilation beyond N: each row sees only itself
    # d = 64 with an odd group size: pairs of query heads at the same query
    # tile, each with its own KV head (heads 2 and 3 of group 3 straddle two)
    ("swa", 2, 4, 4, 500, 64, 100, 0),      # group 1, two batches
    # group 3, stride tiles. N = 700 (seed 740) has two-key rows at |o| ~ 2.1,
    # where the output's own bf16 rounding is up to 7.8e-3: it measured 1.12e-2
    # while the row sum added unrounded weights that the PV product never
    # used (the weights applied to V did not sum to one)
    ("strided", 2, 6, 2, 700, 64, 40, 9),
    ("strided", 2, 6, 2, 701, 64, 40, 9),
    ("global", 1, 6, 2, 600, 64, 64, 70),   # group 3, global keys
    ("dilated", 1, 6, 2, 900, 64, 50, 2),   # group 3, dilation 2
]


@pytest.mark.parametrize("kind,B,Hq,Hkv,N,d,W,S", EDGE)
def test_edge_cases_full(orc, kind, B, Hq, Hkv, N, d, W, S):
    q, k, v = attn_inputs(B, Hq, Hkv, N, d, seed=N + W)
    out = run_prefill(kind, q, k, v, W, S)
    ref = orc.attention(kind, q, k, v, W=W, S=S, scale=1 / math.sqrt(d))
    compare(out, ref, f"{kind} N{N} W{W} S{S}")


# Rows with one to three attended keys and outputs of magnitude 2 and more
# sit at the flat bar's bf16 edge. Their error is bounded by the two roundings
# the kernels make: each weight is rounded to bf16 (relative error u = 2^-8)
# before the PV product, and the output is rounded to bf16. With the row sum
# taken over the rounded weights (so that the weights applied to V sum to
# one), o' - o = sum_j w_j (d_j - dbar) (v_j - o) / (1 + dbar), |d_j| <= u,
# which gives the per-element bound below; a row sum of the unrounded weights
# adds sum_j w_j d_j v_j instead, which this bound catches. With W = 2 that
# bound plus the output's half-ulp (7.8e-3 from |o| = 2) can pass 1e-2: the
# flat bar cannot hold for every such row with bf16 weights.
U = 2.0 ** -8
SHORT_ROWS = [(kind, W, S, d, seed) for kind, W, S, d in [
    ("swa", 1, 0, 64), ("swa", 2, 0, 64), ("swa", 3, 0, 64), ("swa", 1, 0, 128), ("swa", 2, 0, 128),
    ("swa", 3, 0, 128), ("strided", 1, 5, 64), ("strided", 2, 7, 64), ("strided", 3, 9, 64), ("strided", 2, 3, 128),
    ("global", 1, 2, 64), ("global", 2, 3, 64), ("global", 3, 5, 128)] for seed in range(8)]


def half_ulp_bf16(x):
    x = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(x)) - 8)


@pytest.mark.parametrize("kind,W,S,d,seed", SHORT_ROWS)
def test_short_rows_at_the_bf16_edge(orc, kind, W, S, d, seed):
    N, H = 260, 2
    q, k, v = attn_inputs(1, H, 1, N, d, seed=1000 + seed)
    out = run_prefill(kind, q, k, v, W, S).float().cpu().numpy().astype(np.float64)[0]
    if kind == "swa" and W == 1:  # one key: weight exactly 1, the output is V bit for bit
        assert np.array_equal(out, np.broadcast_to(v.float().numpy()[0, 0], out.shape))
        return
    scale = 1 / math.sqrt(d)
    qf, kf, vf = (t.float().numpy().astype(np.float64) for t in (q, k, v))
    for h in range(H):
        for i in range(N):
            o, w = orc.attention_row(qf[0, h, i], kf[0, 0], vf[0, 0], orc.mask_row(kind, N, i, W, S), scale)
            e1 = 2 * U / (1 - U) * (w[:, None] * np.abs(vf[0, 0] - o[None, :])).sum(0) + 1e-5
            bound = e1 + half_ulp_bf16(np.abs(o) + e1)
            err = np.abs(out[h, i] - o)
            assert (err <= bound).all(), (h, i, err.max(), bound[err.argmax()], o[err.argmax()])
    ref = orc.attention(kind, q, k, v, W=W, S=S, scale=scale)
    assert np.abs(out - ref[0]).mean() <= MEAN_TOL


@pytest.mark.parametrize("kind,N,W,S,Hq,Hkv,d", [
    ("swa", 256, 64, 0, 2, 2, 64), ("strided", 256, 16, 8, 2, 2, 64), ("swa", 1000, 300, 0, 4, 2, 128),
    ("strided", 1500, 100, 9, 2, 2, 64), ("swa", 385, 5000, 0, 3, 1, 64), ("strided", 2048, 128, 128, 2, 1, 64),
    ("global", 1500, 100, 300, 2, 2, 64), ("global", 1000, 512, 64, 4, 2, 128), ("global", 777, 64, 0, 3, 1, 64),
    ("strided", 700, 40, 9, 6, 2, 64), ("global", 600, 64, 70, 6, 2, 64)])
def test_visited_tiles_and_cells_bit_exact(orc, kind, N, W, S, Hq, Hkv, d):
    q, k, v = attn_inputs(1, Hq, Hkv, N, d, seed=7)
    qd, kd, vd = gpu(q, k, v)
    out, cells, tiles, ntiles = swa.prefill_debug(KIND[kind], qd, kd, vd, W, S, tiles_cap=64)
    assert swa.last_device_error() == swa.OK
    lists, want_cells = orc.schedule(kind, N, W, S, 128, 128)
    cells, tiles, ntiles = cells.cpu(), tiles.cpu(), ntiles.cpu()
    for h in range(Hq):
        for qt, (lst, c) in enumerate(zip(lists, want_cells)):
            assert int(ntiles[0, h, qt]) == len(lst), (h, qt)
            assert tiles[0, h, qt, :len(lst)].tolist() == lst, (h, qt)
            assert int(cells[0, h, qt]) == c, (h, qt)
    ref = orc.attention(kind, q, k, v, W=W, S=S, scale=1 / math.sqrt(d))
    compare(out, ref, "debug path output")


# The kernel's own visiting lists and per-tile attended-cell counts at the
# workloads' sequence lengths and masks (cost proportional to ||M||_0, "Learn:
# Sparse & Sliding-Window Attention", section 3), on one batch and two heads
# (same unit layout as the workload: head pairs for even groups, head pairs
# with their own KV heads for group 1 at d = 64). Query tiles: all of them,
# or a spread sample plus the edges at 128K.
FULL_SIZE = [
    ("swa", 8192, 4096, 0, 2, 1, 128, None),           # Mistral-style
    ("strided", 16384, 128, 128, 2, 2, 64, None),      # local + strided
    ("global", 16384, 512, 64, 2, 2, 64, None),        # window + global tokens
    ("swa", 131072, 1024, 0, 2, 1, 128, 48),           # Gemma-style, 128K
]


@pytest.mark.parametrize("kind,N,W,S,Hq,Hkv,d,nsample", FULL_SIZE)
def test_visited_tiles_bit_exact_at_workload_sizes(orc, kind, N, W, S, Hq, Hkv, d, nsample):
    q, k, v = attn_inputs(1, Hq, Hkv, N, d, seed=11)
    qd, kd, vd = gpu(q, k, v)
    del q, k, v
    out, cells, tiles, ntiles = swa.prefill_debug(KIND[kind], qd, kd, vd, W, S, tiles_cap=64)
    assert swa.last_device_error() == swa.OK
    cells, tiles, ntiles = cells.cpu(), tiles.cpu(), ntiles.cpu()
    nq = (N + 127) // 128
    qts = range(nq)
    if nsample:
        rng = np.random.default_rng(5)
        qts = sorted(set(rng.integers(0, nq, nsample).tolist()) | {0, 1, 7, 8, 9, nq // 2, nq - 2, nq - 1})
    total = 0
    for qt in qts:
        lst, c = orc.schedule_qtile(kind, N, W, S, 128, 128, qt)
        assert len(lst) <= 64
        for h in range(Hq):
            assert int(ntiles[0, h, qt]) == len(lst), (h, qt)
            assert tiles[0, h, qt, :len(lst)].tolist() == lst, (h, qt)
            assert int(cells[0, h, qt]) == c, (h, qt)
        total += c
    if not nsample:  # every query tile: the counts add up to ||M||_0
        assert total == swa.count_nonmasked(KIND[kind], N, W, S)
        assert int(cells.sum()) == Hq * total
    assert torch.isfinite(out.float()).all()


def test_timeout_is_reported_and_context_survives(orc):
    q, k, v = attn_inputs(1, 2, 2, 256, 64, seed=1)
    qd, kd, vd = gpu(q, k, v)
    swa.prefill_debug(swa.MASK_WINDOW, qd, kd, vd, 64, inject_timeout=True)
    assert swa.last_device_error() == swa.ERR_TIMEOUT
    assert swa.last_device_error() == swa.OK  # cleared
    out = swa.swa_attn_fwd(qd, kd, vd, 64)
    assert swa.last_device_error() == swa.OK
    compare(out, orc.attention("swa", q, k, v, W=64, scale=0.125), "after timeout")


# ---------------------------------------------------------- differential --

@pytest.mark.parametrize("N,W,dv,Hq,Hkv", [(256, None, 128, 2, 2), (300, 70, 128, 2, 1), (513, None, 64, 4, 2)])
def test_diff_small_full(orc, N, W, dv, Hq, Hkv):
    q1, k1, q2, k2, v = diff_inputs(1, Hq, Hkv, N, 64, dv, seed=3)
    lam = torch.tensor([0.8, 0.5, 0.2, 1.0][:Hq], dtype=torch.float32)
    out = swa.diff_attn_fwd(*gpu(q1, k1, q2, k2, v), lam.cuda(), window=W, scale=0.125)
    assert swa.last_device_error() == swa.OK
    ref = orc.diff_attention(q1, k1, q2, k2, v, lam, W=W, scale=0.125)
    compare(out, ref, "diff")


@pytest.mark.parametrize("case", ["lambda0", "same_maps", "window_ragged"])
def test_diff_degenerate_cases(orc, case):
    """Differential attention where it reduces to something plainer: lambda = 0
    is the causal attention of (Q1, K1, V); Q2 = Q1, K2 = K1 gives (1 - lambda)
    times it ("Attention Variants -- Sliding Window, Sparse, Differential",
    The Problem: one map subtracted from the other); and a window with a
    ragged last tile."""
    N, Hq, Hkv, dv = (200, 2, 2, 128) if case != "window_ragged" else (333, 4, 2, 64)
    q1, k1, q2, k2, v = diff_inputs(1, Hq, Hkv, N, 64, dv, seed=17)
    if case == "same_maps":
        q2, k2 = q1.clone(), k1.clone()
    lam = torch.zeros(Hq) if case == "lambda0" else torch.tensor([0.25, 0.8, 0.5, 0.1][:Hq])
    W = 50 if case == "window_ragged" else None
    out = swa.diff_attn_fwd(*gpu(q1, k1, q2, k2, v), lam.float().cuda(), window=W, scale=0.125)
    assert swa.last_device_error() == swa.OK
    ref = orc.diff_attention(q1, k1, q2, k2, v, lam, W=W, scale=0.125)
    compare(out, ref, f"diff {case}")
    if case == "lambda0":  # equal to the plain causal attention of (Q1, K1, V), within the same bar
        plain = orc.attention("causal", q1, k1, v, scale=0.125)
        compare(out, plain, "diff lambda 0 vs causal attention")
    if case == "same_maps":
        plain = orc.attention("causal", q1, k1, v, scale=0.125)
        compare(out, plain * (1 - lam.numpy().astype(np.float64))[None, :, None, None], "diff same maps")


# ---------------------------------------------------------------- decode --

@pytest.mark.parametrize("B,Hq,Hkv,d,W,pos0,T", [(2, 4, 2, 128, 64, 3, 70), (3, 16, 8, 128, 1024, 131072, 3),
                                                  (2, 2, 2, 64, 100, 0, 5), (1, 8, 1, 128, 256, 250, 10),
                                                  (1, 2, 1, 128, 4096, 4090, 8),   # one group, long window
                                                  (5, 8, 8, 64, 1500, 1400, 3),   # last split ragged
                                                  (40, 8, 8, 128, 2048, 5000, 2)])  # many groups, 2048 slots
def test_decode_steps_vs_oracle(orc, B, Hq, Hkv, d, W, pos0, T):
    q, k_new, v_new, k_cache, v_cache = decode_inputs(T, B, Hq, Hkv, d, W, seed=5)
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    ref, kc_ref, vc_ref = orc.decode(q, k_new, v_new, k_cache, v_cache, pos)
    kc, vc = gpu(k_cache, v_cache)
    posd = torch.from_numpy(pos).cuda()
    qd, knd, vnd = gpu(q, k_new, v_new)
    outs = []
    for t in range(T):
        outs.append(swa.swa_decode_step(qd[t], knd[t], vnd[t], kc, vc, posd[t]))
    assert swa.last_device_error() == swa.OK
    compare(torch.stack(outs), ref, "decode")
    assert np.array_equal(kc.float().cpu().numpy(), kc_ref)
    assert np.array_equal(vc.float().cpu().numpy(), vc_ref)


@pytest.mark.parametrize("B,Hq,Hkv,d,n_sink,W,pos0,T", [(2, 4, 2, 128, 4, 64, 0, 70), (2, 4, 2, 128, 4, 64, 200, 3),
                                                         (3, 16, 8, 128, 4, 1024, 131072, 2),
                                                         (1, 8, 1, 64, 2, 100, 5, 20), (2, 2, 2, 128, 1, 1, 0, 6)])
def test_sink_decode_vs_oracle(orc, B, Hq, Hkv, d, n_sink, W, pos0, T):
    q, k_new, v_new, k_cache, v_cache = decode_inputs(T, B, Hq, Hkv, d, n_sink + W, seed=9)
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    ref, kc_ref, vc_ref = orc.sink_decode(q, k_new, v_new, k_cache, v_cache, pos, n_sink)
    kc, vc = gpu(k_cache, v_cache)
    posd = torch.from_numpy(pos).cuda()
    qd, knd, vnd = gpu(q, k_new, v_new)
    outs = [swa.swa_sink_decode_step(qd[t], knd[t], vnd[t], kc, vc, posd[t], n_sink) for t in range(T)]
    assert swa.last_device_error() == swa.OK
    compare(torch.stack(outs), ref, "sink decode")
    assert np.array_equal(kc.float().cpu().numpy(), kc_ref)
    assert np.array_equal(vc.float().cpu().numpy(), vc_ref)


def run_diff_decode(orc, B, Hq, Hkv, W, pos0, T, seed, lam=None):
    dk, dv = 64, 128
    ins = diff_decode_inputs(T, B, Hq, Hkv, dk, dv, W, seed=seed)
    q1, q2, k1n, k2n, vn, k1c, k2c, vc = ins
    # lambda in the range the method uses (0 < lambda < 1): with it the
    # outputs stay below 4, where bf16's half-ulp (1.56e-2 from 4 up) would
    # exceed the bar by itself; the oracle's pins cover negative lambda
    lam = torch.linspace(0.2, 0.8, Hq) if lam is None else lam
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    ref, k1r, k2r, vr = orc.diff_decode(q1, q2, k1n, k2n, vn, k1c, k2c, vc, lam, pos)
    k1d, k2d, vd = gpu(k1c, k2c, vc)
    q1d, q2d, k1nd, k2nd, vnd = gpu(q1, q2, k1n, k2n, vn)
    posd, lamd = torch.from_numpy(pos).cuda(), lam.float().cuda()
    outs = [swa.swa_diff_decode_step(q1d[t], q2d[t], k1nd[t], k2nd[t], vnd[t], k1d, k2d, vd, posd[t], lamd)
            for t in range(T)]
    assert swa.last_device_error() == swa.OK
    return torch.stack(outs), ref, (k1d, k2d, vd), (k1r, k2r, vr)


@pytest.mark.parametrize("B,Hq,Hkv,W,pos0,T", [(2, 4, 2, 64, 0, 70), (3, 16, 8, 4096, 4096, 2), (1, 8, 1, 100, 5, 20),
                                               (2, 2, 2, 1, 0, 4), (5, 4, 1, 1500, 1400, 3), (2, 16, 16, 300, 900, 2)])
def test_diff_decode_vs_oracle(orc, B, Hq, Hkv, W, pos0, T):
    """Both maps over the rolling window, V read once: early positions,
    wrap-around, GQA groups 1-8, W = 1 and a ragged last split."""
    out, ref, caches, caches_ref = run_diff_decode(orc, B, Hq, Hkv, W, pos0, T, seed=31)
    compare(out, ref, "diff decode")
    for c, r in zip(caches, caches_ref):  # each new token stored in slot pos % W, nothing else touched
        assert np.array_equal(c.float().cpu().numpy(), r)


# ------------------------------------------------------ workload sizes ----

def sampled_rows(B, H, N, n, seed):
    rng = np.random.default_rng(seed)
    i = np.concatenate([rng.integers(0, N, n), [0, 1, 127, 128, N - 1, N - 2]])
    bh = rng.integers(0, B * H, i.size)
    return np.unique(bh.astype(np.int64) * N + i)


@pytest.mark.parametrize("name", ["mistral_swa_prefill", "local_strided_prefill", "gemma_swa_prefill",
                                  "longformer_global_prefill", "longformer_dilated_prefill"])
def test_workload_sampled_rows(orc, name):
    w = WORKLOADS[name]
    q, k, v = attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=0)
    out = run_prefill(w.kind, q, k, v, w.W, w.S).reshape(-1, w.d)
    rows = sampled_rows(w.B, w.Hq, w.N, 1500, 1)
    ref = orc.attention(w.kind, q, k, v, W=w.W, S=w.S, scale=w.scale, rows=rows)
    compare(out[torch.from_numpy(rows).cuda()], ref, name)
    assert torch.isfinite(out.float()).all()


def test_diff_workload_sampled_rows(orc):
    w = WORKLOADS["diff_causal"]
    q1, k1, q2, k2, v = diff_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, seed=0)
    lam = torch.full((w.Hq,), w.lam, dtype=torch.float32)
    out = swa.diff_attn_fwd(*gpu(q1, k1, q2, k2, v), lam.cuda(), window=w.W, scale=w.scale)
    assert swa.last_device_error() == swa.OK
    rows = sampled_rows(w.B, w.Hq, w.N, 1500, 2)
    ref = orc.diff_attention(q1, k1, q2, k2, v, lam, W=w.W, scale=w.scale, rows=rows)
    compare(out.reshape(-1, w.dv)[torch.from_numpy(rows).cuda()], ref, "diff workload")


def test_diff_decode_workload_first_step(orc):
    w = WORKLOADS["diff_gqa_decode"]
    lam = torch.full((w.Hq,), w.lam)
    out, ref, _, _ = run_diff_decode(orc, w.B, w.Hq, w.Hkv, w.W, w.pos0, 1, seed=0, lam=lam)
    compare(out, ref, "diff decode workload")


def test_decode_workload_first_steps(orc):
    w = WORKLOADS["gemma_swa_decode"]
    T = 3
    q, k_new, v_new, k_cache, v_cache = decode_inputs(T, w.B, w.Hq, w.Hkv, w.d, w.W, seed=0)
    pos = np.array([[w.pos0 + t] * w.B for t in range(T)], dtype=np.int32)
    ref, _, _ = orc.decode(q, k_new, v_new, k_cache, v_cache, pos)
    kc, vc = gpu(k_cache, v_cache)
    posd = torch.from_numpy(pos).cuda()
    qd, knd, vnd = gpu(q, k_new, v_new)
    outs = [swa.swa_decode_step(qd[t], knd[t], vnd[t], kc, vc, posd[t]) for t in range(T)]
    assert swa.last_device_error() == swa.OK
    compare(torch.stack(outs), ref, "decode workload")


def test_dilated_lse_at_original_rows(orc):
    """The per-class launches write the log-sum-exp at each row's own index."""
    q, k, v = attn_inputs(1, 2, 2, 500, 64, seed=77)
    out, lse = run_prefill("dilated", q, k, v, 40, 3, lse=True)
    ref, ref_lse = orc.attention("dilated", q, k, v, W=40, S=3, scale=0.125, with_lse=True)
    compare(out, ref, "dilated with lse")
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 2e-3
