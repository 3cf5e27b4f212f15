"""The backward of the window attention (swa_attn_bwd) against the oracle's
fp64 chain rule, on the same seeded inputs. The kernel uses its own forward
output and log-sum-exp and rounds P and dS to bf16 before the products that
consume them (as the forward rounds P), so its error grows with the number
of attended keys; the bar is relative to each gradient's largest entry."""
import math

import numpy as np
import pytest
import torch

import differential_attention_swa_b200 as swa
from differential_attention_swa_b200.inputs import attn_inputs, randn_bf16

pytestmark = pytest.mark.gpu

# bf16 products (P, dS) and bf16 outputs: each term carries a relative
# error of about 2^-9; the sums stay within ~1 % of the largest entry
REL_MAX = 2e-2
REL_MEAN = 2e-3
# where a gradient is exactly zero (window 1: dS = P (dP - D) = 0 because
# D = dO . O = dO . v_i = dP), only rounding residue remains
ABS_FLOOR = 1e-4


def compare_grad(got, want, what):
    got = got.float().cpu().numpy().astype(np.float64).reshape(want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    scale = max(np.abs(want).max(), ABS_FLOOR / REL_MAX)
    diff = np.abs(got - want)
    assert diff.max() <= REL_MAX * scale and diff.mean() <= REL_MEAN * scale, \
        f"{what}: max {diff.max():.3e} mean {diff.mean():.3e} (largest entry {scale:.3e})"
    return diff.max() / scale


def run(B, Hq, Hkv, N, d, W, seed, S=0):
    q, k, v = attn_inputs(B, Hq, Hkv, N, d, seed=seed)
    d_o = randn_bf16((B, Hq, N, d), seed + 10)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, d_o))
    if S:
        o, lse = swa.strided_attn_fwd(qd, kd, vd, W, S, return_lse=True)
    else:
        o, lse = swa.swa_attn_fwd(qd, kd, vd, W, return_lse=True)
    dq, dk, dv = swa.swa_attn_bwd(qd, kd, vd, o, dod, lse, W, stride=S)
    torch.cuda.synchronize()
    assert swa.last_device_error() == swa.OK
    return (q, k, v, d_o), (dq, dk, dv)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W", [
    (1, 2, 2, 256, 64, 64),      # two tiles, window of half a tile
    (1, 4, 2, 300, 128, 100),    # ragged tail, GQA group 2
    (2, 2, 1, 200, 64, 5000),    # window beyond N: causal, group 2
    (1, 2, 2, 129, 128, 1),      # window 1, one row in the last tile
    (1, 6, 2, 257, 64, 130),     # group 3, window just over a tile
    (1, 8, 1, 384, 128, 256),    # group 8, three tiles
])
def test_backward_vs_oracle(orc, B, Hq, Hkv, N, d, W):
    (q, k, v, d_o), (dq, dk, dv) = run(B, Hq, Hkv, N, d, W, seed=N + W)
    rq, rk, rv = orc.attention_bwd("swa", q, k, v, d_o, W=W, scale=1 / math.sqrt(d))
    compare_grad(dq, rq, "dq")
    compare_grad(dk, rk, "dk")
    compare_grad(dv, rv, "dv")


def test_backward_sampled_rows_at_size(orc):
    """A Mistral-like head shape at N = 4096 (W = 1024, GQA group 4): sampled
    rows of dQ and of dK/dV, each from the oracle's per-row chain rule."""
    B, Hq, Hkv, N, d, W = 1, 8, 2, 4096, 128, 1024
    (q, k, v, d_o), (dq, dk, dv) = run(B, Hq, Hkv, N, d, W, seed=3)
    rng = np.random.default_rng(4)
    qr = np.unique(np.concatenate([rng.integers(0, B * Hq * N, 40), [0, N - 1, 128, 2 * N + 1023]]))
    kr = np.unique(np.concatenate([rng.integers(0, B * Hkv * N, 6), [0, N - 1, N + 127]]))
    rq, rk, rv = orc.attention_bwd("swa", q, k, v, d_o, W=W, scale=1 / math.sqrt(d), dq_rows=qr, dkv_rows=kr)
    compare_grad(dq.reshape(-1, d)[torch.from_numpy(qr).cuda()], rq, "dq rows")
    compare_grad(dk.reshape(-1, d)[torch.from_numpy(kr).cuda()], rk, "dk rows")
    compare_grad(dv.reshape(-1, d)[torch.from_numpy(kr).cuda()], rv, "dv rows")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W,S", [
    (1, 2, 2, 300, 64, 17, 5),      # N not a multiple of S, several stride tiles per row block
    (1, 4, 2, 1000, 128, 64, 7),    # group 2, stride keys spread over the sequence
    (1, 2, 2, 256, 64, 3, 1),       # stride 1: every key (full causal)
    (1, 2, 2, 333, 64, 20, 400),    # stride beyond N: window + key 0
    (1, 3, 1, 700, 64, 1, 3),       # window 1 + stride, group 3
    (1, 2, 2, 16384, 64, 128, 128), # the local+strided workload's mask at one batch and two heads
])
def test_strided_backward_vs_oracle(orc, B, Hq, Hkv, N, d, W, S):
    (q, k, v, d_o), (dq, dk, dv) = run(B, Hq, Hkv, N, d, W, seed=N + S, S=S)
    if N <= 1024:
        rq, rk, rv = orc.attention_bwd("strided", q, k, v, d_o, W=W, S=S, scale=1 / math.sqrt(d))
        compare_grad(dq, rq, "dq")
        compare_grad(dk, rk, "dk")
        compare_grad(dv, rv, "dv")
    else:  # sampled rows, stride keys among them
        rng = np.random.default_rng(5)
        qr = np.unique(np.concatenate([rng.integers(0, B * Hq * N, 30), [0, N - 1, 128 * 5 + 3]]))
        kr = np.unique(np.concatenate([rng.integers(0, B * Hkv * N, 4), [0, S, 5 * S, N - 1]]))
        rq, rk, rv = orc.attention_bwd("strided", q, k, v, d_o, W=W, S=S, scale=1 / math.sqrt(d), dq_rows=qr,
                                       dkv_rows=kr)
        compare_grad(dq.reshape(-1, d)[torch.from_numpy(qr).cuda()], rq, "dq rows")
        compare_grad(dk.reshape(-1, d)[torch.from_numpy(kr).cuda()], rk, "dk rows")
        compare_grad(dv.reshape(-1, d)[torch.from_numpy(kr).cuda()], rv, "dv rows")


def _sampled_rows_check(orc, kind, B, Hq, Hkv, N, d, W, S, seed):
    (q, k, v, d_o), (dq, dk, dv) = run(B, Hq, Hkv, N, d, W, seed=seed, S=S)
    rng = np.random.default_rng(seed)
    # dK/dV rows from every (batch, KV head): the first, last and a few inner
    # keys of each (stride keys among them), plus random ones
    keys = [0, 127, 133, 2 * 128 + 64, N // 2 + 77, N - 1] + ([S, 7 * S] if S else [])
    kr = np.unique(np.concatenate([[y * N + key for y in range(B * Hkv) for key in keys],
                                   rng.integers(0, B * Hkv * N, 24)]))
    qr = np.unique(np.concatenate([rng.integers(0, B * Hq * N, 24), [0, N - 1, (B * Hq - 1) * N + 5]]))
    rq, rk, rv = orc.attention_bwd(kind, q, k, v, d_o, W=W, S=S, scale=1 / math.sqrt(d), dq_rows=qr, dkv_rows=kr)
    compare_grad(dq.reshape(-1, d)[torch.from_numpy(qr).cuda()], rq, "dq rows")
    compare_grad(dk.reshape(-1, d)[torch.from_numpy(kr).cuda()], rk, "dk rows")
    compare_grad(dv.reshape(-1, d)[torch.from_numpy(kr).cuda()], rv, "dv rows")


def test_backward_multi_tile_sets_reused(orc):
    """At d = 64 the dK/dV kernel runs several key tiles per CTA (one CTA per
    SM, two sets of fixed K/V tiles and of accumulators): 2 x 4 KV heads x 64
    key tiles = 512 tiles give every CTA three or four, so each set is
    refilled and its accumulators overwritten after an epilogue. Window 96
    (cut tiles at both edges), GQA group 2."""
    _sampled_rows_check(orc, "swa", 2, 8, 4, 8192, 64, 96, 0, seed=21)


def test_strided_backward_multi_tile_sets_reused(orc):
    """The same multi-tile dK/dV path with the local + strided mask: the
    window pass's 512 tiles add the stride pass's fp32 partials to their
    stride keys (every 64th key) before rounding."""
    _sampled_rows_check(orc, "strided", 2, 8, 4, 8192, 64, 64, 64, seed=22)


def test_backward_multi_tile_odd_step_counts(orc):
    """Group 1 and W = 300: a key tile has one to four query-tile steps, so
    the stage ring and the half-step barriers run on across tiles at odd as
    well as even alignments (2 x 8 KV heads x 32 key tiles = 512 tiles)."""
    _sampled_rows_check(orc, "swa", 2, 8, 8, 4096, 64, 300, 0, seed=23)
