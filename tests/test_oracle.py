"""Pins for the fp64 oracle: what the pages print or fix, closed forms,
textbook special cases (torch's fp64 scaled_dot_product_attention), and
brute force on tiny inputs. Each test would fail on a plausible slip in the
oracle: a dropped term, a wrong sign, an off-by-one window, a swapped
operand, a wrong GQA map."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from conftest import read_grid, read_numbers
from differential_attention_swa_b200.inputs import attn_inputs, diff_inputs, randn_bf16


def grid_of(M):
    return ["".join("x" if v == 0.0 else "." for v in row) for row in M]


# ------------------------------------------------------------------ masks --

def test_swa_mask_8_4_matches_hand_derived_grid(orc):
    M = orc.swa_mask(8, 4)
    assert grid_of(M) == read_grid("swa_mask_n8_w4.txt")
    assert set(np.unique(M).tolist()) == {0.0, -math.inf}
    assert orc.count_nonmasked(M) == 26


def test_strided_mask_8_2_3_matches_hand_derived_grid(orc):
    M = orc.strided_mask(8, 2, 3)
    assert grid_of(M) == read_grid("strided_mask_n8_w2_s3.txt")
    assert orc.count_nonmasked(M) == 24


def test_causal_8_count(orc):
    assert orc.count_nonmasked(orc.causal_mask(8)) == 36


@pytest.mark.parametrize("n", [1, 2, 7, 33])
def test_window_at_least_n_is_full_causal(orc, n):
    C = orc.causal_mask(n)
    for W in (n, n + 1, 10 * n):
        assert np.array_equal(orc.swa_mask(n, W), C)
        for S in (1, 2, 5, n + 3):
            assert np.array_equal(orc.strided_mask(n, W, S), C)


def test_brute_force_masks_all_small(orc):
    """The cheatsheet's loops against the lesson's predicate form
    M_ij = 1[i - w < j <= i] (and its OR with j % S == 0, j <= i), for every
    n <= 24, every window and every stride."""
    for n in range(1, 25):
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        for W in range(1, n + 2):
            band = (ii - W < jj) & (jj <= ii)
            assert np.array_equal(orc.swa_mask(n, W) == 0.0, band), (n, W)
            for S in range(1, n + 2):
                want = band | ((jj % S == 0) & (jj <= ii))
                assert np.array_equal(orc.strided_mask(n, W, S) == 0.0, want), (n, W, S)


def band_closed(N, W):
    return N * (N + 1) // 2 if W >= N else N * W - W * (W - 1) // 2


def strided_closed(N, W, S):
    # sum over rows of min(i+1, W) window keys plus the multiples of S below lo_i
    i = np.arange(N, dtype=np.int64)
    lo = np.maximum(0, i - W + 1)
    return int(np.minimum(i + 1, W).sum() + ((lo + S - 1) // S).sum())


@pytest.mark.parametrize("N,W,S,want", [
    (256, 64, 0, 14368), (256, 16, 8, 7696), (8192, 4096, 0, 25167872),
    (16384, 128, 128, 3129408), (131072, 1024, 0, 133693952), (4096, 4096, 0, 8390656)])
def test_closed_form_counts(N, W, S, want):
    got = strided_closed(N, W, S) if S else band_closed(N, W)
    assert got == want


@pytest.mark.parametrize("N,W,S", [(256, 64, 0), (256, 16, 8), (300, 17, 5), (8192, 4096, 0),
                                   (1000, 1, 3), (513, 600, 7)])
def test_explicit_count_matches_closed_form(orc, N, W, S):
    if N <= 1024:
        M = orc.strided_mask(N, W, S) if S else orc.swa_mask(N, W)
        got = orc.count_nonmasked(M)
    else:  # row by row: the full matrix is 8 bytes per cell
        kind = "strided" if S else "swa"
        got = sum(orc.count_nonmasked(orc.mask_row(kind, N, i, W, S)) for i in range(N))
    want = strided_closed(N, W, S) if S else band_closed(N, W)
    assert got == want


def test_stride_at_least_n_adds_only_key_zero(orc):
    n, W = 40, 6
    for S in (n, n + 1, 100):
        want = orc.swa_mask(n, W).copy()
        want[:, 0] = 0.0
        assert np.array_equal(orc.strided_mask(n, W, S), want)


# ----------------------------------------------------- softmax & rows ------

def test_rows_sum_to_one_and_masked_weights_are_zero(orc):
    rng = np.random.default_rng(0)
    n, d = 37, 8
    K, V = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    M = orc.strided_mask(n, 5, 4)
    for i in range(n):
        out, w = orc.attention_row(rng.normal(size=d), K, V, M[i], 1 / math.sqrt(d))
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(w[M[i] != 0.0] == 0.0)
        assert np.all(w[M[i] == 0.0] > 0.0)
        assert np.allclose(out, w @ V, rtol=0, atol=1e-12)


def test_attention_row_matches_page_example_shape(orc):
    """The instagit snippet: n = 8, d = 8, rng seed 0, SWA window 4, the last
    token's row. Checked against a softmax written out with numpy."""
    rng = np.random.default_rng(0)
    n, d = 8, 8
    q = rng.normal(size=d)
    K = rng.normal(size=(n, d))
    V = rng.normal(size=(n, d))
    row = orc.swa_mask(n, 4)[7]
    out, w = orc.attention_row(q, K, V, row, 1.0 / math.sqrt(d))
    s = K[4:8] @ q / math.sqrt(d)
    e = np.exp(s - s.max())
    want_w = np.zeros(n)
    want_w[4:8] = e / e.sum()
    assert np.allclose(w, want_w, rtol=0, atol=1e-14)
    assert np.allclose(out, want_w @ V, rtol=0, atol=1e-13)


@pytest.mark.parametrize("tile", [1, 3, 4, 37])
def test_tiled_softmax_equals_full_softmax(orc, tile):
    rng = np.random.default_rng(1)
    n, dk, dv = 37, 8, 5
    K, V = rng.normal(size=(n, dk)) * 3, rng.normal(size=(n, dv))
    M = orc.strided_mask(n, 6, 5)
    for i in range(n):
        q = rng.normal(size=dk)
        full, _ = orc.attention_row(q, K, V, M[i], 0.7)
        tiled = orc.tiled_softmax_dot(q, K, V, M[i], 0.7, tile)
        assert np.allclose(tiled, full, rtol=1e-12, atol=1e-12)


def test_row_zero_is_v0_and_window_one_is_identity(orc):
    q, k, v = attn_inputs(1, 2, 2, 50, 16, seed=3)
    out = orc.attention("swa", q, k, v, W=8)
    assert np.array_equal(out[0, :, 0, :], v[0, :, 0, :].float().numpy().astype(np.float64))
    out1 = orc.attention("swa", q, k, v, W=1)
    assert np.array_equal(out1, v.float().numpy().astype(np.float64))
    out1s = orc.attention("strided", q, k, v, W=1, S=1000)
    # window 1 plus key 0: row i mixes only v_0 and v_i
    assert np.array_equal(out1s[:, :, 0], out1[:, :, 0])


# ---------------------------------------------- textbook library routine ---

def sdpa_ref(q, k, v, allowed, scale):
    """torch's fp64 scaled_dot_product_attention with a boolean mask,
    KV heads repeated to the query heads (consecutive grouping)."""
    G = q.shape[1] // k.shape[1]
    q64, k64, v64 = (t.double() for t in (q, k, v))
    k64 = k64.repeat_interleave(G, dim=1)
    v64 = v64.repeat_interleave(G, dim=1)
    return F.scaled_dot_product_attention(q64, k64, v64, attn_mask=torch.from_numpy(allowed),
                                          scale=scale).numpy()


@pytest.mark.parametrize("kind,B,Hq,Hkv,N,d,dv,W,S", [
    ("swa", 1, 2, 2, 64, 16, 16, 9, 0),
    ("swa", 2, 4, 2, 130, 32, 32, 40, 0),
    ("swa", 1, 6, 2, 77, 16, 24, 1000, 0),
    ("strided", 1, 2, 1, 150, 16, 16, 7, 11),
    ("strided", 2, 4, 4, 97, 8, 8, 3, 1),
    ("causal", 1, 3, 1, 55, 16, 16, 0, 0),
    ("global", 1, 4, 2, 140, 16, 16, 9, 5),
    ("global", 2, 2, 2, 70, 8, 24, 3, 40),
])
def test_attention_matches_torch_sdpa_fp64(orc, kind, B, Hq, Hkv, N, d, dv, W, S):
    q, k, v = attn_inputs(B, Hq, Hkv, N, d, dv, seed=11)
    scale = 1.0 / math.sqrt(d)
    out, lse = orc.attention(kind, q, k, v, W=W, S=S, scale=scale, with_lse=True)
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    if kind == "causal":
        allowed = jj <= ii
    else:
        allowed = (ii - W < jj) & (jj <= ii)
        if kind == "strided":
            allowed |= (jj % S == 0) & (jj <= ii)
        if kind == "global":  # S carries the number of global tokens
            allowed |= ((jj < S) | (ii < S)) & (jj <= ii)
    ref = sdpa_ref(q, k, v, allowed, scale)
    assert np.abs(out - ref).max() < 1e-12
    # natural-log sum of exp over the attended scores
    G = Hq // Hkv
    s = np.einsum("bhid,bhjd->bhij", q.double().numpy(),
                  k.double().repeat_interleave(G, dim=1).numpy()) * scale
    s = np.where(allowed, s, -np.inf)
    mx = s.max(-1, keepdims=True)
    want_lse = (mx + np.log(np.exp(s - mx).sum(-1, keepdims=True)))[..., 0]
    assert np.abs(lse - want_lse).max() < 1e-12


def test_attention_row_subset_matches_full(orc):
    q, k, v = attn_inputs(2, 4, 2, 90, 16, seed=5)
    full = orc.attention("strided", q, k, v, W=10, S=7)
    rows = np.array([0, 5, 89, 90, 179, 4 * 90 + 33, 8 * 90 - 1])
    part = orc.attention("strided", q, k, v, W=10, S=7, rows=rows)
    assert np.array_equal(part, full.reshape(-1, 16)[rows])
    with pytest.raises(ValueError):
        orc.attention("strided", q, k, v, W=10, S=7, rows=[2 * 4 * 90])


# ------------------------------------------------------------ differential --

def test_diff_lambda_zero_is_plain_attention(orc):
    q1, k1, q2, k2, v = diff_inputs(1, 2, 2, 70, 16, 24, seed=2)
    lam = np.zeros(2, dtype=np.float32)
    out = orc.diff_attention(q1, k1, q2, k2, v, lam)
    plain = orc.attention("causal", q1, k1, v, scale=1 / 4)
    assert np.abs(out - plain).max() < 1e-13


def test_diff_same_maps_is_one_minus_lambda(orc):
    q1, k1, _, _, v = diff_inputs(1, 2, 2, 70, 16, 24, seed=2)
    lam = np.array([0.8, 0.3], dtype=np.float32)
    out = orc.diff_attention(q1, k1, q1, k1, v, lam)
    plain = orc.attention("causal", q1, k1, v, scale=1 / 4)
    want = plain * (1.0 - lam.astype(np.float64))[None, :, None, None]
    assert np.abs(out - want).max() < 1e-12


@pytest.mark.parametrize("W", [None, 13])
def test_diff_matches_sdpa_difference(orc, W):
    B, Hq, Hkv, N, dqk, dv = 1, 4, 2, 66, 16, 32
    q1, k1, q2, k2, v = diff_inputs(B, Hq, Hkv, N, dqk, dv, seed=9)
    lam = np.array([0.8, 0.5, 0.1, 1.2], dtype=np.float32)
    out = orc.diff_attention(q1, k1, q2, k2, v, lam, W=W, scale=0.125)
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    Wv = N if W is None else W
    allowed = (ii - Wv < jj) & (jj <= ii)
    a1 = sdpa_ref(q1, k1, v, allowed, 0.125)
    a2 = sdpa_ref(q2, k2, v, allowed, 0.125)
    want = a1 - lam.astype(np.float64)[None, :, None, None] * a2
    assert np.abs(out - want).max() < 1e-12


# ----------------------------------------------------------------- decode --

@pytest.mark.parametrize("W,pos0,T", [(8, 3, 12), (8, 20, 9), (5, 0, 7), (16, 16, 3)])
def test_decode_equals_window_softmax_over_history(orc, W, pos0, T):
    """Step t attends exactly the W most recent positions of the history,
    whatever slot order the rolling buffer holds them in, across wrap-around
    and before the buffer first fills (pos < W - 1)."""
    B, Hq, Hkv, d = 2, 4, 2, 16
    L = pos0 + T
    Kh = randn_bf16((B, Hkv, L, d), 1).float()
    Vh = randn_bf16((B, Hkv, L, d), 2).float()
    q = randn_bf16((T, B, Hq, d), 3).float()
    kc = torch.full((B, Hkv, W, d), float("nan"))  # unfilled slots must never be read
    vc = torch.full((B, Hkv, W, d), float("nan"))
    for p in range(max(0, pos0 - W), pos0):
        kc[:, :, p % W] = Kh[:, :, p]
        vc[:, :, p % W] = Vh[:, :, p]
    k_new = Kh[:, :, pos0:].permute(2, 0, 1, 3).contiguous()
    v_new = Vh[:, :, pos0:].permute(2, 0, 1, 3).contiguous()
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    out, kc2, vc2 = orc.decode(q, k_new, v_new, kc, vc, pos)
    G = Hq // Hkv
    for t in range(T):
        p = pos0 + t
        lo = max(0, p - W + 1)
        Kw = Kh[:, :, lo:p + 1].double().repeat_interleave(G, dim=1)
        Vw = Vh[:, :, lo:p + 1].double().repeat_interleave(G, dim=1)
        ref = F.scaled_dot_product_attention(q[t].double()[:, :, None], Kw, Vw, scale=1 / 4)[:, :, 0]
        assert np.abs(out[t] - ref.numpy()).max() < 1e-12
    # the cache afterwards holds the last W positions at slot p % W
    last = pos0 + T - 1
    for p in range(max(0, last - W + 1), last + 1):
        assert np.array_equal(kc2[:, :, p % W], Kh[:, :, p].numpy())


# --------------------------------------------------------------- schedule --

def tiles_touched_from_mask(allowed, band_allowed, Bq, Bk, S, global_keys=False):
    """Block-reduce boolean masks: which key tiles / stride tiles hold an
    attended cell for each query tile."""
    N = allowed.shape[0]
    out = []
    for qt in range((N + Bq - 1) // Bq):
        rows = slice(qt * Bq, min(N, qt * Bq + Bq))
        a, b = allowed[rows], band_allowed[rows]
        extra = a & ~b
        unit = 1 if global_keys else S  # global keys are tiled as they are; stride keys m*S compacted
        st = sorted({(j // unit) // Bk for j in np.nonzero(extra.any(0))[0]}) if S else []
        kt = sorted({j // Bk for j in np.nonzero(b.any(0))[0]})
        out.append(([0x40000000 | t for t in st] + kt, int(a.sum())))
    return out


@pytest.mark.parametrize("kind,N,W,S,Bq,Bk", [
    ("swa", 256, 64, 0, 128, 128), ("strided", 256, 16, 8, 128, 128), ("swa", 300, 50, 0, 64, 32),
    ("strided", 517, 33, 5, 128, 16), ("swa", 100, 1000, 0, 32, 32), ("strided", 130, 1, 1, 64, 64),
    ("causal", 200, 0, 0, 64, 32), ("global", 256, 16, 8, 128, 128), ("global", 517, 33, 200, 128, 16),
    ("global", 300, 64, 300, 64, 32), ("global", 130, 1, 1, 64, 64)])
def test_schedule_matches_block_reduction(orc, kind, N, W, S, Bq, Bk):
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    if kind == "causal":
        allowed = jj <= ii
        band = allowed
    else:
        band = (ii - W < jj) & (jj <= ii)
        allowed = band
        if kind == "strided":
            allowed = band | ((jj % S == 0) & (jj <= ii))
        if kind == "global":
            allowed = band | (((jj < S) | (ii < S)) & (jj <= ii))
    lists, cells = orc.schedule(kind, N, W, S, Bq, Bk)
    want = tiles_touched_from_mask(allowed, band, Bq, Bk, S, global_keys=(kind == "global"))
    assert lists == [w[0] for w in want]
    assert cells == [w[1] for w in want]
    assert sum(cells) == int(allowed.sum())


def test_schedule_tile_totals_at_workload_sizes(orc):
    """Band tiles per (b, h) at 128 x 128 tiles; sampled tiles checked
    against the explicit mask, totals against the interval count."""
    def total(N, W, S):
        t = 0
        for qt in range((N + 127) // 128):
            r0, r1 = qt * 128, min(N - 1, qt * 128 + 127)
            t += r1 // 128 - max(0, r0 - W + 1) // 128 + 1
            if S:
                m = (max(0, r1 - W + 1) + S - 1) // S
                t += (m + 127) // 128
        return t
    assert total(8192, 4096, 0) == 1584
    assert total(131072, 1024, 0) == 9180
    assert total(16384, 128, 128) == 382
    for qt in (0, 1, 31, 63):
        tiles, cells = orc.schedule_qtile("swa", 8192, 4096, 0, 128, 128, qt)
        lo = max(0, qt * 128 - 4095) // 128
        assert tiles == list(range(lo, qt + 1))
    for qt in (0, 1, 2, 127):
        tiles, cells = orc.schedule_qtile("strided", 16384, 128, 128, 128, 128, qt)
        r1 = qt * 128 + 127
        want_st = [0x40000000] if max(0, r1 - 127) > 0 else []
        assert tiles == want_st + list(range(max(0, qt * 128 - 127) // 128, qt + 1))
        assert cells == strided_closed(r1 + 1, 128, 128) - strided_closed(qt * 128, 128, 128)


# ------------------------------------------------------- printed numbers ---

def test_nsa_keys_printed_on_cheatsheet(orc):
    nums = read_numbers("page_numbers.txt")
    n = orc.count_nsa(1024, 32, 4, 128)
    assert n == nums["nsa_keys_N1024_l32_k4_w128"] == 288
    assert math.floor(10 * 1024 / n) / 10 == nums["nsa_reduction_printed"]


def test_kv_cache_bytes_scales_with_window(orc):
    nums = read_numbers("page_numbers.txt")
    L, H, d = nums["kv_example_layers"], nums["kv_example_kv_heads"], nums["kv_example_d_head"]
    N, W = nums["kv_example_seq_len"], nums["kv_example_window"]
    full = orc.kv_cache_bytes(N, L, H, d, dtype=2)
    swa = orc.kv_cache_bytes(N, L, H, d, dtype=2, window=W)
    assert full == 2 * 80 * 8 * 128 * 131072 * 2 == 42949672960
    assert swa == 1342177280
    # the page's own scaling rule swa_kv = full_kv * (window / seq_len)
    assert swa == full * W // N
    # linear in min(N, W): doubling N past W changes nothing
    assert orc.kv_cache_bytes(2 * N, L, H, d, window=W) == swa
    assert orc.kv_cache_bytes(W // 2, L, H, d, window=W) * 2 == swa
    # lesson quiz: 32k-token cache vs a 2048 window is 16x smaller
    assert orc.kv_cache_bytes(32768, 1, 1, 1) // orc.kv_cache_bytes(32768, 1, 1, 1, window=2048) == \
        nums["kv_reduction_w2048_s32768"]


def test_core_flops_table(orc):
    nums = read_numbers("page_numbers.txt")
    b, s, d, w = 2, 64, 16, 8
    dense = np.zeros((s, s))  # every pair allowed
    assert orc.core_flops(orc.count_nonmasked(dense), d, b) == 4 * b * s * s * d
    # a two-sided window of exactly w keys per row: s*w entries -> 4bswd
    assert orc.core_flops(s * w, d, b) == 4 * b * s * w * d
    assert (32768 * 32768) // (32768 * 2048) == nums["score_flops_reduction_w2048_s32768"]


# ------------------------------------------------------ attention sinks ---

def _sink_history(B, Hkv, Hq, d, n_sink, W, pos0, T, seed):
    """A K/V history of pos0 + T tokens, a cache holding what a sink cache
    holds before step pos0, and the T new tokens."""
    L = pos0 + T
    Kh = randn_bf16((B, Hkv, L, d), seed).float()
    Vh = randn_bf16((B, Hkv, L, d), seed + 1).float()
    q = randn_bf16((T, B, Hq, d), seed + 2).float()
    kc = torch.full((B, Hkv, n_sink + W, d), float("nan"))  # unfilled slots must never be read
    vc = torch.full((B, Hkv, n_sink + W, d), float("nan"))
    for p in range(pos0):
        if p < n_sink:
            slot = p
        elif p >= pos0 - W:
            slot = n_sink + (p - n_sink) % W
        else:
            continue
        kc[:, :, slot] = Kh[:, :, p]
        vc[:, :, slot] = Vh[:, :, p]
    k_new = Kh[:, :, pos0:].permute(2, 0, 1, 3).contiguous()
    v_new = Vh[:, :, pos0:].permute(2, 0, 1, 3).contiguous()
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    return Kh, Vh, q, kc, vc, k_new, v_new, pos


@pytest.mark.parametrize("n_sink,W,pos0,T", [(4, 8, 0, 20), (4, 8, 30, 9), (1, 5, 2, 12), (3, 16, 10, 4),
                                             (4, 6, 9, 1)])
def test_sink_decode_equals_softmax_over_sinks_and_window(orc, n_sink, W, pos0, T):
    """Step at pos attends positions 0 .. n_sink-1 (those <= pos) and the W
    most recent positions above the sinks, whatever slots hold them."""
    B, Hq, Hkv, d = 2, 4, 2, 16
    Kh, Vh, q, kc, vc, k_new, v_new, pos = _sink_history(B, Hkv, Hq, d, n_sink, W, pos0, T, 40)
    out, kc2, vc2 = orc.sink_decode(q, k_new, v_new, kc, vc, pos, n_sink)
    G = Hq // Hkv
    for t in range(T):
        p = pos0 + t
        keys = sorted(set(range(min(n_sink, p + 1))) | set(range(max(n_sink, p - W + 1), p + 1)))
        assert len(keys) <= n_sink + W  # bounded cache, O(k + w)
        Kw = Kh[:, :, keys].double().repeat_interleave(G, dim=1)
        Vw = Vh[:, :, keys].double().repeat_interleave(G, dim=1)
        ref = F.scaled_dot_product_attention(q[t].double()[:, :, None], Kw, Vw, scale=1 / 4)[:, :, 0]
        assert np.abs(out[t] - ref.numpy()).max() < 1e-12
    last = pos0 + T - 1
    for p in range(min(n_sink, last + 1)):  # sinks never leave
        assert np.array_equal(kc2[:, :, p], Kh[:, :, p].numpy())
    for p in range(max(n_sink, last - W + 1), last + 1):
        assert np.array_equal(vc2[:, :, n_sink + (p - n_sink) % W], Vh[:, :, p].numpy())


def test_sink_decode_without_sinks_is_the_rolling_window(orc):
    T, B, Hq, Hkv, d, W = 6, 2, 4, 2, 16, 8
    q = randn_bf16((T, B, Hq, d), 1)
    k_new, v_new = randn_bf16((T, B, Hkv, d), 2), randn_bf16((T, B, Hkv, d), 3)
    kc, vc = randn_bf16((B, Hkv, W, d), 4), randn_bf16((B, Hkv, W, d), 5)
    pos = np.array([[20 + t, 3 + t] for t in range(T)], dtype=np.int32)
    a, ka, va = orc.decode(q, k_new, v_new, kc, vc, pos)
    b, kb, vb = orc.sink_decode(q, k_new, v_new, kc, vc, pos, 0)
    assert np.array_equal(a, b) and np.array_equal(ka, kb) and np.array_equal(va, vb)


# ------------------------------------------------------ differential decode --

def _diff_history(B, Hkv, Hq, dk, dv, W, pos0, T, seed):
    """Histories of K1, K2, V over pos0 + T tokens, caches holding what a
    W-slot rolling cache holds before step pos0, and the T new tokens."""
    L = pos0 + T
    K1h = randn_bf16((B, Hkv, L, dk), seed).float()
    K2h = randn_bf16((B, Hkv, L, dk), seed + 1).float()
    Vh = randn_bf16((B, Hkv, L, dv), seed + 2).float()
    q1 = randn_bf16((T, B, Hq, dk), seed + 3).float()
    q2 = randn_bf16((T, B, Hq, dk), seed + 4).float()
    caches = [torch.full((B, Hkv, W, x), float("nan")) for x in (dk, dk, dv)]  # unfilled slots never read
    for p in range(max(0, pos0 - W), pos0):
        for c, h in zip(caches, (K1h, K2h, Vh)):
            c[:, :, p % W] = h[:, :, p]
    new = [h[:, :, pos0:].permute(2, 0, 1, 3).contiguous() for h in (K1h, K2h, Vh)]
    pos = np.array([[pos0 + t] * B for t in range(T)], dtype=np.int32)
    return (K1h, K2h, Vh), (q1, q2), caches, new, pos


@pytest.mark.parametrize("W,pos0,T,G", [(8, 0, 12, 2), (8, 30, 9, 1), (5, 2, 10, 4), (16, 40, 3, 2)])
def test_diff_decode_is_difference_of_two_window_softmaxes(orc, W, pos0, T, G):
    """Each step equals SDPA(q1, K1w, Vw) - lambda_h SDPA(q2, K2w, Vw) over
    the window positions max(0, p-W+1) .. p, whatever slots hold them; V is
    the same for both maps."""
    B, Hkv, dk, dv = 2, 2, 16, 24
    Hq = Hkv * G
    (K1h, K2h, Vh), (q1, q2), (k1c, k2c, vc), (k1n, k2n, vn), pos = _diff_history(B, Hkv, Hq, dk, dv, W, pos0, T, 60)
    lam = torch.linspace(-0.5, 0.9, Hq)
    out, k1a, k2a, va = orc.diff_decode(q1, q2, k1n, k2n, vn, k1c, k2c, vc, lam, pos)
    for t in range(T):
        p = pos0 + t
        keys = list(range(max(0, p - W + 1), p + 1))
        K1w, K2w, Vw = (h[:, :, keys].double().repeat_interleave(G, dim=1) for h in (K1h, K2h, Vh))
        a1 = F.scaled_dot_product_attention(q1[t].double()[:, :, None], K1w, Vw, scale=1 / 4)[:, :, 0]
        a2 = F.scaled_dot_product_attention(q2[t].double()[:, :, None], K2w, Vw, scale=1 / 4)[:, :, 0]
        ref = a1 - lam.double()[None, :, None] * a2
        assert np.abs(out[t] - ref.numpy()).max() < 1e-12
    last = pos0 + T - 1
    for p in range(max(0, last - W + 1), last + 1):  # the window's tokens sit in slot p % W
        assert np.array_equal(k2a[:, :, p % W], K2h[:, :, p].numpy())
        assert np.array_equal(va[:, :, p % W], Vh[:, :, p].numpy())


def test_diff_decode_with_lambda_zero_is_the_plain_decode(orc):
    T, B, Hq, Hkv, d, W = 5, 2, 4, 2, 16, 8
    (K1h, K2h, Vh), (q1, q2), (k1c, k2c, vc), (k1n, k2n, vn), pos = _diff_history(B, Hkv, Hq, d, d, W, 20, T, 70)
    out, k1a, _, va = orc.diff_decode(q1, q2, k1n, k2n, vn, k1c, k2c, vc, np.zeros(Hq), pos)
    ref, kr, vr = orc.decode(q1, k1n, vn, k1c, vc, pos)
    assert np.abs(out - ref).max() < 1e-12
    assert np.array_equal(k1a, kr) and np.array_equal(va, vr)



# ------------------------------------------------------- global tokens -----

def global_closed(N, W, g):
    # per row: min(i+1, W) window keys plus the global keys below the window
    i = np.arange(N, dtype=np.int64)
    lo = np.maximum(0, i - W + 1)
    return int(np.minimum(i + 1, W).sum() + np.minimum(g, lo).sum())


def test_global_mask_8_2_3_matches_hand_derived_grid(orc):
    M = orc.mask("global", 8, 2, 3)
    assert grid_of(M) == read_grid("global_mask_n8_w2_g3.txt")
    assert orc.count_nonmasked(M) == 30 == global_closed(8, 2, 3)


def test_global_mask_brute_force_all_small(orc):
    """Against the predicate j <= i and (i - W < j or j < g or i < g), for
    every n <= 20, every window and every number of global tokens; the
    count against the closed form."""
    for n in range(1, 21):
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        for W in range(1, n + 2):
            for g in range(0, n + 2):
                want = (jj <= ii) & ((ii - W < jj) | (jj < g) | (ii < g))
                M = orc.mask("global", n, W, g)
                assert np.array_equal(M == 0.0, want), (n, W, g)
                assert orc.count_nonmasked(M) == global_closed(n, W, g), (n, W, g)


def test_global_mask_special_cases(orc):
    n, W = 40, 6
    assert np.array_equal(orc.mask("global", n, W, 0), orc.swa_mask(n, W))  # no global token
    assert np.array_equal(orc.mask("global", n, W, 1), orc.strided_mask(n, W, n + 5))  # only key 0
    for g in (n, n + 3):
        assert np.array_equal(orc.mask("global", n, W, g), orc.causal_mask(n))
    assert np.array_equal(orc.mask("global", n, n, 7), orc.causal_mask(n))


@pytest.mark.parametrize("n_sink,W,pos", [(4, 8, 3), (4, 8, 9), (4, 8, 40), (2, 16, 17), (1, 5, 30)])
def test_global_prefill_row_equals_sink_decode_step(orc, n_sink, W, pos):
    """A decode step with n_sink attention sinks and a W-token window sees
    exactly row pos of the window + global-token mask with g = n_sink: the
    two oracle functions are written separately and must agree."""
    B, Hq, Hkv, d = 1, 4, 2, 16
    Kh, Vh, q, kc, vc, k_new, v_new, posarr = _sink_history(B, Hkv, Hq, d, n_sink, W, pos, 1, 90)
    dec, _, _ = orc.sink_decode(q, k_new, v_new, kc, vc, posarr, n_sink)
    Q = torch.zeros(B, Hq, pos + 1, d)
    Q[:, :, pos] = q[0]
    pre = orc.attention("global", Q, Kh, Vh, W=W, S=n_sink, scale=0.25)
    assert np.abs(pre[:, :, pos] - dec[0]).max() < 1e-12


# ------------------------------------------------------ dilated window -----

def dilated_closed(N, W, dil):
    # row i attends min(W, floor(i / dil) + 1) keys
    i = np.arange(N, dtype=np.int64)
    return int(np.minimum(W, i // dil + 1).sum())


def test_dilated_mask_brute_force_all_small(orc):
    """Against the predicate j <= i, (i - j) % dil == 0, (i - j) / dil < W,
    for every n <= 20, window and dilation; count against the closed form."""
    for n in range(1, 21):
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        for W in range(1, n + 2):
            for dil in range(1, n + 2):
                want = (jj <= ii) & ((ii - jj) % dil == 0) & ((ii - jj) // dil < W)
                M = orc.mask("dilated", n, W, dil)
                assert np.array_equal(M == 0.0, want), (n, W, dil)
                assert orc.count_nonmasked(M) == dilated_closed(n, W, dil)


def test_dilation_one_is_the_window(orc):
    for n, W in ((40, 6), (17, 17), (9, 30)):
        assert np.array_equal(orc.mask("dilated", n, W, 1), orc.swa_mask(n, W))


@pytest.mark.parametrize("n,W,dil", [(50, 4, 3), (64, 7, 2), (33, 5, 4), (20, 30, 6)])
def test_dilated_mask_is_dil_interleaved_windows(orc, n, W, dil):
    """Rows and keys of one residue class mod dil form a plain window mask of
    W keys on that subsequence; keys of other classes are never attended.
    The kernels rest on this decomposition."""
    M = orc.mask("dilated", n, W, dil)
    ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    assert np.all(M[(ii - jj) % dil != 0] == -np.inf)
    for r in range(dil):
        idx = np.arange(r, n, dil)
        assert np.array_equal(M[np.ix_(idx, idx)], orc.swa_mask(idx.size, W))


@pytest.mark.parametrize("B,Hq,Hkv,N,d,W,dil", [(1, 2, 1, 90, 16, 5, 3), (2, 4, 4, 64, 8, 9, 2)])
def test_dilated_attention_matches_torch_sdpa_fp64(orc, B, Hq, Hkv, N, d, W, dil):
    q, k, v = attn_inputs(B, Hq, Hkv, N, d, seed=13)
    out = orc.attention("dilated", q, k, v, W=W, S=dil, scale=0.25)
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    allowed = (jj <= ii) & ((ii - jj) % dil == 0) & ((ii - jj) // dil < W)
    assert np.abs(out - sdpa_ref(q, k, v, allowed, 0.25)).max() < 1e-12


# ------------------------------------------------------------- backward ----

def _allowed(kind, N, W, S):
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    if kind == "causal":
        return jj <= ii
    band = (ii - W < jj) & (jj <= ii)
    if kind == "strided":
        return band | ((jj % S == 0) & (jj <= ii))
    if kind == "global":
        return band | (((jj < S) | (ii < S)) & (jj <= ii))
    return band


@pytest.mark.parametrize("kind,B,Hq,Hkv,N,dk,dv,W,S", [
    ("swa", 1, 2, 2, 40, 8, 8, 7, 0), ("swa", 1, 4, 2, 33, 16, 12, 5, 0), ("causal", 2, 2, 1, 25, 8, 8, 0, 0),
    ("strided", 1, 2, 2, 45, 8, 8, 4, 6), ("global", 1, 2, 1, 38, 8, 8, 5, 3)])
def test_backward_matches_torch_autograd_fp64(orc, kind, B, Hq, Hkv, N, dk, dv, W, S):
    """The oracle's per-row chain rule against torch autograd through fp64
    scaled_dot_product_attention with the explicit mask (GQA by repeating
    K/V heads, whose gradients autograd sums)."""
    q, k, v = attn_inputs(B, Hq, Hkv, N, dk, dv, seed=17)
    dO = randn_bf16((B, Hq, N, dv), 99)
    scale = 1 / math.sqrt(dk)
    dq, dkk, dvv = orc.attention_bwd(kind, q, k, v, dO, W=W, S=S, scale=scale)
    G = Hq // Hkv
    q64, k64, v64 = (t.double().requires_grad_(True) for t in (q, k, v))
    o = F.scaled_dot_product_attention(q64, k64.repeat_interleave(G, dim=1), v64.repeat_interleave(G, dim=1),
                                       attn_mask=torch.from_numpy(_allowed(kind, N, W, S)), scale=scale)
    (o * dO.double()).sum().backward()
    assert np.abs(dq - q64.grad.numpy()).max() < 1e-12
    assert np.abs(dkk - k64.grad.numpy()).max() < 1e-12
    assert np.abs(dvv - v64.grad.numpy()).max() < 1e-12


def test_backward_matches_finite_differences_of_the_oracle_forward(orc):
    """Central differences of f = sum(O * dO), O from the oracle's forward,
    for a few entries of Q, K and V (steps of 2^-10 are exact in float32)."""
    B, Hq, Hkv, N, d, W = 1, 2, 1, 12, 4, 5
    q, k, v = (t.float() for t in attn_inputs(B, Hq, Hkv, N, d, seed=23))
    dO = randn_bf16((B, Hq, N, d), 7).float()
    dq, dkk, dvv = orc.attention_bwd("swa", q, k, v, dO, W=W, scale=0.5)
    h = 2.0 ** -10

    def f(qq, kk, vv):
        return float((orc.attention("swa", qq, kk, vv, W=W, scale=0.5) * dO.double().numpy()).sum())

    for name, t, g, idx in (("q", q, dq, (0, 1, 7, 2)), ("k", k, dkk, (0, 0, 4, 1)), ("v", v, dvv, (0, 0, 9, 3)),
                            ("k0", k, dkk, (0, 0, 0, 0))):
        plus, minus = t.clone(), t.clone()
        plus[idx] += h
        minus[idx] -= h
        args_p = {"q": (plus, k, v), "k": (q, plus, v), "v": (q, k, plus), "k0": (q, plus, v)}[name]
        args_m = {"q": (minus, k, v), "k": (q, minus, v), "v": (q, k, minus), "k0": (q, minus, v)}[name]
        num = (f(*args_p) - f(*args_m)) / (2 * h)
        assert abs(num - g[idx]) < 2e-5 * max(1.0, abs(g[idx])), (name, num, g[idx])


def test_backward_row_subsets_match_full(orc):
    q, k, v = attn_inputs(2, 4, 2, 30, 8, seed=31)
    dO = randn_bf16((2, 4, 30, 8), 32)
    dq, dkk, dvv = orc.attention_bwd("swa", q, k, v, dO, W=6)
    qr, kr = np.array([0, 29, 31, 4 * 30 + 17, 8 * 30 - 1]), np.array([0, 5, 30 + 29, 3 * 30 + 2])
    a, b, c = orc.attention_bwd("swa", q, k, v, dO, W=6, dq_rows=qr, dkv_rows=kr)
    assert np.array_equal(a, dq.reshape(-1, 8)[qr])
    assert np.array_equal(b, dkk.reshape(-1, 8)[kr]) and np.array_equal(c, dvv.reshape(-1, 8)[kr])
