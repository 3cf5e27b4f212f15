// schedule.cuh -- which key tiles a query tile touches.
//
// One definition, compiled for both sides: the prefill kernel enumerates its
// key tiles with these functions and swa_schedule() exports the same lists
// for the parity tests. The mask is never stored; each function evaluates
// the window / stride predicate on the tile's edge rows.
//
// Masks ("Learn: Sparse & Sliding-Window Attention", section 3; "Attention
// Variants Compared", swa_mask / strided_mask code):
//   window:  key j attended by row i iff  lo_i <= j <= i,  lo_i = max(0, i-W+1)
//   strided: window OR (j % S == 0 and j <= i).
//   global:  window OR j < g OR i < g, with j <= i ("Learn: Sparse &
//            Sliding-Window Attention", section 3b, Longformer's global
//            tokens, here positions 0 .. g-1; a global row i < g attends
//            keys j <= i < g, all of them global, so it needs no own term).
// A cell outside the window is an "extra" cell iff it is a stride key
// (j % S == 0) or a global key (j < g) below lo_i, so the union splits into
// disjoint window cells and extra cells, and each attended cell is visited
// exactly once.
//
// Extra cells are read through a second view of K/V whose row m holds key
// m*S (strided) or key m (global: the global keys are the first g rows). An
// "extra tile" ct holds rows ct*Bk .. ct*Bk+Bk-1 of that view.
#pragma once

#ifdef __CUDACC__
#define SWA_HD __host__ __device__ __forceinline__
#else
#define SWA_HD inline
#endif

#include <cstdint>

namespace swa {

// n / d for 0 <= n < 2^31 by a fixed divisor d >= 1, as a multiply-high and
// a shift (the round-up method: s = ceil(log2 d), m = floor(2^32 (2^s - d) / d)
// + 1, n / d = (umulhi(n, m) + n) >> s). Built once on the host; the kernels
// use it for their per-unit index arithmetic, where a runtime division costs
// tens of instructions.
struct FastDiv {
  uint32_t d, m, s;
  SWA_HD int operator()(int n) const {
#ifdef __CUDA_ARCH__
    const uint32_t hi = __umulhi(static_cast<uint32_t>(n), m);
#else
    const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * m) >> 32);
#endif
    return static_cast<int>((hi + static_cast<uint32_t>(n)) >> s);
  }
};

inline FastDiv make_fastdiv(int d) {
  FastDiv f;
  f.d = static_cast<uint32_t>(d < 1 ? 1 : d);
  f.s = 0;
  while ((1ull << f.s) < f.d) ++f.s;
  f.m = static_cast<uint32_t>((((1ull << 32) * ((1ull << f.s) - f.d)) / f.d) + 1);
  return f;
}

// Plain division, for the host-side schedule export.
struct PlainDiv {
  int d;
  SWA_HD int operator()(int n) const { return n / d; }
};

constexpr int kStrideTag = 0x40000000;

enum MaskKind { kMaskWindow = 0, kMaskStrided = 1, kMaskCausal = 2, kMaskGlobal = 3 };

SWA_HD int imin(int a, int b) { return a < b ? a : b; }
SWA_HD int imax(int a, int b) { return a > b ? a : b; }

// First attended key of row i under the window.
SWA_HD int window_lo(int i, int W) { return imax(0, i - W + 1); }

// Number of stride rows m with m*S < lo (keys below the window of a row
// whose window starts at lo). `div` divides by S.
template <class Div>
SWA_HD int stride_rows_below(int lo, int S, Div div) { return lo > 0 ? div(lo - 1) + 1 : 0; }
SWA_HD int stride_rows_below(int lo, int S) { return stride_rows_below(lo, S, PlainDiv{S}); }

// Extra-view rows attended by a row whose window starts at lo: stride rows
// below lo (strided), the global keys below lo (global; S carries g).
template <class Div>
SWA_HD int extra_rows_below(int kind, int lo, int S, Div div) {
  if (kind == kMaskStrided && S > 0) return stride_rows_below(lo, S, div);
  if (kind == kMaskGlobal && S > 0) return imin(S, lo);
  return 0;
}
SWA_HD int extra_rows_below(int kind, int lo, int S) { return extra_rows_below(kind, lo, S, PlainDiv{S > 0 ? S : 1}); }

struct QTileKeys {
  int band_lo;   // first window key tile
  int band_hi;   // last window key tile
  int n_stride;  // stride tiles 0 .. n_stride-1
};

// Key tiles of query tile qt (rows qt*Bq .. min(N, qt*Bq+Bq) - 1). W >= N
// (or kind == causal) is full causal. The window part is the contiguous
// range from the tile holding the first row's lo to the tile holding the
// last row; every tile in it has an attended cell because consecutive rows'
// windows overlap or abut. Extra tiles are those with an extra-view row
// below the last row's lo (the largest lo in the tile).
template <class Div>
SWA_HD QTileKeys qtile_keys(int kind, int N, int W, int S, int Bq, int Bk, int qt, Div div) {
  QTileKeys r;
  const int r0 = qt * Bq;
  const int r1 = imin(N - 1, r0 + Bq - 1);
  const int Wc = (kind == kMaskCausal) ? N : W;
  r.band_lo = window_lo(r0, Wc) / Bk;
  r.band_hi = r1 / Bk;
  r.n_stride = 0;
  if ((kind == kMaskStrided || kind == kMaskGlobal) && S > 0) {
    const int m = extra_rows_below(kind, window_lo(r1, Wc), S, div);
    r.n_stride = (m + Bk - 1) / Bk;
  }
  return r;
}

// The same for the window, strided and causal kinds only (no global-token
// branch), for kernels built without the global kind.
template <class Div>
SWA_HD QTileKeys qtile_keys_basic(int kind, int N, int W, int S, int Bq, int Bk, int qt, Div div) {
  QTileKeys r;
  const int r0 = qt * Bq;
  const int r1 = imin(N - 1, r0 + Bq - 1);
  const int Wc = (kind == kMaskCausal) ? N : W;
  r.band_lo = window_lo(r0, Wc) / Bk;
  r.band_hi = r1 / Bk;
  r.n_stride = 0;
  if (kind == kMaskStrided && S > 0) {
    const int m = stride_rows_below(window_lo(r1, Wc), S, div);
    r.n_stride = (m + Bk - 1) / Bk;
  }
  return r;
}

SWA_HD QTileKeys qtile_keys(int kind, int N, int W, int S, int Bq, int Bk, int qt) {
  return qtile_keys(kind, N, W, S, Bq, Bk, qt, PlainDiv{S > 0 ? S : 1});
}

SWA_HD int qtile_nkeys(const QTileKeys& k) { return k.n_stride + (k.band_hi - k.band_lo + 1); }

// Entry e of the query tile's visiting order: stride tiles first (oldest
// keys), then window tiles ascending. Encoded as in swa_debug_t.
SWA_HD int qtile_entry(const QTileKeys& k, int e) {
  return e < k.n_stride ? (kStrideTag | e) : (k.band_lo + (e - k.n_stride));
}

// Closed-form ||M||_0 of one N x N mask.
SWA_HD long long count_attended(int kind, int N, int W, int S) {
  if (kind == kMaskCausal || W >= N) {
    long long n = N;
    long long band = n * (n + 1) / 2;
    return band;  // no stride cells: every lo_i is 0
  }
  long long n = N, w = W;
  long long band = n * w - w * (w - 1) / 2;
  if (kind == kMaskGlobal && S > 0) {
    // rows i >= W have lo_i = t for t = 1 .. N-W and add min(g, t) keys
    const long long T = n - w, g = S;
    if (T <= g) return band + T * (T + 1) / 2;
    return band + g * (g + 1) / 2 + (T - g) * g;
  }
  if (kind != kMaskStrided || S <= 0) return band;
  // stride cells: sum over rows i >= W of ceil((i - W + 1) / S)
  // = sum over t = 1 .. N-W of ceil(t / S)
  long long T = n - w;  // rows with lo_i = t for t = 1 .. T
  long long s = S;
  long long q = T / s, rem = T % s;
  // t = 1..q*s: ceil(t/s) = block index b+1 for t in (b*s, (b+1)*s]
  long long full = s * q * (q + 1) / 2;
  long long tail = rem * (q + 1);
  return band + full + tail;
}

}  // namespace swa
