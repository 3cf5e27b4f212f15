// backward.cu -- gradients of the sliding-window attention forward on sm_100a.
//
// The pages define the forward only (A = softmax(Q K^T * scale + log M) V,
// "Learn: Sparse & Sliding-Window Attention", section 3); its training use
// ("Attention Variants -- Sliding Window, Sparse, Differential", opening)
// needs the gradients. This is the chain rule of that forward, in the
// flash-attention arrangement that never stores the N x N matrices: with
// the forward's log-sum-exp L_i and D_i = dO_i . O_i,
//     P_ij  = exp(scale q_i.k_j - L_i) on attended cells, else 0
//     dV_j  = sum_i P_ij dO_i,        dP_ij = dO_i . v_j
//     dS_ij = P_ij (dP_ij - D_i)
//     dQ_i  = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i
// over the same window mask, summed over the query heads of a KV head.
//
// Three kernels:
//   bwd_prep      D_i and L_i * log2(e) per query row into a padded
//                 workspace (one thread per row).
//   bwd_dkdv      one CTA per (b, KV head, 128-key tile): K and V of the tile
//                 stay in shared memory; for every query head of the group
//                 and every query tile that sees the keys, S^T = K Q^T and
//                 dP^T = V dO^T go to tensor memory, four warps (one key per
//                 TMEM lane) turn them into P^T and dS^T (bf16, written back
//                 over them), and dV += P^T dO, dK += dS^T Q accumulate in
//                 tensor memory (A operand read from TMEM).
//   bwd_dq        one CTA per (b, head, 128-query tile): Q and dO stay; for
//                 every key tile of the row block's window, S = Q K^T and
//                 dP = dO V^T, then dS (bf16 over S) and dQ += dS K.
// Operand layouts follow the forward's: 128-byte swizzled TMA tiles,
// K-major for the score products, MN-major for the products that run over
// the 128 tile rows. Waits are bounded; a timeout records SWA_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "schedule.cuh"

namespace swa {

namespace {

constexpr int kBwdThreads = 192;  // producer, MMA, four elementwise warps
// dQ kernel: producer, MMA, then four elementwise warps per 64-key half
// (warps 2-5 take half 0, warps 6-9 half 1, one lane quarter each), so the
// halves' elementwise work runs side by side
constexpr int kDqThreads = 320;
constexpr int kBT = 128;          // rows of a query or key tile

template <int D>
struct BwdCfg {
  static constexpr int kTile = kBT * D * 2;              // one tile of D bf16 columns
  static constexpr int kStage = 2 * kTile + 2 * kBT * 4; // two tiles + two fp32 row tables
  static constexpr int kStages = 2;
  // the dK/dV kernel at d = 64 runs several key tiles per CTA: two sets of
  // its fixed K and V tiles (the next tile's load overlaps this tile's
  // steps) and of its TMEM accumulators (the second in the 128 columns one
  // set leaves free), so a tile's epilogue overlaps the next tile's steps
  static constexpr int kFixedSets = D == 64 ? 2 : 1;
  static constexpr int kOffA = 0;                        // the CTA's fixed tiles (set f: + f * 2 * kTile)
  static constexpr int kOffB = kTile;
  static constexpr int kOffStages = 2 * kTile * kFixedSets;
  static constexpr int kOffBar = kOffStages + kStages * kStage;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;  // barriers area + alignment slack
  static constexpr uint32_t kColS = 0;      // S (or S^T), then P / dS as bf16 pairs
  static constexpr uint32_t kColDP = 128;   // dP (or dP^T), then dS^T as bf16 pairs
  static constexpr uint32_t kColAcc = 256;  // dQ, or dV then dK (set f: + f * kAccSet)
  static constexpr uint32_t kAccSet = 2 * D;
  // dQ kernel: Q and dO rows as the score products' A operands (bf16 pairs)
  static constexpr uint32_t kColQ = 256 + D;
  static constexpr uint32_t kColDO = kColQ + D / 2;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(256 + kFixedSets * 2 * D <= 512, "tensor memory");
  static_assert(kColDO + D / 2 <= 512, "tensor memory (dQ kernel)");
};

// Each step's score products run as two halves of 64 columns (queries in
// the dK/dV kernel, keys in the dQ kernel), each with its own barriers, so
// the tensor core works on one half (its accumulation, then the next step's
// scores) while the elementwise warps process the other.
constexpr int kBH = 64;  // columns of a half

struct BwdBar {
  static constexpr int kFixed = 0;      // + set: the fixed tiles landed
  static constexpr int kFull = 2;       // + stage
  static constexpr int kEmpty = 4;      // + stage
  static constexpr int kS = 6;          // + half: score products of the half in TMEM
  static constexpr int kP = 8;          // + half: elementwise done, P / dS of the half written
  static constexpr int kAcc = 10;       // + set: accumulators final
  static constexpr int kFinal = 12;     // MMA drain on abort
  static constexpr int kA = 13;         // dQ kernel: Q and dO rows copied into TMEM
  static constexpr int kFixedFree = 14; // + set: the set's fixed tiles no longer read (multi-tile dK/dV)
  static constexpr int kAccFree = 16;   // + set: the set's accumulators read out (multi-tile dK/dV)
  static constexpr int kWordsOff = 256;
  static_assert(18 * 8 <= kWordsOff, "barrier block");
};

__device__ __forceinline__ void bwd_timeout(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicExch(err, 4 /* SWA_ERR_TIMEOUT */);
}

// Four consecutive floats from shared memory (16-byte aligned address).
// Volatile: it stays after the barrier wait that makes the data visible.
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// p[0..3] += (a, b, c, d) as one relaxed device-scope reduction (p 16-byte
// aligned): a quarter of the atomic operations of four scalar adds.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// D_i = dO_i . O_i and L_i * log2(e), rows past N padded with zeros. Each
// row is read by D / 8 lanes, 16 bytes of O and of dO each (a warp's loads
// cover consecutive rows whole), whose partial dot products meet through
// shuffles within the row's lane group.
constexpr int kPrepThreads = 256;
template <int D>
__global__ void __launch_bounds__(kPrepThreads) bwd_prep_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;               // lanes per row
  constexpr int RPB = kPrepThreads / LPR;  // rows per block
  const int64_t total = (int64_t)p.B * p.Hq * p.npad;
  const int64_t r = (int64_t)blockIdx.x * RPB + threadIdx.x / LPR;  // (b*Hq + hq) * npad + i
  const int e = threadIdx.x % LPR;
  const bool valid = r < total;  // every lane stays for the shuffles
  const int64_t bh = valid ? r / p.npad : 0;
  const int i = valid ? (int)(r % p.npad) : p.N;
  const int64_t row = bh * p.N + i;
  float d = 0.f;
  if (i < p.N) {
    const uint4 a = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.o) + row * D)[e];
    const uint4 b = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.dO) + row * D)[e];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      d = fmaf(__uint_as_float(wa[k] << 16), __uint_as_float(wb[k] << 16), d);
      d = fmaf(__uint_as_float(wa[k] & 0xffff0000u), __uint_as_float(wb[k] & 0xffff0000u), d);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
  if (valid && e == 0) {
    float l2 = 0.f;
    if (i < p.N && SWA_IN(row, 0, (int64_t)p.B * p.Hq * p.N, p.err_flag)) l2 = p.lse[row] * 1.4426950408889634f;
    p.dd[r] = d;
    p.lse2[r] = l2;
  }
  // the stride pass adds its partials into zeroed memory
  if (p.S > 0) {
    const int64_t nz = (int64_t)p.B * p.Hkv * p.nspad * D;
    const int64_t nthreads = (int64_t)gridDim.x * kPrepThreads;
    for (int64_t z = (int64_t)blockIdx.x * kPrepThreads + threadIdx.x; z < nz; z += nthreads) {
      p.sdk[z] = 0.f;
      p.sdv[z] = 0.f;
    }
  }
}

// MODE 0: 128 window keys of the tile. MODE 1: the same, plus the stride
// pass's fp32 partials added to the stride keys before rounding (local +
// strided mask). MODE 2 (stride pass): the CTA owns 128 compacted stride
// keys (m*S for m in ct*128 .. ct*128+127) and one chunk of the later query
// tiles whose rows have them below their window; it adds its fp32 partial
// dK / dV into the workspace (several chunks per stride tile).
constexpr int kStrideChunk = 8;  // query tiles per stride-pass CTA

template <int D, int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                    const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  constexpr bool MULTI = C::kFixedSets == 2;  // several key tiles per CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * i; };
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + C::kOffBar + BwdBar::kWordsOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(words + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  constexpr bool STRIDE = MODE == 2;
  const int Wc = imin(p.W, p.N);
  // Work tiles in one linear order: column x = key tile (stride pass: stride
  // tile and chunk of query tiles), row y = b * Hkv + hkv. The CTA takes
  // the tile of its grid cell, or (multi-tile) every gridDim.x-th tile from
  // blockIdx.x; every role walks the same list.
  const int nchunk = STRIDE ? (p.nq + kStrideChunk - 1) / kStrideChunk : 1;
  const int ncol = STRIDE ? p.nspad / kBT * nchunk : p.nq;
  const int ntiles = ncol * p.B * p.Hkv;
  const int t_first = MULTI ? (int)blockIdx.x : (int)(blockIdx.y * ncol + blockIdx.x);
  const int t_step = MULTI ? (int)gridDim.x : ntiles;
  struct Tile {
    int b, hkv, kt, qt_lo, nqt, nsteps;
  };
  // query tiles that see keys kt*128 .. kt*128+127: from the diagonal up to
  // the last row whose window still reaches the tile's last key
  auto tile_of = [&](int t) -> Tile {
    Tile w;
    const int x = t % ncol, y = t / ncol;
    w.b = y / p.Hkv;
    w.hkv = y % p.Hkv;
    int qt_hi;
    if (STRIDE) {
      // row i has stride key m below its window iff m * S < i - W + 1
      w.kt = x / nchunk;
      const int chunk = x % nchunk;
      const int64_t first = (int64_t)w.kt * kBT * p.S + Wc;  // first row that sees m = kt * 128
      const int q0 = (int)(first < p.N ? first / kBT : p.nq);
      w.qt_lo = q0 + chunk * kStrideChunk;
      qt_hi = imin(p.nq - 1, w.qt_lo + kStrideChunk - 1);  // empty when past the last tile
    } else {
      w.kt = x;
      w.qt_lo = x;
      const int reach = x * kBT + kBT - 1 + Wc - 1;  // last query row that sees the tile's last key
      qt_hi = imin(p.nq - 1, reach / kBT);
    }
    w.nqt = qt_hi - w.qt_lo + 1;
    w.nsteps = w.nqt > 0 ? p.G * w.nqt : 0;
    return w;
  };

  if (threadIdx.x == 0) {
    for (int f = 0; f < 2; ++f) {
      mbar_init(bar(BwdBar::kFixed + f), 1);
      mbar_init(bar(BwdBar::kAcc + f), 1);
      mbar_init(bar(BwdBar::kFixedFree + f), 1);
      mbar_init(bar(BwdBar::kAccFree + f), 128);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(BwdBar::kFull + s), 1);
      mbar_init(bar(BwdBar::kEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(BwdBar::kS + h), 1);
      mbar_init(bar(BwdBar::kP + h), 128);
    }
    mbar_init(bar(BwdBar::kFinal), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(words), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];

  if (warp == 0) {
    // ------------------------------------------------------ producer ---
    if (lane == 0) {
      int issued[C::kStages] = {0, 0};
      int fixed_issued[2] = {0, 0};
      int g = 0;   // steps, across the CTA's tiles (stage ring)
      int jj = 0;  // non-empty tiles (fixed-tile sets)
      bool ok = true;
      for (int t = t_first; t < ntiles && ok; t += t_step) {
        const Tile w = tile_of(t);
        if (w.nsteps == 0) continue;
        const int fs = MULTI ? (jj & 1) : 0, fuse = MULTI ? (jj >> 1) : jj;
        ++jj;
        // the set's K and V are free once the tile before last has run its scores
        if (fuse > 0 && !mbar_wait(bar(BwdBar::kFixedFree + fs), (fuse - 1) & 1, abort_flag)) {
          bwd_timeout(abort_flag, p.err_flag);
          break;
        }
        const int zkv = w.b * p.Hkv + w.hkv;
        const int krows = STRIDE ? (p.N - 1) / p.S + 1 : p.N;  // rows of the stride view, or of K/V
        (void)krows;
        const uint32_t set_off = fs * 2 * C::kTile;
        mbar_arrive_expect_tx(bar(BwdBar::kFixed + fs), 2 * C::kTile);
        for (int bx = 0; bx < D / 64; ++bx) {
          if (!SWA_TMA_IN(bx * 64, D, w.kt * kBT, krows, zkv, p.B * p.Hkv, p.err_flag)) continue;
          tma_load_3d(sbase + C::kOffA + set_off + bx * 16384, STRIDE ? &tm_ks : &tm_k, bar(BwdBar::kFixed + fs),
                      bx * 64, w.kt * kBT, zkv);
          tma_load_3d(sbase + C::kOffB + set_off + bx * 16384, STRIDE ? &tm_vs : &tm_v, bar(BwdBar::kFixed + fs),
                      bx * 64, w.kt * kBT, zkv);
        }
        fixed_issued[fs] = fuse + 1;
        for (int s = 0; s < w.nsteps; ++s, ++g) {
          const int st = g & 1, use = g >> 1;
          if (use > 0 && !mbar_wait(bar(BwdBar::kEmpty + st), (use - 1) & 1, abort_flag)) {
            bwd_timeout(abort_flag, p.err_flag);
            ok = false;
            break;
          }
          const int hq = w.hkv * p.G + s / w.nqt, qt = w.qt_lo + s % w.nqt;
          const int zq = w.b * p.Hq + hq;
          const uint32_t base = sbase + C::kOffStages + st * C::kStage;
          mbar_arrive_expect_tx(bar(BwdBar::kFull + st), 2 * C::kTile + 2 * kBT * 4);
          for (int bx = 0; bx < D / 64; ++bx) {
            if (!SWA_TMA_IN(bx * 64, D, qt * kBT, p.N, zq, p.B * p.Hq, p.err_flag)) continue;
            tma_load_3d(base + bx * 16384, &tm_q, bar(BwdBar::kFull + st), bx * 64, qt * kBT, zq);
            tma_load_3d(base + C::kTile + bx * 16384, &tm_do, bar(BwdBar::kFull + st), bx * 64, qt * kBT, zq);
          }
          const int64_t rt = (int64_t)zq * p.npad + qt * kBT;
          if (SWA_IN(rt, 0, (int64_t)p.B * p.Hq * p.npad - kBT + 1, p.err_flag)) {
            bulk_load(base + 2 * C::kTile, p.lse2 + rt, kBT * 4, bar(BwdBar::kFull + st));
            bulk_load(base + 2 * C::kTile + kBT * 4, p.dd + rt, kBT * 4, bar(BwdBar::kFull + st));
          }
          issued[st] = use + 1;
        }
      }
      if (*abort_flag) {  // drain: every copy issued lands before the CTA may exit
        for (int f = 0; f < 2; ++f)
          if (fixed_issued[f] > 0) mbar_wait_timed(bar(BwdBar::kFixed + f), (fixed_issued[f] - 1) & 1);
        for (int st = 0; st < C::kStages; ++st)
          if (issued[st] > 0) mbar_wait_timed(bar(BwdBar::kFull + st), (issued[st] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA ---
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kBT, kBH, false);
      const uint32_t idesc_acc = idesc_bf16_f32(kBT, D, true);
      bool ok = true;
      int g = 0, jj = 0;
      for (int t = t_first; t < ntiles && ok; t += t_step) {
        const Tile w = tile_of(t);
        if (w.nsteps == 0) continue;
        const int fs = MULTI ? (jj & 1) : 0, fuse = MULTI ? (jj >> 1) : jj;
        ++jj;
        const uint32_t set_off = fs * 2 * C::kTile;
        const uint64_t k_desc = sw128_desc(sbase + C::kOffA + set_off, 16, 1024);
        const uint64_t v_desc = sw128_desc(sbase + C::kOffB + set_off, 16, 1024);
        const uint32_t acc_col = C::kColAcc + fs * C::kAccSet;
        if (!mbar_wait(bar(BwdBar::kFixed + fs), fuse & 1, abort_flag)) {
          ok = false;
          break;
        }
        // the set's accumulators: read out by the epilogue of the tile before last
        if (fuse > 0 && !mbar_wait(bar(BwdBar::kAccFree + fs), (fuse - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S^T = K Q^T and dP^T = V dO^T of queries 64h .. 64h+63 of step gs
        // (rows: keys, columns: queries; the half's Q and dO rows start 64
        // rows = 8192 bytes into each 64-column box)
        auto scores = [&](int gs, int h) {
          const uint32_t cur = sbase + C::kOffStages + (gs & 1) * C::kStage + h * 8192;
          const uint64_t q_k = sw128_desc(cur, 16, 1024);
          const uint64_t do_k = sw128_desc(cur + C::kTile, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + C::kColS + kBH * h, k_desc + off, q_k + off, idesc_s, kk > 0 ? 1u : 0u);
            umma_bf16_ss(tmem + C::kColDP + kBH * h, v_desc + off, do_k + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(BwdBar::kS + h));
        };
        // dV += P^T dO and dK += dS^T Q over the half's 64 queries (P^T, dS^T
        // as bf16 pairs in the half's first 32 columns); the tile's first
        // product overwrites the set's accumulators
        auto accumulate = [&](int gs, bool first, int h) {
          const uint32_t cur = sbase + C::kOffStages + (gs & 1) * C::kStage;
          const uint64_t q_mn = sw128_desc(cur, 16384, 1024);
          const uint64_t do_mn = sw128_desc(cur + C::kTile, 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < kBH / 16; ++kk) {
            const uint32_t acc = (first && h == 0 && kk == 0) ? 0u : 1u;
            const uint64_t row = (uint64_t)(((kBH / 16) * h + kk) * 2048 >> 4);
            umma_bf16_ts(tmem + acc_col, tmem + C::kColS + kBH * h + kk * 8, do_mn + row, idesc_acc, acc);
            umma_bf16_ts(tmem + acc_col + D, tmem + C::kColDP + kBH * h + kk * 8, q_mn + row, idesc_acc, acc);
          }
        };
        const int g0 = g;  // the tile's first step
        if (!mbar_wait(bar(BwdBar::kFull + (g0 & 1)), (g0 >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        scores(g0, 0);
        scores(g0, 1);
        for (int s = 0; ok && s < w.nsteps; ++s) {
          const int gs = g0 + s;
          for (int h = 0; h < 2 && ok; ++h) {
            if (!mbar_wait(bar(BwdBar::kP + h), gs & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            accumulate(gs, s == 0, h);
            if (h == 1) umma_commit(bar(BwdBar::kEmpty + (gs & 1)));  // Q, dO and the row tables of the step read
            if (s + 1 < w.nsteps) {
              if (h == 0) {
                if (!mbar_wait(bar(BwdBar::kFull + ((gs + 1) & 1)), ((gs + 1) >> 1) & 1, abort_flag)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              // into the columns the accumulation above reads first (MMAs run in issue order)
              scores(gs + 1, h);
            }
          }
        }
        g = g0 + w.nsteps;
        if (ok) {
          umma_commit(bar(BwdBar::kAcc + fs));                    // the tile's dV and dK final
          if (MULTI) umma_commit(bar(BwdBar::kFixedFree + fs));  // its K and V read by every score product
        }
      }
      if (!ok) bwd_timeout(abort_flag, p.err_flag);
      if (!ok || *abort_flag) {
        umma_commit(bar(BwdBar::kFinal));
        mbar_wait_timed(bar(BwdBar::kFinal), 0);
      }
    }
  } else {
    // --------------------------------------------------- elementwise ---
    const int qw = warp & 3;             // TMEM lane quarter
    const int kr = qw * 32 + lane;       // key row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(qw * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0, jj = 0;
    for (int t = t_first; t < ntiles && ok; t += t_step) {
      const Tile w = tile_of(t);
      if (w.nsteps == 0) continue;
      const int fs = MULTI ? (jj & 1) : 0, fuse = MULTI ? (jj >> 1) : jj;
      ++jj;
      const uint32_t acc_col = C::kColAcc + fs * C::kAccSet;
      const int key = w.kt * kBT + kr;  // (STRIDE: the compacted index m; the key is m * S)
      // query rows [ilo, ihi] that attend this lane's key (empty: ilo > ihi):
      // the window's rows key .. key + W - 1, or, for the stride key m*S, every
      // row whose window starts after it (m*S < i - W + 1, i.e. i >= m*S + W);
      // rows below N
      int ilo, ihi;
      if constexpr (STRIDE) {
        const int64_t first = (int64_t)key * p.S + Wc;
        ilo = (int)(first < p.N ? first : p.N);
        ihi = p.N - 1;
      } else {
        const int64_t last = (int64_t)key + Wc - 1;
        ilo = key;
        ihi = key < p.N ? (int)(last < p.N - 1 ? last : p.N - 1) : -1;
      }
      for (int s = 0; s < w.nsteps && ok; ++s, ++g) {
        const int qt = w.qt_lo + s % w.nqt;
        // the step's row tables: L * log2(e), then D, 128 floats each
        const uint32_t tables = sbase + C::kOffStages + (g & 1) * C::kStage + 2 * C::kTile;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {  // two halves of 64 queries, each on its own barriers
          const bool got = mbar_wait(bar(BwdBar::kS + h), g & 1, abort_flag);
          // the row tables were written by the copy engine: acquire them from
          // the stage's own barrier (complete already; the stage cannot be
          // refilled before this step's P^T and dS^T are consumed)
          const bool have = got && (h == 1 || mbar_wait(bar(BwdBar::kFull + (g & 1)), (g >> 1) & 1, abort_flag));
          if (!__all_sync(0xffffffffu, have)) {
            if (lane == 0) bwd_timeout(abort_flag, p.err_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const int c_lo = ilo - (qt * kBT + kBH * h), c_hi = ihi - (qt * kBT + kBH * h);  // attended columns
          const uint32_t s_col = tmem + lane_addr + C::kColS + kBH * h;
          const uint32_t dp_col = tmem + lane_addr + C::kColDP + kBH * h;
          uint32_t pk[32], dk[32];
          if (__all_sync(0xffffffffu, c_hi < 0 || c_lo > kBH - 1 || c_lo > c_hi)) {
            // no query of this half attends a key of this warp: P^T = dS^T = 0,
            // the scores are not read
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = dk[e] = 0u;
          } else {
            float sv[64], dp[64];
            tmem_ld64(s_col, sv);
            tmem_ld64(dp_col, dp);
            const uint32_t tab = tables + 4 * kBH * h;  // the half's rows (same for every lane)
            auto body = [&](auto attended) {
#pragma unroll
              for (int c = 0; c < 64; c += 4) {
                const float4 l4 = ld_shared_f4(tab + 4 * c), d4 = ld_shared_f4(tab + 4 * kBT + 4 * c);
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                  const bool a0 = attended(c + e), a1 = attended(c + e + 1);
                  const float p0 = a0 ? ex2_approx(fmaf(sv[c + e], sl2, -lv[e])) : 0.f;
                  const float p1 = a1 ? ex2_approx(fmaf(sv[c + e + 1], sl2, -lv[e + 1])) : 0.f;
                  pk[(c + e) >> 1] = pack_bf16(p0, p1);
                  dk[(c + e) >> 1] = pack_bf16(p0 * (dp[c + e] - dv[e]), p1 * (dp[c + e + 1] - dv[e + 1]));
                }
              }
            };
            // every (key, query) cell of the warp's 32 x 64 block attended: no per-cell test
            if (__all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kBH - 1))
              body([](int) { return true; });
            else
              body([&](int c) { return c >= c_lo && c <= c_hi; });
          }
          // P^T over S^T and dS^T over dP^T as bf16 pairs: the half's 64
          // queries land in its own first 32 columns, already read
          tmem_st32_u(s_col, pk);
          tmem_st32_u(dp_col, dk);
          tc_fence_before();
          mbar_arrive(bar(BwdBar::kP + h));
        }
      }
      if (!ok) break;
      {
        const bool got = mbar_wait(bar(BwdBar::kAcc + fs), fuse & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) bwd_timeout(abort_flag, p.err_flag);
          ok = false;
        }
      }
      if (ok && STRIDE) {
        // this chunk's fp32 partials of the stride keys, added to the others'
        tc_fence_after();
        const int64_t row = ((int64_t)(w.b * p.Hkv + w.hkv) * p.nspad + key) * D;
#pragma unroll 1
        for (int c = 0; c < D && SWA_IN(row, 0, (int64_t)p.B * p.Hkv * p.nspad * D - D + 1, p.err_flag); c += 32) {
          float a[32], gk[32];
          tmem_ld32(tmem + lane_addr + acc_col + c, a);
          tmem_ld32(tmem + lane_addr + acc_col + D + c, gk);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            red_add_v4(p.sdv + row + c + e, a[e], a[e + 1], a[e + 2], a[e + 3]);
            red_add_v4(p.sdk + row + c + e, gk[e], gk[e + 1], gk[e + 2], gk[e + 3]);
          }
        }
      } else if (ok) {
        tc_fence_after();
        const int64_t row = ((int64_t)(w.b * p.Hkv + w.hkv) * p.N + key) * D;
        __nv_bfloat16* dv = reinterpret_cast<__nv_bfloat16*>(p.dv) + row;
        __nv_bfloat16* dkp = reinterpret_cast<__nv_bfloat16*>(p.dk) + row;
        // a stride key also gets the stride pass's partials before the one rounding
        const bool add = MODE == 1 && key < p.N && key % p.S == 0;
        const int64_t srow = ((int64_t)(w.b * p.Hkv + w.hkv) * p.nspad + (add ? key / p.S : 0)) * D;
        const bool in_rows = key >= p.N || SWA_IN(row, 0, (int64_t)p.B * p.Hkv * p.N * D - D + 1, p.err_flag);
        const bool in_srow = !add || SWA_IN(srow, 0, (int64_t)p.B * p.Hkv * p.nspad * D - D + 1, p.err_flag);
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float a[32], gk[32];
          tmem_ld32(tmem + lane_addr + acc_col + c, a);
          tmem_ld32(tmem + lane_addr + acc_col + D + c, gk);
          if (add && in_srow) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              a[e] += p.sdv[srow + c + e];
              gk[e] += p.sdk[srow + c + e];
            }
          }
          if (key < p.N && in_rows) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              st_global_v4(dv + c + e, pack_bf16(a[e], a[e + 1]), pack_bf16(a[e + 2], a[e + 3]),
                           pack_bf16(a[e + 4], a[e + 5]), pack_bf16(a[e + 6], a[e + 7]));
              st_global_v4(dkp + c + e, pack_bf16(gk[e] * p.scale, gk[e + 1] * p.scale),
                           pack_bf16(gk[e + 2] * p.scale, gk[e + 3] * p.scale),
                           pack_bf16(gk[e + 4] * p.scale, gk[e + 5] * p.scale),
                           pack_bf16(gk[e + 6] * p.scale, gk[e + 7] * p.scale));
            }
          }
        }
      }
      if (MULTI && ok) {  // the set's accumulators read: a later tile may overwrite them
        tc_fence_before();
        mbar_arrive(bar(BwdBar::kAccFree + fs));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// SM: the local + strided mask (stride tiles before the window tiles).
template <int D, bool SM>
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                  const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * i; };
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + C::kOffBar + BwdBar::kWordsOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(words + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int qt = blockIdx.x;
  const int b = blockIdx.y / p.Hq, hq = blockIdx.y % p.Hq;
  const int hkv = hq / p.G;
  // key tiles of the row block: the compacted stride tiles with a key below
  // the last row's window (strided mask), then the window tiles from the one
  // holding the first row's window start to the diagonal tile
  const int Wc = imin(p.W, p.N);
  const int kt_lo = imax(0, qt * kBT - Wc + 1) / kBT;
  int nst = 0;
  if (SM) {
    const int r1 = imin(p.N - 1, qt * kBT + kBT - 1);
    nst = (stride_rows_below(imax(0, r1 - Wc + 1), p.S) + kBT - 1) / kBT;
  }
  const int nsteps = nst + (qt - kt_lo + 1);

  if (threadIdx.x == 0) {
    mbar_init(bar(BwdBar::kFixed), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(BwdBar::kFull + s), 1);
      mbar_init(bar(BwdBar::kEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(BwdBar::kS + h), 1);
      mbar_init(bar(BwdBar::kP + h), 128);
    }
    mbar_init(bar(BwdBar::kAcc), 1);
    mbar_init(bar(BwdBar::kFinal), 1);
    mbar_init(bar(BwdBar::kA), 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(words), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];

  if (warp == 0) {
    // ------------------------------------------------------ producer ---
    if (lane == 0) {
      const int zq = b * p.Hq + hq, zkv = b * p.Hkv + hkv;
      mbar_arrive_expect_tx(bar(BwdBar::kFixed), 2 * C::kTile);
      for (int bx = 0; bx < D / 64; ++bx) {
        if (!SWA_TMA_IN(bx * 64, D, qt * kBT, p.N, zq, p.B * p.Hq, p.err_flag)) continue;
        tma_load_3d(sbase + C::kOffA + bx * 16384, &tm_q, bar(BwdBar::kFixed), bx * 64, qt * kBT, zq);
        tma_load_3d(sbase + C::kOffB + bx * 16384, &tm_do, bar(BwdBar::kFixed), bx * 64, qt * kBT, zq);
      }
      int issued[C::kStages] = {0, 0};
      for (int s = 0; s < nsteps; ++s) {
        const int st = s & 1, use = s >> 1;
        if (use > 0 && !mbar_wait(bar(BwdBar::kEmpty + st), (use - 1) & 1, abort_flag)) {
          bwd_timeout(abort_flag, p.err_flag);
          break;
        }
        const bool strided = s < nst;
        const int row = (strided ? s : kt_lo + (s - nst)) * kBT;
        const uint32_t base = sbase + C::kOffStages + st * C::kStage;
        mbar_arrive_expect_tx(bar(BwdBar::kFull + st), 2 * C::kTile);
        const int krows = strided ? (p.N - 1) / p.S + 1 : p.N;
        (void)krows;
        for (int bx = 0; bx < D / 64; ++bx) {
          if (!SWA_TMA_IN(bx * 64, D, row, krows, zkv, p.B * p.Hkv, p.err_flag)) continue;
          tma_load_3d(base + bx * 16384, strided ? &tm_ks : &tm_k, bar(BwdBar::kFull + st), bx * 64, row, zkv);
          tma_load_3d(base + C::kTile + bx * 16384, strided ? &tm_vs : &tm_v, bar(BwdBar::kFull + st), bx * 64, row,
                      zkv);
        }
        issued[st] = use + 1;
      }
      if (*abort_flag) {
        mbar_wait_timed(bar(BwdBar::kFixed), 0);
        for (int st = 0; st < C::kStages; ++st)
          if (issued[st] > 0) mbar_wait_timed(bar(BwdBar::kFull + st), (issued[st] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA ---
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kBT, kBH, false);
      const uint32_t idesc_acc = idesc_bf16_f32(kBT, D, true);
      // the score products take Q and dO from TMEM (copied there once by the
      // elementwise warps): only the half's K or V tile is read from shared
      // memory, which an N = 64 product with both operands in shared memory
      // would be bound by
      bool ok = mbar_wait(bar(BwdBar::kA), 0, abort_flag);
      if (!ok) bwd_timeout(abort_flag, p.err_flag);
      tc_fence_after();
      // S = Q K^T and dP = dO V^T over keys 64h .. 64h+63 of step s (rows:
      // queries, columns: keys; the half's K and V rows start 8192 bytes
      // into each 64-column box)
      auto scores = [&](int s, int h) {
        const uint32_t cur = sbase + C::kOffStages + (s & 1) * C::kStage + h * 8192;
        const uint64_t k_k = sw128_desc(cur, 16, 1024);
        const uint64_t v_k = sw128_desc(cur + C::kTile, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          umma_bf16_ts(tmem + C::kColS + kBH * h, tmem + C::kColQ + kk * 8, k_k + off, idesc_s, kk > 0 ? 1u : 0u);
          umma_bf16_ts(tmem + C::kColDP + kBH * h, tmem + C::kColDO + kk * 8, v_k + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(BwdBar::kS + h));
      };
      // dQ += dS K over the half's 64 keys (dS as bf16 pairs in the half's
      // first 32 columns)
      auto accumulate = [&](int s, int h) {
        const uint64_t k_mn = sw128_desc(sbase + C::kOffStages + (s & 1) * C::kStage, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < kBH / 16; ++kk)
          umma_bf16_ts(tmem + C::kColAcc, tmem + C::kColS + kBH * h + kk * 8,
                       k_mn + (uint64_t)(((kBH / 16) * h + kk) * 2048 >> 4), idesc_acc,
                       (s == 0 && h == 0 && kk == 0) ? 0u : 1u);
      };
      if (ok && nsteps > 0) {
        ok = mbar_wait(bar(BwdBar::kFull), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          scores(0, 0);
          scores(0, 1);
        }
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        for (int h = 0; h < 2 && ok; ++h) {
          if (!mbar_wait(bar(BwdBar::kP + h), s & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          accumulate(s, h);
          if (h == 1) umma_commit(bar(BwdBar::kEmpty + (s & 1)));  // K and V of step s read
          if (s + 1 < nsteps) {
            if (h == 0) {
              if (!mbar_wait(bar(BwdBar::kFull + ((s + 1) & 1)), ((s + 1) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            scores(s + 1, h);  // into the columns the accumulation above reads first
          }
        }
      }
      if (ok) umma_commit(bar(BwdBar::kAcc));
      else bwd_timeout(abort_flag, p.err_flag);
      if (!ok || *abort_flag) {
        umma_commit(bar(BwdBar::kFinal));
        mbar_wait_timed(bar(BwdBar::kFinal), 0);
      }
    }
  } else {
    // --------------------------------------------------- elementwise ---
    const int qw = warp & 3;
    const int hh = (warp - 2) >> 2;  // the 64-key half this warp takes
    const int r = qw * 32 + lane;  // query row within the tile
    const int i = qt * kBT + r;
    const uint32_t lane_addr = static_cast<uint32_t>(qw * 32) << 16;
    const float sl2 = p.scale_log2;
    const int64_t rt = (int64_t)(b * p.Hq + hq) * p.npad + i;  // padded: always in bounds
    const bool rt_ok = SWA_IN(rt, 0, (int64_t)p.B * p.Hq * p.npad, p.err_flag);
    const float lse2 = rt_ok ? p.lse2[rt] : 0.f, dd = rt_ok ? p.dd[rt] : 0.f;
    // keys this row attends: the window's [wlo, whi], and the compacted
    // stride keys m < mst (those below the window start); none past N
    int wlo = 1, whi = 0, mst = 0;
    if (i < p.N) {
      wlo = imax(0, i - Wc + 1);
      whi = i;
      if (SM) mst = stride_rows_below(wlo, p.S);
    }
    bool ok = true;
    {
      // this row of Q (half-0 warps) or of dO (half-1 warps) into TMEM, the
      // score products' A operands: column j holds elements 2j and 2j + 1
      // (low half first), which is the row's own word order; the tiles
      // arrived with the 128-byte swizzle (16-byte chunk c of row r at chunk
      // c ^ (r % 8))
      const bool got = mbar_wait(bar(BwdBar::kFixed), 0, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) bwd_timeout(abort_flag, p.err_flag);
        ok = false;
      } else {
        const uint8_t* tile = smem + (hh ? C::kOffB : C::kOffA);
        uint32_t w[D / 2];
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + bx * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
            w[bx * 32 + 4 * c] = v.x;
            w[bx * 32 + 4 * c + 1] = v.y;
            w[bx * 32 + 4 * c + 2] = v.z;
            w[bx * 32 + 4 * c + 3] = v.w;
          }
        const uint32_t col = tmem + lane_addr + (hh ? C::kColDO : C::kColQ);
#pragma unroll
        for (int j = 0; j < D / 2; j += 32) tmem_st32_u(col + j, w + j);
        tc_fence_before();
        mbar_arrive(bar(BwdBar::kA));
      }
    }
    for (int s = 0; s < nsteps && ok; ++s) {
      const bool strided = SM && s < nst;
      const int kt = strided ? s : kt_lo + (s - nst);  // strided: compacted stride rows kt*128 ..
      const int h = hh;
      const bool got = mbar_wait(bar(BwdBar::kS + h), s & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) bwd_timeout(abort_flag, p.err_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const int kb = kt * kBT + kBH * h;  // the half's first key (strided: compacted index)
      const int c_lo = (strided ? 0 : wlo) - kb, c_hi = (strided ? mst - 1 : whi) - kb;  // attended columns
      const uint32_t s_col = tmem + lane_addr + C::kColS + kBH * h;
      uint32_t pk[32];
      if (__all_sync(0xffffffffu, c_hi < 0 || c_lo > kBH - 1 || c_lo > c_hi)) {
        // no row of this warp attends a key of this half: dS = 0, the scores
        // are not read
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = 0u;
      } else {
        float sv[64], dp[64];
        tmem_ld64(s_col, sv);
        tmem_ld64(tmem + lane_addr + C::kColDP + kBH * h, dp);
        auto body = [&](auto attended) {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const bool a0 = attended(c), a1 = attended(c + 1);
            const float p0 = a0 ? ex2_approx(fmaf(sv[c], sl2, -lse2)) : 0.f;
            const float p1 = a1 ? ex2_approx(fmaf(sv[c + 1], sl2, -lse2)) : 0.f;
            pk[c >> 1] = pack_bf16(p0 * (dp[c] - dd), p1 * (dp[c + 1] - dd));
          }
        };
        // every (query, key) cell of the warp's 32 x 64 block attended: no per-cell test
        if (__all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kBH - 1))
          body([](int) { return true; });
        else
          body([&](int c) { return c >= c_lo && c <= c_hi; });
      }
      // dS over S as bf16 pairs: the half's 64 keys in its own first 32
      // columns, already read
      tmem_st32_u(s_col, pk);
      tc_fence_before();
      mbar_arrive(bar(BwdBar::kP + h));
    }
    if (ok) {
      const bool got = mbar_wait(bar(BwdBar::kAcc), 0, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) bwd_timeout(abort_flag, p.err_flag);
        ok = false;
      }
    }
    if (ok) {  // the half's warps write their half of dQ's columns
      tc_fence_after();
      __nv_bfloat16* dq = reinterpret_cast<__nv_bfloat16*>(p.dq) + ((int64_t)(b * p.Hq + hq) * p.N + i) * D;
#pragma unroll 1
      for (int c = hh * (D / 2); c < (hh + 1) * (D / 2); c += 32) {
        float a[32];
        tmem_ld32(tmem + lane_addr + C::kColAcc + c, a);
        if (i < p.N && SWA_IN((int64_t)(b * p.Hq + hq) * p.N + i, 0, (int64_t)p.B * p.Hq * p.N, p.err_flag)) {
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            st_global_v4(dq + c + e, pack_bf16(a[e] * p.scale, a[e + 1] * p.scale),
                         pack_bf16(a[e + 2] * p.scale, a[e + 3] * p.scale),
                         pack_bf16(a[e + 4] * p.scale, a[e + 5] * p.scale),
                         pack_bf16(a[e + 6] * p.scale, a[e + 7] * p.scale));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_bwd_d(const BwdMaps& m, const BwdParams& p, cudaStream_t stream) {
  using C = BwdCfg<D>;
  {
    const void* kernels[5] = {reinterpret_cast<const void*>(bwd_dkdv_kernel<D, 0>),
                              reinterpret_cast<const void*>(bwd_dkdv_kernel<D, 1>),
                              reinterpret_cast<const void*>(bwd_dkdv_kernel<D, 2>),
                              reinterpret_cast<const void*>(bwd_dq_kernel<D, false>),
                              reinterpret_cast<const void*>(bwd_dq_kernel<D, true>)};
    for (const void* k : kernels) {
      const cudaError_t e = ensure_dynamic_smem(k, C::kSmemBytes);
      if (e != cudaSuccess) return e;
    }
  }
  const int64_t rows = (int64_t)p.B * p.Hq * p.npad;
  constexpr int kPrepRows = kPrepThreads / (D / 8);
  bwd_prep_kernel<D><<<(unsigned)((rows + kPrepRows - 1) / kPrepRows), kPrepThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nk = p.nq;  // key tiles of 128 (same count as query tiles)
  const dim3 gq(p.nq, p.B * p.Hq);
  // dK/dV grid over ncol x (B * Hkv) work tiles: a CTA per tile, or, when
  // the kernel runs several tiles per CTA, one CTA per SM
  auto dkdv_grid = [&](int ncol) -> dim3 {
    if (C::kFixedSets == 1) return dim3(ncol, p.B * p.Hkv);
    const int64_t ntiles = (int64_t)ncol * p.B * p.Hkv;
    return dim3((unsigned)(ntiles < p.num_ctas ? ntiles : p.num_ctas));
  };
  if (p.S > 0) {  // stride keys first: their partials feed the window pass
    const int nchunk = (p.nq + kStrideChunk - 1) / kStrideChunk;
    bwd_dkdv_kernel<D, 2><<<dkdv_grid(p.nspad / kBT * nchunk), kBwdThreads, C::kSmemBytes, stream>>>(
        m.q, m.k, m.v, m.dO, m.ks, m.vs, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_dkdv_kernel<D, 1><<<dkdv_grid(nk), kBwdThreads, C::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, m.ks, m.vs,
                                                                                    p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<D, true><<<gq, kDqThreads, C::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, m.ks, m.vs, p);
    return cudaGetLastError();
  }
  bwd_dkdv_kernel<D, 0><<<dkdv_grid(nk), kBwdThreads, C::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, m.ks, m.vs, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D, false><<<gq, kDqThreads, C::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, m.ks, m.vs, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BwdMaps& m, const BwdParams& p, int d, cudaStream_t stream) {
  if (d == 128) return launch_bwd_d<128>(m, p, stream);
  if (d == 64) return launch_bwd_d<64>(m, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
