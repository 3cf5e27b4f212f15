// prefill.cu -- masked attention forward on sm_100a (tcgen05 + TMA).
//
// Computes A = softmax(Q K^T * scale + log M) V ("Learn: Sparse &
// Sliding-Window Attention", section 3) for the window, local+strided and
// differential masks. The flash-style online softmax ("Attention Variants
// Compared", tiled_softmax_dot; "Exploring Attention Variants", Flash
// Attention section) keeps the N x N matrix off HBM.
//
// One CTA = one work unit of two "subs". A sub is 128 query rows of one head
// with its own score tile S and output accumulator O in tensor memory and its
// own softmax warpgroup. The two subs share the stream of K/V tiles:
//   * two heads of one GQA group, same rows (Hq/Hkv even);
//   * two consecutive 128-row query tiles of one head (otherwise);
//   * the two maps of differential attention (Q1/K1 and Q2/K2, shared V).
// While one softmax warpgroup works on its scores, the tensor core runs the
// other sub's MMAs, so the exponentials overlap the matrix products.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q once, then K and V tiles through a ring of
//               shared-memory slots.
//   warp 1      TMEM owner and MMA issuer. A sub's 128 score columns hold
//               one 128-key S (d = 128 and differential kernels) or two
//               64-key buffers, one per half of the key tile (d = 64 window
//               kernels). Per key tile (or half), as soon as a sub's P is
//               written, one elected lane issues for that sub
//               O_t += P V(prev) (A operand read from TMEM), then
//               S_t = Q_t K^T into the columns that held P, and the commits.
//               The tensor core runs MMAs in issue order, so P is read
//               before S overwrites it. The sub whose softmax finishes first
//               gets its next S first, so one sub's MMAs overlap the other
//               sub's exponentials; with two halves, S of one half also
//               overlaps the softmax of the other. The whole warp keeps the
//               bookkeeping, so the MMA operands are warp-uniform values.
//   warps 4-7   softmax of sub 0, warps 8-11 softmax of sub 1: one thread
//               per query row (TMEM lane), fp32 online softmax in the log2
//               domain, P as bf16 back into TMEM over the consumed scores,
//               lazy rescaling of O, then the epilogue O / l -> bf16.
// Every wait is bounded; on a timeout the CTA records SWA_ERR_TIMEOUT,
// drains what it has in flight, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "schedule.cuh"

namespace swa {

constexpr int BM = 128;  // query rows per sub (TMEM lanes)
constexpr int BN = 128;  // keys per tile (S columns of a sub)


// warp 0 producer, warp 1 MMA issuer, warps 4-11 softmax (warp w reaches
// TMEM lanes 32 * (w % 4) .. + 31). Warps 2-3 have no role: registers are
// allocated to whole groups of four warps, so dropping them would not raise
// the 168 registers a thread gets.
constexpr int kSmxWarp0 = 4;
constexpr int kThreads = 384;
// Lazy rescale threshold (log2 units): O and l keep a stale row max until a
// new score exceeds it by more than this, so P stays below 2^8.
constexpr float kRescaleTau = 8.0f;
// Scale of the mask's saturated FMA: |c - c0 +- 1/2| >= 1/2, so the product
// is far outside [0, 1] for every column either side of the edge.
constexpr float kMaskScale = 1e30f;


// Per-instantiation choices, measured on B200 (tcgen05 MMAs with M = 128 and
// both operands in shared memory cost about as much at N = 64 as at N = 128,
// because reading the operands takes as long as the math):
//   NH    score buffers per key tile and sub: 1 = one 128-key S (N = 128
//         MMAs), 2 = two 64-key halves, so S of one half runs during the
//         softmax of the other at twice the MMA cost per score;
//   POLY  of every 8 pairs of exponentials, how many are evaluated on the FMA
//         pipe (exp2_fma2) instead of the MUFU unit.
// d = 128 window kernels: one buffer (the MMA cost dominates); differential
// (d_qk = 64, d_v = 128): one buffer, 1 of 8 pairs on the FMA pipe; d = 64
// window and strided kernels (short units, MUFU-bound): two halves.
template <int DQK, int DV, bool DIFF>
struct PrefillTune {
#ifdef SWA_NH
  static constexpr int NH = SWA_NH;
#else
  static constexpr int NH = (DQK == 128 || DIFF) ? 1 : 2;
#endif
#ifdef SWA_POLY_PAIRS_PER_8
  static constexpr int POLY = SWA_POLY_PAIRS_PER_8;
#else
  static constexpr int POLY = DIFF ? 1 : 0;
#endif
  static_assert(NH == 1 || NH == 2, "one or two score buffers per tile");
};

// 2^x for a pair of floats on the FMA pipe (packed f32x2 arithmetic).
// Cody-Waite range reduction with round-to-nearest: x = n + f, n integer,
// f in [-1/2, 1/2]; adding and subtracting 1.5 * 2^23 rounds x to an integer
// held in the low mantissa bits of j. 2^f comes from a cubic with p(0) = 1
// whose other coefficients are a discrete minimax fit (linear programming)
// of the relative error on [-1/2, 1/2]; 2^n is added to the exponent field:
// the bit pattern of j times 2^23 is n << 23 modulo 2^32. Inputs at or
// below -127 (-inf included) are clamped to -127, where f = 0, p(0) = 1 and
// the result is exactly 0. Relative error of the fp32 evaluation: at most
// 1.02e-4 on [-125, 8].
constexpr float kExp2C1 = 0.6932829022407532f;
constexpr float kExp2C2 = 0.24221095442771912f;
constexpr float kExp2C3 = 0.05500892922282219f;
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 j = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(j, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  q = __ffma2_rn(q, f, make_float2(kExp2C1, kExp2C1));
  q = __ffma2_rn(q, f, make_float2(1.f, 1.f));
  return make_float2(__uint_as_float(__float_as_uint(j.x) * 8388608u + __float_as_uint(q.x)),
                     __uint_as_float(__float_as_uint(j.y) * 8388608u + __float_as_uint(q.y)));
}


// KV2: the two subs read different KV heads (kModeKvPairs); a ring slot then
// holds the K (or V) tiles of both.
template <int DQK, int DV, bool DIFF, bool KV2 = false>
struct PrefillCfg {
  static constexpr int kQBytes = BM * DQK * 2;
  static constexpr int kKBytes = BN * DQK * 2 * ((DIFF || KV2) ? 2 : 1);
  static constexpr int kVBytes = BN * DV * 2 * (KV2 ? 2 : 1);
  static constexpr int kSlot = kKBytes > kVBytes ? kKBytes : kVBytes;
  static constexpr int kStageBytes = 8 * 32 * 64 * 2;  // per softmax warp: 32 rows x 64 columns of bf16
  static constexpr int kTiles = 2 * kQBytes + kStageBytes;
  static constexpr int kBudget = 227 * 1024 - 1024 - 1024;  // minus alignment slack and barriers
  static constexpr int kSlotsRaw = (kBudget - kTiles) / kSlot;
  static constexpr int kSlots = kSlotsRaw > 8 ? 8 : kSlotsRaw;
  static_assert(kSlots >= 2, "shared memory too small for the K/V ring");
  static constexpr int kOffQ = 0;
  static constexpr int kOffStage = 2 * kQBytes;
  static constexpr int kOffSlots = kTiles;
  static constexpr int kOffBar = kTiles + kSlots * kSlot;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;  // barriers area + alignment slack
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol0 = 256;
  static constexpr int kOCol1 = 256 + DV;
  static_assert(256 + 2 * DV <= kTmemCols, "TMEM budget");
  static_assert(DQK == 64 || DQK == 128, "score bursts cover K = 64 or 128");
};

// Barrier block layout (8-byte mbarriers, then a few words).
struct BarLayout {
  static constexpr int kQ = 0;
  static constexpr int kFull = 1;       // + slot
  static constexpr int kEmpty = 9;      // + slot
  static constexpr int kS = 17;         // + 2 * sub + half: S_t,h written
  static constexpr int kP = 21;         // + 2 * sub + half: P_t,h written
  static constexpr int kO = 25;         // + sub: the unit's last PV done
  static constexpr int kX = 27;         // differential hand-off of 1/l2
  static constexpr int kFinal = 28;     // MMA drain on abort
  static constexpr int kQEmpty = 29;    // every S MMA of the unit done: Q may be replaced
  static constexpr int kOFree = 30;     // + sub: epilogue done reading O_t
  static constexpr int kLast = 32;      // + sub: PV of half 0 done where no S of half 0 follows
  static constexpr int kCount = 34;
  static constexpr int kWordsOff = 384; // bytes: tmem base, abort flag
  static constexpr int kF2Off = 512;    // bytes: 128 floats
  static_assert(kCount * 8 <= kWordsOff, "barrier block");
};

struct Unit {
  int b, hkv;
  int hkv1;  // KV head of sub 1 (differs from hkv in kModeKvPairs only)
  int hq[2];
  int qt[2];
  int valid[2];
};

// Unit u of the launch (heaviest query tiles first). The divisions by the
// group sizes go through the FastDivs the host builds (fd_u1: units per query
// tile, fd_u2: units per batch, fd_u3: head pairs per KV head, fd_g: Hq/Hkv).
__device__ __forceinline__ Unit decode_unit(const PrefillParams& p, int u) {
  Unit r;
  const int q1 = p.fd_u1(u);  // query tile (or tile pair) counted from the last
  const int bh = u - q1 * (int)p.fd_u1.d;
  r.b = p.fd_u2(bh);
  const int rem = bh - r.b * (int)p.fd_u2.d;
  if (p.mode == kModeHeadPairs) {
    r.hkv = p.fd_u3(rem);
    const int gp = rem - r.hkv * (int)p.fd_u3.d;
    r.hq[0] = r.hkv * p.G + 2 * gp;
    r.hq[1] = r.hq[0] + 1;
    r.qt[0] = r.qt[1] = p.nq - 1 - q1;
    r.valid[0] = r.valid[1] = 1;
  } else if (p.mode == kModeKvPairs) {
    // consecutive query heads 2j, 2j+1 at the same query tile; each reads
    // its own KV head (odd group sizes)
    r.hq[0] = 2 * rem;
    r.hq[1] = r.hq[0] + 1;
    r.hkv = p.fd_g(r.hq[0]);
    r.hkv1 = p.fd_g(r.hq[1]);
    r.qt[0] = r.qt[1] = p.nq - 1 - q1;
    r.valid[0] = r.valid[1] = 1;
    return r;
  } else if (p.mode == kModeTilePairs) {
    const int qp = (p.nq + 1) / 2 - 1 - q1;
    r.hq[0] = r.hq[1] = rem;
    r.hkv = p.fd_g(rem);
    r.qt[0] = 2 * qp;
    r.qt[1] = 2 * qp + 1;
    r.valid[0] = 1;
    r.valid[1] = r.qt[1] < p.nq;
  } else {  // differential: both maps of the same rows
    r.hq[0] = r.hq[1] = rem;
    r.hkv = p.fd_g(rem);
    r.qt[0] = r.qt[1] = p.nq - 1 - q1;
    r.valid[0] = r.valid[1] = 1;
  }
  r.hkv1 = r.hkv;
  return r;
}

// The unit's key items: stride tiles 0 .. nst-1, then window tiles
// blo .. bhi (union over the two subs, which is contiguous).
struct Items {
  QTileKeys k[2];
  int nst, blo, bhi, n;
};

// GEN: also the window + global-token kind (extra tiles of K/V itself); the
// window and strided kinds compile without that branch.
template <bool GEN>
__device__ __forceinline__ Items unit_items(const PrefillParams& p, const Unit& un) {
  Items it;
  it.nst = 0;
  it.blo = 0x7fffffff;
  it.bhi = -1;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (un.valid[t]) {
      it.k[t] = GEN ? qtile_keys(p.kind, p.N, p.W, p.S, BM, BN, un.qt[t], p.fd_s)
                    : qtile_keys_basic(p.kind, p.N, p.W, p.S, BM, BN, un.qt[t], p.fd_s);
      it.nst = imax(it.nst, it.k[t].n_stride);
      it.blo = imin(it.blo, it.k[t].band_lo);
      it.bhi = imax(it.bhi, it.k[t].band_hi);
    } else {
      it.k[t].band_lo = 1;
      it.k[t].band_hi = 0;
      it.k[t].n_stride = 0;
    }
  }
  it.n = it.nst + (it.bhi - it.blo + 1);
  return it;
}

__device__ __forceinline__ bool item_is_stride(const Items& it, int u) { return u < it.nst; }
__device__ __forceinline__ int item_tile(const Items& it, int u) {
  return u < it.nst ? u : it.blo + (u - it.nst);
}
__device__ __forceinline__ bool item_in_sub(const Items& it, int t, int u) {
  if (u < it.nst) return u < it.k[t].n_stride;
  const int kt = it.blo + (u - it.nst);
  return kt >= it.k[t].band_lo && kt <= it.k[t].band_hi;
}

__device__ __forceinline__ void record_timeout(volatile int* abort_flag, int* err_flag) {
  *abort_flag = 1;
  atomicExch(err_flag, 4 /* SWA_ERR_TIMEOUT */);
}

// GEN instantiations serve the window + global-token kind and strided views
// (dilated windows: rows r, r + dil, ... of each head, with the log-sum-exp
// written at the original rows); the others compile without that code.
template <int DQK, int DV, bool DIFF, bool GEN, bool KV2>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q2,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_k2,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ks,
                   const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_o,
                   const PrefillParams p, const RowMap rmap) {
  using C = PrefillCfg<DQK, DV, DIFF, KV2>;
  constexpr int NH = PrefillTune<DQK, DV, DIFF>::NH;
  constexpr int BH = BN / NH;  // keys per score buffer
  constexpr int kPolyPairsPer8 = PrefillTune<DQK, DV, DIFF>::POLY;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * i; };
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + C::kOffBar + BarLayout::kWordsOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(words + 1);
  float* f2s = reinterpret_cast<float*>(smem + C::kOffBar + BarLayout::kF2Off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // persistent CTAs: round r gives CTA c unit r*P + c (r even) or
  // r*P + P-1-c (r odd). Units come heaviest first, so the alternating
  // direction evens out the per-CTA totals.
  const int nunits = p.nunits, P = gridDim.x, c_id = blockIdx.x;
  auto unit_of = [&](int rnd) -> int { return rnd * P + ((rnd & 1) ? (P - 1 - c_id) : c_id); };
  // The first round from r on that gives this CTA a unit (-1: none left),
  // with the unit decoded and its key items listed. The MMA and softmax
  // warps call it for the next unit before they drain the current one, so
  // its integer work is off the path between units.
  auto next_unit = [&](int r, Unit& un, Items& it) -> int {
    for (; r * P < nunits; ++r) {
      const int ui = unit_of(r);
      if (ui < nunits) {
        un = decode_unit(p, ui);
        it = unit_items<GEN>(p, un);
        return r;
      }
    }
    return -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(BarLayout::kQ), 1);
    mbar_init(bar(BarLayout::kQEmpty), 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar(BarLayout::kFull + s), 1);
      mbar_init(bar(BarLayout::kEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      for (int h = 0; h < 2; ++h) {
        mbar_init(bar(BarLayout::kS + 2 * t + h), 1);
        mbar_init(bar(BarLayout::kP + 2 * t + h), 128);
      }
      mbar_init(bar(BarLayout::kO + t), 1);
      mbar_init(bar(BarLayout::kOFree + t), 128);
      mbar_init(bar(BarLayout::kLast + t), 1);
    }
    mbar_init(bar(BarLayout::kX), 128);
    mbar_init(bar(BarLayout::kFinal), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(words), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];

  if (warp == 0) {
    // ------------------------------------------------------ producer ---
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      if (DIFF) {
        tma_prefetch_map(&tm_q2);
        tma_prefetch_map(&tm_k2);
      }
      if (p.kind == kMaskStrided) {
        tma_prefetch_map(&tm_ks);
        tma_prefetch_map(&tm_vs);
      }
      int L = 0;      // K/V loads issued, across units
      int nq_ld = 0;  // Q loads issued (one per unit)
      int issued[8];
      for (int s = 0; s < 8; ++s) issued[s] = 0;
      bool ok = true;
      for (int rnd = 0; rnd * P < nunits && ok; ++rnd) {
        const int ui = unit_of(rnd);
        if (ui >= nunits) continue;
        const Unit un = decode_unit(p, ui);
        const Items it = unit_items<GEN>(p, un);
        // Q of this unit once every S MMA of the previous unit is done
        if (nq_ld > 0 && !mbar_wait(bar(BarLayout::kQEmpty), (nq_ld - 1) & 1, abort_flag)) {
          record_timeout(abort_flag, p.err_flag);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(BarLayout::kQ), (un.valid[0] + un.valid[1]) * C::kQBytes);
        for (int t = 0; t < 2; ++t) {
          if (!un.valid[t]) continue;
          const CUtensorMap* m = (DIFF && t == 1) ? &tm_q2 : &tm_q;
          for (int bx = 0; bx < DQK / 64; ++bx)
            if (SWA_TMA_IN(bx * 64, DQK, un.qt[t] * BM, p.N, un.b * p.Hq + un.hq[t], p.B * p.Hq, p.err_flag))
              tma_load_3d(sbase + C::kOffQ + t * C::kQBytes + bx * 16384, m, bar(BarLayout::kQ), bx * 64,
                          un.qt[t] * BM, un.b * p.Hq + un.hq[t]);
        }
        ++nq_ld;
        const int zkv = un.b * p.Hkv + un.hkv;
        const int zkv1 = un.b * p.Hkv + un.hkv1;
        for (int u = 0; u < it.n && ok; ++u) {
          const bool st = item_is_stride(it, u);
          const int row = item_tile(it, u) * BN;
          // rows of the view the tile comes from: the stride view holds
          // ceil(N / S) rows, the global keys' view is K/V itself
          const int vrows = (st && p.kind == kMaskStrided) ? (p.N - 1) / p.S + 1 : p.N;
          (void)vrows;
          {  // K (or K1 and K2)
            const int slot = L % C::kSlots, use = L / C::kSlots;
            ++L;
            if (use > 0 && !mbar_wait(bar(BarLayout::kEmpty + slot), (use - 1) & 1, abort_flag)) {
              record_timeout(abort_flag, p.err_flag);
              ok = false;
              break;
            }
            if (!(p.inject_timeout && ui == 0 && u == 0)) {
              mbar_arrive_expect_tx(bar(BarLayout::kFull + slot), C::kKBytes);
              const uint32_t dst = sbase + C::kOffSlots + slot * C::kSlot;
              const CUtensorMap* m = st ? &tm_ks : &tm_k;
              for (int bx = 0; bx < DQK / 64; ++bx)
                if (SWA_TMA_IN(bx * 64, DQK, row, vrows, zkv, p.B * p.Hkv, p.err_flag))
                  tma_load_3d(dst + bx * 16384, m, bar(BarLayout::kFull + slot), bx * 64, row, zkv);
              if (DIFF)
                for (int bx = 0; bx < DQK / 64; ++bx)
                  if (SWA_TMA_IN(bx * 64, DQK, row, vrows, zkv, p.B * p.Hkv, p.err_flag))
                    tma_load_3d(dst + BN * DQK * 2 + bx * 16384, &tm_k2, bar(BarLayout::kFull + slot), bx * 64,
                                row, zkv);
              if (KV2)  // sub 1's KV head
                for (int bx = 0; bx < DQK / 64; ++bx)
                  if (SWA_TMA_IN(bx * 64, DQK, row, vrows, zkv1, p.B * p.Hkv, p.err_flag))
                    tma_load_3d(dst + BN * DQK * 2 + bx * 16384, m, bar(BarLayout::kFull + slot), bx * 64, row,
                                zkv1);
              issued[slot] = use + 1;
            }
          }
          {  // V
            const int slot = L % C::kSlots, use = L / C::kSlots;
            ++L;
            if (use > 0 && !mbar_wait(bar(BarLayout::kEmpty + slot), (use - 1) & 1, abort_flag)) {
              record_timeout(abort_flag, p.err_flag);
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(BarLayout::kFull + slot), C::kVBytes);
            const uint32_t dst = sbase + C::kOffSlots + slot * C::kSlot;
            const CUtensorMap* m = st ? &tm_vs : &tm_v;
            for (int bx = 0; bx < DV / 64; ++bx)
              if (SWA_TMA_IN(bx * 64, DV, row, vrows, zkv, p.B * p.Hkv, p.err_flag))
                tma_load_3d(dst + bx * 16384, m, bar(BarLayout::kFull + slot), bx * 64, row, zkv);
            if (KV2)
              for (int bx = 0; bx < DV / 64; ++bx)
                if (SWA_TMA_IN(bx * 64, DV, row, vrows, zkv1, p.B * p.Hkv, p.err_flag))
                  tma_load_3d(dst + BN * DV * 2 + bx * 16384, m, bar(BarLayout::kFull + slot), bx * 64, row, zkv1);
            issued[slot] = use + 1;
          }
        }
      }
      if (!ok || *abort_flag) {
        // drain: every load issued lands before the CTA may exit
        for (int s = 0; s < C::kSlots; ++s)
          if (issued[s] > 0) mbar_wait_timed(bar(BarLayout::kFull + s), (issued[s] - 1) & 1);
        if (nq_ld > 0) mbar_wait_timed(bar(BarLayout::kQ), (nq_ld - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA ---
    // The whole warp runs the bookkeeping, so every operand is warp-uniform;
    // one elected lane issues each MMA burst and commit. Sub and half indices
    // are compile-time constants (generic lambdas over integral_constant),
    // so the issuer's state stays in registers.
    {
      // all lanes wait; the result is made warp-uniform
      auto wait = [&](uint32_t b, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag));
      };
      auto commit = [&](uint32_t b) {
        if (elect_one()) umma_commit(b);
        __syncwarp();
      };
      using I0 = std::integral_constant<int, 0>;
      using I1 = std::integral_constant<int, 1>;
      const uint32_t idesc_s = idesc_bf16_f32(BM, BH, false);
      const uint32_t idesc_pv = idesc_bf16_f32(BM, DV, true);
      const uint64_t q_desc_0 = sw128_desc(sbase + C::kOffQ, 16, 1024);
      const uint64_t q_desc_1 = sw128_desc(sbase + C::kOffQ + C::kQBytes, 16, 1024);
      struct SubMma {
        int npv0, npv1;  // PV products of half 0 / 1, across units (P phases)
        int nunit;       // units in which the sub took part (O-free phases)
        int ntot;        // key tiles of the sub in this unit
        int kcount;      // S tiles issued in this unit
        int pv_done;     // key tiles of this unit whose PVs (both halves) are issued
        bool pending;    // the previous item's PVs are still to issue
        int64_t dbg_row;
      };
      SubMma sm0 = {0, 0, 0, 0, 0, 0, false, -1}, sm1 = {0, 0, 0, 0, 0, 0, false, -1};
      int L = 0;
      int nq = 0;  // units started (Q phases)
      bool ok = true;
      Unit un;
      Items it;
      for (int rnd = next_unit(0, un, it); rnd >= 0 && ok;) {
        sm0.ntot = un.valid[0] ? qtile_nkeys(it.k[0]) : 0;
        sm1.ntot = un.valid[1] ? qtile_nkeys(it.k[1]) : 0;
        sm0.kcount = sm1.kcount = 0;
        sm0.pv_done = sm1.pv_done = 0;
        sm0.pending = sm1.pending = false;
        sm0.dbg_row = (un.valid[0] && p.dbg_tiles) ? (int64_t)(un.b * p.Hq + un.hq[0]) * p.nq + un.qt[0] : -1;
        sm1.dbg_row = (un.valid[1] && p.dbg_tiles && !DIFF) ? (int64_t)(un.b * p.Hq + un.hq[1]) * p.nq + un.qt[1] : -1;
        if (!wait(bar(BarLayout::kQ), nq & 1)) {
          if (lane == 0) record_timeout(abort_flag, p.err_flag);
          ok = false;
          break;
        }
        ++nq;
        tc_fence_after();
        int prev_vslot = -1, prev_vuse = 0;
        // One half-step of both subs: wait for both P_t,h, then one elected
        // lane issues, per sub, O_t += P_t,h V_h(prev) (P read from score
        // buffer h) and S_t,h = Q_t K_h^T into the same buffer, with their
        // commits. The tensor core runs MMAs in issue order, so P is read
        // before S overwrites it. `drain` issues the last item's PVs only.
        auto half_step = [&](auto hc, bool in0, bool in1, int kslot, int u, bool drain) -> bool {
          constexpr int h = decltype(hc)::value;
          int& npv0 = h ? sm0.npv1 : sm0.npv0;
          int& npv1 = h ? sm1.npv1 : sm1.npv0;
          const bool f0 = (h == 0 && sm0.pv_done == 0), f1 = (h == 0 && sm1.pv_done == 0);
          const uint64_t vdesc =
              sw128_desc(sbase + C::kOffSlots + prev_vslot * C::kSlot + h * (BH / 16) * 2048, 16384, 1024);
          const uint32_t kbase = sbase + C::kOffSlots + kslot * C::kSlot + h * BH * 128;
          const uint64_t kdesc0 = sw128_desc(kbase, 16, 1024);
          const uint64_t kdesc1 = sw128_desc(kbase + ((DIFF || KV2) ? BN * DQK * 2 : 0), 16, 1024);
          // sub 1's V tile (KV2: the second tile in the slot); the start
          // address field counts 16-byte units
          const uint64_t vdesc1 = vdesc + (KV2 ? (BN * DV * 2) >> 4 : 0);
          const bool o_done0 = h == NH - 1 && sm0.pending && sm0.pv_done + 1 == sm0.ntot;
          const bool o_done1 = h == NH - 1 && sm1.pending && sm1.pv_done + 1 == sm1.ntot;
          // PV of the previous key tile (A = P in TMEM over its scores), then S
          // of this one into the same columns; BH keys of P per PV
          auto pv = [&](uint32_t d, uint32_t a, uint64_t vd, uint32_t acc) {
            if (BH == 128) umma_ts_k8(d, a, vd, idesc_pv, acc);
            else umma_ts_k4(d, a, vd, idesc_pv, acc);
          };
          auto qk = [&](uint32_t d, uint64_t qd, uint64_t kd) {
            if (DQK == 128) umma_ss_k8(d, qd, kd, idesc_s, 0u);
            else umma_ss_k4(d, qd, kd, idesc_s, 0u);
          };
          // each sub's burst goes out as soon as that sub's P is written, so a
          // sub that finishes its softmax first gets its next S first
          if (sm0.pending && !wait(bar(BarLayout::kP + 0 + h), npv0 & 1)) return false;
          if (sm0.pending && f0 && sm0.nunit > 0 && !wait(bar(BarLayout::kOFree + 0), (sm0.nunit - 1) & 1))
            return false;
          tc_fence_after();
          if (elect_one()) {
            if (sm0.pending) {
              pv(tmem + C::kOCol0, tmem + h * BH, vdesc, f0 ? 0u : 1u);
              if (NH == 2 && h == 0 && !in0) umma_commit(bar(BarLayout::kLast + 0));  // no S of half 0 follows
              if (o_done0) umma_commit(bar(BarLayout::kO + 0));
            }
            if (in0) {
              qk(tmem + h * BH, q_desc_0, kdesc0);
              umma_commit(bar(BarLayout::kS + 0 + h));
            }
          }
          __syncwarp();
          if (sm1.pending && !wait(bar(BarLayout::kP + 2 + h), npv1 & 1)) return false;
          if (sm1.pending && f1 && sm1.nunit > 0 && !wait(bar(BarLayout::kOFree + 1), (sm1.nunit - 1) & 1))
            return false;
          tc_fence_after();
          if (elect_one()) {
            if (sm1.pending) {
              pv(tmem + C::kOCol1, tmem + BN + h * BH, vdesc1, f1 ? 0u : 1u);
              if (NH == 2 && h == 0 && !in1) umma_commit(bar(BarLayout::kLast + 1));
              if (o_done1) umma_commit(bar(BarLayout::kO + 1));
            }
            if (in1) {
              qk(tmem + BN + h * BH, q_desc_1, kdesc1);
              umma_commit(bar(BarLayout::kS + 2 + h));
            }
            if (h == NH - 1) {
              if (!drain) umma_commit(bar(BarLayout::kEmpty + kslot));                // K(u) read by its S
              if (prev_vslot >= 0) umma_commit(bar(BarLayout::kEmpty + prev_vslot));  // V(u-1) by its PVs
              if (!drain && u == it.n - 1) umma_commit(bar(BarLayout::kQEmpty));      // last S of the unit
            }
          }
          __syncwarp();
          if (sm0.pending) {
            ++npv0;
            if (h == NH - 1) ++sm0.pv_done;
          }
          if (sm1.pending) {
            ++npv1;
            if (h == NH - 1) ++sm1.pv_done;
          }
          if (h == 0 && lane == 0 && !drain) {
            const int tag = item_is_stride(it, u) ? (kStrideTag | item_tile(it, u)) : item_tile(it, u);
            const int64_t ndbg = (int64_t)p.B * p.Hq * p.nq;
            (void)ndbg;
            if (in0 && sm0.dbg_row >= 0 && sm0.kcount < p.dbg_cap && SWA_IN(sm0.dbg_row, 0, ndbg, p.err_flag))
              p.dbg_tiles[sm0.dbg_row * p.dbg_cap + sm0.kcount] = tag;
            if (in1 && sm1.dbg_row >= 0 && sm1.kcount < p.dbg_cap && SWA_IN(sm1.dbg_row, 0, ndbg, p.err_flag))
              p.dbg_tiles[sm1.dbg_row * p.dbg_cap + sm1.kcount] = tag;
          }
          if (h == 0) {
            sm0.kcount += in0;
            sm1.kcount += in1;
          }
          return true;
        };
        for (int u = 0; u < it.n; ++u) {
          const int kslot = L % C::kSlots, kuse = L / C::kSlots;
          ++L;
          const int vslot = L % C::kSlots, vuse = L / C::kSlots;
          ++L;
          if (!wait(bar(BarLayout::kFull + kslot), kuse & 1) ||
              ((sm0.pending || sm1.pending) && !wait(bar(BarLayout::kFull + prev_vslot), prev_vuse & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool in0 = item_in_sub(it, 0, u), in1 = item_in_sub(it, 1, u);
          if (!half_step(I0{}, in0, in1, kslot, u, false) ||
              (NH == 2 && !half_step(I1{}, in0, in1, kslot, u, false))) {
            ok = false;
            break;
          }
          sm0.pending = in0;
          sm1.pending = in1;
          prev_vslot = vslot;
          prev_vuse = vuse;
        }
        Unit un_next;
        Items it_next;
        const int rnd_next = ok ? next_unit(rnd + 1, un_next, it_next) : -1;
        if (ok && (sm0.pending || sm1.pending)) {
          ok = wait(bar(BarLayout::kFull + prev_vslot), prev_vuse & 1);
          if (ok) tc_fence_after();
          ok = ok && half_step(I0{}, false, false, 0, 0, true) &&
               (NH == 1 || half_step(I1{}, false, false, 0, 0, true));
        }
        if (!ok) {
          if (lane == 0) record_timeout(abort_flag, p.err_flag);
          break;
        }
        if (lane == 0 && sm0.dbg_row >= 0 && SWA_IN(sm0.dbg_row, 0, (int64_t)p.B * p.Hq * p.nq, p.err_flag))
          p.dbg_ntiles[sm0.dbg_row] = sm0.kcount;
        if (lane == 0 && sm1.dbg_row >= 0 && SWA_IN(sm1.dbg_row, 0, (int64_t)p.B * p.Hq * p.nq, p.err_flag))
          p.dbg_ntiles[sm1.dbg_row] = sm1.kcount;
        if (un.valid[0]) ++sm0.nunit;
        if (un.valid[1]) ++sm1.nunit;
        un = un_next;
        it = it_next;
        rnd = rnd_next;
      }
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) {
        commit(bar(BarLayout::kFinal));
        mbar_wait_timed(bar(BarLayout::kFinal), 0);
      }
    }
  } else if (warp >= kSmxWarp0) {
    // ------------------------------------------------------- softmax ---
    const int t = (warp - kSmxWarp0) >> 2;  // sub
    const int qw = warp & 3;             // TMEM lane quarter
    const int r = qw * 32 + lane;        // row within the sub's tile
    const uint32_t lane_addr = static_cast<uint32_t>(qw * 32) << 16;
    const uint32_t s_tmem = tmem + lane_addr + t * BN;
    const uint32_t o_tmem = tmem + lane_addr + (t == 0 ? C::kOCol0 : C::kOCol1);
    const int Wc = (p.kind == kMaskCausal) ? p.N : p.W;
    const float cl2 = p.scale_log2;
    const bool want_lse = !DIFF && p.lse != nullptr;
    // Epilogue store: this warp's 32 output rows go through a 4 KB
    // shared-memory box (128-byte swizzle), 64 columns at a time, and lane 0
    // writes the box with one TMA store; rows past N are clipped by TMA.
    const uint32_t stage = sbase + C::kOffStage + (warp - kSmxWarp0) * 4096;
    bool stage_used = false;
    auto store_rows = [&](bool& used, auto&& fetch, int zrow, int row0) {
#pragma unroll 1
      for (int h = 0; h < DV / 64; ++h) {
        if (used && lane == 0) bulk_wait_read();  // the previous box has been read out
        __syncwarp();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float v[32];
          fetch(64 * h + 32 * half, v);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t chunk = 4 * half + q4;  // 16-byte chunk of the 128-byte row
            const uint32_t addr = stage + lane * 128 + ((chunk ^ (lane & 7)) << 4);
            st_shared_v4(addr, pack_bf16(v[8 * q4], v[8 * q4 + 1]), pack_bf16(v[8 * q4 + 2], v[8 * q4 + 3]),
                         pack_bf16(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16(v[8 * q4 + 6], v[8 * q4 + 7]));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // a box whose rows all lie past N is clipped whole by the TMA unit
          if (SWA_TMA_IN(64 * h, DV, row0, p.nq * BM, zrow, p.B * p.Hq, p.err_flag))
            tma_store_3d(&tm_o, stage, 64 * h, row0, zrow);
          bulk_commit();
        }
        used = true;
      }
    };
    int kglob = 0;   // key tiles consumed, across units (S / P phases)
    int nlast = 0;   // kLast signals this sub's MMAs produce, across units
    int nunit = 0;   // units this sub took part in
    int nx = 0;      // differential hand-offs
    bool ok = true;

    Unit un;
    Items it;
    for (int rnd = next_unit(0, un, it); rnd >= 0 && ok;) {
      // this sub's fields as scalars: a run-time index into the unit's
      // arrays would keep them in local memory
      const bool valid_t = t ? un.valid[1] : un.valid[0];
      if (!valid_t) {
        rnd = next_unit(rnd + 1, un, it);
        continue;
      }
      const int qt_t = t ? un.qt[1] : un.qt[0];
      const int hq = t ? un.hq[1] : un.hq[0];
      const int ks_lo = t ? it.k[1].band_lo : it.k[0].band_lo;
      const int ks_hi = t ? it.k[1].band_hi : it.k[0].band_hi;
      const int ks_nst = t ? it.k[1].n_stride : it.k[0].n_stride;
      auto in_sub = [&](int u) -> bool {
        if (u < it.nst) return u < ks_nst;
        const int kt = it.blo + (u - it.nst);
        return kt >= ks_lo && kt <= ks_hi;
      };
      const int i = qt_t * BM + r;  // query index
      const bool row_ok = i < p.N;
      const int lo = window_lo(i, Wc);
      const int mst = GEN ? extra_rows_below(p.kind, lo, p.S, p.fd_s)  // extra-view rows below lo
                          : ((p.kind == kMaskStrided) ? stride_rows_below(lo, p.S, p.fd_s) : 0);
      float m_run = -INFINITY;  // running max, log2 units (scores * scale * log2 e)
      float l_run = 0.f;  // sum of the bf16 weights the PV products consume
      float l_exact = 0.f;  // sum of the unrounded weights (log-sum-exp only)
      long long cells = 0;

      for (int u = 0; u < it.n && ok; ++u) {
        if (!in_sub(u)) continue;
        // no S of half 0 follows this tile's PV of half 0 in this unit when
        // the next item is not this sub's: the MMA issuer signals kLast
        const bool last_run = !(u + 1 < it.n && in_sub(u + 1));
        // attended columns [c0, c1] of this row in this tile
        int c0, c1;
        const int tile = item_tile(it, u);
        if (item_is_stride(it, u)) {
          c0 = 0;
          c1 = imin(mst - 1 - tile * BN, BN - 1);
        } else {
          c0 = imax(lo - tile * BN, 0);
          c1 = imin(i - tile * BN, BN - 1);
        }
        if (!row_ok) { c0 = 1; c1 = 0; }
        if (c1 >= c0) cells += c1 - c0 + 1;

#pragma unroll 1
        for (int h = 0; h < NH; ++h) {
          const int c0h = c0 - h * BH, c1h = c1 - h * BH;  // attended columns of this half
          const bool full = (c0h <= 0 && c1h >= BH - 1);
          const bool got = mbar_wait(bar(BarLayout::kS + 2 * t + h), kglob & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got)) { if (lane == 0) record_timeout(abort_flag, p.err_flag); ok = false; break; }
          tc_fence_after();
          if (BH == 64 && __all_sync(0xffffffffu, c1h < c0h || c1h < 0 || c0h > BH - 1)) {
            // no row of this warp attends a column of this half (a window
            // edge, the stride view's unused keys, rows past N): P = 0 and
            // the row max and sum stand, so the scores are not read. (The
            // 128-column buffers of the d = 128 and differential kernels
            // meet such a tile only at rows past N: the vote would cost more
            // than it saves.)
            uint32_t zero[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) zero[e] = 0u;
            tmem_st32_u(s_tmem + h * BH, zero);
            tc_fence_before();
            mbar_arrive(bar(BarLayout::kP + 2 * t + h));
            continue;
          }

          float s[BH];
          if (BH == 128) tmem_ld128(s_tmem, s);
          else tmem_ld64(s_tmem + h * BH, s);
          float m_tile;
          if constexpr (BH == 64) {
            if (!__all_sync(0xffffffffu, full)) {
              // Masked columns become -FLT_MAX through FMA-pipe arithmetic
              // (the ALU pipe, at half the rate, carries the row max): a
              // saturated FMA gives the weight w = 1 for an attended column
              // and 0 for a masked one, then s' = s w + (w - 1) FLT_MAX, exact
              // in both cases. Most partial halves are cut on one side only
              // (the window's start, or the diagonal): test only the side
              // some row needs.
              const bool cut_lo = __any_sync(0xffffffffu, c0h > 0), cut_hi = __any_sync(0xffffffffu, c1h < BH - 1);
              const float blo = (0.5f - static_cast<float>(c0h)) * kMaskScale;  // c >= c0h: c k + blo > 0
              const float bhi = (static_cast<float>(c1h) + 0.5f) * kMaskScale;  // c <= c1h: bhi - c k > 0
              auto apply = [&](auto lo_side, auto hi_side) {
#pragma unroll
                for (int c = 0; c < BH; ++c) {
                  float w = 1.f;
                  if (decltype(lo_side)::value) w = fma_sat(static_cast<float>(c), kMaskScale, blo);
                  if (decltype(hi_side)::value) w *= fma_sat(static_cast<float>(c), -kMaskScale, bhi);
                  s[c] = fmaf(s[c], w, fmaf(w, FLT_MAX, -FLT_MAX));
                }
              };
              using T = std::true_type;
              using F = std::false_type;
              if (cut_lo && cut_hi) apply(T{}, T{});
              else if (cut_lo) apply(T{}, F{});
              else apply(F{}, T{});
            }
            // row max over 8 independent chains of three-input maxima
            float mx8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mx8[j] = s[j];
#pragma unroll
            for (int c = 8; c < BH; c += 2) mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], s[c], s[c + 1]);
            const float mx =
                fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
            // a row with no attended column here has the maximum -FLT_MAX
            m_tile = (mx == -FLT_MAX) ? -INFINITY : mx * cl2;
          } else {
            // 128-column tiles are partial only at a band's edges: select
            // -inf for masked columns; three-input maxima
            if (!__all_sync(0xffffffffu, full)) {
              const bool cut_lo = __any_sync(0xffffffffu, c0h > 0), cut_hi = __any_sync(0xffffffffu, c1h < BH - 1);
              if (cut_lo && cut_hi) {
#pragma unroll
                for (int c = 0; c < BH; ++c) s[c] = (c >= c0h && c <= c1h) ? s[c] : -INFINITY;
              } else if (cut_lo) {
#pragma unroll
                for (int c = 0; c < BH; ++c) s[c] = (c >= c0h) ? s[c] : -INFINITY;
              } else {
#pragma unroll
                for (int c = 0; c < BH; ++c) s[c] = (c <= c1h) ? s[c] : -INFINITY;
              }
            }
            float mx8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mx8[j] = s[j];
#pragma unroll
            for (int c = 8; c < BH; c += 2) mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], s[c], s[c + 1]);
            const float mx =
                fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
            m_tile = mx * cl2;  // -inf stays -inf
          }
          float m_use = m_run, alpha = 1.f;
          bool rescale = false;
          if (m_tile > m_run) {
            if (m_run == -INFINITY) {
              m_use = m_tile;  // nothing accumulated yet: the O row is 0 (or not yet written)
              alpha = 0.f;
            } else if (m_tile - m_run > kRescaleTau) {
              m_use = m_tile;
              alpha = ex2_approx(m_run - m_tile);
              rescale = true;
            }
          }
          const float msub = (m_use == -INFINITY) ? 0.f : m_use;
          // p = 2^(s * scale * log2 e - m): packed fp32 pairs for the scaling
          // and the row sum, MUFU ex2 for the exponential
          const float2 cl2x2 = make_float2(cl2, cl2), negm = make_float2(-msub, -msub);
          float2 rs2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
          float2 ex2s[2] = {{0.f, 0.f}, {0.f, 0.f}};
          uint32_t pk[BH / 2];
#pragma unroll
          for (int j = 0; j < BH / 2; ++j) {
            const float2 x = __ffma2_rn(make_float2(s[2 * j], s[2 * j + 1]), cl2x2, negm);
            float p0, p1;
            if ((j & 7) < kPolyPairsPer8) {
              const float2 e = exp2_fma2(x);
              p0 = e.x;
              p1 = e.y;
            } else {
              p0 = ex2_approx(x.x);
              p1 = ex2_approx(x.y);
            }
            pk[j] = pack_bf16(p0, p1);
            // the row sum adds the bf16 values the PV product consumes, so
            // the weights applied to V sum to one
            rs2[j & 3] = __fadd2_rn(rs2[j & 3], unpack_bf16(pk[j]));
            if (want_lse) ex2s[j & 1] = __fadd2_rn(ex2s[j & 1], make_float2(p0, p1));
          }
          const float2 rsum = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
          const float rs = rsum.x + rsum.y;
          l_run = l_run * alpha + rs;
          if (want_lse) {
            const float2 es = __fadd2_rn(ex2s[0], ex2s[1]);
            l_exact = l_exact * alpha + (es.x + es.y);
          }
          m_run = m_use;

          // P over the consumed scores: bf16 pairs, 32 columns per 64 keys
          tmem_st32_u(s_tmem + h * BH, pk);
          if (BH == 128) tmem_st32_u(s_tmem + 32, pk + 32);
          if (__any_sync(0xffffffffu, rescale)) {
            // O_t must hold every earlier PV before it is rescaled. One
            // buffer per tile: the commit of S_t (waited for above) follows
            // the PV of the previous tile, so O_t is complete already. Two
            // halves: for half 0, the S commit of this tile's half 1 follows
            // the previous PV of half 1; for half 1, this tile's PV of half 0
            // is followed by the next tile's S of half 0, or else by kLast.
            bool g = true;
            if (NH == 1) g = true;
            else if (h == 0) g = mbar_wait(bar(BarLayout::kS + 2 * t + 1), kglob & 1, abort_flag);
            else if (!last_run) g = mbar_wait(bar(BarLayout::kS + 2 * t), (kglob + 1) & 1, abort_flag);
            else g = mbar_wait(bar(BarLayout::kLast + t), nlast & 1, abort_flag);
            if (!__all_sync(0xffffffffu, g)) { if (lane == 0) record_timeout(abort_flag, p.err_flag); ok = false; break; }
            tc_fence_after();
            const float f = rescale ? alpha : 1.f;
#pragma unroll 1
            for (int c = 0; c < DV; c += 32) {
              float o[32];
              tmem_ld32(o_tmem + c, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= f;
              tmem_st32(o_tmem + c, o);
            }
          }
          tc_fence_before();
          mbar_arrive(bar(BarLayout::kP + 2 * t + h));
        }
        if (last_run) ++nlast;
        ++kglob;
      }
      if (!ok) break;
      Unit un_next;
      Items it_next;
      const int rnd_next = next_unit(rnd + 1, un_next, it_next);  // while the last PV runs

      // -------------------------------------------------- epilogue ---
      {
        const bool got = mbar_wait(bar(BarLayout::kO + t), nunit & 1, abort_flag);  // the sub's last PV
        if (!__all_sync(0xffffffffu, got)) { if (lane == 0) record_timeout(abort_flag, p.err_flag); ok = false; break; }
      }
      ++nunit;
      tc_fence_after();
      const int64_t orow = GEN ? (int64_t)(un.b * p.Hq + hq) * rmap.n + rmap.off + (int64_t)i * rmap.mul
                               : ((int64_t)(un.b * p.Hq + hq) * p.N + i);
      if (DIFF) {
        if (t == 1) {
          // hands lambda / l2 to sub 0, which reads both accumulators
          const float lam = SWA_IN(hq, 0, p.Hq, p.err_flag) ? p.lambda[hq] : 0.f;
          f2s[r] = (l_run > 0.f) ? lam / l_run : 0.f;
          tc_fence_before();
          mbar_arrive(bar(BarLayout::kX));
        } else {
          const bool g2 = mbar_wait(bar(BarLayout::kX), nx & 1, abort_flag);
          if (!__all_sync(0xffffffffu, g2)) { if (lane == 0) record_timeout(abort_flag, p.err_flag); ok = false; break; }
          ++nx;
          tc_fence_after();
          const float inv1 = 1.f / l_run;
          const float f2 = f2s[r];
          const uint32_t o2_tmem = tmem + lane_addr + C::kOCol1;
          store_rows(stage_used, [&](int c, float* v) {
            float b2[32];
            tmem_ld32(o_tmem + c, v);
            tmem_ld32(o2_tmem + c, b2);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = v[e] * inv1 - b2[e] * f2;
          }, un.b * p.Hq + hq, qt_t * BM + qw * 32);
          // both accumulators read: the next unit's first PVs may overwrite them
          tc_fence_before();
          mbar_arrive(bar(BarLayout::kOFree + 0));
          mbar_arrive(bar(BarLayout::kOFree + 1));
        }
      } else {
        const float inv = 1.f / l_run;
        store_rows(stage_used, [&](int c, float* v) {
          tmem_ld32(o_tmem + c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= inv;
        }, un.b * p.Hq + hq, qt_t * BM + qw * 32);
        tc_fence_before();
        mbar_arrive(bar(BarLayout::kOFree + t));  // O_t read: the next unit may overwrite it
        if (want_lse && row_ok && SWA_IN(orow, 0, (int64_t)p.B * p.Hq * (GEN ? rmap.n : p.N), p.err_flag))
          p.lse[orow] = (m_run + __log2f(l_exact)) * 0.6931471805599453f;
      }
      if (p.dbg_cells && !(DIFF && t == 1)) {
        long long c = row_ok ? cells : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
        const int64_t ci = (int64_t)(un.b * p.Hq + hq) * p.nq + qt_t;
        if (lane == 0 && SWA_IN(ci, 0, (int64_t)p.B * p.Hq * p.nq, p.err_flag))
          atomicAdd(reinterpret_cast<unsigned long long*>(p.dbg_cells + ci), static_cast<unsigned long long>(c));
      }
      un = un_next;
      it = it_next;
      rnd = rnd_next;
    }
  }

  if (warp >= kSmxWarp0 && lane == 0) bulk_wait_all();  // output stores complete before exit
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int DQK, int DV, bool DIFF, bool GEN = false, bool KV2 = false>
static cudaError_t launch_one(const PrefillMaps& maps, const PrefillParams& p, const RowMap& rows, int nunits,
                              cudaStream_t stream) {
  using C = PrefillCfg<DQK, DV, DIFF, KV2>;
  auto kern = prefill_kernel<DQK, DV, DIFF, GEN, KV2>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = nunits < p.num_ctas ? nunits : p.num_ctas;
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(maps.q, maps.q2, maps.k, maps.k2, maps.v, maps.ks, maps.vs,
                                                  maps.o, p, rows);
  return cudaGetLastError();
}

// Evaluates exp2_fma2 elementwise (y[i] = 2^x[i]), so that the polynomial
// the differential kernel uses for part of its exponentials can be checked
// against an error bound on its own.
__global__ void exp2_fma2_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t npair = (n + 1) / 2;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < npair; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = 2 * t;
    const bool two = i + 1 < n;
    const float2 r = exp2_fma2(make_float2(x[i], two ? x[i + 1] : x[i]));
    y[i] = r.x;
    if (two) y[i + 1] = r.y;
  }
}

cudaError_t launch_exp2_fma2(const float* x, float* y, int64_t n, cudaStream_t stream) {
  const int64_t npair = (n + 1) / 2;
  const int64_t blocks = (npair + 255) / 256;
  exp2_fma2_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillParams& p, const RowMap& rows, int dqk, int dv,
                           bool diff, int nunits, cudaStream_t stream) {
  if (diff) {
    if (dqk == 64 && dv == 128) return launch_one<64, 128, true>(maps, p, rows, nunits, stream);
    if (dqk == 64 && dv == 64) return launch_one<64, 64, true>(maps, p, rows, nunits, stream);
    return cudaErrorInvalidValue;
  }
  const bool gen = p.kind == kMaskGlobal || rows.mul != 1 || rows.off != 0 || rows.n != p.N;
  const bool kv2 = p.mode == kModeKvPairs;
  if (kv2 && !(dqk == 64 && dv == 64)) return cudaErrorInvalidValue;  // the host picks it at d = 64 only
  if (gen) {
    if (dqk == 128 && dv == 128) return launch_one<128, 128, false, true>(maps, p, rows, nunits, stream);
    if (dqk == 64 && dv == 64)
      return kv2 ? launch_one<64, 64, false, true, true>(maps, p, rows, nunits, stream)
                 : launch_one<64, 64, false, true>(maps, p, rows, nunits, stream);
    return cudaErrorInvalidValue;
  }
  if (dqk == 128 && dv == 128) return launch_one<128, 128, false>(maps, p, rows, nunits, stream);
  if (dqk == 64 && dv == 64)
    return kv2 ? launch_one<64, 64, false, false, true>(maps, p, rows, nunits, stream)
               : launch_one<64, 64, false>(maps, p, rows, nunits, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
