// diff_decode.cu -- one differential-attention decode step over a rolling
// W-slot cache on sm_100a.
//
// "Attention Variants -- Sliding Window, Sparse, Differential", The Problem:
// two softmax maps, softmax(q1 K1^T s) and softmax(q2 K2^T s), over the same
// keys, one subtracted from the other (w1 - lambda_h w2) and applied to one
// V. "Attention Variants Compared", symptom table: the first differential
// version's decode loads the value cache twice per step; here one pass reads
// every slot's K1, K2 and V bytes exactly once and feeds both maps.
// The window is the sliding one of "Learn: Sparse & Sliding-Window
// Attention", section 4: position p lives in slot p % W.
//
// Bound by HBM bandwidth, like the single-map step:
//   kernel 1 (split-KV): grid = (splits, B * Hkv). A slot row is 512 bytes
//     (K1 and K2 64 bf16 each, V 128 bf16) spread over 16 lanes: lane e
//     holds 8 columns of K1 (e < 8) or of K2 (e >= 8) and 8 columns of V.
//     Half-warp shuffles give map 1's score on lanes 0-7 and map 2's on
//     lanes 8-15; one more shuffle hands each lane both. Two fp32 online
//     softmaxes (log2 domain) per query head of the GQA group; partials
//     (m1, l1, m2, l2, o1, o2) go to the caller's workspace. The CTA that
//     holds slot pos % W stores the new token there first.
//   kernel 2 (combine): merges the splits of each map in a fixed order and
//     writes bf16(o1 / l1 - lambda_h o2 / l2).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace swa {

namespace {

constexpr int kDdThreads = 128;  // 4 warps
constexpr int kDdUnroll = 6;     // slot rows in flight per lane group
// registers capped so that 4 CTAs share an SM for groups of 1-2 query heads
// (larger groups hold more state per lane: 2 CTAs at G = 4, no cap at 8)
template <int G>
constexpr int dd_min_blocks() { return G <= 2 ? 4 : (G == 4 ? 2 : 1); }
constexpr int kDk = 64;          // query/key head dim of each map
constexpr int kDv = 128;         // value head dim
constexpr int kLpr = 16;         // lanes per slot row
constexpr int kRpw = 32 / kLpr;  // slot rows per warp per load
constexpr int kRowsPerIter = 4 * kRpw * kDdUnroll;

__host__ __device__ constexpr int diff_partial_stride() { return 4 + 2 * kDv; }

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// (m, l, acc) of one map merged with another lane's copy
__device__ __forceinline__ void merge_state(float& m, float& l, float* acc, int off) {
  const float mo = __shfl_xor_sync(0xffffffffu, m, off);
  const float lo = __shfl_xor_sync(0xffffffffu, l, off);
  const float mn = fmaxf(m, mo);
  const float a = (mn == -INFINITY) ? 0.f : ex2_approx(m - mn);
  const float ao = (mn == -INFINITY) ? 0.f : ex2_approx(mo - mn);
  l = l * a + lo * ao;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float xo = __shfl_xor_sync(0xffffffffu, acc[c], off);
    acc[c] = acc[c] * a + xo * ao;
  }
  m = mn;
}

template <int G>
__global__ void __launch_bounds__(kDdThreads, dd_min_blocks<G>()) diff_decode_split_kernel(const DiffDecodeParams p) {
  // a step may start while the previous step's merge runs; its partials and
  // cache writes wait until that grid is complete (programmatic dependent
  // launch), and the merge that follows may launch early
  grid_dependency_wait();
  launch_dependents();
  const int split = blockIdx.x;
  const int bk = blockIdx.y;  // b * Hkv + hkv
  const int b = bk / p.Hkv;
  const int hkv = bk % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = lane / kLpr;  // row within the warp's load
  const int e = lane % kLpr;   // 8-column group
  const bool map2 = e >= 8;    // this lane's key columns belong to K2
  const int kc8 = 8 * (e & 7); // first key column of the lane within its map

  const int pos = p.pos[b];
  const int nvalid = pos + 1 < p.W ? pos + 1 : p.W;  // slots in use: a prefix until the cache is full
  const int new_slot = pos % p.W;
  const int s0 = split * p.chunk;
  const int s1 = (s0 + p.chunk) < nvalid ? (s0 + p.chunk) : nvalid;

  // the lane's 8 query columns of its map, pre-scaled into the log2 domain
  const __nv_bfloat16* qsrc = reinterpret_cast<const __nv_bfloat16*>(map2 ? p.q2 : p.q1);
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(qsrc + ((int64_t)b * p.Hq + hkv * G + g) * kDk + kc8), f);
#pragma unroll
    for (int c = 0; c < 8; ++c) qv[g][c] = f[c] * p.scale_log2;
  }

  float m1[G], l1[G], a1[G][8], m2[G], l2[G], a2[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m1[g] = m2[g] = -INFINITY;
    l1[g] = l2[g] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) a1[g][c] = a2[g][c] = 0.f;
  }

  const int64_t row0 = (int64_t)bk * p.W;  // first slot row of this (b, kv head)
  const __nv_bfloat16* kcache = reinterpret_cast<const __nv_bfloat16*>(map2 ? p.k2_cache : p.k1_cache);
  const __nv_bfloat16* vcache = reinterpret_cast<const __nv_bfloat16*>(p.v_cache);
  const __nv_bfloat16* knew = reinterpret_cast<const __nv_bfloat16*>(map2 ? p.k2_new : p.k1_new) + (int64_t)bk * kDk;
  const __nv_bfloat16* vnew = reinterpret_cast<const __nv_bfloat16*>(p.v_new) + (int64_t)bk * kDv;

  for (int base = s0; base < s1; base += kRowsPerIter) {
    uint4 kr[kDdUnroll], vr[kDdUnroll];
    int slot[kDdUnroll];
#pragma unroll
    for (int u = 0; u < kDdUnroll; ++u) {
      slot[u] = base + (u * 4 + warp) * kRpw + rr;
      if (slot[u] < s1 && SWA_IN(slot[u], 0, p.W, p.err_flag)) {
        const int64_t kofs = (row0 + slot[u]) * kDk + kc8;
        const int64_t vofs = (row0 + slot[u]) * kDv + 8 * e;
        if (slot[u] == new_slot) {
          // the step writes before it attends: the new token replaces the oldest
          kr[u] = *reinterpret_cast<const uint4*>(knew + kc8);
          vr[u] = *reinterpret_cast<const uint4*>(vnew + 8 * e);
          *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(kcache) + kofs) = kr[u];
          *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(vcache) + vofs) = vr[u];
        } else {
          kr[u] = ld_stream(kcache + kofs);
          vr[u] = ld_stream(vcache + vofs);
        }
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    // scores: map 1 on lanes 0-7 of each 16-lane group, map 2 on lanes 8-15,
    // then every lane gets both
    float sc1[kDdUnroll][G], sc2[kDdUnroll][G];
#pragma unroll
    for (int u = 0; u < kDdUnroll; ++u) {
      float kf[8];
      unpack8(kr[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d0 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) d0 = fmaf(qv[g][c], kf[c], d0);
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) d0 += __shfl_xor_sync(0xffffffffu, d0, off);
        const float other = __shfl_xor_sync(0xffffffffu, d0, 8);
        const bool ok = slot[u] < s1;
        sc1[u][g] = ok ? (map2 ? other : d0) : -INFINITY;
        sc2[u][g] = ok ? (map2 ? d0 : other) : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx1 = m1[g], mx2 = m2[g];
#pragma unroll
      for (int u = 0; u < kDdUnroll; ++u) {
        mx1 = fmaxf(mx1, sc1[u][g]);
        mx2 = fmaxf(mx2, sc2[u][g]);
      }
      if (mx1 == -INFINITY) continue;  // nothing valid yet in this lane group (both maps alike)
      const float c1 = ex2_approx(m1[g] - mx1), c2 = ex2_approx(m2[g] - mx2);  // m = -inf -> 0
      l1[g] *= c1;
      l2[g] *= c2;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        a1[g][c] *= c1;
        a2[g][c] *= c2;
      }
#pragma unroll
      for (int u = 0; u < kDdUnroll; ++u) {
        const float w1 = ex2_approx(sc1[u][g] - mx1), w2 = ex2_approx(sc2[u][g] - mx2);
        float vf[8];
        unpack8(vr[u], vf);  // V read once, used by both maps
        l1[g] += w1;
        l2[g] += w2;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          a1[g][c] = fmaf(w1, vf[c], a1[g][c]);
          a2[g][c] = fmaf(w2, vf[c], a2[g][c]);
        }
      }
      m1[g] = mx1;
      m2[g] = mx2;
    }
  }

  // merge the two row groups of the warp (lanes e and e + 16)
#pragma unroll
  for (int g = 0; g < G; ++g) {
    merge_state(m1[g], l1[g], a1[g], kLpr);
    merge_state(m2[g], l2[g], a2[g], kLpr);
  }

  // merge the 4 warps through shared memory
  __shared__ float sm_ml[4][G][4];
  __shared__ __align__(16) float sm_acc[4][G][2][kDv];
  if (lane < kLpr) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (lane == 0) {
        sm_ml[warp][g][0] = m1[g];
        sm_ml[warp][g][1] = l1[g];
        sm_ml[warp][g][2] = m2[g];
        sm_ml[warp][g][3] = l2[g];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        sm_acc[warp][g][0][8 * e + c] = a1[g][c];
        sm_acc[warp][g][1][8 * e + c] = a2[g][c];
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * 2 * kDv; idx += kDdThreads) {
    const int g = idx / (2 * kDv), mp = (idx / kDv) & 1, c = idx % kDv;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_ml[w][g][2 * mp]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float a = (M == -INFINITY) ? 0.f : ex2_approx(sm_ml[w][g][2 * mp] - M);
      L += sm_ml[w][g][2 * mp + 1] * a;
      O += sm_acc[w][g][mp][c] * a;
    }
    const int64_t ri = (int64_t)(b * p.Hq + hkv * G + g) * p.nsplit + split;
    if (!SWA_IN(ri, 0, (int64_t)p.B * p.Hq * p.nsplit, p.err_flag)) continue;
    float* rec = p.partial + ri * diff_partial_stride();
    if (c == 0) {
      rec[2 * mp] = M;
      rec[2 * mp + 1] = L;
    }
    rec[4 + mp * kDv + c] = O;
  }
}

__global__ void __launch_bounds__(kDv) diff_decode_combine_kernel(const DiffDecodeParams p) {
  grid_dependency_wait();  // the split kernel's partials are complete and visible
  const int bh = blockIdx.x;  // b * Hq + hq
  const int c = threadIdx.x;
  if (!SWA_IN(bh, 0, p.B * p.Hq, p.err_flag)) return;
  const float* recs = p.partial + (int64_t)bh * p.nsplit * diff_partial_stride();
  float M1 = -INFINITY, M2 = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) {
    M1 = fmaxf(M1, recs[s * diff_partial_stride()]);
    M2 = fmaxf(M2, recs[s * diff_partial_stride() + 2]);
  }
  float L1 = 0.f, O1 = 0.f, L2 = 0.f, O2 = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float* r = recs + s * diff_partial_stride();
    const float x1 = (r[0] == -INFINITY) ? 0.f : ex2_approx(r[0] - M1);
    const float x2 = (r[2] == -INFINITY) ? 0.f : ex2_approx(r[2] - M2);
    L1 += r[1] * x1;
    O1 += r[4 + c] * x1;
    L2 += r[3] * x2;
    O2 += r[4 + kDv + c] * x2;
  }
  const float lam = p.lambda[bh % p.Hq];
  reinterpret_cast<__nv_bfloat16*>(p.o)[(int64_t)bh * kDv + c] = __float2bfloat16_rn(O1 / L1 - lam * (O2 / L2));
}

template <int G>
cudaError_t launch_dd(const DiffDecodeParams& p, cudaStream_t stream) {
  dim3 grid(p.nsplit, p.B * p.Hkv);
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t scfg = {};
  scfg.gridDim = grid;
  scfg.blockDim = dim3(kDdThreads);
  scfg.dynamicSmemBytes = 0;
  scfg.stream = stream;
  scfg.attrs = &pdl;
  scfg.numAttrs = 1;
  cudaLaunchKernelEx(&scfg, diff_decode_split_kernel<G>, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the merge may launch while the split grid drains; it waits on the
  // device for the split grid's partials (programmatic dependent launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * p.Hq);
  cfg.blockDim = dim3(kDv);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, diff_decode_combine_kernel, p);
  return cudaGetLastError();
}

}  // namespace

// Splits per (b, kv head): about 16 CTAs per SM in total (measured best on
// the 64 x 8 x 4096-slot step among 8, 16, 24 and 32), each a whole number
// of 64-slot blocks.
static int diff_decode_nsplit(int B, int Hkv, int W) {
  const int groups = B * Hkv;
  int ns = (16 * 148 + groups - 1) / groups;
  if (ns < 1) ns = 1;
  const int chunk = ((W + ns - 1) / ns + 63) / 64 * 64;
  return (W + chunk - 1) / chunk;
}

size_t diff_decode_partial_bytes(int B, int Hq, int Hkv, int W) {
  return (size_t)B * Hq * diff_decode_nsplit(B, Hkv, W) * diff_partial_stride() * sizeof(float);
}

cudaError_t launch_diff_decode(const DiffDecodeParams& p0, cudaStream_t stream) {
  DiffDecodeParams p = p0;
  p.err_flag = device_error_ptr();
  if (p.err_flag == nullptr) return cudaErrorUnknown;
  p.nsplit = diff_decode_nsplit(p.B, p.Hkv, p.W);
  p.chunk = ((p.W + p.nsplit - 1) / p.nsplit + 63) / 64 * 64;
  switch (p.G) {
    case 1: return launch_dd<1>(p, stream);
    case 2: return launch_dd<2>(p, stream);
    case 4: return launch_dd<4>(p, stream);
    case 8: return launch_dd<8>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace swa
