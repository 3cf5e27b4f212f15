// decode.cu -- one decode step over a rolling W-slot KV cache on sm_100a.
//
// "Learn: Sparse & Sliding-Window Attention", section 4: at decode time keep
// only the most recent w tokens' K/V, evicting the oldest; section 6: the
// cache stays O(w). Position p lives in slot p % W, so the W slots always
// hold positions max(0, pos-W+1) .. pos, in rotated order; softmax does not
// care about the order.
//
// The step reads the whole cache once, so it is bound by HBM bandwidth:
//   kernel 1 (split-KV): grid = (splits, B * Hkv). Each CTA streams one
//     contiguous slot range of one (b, kv head) with 16-byte loads and serves
//     all G = Hq/Hkv query heads of that group from the same K/V bytes
//     (GQA: each K/V byte is read once). A row of d bf16 is split over d/8
//     lanes; scores are reduced with shuffles; an fp32 online softmax in the
//     log2 domain keeps (m, l, o) per head. The CTA holding slot pos % W
//     takes the new token from k_new / v_new and stores it into that slot.
//     Partials (m, l, unnormalised o) go to the caller's workspace.
//   kernel 2 (combine): merges the splits of each (b, hq) in a fixed order
//     (deterministic) and writes bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/swa_attn.h"
#include "internal.h"
#include "ptx.cuh"

namespace swa {

constexpr int kDecThreads = 128;  // 4 warps
constexpr int kDecUnroll = 8;     // rows in flight per lane group
// registers capped so that 4 CTAs share an SM for groups of 1-2 query heads
// (larger groups hold more state per lane: 2 CTAs at G = 4, no cap at 8)
template <int G>
constexpr int dec_min_blocks() { return G <= 2 ? 4 : (G == 4 ? 2 : 1); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ int imin_dec(int a, int b) { return a < b ? a : b; }

// Record of one split's partial result: m, l, two pad words, then d floats.
__host__ __device__ constexpr int partial_stride(int d) { return d + 4; }

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, dec_min_blocks<G>())
    decode_split_kernel(const DecodeParams p) {
  // a step may start while the previous step's merge runs; its partials and
  // cache writes wait until that grid is complete (programmatic dependent
  // launch), and the merge that follows may launch early
  grid_dependency_wait();
  launch_dependents();
  constexpr int LPR = D / 8;         // lanes per cache row
  constexpr int RPW = 32 / LPR;      // rows per warp per load
  constexpr int ROWS_PER_ITER = 4 * RPW * kDecUnroll;

  const int split = blockIdx.x;
  const int bk = blockIdx.y;  // b * Hkv + hkv
  const int b = bk / p.Hkv;
  const int hkv = bk % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = lane / LPR;   // row within the warp's load
  const int e = lane % LPR;    // 8-element column group

  // Slots 0 .. n_sink-1 hold positions 0 .. n_sink-1 for good (attention
  // sinks); a later position p rotates through slot n_sink + (p-n_sink) % W.
  // The slots in use are always a prefix [0, nvalid) of the n_sink + W.
  const int pos = p.pos[b];
  const int nvalid = pos < p.n_sink ? pos + 1 : p.n_sink + imin_dec(p.W, pos + 1 - p.n_sink);
  const int new_slot = pos < p.n_sink ? pos : p.n_sink + (pos - p.n_sink) % p.W;
  const int s0 = split * p.chunk;
  const int s1 = (s0 + p.chunk) < nvalid ? (s0 + p.chunk) : nvalid;

  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q) + ((int64_t)b * p.Hq + hkv * G) * D;
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float f[8];
    bf16x8_to_float(*reinterpret_cast<const uint4*>(qb + g * D + 8 * e), f);
#pragma unroll
    for (int c = 0; c < 8; ++c) qv[g][c] = f[c] * p.scale_log2;
  }

  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[g][c] = 0.f;
  }

  const int64_t cache_base = (int64_t)bk * (p.n_sink + p.W) * D;
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.k_cache) + cache_base;
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.v_cache) + cache_base;
  const __nv_bfloat16* kn = reinterpret_cast<const __nv_bfloat16*>(p.k_new) + (int64_t)bk * D;
  const __nv_bfloat16* vn = reinterpret_cast<const __nv_bfloat16*>(p.v_new) + (int64_t)bk * D;

  for (int base = s0; base < s1; base += ROWS_PER_ITER) {
    uint4 kr[kDecUnroll], vr[kDecUnroll];
    int slot[kDecUnroll];
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      slot[u] = base + (u * 4 + warp) * RPW + rr;
      if (slot[u] < s1 && SWA_IN(slot[u], 0, p.n_sink + p.W, p.err_flag)) {
        if (slot[u] == new_slot) {
          kr[u] = *reinterpret_cast<const uint4*>(kn + 8 * e);
          vr[u] = *reinterpret_cast<const uint4*>(vn + 8 * e);
          // the step writes before it attends: the new token replaces the oldest
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.k_cache) + cache_base + (int64_t)slot[u] * D + 8 * e) = kr[u];
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.v_cache) + cache_base + (int64_t)slot[u] * D + 8 * e) = vr[u];
        } else {
          kr[u] = ld_stream_v4(kc + (int64_t)slot[u] * D + 8 * e);
          vr[u] = ld_stream_v4(vc + (int64_t)slot[u] * D + 8 * e);
        }
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float sc[kDecUnroll][G];
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      float kf[8];
      bf16x8_to_float(kr[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d0 = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) d0 = fmaf(qv[g][c], kf[c], d0);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) d0 += __shfl_xor_sync(0xffffffffu, d0, off);
        sc[u][g] = (slot[u] < s1) ? d0 : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = m[g];
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) mx = fmaxf(mx, sc[u][g]);
      if (mx == -INFINITY) continue;  // nothing valid yet in this lane group
      const float a = ex2_approx(m[g] - mx);  // m = -inf -> 0
      l[g] *= a;
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[g][c] *= a;
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const float w = ex2_approx(sc[u][g] - mx);
        float vf[8];
        bf16x8_to_float(vr[u], vf);
        l[g] += w;
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[g][c] = fmaf(w, vf[c], acc[g][c]);
      }
      m[g] = mx;
    }
  }

  // merge the RPW row groups of the warp (lanes e, e+LPR, ...)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[g], off);
      const float mn = fmaxf(m[g], mo);
      const float a = (mn == -INFINITY) ? 0.f : ex2_approx(m[g] - mn);
      const float ao = (mn == -INFINITY) ? 0.f : ex2_approx(mo - mn);
      l[g] = l[g] * a + lo * ao;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float xo = __shfl_xor_sync(0xffffffffu, acc[g][c], off);
        acc[g][c] = acc[g][c] * a + xo * ao;
      }
      m[g] = mn;
    }
  }

  // merge the 4 warps through shared memory
  __shared__ float sm_m[4][G], sm_l[4][G];
  __shared__ __align__(16) float sm_acc[4][G][D];
  if (lane < LPR) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (lane == 0) {
        sm_m[warp][g] = m[g];
        sm_l[warp][g] = l[g];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sm_acc[warp][g][8 * e + c] = acc[g][c];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += kDecThreads) {
    const int g = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float a = (M == -INFINITY) ? 0.f : ex2_approx(sm_m[w][g] - M);
      L += sm_l[w][g] * a;
      O += sm_acc[w][g][c] * a;
    }
    const int64_t ri = (int64_t)(b * p.Hq + hkv * G + g) * p.nsplit + split;
    if (!SWA_IN(ri, 0, (int64_t)p.B * p.Hq * p.nsplit, p.err_flag)) continue;
    float* rec = p.partial + ri * partial_stride(D);
    if (c == 0) {
      rec[0] = M;
      rec[1] = L;
    }
    rec[4 + c] = O;
  }
}

template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const DecodeParams p) {
  grid_dependency_wait();  // the split kernel's partials are complete and visible
  const int bh = blockIdx.x;  // b * Hq + hq
  const int c = threadIdx.x;
  if (!SWA_IN(bh, 0, p.B * p.Hq, p.err_flag)) return;
  const float* recs = p.partial + (int64_t)bh * p.nsplit * partial_stride(D);
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, recs[s * partial_stride(D)]);
  float L = 0.f, O = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float* r = recs + s * partial_stride(D);
    const float a = (r[0] == -INFINITY) ? 0.f : ex2_approx(r[0] - M);
    L += r[1] * a;
    O += r[4 + c] * a;
  }
  reinterpret_cast<__nv_bfloat16*>(p.o)[(int64_t)bh * D + c] = __float2bfloat16_rn(O / L);
}

int decode_nsplit(int B, int Hkv, int W) {
  const int groups = B * Hkv;
  // about 24 CTAs per SM in total (measured best on the 64 x 8 x 1024-slot
  // step among 8, 16, 24 and 32), each a whole number of 64-slot blocks
  int ns = (24 * 148 + groups - 1) / groups;
  if (ns < 1) ns = 1;
  int chunk = (W + ns - 1) / ns;
  chunk = ((chunk + 63) / 64) * 64;           // whole iterations of the load loop
  return (W + chunk - 1) / chunk;
}

static int decode_chunk(int B, int Hkv, int W) {
  const int ns = decode_nsplit(B, Hkv, W);
  int chunk = (W + ns - 1) / ns;
  return ((chunk + 63) / 64) * 64;
}

size_t decode_partial_bytes(int B, int Hq, int Hkv, int d, int slots) {
  return (size_t)B * Hq * decode_nsplit(B, Hkv, slots) * partial_stride(d) * sizeof(float);
}

template <int D, int G>
static cudaError_t launch_g(DecodeParams p, cudaStream_t stream) {
  dim3 grid(p.nsplit, p.B * p.Hkv);
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t scfg = {};
  scfg.gridDim = grid;
  scfg.blockDim = dim3(kDecThreads);
  scfg.dynamicSmemBytes = 0;
  scfg.stream = stream;
  scfg.attrs = &pdl;
  scfg.numAttrs = 1;
  cudaLaunchKernelEx(&scfg, decode_split_kernel<D, G>, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the merge may launch while the split grid drains; it waits on the
  // device for the split grid's partials (programmatic dependent launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * p.Hq);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p0, cudaStream_t stream) {
  DecodeParams p = p0;
  p.err_flag = device_error_ptr();
  if (p.err_flag == nullptr) return cudaErrorUnknown;
  p.nsplit = decode_nsplit(p.B, p.Hkv, p.n_sink + p.W);
  p.chunk = decode_chunk(p.B, p.Hkv, p.n_sink + p.W);
  if (p.d == 128) {
    switch (p.G) {
      case 1: return launch_g<128, 1>(p, stream);
      case 2: return launch_g<128, 2>(p, stream);
      case 4: return launch_g<128, 4>(p, stream);
      case 8: return launch_g<128, 8>(p, stream);
    }
  } else if (p.d == 64) {
    switch (p.G) {
      case 1: return launch_g<64, 1>(p, stream);
      case 2: return launch_g<64, 2>(p, stream);
      case 4: return launch_g<64, 4>(p, stream);
      case 8: return launch_g<64, 8>(p, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace swa

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: a plugin host that hands
// a library raw tensors but no allocator, or a serving loop that forbids
// allocation on its hot path. For them the split partials live in one fixed
// array compiled into this library. Every GPU that loads the library holds
// these bytes until the process exits, and every call shares them.

namespace swa {

constexpr size_t kStaticDecodeScratchBytes = 4u << 20;  // SWA_DECODE_STATIC_SCRATCH_BYTES
static_assert(kStaticDecodeScratchBytes == SWA_DECODE_STATIC_SCRATCH_BYTES, "header and library disagree");

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticDecodeScratchBytes];

// In host code `g_decode_scratch` names a host-side stand-in, not device
// memory, so the kernels receive the array's device address instead. It is
// looked up once per device, with that device current, on the first call.
static float* static_decode_scratch() {
  static float* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_decode_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<float*>(a);
  }
  return ptrs[dev];
}

}  // namespace swa

extern "C" swa_status_t swa_decode_step_static(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                               void* v_cache, const int32_t* pos, void* o, int B, int Hq, int Hkv,
                                               int d, int W, float scale, void* stream) {
  using namespace swa;
  auto a16 = [](const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(k_new) || !a16(v_new) || !a16(k_cache) || !a16(v_cache) || !a16(o) || pos == nullptr ||
      (reinterpret_cast<uintptr_t>(pos) & 3u))
    return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || W > (1 << 30) || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SWA_ERR_UNSUPPORTED;
  if (decode_partial_bytes(B, Hq, Hkv, d, W) > kStaticDecodeScratchBytes) return SWA_ERR_SCRATCH_TOO_SMALL;
  float* scratch = static_decode_scratch();
  if (scratch == nullptr) return SWA_ERR_CUDA;
  // Each split writes its whole record before the combine reads it, so the
  // array needs no clearing between calls.
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.q = q; p.k_new = k_new; p.v_new = v_new; p.k_cache = k_cache; p.v_cache = v_cache; p.pos = pos; p.o = o;
  p.partial = scratch;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.d = d; p.W = W; p.G = G;
  p.n_sink = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  return launch_decode(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}
