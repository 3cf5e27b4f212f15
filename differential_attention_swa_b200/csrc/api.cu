// api.cu -- the extern "C" entry points declared in include/swa_attn.h:
// argument checks (before any launch), TMA descriptor encoding, launches,
// the schedule export and the device error flag.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/swa_attn.h"
#include "internal.h"
#include "schedule.cuh"

namespace swa {

// Device word the kernels set when a bounded wait runs out.
__device__ int g_device_error = 0;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 3-D bf16 view (inner = head dim, rows, outer = batch*heads) with a
// 64 x 128 box and the 128-byte swizzle the MMA descriptors expect.
bool encode_rows(CUtensorMap* m, const void* base, int d, int64_t rows, int64_t outer, int64_t row_stride_el,
                 int64_t outer_stride_el, uint32_t box_rows = 128) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)row_stride_el * 2, (cuuint64_t)outer_stride_el * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device (cached per device; host
// threads may race to fill an entry, all with the same value).
int sm_count() {
  static std::atomic<int> counts[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dim_ok(int d) { return d == 64 || d == 128; }

// Row r of the attention problem (r < N) is row row_off + r*row_mul of each
// (b, head) in memory, whose heads hold N_full rows each (N_full < 0: N).
// The dilated window runs one such strided view per residue class.
swa_status_t run_prefill(int kind, bool diff, const void* q, const void* k, const void* q2, const void* k2,
                         const void* v, void* o, float* lse, const float* lambda, int B, int Hq, int Hkv, int N,
                         int dqk, int dv, int W, int S, float scale, const swa_debug_t* dbg, void* stream,
                         int N_full = -1, int row_mul = 1, int row_off = 0) {
  if (N_full < 0) N_full = N;
  if (row_mul < 1 || row_off < 0 || (int64_t)row_off + (int64_t)(N - 1) * row_mul >= N_full) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SWA_ERR_INVALID_ARG;
  if (diff && (!aligned16(q2) || !aligned16(k2) || lambda == nullptr)) return SWA_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || W < 1 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if (kind == kMaskStrided && S < 1) return SWA_ERR_INVALID_ARG;
  if (kind == kMaskGlobal && S < 0) return SWA_ERR_INVALID_ARG;
  // masked scores are carried as -FLT_MAX; scale * log2(e) >= 1e-30 keeps
  // their weights at exactly 0
  if (!(scale >= 1e-30f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if ((int64_t)B * Hq > (1 << 30) / 8) return SWA_ERR_INVALID_ARG;
  if (!head_dim_ok(dqk) || !head_dim_ok(dv)) return SWA_ERR_UNSUPPORTED;
  if (!diff && dqk != dv) return SWA_ERR_UNSUPPORTED;
  if (diff && dqk != 64) return SWA_ERR_UNSUPPORTED;  // K1 and K2 share one ring slot
  if (dbg && dbg->tiles && (dbg->tiles_cap < 1 || dbg->ntiles == nullptr)) return SWA_ERR_INVALID_ARG;
  if (!get_encoder()) return SWA_ERR_CUDA;

  const int G = Hq / Hkv;
  PrefillMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int64_t nB = (int64_t)B;
  auto at = [&](const void* base, int d) {  // first row of the view
    return static_cast<const void*>(static_cast<const uint16_t*>(base) + (int64_t)row_off * d);
  };
  const int64_t nf = N_full;
  bool ok = encode_rows(&maps.q, at(q, dqk), dqk, N, nB * Hq, (int64_t)row_mul * dqk, nf * dqk) &&
            encode_rows(&maps.k, at(k, dqk), dqk, N, nB * Hkv, (int64_t)row_mul * dqk, nf * dqk) &&
            encode_rows(&maps.v, at(v, dv), dv, N, nB * Hkv, (int64_t)row_mul * dv, nf * dv) &&
            encode_rows(&maps.o, at(o, dv), dv, N, nB * Hq, (int64_t)row_mul * dv, nf * dv, 32);
  if (ok && diff)
    ok = encode_rows(&maps.q2, at(q2, dqk), dqk, N, nB * Hq, (int64_t)row_mul * dqk, nf * dqk) &&
         encode_rows(&maps.k2, at(k2, dqk), dqk, N, nB * Hkv, (int64_t)row_mul * dqk, nf * dqk);
  if (ok && kind == kMaskStrided) {
    // stride row m is key m*S: a view whose row stride is S rows of K/V
    const int64_t rows = (N + (int64_t)S - 1) / S;
    ok = encode_rows(&maps.ks, k, dqk, rows, nB * Hkv, (int64_t)S * dqk, (int64_t)N * dqk) &&
         encode_rows(&maps.vs, v, dv, rows, nB * Hkv, (int64_t)S * dv, (int64_t)N * dv);
  }
  if (!ok) return SWA_ERR_INVALID_ARG;
  if (!diff) maps.q2 = maps.q, maps.k2 = maps.k;
  // global keys are the first rows of K/V themselves: the extra view is K/V
  if (kind != kMaskStrided) maps.ks = maps.k, maps.vs = maps.v;

  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.W = W;
  p.S = (kind == kMaskStrided || kind == kMaskGlobal) ? S : 0;  // stride, or number of global tokens
  p.G = G; p.kind = kind;
  p.nq = (N + 127) / 128;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o; p.lse = lse; p.lambda = lambda;
  if (dbg) {
    p.dbg_cells = dbg->cells;
    p.dbg_tiles = dbg->tiles;
    p.dbg_ntiles = dbg->ntiles;
    p.dbg_cap = dbg->tiles_cap;
    p.inject_timeout = dbg->inject_timeout;
  }
  int64_t nunits;
  if (diff) {
    p.mode = kModeDiff;
    nunits = nB * Hq * p.nq;
  } else if (G % 2 == 0) {
    p.mode = kModeHeadPairs;
    nunits = nB * Hkv * (G / 2) * p.nq;
  } else if (Hq % 2 == 0 && dqk == 64) {
    // odd group size: pair consecutive query heads at the same query tile,
    // each with its own KV head, so both subs visit the same key tiles
    p.mode = kModeKvPairs;
    nunits = nB * (Hq / 2) * p.nq;
  } else {
    p.mode = kModeTilePairs;
    nunits = nB * Hq * ((p.nq + 1) / 2);
  }
  if (nunits > 0x7fffffff) return SWA_ERR_INVALID_ARG;
  p.nunits = (int)nunits;
  // the divisors decode_unit uses (units per query tile, per batch, per KV
  // head), the group size, and the stride clamped to N (a stride at or
  // beyond N leaves key 0 as the only stride key either way)
  if (p.mode == kModeHeadPairs) {
    p.fd_u1 = make_fastdiv(B * Hkv * (G / 2));
    p.fd_u2 = make_fastdiv(Hkv * (G / 2));
    p.fd_u3 = make_fastdiv(G / 2);
  } else if (p.mode == kModeKvPairs) {
    p.fd_u1 = make_fastdiv(B * (Hq / 2));
    p.fd_u2 = make_fastdiv(Hq / 2);
    p.fd_u3 = make_fastdiv(1);
  } else {
    p.fd_u1 = make_fastdiv(B * Hq);
    p.fd_u2 = make_fastdiv(Hq);
    p.fd_u3 = make_fastdiv(1);
  }
  p.fd_g = make_fastdiv(G);
  p.fd_s = make_fastdiv(kind == kMaskStrided ? (S < N ? S : N) : 1);
  p.num_ctas = sm_count();
  if (p.num_ctas <= 0) return SWA_ERR_CUDA;
  p.err_flag = device_error_ptr();
  if (p.err_flag == nullptr) return SWA_ERR_CUDA;
  RowMap rows;
  rows.n = N_full;
  rows.off = row_off;
  rows.mul = row_mul;
  cudaError_t e = launch_prefill(maps, p, rows, dqk, dv, diff, (int)nunits, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

}  // namespace

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;  // (kernel, device)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done.insert({kernel, dev});
  return cudaSuccess;
}

int* device_error_ptr() {
  static int* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(a);
  }
  return ptrs[dev];
}

int read_and_clear_device_error(cudaStream_t stream, int* err) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
  int zero = 0;
  if (cudaMemcpyFromSymbol(err, g_device_error, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  return 0;
}

}  // namespace swa

namespace swa {
namespace {
swa_status_t run_decode(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                        const int32_t* pos, void* o, int B, int Hq, int Hkv, int d, int n_sink, int W, float scale,
                        void* workspace, size_t ws_bytes, void* stream) {
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(o) || pos == nullptr || (reinterpret_cast<uintptr_t>(pos) & 3u))
    return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || n_sink < 0 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if ((int64_t)n_sink + W > (1 << 30)) return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SWA_ERR_UNSUPPORTED;
  const size_t need = decode_partial_bytes(B, Hq, Hkv, d, n_sink + W);
  if (!aligned16(workspace) || ws_bytes < need) return SWA_ERR_INVALID_ARG;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.k_new = k_new; p.v_new = v_new; p.k_cache = k_cache; p.v_cache = v_cache; p.pos = pos; p.o = o;
  p.partial = static_cast<float*>(workspace);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.d = d; p.W = W; p.G = G; p.n_sink = n_sink;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = launch_decode(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}
// Backward of the window (S = 0) or local + strided (S >= 1) attention.
swa_status_t run_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int W, int S, float scale,
                     void* workspace, size_t ws_bytes, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || W < 1 || S < 0 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if ((int64_t)B * Hq > (1 << 30) / 8 || N > (1 << 30)) return SWA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SWA_ERR_UNSUPPORTED;
  const int64_t npad = ((int64_t)N + 127) / 128 * 128;
  const int64_t nspad = S > 0 ? (((int64_t)N + S - 1) / S + 127) / 128 * 128 : 0;
  const size_t need = (size_t)(2 * (int64_t)B * Hq * npad * 4 + 2 * (int64_t)B * Hkv * nspad * d * 4);
  if (!aligned16(workspace) || ws_bytes < need) return SWA_ERR_INVALID_ARG;
  if (!get_encoder()) return SWA_ERR_CUDA;
  const int64_t nB = B;
  BwdMaps m;
  std::memset(&m, 0, sizeof(m));
  bool ok = encode_rows(&m.q, q, d, N, nB * Hq, d, (int64_t)N * d) &&
            encode_rows(&m.k, k, d, N, nB * Hkv, d, (int64_t)N * d) &&
            encode_rows(&m.v, v, d, N, nB * Hkv, d, (int64_t)N * d) &&
            encode_rows(&m.dO, d_o, d, N, nB * Hq, d, (int64_t)N * d);
  if (ok && S > 0) {
    // stride row m is key m*S: a view whose row stride is S rows of K/V
    const int64_t rows = ((int64_t)N + S - 1) / S;
    ok = encode_rows(&m.ks, k, d, rows, nB * Hkv, (int64_t)S * d, (int64_t)N * d) &&
         encode_rows(&m.vs, v, d, rows, nB * Hkv, (int64_t)S * d, (int64_t)N * d);
  } else {
    m.ks = m.k;
    m.vs = m.v;
  }
  if (!ok) return SWA_ERR_INVALID_ARG;
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.o = o; p.dO = d_o; p.dq = dq; p.dk = dk; p.dv = dv; p.lse = lse;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.W = W; p.G = Hq / Hkv;
  p.nq = (int)(npad / 128);
  p.npad = (int)npad;
  p.S = S;
  p.nspad = (int)nspad;
  p.lse2 = static_cast<float*>(workspace);
  p.dd = p.lse2 + (int64_t)B * Hq * npad;
  p.sdk = S > 0 ? p.dd + (int64_t)B * Hq * npad : nullptr;
  p.sdv = S > 0 ? p.sdk + (int64_t)B * Hkv * nspad * d : nullptr;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_ctas = sm_count();
  if (p.num_ctas < 1) return SWA_ERR_CUDA;
  p.err_flag = device_error_ptr();
  if (p.err_flag == nullptr) return SWA_ERR_CUDA;
  cudaError_t e = launch_backward(m, p, d, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}
}  // namespace
}  // namespace swa

using namespace swa;

extern "C" {

swa_status_t swa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int N, int d, int W, float scale, void* stream) {
  return run_prefill(kMaskWindow, false, q, k, nullptr, nullptr, v, o, lse, nullptr, B, Hq, Hkv, N, d, d, W, 0,
                     scale, nullptr, stream);
}

swa_status_t strided_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int N, int d, int W, int stride, float scale, void* stream) {
  if (stride < 1) return SWA_ERR_INVALID_ARG;
  return run_prefill(kMaskStrided, false, q, k, nullptr, nullptr, v, o, lse, nullptr, B, Hq, Hkv, N, d, d, W,
                     stride, scale, nullptr, stream);
}

swa_status_t global_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                             int Hkv, int N, int d, int W, int n_global, float scale, void* stream) {
  if (n_global < 0) return SWA_ERR_INVALID_ARG;
  return run_prefill(kMaskGlobal, false, q, k, nullptr, nullptr, v, o, lse, nullptr, B, Hq, Hkv, N, d, d, W,
                     n_global, scale, nullptr, stream);
}

swa_status_t dilated_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int N, int d, int W, int dilation, float scale, void* stream) {
  if (dilation < 1 || N < 1) return SWA_ERR_INVALID_ARG;
  // residue class r (rows r, r + dilation, ...) is a plain window of W keys
  // over the same class of keys: one strided view each
  for (int r = 0; r < dilation && r < N; ++r) {
    const int rows = (N - r + dilation - 1) / dilation;
    const swa_status_t st = run_prefill(kMaskWindow, false, q, k, nullptr, nullptr, v, o, lse, nullptr, B, Hq, Hkv,
                                        rows, d, d, W, 0, scale, nullptr, stream, N, dilation, r);
    if (st != SWA_OK) return st;
  }
  return SWA_OK;
}

swa_status_t diff_attn_fwd(const void* q1, const void* k1, const void* q2, const void* k2, const void* v, void* o,
                           const float* lambda, int B, int Hq, int Hkv, int N, int d_qk, int d_v, int W, float scale,
                           void* stream) {
  return run_prefill(kMaskWindow, true, q1, k1, q2, k2, v, o, nullptr, lambda, B, Hq, Hkv, N, d_qk, d_v, W, 0,
                     scale, nullptr, stream);
}

swa_status_t swa_prefill_debug(int kind, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                               int Hq, int Hkv, int N, int d, int W, int stride, float scale, const swa_debug_t* dbg,
                               void* stream) {
  if (kind != kMaskWindow && kind != kMaskStrided && kind != kMaskGlobal) return SWA_ERR_INVALID_ARG;
  return run_prefill(kind, false, q, k, nullptr, nullptr, v, o, lse, nullptr, B, Hq, Hkv, N, d, d, W, stride, scale,
                     dbg, stream);
}

size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W) {
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || W > (1 << 30) || Hq % Hkv != 0 || (d != 64 && d != 128)) return 0;
  return decode_partial_bytes(B, Hq, Hkv, d, W);
}

swa_status_t swa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* pos, void* o, int B, int Hq, int Hkv, int d, int W, float scale,
                             void* workspace, size_t ws_bytes, void* stream) {
  return run_decode(q, k_new, v_new, k_cache, v_cache, pos, o, B, Hq, Hkv, d, 0, W, scale, workspace, ws_bytes,
                    stream);
}

swa_status_t swa_sink_decode_step(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                  void* v_cache, const int32_t* pos, void* o, int B, int Hq, int Hkv, int d,
                                  int n_sink, int W, float scale, void* workspace, size_t ws_bytes, void* stream) {
  return run_decode(q, k_new, v_new, k_cache, v_cache, pos, o, B, Hq, Hkv, d, n_sink, W, scale, workspace,
                    ws_bytes, stream);
}

size_t swa_sink_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int n_sink, int W) {
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || n_sink < 0 || (int64_t)n_sink + W > (1 << 30) || Hq % Hkv != 0 ||
      (d != 64 && d != 128))
    return 0;
  return decode_partial_bytes(B, Hq, Hkv, d, n_sink + W);
}

size_t swa_diff_decode_workspace_bytes(int B, int Hq, int Hkv, int d_qk, int d_v, int W) {
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || W > (1 << 30) || Hq % Hkv != 0 || d_qk != 64 || d_v != 128) return 0;
  return diff_decode_partial_bytes(B, Hq, Hkv, W);
}

swa_status_t swa_diff_decode_step(const void* q1, const void* q2, const void* k1_new, const void* k2_new,
                                  const void* v_new, void* k1_cache, void* k2_cache, void* v_cache,
                                  const int32_t* pos, const float* lambda, void* o, int B, int Hq, int Hkv, int d_qk,
                                  int d_v, int W, float scale, void* workspace, size_t ws_bytes, void* stream) {
  if (!aligned16(q1) || !aligned16(q2) || !aligned16(k1_new) || !aligned16(k2_new) || !aligned16(v_new) ||
      !aligned16(k1_cache) || !aligned16(k2_cache) || !aligned16(v_cache) || !aligned16(o) || pos == nullptr ||
      (reinterpret_cast<uintptr_t>(pos) & 3u) || lambda == nullptr || (reinterpret_cast<uintptr_t>(lambda) & 3u))
    return SWA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || W < 1 || Hq % Hkv != 0 || W > (1 << 30)) return SWA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SWA_ERR_INVALID_ARG;
  if (d_qk != 64 || d_v != 128) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SWA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || ws_bytes < diff_decode_partial_bytes(B, Hq, Hkv, W)) return SWA_ERR_INVALID_ARG;
  DiffDecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q1 = q1; p.q2 = q2; p.k1_new = k1_new; p.k2_new = k2_new; p.v_new = v_new;
  p.k1_cache = k1_cache; p.k2_cache = k2_cache; p.v_cache = v_cache; p.o = o;
  p.pos = pos; p.lambda = lambda; p.partial = static_cast<float*>(workspace);
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.W = W; p.G = G;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = launch_diff_decode(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

size_t swa_attn_bwd_workspace_bytes(int B, int Hq, int N) {
  if (B < 1 || Hq < 1 || N < 1) return 0;
  const int64_t npad = ((int64_t)N + 127) / 128 * 128;
  return (size_t)(2 * (int64_t)B * Hq * npad * (int64_t)sizeof(float));
}

size_t strided_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int stride) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || stride < 1 || (d != 64 && d != 128)) return 0;
  const int64_t nspad = (((int64_t)N + stride - 1) / stride + 127) / 128 * 128;
  return swa_attn_bwd_workspace_bytes(B, Hq, N) + (size_t)(2 * (int64_t)B * Hkv * nspad * d * (int64_t)sizeof(float));
}

swa_status_t swa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                          const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int W,
                          float scale, void* workspace, size_t ws_bytes, void* stream) {
  return run_bwd(q, k, v, o, d_o, lse, dq, dk, dv, B, Hq, Hkv, N, d, W, 0, scale, workspace, ws_bytes, stream);
}

swa_status_t strided_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                              const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                              int W, int stride, float scale, void* workspace, size_t ws_bytes, void* stream) {
  if (stride < 1) return SWA_ERR_INVALID_ARG;
  return run_bwd(q, k, v, o, d_o, lse, dq, dk, dv, B, Hq, Hkv, N, d, W, stride, scale, workspace, ws_bytes, stream);
}

int64_t swa_schedule(int kind, int N, int W, int stride, int Bq, int Bk, int32_t* qtile_offsets, int32_t* tiles,
                     int64_t cap) {
  if (N < 1 || Bq < 1 || Bk < 1 || kind < 0 || kind > 3) return -1;
  if (kind != kMaskCausal && W < 1) return -1;
  if (kind == kMaskStrided && stride < 1) return -1;
  if (kind == kMaskGlobal && stride < 0) return -1;
  const int nq = (N + Bq - 1) / Bq;
  int64_t n = 0;
  for (int qt = 0; qt < nq; ++qt) {
    if (qtile_offsets) qtile_offsets[qt] = (int32_t)n;
    const QTileKeys keys = qtile_keys(kind, N, W, stride, Bq, Bk, qt);
    const int cnt = qtile_nkeys(keys);
    for (int e = 0; e < cnt; ++e, ++n)
      if (tiles && n < cap) tiles[n] = qtile_entry(keys, e);
  }
  if (qtile_offsets) qtile_offsets[nq] = (int32_t)n;
  return n;
}

int64_t swa_count_nonmasked(int kind, int N, int W, int stride) {
  if (N < 0 || kind < 0 || kind > 3) return -1;
  if (kind != kMaskCausal && W < 1) return -1;
  if (kind == kMaskStrided && stride < 1) return -1;
  if (kind == kMaskGlobal && stride < 0) return -1;
  if (N == 0) return 0;
  return count_attended(kind, N, W, stride);
}

swa_status_t swa_debug_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return SWA_ERR_INVALID_ARG;
  if (n == 0) return SWA_OK;
  if (x == nullptr || y == nullptr || (reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u))
    return SWA_ERR_INVALID_ARG;
  return launch_exp2_fma2(x, y, n, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

swa_status_t swa_last_device_error(void* stream) {
  int err = 0;
  if (read_and_clear_device_error(static_cast<cudaStream_t>(stream), &err) != 0) return SWA_ERR_CUDA;
  return static_cast<swa_status_t>(err);
}

const char* swa_status_string(swa_status_t s) {
  switch (s) {
    case SWA_OK: return "ok";
    case SWA_ERR_INVALID_ARG: return "invalid argument";
    case SWA_ERR_UNSUPPORTED: return "unsupported head dimension or group size";
    case SWA_ERR_CUDA: return "CUDA error";
    case SWA_ERR_TIMEOUT: return "in-kernel wait timed out";
    case SWA_ERR_SCRATCH_TOO_SMALL: return "sizes need more scratch than the static decode array holds";
    case SWA_ERR_BOUNDS: return "debug bounds check failed: an index fell outside its tensor";
  }
  return "unknown status";
}

}  // extern "C"
