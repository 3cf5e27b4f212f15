// internal.h -- declarations shared by the library's translation units (not
// part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "schedule.cuh"

namespace swa {

// Work-unit layouts of the prefill kernel (two 128-row "subs" per CTA).
enum UnitMode {
  kModeHeadPairs = 0,  // two query heads of one KV group, same rows
  kModeTilePairs = 1,  // two consecutive query tiles of one head
  kModeDiff = 2,       // the two maps of differential attention
  kModeKvPairs = 3     // two query heads of different KV groups, same rows
};

struct PrefillParams {
  int B, Hq, Hkv, N, W, S;
  int G;     // Hq / Hkv
  int kind;  // MaskKind
  int mode;  // UnitMode
  int nq;    // query tiles of 128 rows
  int nunits;    // work units of two subs
  int num_ctas;  // persistent CTAs (one per SM)
  float scale_log2;  // scale * log2(e)
  void* o;
  float* lse;
  const float* lambda;
  int64_t* dbg_cells;
  int32_t* dbg_tiles;
  int32_t* dbg_ntiles;
  int dbg_cap;
  int inject_timeout;
  int* err_flag;  // device word that receives SWA_ERR_TIMEOUT
  // divisions of the work-unit index (see decode_unit), by the group size
  // and by the stride (clamped to N, which leaves the stride keys unchanged)
  FastDiv fd_u1, fd_u2, fd_u3, fd_g, fd_s;
};

// Backward of the window attention (dQ, dK, dV from dO and the forward's
// O and log-sum-exp). The workspace holds D_i and L_i log2(e) per query row,
// padded to whole 128-row tiles (npad rows per head).
struct BwdParams {
  const void *q, *k, *v, *o, *dO;
  void *dq, *dk, *dv;
  const float* lse;
  float *lse2, *dd;
  float *sdk, *sdv;  // strided mask: fp32 partial dK, dV of the stride keys [B*Hkv, nspad, d]
  int B, Hq, Hkv, N, W, G, nq, npad;
  int S, nspad;      // stride (0: window mask only), compacted stride rows padded to tiles
  float scale, scale_log2;
  int num_ctas;      // SMs of the device: the multi-tile dK/dV grid
  int* err_flag;
};
struct BwdMaps {
  CUtensorMap q, k, v, dO, ks, vs;  // ks, vs: stride row m is key m*S (or K, V when S = 0)
};
cudaError_t launch_backward(const BwdMaps& m, const BwdParams& p, int d, cudaStream_t stream);

// Row map of a strided view (dilated windows): row i of the problem is row
// off + i*mul of a head holding n rows, which is where its log-sum-exp goes.
struct RowMap {
  int n, off, mul;
};

struct PrefillMaps {
  CUtensorMap q, q2, k, k2, v, ks, vs;
  CUtensorMap o;  // output, 64 x 32-row boxes (one warp's rows)
};

cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillParams& p, const RowMap& rows, int dqk, int dv,
                           bool diff, int nunits, cudaStream_t stream);

struct DecodeParams {
  const void* q;
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  const int32_t* pos;
  void* o;
  float* partial;  // [B*Hq][nsplit][d + 2]
  int B, Hq, Hkv, d, W, G;
  int n_sink;  // attention-sink slots ahead of the W window slots (0: none)
  int nsplit, chunk;
  float scale_log2;
  int* err_flag;  // device error word (bounds-checking debug builds report here)
};

// Differential decode: two maps (q1/K1, q2/K2) over one rolling window and
// one shared V cache; d_qk = 64, d_v = 128.
struct DiffDecodeParams {
  const void *q1, *q2, *k1_new, *k2_new, *v_new;
  void *k1_cache, *k2_cache, *v_cache, *o;
  const int32_t* pos;
  const float* lambda;
  float* partial;
  int B, Hq, Hkv, W, G;
  int nsplit, chunk;
  float scale_log2;
  int* err_flag;
};
size_t diff_decode_partial_bytes(int B, int Hq, int Hkv, int W);
cudaError_t launch_diff_decode(const DiffDecodeParams& p, cudaStream_t stream);

int decode_nsplit(int B, int Hkv, int W);
size_t decode_partial_bytes(int B, int Hq, int Hkv, int d, int slots);
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device): function attributes live in each
// device's context. Safe to call from several host threads.
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);

// y[i] = 2^x[i] through the prefill kernels' FMA-pipe exponential.
cudaError_t launch_exp2_fma2(const float* x, float* y, int64_t n, cudaStream_t stream);

int* device_error_ptr();
int read_and_clear_device_error(cudaStream_t stream, int* err);

}  // namespace swa
