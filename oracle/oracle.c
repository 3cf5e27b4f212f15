/*
 * oracle.c -- plain, slow, fp64 CPU reference for masked causal attention.
 *
 * TEST INFRASTRUCTURE ONLY. The library's product path never calls, links or
 * loads this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header or constant with the CUDA
 * kernels.
 *
 * Every function follows the definitions on these pages:
 *   [CS] "Attention Variants Compared" (cheatsheet): the code of swa_mask and
 *        strided_mask, and its table of helper functions (count_nonmasked,
 *        tiled_softmax_dot).
 *   [SW] "Learn: Sparse & Sliding-Window Attention": section 3 "The math"
 *        (A = softmax(QK^T/sqrt(d_k) + log M) V, log M in {0, -inf}, dense
 *        causal M_ij = 1[j <= i], band M_ij = 1[i-w < j <= i]); section 3b
 *        (Longformer: window plus global tokens); section 4
 *        (rolling KV window at decode: keep the last w tokens, evict the
 *        oldest).
 *   [IG] "Exploring Attention Variants: Flash Attention, Sliding-Window, and
 *        Sparse Attention Implementation": SWA mask M[i][j] = 0 for
 *        j in [i-W+1, i] else -inf; strided = logical OR of the window mask
 *        and the stride mask; attention_row(q, K, V, mask_row) -> (out,
 *        weights).
 *   [DA] "Attention Variants -- Sliding Window, Sparse, Differential": the
 *        problem statement (two attention maps from separate Q/K
 *        projections, one subtracted from the other).
 *
 * Readings taken where the pages are silent (each listed in the design
 * notes): the window holds W keys (i-W+1 .. i); stride keys are the absolute
 * multiples of S from 0 (range(0, i+1, stride)); the differential output is
 * sum_j (w1_ij - lambda_h * w2_ij) v_j with both maps under the same mask;
 * query head h reads KV head h / (Hq/Hkv); a decode step writes the new
 * token into slot pos % W and then attends.
 *
 * Inputs are float32 arrays holding bf16 values exactly; every product and
 * sum is taken in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MASK_SWA 0
#define ORC_MASK_STRIDED 1
#define ORC_MASK_CAUSAL 2
#define ORC_MASK_GLOBAL 3
#define ORC_MASK_DILATED 4

/* ---------------------------------------------------------------------- */
/* Masks, one row at a time, in the pages' additive form: 0.0 = attends,  */
/* -inf = masked.                                                          */
/* ---------------------------------------------------------------------- */

/* [CS] swa_mask / [IG]: row i starts all -inf, then j = lo .. i set to 0.0
 * with lo = max(0, i - window + 1). window >= n gives full causal. */
void orc_swa_mask_row(int n, int window, int i, double* row) {
  for (int j = 0; j < n; ++j) row[j] = -INFINITY;
  int lo = i - window + 1;
  if (lo < 0) lo = 0;
  for (int j = lo; j <= i; ++j) row[j] = 0.0;
}

/* [CS] strided_mask: the local window first, then every stride-th key from 0
 * up to and including i is set to 0.0; [IG]: the union (logical OR). */
void orc_strided_mask_row(int n, int window, int stride, int i, double* row) {
  orc_swa_mask_row(n, window, i, row);
  for (int j = 0; j < i + 1; j += stride) row[j] = 0.0;
}

/* [SW] section 3: dense causal attention is M_ij = 1[j <= i]. Written on its
 * own (not as swa_mask with a large window) so that the two can be compared. */
void orc_causal_mask_row(int n, int i, double* row) {
  for (int j = 0; j < n; ++j) row[j] = (j <= i) ? 0.0 : -INFINITY;
}

/* [SW] section 3b (Longformer): the sliding window plus g global tokens
 * that attend to everything and are attended to by everything, each adding
 * a full row and a full column to M. Reading for this causal path: the
 * global tokens are positions 0 .. g-1 (a [CLS] or question prefix), and
 * "everything" is every position the causal mask allows. Row i of the
 * window is taken first, then global column j (j < g, j <= i), then, when
 * i itself is global, its whole causal row. */
void orc_global_mask_row(int n, int window, int g, int i, double* row) {
  orc_swa_mask_row(n, window, i, row);
  for (int j = 0; j < g && j <= i; ++j) row[j] = 0.0;
  if (i < g)
    for (int j = 0; j <= i; ++j) row[j] = 0.0;
}

/* [SW] section 3b (Longformer): dilation puts gaps of size d_dil inside
 * the window, so the same budget of allowed keys reaches d_dil times
 * further. Reading: the W keys i, i - dil, i - 2 dil, ..., i - (W-1) dil
 * (those >= 0); dil = 1 is the plain window. */
void orc_dilated_mask_row(int n, int window, int dil, int i, double* row) {
  for (int j = 0; j < n; ++j) row[j] = -INFINITY;
  for (int k = 0; k < window; ++k) {
    const int64_t j = (int64_t)i - (int64_t)k * dil;
    if (j < 0) break;
    row[j] = 0.0;
  }
}

/* kind: swa / strided / causal / global / dilated; `stride` carries S for
 * strided, the number of global tokens g for global, the dilation for
 * dilated. */
void orc_mask_row(int kind, int n, int window, int stride, int i, double* row) {
  if (kind == ORC_MASK_SWA) orc_swa_mask_row(n, window, i, row);
  else if (kind == ORC_MASK_STRIDED) orc_strided_mask_row(n, window, stride, i, row);
  else if (kind == ORC_MASK_GLOBAL) orc_global_mask_row(n, window, stride, i, row);
  else if (kind == ORC_MASK_DILATED) orc_dilated_mask_row(n, window, stride, i, row);
  else orc_causal_mask_row(n, i, row);
}

/* The full n x n matrix, row-major, built row by row. */
void orc_mask(int kind, int n, int window, int stride, double* M) {
  for (int i = 0; i < n; ++i) orc_mask_row(kind, n, window, stride, i, M + (int64_t)i * n);
}

/* [CS] count_nonmasked(M): the number of attended cells, ||M||_0 in [SW]. */
int64_t orc_count_nonmasked(const double* M, int64_t count) {
  int64_t c = 0;
  for (int64_t t = 0; t < count; ++t) c += (M[t] == 0.0);
  return c;
}

/* ---------------------------------------------------------------------- */
/* One attention row.                                                      */
/* ---------------------------------------------------------------------- */

/* [IG] attention_row / [SW] section 3: s_j = scale * q.k_j + M_ij,
 * w = softmax(s) (max subtracted), out = sum_j w_j v_j. K is n x dk, V is
 * n x dv, both row-major float. weights may be NULL. A masked entry's score
 * is -inf whatever q.k_j is, so its dot product is not formed. */
void orc_attention_row(const double* q, const float* K, const float* V, const double* mask_row,
                       int n, int dk, int dv, double scale, double* out, double* weights,
                       double* scratch_s, double* lse) {
  double mx = -INFINITY;
  for (int j = 0; j < n; ++j) {
    double s = -INFINITY;
    if (mask_row[j] == 0.0) {
      double dot = 0.0;
      const float* kj = K + (int64_t)j * dk;
      for (int c = 0; c < dk; ++c) dot += q[c] * (double)kj[c];
      s = scale * dot + mask_row[j];
    }
    scratch_s[j] = s;
    if (s > mx) mx = s;
  }
  double denom = 0.0;
  for (int j = 0; j < n; ++j) {
    double e = (scratch_s[j] == -INFINITY) ? 0.0 : exp(scratch_s[j] - mx);
    scratch_s[j] = e;
    denom += e;
  }
  for (int c = 0; c < dv; ++c) out[c] = 0.0;
  for (int j = 0; j < n; ++j) {
    double w = scratch_s[j] / denom;
    if (weights) weights[j] = w;
    if (w == 0.0) continue;
    const float* vj = V + (int64_t)j * dv;
    for (int c = 0; c < dv; ++c) out[c] += w * (double)vj[c];
  }
  if (lse) *lse = mx + log(denom);
}

/* Stand-alone form on double inputs (used by the tests on tiny cases). */
void orc_attention_row_f64(const double* q, const double* K, const double* V, const double* mask_row,
                           int n, int dk, int dv, double scale, double* out, double* weights) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY;
  for (int j = 0; j < n; ++j) {
    double v = -INFINITY;
    if (mask_row[j] == 0.0) {
      double dot = 0.0;
      for (int c = 0; c < dk; ++c) dot += q[c] * K[(int64_t)j * dk + c];
      v = scale * dot + mask_row[j];
    }
    s[j] = v;
    if (v > mx) mx = v;
  }
  double denom = 0.0;
  for (int j = 0; j < n; ++j) {
    s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - mx);
    denom += s[j];
  }
  for (int c = 0; c < dv; ++c) out[c] = 0.0;
  for (int j = 0; j < n; ++j) {
    double w = s[j] / denom;
    if (weights) weights[j] = w;
    for (int c = 0; c < dv; ++c) out[c] += w * V[(int64_t)j * dv + c];
  }
  free(s);
}

/* [CS] tiled_softmax_dot(q, Ks, Vs, tile): the flash-style softmax. Keys are
 * taken `tile` at a time; a running max m, running sum l and a running
 * output are rescaled by exp(m_old - m_new) whenever the max grows. Only
 * used to check that the tiled form equals the full softmax. */
void orc_tiled_softmax_dot(const double* q, const double* K, const double* V, const double* mask_row,
                           int n, int dk, int dv, double scale, int tile, double* out) {
  double m = -INFINITY, l = 0.0;
  for (int c = 0; c < dv; ++c) out[c] = 0.0;
  for (int t0 = 0; t0 < n; t0 += tile) {
    int t1 = t0 + tile < n ? t0 + tile : n;
    double tm = -INFINITY;
    for (int j = t0; j < t1; ++j) {
      if (mask_row[j] != 0.0) continue;
      double dot = 0.0;
      for (int c = 0; c < dk; ++c) dot += q[c] * K[(int64_t)j * dk + c];
      double s = scale * dot;
      if (s > tm) tm = s;
    }
    if (tm == -INFINITY) continue; /* nothing attended in this tile */
    double m_new = m > tm ? m : tm;
    double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
    l *= alpha;
    for (int c = 0; c < dv; ++c) out[c] *= alpha;
    for (int j = t0; j < t1; ++j) {
      if (mask_row[j] != 0.0) continue;
      double dot = 0.0;
      for (int c = 0; c < dk; ++c) dot += q[c] * K[(int64_t)j * dk + c];
      double p = exp(scale * dot - m_new);
      l += p;
      for (int c = 0; c < dv; ++c) out[c] += p * V[(int64_t)j * dv + c];
    }
    m = m_new;
  }
  for (int c = 0; c < dv; ++c) out[c] /= l;
}

/* ---------------------------------------------------------------------- */
/* Whole tensors: [B, H, N, d] row-major, query head h reads KV head       */
/* h / (Hq / Hkv). Rows are split over threads.                            */
/* ---------------------------------------------------------------------- */

typedef struct {
  int kind, B, Hq, Hkv, N, dk, dv, W, S;
  double scale;
  const float *q, *k, *v;        /* plain attention */
  const float *q1, *k1, *q2, *k2; /* differential */
  const float* lambda;
  const int64_t* rows; /* flat row ids (b*Hq + h)*N + i, or NULL for all */
  int64_t nrows;
  double* out; /* nrows x dv */
  double* lse; /* nrows, may be NULL */
  int nthreads, tid;
} orc_job_t;

static void row_coords(const orc_job_t* J, int64_t r, int* b, int* hq, int* i) {
  int64_t flat = J->rows ? J->rows[r] : r;
  *i = (int)(flat % J->N);
  int64_t bh = flat / J->N;
  *hq = (int)(bh % J->Hq);
  *b = (int)(bh / J->Hq);
}

static void* attn_worker(void* arg) {
  orc_job_t* J = (orc_job_t*)arg;
  int G = J->Hq / J->Hkv;
  double* mrow = (double*)malloc(sizeof(double) * (size_t)J->N);
  double* s = (double*)malloc(sizeof(double) * (size_t)J->N);
  double* qd = (double*)malloc(sizeof(double) * (size_t)J->dk);
  for (int64_t r = J->tid; r < J->nrows; r += J->nthreads) {
    int b, hq, i;
    row_coords(J, r, &b, &hq, &i);
    int hk = hq / G;
    const float* qrow = J->q + (((int64_t)b * J->Hq + hq) * J->N + i) * J->dk;
    for (int c = 0; c < J->dk; ++c) qd[c] = (double)qrow[c];
    const float* K = J->k + ((int64_t)b * J->Hkv + hk) * J->N * (int64_t)J->dk;
    const float* V = J->v + ((int64_t)b * J->Hkv + hk) * J->N * (int64_t)J->dv;
    orc_mask_row(J->kind, J->N, J->W, J->S, i, mrow);
    orc_attention_row(qd, K, V, mrow, J->N, J->dk, J->dv, J->scale, J->out + r * J->dv, NULL, s,
                      J->lse ? J->lse + r : NULL);
  }
  free(mrow);
  free(s);
  free(qd);
  return NULL;
}

/* [DA] problem statement: two maps from separate Q/K, one subtracted from
 * the other, over the shared V: out_i = sum_j (w1_ij - lambda_h w2_ij) v_j. */
static void* diff_worker(void* arg) {
  orc_job_t* J = (orc_job_t*)arg;
  int G = J->Hq / J->Hkv;
  int N = J->N;
  double* mrow = (double*)malloc(sizeof(double) * (size_t)N);
  double* s = (double*)malloc(sizeof(double) * (size_t)N);
  double* w1 = (double*)malloc(sizeof(double) * (size_t)N);
  double* w2 = (double*)malloc(sizeof(double) * (size_t)N);
  double* o = (double*)malloc(sizeof(double) * (size_t)J->dv);
  double* qd = (double*)malloc(sizeof(double) * (size_t)J->dk);
  for (int64_t r = J->tid; r < J->nrows; r += J->nthreads) {
    int b, hq, i;
    row_coords(J, r, &b, &hq, &i);
    int hk = hq / G;
    int64_t qoff = (((int64_t)b * J->Hq + hq) * N + i) * J->dk;
    int64_t koff = ((int64_t)b * J->Hkv + hk) * N * (int64_t)J->dk;
    const float* V = J->v + ((int64_t)b * J->Hkv + hk) * N * (int64_t)J->dv;
    orc_mask_row(J->kind, N, J->W, J->S, i, mrow);
    for (int c = 0; c < J->dk; ++c) qd[c] = (double)J->q1[qoff + c];
    orc_attention_row(qd, J->k1 + koff, V, mrow, N, J->dk, J->dv, J->scale, o, w1, s, NULL);
    for (int c = 0; c < J->dk; ++c) qd[c] = (double)J->q2[qoff + c];
    orc_attention_row(qd, J->k2 + koff, V, mrow, N, J->dk, J->dv, J->scale, o, w2, s, NULL);
    double lam = (double)J->lambda[hq];
    double* out = J->out + r * J->dv;
    for (int c = 0; c < J->dv; ++c) out[c] = 0.0;
    for (int j = 0; j < N; ++j) {
      double w = w1[j] - lam * w2[j];
      if (w == 0.0) continue;
      const float* vj = V + (int64_t)j * J->dv;
      for (int c = 0; c < J->dv; ++c) out[c] += w * (double)vj[c];
    }
  }
  free(mrow);
  free(s);
  free(w1);
  free(w2);
  free(o);
  free(qd);
  return NULL;
}

static int run_threads(orc_job_t* proto, void* (*fn)(void*)) {
  int nt = proto->nthreads < 1 ? 1 : proto->nthreads;
  if (nt > 256) nt = 256;
  pthread_t th[256];
  orc_job_t jobs[256];
  for (int t = 0; t < nt; ++t) {
    jobs[t] = *proto;
    jobs[t].nthreads = nt;
    jobs[t].tid = t;
  }
  int started = 0;
  for (int t = 1; t < nt; ++t) {
    if (pthread_create(&th[t], NULL, fn, &jobs[t]) != 0) break;
    started = t;
  }
  fn(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  if (started != nt - 1) { /* a thread failed to start: do its share here */
    for (int t = started + 1; t < nt; ++t) fn(&jobs[t]);
  }
  return 0;
}

/* Masked attention (kind = swa / strided / causal) over [B,H,N,d] tensors.
 * rows: flat row ids to compute, or NULL with nrows = B*Hq*N for all rows.
 * out: nrows x dv doubles; lse: nrows natural-log sums (may be NULL). */
int orc_attention(int kind, const float* q, const float* k, const float* v, int B, int Hq, int Hkv,
                  int N, int dk, int dv, int W, int S, double scale, const int64_t* rows,
                  int64_t nrows, double* out, double* lse, int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0 || N <= 0) return 1;
  orc_job_t J;
  memset(&J, 0, sizeof(J));
  J.kind = kind; J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.N = N; J.dk = dk; J.dv = dv;
  J.W = W; J.S = S; J.scale = scale; J.q = q; J.k = k; J.v = v;
  J.rows = rows; J.nrows = nrows; J.out = out; J.lse = lse; J.nthreads = nthreads;
  return run_threads(&J, attn_worker);
}

int orc_diff_attention(int kind, const float* q1, const float* k1, const float* q2, const float* k2,
                       const float* v, const float* lambda, int B, int Hq, int Hkv, int N, int dk,
                       int dv, int W, int S, double scale, const int64_t* rows, int64_t nrows,
                       double* out, int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0 || N <= 0) return 1;
  orc_job_t J;
  memset(&J, 0, sizeof(J));
  J.kind = kind; J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.N = N; J.dk = dk; J.dv = dv;
  J.W = W; J.S = S; J.scale = scale; J.q1 = q1; J.k1 = k1; J.q2 = q2; J.k2 = k2; J.v = v;
  J.lambda = lambda; J.rows = rows; J.nrows = nrows; J.out = out; J.nthreads = nthreads;
  return run_threads(&J, diff_worker);
}

/* ---------------------------------------------------------------------- */
/* Decode over a rolling W-slot cache ([SW] section 4: keep only the most  */
/* recent w tokens' K/V, evict the oldest).                                */
/* ---------------------------------------------------------------------- */

/* T steps. q: [T,B,Hq,d]; k_new, v_new: [T,B,Hkv,d]; caches: [B,Hkv,W,d]
 * (updated in place); pos: [T,B] absolute position of each step's token.
 * Each step first stores the new token in slot pos % W (overwriting the
 * token at pos - W, the oldest), then attends over the positions still in
 * the window, max(0, pos-W+1) .. pos, each read from its slot p % W. */
int orc_decode(const float* q, const float* k_new, const float* v_new, float* k_cache,
               float* v_cache, const int32_t* pos, int T, int B, int Hq, int Hkv, int d, int W,
               double scale, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0 || W <= 0) return 1;
  int G = Hq / Hkv;
  double* s = (double*)malloc(sizeof(double) * (size_t)W);
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  for (int t = 0; t < T; ++t) {
    for (int b = 0; b < B; ++b) {
      int p = pos[(int64_t)t * B + b];
      int slot = p % W;
      for (int hk = 0; hk < Hkv; ++hk) {
        int64_t src = (((int64_t)t * B + b) * Hkv + hk) * d;
        int64_t dst = (((int64_t)b * Hkv + hk) * W + slot) * d;
        memcpy(k_cache + dst, k_new + src, sizeof(float) * (size_t)d);
        memcpy(v_cache + dst, v_new + src, sizeof(float) * (size_t)d);
      }
      int first = p - W + 1;
      if (first < 0) first = 0;
      int cnt = p - first + 1;
      for (int hq = 0; hq < Hq; ++hq) {
        int hk = hq / G;
        const float* qrow = q + (((int64_t)t * B + b) * Hq + hq) * d;
        for (int c = 0; c < d; ++c) qd[c] = (double)qrow[c];
        const float* Kc = k_cache + ((int64_t)b * Hkv + hk) * (int64_t)W * d;
        const float* Vc = v_cache + ((int64_t)b * Hkv + hk) * (int64_t)W * d;
        double mx = -INFINITY;
        for (int u = 0; u < cnt; ++u) {
          int sl = (first + u) % W;
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += qd[c] * (double)Kc[(int64_t)sl * d + c];
          s[u] = scale * dot;
          if (s[u] > mx) mx = s[u];
        }
        double denom = 0.0;
        for (int u = 0; u < cnt; ++u) {
          s[u] = exp(s[u] - mx);
          denom += s[u];
        }
        double* o = out + (((int64_t)t * B + b) * Hq + hq) * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int u = 0; u < cnt; ++u) {
          int sl = (first + u) % W;
          double w = s[u] / denom;
          for (int c = 0; c < d; ++c) o[c] += w * (double)Vc[(int64_t)sl * d + c];
        }
      }
    }
  }
  free(s);
  free(qd);
  return 0;
}

/* ---------------------------------------------------------------------- */
/* Which key tiles a query tile touches, read off the explicit mask.       */
/* ---------------------------------------------------------------------- */

/* For query tile qt (rows qt*Bq .. qt*Bq+Bq-1, clipped to N) scan every cell
 * of the explicit mask row. An attended cell that the window mask also
 * attends marks key tile j / Bk; an attended cell outside the window (only
 * the strided mask has those; they are multiples of S) marks stride tile
 * (j / S) / Bk. cells += every attended cell. Writes the marked tiles into
 * tiles[] as stride tiles first (0x40000000 | ct, ascending) then window
 * tiles (kt, ascending); returns their number, or -1 if cap is too small, or
 * -2 if an outside-window cell is not a multiple of S. */
int64_t orc_schedule_qtile(int kind, int N, int W, int S, int Bq, int Bk, int qt, int32_t* tiles,
                           int64_t cap, int64_t* cells) {
  if (kind == ORC_MASK_DILATED) return -3; /* visited per residue class, as window masks */
  int nkt = (N + Bk - 1) / Bk;
  /* extra key tiles: stride keys m*S (tile m / Bk) or global keys j < g
   * (tile j / Bk), tagged 0x40000000 | tile */
  int nst = 0;
  if (kind == ORC_MASK_STRIDED && S > 0) nst = ((N + S - 1) / S + Bk - 1) / Bk;
  if (kind == ORC_MASK_GLOBAL && S > 0) nst = ((S < N ? S : N) + Bk - 1) / Bk;
  uint8_t* band = (uint8_t*)calloc((size_t)nkt + 1, 1);
  uint8_t* strd = (uint8_t*)calloc((size_t)nst + 1, 1);
  double* row = (double*)malloc(sizeof(double) * (size_t)N);
  double* wrow = (double*)malloc(sizeof(double) * (size_t)N);
  int64_t c = 0;
  int bad = 0;
  int r0 = qt * Bq, r1 = qt * Bq + Bq;
  if (r1 > N) r1 = N;
  for (int i = r0; i < r1; ++i) {
    orc_mask_row(kind, N, W, S, i, row);
    /* the window part of the same row: for the strided and global masks
     * the band is the swa_mask row (their first loop); for swa/causal the
     * whole row is band */
    const int split = (kind == ORC_MASK_STRIDED || kind == ORC_MASK_GLOBAL);
    if (split) orc_swa_mask_row(N, W, i, wrow);
    for (int j = 0; j < N; ++j) {
      if (row[j] != 0.0) continue;
      ++c;
      int in_band = split ? (wrow[j] == 0.0) : 1;
      if (in_band) {
        band[j / Bk] = 1;
      } else if (kind == ORC_MASK_STRIDED) {
        if (j % S != 0) bad = 1;
        strd[(j / S) / Bk] = 1;
      } else {
        if (j >= S) bad = 1; /* outside the window only global keys may be attended */
        strd[j / Bk] = 1;
      }
    }
  }
  int64_t n = 0;
  for (int t = 0; t < nst; ++t)
    if (strd[t]) {
      if (n < cap) tiles[n] = 0x40000000 | t;
      ++n;
    }
  for (int t = 0; t < nkt; ++t)
    if (band[t]) {
      if (n < cap) tiles[n] = t;
      ++n;
    }
  free(band);
  free(strd);
  free(row);
  free(wrow);
  if (cells) *cells = c;
  if (bad) return -2;
  return n > cap ? -1 : n;
}

/* ---------------------------------------------------------------------- */
/* Decode with attention sinks ("Learn: Sparse & Sliding-Window           */
/* Attention", section 4, StreamingLLM: keep the first k tokens for good  */
/* plus the most recent w tokens, drop the middle; section 6: O(k + w)).  */
/* ---------------------------------------------------------------------- */

/* Caches: [B,Hkv,n_sink+W,d]. Positions p < n_sink stay in slot p for good;
 * a later position p takes slot n_sink + (p - n_sink) % W, overwriting the
 * oldest non-sink token. Each step first stores its token, then attends over
 * the sink positions 0 .. min(n_sink, pos+1)-1 and the recent positions
 * max(n_sink, pos-W+1) .. pos, each read from its slot. Shapes as
 * orc_decode; n_sink = 0 is the plain rolling window. */
int orc_sink_decode(const float* q, const float* k_new, const float* v_new, float* k_cache,
                    float* v_cache, const int32_t* pos, int T, int B, int Hq, int Hkv, int d,
                    int n_sink, int W, double scale, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0 || W <= 0 || n_sink < 0) return 1;
  const int G = Hq / Hkv;
  const int slots = n_sink + W;
  int* key_slot = (int*)malloc(sizeof(int) * (size_t)slots);
  double* s = (double*)malloc(sizeof(double) * (size_t)slots);
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  for (int t = 0; t < T; ++t) {
    for (int b = 0; b < B; ++b) {
      const int p = pos[(int64_t)t * B + b];
      const int slot = (p < n_sink) ? p : n_sink + (p - n_sink) % W;
      for (int hk = 0; hk < Hkv; ++hk) {
        const int64_t src = (((int64_t)t * B + b) * Hkv + hk) * d;
        const int64_t dst = (((int64_t)b * Hkv + hk) * slots + slot) * d;
        memcpy(k_cache + dst, k_new + src, sizeof(float) * (size_t)d);
        memcpy(v_cache + dst, v_new + src, sizeof(float) * (size_t)d);
      }
      /* the attended positions, each mapped to its slot */
      int cnt = 0;
      for (int u = 0; u < n_sink && u <= p; ++u) key_slot[cnt++] = u;
      int first = p - W + 1;
      if (first < n_sink) first = n_sink;
      for (int u = first; u <= p; ++u) key_slot[cnt++] = n_sink + (u - n_sink) % W;
      for (int hq = 0; hq < Hq; ++hq) {
        const int hk = hq / G;
        const float* qrow = q + (((int64_t)t * B + b) * Hq + hq) * d;
        for (int c = 0; c < d; ++c) qd[c] = (double)qrow[c];
        const float* Kc = k_cache + ((int64_t)b * Hkv + hk) * (int64_t)slots * d;
        const float* Vc = v_cache + ((int64_t)b * Hkv + hk) * (int64_t)slots * d;
        double mx = -INFINITY;
        for (int u = 0; u < cnt; ++u) {
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += qd[c] * (double)Kc[(int64_t)key_slot[u] * d + c];
          s[u] = scale * dot;
          if (s[u] > mx) mx = s[u];
        }
        double denom = 0.0;
        for (int u = 0; u < cnt; ++u) {
          s[u] = exp(s[u] - mx);
          denom += s[u];
        }
        double* o = out + (((int64_t)t * B + b) * Hq + hq) * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int u = 0; u < cnt; ++u) {
          const double w = s[u] / denom;
          for (int c = 0; c < d; ++c) o[c] += w * (double)Vc[(int64_t)key_slot[u] * d + c];
        }
      }
    }
  }
  free(key_slot);
  free(s);
  free(qd);
  return 0;
}

/* Differential attention, one decode step per (t, b), over a rolling W-slot
 * cache ("Attention Variants -- Sliding Window, Sparse, Differential", The
 * Problem: two softmax maps over the same keys, combined as w1 - lambda_h w2
 * and applied to one shared V; window as orc_decode).
 * q1, q2: [T,B,Hq,dk]; k1_new, k2_new: [T,B,Hkv,dk]; v_new: [T,B,Hkv,dv];
 * caches k1c, k2c: [B,Hkv,W,dk], vc: [B,Hkv,W,dv], updated in place; lambda:
 * [Hq]. Each step writes its token into slot pos % W, then attends over the
 * positions max(0, pos-W+1) .. pos. out: [T,B,Hq,dv] doubles. */
int orc_diff_decode(const float* q1, const float* q2, const float* k1_new, const float* k2_new,
                    const float* v_new, float* k1c, float* k2c, float* vc, const float* lambda,
                    const int32_t* pos, int T, int B, int Hq, int Hkv, int dk, int dv, int W,
                    double scale, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0 || W <= 0) return 1;
  const int G = Hq / Hkv;
  double* s1 = (double*)malloc(sizeof(double) * (size_t)W);
  double* s2 = (double*)malloc(sizeof(double) * (size_t)W);
  int* key_slot = (int*)malloc(sizeof(int) * (size_t)W);
  for (int t = 0; t < T; ++t) {
    for (int b = 0; b < B; ++b) {
      const int p = pos[(int64_t)t * B + b];
      const int slot = p % W;
      for (int hk = 0; hk < Hkv; ++hk) {
        const int64_t src = ((int64_t)t * B + b) * Hkv + hk;
        const int64_t dst = ((int64_t)b * Hkv + hk) * W + slot;
        memcpy(k1c + dst * dk, k1_new + src * dk, sizeof(float) * (size_t)dk);
        memcpy(k2c + dst * dk, k2_new + src * dk, sizeof(float) * (size_t)dk);
        memcpy(vc + dst * dv, v_new + src * dv, sizeof(float) * (size_t)dv);
      }
      int cnt = 0;
      for (int u = (p - W + 1 > 0 ? p - W + 1 : 0); u <= p; ++u) key_slot[cnt++] = u % W;
      for (int hq = 0; hq < Hq; ++hq) {
        const int hk = hq / G;
        const float* a1 = q1 + (((int64_t)t * B + b) * Hq + hq) * dk;
        const float* a2 = q2 + (((int64_t)t * B + b) * Hq + hq) * dk;
        const int64_t cb = ((int64_t)b * Hkv + hk) * W;
        double m1 = -INFINITY, m2 = -INFINITY;
        for (int u = 0; u < cnt; ++u) {
          double d1 = 0.0, d2 = 0.0;
          const float* r1 = k1c + (cb + key_slot[u]) * dk;
          const float* r2 = k2c + (cb + key_slot[u]) * dk;
          for (int c = 0; c < dk; ++c) {
            d1 += (double)a1[c] * (double)r1[c];
            d2 += (double)a2[c] * (double)r2[c];
          }
          s1[u] = scale * d1;
          s2[u] = scale * d2;
          if (s1[u] > m1) m1 = s1[u];
          if (s2[u] > m2) m2 = s2[u];
        }
        double z1 = 0.0, z2 = 0.0;
        for (int u = 0; u < cnt; ++u) {
          s1[u] = exp(s1[u] - m1);
          s2[u] = exp(s2[u] - m2);
          z1 += s1[u];
          z2 += s2[u];
        }
        const double lam = (double)lambda[hq];
        double* o = out + (((int64_t)t * B + b) * Hq + hq) * dv;
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        for (int u = 0; u < cnt; ++u) {
          const double w = s1[u] / z1 - lam * (s2[u] / z2);
          const float* vr = vc + (cb + key_slot[u]) * dv;
          for (int c = 0; c < dv; ++c) o[c] += w * (double)vr[c];
        }
      }
    }
  }
  free(s1);
  free(s2);
  free(key_slot);
  return 0;
}

/* ---------------------------------------------------------------------- */
/* Backward of the masked attention forward. The pages give no backward   */
/* pass; these functions apply the chain rule to the forward definition   */
/* ([SW] section 3: o_i = sum_j w_ij v_j, w_i = softmax_j(scale q_i.k_j    */
/* + log M_ij)), with dO the gradient of the loss with respect to O:      */
/*   dv_j  = sum_i w_ij do_i                                              */
/*   dw_ij = do_i . v_j,   D_i = sum_j w_ij dw_ij (= do_i . o_i)          */
/*   ds_ij = w_ij (dw_ij - D_i)                                           */
/*   dq_i  = scale sum_j ds_ij k_j,   dk_j = scale sum_i ds_ij q_i        */
/* summed over the query heads that share a KV head. Written per output   */
/* row, straight from these sums; slow, for tests only.                   */
/* ---------------------------------------------------------------------- */

/* Forward weights w_i (length N) and D_i of query row (b, hq, i). */
static double bwd_row_weights(int kind, const float* q, const float* k, const float* v, const float* dO,
                              int B, int Hq, int Hkv, int N, int dk, int dv, int W, int S, double scale,
                              int b, int hq, int i, double* w, double* mrow, double* s, double* qd,
                              double* o) {
  const int G = Hq / Hkv, hk = hq / G;
  const float* qrow = q + (((int64_t)b * Hq + hq) * N + i) * dk;
  for (int c = 0; c < dk; ++c) qd[c] = (double)qrow[c];
  const float* K = k + ((int64_t)b * Hkv + hk) * (int64_t)N * dk;
  const float* V = v + ((int64_t)b * Hkv + hk) * (int64_t)N * dv;
  orc_mask_row(kind, N, W, S, i, mrow);
  orc_attention_row(qd, K, V, mrow, N, dk, dv, scale, o, w, s, NULL);
  const float* dorow = dO + (((int64_t)b * Hq + hq) * N + i) * dv;
  double D = 0.0;
  for (int c = 0; c < dv; ++c) D += (double)dorow[c] * o[c];
  return D;
}

/* dq of query row (b, hq, i): dk doubles. */
void orc_attention_bwd_dq_row(int kind, const float* q, const float* k, const float* v, const float* dO,
                              int B, int Hq, int Hkv, int N, int dk, int dv, int W, int S, double scale,
                              int b, int hq, int i, double* dq) {
  double* w = (double*)malloc(sizeof(double) * (size_t)N);
  double* mrow = (double*)malloc(sizeof(double) * (size_t)N);
  double* s = (double*)malloc(sizeof(double) * (size_t)N);
  double* qd = (double*)malloc(sizeof(double) * (size_t)dk);
  double* o = (double*)malloc(sizeof(double) * (size_t)dv);
  const double D = bwd_row_weights(kind, q, k, v, dO, B, Hq, Hkv, N, dk, dv, W, S, scale, b, hq, i, w, mrow, s,
                                   qd, o);
  const int hk = hq / (Hq / Hkv);
  const float* K = k + ((int64_t)b * Hkv + hk) * (int64_t)N * dk;
  const float* V = v + ((int64_t)b * Hkv + hk) * (int64_t)N * dv;
  const float* dorow = dO + (((int64_t)b * Hq + hq) * N + i) * dv;
  for (int c = 0; c < dk; ++c) dq[c] = 0.0;
  for (int j = 0; j < N; ++j) {
    if (w[j] == 0.0) continue;
    double dw = 0.0;
    for (int c = 0; c < dv; ++c) dw += (double)dorow[c] * (double)V[(int64_t)j * dv + c];
    const double ds = w[j] * (dw - D);
    for (int c = 0; c < dk; ++c) dq[c] += scale * ds * (double)K[(int64_t)j * dk + c];
  }
  free(w); free(mrow); free(s); free(qd); free(o);
}

/* dk and dv of key row (b, hk, j): dk and dv doubles, summed over every
 * query row of every query head of KV head hk. */
void orc_attention_bwd_dkv_row(int kind, const float* q, const float* k, const float* v, const float* dO,
                               int B, int Hq, int Hkv, int N, int dk, int dv, int W, int S, double scale,
                               int b, int hk, int j, double* dkj, double* dvj) {
  double* w = (double*)malloc(sizeof(double) * (size_t)N);
  double* mrow = (double*)malloc(sizeof(double) * (size_t)N);
  double* s = (double*)malloc(sizeof(double) * (size_t)N);
  double* qd = (double*)malloc(sizeof(double) * (size_t)dk);
  double* o = (double*)malloc(sizeof(double) * (size_t)dv);
  const int G = Hq / Hkv;
  const float* V = v + ((int64_t)b * Hkv + hk) * (int64_t)N * dv;
  for (int c = 0; c < dk; ++c) dkj[c] = 0.0;
  for (int c = 0; c < dv; ++c) dvj[c] = 0.0;
  for (int hq = hk * G; hq < hk * G + G; ++hq) {
    for (int i = 0; i < N; ++i) {
      orc_mask_row(kind, N, W, S, i, mrow);
      if (mrow[j] != 0.0) continue; /* row i does not attend key j */
      const double D = bwd_row_weights(kind, q, k, v, dO, B, Hq, Hkv, N, dk, dv, W, S, scale, b, hq, i, w, mrow,
                                       s, qd, o);
      const float* dorow = dO + (((int64_t)b * Hq + hq) * N + i) * dv;
      double dw = 0.0;
      for (int c = 0; c < dv; ++c) dw += (double)dorow[c] * (double)V[(int64_t)j * dv + c];
      const double ds = w[j] * (dw - D);
      for (int c = 0; c < dv; ++c) dvj[c] += w[j] * (double)dorow[c];
      for (int c = 0; c < dk; ++c) dkj[c] += scale * ds * qd[c];
    }
  }
  free(w); free(mrow); free(s); free(qd); free(o);
}
