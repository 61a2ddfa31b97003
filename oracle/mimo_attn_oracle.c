/*
 * mimo_attn_oracle.c -- plain, slow FP64 CPU oracle for the MiMo-V2 attention
 * forward (sliding-window layer with a learnable sink, and global causal layer).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header or constant
 * table with the CUDA library.
 *
 * What it computes is the plain definition of the layer, written out in FP64
 * from BF16 inputs converted exactly, with no intermediate rounding and no
 * blocking or reordering:
 *
 *   For sequence b (tokens s_b .. s_b+L_b-1 of the THD-packed tensors), local
 *   position p, query head h and its KV head g = floor(h / (Hq/Hkv)):
 *
 *   1. RoPE on the first R = rope_dims dims (rotate-half pairing (i, i+R/2),
 *      theta_i = base^(-2i/R), angle = pos * theta_i, positions restart at 0
 *      for every sequence):
 *        q~ = rope(q[s_b+p, h], p),  k~_j = rope(k[s_b+j, g], j).
 *      Sources: miles docs "MiMo-V2.6-Flash" section 1 Model Introduction
 *      (partial RoPE, 64 of 192 dims; bases 1e4 / 1e7); Megatron-Bridge API doc
 *      "mimo_v2_flash_bridge" module summary (partial rotary, dual RoPE bases).
 *   2. Allowed keys A(p) = { j : 0 <= j <= p and p - j <= W }; W = infinity for
 *      the global layer.  With W = 128 a query sees itself plus 128 previous
 *      keys, 129 in total (miles docs section 5.4 "Sliding window"; miles PR
 *      #3648 commit "SGLang's RadixAttention window excludes the query token").
 *   3. s_j = q~ . k~_j / sqrt(d_qk).
 *   4. M = max(max_j s_j, sigma_h) with the per-head sink logit sigma_h
 *      (sliding-window layers only; miles PR #3648 Motivation / Design Notes).
 *   5. Z = sum_j exp(s_j - M) + exp(sigma_h - M)    (sink term only with a sink).
 *   6. lse = M + ln Z   (natural log, includes the sink term).
 *   7. out = sum_j exp(s_j - lse) * (v_scale * v[s_b+j, g])  (V scaled by 0.707
 *      before attention: miles PR #3648 Motivation; miles docs section 1).
 *
 * Each rotated key row is computed once per call (the same value every query
 * would compute); this is the only precomputation.
 *
 * Inputs may be given as BF16 bit patterns or as FP64 values (the FP64 form
 * lets the tests differentiate the forward numerically).
 *
 * The backward (oracle_attn_bwd) differentiates the same definition: given
 * the upstream gradients dO = dL/dout and dLSE = dL/dlse, with
 * P_j = exp(s_j - lse), P_sink = exp(sigma_h - lse) and D = dO . out,
 *   dL/ds_j     = P_j (dO . v'_j - D + dLSE)          (v'_j = v_scale v_j)
 *   dL/dsigma_h = sum over the head's rows of P_sink (dLSE - D)
 *   dL/dv_j     = v_scale sum over rows attending j of P_j dO
 *   dL/dq~      = sum_j dL/ds_j k~_j / sqrt(d_qk),  dL/dk~_j = sum over rows of dL/ds_j q~ / sqrt(d_qk)
 *   dL/dq = R(-phi) dL/dq~ and dL/dk = R(-phi) dL/dk~ (the transpose of the rotation).
 * It is single-threaded and meant for the small shapes the tests use.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Element i of an input tensor given as BF16 bits (f64 == 0) or FP64 values. */
static double ld(const void* p, size_t i, int f64) {
  return f64 ? ((const double*)p)[i] : bf16_bits_to_double(((const uint16_t*)p)[i]);
}

/* Step 1: rotate the first rope_dims entries of x (length dim) by position pos. */
void oracle_rope(const double* x, int64_t pos, double base, int32_t rope_dims, int32_t dim, double* y) {
  int32_t half = rope_dims / 2;
  for (int32_t d = 0; d < dim; ++d) y[d] = x[d];
  for (int32_t i = 0; i < half; ++i) {
    double theta = pow(base, -2.0 * (double)i / (double)rope_dims);
    double phi = (double)pos * theta;
    double c = cos(phi), s = sin(phi);
    y[i] = x[i] * c - x[i + half] * s;
    y[i + half] = x[i + half] * c + x[i] * s;
  }
}

typedef struct {
  /* inputs */
  const void* q;
  const void* v;
  int f64;
  const float* sink;
  const int32_t* cu;
  int32_t num_seqs;
  int64_t total_tokens;
  int32_t hq, hkv, dqk, dv, window, rope_dims;
  double rope_base, v_scale;
  const int64_t* rows;
  int64_t n_rows;
  const double* k_rot; /* [T, hkv, dqk] rotated keys */
  /* outputs */
  double* out; /* [n_rows, hq, dv] */
  double* lse; /* [hq, n_rows] */
  /* work split */
  int64_t r0, r1;
  int32_t status;
} oracle_job;

typedef struct {
  const void* k;
  int f64;
  int64_t t0, t1;
  const int32_t* cu;
  int32_t num_seqs, hkv, dqk, rope_dims;
  double rope_base;
  double* k_rot;
} rot_job;

static int32_t seq_of_token(const int32_t* cu, int32_t num_seqs, int64_t t) {
  /* largest b with cu[b] <= t and cu[b+1] > t (skips empty sequences) */
  int32_t lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) / 2;
    if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

static void* rotate_keys(void* arg) {
  rot_job* j = (rot_job*)arg;
  double* x = (double*)malloc(sizeof(double) * (size_t)j->dqk);
  if (!x) return NULL;
  for (int64_t t = j->t0; t < j->t1; ++t) {
    int32_t b = seq_of_token(j->cu, j->num_seqs, t);
    int64_t pos = t - (int64_t)j->cu[b];
    for (int32_t g = 0; g < j->hkv; ++g) {
      const size_t base = ((size_t)t * j->hkv + g) * j->dqk;
      for (int32_t d = 0; d < j->dqk; ++d) x[d] = ld(j->k, base + d, j->f64);
      oracle_rope(x, pos, j->rope_base, j->rope_dims, j->dqk, j->k_rot + ((size_t)t * j->hkv + g) * j->dqk);
    }
  }
  free(x);
  return NULL;
}

static void* run_rows(void* arg) {
  oracle_job* J = (oracle_job*)arg;
  const int32_t group = J->hq / J->hkv;
  const double inv_sqrt_d = 1.0 / sqrt((double)J->dqk);
  int64_t max_len = 0;
  for (int32_t b = 0; b < J->num_seqs; ++b) {
    int64_t L = (int64_t)J->cu[b + 1] - J->cu[b];
    if (L > max_len) max_len = L;
  }
  double* qx = (double*)malloc(sizeof(double) * (size_t)J->dqk);
  double* qr = (double*)malloc(sizeof(double) * (size_t)J->dqk);
  double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
  double* o = (double*)malloc(sizeof(double) * (size_t)J->dv);
  if (!qx || !qr || !s || !o) {
    J->status = ORACLE_ERR_NOMEM;
    free(qx); free(qr); free(s); free(o);
    return NULL;
  }
  for (int64_t r = J->r0; r < J->r1; ++r) {
    int64_t t = J->rows ? J->rows[r] : r;
    int32_t b = seq_of_token(J->cu, J->num_seqs, t);
    int64_t sb = J->cu[b];
    int64_t p = t - sb;
    int64_t lo = 0;
    if (J->window >= 0 && p - J->window > 0) lo = p - J->window;
    for (int32_t h = 0; h < J->hq; ++h) {
      int32_t g = h / group;
      const size_t qbase = ((size_t)t * J->hq + h) * J->dqk;
      for (int32_t d = 0; d < J->dqk; ++d) qx[d] = ld(J->q, qbase + d, J->f64);
      oracle_rope(qx, p, J->rope_base, J->rope_dims, J->dqk, qr);
      /* steps 3-4 */
      int has_sink = J->sink != NULL;
      double sigma = has_sink ? (double)J->sink[h] : 0.0;
      double M = has_sink ? sigma : -INFINITY;
      for (int64_t j = lo; j <= p; ++j) {
        const double* kr = J->k_rot + ((size_t)(sb + j) * J->hkv + g) * J->dqk;
        double acc = 0.0;
        for (int32_t d = 0; d < J->dqk; ++d) acc += qr[d] * kr[d];
        s[j - lo] = acc * inv_sqrt_d;
        if (s[j - lo] > M) M = s[j - lo];
      }
      /* step 5 */
      double Z = has_sink ? exp(sigma - M) : 0.0;
      for (int64_t j = lo; j <= p; ++j) Z += exp(s[j - lo] - M);
      /* step 6 */
      double L = M + log(Z);
      J->lse[(size_t)h * J->n_rows + r] = L;
      /* step 7 */
      for (int32_t d = 0; d < J->dv; ++d) o[d] = 0.0;
      for (int64_t j = lo; j <= p; ++j) {
        double w = exp(s[j - lo] - L);
        const size_t vbase = ((size_t)(sb + j) * J->hkv + g) * J->dv;
        for (int32_t d = 0; d < J->dv; ++d) o[d] += w * (J->v_scale * ld(J->v, vbase + d, J->f64));
      }
      double* dst = J->out + ((size_t)r * J->hq + h) * J->dv;
      for (int32_t d = 0; d < J->dv; ++d) dst[d] = o[d];
    }
  }
  free(qx); free(qr); free(s); free(o);
  return NULL;
}

/* Shape and argument checks shared by the entry points. */
static int32_t check_args(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                          int32_t num_seqs, int64_t total_tokens, int32_t hq, int32_t hkv, int32_t dqk,
                          int32_t dv, int32_t rope_dims) {
  if (!q || !k || !v || !cu_seqlens) return ORACLE_ERR_ARG;
  if (num_seqs < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || dqk < 1 || dv < 1) return ORACLE_ERR_ARG;
  if (rope_dims < 0 || rope_dims % 2 != 0 || rope_dims > dqk) return ORACLE_ERR_ARG;
  if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != total_tokens) return ORACLE_ERR_ARG;
  for (int32_t b = 0; b < num_seqs; ++b)
    if (cu_seqlens[b + 1] < cu_seqlens[b]) return ORACLE_ERR_ARG;
  return ORACLE_OK;
}

/* The forward for BF16-bit (f64 == 0) or FP64 (f64 == 1) inputs. */
static int32_t attn_fwd_impl(const void* q, const void* k, const void* v, int f64, const float* sink,
                             const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                             int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, int32_t window,
                             double rope_base, int32_t rope_dims, double v_scale,
                             const int64_t* rows, int64_t n_rows, int32_t nthreads,
                             double* out, double* lse) {
  if (!out || !lse) return ORACLE_ERR_ARG;
  int32_t chk = check_args(q, k, v, cu_seqlens, num_seqs, total_tokens, hq, hkv, dqk, dv, rope_dims);
  if (chk != ORACLE_OK) return chk;
  if (rows == NULL && n_rows != total_tokens) return ORACLE_ERR_ARG;
  for (int64_t r = 0; rows && r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= total_tokens) return ORACLE_ERR_ARG;
  if (nthreads < 1) nthreads = 1;
  if (total_tokens == 0 || n_rows == 0) return ORACLE_OK;

  double* k_rot = (double*)malloc(sizeof(double) * (size_t)total_tokens * hkv * dqk);
  if (!k_rot) return ORACLE_ERR_NOMEM;
  pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  rot_job* rj = (rot_job*)malloc(sizeof(rot_job) * (size_t)nthreads);
  oracle_job* jobs = (oracle_job*)malloc(sizeof(oracle_job) * (size_t)nthreads);
  if (!tid || !rj || !jobs) {
    free(k_rot); free(tid); free(rj); free(jobs);
    return ORACLE_ERR_NOMEM;
  }
  for (int32_t i = 0; i < nthreads; ++i) {
    rj[i].k = k; rj[i].f64 = f64; rj[i].cu = cu_seqlens; rj[i].num_seqs = num_seqs; rj[i].hkv = hkv; rj[i].dqk = dqk;
    rj[i].rope_dims = rope_dims; rj[i].rope_base = rope_base; rj[i].k_rot = k_rot;
    rj[i].t0 = total_tokens * i / nthreads; rj[i].t1 = total_tokens * (i + 1) / nthreads;
    pthread_create(&tid[i], NULL, rotate_keys, &rj[i]);
  }
  for (int32_t i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);

  for (int32_t i = 0; i < nthreads; ++i) {
    oracle_job* J = &jobs[i];
    J->q = q; J->v = v; J->f64 = f64; J->sink = sink; J->cu = cu_seqlens; J->num_seqs = num_seqs;
    J->total_tokens = total_tokens; J->hq = hq; J->hkv = hkv; J->dqk = dqk; J->dv = dv;
    J->window = window; J->rope_dims = rope_dims; J->rope_base = rope_base; J->v_scale = v_scale;
    J->rows = rows; J->n_rows = n_rows; J->k_rot = k_rot; J->out = out; J->lse = lse;
    J->r0 = n_rows * i / nthreads; J->r1 = n_rows * (i + 1) / nthreads; J->status = ORACLE_OK;
    pthread_create(&tid[i], NULL, run_rows, J);
  }
  int32_t status = ORACLE_OK;
  for (int32_t i = 0; i < nthreads; ++i) {
    pthread_join(tid[i], NULL);
    if (jobs[i].status != ORACLE_OK) status = jobs[i].status;
  }
  free(k_rot); free(tid); free(rj); free(jobs);
  return status;
}

/*
 * Full forward (rows == NULL: every token, n_rows must equal total_tokens) or a
 * selection of token rows.  Inputs are BF16 bit patterns in THD layout:
 * q [T, hq, dqk], k [T, hkv, dqk], v [T, hkv, dv]; sink is FP32 [hq] or NULL.
 * window < 0 selects the global causal layer.  Outputs: out [n_rows, hq, dv]
 * and lse [hq, n_rows] in FP64.  Returns 0 on success.
 */
int32_t oracle_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* sink,
                        const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                        int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, int32_t window,
                        double rope_base, int32_t rope_dims, double v_scale,
                        const int64_t* rows, int64_t n_rows, int32_t nthreads,
                        double* out, double* lse) {
  return attn_fwd_impl(q, k, v, 0, sink, cu_seqlens, num_seqs, total_tokens, hq, hkv, dqk, dv, window, rope_base,
                       rope_dims, v_scale, rows, n_rows, nthreads, out, lse);
}

/* The same forward with FP64 inputs (q, k, v as doubles, same layout). */
int32_t oracle_attn_fwd_f64(const double* q, const double* k, const double* v, const float* sink,
                            const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                            int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, int32_t window,
                            double rope_base, int32_t rope_dims, double v_scale,
                            const int64_t* rows, int64_t n_rows, int32_t nthreads,
                            double* out, double* lse) {
  return attn_fwd_impl(q, k, v, 1, sink, cu_seqlens, num_seqs, total_tokens, hq, hkv, dqk, dv, window, rope_base,
                       rope_dims, v_scale, rows, n_rows, nthreads, out, lse);
}

/* Transpose of oracle_rope: each pair is a plane rotation by phi = pos * theta_i,
 * whose transpose is the rotation by -phi, i.e. oracle_rope at position -pos. */
void oracle_rope_transpose(const double* x, int64_t pos, double base, int32_t rope_dims, int32_t dim, double* y) {
  oracle_rope(x, -pos, base, rope_dims, dim, y);
}

/*
 * Backward of the forward above, single-threaded.  Inputs as oracle_attn_fwd
 * (f64 selects FP64 inputs instead of BF16 bits) plus dout [T, hq, dv] and
 * dlse [hq, T] (NULL = 0) in FP64.  Outputs (FP64, overwritten): dq [T, hq, dqk],
 * dk [T, hkv, dqk], dv [T, hkv, dv] and dsink [hq] (may be NULL without a sink).
 */
int32_t oracle_attn_bwd(const void* q, const void* k, const void* v, int32_t f64, const float* sink,
                        const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                        int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, int32_t window,
                        double rope_base, int32_t rope_dims, double v_scale,
                        const double* dout, const double* dlse,
                        double* dq, double* dk, double* dvv, double* dsink) {
  int32_t chk = check_args(q, k, v, cu_seqlens, num_seqs, total_tokens, hq, hkv, dqk, dv, rope_dims);
  if (chk != ORACLE_OK) return chk;
  if (!dout || !dq || !dk || !dvv || (sink && !dsink)) return ORACLE_ERR_ARG;
  const int32_t group = hq / hkv;
  const double inv_sqrt_d = 1.0 / sqrt((double)dqk);
  const size_t T = (size_t)total_tokens;
  memset(dq, 0, sizeof(double) * T * hq * dqk);
  memset(dk, 0, sizeof(double) * T * hkv * dqk);
  memset(dvv, 0, sizeof(double) * T * hkv * dv);
  if (dsink) memset(dsink, 0, sizeof(double) * (size_t)hq);
  if (T == 0) return ORACLE_OK;

  int64_t max_len = 0;
  for (int32_t b = 0; b < num_seqs; ++b) {
    int64_t L = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
    if (L > max_len) max_len = L;
  }
  double* k_rot = (double*)malloc(sizeof(double) * T * hkv * dqk);
  double* dk_rot = (double*)calloc(T * hkv * dqk, sizeof(double));
  double* qx = (double*)malloc(sizeof(double) * (size_t)dqk);
  double* qr = (double*)malloc(sizeof(double) * (size_t)dqk);
  double* dqr = (double*)malloc(sizeof(double) * (size_t)dqk);
  double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
  double* o = (double*)malloc(sizeof(double) * (size_t)dv);
  if (!k_rot || !dk_rot || !qx || !qr || !dqr || !s || !o) {
    free(k_rot); free(dk_rot); free(qx); free(qr); free(dqr); free(s); free(o);
    return ORACLE_ERR_NOMEM;
  }
  rot_job rj;
  rj.k = k; rj.f64 = f64; rj.t0 = 0; rj.t1 = total_tokens; rj.cu = cu_seqlens; rj.num_seqs = num_seqs;
  rj.hkv = hkv; rj.dqk = dqk; rj.rope_dims = rope_dims; rj.rope_base = rope_base; rj.k_rot = k_rot;
  rotate_keys(&rj);

  for (size_t t = 0; t < T; ++t) {
    int32_t b = seq_of_token(cu_seqlens, num_seqs, (int64_t)t);
    int64_t sb = cu_seqlens[b];
    int64_t p = (int64_t)t - sb;
    int64_t lo = 0;
    if (window >= 0 && p - window > 0) lo = p - window;
    for (int32_t h = 0; h < hq; ++h) {
      int32_t g = h / group;
      for (int32_t d = 0; d < dqk; ++d) qx[d] = ld(q, (t * hq + h) * dqk + d, f64);
      oracle_rope(qx, p, rope_base, rope_dims, dqk, qr);
      /* forward of this row: scores, lse, out */
      int has_sink = sink != NULL;
      double sigma = has_sink ? (double)sink[h] : 0.0;
      double M = has_sink ? sigma : -INFINITY;
      for (int64_t j = lo; j <= p; ++j) {
        const double* kr = k_rot + ((size_t)(sb + j) * hkv + g) * dqk;
        double acc = 0.0;
        for (int32_t d = 0; d < dqk; ++d) acc += qr[d] * kr[d];
        s[j - lo] = acc * inv_sqrt_d;
        if (s[j - lo] > M) M = s[j - lo];
      }
      double Z = has_sink ? exp(sigma - M) : 0.0;
      for (int64_t j = lo; j <= p; ++j) Z += exp(s[j - lo] - M);
      double L = M + log(Z);
      for (int32_t d = 0; d < dv; ++d) o[d] = 0.0;
      for (int64_t j = lo; j <= p; ++j) {
        double w = exp(s[j - lo] - L);
        for (int32_t d = 0; d < dv; ++d) o[d] += w * (v_scale * ld(v, ((size_t)(sb + j) * hkv + g) * dv + d, f64));
      }
      /* backward of this row */
      const double* go = dout + (t * hq + h) * dv;
      double gl = dlse ? dlse[(size_t)h * T + t] : 0.0;
      double D = 0.0;
      for (int32_t d = 0; d < dv; ++d) D += go[d] * o[d];
      if (has_sink) dsink[h] += exp(sigma - L) * (gl - D);
      for (int32_t d = 0; d < dqk; ++d) dqr[d] = 0.0;
      for (int64_t j = lo; j <= p; ++j) {
        double pj = exp(s[j - lo] - L);
        size_t vrow = ((size_t)(sb + j) * hkv + g) * dv;
        double dpj = 0.0;
        for (int32_t d = 0; d < dv; ++d) dpj += go[d] * (v_scale * ld(v, vrow + d, f64));
        double ds = pj * (dpj - D + gl);
        for (int32_t d = 0; d < dv; ++d) dvv[vrow + d] += v_scale * pj * go[d];
        const double* kr = k_rot + ((size_t)(sb + j) * hkv + g) * dqk;
        double* dkr = dk_rot + ((size_t)(sb + j) * hkv + g) * dqk;
        for (int32_t d = 0; d < dqk; ++d) {
          dqr[d] += ds * kr[d] * inv_sqrt_d;
          dkr[d] += ds * qr[d] * inv_sqrt_d;
        }
      }
      oracle_rope_transpose(dqr, p, rope_base, rope_dims, dqk, dq + (t * hq + h) * dqk);
    }
  }
  for (size_t t = 0; t < T; ++t) {
    int32_t b = seq_of_token(cu_seqlens, num_seqs, (int64_t)t);
    int64_t p = (int64_t)t - cu_seqlens[b];
    for (int32_t g = 0; g < hkv; ++g)
      oracle_rope_transpose(dk_rot + (t * hkv + g) * dqk, p, rope_base, rope_dims, dqk, dk + (t * hkv + g) * dqk);
  }
  free(k_rot); free(dk_rot); free(qx); free(qr); free(dqr); free(s); free(o);
  return ORACLE_OK;
}
