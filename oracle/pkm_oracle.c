/*
 * pkm_oracle.c -- plain, slow, fp64 CPU oracle for the product-key memory layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The CUDA library never calls it and
 * shares no code with it.
 *
 * What it computes, per token t and head h, with the step each function follows
 * ("Large Memory Layers with Product Keys", gptget.net summary, Methodology and
 * the Deep Analysis / Methodology list, unless another page is named):
 *   1. q = BN(x W_q^T): the query network q(x) is a linear map followed by
 *      inference-mode BatchNorm ("batch normalization in the query network").
 *   2. q_h is split into halves q1, q2 of size dq/2.
 *   3. Each half is scored against its own sub-key codebook (C for q1, C' for q2,
 *      n sub-keys of size dq/2 each): local inner-product search per subspace.
 *   4. The top-k sub-keys of each half are kept (the sets IC and IC').
 *   5. The k x k combined candidates (i, j) score s1[i] + s2[j] -- a key's score is
 *      its left score plus its right score ("Product Keys Give Transformers
 *      Million-Slot Memory Layers", section "Why top-k of each half is enough") --
 *      and the k best are kept. Key (i, j) is left sub-key i joined with right
 *      sub-key j (same page, "Implied keys vs stored sub-keys"); its flat slot is
 *      i*n + j.
 *   6. The k kept scores are turned into weights by a softmax (the pages only say
 *      "weighted sum"; softmax is the reading this library takes).
 *   7. out[t] += sum_j w_j V[slot_j]; heads add into one output.
 * Ordering: every top-k here is by (score descending, id ascending), so ties go to
 * the lower id.
 *
 * All arithmetic is fp64. bf16 inputs are widened exactly (bits << 16).
 * OpenMP runs tokens in parallel; each token's arithmetic is sequential.
 *
 * Pins (tests/test_oracle_pins.py): brute-force top-k over all n^2 explicit keys,
 * library matmul / batch_norm / sort, hand-worked 3x3 example, softmax and
 * identity-table closed forms, finite differences for the backward.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };

static double widen(const void* p, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float*)p)[i];
  uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

typedef struct {
  double s;
  int64_t id;
} scored_t;

/* Total order used everywhere: higher score first; equal scores, lower id first. */
static int better_first(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  if (x->id < y->id) return -1;
  if (x->id > y->id) return 1;
  return 0;
}

/* Step 1: q[f] = ((sum_c x[c] W[f][c]) - mean[f]) / sqrt(var[f] + eps) * gamma[f] + beta[f]. */
static void query_one(const void* x, const void* Wq, int dtype, int64_t t, int d, int F,
                      const float* mean, const float* var, const float* gamma,
                      const float* beta, double eps, double* q) {
  for (int f = 0; f < F; ++f) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c)
      acc += widen(x, dtype, t * (int64_t)d + c) * widen(Wq, dtype, (int64_t)f * d + c);
    q[f] = (acc - (double)mean[f]) / sqrt((double)var[f] + eps) * (double)gamma[f] +
           (double)beta[f];
  }
}

/* Step 3: s[i] = <q_half, sub-key i> for one codebook of n sub-keys of size half. */
static void half_scores(const double* qh, const void* book, int dtype, int64_t book_off,
                        int n, int half, double* s) {
  for (int i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int e = 0; e < half; ++e)
      acc += qh[e] * widen(book, dtype, book_off + (int64_t)i * half + e);
    s[i] = acc;
  }
}

/* Steps 4 and 5: sort all entries in the total order; the caller keeps the first k. */
static void sort_best_first(scored_t* all, int64_t count) {
  qsort(all, (size_t)count, sizeof(scored_t), better_first);
}

/* One token, all heads, steps 2-7 from its query q [H*dq]. Scratch is allocated per
 * call. */
static int search_token(int64_t t, int H, int dq, int n, int k, int v, int dtype,
                        const double* q, const void* subkeys, const void* values, double* out,
                        int32_t* indices, double* weights, double* scores, double* half_out) {
  const int half = dq / 2;
  double* s = (double*)malloc(sizeof(double) * 2 * n);
  scored_t* lists = (scored_t*)malloc(sizeof(scored_t) * 2 * (size_t)n);
  scored_t* cand = (scored_t*)malloc(sizeof(scored_t) * (size_t)k * k);
  if (!s || !lists || !cand) {
    free(s); free(lists); free(cand);
    return -1;
  }
  if (out)
    for (int c = 0; c < v; ++c) out[t * (int64_t)v + c] = 0.0;

  for (int h = 0; h < H; ++h) {
    /* Steps 2-4 for both halves. */
    for (int sh = 0; sh < 2; ++sh) {
      const double* qh = q + h * dq + sh * half;
      int64_t book_off = ((int64_t)(h * 2 + sh) * n) * half;
      half_scores(qh, subkeys, dtype, book_off, n, half, s + sh * n);
      if (half_out)
        memcpy(half_out + ((t * H + h) * 2 + sh) * (int64_t)n, s + sh * n,
               sizeof(double) * n);
      scored_t* L = lists + sh * n;
      for (int i = 0; i < n; ++i) {
        L[i].s = s[sh * n + i];
        L[i].id = i;
      }
      sort_best_first(L, n);
    }
    /* Step 5: the k x k candidates, flat slot i*n + j. */
    for (int a = 0; a < k; ++a)
      for (int b = 0; b < k; ++b) {
        cand[a * k + b].s = lists[a].s + lists[n + b].s;
        cand[a * k + b].id = lists[a].id * (int64_t)n + lists[n + b].id;
      }
    sort_best_first(cand, (int64_t)k * k);
    /* Step 6: softmax over the k kept scores (max subtracted). */
    double mx = cand[0].s, den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(cand[j].s - mx);
    for (int j = 0; j < k; ++j) {
      int64_t o = (t * H + h) * (int64_t)k + j;
      double w = exp(cand[j].s - mx) / den;
      if (indices) indices[o] = (int32_t)cand[j].id;
      if (weights) weights[o] = w;
      if (scores) scores[o] = cand[j].s;
      /* Step 7: weighted value rows, summed over heads. */
      if (out)
        for (int c = 0; c < v; ++c)
          out[t * (int64_t)v + c] += w * widen(values, dtype, cand[j].id * (int64_t)v + c);
    }
  }
  free(s); free(lists); free(cand);
  return 0;
}

/* One token, all heads: steps 1-7. */
static int forward_token(int64_t t, int d, int H, int dq, int n, int k, int v, int dtype,
                         double eps, const void* x, const void* Wq, const float* mean,
                         const float* var, const float* gamma, const float* beta,
                         const void* subkeys, const void* values, double* out,
                         int32_t* indices, double* weights, double* scores, double* q_out,
                         double* half_out) {
  const int F = H * dq;
  double* q = (double*)malloc(sizeof(double) * F);
  if (!q) return -1;
  query_one(x, Wq, dtype, t, d, F, mean, var, gamma, beta, eps, q);
  if (q_out) memcpy(q_out + t * F, q, sizeof(double) * F);
  const int rc = search_token(t, H, dq, n, k, v, dtype, q, subkeys, values, out, indices,
                              weights, scores, half_out);
  free(q);
  return rc;
}

/* acc[t][f] = sum_c x[t][c] W[f][c] for every token (the linear map of step 1). */
static void linear_all(int64_t B, int d, int F, int dtype, const void* x, const void* Wq,
                       double* acc) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t t = 0; t < B; ++t)
    for (int f = 0; f < F; ++f) {
      double a = 0.0;
      for (int c = 0; c < d; ++c)
        a += widen(x, dtype, t * (int64_t)d + c) * widen(Wq, dtype, (int64_t)f * d + c);
      acc[t * F + f] = a;
    }
}

/* BatchNorm training-mode statistics of acc over the batch, per feature:
 * mean = (1/B) sum_t acc, var = (1/B) sum_t (acc - mean)^2 (the biased variance that
 * normalises the batch). Two passes, tokens in order. */
static void batch_stats(int64_t B, int F, const double* acc, double* mean, double* var) {
  for (int f = 0; f < F; ++f) {
    double s = 0.0;
    for (int64_t t = 0; t < B; ++t) s += acc[t * F + f];
    const double mu = s / (double)B;
    double m2 = 0.0;
    for (int64_t t = 0; t < B; ++t) m2 += (acc[t * F + f] - mu) * (acc[t * F + f] - mu);
    mean[f] = mu;
    var[f] = m2 / (double)B;
  }
}

/*
 * Forward for B tokens. Outputs (any may be NULL):
 *   out [B][v], indices [B][H][k] (flat slot i*n+j), weights [B][H][k],
 *   scores [B][H][k] (kept key scores), q_out [B][H*dq], half_out [B][H][2][n].
 * Layouts of the inputs: x [B][d], Wq [H*dq][d], BN vectors [H*dq] (fp32),
 * subkeys [H][2][n][dq/2], values [n*n][v]. dtype 0 = fp32, 1 = bf16 bit patterns.
 * Returns 0, or -1 on bad sizes / allocation failure.
 */
int pkm_oracle_forward(int64_t B, int d, int H, int dq, int n, int k, int v, int dtype,
                       double eps, const void* x, const void* Wq, const float* mean,
                       const float* var, const float* gamma, const float* beta,
                       const void* subkeys, const void* values, double* out,
                       int32_t* indices, double* weights, double* scores, double* q_out,
                       double* half_out, int nthreads) {
  if (B < 0 || d < 1 || H < 1 || dq < 2 || dq % 2 || n < 1 || k < 1 || k > n || v < 0)
    return -1;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
  for (int64_t t = 0; t < B; ++t)
    err |= forward_token(t, d, H, dq, n, k, v, dtype, eps, x, Wq, mean, var, gamma, beta,
                         subkeys, values, out, indices, weights, scores, q_out, half_out)
               ? 1 : 0;
  (void)nthreads;
  return err ? -1 : 0;
}

/*
 * Forward with BatchNorm in training mode (the query network's "batch
 * normalization" while the model trains): the batch's own statistics normalise it,
 *   q = (acc - mean_B) / sqrt(var_B + eps) * gamma + beta,
 * mean_B, var_B from batch_stats, and the running statistics move towards them:
 *   running_mean' = (1 - momentum) running_mean + momentum mean_B
 *   running_var'  = (1 - momentum) running_var  + momentum var_B B / (B - 1)
 * (the unbiased variance, as the common BatchNorm layers keep it). Steps 2-7 as in
 * pkm_oracle_forward. Outputs as pkm_oracle_forward plus batch_mean, batch_var,
 * new_running_mean, new_running_var [H*dq] (fp64; any may be NULL). B >= 2.
 */
int pkm_oracle_forward_train(int64_t B, int d, int H, int dq, int n, int k, int v, int dtype,
                             double eps, double momentum, const void* x, const void* Wq,
                             const float* running_mean, const float* running_var,
                             const float* gamma, const float* beta, const void* subkeys,
                             const void* values, double* out, int32_t* indices,
                             double* weights, double* scores, double* q_out, double* half_out,
                             double* batch_mean, double* batch_var, double* new_running_mean,
                             double* new_running_var, int nthreads) {
  if (B < 2 || d < 1 || H < 1 || dq < 2 || dq % 2 || n < 1 || k < 1 || k > n || v < 0)
    return -1;
  const int F = H * dq;
  double* acc = (double*)malloc(sizeof(double) * (size_t)B * F);
  double* mu = (double*)malloc(sizeof(double) * F);
  double* var = (double*)malloc(sizeof(double) * F);
  double* q = (double*)malloc(sizeof(double) * (size_t)B * F);
  if (!acc || !mu || !var || !q) {
    free(acc); free(mu); free(var); free(q);
    return -1;
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
  linear_all(B, d, F, dtype, x, Wq, acc);
  batch_stats(B, F, acc, mu, var);
  for (int64_t t = 0; t < B; ++t)
    for (int f = 0; f < F; ++f)
      q[t * F + f] = (acc[t * F + f] - mu[f]) / sqrt(var[f] + eps) * (double)gamma[f] +
                     (double)beta[f];
  int err = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
  for (int64_t t = 0; t < B; ++t)
    err |= search_token(t, H, dq, n, k, v, dtype, q + t * F, subkeys, values, out, indices,
                        weights, scores, half_out) ? 1 : 0;
  if (q_out) memcpy(q_out, q, sizeof(double) * (size_t)B * F);
  for (int f = 0; f < F; ++f) {
    if (batch_mean) batch_mean[f] = mu[f];
    if (batch_var) batch_var[f] = var[f];
    if (new_running_mean)
      new_running_mean[f] = (1.0 - momentum) * (double)running_mean[f] + momentum * mu[f];
    if (new_running_var)
      new_running_var[f] = (1.0 - momentum) * (double)running_var[f] +
                           momentum * var[f] * (double)B / (double)(B - 1);
  }
  free(acc); free(mu); free(var); free(q);
  (void)nthreads;
  return err ? -1 : 0;
}

/*
 * Brute force over the implied keys ("Product Keys Give Transformers Million-Slot
 * Memory Layers", sections "Implied keys vs stored sub-keys" and "Search cost:
 * flat vs product keys"): for every (i, j) build the full dq-long key
 * C[i] joined with C'[j], take its inner product with the whole query head q_h,
 * and keep the top-k of all n*n keys. Uses no per-half score at all.
 * q [B][H*dq] fp64 (from pkm_oracle_forward's q_out), out_idx / out_score [B][H][k].
 */
int pkm_oracle_flat_topk(int64_t B, int H, int dq, int n, int k, int dtype, const double* q,
                         const void* subkeys, int32_t* out_idx, double* out_score,
                         int nthreads) {
  if (B < 0 || H < 1 || dq < 2 || dq % 2 || n < 1 || k < 1 || k > n * n) return -1;
  const int half = dq / 2;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
  for (int64_t th = 0; th < B * H; ++th) {
    int64_t t = th / H;
    int h = (int)(th % H);
    scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)n * n);
    double* key = (double*)malloc(sizeof(double) * dq);
    if (!all || !key) {
      free(all); free(key);
      err |= 1;
      continue;
    }
    const double* qh = q + t * (int64_t)H * dq + (int64_t)h * dq;
    int64_t offC = ((int64_t)(h * 2 + 0) * n) * half;
    int64_t offCp = ((int64_t)(h * 2 + 1) * n) * half;
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) {
        for (int e = 0; e < half; ++e) {
          key[e] = widen(subkeys, dtype, offC + (int64_t)i * half + e);
          key[half + e] = widen(subkeys, dtype, offCp + (int64_t)j * half + e);
        }
        double acc = 0.0;
        for (int e = 0; e < dq; ++e) acc += qh[e] * key[e];
        all[(int64_t)i * n + j].s = acc;
        all[(int64_t)i * n + j].id = (int64_t)i * n + j;
      }
    sort_best_first(all, (int64_t)n * n);
    for (int j = 0; j < k; ++j) {
      out_idx[th * k + j] = (int32_t)all[j].id;
      out_score[th * k + j] = all[j].s;
    }
    free(all); free(key);
  }
  (void)nthreads;
  return err ? -1 : 0;
}

/*
 * Steps 6-7 alone, for given kept scores and slots: softmax, then the weighted
 * value sum over heads. scores/indices [B][H][k]; weights [B][H][k]; out [B][v].
 * Used for finite differences and to re-finish a selection made elsewhere.
 */
int pkm_oracle_finish(int64_t B, int H, int k, int v, int dtype, const double* scores,
                      const int32_t* indices, const void* values, double* weights,
                      double* out) {
  if (B < 0 || H < 1 || k < 1 || v < 0) return -1;
  for (int64_t t = 0; t < B; ++t) {
    if (out)
      for (int c = 0; c < v; ++c) out[t * (int64_t)v + c] = 0.0;
    for (int h = 0; h < H; ++h) {
      const double* s = scores + (t * H + h) * (int64_t)k;
      double mx = s[0];
      for (int j = 1; j < k; ++j)
        if (s[j] > mx) mx = s[j];
      double den = 0.0;
      for (int j = 0; j < k; ++j) den += exp(s[j] - mx);
      for (int j = 0; j < k; ++j) {
        double w = exp(s[j] - mx) / den;
        int64_t o = (t * H + h) * (int64_t)k + j;
        if (weights) weights[o] = w;
        if (out)
          for (int c = 0; c < v; ++c)
            out[t * (int64_t)v + c] +=
                w * widen(values, dtype, (int64_t)indices[o] * v + c);
      }
    }
  }
  return 0;
}

/*
 * Sparse value backward ("trained end-to-end with sparse updates"; the Deep
 * Analysis / Methodology list: all parameters learn by backpropagation and only
 * a few memory slots are updated). With L = <grad_out, out>:
 *   g_w[j]   = <grad_out[t], V[slot_j]>
 *   g_s[j]   = w_j * (g_w[j] - sum_l w_l g_w[l])        (softmax Jacobian)
 *   G[slot] += w_j * grad_out[t]                         (only the kept slots)
 * grad_out [B][v] in dtype; indices/weights [B][H][k]; grad_scores [B][H][k].
 * row_slot [n*n] maps a slot to a row of grad_values (-1 = not stored; NULL =
 * identity); grad_values [rows][v] is ACCUMULATED into.
 */
int pkm_oracle_backward(int64_t B, int H, int k, int v, int dtype, const void* values,
                        const void* grad_out, const int32_t* indices, const double* weights,
                        const int64_t* row_slot, double* grad_values, double* grad_scores) {
  if (B < 0 || H < 1 || k < 1 || v < 0) return -1;
  double* gw = (double*)malloc(sizeof(double) * (size_t)k);
  if (!gw) return -1;
  for (int64_t t = 0; t < B; ++t)
    for (int h = 0; h < H; ++h) {
      int64_t base = (t * H + h) * (int64_t)k;
      double wsum = 0.0;
      for (int j = 0; j < k; ++j) {
        double acc = 0.0;
        for (int c = 0; c < v; ++c)
          acc += widen(grad_out, dtype, t * (int64_t)v + c) *
                 widen(values, dtype, (int64_t)indices[base + j] * v + c);
        gw[j] = acc;
        wsum += weights[base + j] * acc;
      }
      for (int j = 0; j < k; ++j) {
        if (grad_scores) grad_scores[base + j] = weights[base + j] * (gw[j] - wsum);
        if (grad_values) {
          int64_t r = row_slot ? row_slot[indices[base + j]] : indices[base + j];
          if (r < 0) continue;
          for (int c = 0; c < v; ++c)
            grad_values[r * v + c] += weights[base + j] * widen(grad_out, dtype, t * (int64_t)v + c);
        }
      }
    }
  free(gw);
  return 0;
}

/*
 * Memory utilisation of one batch: the number of distinct slots among the B*H*k picks
 * (the pages report the share of memory slots a trained layer uses, with and without
 * BatchNorm in the query network). indices [B][H][k]; slots = n*n. Ids outside
 * [0, slots) are not counted; their number goes to *bad (if not NULL).
 * Returns the count of distinct slots, or -1 on bad sizes / allocation failure.
 */
int64_t pkm_oracle_slot_usage(int64_t picks, const int32_t* indices, int64_t slots,
                              int64_t* bad) {
  if (picks < 0 || slots < 1) return -1;
  unsigned char* seen = (unsigned char*)calloc((size_t)slots, 1);
  if (!seen) return -1;
  int64_t distinct = 0, nbad = 0;
  for (int64_t e = 0; e < picks; ++e) {
    const int64_t r = indices[e];
    if (r < 0 || r >= slots) {
      ++nbad;
      continue;
    }
    if (!seen[r]) {
      seen[r] = 1;
      ++distinct;
    }
  }
  free(seen);
  if (bad) *bad = nbad;
  return distinct;
}

/*
 * Full backward of the layer with the selection held fixed (the top-k choice is
 * piecewise constant, so no gradient flows through it). With L = <grad_out, out>,
 * for token t, head h and kept key j = (i_j, i'_j) (slot = i_j*n + i'_j):
 *   g_c[j]  = w_j (g_j - sum_l w_l g_l),  g_j = <grad_out[t], V[slot_j]>
 *   dL/dq1  = sum_j g_c[j] C_h[i_j]          dL/dq2 = sum_j g_c[j] C'_h[i'_j]
 *   dL/dC_h[i]   += sum over (t, j) with i_j = i  of g_c[t,j] q1[t]   (same for C')
 *   q = (acc - mean) / sqrt(var + eps) * gamma + beta,  acc = x W^T,
 *   xhat = (acc - mean) / sqrt(var + eps):
 *   dL/dgamma = sum_t dL/dq xhat;  dL/dbeta = sum_t dL/dq;
 *   dL/dW = dL/dacc^T x;  dL/dx = dL/dacc W, where
 *     inference BatchNorm (bn_training = 0; mean, var are the running statistics,
 *     constants):  dL/dacc = dL/dq gamma / sqrt(var + eps)
 *     training BatchNorm (bn_training = 1; mean, var are the batch's own, recomputed
 *     here from acc, and depend on every token -- the backward of batch
 *     normalisation, Ioffe and Szegedy 2015):
 *       dL/dacc = gamma / sqrt(var + eps) (dL/dq - (1/B) sum_t dL/dq
 *                                          - xhat (1/B) sum_t dL/dq xhat)
 * Outputs (fp64, overwritten; any may be NULL): grad_x [B][d], grad_W [H*dq][d],
 * grad_gamma, grad_beta [H*dq], grad_subkeys [H][2][n][dq/2], grad_q [B][H*dq].
 * indices / weights [B][H][k] are the forward's picks; grad_out [B][v] in dtype.
 * Every sum over tokens runs in token order; independent outputs run in parallel.
 */
int pkm_oracle_backward_full(int64_t B, int d, int H, int dq, int n, int k, int v, int dtype,
                             double eps, int bn_training, const void* x, const void* Wq,
                             const float* mean, const float* var, const float* gamma,
                             const float* beta, const void* subkeys, const void* values,
                             const int32_t* indices, const double* weights,
                             const void* grad_out, double* grad_x, double* grad_W,
                             double* grad_gamma, double* grad_beta, double* grad_subkeys,
                             double* grad_q_out) {
  if (B < 0 || d < 1 || H < 1 || dq < 2 || dq % 2 || n < 1 || k < 1 || k > n || v < 1) return -1;
  if (bn_training && B < 2) return -1;
  const int F = H * dq, half = dq / 2;
  const size_t BF = (size_t)B * F;
  double* acc = (double*)malloc(sizeof(double) * (BF ? BF : 1));
  double* gq = (double*)calloc(BF ? BF : 1, sizeof(double));
  double* gacc = (double*)malloc(sizeof(double) * (BF ? BF : 1));
  double* mu = (double*)malloc(sizeof(double) * F);
  double* sd = (double*)malloc(sizeof(double) * F);   /* sqrt(var + eps) */
  double* q = (double*)malloc(sizeof(double) * F);
  double* gw = (double*)malloc(sizeof(double) * k);
  double* gc = (double*)malloc(sizeof(double) * k);
  if (!acc || !gq || !gacc || !mu || !sd || !q || !gw || !gc) {
    free(acc); free(gq); free(gacc); free(mu); free(sd); free(q); free(gw); free(gc);
    return -1;
  }
  if (grad_subkeys) memset(grad_subkeys, 0, sizeof(double) * (size_t)H * 2 * n * half);
  /* Step 1 again (acc = x W^T), and the statistics BatchNorm used. */
  linear_all(B, d, F, dtype, x, Wq, acc);
  if (bn_training) {
    batch_stats(B, F, acc, mu, sd);
    for (int f = 0; f < F; ++f) sd[f] = sqrt(sd[f] + eps);
  } else {
    for (int f = 0; f < F; ++f) {
      mu[f] = (double)mean[f];
      sd[f] = sqrt((double)var[f] + eps);
    }
  }
  for (int64_t t = 0; t < B; ++t) {
    for (int f = 0; f < F; ++f)
      q[f] = (acc[t * F + f] - mu[f]) / sd[f] * (double)gamma[f] + (double)beta[f];
    double* g = gq + t * F;
    for (int h = 0; h < H; ++h) {
      const int64_t base = (t * H + h) * (int64_t)k;
      /* Gradient wrt the kept scores (softmax Jacobian). */
      double wsum = 0.0;
      for (int j = 0; j < k; ++j) {
        double a = 0.0;
        for (int c = 0; c < v; ++c)
          a += widen(grad_out, dtype, t * (int64_t)v + c) *
               widen(values, dtype, (int64_t)indices[base + j] * v + c);
        gw[j] = a;
        wsum += weights[base + j] * a;
      }
      for (int j = 0; j < k; ++j) gc[j] = weights[base + j] * (gw[j] - wsum);
      /* A kept score is s1[i] + s2[i']: its gradient goes to both halves. */
      for (int j = 0; j < k; ++j) {
        const int64_t slot = indices[base + j];
        const int64_t sub[2] = {slot / n, slot % n};
        for (int side = 0; side < 2; ++side) {
          const int64_t row = ((int64_t)(h * 2 + side) * n + sub[side]) * half;
          for (int e = 0; e < half; ++e) {
            const int f = h * dq + side * half + e;
            g[f] += gc[j] * widen(subkeys, dtype, row + e);
            if (grad_subkeys) grad_subkeys[row + e] += gc[j] * q[f];
          }
        }
      }
    }
  }
  if (grad_q_out) memcpy(grad_q_out, gq, sizeof(double) * BF);
  /* Through BatchNorm. */
  for (int f = 0; f < F; ++f) {
    double sb = 0.0, sg = 0.0;
    for (int64_t t = 0; t < B; ++t) {
      sb += gq[t * F + f];
      sg += gq[t * F + f] * ((acc[t * F + f] - mu[f]) / sd[f]);
    }
    if (grad_beta) grad_beta[f] = sb;
    if (grad_gamma) grad_gamma[f] = sg;
    for (int64_t t = 0; t < B; ++t) {
      const double gt = gq[t * F + f];
      if (bn_training) {
        const double xhat = (acc[t * F + f] - mu[f]) / sd[f];
        gacc[t * F + f] = (double)gamma[f] / sd[f] *
                          (gt - sb / (double)B - xhat * sg / (double)B);
      } else {
        gacc[t * F + f] = gt * (double)gamma[f] / sd[f];
      }
    }
  }
  /* Through the linear map. */
  if (grad_W) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int f = 0; f < F; ++f)
      for (int c = 0; c < d; ++c) {
        double a = 0.0;
        for (int64_t t = 0; t < B; ++t)
          a += gacc[t * F + f] * widen(x, dtype, t * (int64_t)d + c);
        grad_W[(int64_t)f * d + c] = a;
      }
  }
  if (grad_x) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int64_t t = 0; t < B; ++t)
      for (int c = 0; c < d; ++c) {
        double a = 0.0;
        for (int f = 0; f < F; ++f) a += gacc[t * F + f] * widen(Wq, dtype, (int64_t)f * d + c);
        grad_x[t * (int64_t)d + c] = a;
      }
  }
  free(acc); free(gq); free(gacc); free(mu); free(sd); free(q); free(gw); free(gc);
  return 0;
}
