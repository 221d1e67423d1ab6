/*
 * flce_oracle.c -- fp64 CPU oracle for fused linear cross-entropy (FLCE).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or run this file.  The GPU library
 * never calls it and shares no code, header or constant with it.
 *
 * What it computes is the plain definition of the loss that the pages
 * discuss, written out without blocking, chunking or fusion:
 *
 *   z_ij   = sum_k X_ik W_jk                 the "softmax_input" matmul
 *            (PyTorch PR #126348 summary, step 1; nn.Linear(C, V, bias=False)
 *            weight layout V x H from that PR's test fragment)
 *   y_ij   = c*tanh(z_ij/c) when a softcap c is on, else z_ij
 *            (Gemma2 logit softcap named in Liger-Kernel issue #227)
 *   m_i    = max_j y_ij                        (#126348 step 2)
 *   lse_i  = m_i + log sum_j exp(y_ij - m_i)   (#126348 step 3)
 *   valid_i = label_i != ignore_index
 *   N      = sum_i valid_i
 *   loss   = (1/N) sum_{valid i} (lse_i - y_{i,label_i}),  0 when N == 0
 *            (mean NLL against labels, torchtune issue #1228, the
 *            loss_fn(logits, labels) call in the training step)
 *   G_ij   = valid_i (exp(y_ij - lse_i) - [j == label_i]) s_ij dloss / N
 *            with s_ij = 1 - tanh^2(z_ij/c) under a softcap, else 1;
 *            dloss is the upstream scale (the recipe divides the loss by the
 *            gradient-accumulation count before backward, torchtune #1228).
 *            The softmax is rebuilt from z and lse, as #126348 proposes for
 *            the backward pass, rather than saved.
 *   dX     = G W          dW = G^T X
 *
 * Every quantity is fp64.  bf16 and fp32 inputs are widened exactly.
 * Rows are independent, so loops over rows or vocabulary entries run in
 * parallel with OpenMP; every sum over an index is taken in increasing index
 * order inside one thread, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_BF16 0
#define OR_FP32 1
#define OR_FP64 2

#define OR_OK 0
#define OR_INVALID 1
#define OR_BAD_LABEL 2
#define OR_NOMEM 3

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Widen row `row` (length n) of a row-major matrix into dst. */
static void widen_row(double* dst, const void* base, int dtype, int64_t row, int64_t n) {
  int64_t k;
  if (dtype == OR_BF16) {
    const uint16_t* s = (const uint16_t*)base + row * n;
    for (k = 0; k < n; ++k) dst[k] = bf16_bits_to_double(s[k]);
  } else if (dtype == OR_FP32) {
    const float* s = (const float*)base + row * n;
    for (k = 0; k < n; ++k) dst[k] = (double)s[k];
  } else {
    const double* s = (const double*)base + row * n;
    for (k = 0; k < n; ++k) dst[k] = s[k];
  }
}

static int softcap_on(double c) { return c > 0.0 && isfinite(c); }

int flce_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Number of rows whose label is not ignore_index. */
int64_t flce_oracle_count_valid(const int64_t* labels, int64_t BT, int64_t ignore_index) {
  int64_t i, n = 0;
  for (i = 0; i < BT; ++i) n += (labels[i] != ignore_index);
  return n;
}

/*
 * Full forward + backward on BT rows.
 *
 * X: BT x H, W: V x H, both row-major in `dtype` (bf16 bits, fp32 or fp64).
 * n_valid: divisor N of the mean; pass < 0 to count it from these labels
 *          (a caller that runs a subset of rows passes the global count).
 * Outputs (fp64): lse[BT], target[BT] (y_{i,label_i}, NaN on ignored rows),
 *          *n_valid_out, *loss_out, and when non-NULL dX[BT*H], dW[V*H].
 * Returns OR_OK, OR_INVALID, OR_BAD_LABEL (a label outside [0, V) that is not
 * ignore_index) or OR_NOMEM.
 */
int flce_oracle(int64_t BT, int64_t H, int64_t V, int dtype, const void* X, const void* W,
                const int64_t* labels, int64_t ignore_index, double softcap, int64_t n_valid,
                double dloss, double* lse, double* target, int64_t* n_valid_out,
                double* loss_out, double* dX, double* dW) {
  int64_t i, j;
  const int capped = softcap_on(softcap);
  double *Xd = NULL, *Z = NULL, loss = 0.0, scale;

  if (BT < 0 || H <= 0 || V <= 0 || (dtype != OR_BF16 && dtype != OR_FP32 && dtype != OR_FP64))
    return OR_INVALID;
  if (BT > 0 && (!X || !labels)) return OR_INVALID;
  if (!W || !lse || !target || !n_valid_out || !loss_out) return OR_INVALID;
  for (i = 0; i < BT; ++i)
    if (labels[i] != ignore_index && (labels[i] < 0 || labels[i] >= V)) return OR_BAD_LABEL;
  if (n_valid < 0) n_valid = flce_oracle_count_valid(labels, BT, ignore_index);
  *n_valid_out = n_valid;

  Xd = (double*)malloc(sizeof(double) * (size_t)(BT > 0 ? BT : 1) * (size_t)H);
  Z = (double*)malloc(sizeof(double) * (size_t)(BT > 0 ? BT : 1) * (size_t)V);
  if (!Xd || !Z) { free(Xd); free(Z); return OR_NOMEM; }
  for (i = 0; i < BT; ++i) widen_row(Xd + i * H, X, dtype, i, H);

  /* Step 1: z_ij = sum_k X_ik W_jk (sum in increasing k). */
#pragma omp parallel
  {
    double* w = (double*)malloc(sizeof(double) * (size_t)H);
    int64_t jj, ii, kk;
#pragma omp for schedule(static)
    for (jj = 0; jj < V; ++jj) {
      widen_row(w, W, dtype, jj, H);
      for (ii = 0; ii < BT; ++ii) {
        const double* x = Xd + ii * H;
        double acc = 0.0;
        for (kk = 0; kk < H; ++kk) acc += x[kk] * w[kk];
        Z[ii * V + jj] = acc;
      }
    }
    free(w);
  }

  /* Steps 2-3 per row: softcap, max, log-sum-exp, target logit. */
#pragma omp parallel for schedule(static)
  for (i = 0; i < BT; ++i) {
    double* z = Z + i * V;
    double m = -INFINITY, s = 0.0;
    int64_t jj;
    for (jj = 0; jj < V; ++jj) {
      double y = capped ? softcap * tanh(z[jj] / softcap) : z[jj];
      if (y > m) m = y;
    }
    for (jj = 0; jj < V; ++jj) {
      double y = capped ? softcap * tanh(z[jj] / softcap) : z[jj];
      s += exp(y - m);
    }
    lse[i] = m + log(s);
    if (labels[i] != ignore_index) {
      double zt = z[labels[i]];
      target[i] = capped ? softcap * tanh(zt / softcap) : zt;
    } else {
      target[i] = NAN;
    }
  }

  /* Mean NLL over the valid rows, summed in row order. */
  for (i = 0; i < BT; ++i)
    if (labels[i] != ignore_index) loss += lse[i] - target[i];
  *loss_out = n_valid > 0 ? loss / (double)n_valid : 0.0;

  if (!dX && !dW) { free(Xd); free(Z); return OR_OK; }

  /* G overwrites Z:  G_ij = valid_i (p_ij - [j == label_i]) s_ij dloss / N. */
  scale = n_valid > 0 ? dloss / (double)n_valid : 0.0;
#pragma omp parallel for schedule(static)
  for (i = 0; i < BT; ++i) {
    double* z = Z + i * V;
    int64_t jj;
    const int valid = labels[i] != ignore_index;
    for (jj = 0; jj < V; ++jj) {
      double g = 0.0;
      if (valid && n_valid > 0) {
        double t = capped ? tanh(z[jj] / softcap) : 0.0;
        double y = capped ? softcap * t : z[jj];
        double p = exp(y - lse[i]);
        double d = capped ? 1.0 - t * t : 1.0;
        g = (p - (jj == labels[i] ? 1.0 : 0.0)) * d * scale;
      }
      z[jj] = g;
    }
  }

  /* dX = G W : row i of dX is sum_j G_ij W_j (increasing j). */
  if (dX) {
#pragma omp parallel
    {
      double* w = (double*)malloc(sizeof(double) * (size_t)H);
      int64_t ii, jj, kk;
#pragma omp for schedule(static)
      for (ii = 0; ii < BT; ++ii) {
        double* out = dX + ii * H;
        for (kk = 0; kk < H; ++kk) out[kk] = 0.0;
        for (jj = 0; jj < V; ++jj) {
          double g = Z[ii * V + jj];
          if (g == 0.0) continue;
          widen_row(w, W, dtype, jj, H);
          for (kk = 0; kk < H; ++kk) out[kk] += g * w[kk];
        }
      }
      free(w);
    }
  }

  /* dW = G^T X : row j of dW is sum_i G_ij X_i (increasing i). */
  if (dW) {
#pragma omp parallel for schedule(static)
    for (j = 0; j < V; ++j) {
      double* out = dW + j * H;
      int64_t ii, kk;
      for (kk = 0; kk < H; ++kk) out[kk] = 0.0;
      for (ii = 0; ii < BT; ++ii) {
        double g = Z[ii * V + j];
        const double* x = Xd + ii * H;
        if (g == 0.0) continue;
        for (kk = 0; kk < H; ++kk) out[kk] += g * x[kk];
      }
    }
  }
  free(Xd);
  free(Z);
  return OR_OK;
}

/*
 * Cross-entropy for a caller that already holds the logits ("softmax_input"),
 * the exact case of PyTorch PR #126348 ("[AOTAutograd] tweak min-cut
 * partitioner to avoid saving softmax output", summary steps 1-4 and points
 * a./b.): the forward needs only the per-row max and sum (steps 2-3) and the
 * label's entry (point a.); the backward rebuilds the softmax from the
 * logits and those row statistics (point b.) instead of reading a saved
 * softmax_output.  In fp64, with the same softcap, ignore_index and mean
 * conventions as flce_oracle:
 *
 *   y_ij    = c*tanh(z_ij/c) under a softcap c, else z_ij
 *   lse_i   = m_i + log sum_j exp(y_ij - m_i),  m_i = max_j y_ij
 *   loss    = (1/N) sum_{valid i} (lse_i - y_{i,label_i}),  0 when N == 0
 *   dZ_ij   = valid_i (exp(y_ij - lse_i) - [j == label_i]) s_ij dloss / N
 *
 * logits: BT rows of V entries, row i starting at element i*ld (ld >= V), in
 * `dtype` (bf16 bits, fp32 or fp64).  n_valid < 0 counts N from these labels.
 * Outputs: lse[BT], target[BT] (NaN on ignored rows), *n_valid_out,
 * *loss_out and, when non-NULL, dZ (BT x V, dense, fp64).
 */
static double widen_at(const void* base, int dtype, int64_t idx) {
  if (dtype == OR_BF16) return bf16_bits_to_double(((const uint16_t*)base)[idx]);
  if (dtype == OR_FP32) return (double)((const float*)base)[idx];
  return ((const double*)base)[idx];
}

int flce_oracle_ce(int64_t BT, int64_t V, int dtype, const void* logits, int64_t ld,
                   const int64_t* labels, int64_t ignore_index, double softcap, int64_t n_valid,
                   double dloss, double* lse, double* target, int64_t* n_valid_out,
                   double* loss_out, double* dZ) {
  int64_t i;
  const int capped = softcap_on(softcap);
  double loss = 0.0, scale;

  if (BT < 0 || V <= 0 || ld < V || (dtype != OR_BF16 && dtype != OR_FP32 && dtype != OR_FP64))
    return OR_INVALID;
  if (BT > 0 && (!logits || !labels)) return OR_INVALID;
  if (!lse || !target || !n_valid_out || !loss_out) return OR_INVALID;
  for (i = 0; i < BT; ++i)
    if (labels[i] != ignore_index && (labels[i] < 0 || labels[i] >= V)) return OR_BAD_LABEL;
  if (n_valid < 0) n_valid = flce_oracle_count_valid(labels, BT, ignore_index);
  *n_valid_out = n_valid;

  /* Steps 2-3 per row: softcap, max, log-sum-exp; the label's entry. */
#pragma omp parallel for schedule(static)
  for (i = 0; i < BT; ++i) {
    int64_t j;
    double m = -INFINITY, s = 0.0;
    for (j = 0; j < V; ++j) {
      double z = widen_at(logits, dtype, i * ld + j);
      double y = capped ? softcap * tanh(z / softcap) : z;
      if (y > m) m = y;
    }
    for (j = 0; j < V; ++j) {
      double z = widen_at(logits, dtype, i * ld + j);
      double y = capped ? softcap * tanh(z / softcap) : z;
      s += exp(y - m);
    }
    lse[i] = m + log(s);
    if (labels[i] != ignore_index) {
      double zt = widen_at(logits, dtype, i * ld + labels[i]);
      target[i] = capped ? softcap * tanh(zt / softcap) : zt;
    } else {
      target[i] = NAN;
    }
  }

  /* Mean NLL over the valid rows, summed in row order. */
  for (i = 0; i < BT; ++i)
    if (labels[i] != ignore_index) loss += lse[i] - target[i];
  *loss_out = n_valid > 0 ? loss / (double)n_valid : 0.0;
  if (!dZ) return OR_OK;

  /* Backward: the softmax rebuilt from the logits and lse (point b.). */
  scale = n_valid > 0 ? dloss / (double)n_valid : 0.0;
#pragma omp parallel for schedule(static)
  for (i = 0; i < BT; ++i) {
    int64_t j;
    const int valid = labels[i] != ignore_index;
    for (j = 0; j < V; ++j) {
      double g = 0.0;
      if (valid && n_valid > 0) {
        double z = widen_at(logits, dtype, i * ld + j);
        double t = capped ? tanh(z / softcap) : 0.0;
        double y = capped ? softcap * t : z;
        double d = capped ? 1.0 - t * t : 1.0;
        g = (exp(y - lse[i]) - (j == labels[i] ? 1.0 : 0.0)) * d * scale;
      }
      dZ[i * V + j] = g;
    }
  }
  return OR_OK;
}
