/*
 * CPU ORACLE for the predictor-gated sparse FFN decode step.
 *
 * TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
 * baseline leg load this library; the product path never does.  It shares
 * no code with the CUDA path.  Plain loops, double accumulation, every step
 * in the order the method states it; OpenMP only over independent outputs,
 * so results do not depend on the thread count.
 *
 * What the pages fix (PowerInfer write-ups):
 *  - a small per-layer predictor decides, before the FFN runs, which
 *    neurons the input activates; only those neurons are computed
 *    (QbitAI article, r-manual.ru, §"Что такое «разреженная активация»?"
 *    and §"Гибридный дизайн вывода CPU/GPU");
 *  - neurons are split into a frequently active ("hot") group and an
 *    input-dependent ("cold") group, and the partial results of the two
 *    groups are summed (same article, §"Гибридный дизайн вывода CPU/GPU",
 *    the neurons 3, 4, 5 example; aibars.net "SJTU-IPADS/PowerInfer"
 *    §"Mecanismo de Neurônios Quentes e Frios");
 *  - activations are ReLU / ReGLU / squared ReLU (hada.io summary,
 *    §"Hạn chế và FAQ");
 *  - weights may be INT4 Q4_0 (hada.io summary, §"Lượng tử hóa và tương
 *    thích").
 * Readings where the pages are silent (predictor = two bias-free linear
 * maps d->r->d_ff plus an output bias, thresholded through a sigmoid;
 * pre-norm residual stack; bias placement; Q4_0 nibble order) are stated
 * at each function.
 *
 * Parity pins: every function here is pinned by tests that do not reuse it
 * (hand-computed values, float64 library routines, invariants, brute force).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_Q4_0 = 2 };
enum { OR_RELU = 0, OR_REGLU = 1, OR_RELU2 = 2 };

typedef struct {
  int32_t d, F, r, H, act, wdt, pdt;
  const void *wg, *wu, *wd;      /* [F][d] neuron-major; wg unused for ReLU    */
  const uint16_t *sg, *su, *sd;  /* Q4_0 block scales [F][d/32], binary16     */
  const float* bias;             /* [F] on W_gate (ReGLU) or W_up (ReLU); NULL */
  const void *p1, *p2;           /* [r][d], [F][r] in pdt (F32 or F16)        */
  const float* pbias;            /* [F] predictor output bias; NULL = 0        */
} or_layer;

int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the parallel loops below use from now on (results do not depend
 * on it: every output is summed in the same order whatever the count). */
void or_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* IEEE 754 binary16 -> double, from the format's definition: sign, 5-bit
 * exponent with bias 15, 10-bit fraction; exponent 0 = subnormal. */
double or_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp(1.0 + (double)f / 1024.0, e - 15);
  return sign ? -v : v;
}

/* Q4_0 (hada.io summary §"Lượng tử hóa và tương thích": INT4 Q4_0): blocks
 * of 32 consecutive weights of a row share one binary16 scale s; each weight
 * is a 4-bit code q and decodes to (q - 8) * s.  Layout of a row: d/32
 * blocks of 16 bytes; byte k of a block holds element k in its low nibble
 * and element k + 16 in its high nibble. */
double or_q4_0_weight(const uint8_t* qs, const uint16_t* scales, int d, long row, int col) {
  long blk = row * (long)(d / 32) + col / 32;
  int k = col % 32;
  uint8_t byte = qs[blk * 16 + (k % 16)];
  int q = (k < 16) ? (byte & 0x0F) : (byte >> 4);
  return (double)(q - 8) * or_half_to_double(scales[blk]);
}

/* Weight (row, col) of a [rows][cols] matrix stored in dtype dt. */
static double weight(int dt, const void* w, const uint16_t* s, int cols, long row, int col) {
  switch (dt) {
    case OR_F32: return (double)((const float*)w)[row * (long)cols + col];
    case OR_F16: return or_half_to_double(((const uint16_t*)w)[row * (long)cols + col]);
    default:     return or_q4_0_weight((const uint8_t*)w, s, cols, row, col);
  }
}

void or_decode_row(int dt, const void* w, const uint16_t* s, int cols, long row, double* out) {
  for (int c = 0; c < cols; ++c) out[c] = weight(dt, w, s, cols, row, c);
}

/* Pre-norm of the residual stream (a reading: the pages do not describe
 * how FFN layers chain): xh = x / sqrt(mean(x^2) + 1e-6), no learned gain. */
void or_rmsnorm(const float* x, int d, double* xh) {
  double ss = 0.0;
  for (int i = 0; i < d; ++i) ss += (double)x[i] * (double)x[i];
  double inv = 1.0 / sqrt(ss / d + 1e-6);
  for (int i = 0; i < d; ++i) xh[i] = (double)x[i] * inv;
}

/* The activation predictor (QbitAI article §"Что такое «разреженная
 * активация»?": a small model per layer, run on the layer's input, predicts
 * which neurons the input activates).  Reading: u = P1 xh (length r),
 * z_j = P2[j] . u + c_j, and neuron j is predicted active when
 * sigmoid(z_j) > tau, i.e. z_j > logit(tau).  Only cold neurons j >= H are
 * evaluated; z[j] for j < H is left as +INFINITY (hot neurons always run). */
void or_predict(const or_layer* L, const double* xh, double* u, double* z) {
  int d = L->d, r = L->r, F = L->F;
#pragma omp parallel for schedule(static)
  for (int k = 0; k < r; ++k) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += weight(L->pdt, L->p1, NULL, d, k, i) * xh[i];
    u[k] = acc;
  }
#pragma omp parallel for schedule(static)
  for (int j = 0; j < F; ++j) {
    if (j < L->H) { z[j] = INFINITY; continue; }
    double acc = 0.0;
    for (int k = 0; k < r; ++k) acc += weight(L->pdt, L->p2, NULL, r, j, k) * u[k];
    z[j] = acc + (L->pbias ? (double)L->pbias[j] : 0.0);
  }
}

/* Predicted mask: bit j (word j/32, bit j%32) set when neuron j runs: every
 * hot neuron j < H, and every cold neuron with z_j > theta (strict). */
void or_mask(const double* z, int F, int H, double theta, uint32_t* mask) {
  int words = (F + 31) / 32;
  memset(mask, 0, sizeof(uint32_t) * (size_t)words);
  for (int j = 0; j < F; ++j)
    if (j < H || z[j] > theta) mask[j / 32] |= 1u << (j % 32);
}

/* Compaction: the ascending list of neurons j in [begin, F) whose bit is set
 * in the OR of `nmask` masks (one mask = one token; nmask > 1 is the union
 * over a batch).  Returns the count. */
int or_compact(const uint32_t* masks, int nmask, int F, int begin, int32_t* idx) {
  int words = (F + 31) / 32, n = 0;
  for (int j = begin < 0 ? 0 : begin; j < F; ++j) {
    uint32_t w = 0;
    for (int t = 0; t < nmask; ++t) w |= masks[(long)t * words + j / 32];
    if ((w >> (j % 32)) & 1u) idx[n++] = j;
  }
  return n;
}

/* The FFN restricted to a neuron set S (rowset[j] != 0), computing only the
 * neurons in S (QbitAI article §"Что такое «разреженная активация»?":
 * only the activated neurons are computed; the hot/cold sum of
 * §"Гибридный дизайн вывода CPU/GPU" is the sum over S in ascending order):
 *   ReLU : h_j = max(0, W_up[j] . xh + b_j)
 *   ReGLU: h_j = max(0, W_gate[j] . xh + b_j) * (W_up[j] . xh)
 *   squared ReLU (hada.io summary §"Hạn chế và FAQ" names the activation;
 *   reading: applied where ReLU is, no gate): h_j = max(0, W_up[j] . xh + b_j)^2
 *   y_i  = sum over j in S, ascending, of h_j * W_down^T[j][i]
 * h_j = 0 for j not in S.  With S = all neurons this is the dense FFN. */
void or_ffn(const or_layer* L, const double* xh, const uint8_t* rowset, double* h, double* y) {
  int d = L->d, F = L->F;
#pragma omp parallel for schedule(dynamic, 16)
  for (int j = 0; j < F; ++j) {
    h[j] = 0.0;
    if (!rowset[j]) continue;
    double b = L->bias ? (double)L->bias[j] : 0.0;
    if (L->act != OR_REGLU) {
      double g = 0.0;
      for (int i = 0; i < d; ++i) g += weight(L->wdt, L->wu, L->su, d, j, i) * xh[i];
      g += b;
      h[j] = g > 0.0 ? g : 0.0;
      if (L->act == OR_RELU2) h[j] = h[j] * h[j];
    } else {
      double g = 0.0, u = 0.0;
      for (int i = 0; i < d; ++i) g += weight(L->wdt, L->wg, L->sg, d, j, i) * xh[i];
      for (int i = 0; i < d; ++i) u += weight(L->wdt, L->wu, L->su, d, j, i) * xh[i];
      g += b;
      h[j] = (g > 0.0 ? g : 0.0) * u;
    }
  }
  /* down projection: each thread owns a range of output columns and walks
   * the neurons in ascending order, so every y_i has the same order. */
  int nthr = or_num_threads();
  int chunk = (d + nthr - 1) / nthr;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < nthr; ++t) {
    int i0 = t * chunk, i1 = i0 + chunk < d ? i0 + chunk : d;
    for (int i = i0; i < i1; ++i) y[i] = 0.0;
    for (int j = 0; j < F; ++j) {
      if (!rowset[j]) continue;
      double hj = h[j];
      for (int i = i0; i < i1; ++i) y[i] += hj * weight(L->wdt, L->wd, L->sd, d, j, i);
    }
  }
}

/* Neuron set of one token from its list and the hot prefix: S = [0,H) U idx. */
void or_rowset(int F, int H, const int32_t* idx, int n, uint8_t* rowset) {
  memset(rowset, 0, (size_t)F);
  for (int j = 0; j < H && j < F; ++j) rowset[j] = 1;
  for (int t = 0; t < n; ++t) rowset[idx[t]] = 1;
}

/* One decode layer of the stack for one token (reading: pre-norm residual
 * block x <- x + FFN_S(rmsnorm(x)), S = [0,H) U predicted cold neurons).
 * x (fp32 in) is updated in double into x_out; mask receives the predicted
 * mask, z the predictor logits. */
void or_layer_forward(const or_layer* L, const float* x, double theta, double* x_out,
                      uint32_t* mask, double* z) {
  int d = L->d, F = L->F;
  double* xh = (double*)malloc(sizeof(double) * (size_t)d);
  double* u = (double*)malloc(sizeof(double) * (size_t)L->r);
  double* h = (double*)malloc(sizeof(double) * (size_t)F);
  double* y = (double*)malloc(sizeof(double) * (size_t)d);
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)F);
  uint8_t* rs = (uint8_t*)malloc((size_t)F);
  or_rmsnorm(x, d, xh);
  or_predict(L, xh, u, z);
  or_mask(z, F, L->H, theta, mask);
  int n = or_compact(mask, 1, F, L->H, idx);
  or_rowset(F, L->H, idx, n, rs);
  or_ffn(L, xh, rs, h, y);
  for (int i = 0; i < d; ++i) x_out[i] = (double)x[i] + y[i];
  free(xh); free(u); free(h); free(y); free(idx); free(rs);
}
