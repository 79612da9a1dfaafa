/*
 * CPU oracle for the MoE layer's plan -> dispatch -> grouped SwiGLU FFN -> combine.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the package's smoke check and the CPU
 * baseline leg of the benchmark call this file; the product path never does,
 * and it shares no code, header, table or helper with the CUDA library.
 *
 * It is plain and slow on purpose: integer work is written as its definition,
 * floating point is computed in double from the bf16 / fp32 inputs with no
 * intermediate rounding, and nothing is blocked, fused or reordered beyond what
 * each definition states (sums run over their index in ascending order).
 *
 * Source of each definition: the StreamEP README ("How it works"):
 *   - "Pool-layout dispatch": routed (token, k) pairs land in an expert-major,
 *     tile-padded pool, so dispatch's output is the grouped GEMM input.
 *     -> oracle_plan, oracle_pool
 *   - "CuTeDSL compute kernels": forward grouped GEMMs A (up/gate) and Y (down)
 *     over the pool; the expert function is the SwiGLU FFN
 *     W2 (silu(x W1_gate) * (x W1_up)).
 *     -> oracle_expert_ffn, oracle_moe_forward
 *   - "Per-tile streaming" / combine: each token's output is the routing-weighted
 *     sum of its k expert outputs. -> oracle_combine, oracle_moe_forward
 *   - the backward grouped GEMMs A / Y and the backward pass mirroring dispatch and
 *     combine: gradients of the layer with respect to x and the routing weights.
 *     -> oracle_moe_backward; the weight gradients of one expert.
 *     -> oracle_expert_weight_grads
 * Readings where the README is silent (each one also listed in the design notes):
 *   - order inside an expert's pool segment: flat pair id f = t*k + j ascending;
 *   - W1[e] is [H, 2I]: columns [0, I) gate, [I, 2I) up (concatenated);
 *   - padding rows of the pool are all-zero;
 *   - topk_idx == -1 marks a dropped pair (no pool row, no contribution);
 *     any other index outside [0, E) is an error;
 *   - silu(v) = v / (1 + exp(-v));
 *   - the router's choice (oracle_route) is taken on the fp32 scores logit + bias
 *     (one fp32 addition), the precision the GPU decides in; ties go to the lower
 *     expert index; the renormalised weights are computed in double.
 *
 * Pins (tests/test_oracle_pins.py): a hand-worked example, a stable-sort brute
 * force of the plan, invariants, a dense all-experts brute force of the layer,
 * the E=1/k=1 textbook SwiGLU FFN against torch float64 matmuls, closed forms
 * (identity-like W1/W2, identity experts), linearity and permutation
 * equivariance; for the backward, central differences of oracle_moe_forward and
 * torch float64 autograd on the dense E=1 layer; plus planted-mistake variants of
 * this file that must fail them.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_MISSING_EXPERT (-2)
#define ORACLE_ERR_BAD_INDEX (-10)

/* bf16 bit pattern -> double. Exact: bf16 is the top half of an fp32. */
static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

/* Dropless bound on the pool rows: every real pair, plus at most tile-1 padding
 * rows for each expert that receives at least one pair. */
int64_t oracle_pool_rows_max(int64_t T, int32_t k, int32_t E, int32_t tile) {
  int64_t pairs = T * (int64_t)k;
  int64_t nonempty = pairs < (int64_t)E ? pairs : (int64_t)E;
  return round_up(pairs + nonempty * (int64_t)(tile - 1), tile);
}

/*
 * Routing plan (StreamEP README, How it works, "Pool-layout dispatch").
 *   counts[e]      = #{ f : topk_idx[f] == e }
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + ceil(counts[e]/tile)*tile
 *   P              = offsets[E]
 *   pool_row[f]    = offsets[e] + (number of f' < f with topk_idx[f'] == e),
 *                    or -1 for a dropped pair (topk_idx[f] == -1)
 *   row_src[p]     = the f with pool_row[f] == p, or -1 for a padding row
 *                    (rows [P, row_src_len) are -1 as well)
 *   tile_expert[i] = e for the pool tile i = p / tile of rows p in
 *                    [offsets[e], offsets[e+1]); -1 for tiles at or past P/tile
 * Returns ORACLE_ERR_BAD_INDEX if any index is outside [-1, E).
 */
int oracle_plan(int64_t T, int32_t k, int32_t E, int32_t tile, const int32_t *topk_idx,
                int32_t *counts, int32_t *offsets, int32_t *pool_row, int32_t *row_src,
                int64_t row_src_len, int32_t *tile_expert, int64_t tile_expert_len,
                int64_t *P_out) {
  if (T < 0 || k <= 0 || E <= 0 || tile <= 0) return ORACLE_ERR_ARG;
  int64_t pairs = T * (int64_t)k;
  for (int64_t f = 0; f < pairs; ++f) {
    int32_t e = topk_idx[f];
    if (e < -1 || e >= E) return ORACLE_ERR_BAD_INDEX;
  }
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t f = 0; f < pairs; ++f)
    if (topk_idx[f] >= 0) counts[topk_idx[f]] += 1;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e)
    offsets[e + 1] = offsets[e] + (int32_t)round_up(counts[e], tile);
  int64_t P = offsets[E];
  if (P > row_src_len || P / tile > tile_expert_len) return ORACLE_ERR_ARG;

  for (int64_t p = 0; p < row_src_len; ++p) row_src[p] = -1;
  int32_t *seen = (int32_t *)calloc((size_t)E, sizeof(int32_t));
  if (!seen) return ORACLE_ERR_ARG;
  for (int64_t f = 0; f < pairs; ++f) {
    int32_t e = topk_idx[f];
    if (e < 0) {
      pool_row[f] = -1;
      continue;
    }
    int32_t p = offsets[e] + seen[e];
    seen[e] += 1;
    pool_row[f] = p;
    row_src[p] = (int32_t)f;
  }
  free(seen);
  for (int64_t i = 0; i < tile_expert_len; ++i) tile_expert[i] = -1;
  for (int32_t e = 0; e < E; ++e)
    for (int64_t p = offsets[e]; p < offsets[e + 1]; p += tile) tile_expert[p / tile] = e;
  *P_out = P;
  return ORACLE_OK;
}

/*
 * Dispatched pool (StreamEP README, How it works, "Pool-layout dispatch"):
 * row p holds x[row_src[p] / k] for a real row and zeros for a padding row.
 * Bit copy of the bf16 patterns.
 */
void oracle_pool(int64_t P, int32_t H, int32_t k, const int32_t *row_src, const uint16_t *x,
                 uint16_t *pool) {
  for (int64_t p = 0; p < P; ++p) {
    int32_t f = row_src[p];
    for (int32_t h = 0; h < H; ++h)
      pool[p * H + h] = (f >= 0) ? x[(int64_t)(f / k) * H + h] : (uint16_t)0;
  }
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

/*
 * One expert applied to one token row (StreamEP README, How it works,
 * "CuTeDSL compute kernels": GEMM A then GEMM Y), in double:
 *   g[n] = sum_h x[h] * W1e[h][n]          n in [0, I)   (gate)
 *   u[n] = sum_h x[h] * W1e[h][I + n]                     (up)
 *   a[n] = silu(g[n]) * u[n]
 *   z[m] = sum_n a[n] * W2e[n][m]          m in [0, H)
 * W1e is [H, 2I] row-major, W2e is [I, H] row-major. Scratch: g, u, a of I doubles.
 */
void oracle_expert_ffn(int32_t H, int32_t I, const uint16_t *x_row, const uint16_t *W1e,
                       const uint16_t *W2e, double *g, double *u, double *a, double *z) {
  const int64_t two_i = 2 * (int64_t)I;
  for (int32_t n = 0; n < I; ++n) {
    g[n] = 0.0;
    u[n] = 0.0;
  }
  /* h outer so that W1e streams row by row; each g[n], u[n] still sums h ascending. */
  for (int32_t h = 0; h < H; ++h) {
    double xh = bf16_to_double(x_row[h]);
    const uint16_t *w = W1e + (int64_t)h * two_i;
    for (int32_t n = 0; n < I; ++n) {
      g[n] += xh * bf16_to_double(w[n]);
      u[n] += xh * bf16_to_double(w[I + n]);
    }
  }
  for (int32_t n = 0; n < I; ++n) a[n] = silu(g[n]) * u[n];
  for (int32_t m = 0; m < H; ++m) z[m] = 0.0;
  /* n outer: each z[m] sums n ascending. */
  for (int32_t n = 0; n < I; ++n) {
    const uint16_t *w = W2e + (int64_t)n * H;
    for (int32_t m = 0; m < H; ++m) z[m] += a[n] * bf16_to_double(w[m]);
  }
}

/*
 * The layer for a list of tokens, straight from x (never through a pool):
 *   y[t][m] = sum_{j < k, e = topk_idx[t][j] >= 0} w[t][j] * z_{t,j}[m]
 * with z_{t,j} = oracle_expert_ffn(x[t], W1[e], W2[e]); j ascending.
 * x_rows [n, H] bf16, idx_rows / w_rows [n, k], W1 / W2: E pointers to one
 * expert's matrix each (NULL allowed for experts no listed token uses).
 * y [n, H] double. Tokens are independent and run on up to n_threads threads.
 */
int oracle_moe_forward(int64_t n, int32_t H, int32_t I, int32_t E, int32_t k,
                       const uint16_t *x_rows, const int32_t *idx_rows, const float *w_rows,
                       const uint16_t *const *W1, const uint16_t *const *W2, double *y,
                       int n_threads) {
  if (n < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return ORACLE_ERR_ARG;
  for (int64_t f = 0; f < n * k; ++f) {
    int32_t e = idx_rows[f];
    if (e < -1 || e >= E) return ORACLE_ERR_BAD_INDEX;
    if (e >= 0 && (!W1[e] || !W2[e])) return ORACLE_ERR_MISSING_EXPERT;
  }
  int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    double *z = (double *)malloc(sizeof(double) * (size_t)H);
    if (!g || !u || !a || !z) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
      if (!g || !u || !a || !z) continue;
      double *yt = y + t * H;
      for (int32_t m = 0; m < H; ++m) yt[m] = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int32_t e = idx_rows[t * k + j];
        if (e < 0) continue;
        double w = (double)w_rows[t * k + j];
        oracle_expert_ffn(H, I, x_rows + t * H, W1[e], W2[e], g, u, a, z);
        for (int32_t m = 0; m < H; ++m) yt[m] += w * z[m];
      }
    }
    free(g);
    free(u);
    free(a);
    free(z);
  }
  return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/*
 * Backward of the layer for a list of tokens (StreamEP README, How it works: the
 * backward grouped GEMMs A and Y of "CuTeDSL compute kernels", and the backward pass
 * that mirrors dispatch and combine, "Per-tile streaming"), in double. Given dy [n, H],
 * the gradient of a loss with respect to the layer output y, and the forward values
 * g, u, a, z of pair (t, j) with expert e (oracle_expert_ffn):
 *   dw[t][j] = sum_m dy[t][m] * z[m]                            (routing weight)
 *   dz[m]    = w[t][j] * dy[t][m]                               (combine, mirrored)
 *   da[n]    = sum_m W2e[n][m] * dz[m]                          (backward Y)
 *   dg[n]    = da[n] * u[n] * silu'(g[n]),   du[n] = da[n] * silu(g[n])
 *   dx[t][h] = sum over the token's pairs of
 *              sum_n W1e[h][n] * dg[n] + W1e[h][I + n] * du[n]  (backward A; dispatch,
 *                                                                mirrored, sums the pairs)
 * with silu'(v) = s (1 + v (1 - s)), s = 1 / (1 + exp(-v)). Sums run over their index in
 * ascending order, pairs in j order. Dropped pairs (index -1) contribute nothing and get
 * dw = 0. dx [n, H] and dw [n, k] are double.
 */
static double silu_grad(double v) {
  double s = 1.0 / (1.0 + exp(-v));
  return s * (1.0 + v * (1.0 - s));
}

int oracle_moe_backward(int64_t n, int32_t H, int32_t I, int32_t E, int32_t k,
                        const uint16_t *x_rows, const int32_t *idx_rows, const float *w_rows,
                        const uint16_t *const *W1, const uint16_t *const *W2,
                        const uint16_t *dy_rows, double *dx, double *dw, int n_threads) {
  if (n < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return ORACLE_ERR_ARG;
  for (int64_t f = 0; f < n * k; ++f) {
    int32_t e = idx_rows[f];
    if (e < -1 || e >= E) return ORACLE_ERR_BAD_INDEX;
    if (e >= 0 && (!W1[e] || !W2[e])) return ORACLE_ERR_MISSING_EXPERT;
  }
  int err = 0;
  const int64_t two_i = 2 * (int64_t)I;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
  {
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    double *z = (double *)malloc(sizeof(double) * (size_t)H);
    double *dz = (double *)malloc(sizeof(double) * (size_t)H);
    double *dg = (double *)malloc(sizeof(double) * (size_t)I);
    double *du = (double *)malloc(sizeof(double) * (size_t)I);
    if (!g || !u || !a || !z || !dz || !dg || !du) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < n; ++t) {
      if (!g || !u || !a || !z || !dz || !dg || !du) continue;
      double *dxt = dx + t * H;
      for (int32_t h = 0; h < H; ++h) dxt[h] = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int32_t e = idx_rows[t * k + j];
        dw[t * k + j] = 0.0;
        if (e < 0) continue;
        oracle_expert_ffn(H, I, x_rows + t * H, W1[e], W2[e], g, u, a, z);
        const double w = (double)w_rows[t * k + j];
        double s = 0.0;
        for (int32_t m = 0; m < H; ++m) {
          const double dym = bf16_to_double(dy_rows[t * H + m]);
          s += dym * z[m];
          dz[m] = w * dym;
        }
        dw[t * k + j] = s;
        for (int32_t q = 0; q < I; ++q) {
          const uint16_t *w2 = W2[e] + (int64_t)q * H;
          double da = 0.0;
          for (int32_t m = 0; m < H; ++m) da += bf16_to_double(w2[m]) * dz[m];
          dg[q] = da * u[q] * silu_grad(g[q]);
          du[q] = da * silu(g[q]);
        }
        for (int32_t h = 0; h < H; ++h) {
          const uint16_t *w1 = W1[e] + (int64_t)h * two_i;
          double acc = 0.0;
          for (int32_t q = 0; q < I; ++q)
            acc += bf16_to_double(w1[q]) * dg[q] + bf16_to_double(w1[I + q]) * du[q];
          dxt[h] += acc;
        }
      }
    }
    free(g);
    free(u);
    free(a);
    free(z);
    free(dz);
    free(dg);
    free(du);
  }
  return err ? ORACLE_ERR_ARG : ORACLE_OK;
}

/*
 * Weight gradients of one expert e (the backward's weight GEMMs), in double, from the same
 * per-pair values as oracle_moe_backward:
 *   dW1[h][n]     = sum over the pairs (t, j) with topk_idx[t][j] == e of x[t][h] * dg[n]
 *   dW1[h][I + n] = the same sum of x[t][h] * du[n]
 *   dW2[n][m]     = the same sum of a[n] * dz[m],   dz = w[t][j] * dy[t]
 * pairs in flat-pair order t*k + j ascending. dW1 [H, 2I] and dW2 [I, H] are double.
 */
int oracle_expert_weight_grads(int64_t T, int32_t H, int32_t I, int32_t E, int32_t k,
                               const uint16_t *x, const int32_t *topk_idx, const float *topk_w,
                               const uint16_t *W1e, const uint16_t *W2e, int32_t e,
                               const uint16_t *dy, double *dW1, double *dW2) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || e < 0 || e >= E) return ORACLE_ERR_ARG;
  const int64_t two_i = 2 * (int64_t)I;
  double *g = (double *)malloc(sizeof(double) * (size_t)I);
  double *u = (double *)malloc(sizeof(double) * (size_t)I);
  double *a = (double *)malloc(sizeof(double) * (size_t)I);
  double *z = (double *)malloc(sizeof(double) * (size_t)H);
  double *dz = (double *)malloc(sizeof(double) * (size_t)H);
  double *dg = (double *)malloc(sizeof(double) * (size_t)I);
  double *du = (double *)malloc(sizeof(double) * (size_t)I);
  int rc = ORACLE_OK;
  if (!g || !u || !a || !z || !dz || !dg || !du) rc = ORACLE_ERR_ARG;
  for (int64_t i = 0; rc == ORACLE_OK && i < (int64_t)H * two_i; ++i) dW1[i] = 0.0;
  for (int64_t i = 0; rc == ORACLE_OK && i < (int64_t)I * H; ++i) dW2[i] = 0.0;
  for (int64_t f = 0; rc == ORACLE_OK && f < T * k; ++f) {
    if (topk_idx[f] < -1 || topk_idx[f] >= E) {
      rc = ORACLE_ERR_BAD_INDEX;
      break;
    }
    if (topk_idx[f] != e) continue;
    const int64_t t = f / k;
    oracle_expert_ffn(H, I, x + t * H, W1e, W2e, g, u, a, z);
    const double w = (double)topk_w[f];
    for (int32_t m = 0; m < H; ++m) dz[m] = w * bf16_to_double(dy[t * H + m]);
    for (int32_t q = 0; q < I; ++q) {
      const uint16_t *w2 = W2e + (int64_t)q * H;
      double da = 0.0;
      for (int32_t m = 0; m < H; ++m) da += bf16_to_double(w2[m]) * dz[m];
      dg[q] = da * u[q] * silu_grad(g[q]);
      du[q] = da * silu(g[q]);
    }
    for (int32_t h = 0; h < H; ++h) {
      const double xh = bf16_to_double(x[t * H + h]);
      double *row = dW1 + (int64_t)h * two_i;
      for (int32_t q = 0; q < I; ++q) {
        row[q] += xh * dg[q];
        row[I + q] += xh * du[q];
      }
    }
    for (int32_t q = 0; q < I; ++q) {
      double *row = dW2 + (int64_t)q * H;
      for (int32_t m = 0; m < H; ++m) row[m] += a[q] * dz[m];
    }
  }
  free(g);
  free(u);
  free(a);
  free(z);
  free(dz);
  free(dg);
  free(du);
  return rc;
}

/*
 * The layer with identity experts (the expert returns its input row):
 *   y[t][m] = sum_{j < k, topk_idx[t][j] >= 0} w[t][j] * x[t][m]
 */
int oracle_moe_forward_identity(int64_t T, int32_t H, int32_t k, const uint16_t *x,
                                const int32_t *topk_idx, const float *topk_w, double *y) {
  if (T < 0 || H <= 0 || k <= 0) return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t m = 0; m < H; ++m) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j)
        if (topk_idx[t * k + j] >= 0)
          acc += (double)topk_w[t * k + j] * bf16_to_double(x[t * H + m]);
      y[t * H + m] = acc;
    }
  }
  return ORACLE_OK;
}

/*
 * Combine over a given expert-output pool (StreamEP README, How it works,
 * "Per-tile streaming": combine sends each token once its compute is done):
 *   y[t][m] = sum_{j < k, pool_row[t*k+j] >= 0} w[t][j] * ypool[pool_row[t*k+j]][m]
 * ypool [*, H] bf16; y [T, H] double.
 */
int oracle_combine(int64_t T, int32_t H, int32_t k, const int32_t *pool_row,
                   const float *topk_w, const uint16_t *ypool, double *y) {
  if (T < 0 || H <= 0 || k <= 0) return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < T; ++t) {
    for (int32_t m = 0; m < H; ++m) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        int32_t p = pool_row[t * k + j];
        if (p < 0) continue;
        acc += (double)topk_w[t * k + j] * bf16_to_double(ypool[(int64_t)p * H + m]);
      }
      y[t * H + m] = acc;
    }
  }
  return ORACLE_OK;
}

/*
 * Router (the inputs of the StreamEP call: topk_idx / topk_weights from the gate's
 * softmax; "softmax top-k, renormalised"), per token t over E experts:
 *   v_e   = logits[t][e] + bias[e]            (fp32; bias may be NULL)
 *   chosen = the k largest v_e, largest first, equal v_e: lower e first
 *   w_j   = p_j / sum_{chosen i} p_i with p = softmax(v) over all E experts,
 *           which equals exp(v_j - m) / sum_{chosen i} exp(v_i - m), m = max_e v_e
 * idx [T, k] int32, w [T, k] double.
 */
int oracle_route(int64_t T, int32_t E, int32_t k, const float *logits, const float *bias,
                 int32_t *idx, double *w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return ORACLE_ERR_ARG;
  float *v = (float *)malloc(sizeof(float) * (size_t)E);
  unsigned char *taken = (unsigned char *)malloc((size_t)E);
  if (!v || !taken) {
    free(v);
    free(taken);
    return ORACLE_ERR_ARG;
  }
  for (int64_t t = 0; t < T; ++t) {
    float m = -INFINITY;
    for (int32_t e = 0; e < E; ++e) {
      v[e] = bias ? logits[t * E + e] + bias[e] : logits[t * E + e];
      taken[e] = 0;
      if (v[e] > m) m = v[e];
    }
    double sum = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || v[e] > v[best])) best = e;
      taken[best] = 1;
      idx[t * k + j] = best;
      w[t * k + j] = exp((double)v[best] - (double)m);
      sum += w[t * k + j];
    }
    for (int32_t j = 0; j < k; ++j) w[t * k + j] /= sum;
  }
  free(v);
  free(taken);
  return ORACLE_OK;
}
