/*
 * Seeded synthetic inputs for the MoE dispatch / grouped-FFN / combine layer.
 *
 * This module only makes inputs. It holds none of the layer's arithmetic: no
 * plan, no pool, no expert FFN, no weighted sum. Both the CUDA path and the
 * CPU oracle read the arrays it writes, bit for bit.
 *
 * Generator (stated here so that it can be re-implemented from this text):
 *   key(seed, stream)  = SM(seed XOR (stream * 0xD1B54A32D192ED03))
 *   bits(seed,stream,i) = SM(key + (i + 1) * 0x9E3779B97F4A7C15)
 * where SM(z) is the SplitMix64 output function
 *   z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31.
 * so element i of a stream is the i-th SplitMix64 output of a generator seeded
 * with key, and any element can be drawn on its own (counter-based).
 *   uniform(i) = ((bits >> 11) + 0.5) * 2^-53, in the open interval (0, 1).
 *   normal(i)  = Box-Muller on the pair p = i / 2:
 *                r = sqrt(-2 ln u(2p)), a = 2 pi u(2p+1),
 *                r cos a for even i, r sin a for odd i  (double precision).
 * A bf16 value is the double rounded to float (nearest-even), then rounded to
 * bf16 on the bit pattern (nearest-even).
 *
 * Router inputs (the layer takes topk_idx / topk_weights as given):
 *   softmax top-k: fp32 logits (+ optional fp32 per-expert bias added before
 *   the softmax), softmax in double with the max subtracted, the k largest
 *   probabilities (ties: lower expert index first), renormalised over the k
 *   chosen, stored as fp32.
 *   Zipf(alpha): experts ranked by a seeded Fisher-Yates permutation; rank r
 *   (1-based) has mass r^-alpha. Each token draws k distinct experts in turn
 *   without replacement (inverse CDF over the remaining mass, one uniform per
 *   draw). Its weights are the softmax of k N(0,1) logits, stored as fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull
#define STREAM_MUL 0xD1B54A32D192ED03ull

static inline uint64_t sm_out(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return sm_out(seed ^ (stream * STREAM_MUL));
}

static inline uint64_t bits_at(uint64_t key, uint64_t i) {
  return sm_out(key + (i + 1) * GOLDEN);
}

static inline double unif_at(uint64_t key, uint64_t i) {
  return ((double)(bits_at(key, i) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static const double TWO_PI = 6.283185307179586476925286766559;

static inline void normal_pair(uint64_t key, uint64_t p, double *z0, double *z1) {
  double u1 = unif_at(key, 2 * p);
  double u2 = unif_at(key, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = TWO_PI * u2;
  *z0 = r * cos(a);
  *z1 = r * sin(a);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  double z0, z1;
  normal_pair(key, i >> 1, &z0, &z1);
  return (i & 1) ? z1 : z0;
}

static inline uint16_t bf16_from_float(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws: out[j] = bits(seed, stream, first + j). */
void gen_bits(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, uint64_t *out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = bits_at(key, first + (uint64_t)j);
}

/* Uniforms in (0,1): out[j] = uniform(seed, stream, first + j). */
void gen_uniform_f64(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double *out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = unif_at(key, first + (uint64_t)j);
}

/* sigma * N(0,1) in double: out[j] = sigma * normal(seed, stream, first + j). */
void gen_normal_f64(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double sigma,
                    double *out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = sigma * normal_at(key, first + (uint64_t)j);
}

/* sigma * N(0,1) rounded to fp32. */
void gen_normal_f32(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double sigma,
                    float *out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = (float)(sigma * normal_at(key, first + (uint64_t)j));
}

/* sigma * N(0,1) rounded to fp32, then to bf16 (bit patterns as uint16).
 * Element first + j of the stream lands in out[j]; pairs are drawn together. */
void gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double sigma,
                     uint16_t *out) {
  uint64_t key = stream_key(seed, stream);
  const int64_t chunk = 1 << 16;
  int64_t nchunks = (n + chunk - 1) / chunk;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t c = 0; c < nchunks; ++c) {
    int64_t j0 = c * chunk;
    int64_t j1 = j0 + chunk < n ? j0 + chunk : n;
    int64_t j = j0;
    /* odd leading element */
    if (j < j1 && ((first + (uint64_t)j) & 1)) {
      out[j] = bf16_from_float((float)(sigma * normal_at(key, first + (uint64_t)j)));
      ++j;
    }
    for (; j + 1 < j1; j += 2) {
      double z0, z1;
      normal_pair(key, (first + (uint64_t)j) >> 1, &z0, &z1);
      out[j] = bf16_from_float((float)(sigma * z0));
      out[j + 1] = bf16_from_float((float)(sigma * z1));
    }
    if (j < j1) out[j] = bf16_from_float((float)(sigma * normal_at(key, first + (uint64_t)j)));
  }
}

/* Softmax top-k router over fp32 logits [T, E] (+ optional fp32 bias [E]).
 * Writes topk_idx [T, k] (int32) and topk_w [T, k] (fp32). Returns 0, or -1 on bad sizes. */
int gen_router_softmax_topk(int64_t T, int E, int k, const float *logits, const float *bias,
                            int32_t *topk_idx, float *topk_w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  int err = 0;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    if (!p || !taken) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      if (!p || !taken) continue;
      const float *l = logits + t * (int64_t)E;
      double mx = -INFINITY;
      for (int e = 0; e < E; ++e) {
        float v = bias ? l[e] + bias[e] : l[e];
        p[e] = (double)v;
        if (p[e] > mx) mx = p[e];
      }
      double s = 0.0;
      for (int e = 0; e < E; ++e) {
        p[e] = exp(p[e] - mx);
        s += p[e];
      }
      for (int e = 0; e < E; ++e) p[e] /= s;
      memset(taken, 0, (size_t)E);
      double chosen_sum = 0.0;
      for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
          if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
        taken[best] = 1;
        topk_idx[t * k + j] = best;
        chosen_sum += p[best];
      }
      for (int j = 0; j < k; ++j)
        topk_w[t * k + j] = (float)(p[topk_idx[t * k + j]] / chosen_sum);
    }
    free(p);
    free(taken);
  }
  return err ? -1 : 0;
}

/* Zipf(alpha) routing over a seeded expert permutation, k distinct experts per token.
 * Token t uses global token index (t0 + t) for its draws, so a batch can be cut into
 * micro-batches that match one long draw. Streams: perm_stream (permutation),
 * draw_stream (expert draws), logit_stream (weight logits). */
int gen_router_zipf(int64_t T, int64_t t0, int E, int k, double alpha, uint64_t seed,
                    uint64_t perm_stream, uint64_t draw_stream, uint64_t logit_stream,
                    int32_t *topk_idx, float *topk_w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
  double *mass = (double *)malloc(sizeof(double) * (size_t)E);
  if (!perm || !mass) {
    free(perm);
    free(mass);
    return -1;
  }
  uint64_t pkey = stream_key(seed, perm_stream);
  for (int e = 0; e < E; ++e) perm[e] = e;
  for (int i = E - 1; i >= 1; --i) {
    int j = (int)(unif_at(pkey, (uint64_t)i) * (double)(i + 1));
    if (j > i) j = i;
    int32_t tmp = perm[i];
    perm[i] = perm[j];
    perm[j] = tmp;
  }
  for (int r = 0; r < E; ++r) mass[r] = pow((double)(r + 1), -alpha);
  uint64_t dkey = stream_key(seed, draw_stream);
  uint64_t lkey = stream_key(seed, logit_stream);
  int err = 0;
#pragma omp parallel
  {
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    if (!taken) {
#pragma omp atomic write
      err = 1;
    }
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      if (!taken) continue;
      uint64_t g = (uint64_t)(t0 + t);
      memset(taken, 0, (size_t)E);
      double lg[64];
      double mx = -INFINITY, s = 0.0;
      for (int j = 0; j < k; ++j) {
        double rem = 0.0;
        for (int r = 0; r < E; ++r)
          if (!taken[r]) rem += mass[r];
        double target = unif_at(dkey, g * (uint64_t)k + (uint64_t)j) * rem;
        int pick = -1;
        double cum = 0.0;
        for (int r = 0; r < E; ++r) {
          if (taken[r]) continue;
          pick = r;
          cum += mass[r];
          if (cum > target) break;
        }
        taken[pick] = 1;
        topk_idx[t * k + j] = perm[pick];
        if (j < 64) {
          lg[j] = normal_at(lkey, g * (uint64_t)k + (uint64_t)j);
          if (lg[j] > mx) mx = lg[j];
        }
      }
      if (k <= 64) {
        for (int j = 0; j < k; ++j) {
          lg[j] = exp(lg[j] - mx);
          s += lg[j];
        }
        for (int j = 0; j < k; ++j) topk_w[t * k + j] = (float)(lg[j] / s);
      }
    }
    free(taken);
  }
  free(perm);
  free(mass);
  return (err || k > 64) ? -1 : 0;
}
