// Router on the device: per token, the softmax over E experts of the fp32 scores
// logit + bias, the k largest (ties: lower expert index), renormalised over the k
// chosen (the topk_idx / topk_weights the StreamEP call takes as inputs). Because
// the softmax is monotonic and its denominator cancels in the renormalisation, the
// choice is made on the scores themselves and w_j = exp(v_j - m) / sum over the
// chosen exp(v_i - m), m = the largest score.
//
// One warp per token: lane l holds the scores of experts l, l+32, ...; each of the
// k rounds is a warp argmax (shuffle butterfly) over the experts not chosen yet.
// With a plan to fill (and k dividing 256), each block routes the tokens of exactly
// one 256-pair plan chunk and counts its pairs per expert in shared memory, so the
// plan's histogram launch is not needed (the plan's scan and rank launches follow).
#include <float.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// Route token t; lane j < k returns the j-th chosen expert in *e_out and its weight in
// *w_out (other lanes: -1, 0). kPer = scores held per lane (E <= 32 * kPer).
template <int kPer>
__device__ __forceinline__ void route_token(const float *__restrict__ row,
                                            const float *__restrict__ bias, int E, int k,
                                            int lane, int32_t *e_out, float *w_out) {
  float v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = -FLT_MAX;
    if (e < E) v[i] = bias ? row[e] + bias[e] : row[e];
  }
  uint32_t taken = 0;
  int32_t my_e = -1;
  float my_v = 0.0f, m = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bv = -FLT_MAX;
    int32_t be = INT32_MAX;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int32_t oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (j == 0) m = bv;
    if (lane == j) {
      my_e = be;
      my_v = bv;
    }
  }
  const float ex = lane < k ? expf(my_v - m) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  *e_out = my_e;
  *w_out = lane < k ? ex / sum : 0.0f;
}

template <int kPer>
__global__ void __launch_bounds__(256)
    route_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int32_t T,
                 int32_t E, int32_t k, int32_t *__restrict__ topk_idx,
                 float *__restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
       t += warps) {
    int32_t e;
    float w;
    route_token<kPer>(logits + t * E, bias, E, k, lane, &e, &w);
    if (lane < k) {
      topk_idx[t * k + lane] = e;
      topk_w[t * k + lane] = w;
    }
  }
}

// Routing fused with the plan's first launch: block = one 256-pair chunk, its 8 warps
// route the chunk's tokens in turn and count them in one shared histogram.
template <int kPer>
__global__ void __launch_bounds__(kPlanWarps * 32)
    route_hist_kernel(const float *__restrict__ logits, const float *__restrict__ bias,
                      int32_t T, int32_t E, int32_t k, int32_t *__restrict__ topk_idx,
                      float *__restrict__ topk_w, int32_t n_chunks, int32_t *__restrict__ ws,
                      int32_t *__restrict__ done_counter, const PlanResets resets) {
  extern __shared__ int32_t hist[];  // [E] for this block's chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int chunk = blockIdx.x;
  if (chunk < n_chunks) {
    const int per = kPlanChunk / k;  // tokens per chunk
    const int64_t t0 = (int64_t)chunk * per;
    for (int i = warp; i < per; i += kPlanWarps) {
      const int64_t t = t0 + i;
      if (t >= T) break;
      int32_t e;
      float w;
      route_token<kPer>(logits + t * E, bias, E, k, lane, &e, &w);
      if (lane < k) {
        topk_idx[t * k + lane] = e;
        topk_w[t * k + lane] = w;
        atomicAdd(&hist[e], 1);
      }
    }
  }
  __syncthreads();
  if (chunk < n_chunks)
    for (int e = threadIdx.x; e < E; e += blockDim.x) ws[(int64_t)e * n_chunks + chunk] = hist[e];
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t gsz = (int64_t)gridDim.x * blockDim.x;
  if (gtid == 0) *done_counter = 0;
  plan_reset_slice(resets, gtid, gsz);
}

template <int kPer>
static cudaError_t launch_route_t(const moe_shape &s, const float *logits, const float *bias,
                                  int32_t *topk_idx, float *topk_w, const moe_plan_buffers *p,
                                  int num_sms, cudaStream_t st) {
  if (p == nullptr || (kPlanChunk % s.k) != 0) {
    if (s.T > 0) {
      const int64_t blocks = ((int64_t)s.T + 7) / 8;
      const int grid = (int)(blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8);
      route_kernel<kPer><<<grid, 256, 0, st>>>(logits, bias, s.T, s.E, s.k, topk_idx, topk_w);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess || p == nullptr) return e;
    }
    return launch_plan(s, topk_idx, *p, st);
  }
  const PlanGeom g = plan_geom(s);
  const size_t smem = sizeof(int32_t) * (size_t)s.E;
  int32_t *done = p->workspace + (size_t)s.E * (size_t)(g.n_chunks > 0 ? g.n_chunks : 1);
  const int nblk = g.n_chunks > 0 ? g.n_chunks : 1;
  route_hist_kernel<kPer><<<nblk, kPlanWarps * 32, smem, st>>>(
      logits, bias, s.T, s.E, s.k, topk_idx, topk_w, g.n_chunks, p->workspace, done,
      plan_resets(s, *p));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_plan_scan_rank(s, topk_idx, *p, st);
}

cudaError_t launch_route(const moe_shape &s, const float *logits, const float *bias,
                         int32_t *topk_idx, float *topk_w, const moe_plan_buffers *p,
                         int num_sms, cudaStream_t st) {
  const int per = (s.E + 31) / 32;
  if (per <= 1) return launch_route_t<1>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
  if (per <= 2) return launch_route_t<2>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
  if (per <= 4) return launch_route_t<4>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
  if (per <= 8) return launch_route_t<8>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
  if (per <= 16) return launch_route_t<16>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
  return launch_route_t<32>(s, logits, bias, topk_idx, topk_w, p, num_sms, st);
}

}  // namespace moe
