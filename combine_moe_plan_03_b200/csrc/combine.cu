// Combine (StreamEP README, How it works, "Per-tile streaming": combine handles
// a token once its expert outputs exist): out[t] = bf16(sum_j w[t,j] * ypool[row]),
// the routing weight fused here as an fp32 fused multiply-add chain over j
// ascending, rounded once to bf16 (nearest-even). Dropped pairs add nothing.
// With topk_w == nullptr every weight is 1: the backward of dispatch, which sums
// the gradients of a token's k pool rows.
//
// One block of 128 threads per token (grid-stride): the k row ids and weights go
// to shared memory, then each thread gathers 16-byte vectors of the k rows (all
// k loads issued before the FMAs) and writes one 16-byte vector of out.
// HBM traffic per call: live pairs*H*2 read + T*H*2 written (+ T*k*8 for ids/weights).
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kCombThreads = 128;
constexpr int kCombGroup = 8;  // rows gathered before their FMAs

__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], float w, const uint4 &v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(u[i] << 16);
    const float hi = __uint_as_float(u[i] & 0xFFFF0000u);
    acc[2 * i] = fmaf(w, lo, acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, hi, acc[2 * i + 1]);
  }
}

__global__ void __launch_bounds__(kCombThreads)
    combine_kernel(const uint4 *__restrict__ ypool, const float *__restrict__ topk_w,
                   const int32_t *__restrict__ pool_row, uint4 *__restrict__ out, int32_t T,
                   int32_t k, int32_t hv) {
  __shared__ int32_t s_p[kMaxTopK];
  __shared__ float s_w[kMaxTopK];
  const int tid = threadIdx.x;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    if (tid < k) {
      s_p[tid] = pool_row[t * k + tid];
      s_w[tid] = topk_w != nullptr ? topk_w[t * k + tid] : 1.0f;
    }
    __syncthreads();
    for (int v = tid; v < hv; v += kCombThreads) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      for (int j0 = 0; j0 < k; j0 += kCombGroup) {
        uint4 y[kCombGroup];
#pragma unroll
        for (int jj = 0; jj < kCombGroup; ++jj) {
          const int j = j0 + jj;
          if (j < k && s_p[j] >= 0) y[jj] = ld_nc_v4(ypool + (size_t)s_p[j] * hv + v);
        }
#pragma unroll
        for (int jj = 0; jj < kCombGroup; ++jj) {
          const int j = j0 + jj;
          if (j < k && s_p[j] >= 0) fma_bf16x8(acc, s_w[j], y[jj]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      out[(size_t)t * hv + v] = o;
    }
    __syncthreads();
  }
}

cudaError_t launch_combine(const moe_shape &s, const void *ypool, const float *topk_w,
                           const moe_plan_buffers &p, void *out, int num_sms, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  int64_t grid = (int64_t)num_sms * 16;
  if (grid > s.T) grid = s.T;
  combine_kernel<<<(int)grid, kCombThreads, 0, st>>>(static_cast<const uint4 *>(ypool), topk_w,
                                                     p.pool_row, static_cast<uint4 *>(out), s.T,
                                                     s.k, s.H / 8);
  return cudaGetLastError();
}

}  // namespace moe
