// Dispatch (StreamEP README, How it works, "Pool-layout dispatch" and
// "Per-tile streaming"): every live (token, k) pair's row of x lands directly in
// its expert-major, tile-padded pool row, padding rows become zero, and each
// tile's flag counts the rows that have landed (release order), so the grouped
// GEMM can claim a tile as soon as its flag reaches the tile height.
//
// One block of 128 threads per work item, grid-stride over E + T items:
//   item e < E    zero the padding rows of expert e (all in its last tile)
//   item E + t    read x[t] once (16-byte vectors, no L1 allocation) and write it
//                 to the k pool rows of token t
// HBM traffic per call: T*H*2 read + (live pairs + padding rows)*H*2 written.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kDispThreads = 128;
constexpr int kDispVec = 8;  // 16-byte vectors per thread held in registers per pass

__device__ __forceinline__ uint4 ld_stream_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kDispThreads)
    dispatch_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ pool_row,
                    const int32_t *__restrict__ offsets, const int32_t *__restrict__ counts,
                    uint4 *__restrict__ pool, uint32_t *__restrict__ flags, int32_t T, int32_t k,
                    int32_t E, int32_t hv, int32_t tile, int32_t signal) {
  __shared__ int32_t s_rows[kMaxTopK];
  const int tid = threadIdx.x;
  const int64_t items = (int64_t)E + T;
  for (int64_t w = blockIdx.x; w < items; w += gridDim.x) {
    if (w < E) {
      const int e = (int)w;
      const int32_t start = offsets[e] + counts[e];
      const int32_t end = offsets[e + 1];
      const int32_t npad = end - start;
      if (npad <= 0) continue;  // uniform across the block
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int32_t r = 0; r < npad; ++r) {
        uint4 *dst = pool + (size_t)(start + r) * hv;
        for (int v = tid; v < hv; v += kDispThreads) dst[v] = z;
      }
      if (signal) {
        __threadfence();
        __syncthreads();
        if (tid == 0) red_release_gpu_add(flags + (end - 1) / tile, (uint32_t)npad);
      }
    } else {
      const int64_t t = w - E;
      if (tid < k) s_rows[tid] = pool_row[t * k + tid];
      __syncthreads();
      const uint4 *src = x + (size_t)t * hv;
      for (int v0 = 0; v0 < hv; v0 += kDispThreads * kDispVec) {
        uint4 buf[kDispVec];
#pragma unroll
        for (int i = 0; i < kDispVec; ++i) {
          const int v = v0 + i * kDispThreads + tid;
          if (v < hv) buf[i] = ld_stream_v4(src + v);
        }
        for (int j = 0; j < k; ++j) {
          const int32_t p = s_rows[j];
          if (p < 0) continue;
          uint4 *dst = pool + (size_t)p * hv;
#pragma unroll
          for (int i = 0; i < kDispVec; ++i) {
            const int v = v0 + i * kDispThreads + tid;
            if (v < hv) dst[v] = buf[i];
          }
        }
      }
      if (signal) {
        __threadfence();
        __syncthreads();
        if (tid < k && s_rows[tid] >= 0) red_release_gpu_add(flags + s_rows[tid] / tile, 1u);
      }
    }
    __syncthreads();  // s_rows is rewritten by the next item
  }
}

cudaError_t launch_dispatch(const moe_shape &s, const void *x, const moe_plan_buffers &p,
                            void *pool, int signal, int num_sms, cudaStream_t st) {
  const int64_t items = (int64_t)s.E + s.T;
  int64_t grid = (int64_t)num_sms * 8;
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  dispatch_kernel<<<(int)grid, kDispThreads, 0, st>>>(
      static_cast<const uint4 *>(x), p.pool_row, p.offsets, p.counts, static_cast<uint4 *>(pool),
      p.tile_flags, s.T, s.k, s.E, s.H / 8, s.tile, signal);
  return cudaGetLastError();
}

}  // namespace moe
