// Backward of the layer's activation path (StreamEP README, How it works: "The backward
// pass mirrors both overlaps" and the backward grouped GEMMs A and Y of "CuTeDSL compute
// kernels"). Given dy = d loss / d out [T, H] and the forward call's plan, pool and ypool:
//   combine, mirrored:   dypool[p] = bf16(w[t,j] * dy[t])  for p = pool_row[t,j]
//                        dw[t,j]   = sum_h dy[t,h] * ypool[p,h]       (fp32)
//   gate / up recompute: gu[p]     = bf16(pool[p] . W1[e])            (GEMM A without SwiGLU)
//   backward Y:          da[p]     = dypool[p] . W2[e]^T, and in its epilogue
//                        dgu[p]    = bf16(da * u * silu'(g), da * silu(g))
//   backward A:          dpool[p]  = bf16(dgu[p] . W1[e]^T)
//   dispatch, mirrored:  dx[t]     = bf16(sum_j dpool[pool_row[t,j]])  (fp32 sum, j order)
// This file holds the combine backward; the GEMMs are the SM-pair kernel (ffn_gemm_pair.cu)
// with the weights read K-major, and the dispatch backward is the combine kernel with unit
// weights (combine.cu).
#include "ffn_gemm.cuh"

namespace moe {

constexpr int kCbThreads = 128;

__device__ __forceinline__ float dot_bf16x8(const uint4 &a, const uint4 &b) {
  const uint32_t x[4] = {a.x, a.y, a.z, a.w};
  const uint32_t y[4] = {b.x, b.y, b.z, b.w};
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s = fmaf(__uint_as_float(x[i] << 16), __uint_as_float(y[i] << 16), s);
    s = fmaf(__uint_as_float(x[i] & 0xFFFF0000u), __uint_as_float(y[i] & 0xFFFF0000u), s);
  }
  return s;
}

__device__ __forceinline__ uint4 scale_bf16x8(const uint4 &a, float w) {
  const uint32_t x[4] = {a.x, a.y, a.z, a.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = pack_bf16x2(w * __uint_as_float(x[i] << 16), w * __uint_as_float(x[i] & 0xFFFF0000u));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// One block of 128 threads per token (grid-stride); thread v owns the 16-byte vectors v,
// v + 128, ... of the row. Per vector, dy is loaded once and the ypool vectors of up to 8
// pairs are all loaded before they are used; each pair's dypool vector is stored and its
// partial dot product kept in a register. One block reduction per token gives dw (0 for a
// dropped pair). HBM traffic per call: T*H*2 (dy) + 2 * live pairs * H*2 (ypool read,
// dypool written).
constexpr int kCbGroup = 8;

__global__ void __launch_bounds__(kCbThreads)
    combine_backward_kernel(const uint4 *__restrict__ dy, const uint4 *__restrict__ ypool,
                            const float *__restrict__ topk_w, const int32_t *__restrict__ pool_row,
                            uint4 *__restrict__ dypool, float *__restrict__ dw, int32_t T,
                            int32_t k, int32_t hv) {
  __shared__ int32_t s_p[kMaxTopK];
  __shared__ float s_w[kMaxTopK];
  __shared__ float s_red[kCbThreads / 32][kMaxTopK];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    if (tid < k) {
      s_p[tid] = pool_row[t * k + tid];
      s_w[tid] = topk_w[t * k + tid];
    }
    __syncthreads();
    for (int j0 = 0; j0 < k; j0 += kCbGroup) {
      float part[kCbGroup];
#pragma unroll
      for (int jj = 0; jj < kCbGroup; ++jj) part[jj] = 0.0f;
      for (int v = tid; v < hv; v += kCbThreads) {
        const uint4 d = dy[(size_t)t * hv + v];
        uint4 y[kCbGroup];
#pragma unroll
        for (int jj = 0; jj < kCbGroup; ++jj) {
          const int j = j0 + jj;
          if (j < k && s_p[j] >= 0) y[jj] = ypool[(size_t)s_p[j] * hv + v];
        }
#pragma unroll
        for (int jj = 0; jj < kCbGroup; ++jj) {
          const int j = j0 + jj;
          if (j < k && s_p[j] >= 0) {
            part[jj] += dot_bf16x8(d, y[jj]);
            dypool[(size_t)s_p[j] * hv + v] = scale_bf16x8(d, s_w[j]);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < kCbGroup; ++jj) {
        float x = part[jj];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0 && j0 + jj < k) s_red[warp][j0 + jj] = x;
      }
    }
    __syncthreads();
    if (tid < k) {
      float sum = 0.0f;
#pragma unroll
      for (int i = 0; i < kCbThreads / 32; ++i) sum += s_red[i][tid];
      dw[t * k + tid] = s_p[tid] >= 0 ? sum : 0.0f;
    }
    __syncthreads();
  }
}

// Early dispatch backward (the mirror of early combine): before backward A, every token's
// pending count is set to its live pairs x the row counts backward A makes per row (the
// same units of 512 output columns as GEMM Y, so early_combine_arrivals(H)), and a token
// without live pairs goes straight into the ready queue (its dx is zero). One warp per
// token; the queue (ready [T + 4]) must be zero before (moe_backward clears it first).
__global__ void __launch_bounds__(256)
    arm_tokens_kernel(const int32_t *__restrict__ pool_row, int32_t T, int32_t k,
                      int32_t arrivals, int32_t *__restrict__ tok_pending,
                      int32_t *__restrict__ ready) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = w0; t < T; t += nw) {
    const int32_t r = lane < k ? pool_row[t * k + lane] : -1;
    const int live = __popc(__ballot_sync(0xffffffffu, r >= 0));
    if (lane == 0) {
      tok_pending[t] = live * arrivals;
      if (live == 0) {
        const int32_t pos = atomicAdd(ready + T + 1, 1);
        if (pos < T) st_release_gpu(ready + pos, (int32_t)t + 1);
      }
    }
  }
}

cudaError_t launch_arm_tokens(const moe_shape &s, const moe_plan_buffers &p, int num_sms,
                              cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(p.ready, 0, sizeof(int32_t) * ((size_t)s.T + 4), st);
  if (e != cudaSuccess || s.T == 0) return e;
  int64_t grid = ((int64_t)s.T * 32 + 255) / 256;
  if (grid > (int64_t)num_sms * 8) grid = (int64_t)num_sms * 8;
  arm_tokens_kernel<<<(int)grid, 256, 0, st>>>(p.pool_row, s.T, s.k, early_combine_arrivals(s.H),
                                               p.tok_pending, p.ready);
  return cudaGetLastError();
}

// The combine backward in pool-tile order (the mirror of the streaming layer's tile-ordered
// dispatch): a block takes pool tiles in order and, for each live row p of the tile (pair
// f = row_src[p] of token t), writes dypool[p] = bf16(w[f] dy[t]) and dw[f] = dy[t] . ypool[p]
// with the token-ordered kernel's arithmetic (each thread's vectors v, v + 128, ..., the
// same shuffle tree and warp order, so both results are bit-identical); then it raises the
// tile's flag to the tile height (release) for a streaming backward Y. dw of dropped pairs
// is not written (the caller zeroes dw first).
__global__ void __launch_bounds__(kCbThreads)
    combine_backward_tiles_kernel(const uint4 *__restrict__ dy, const uint4 *__restrict__ ypool,
                                  const float *__restrict__ topk_w,
                                  const int32_t *__restrict__ row_src,
                                  const int32_t *__restrict__ meta, uint4 *__restrict__ dypool,
                                  float *__restrict__ dw, uint32_t *__restrict__ flags,
                                  int32_t k, int32_t hv, int32_t tile) {
  __shared__ float s_red[kCbThreads / 32];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int32_t n_tiles = meta[0];  // live tiles of this call's plan
  for (int32_t q = blockIdx.x; q < n_tiles; q += gridDim.x) {
    for (int32_t r = 0; r < tile; ++r) {
      const int64_t p = (int64_t)q * tile + r;
      const int32_t f = row_src[p];
      if (f < 0) continue;  // a padding row: uniform across the block
      const int64_t t = f / k;
      const float w = topk_w[f];
      float part = 0.0f;
      for (int v = tid; v < hv; v += kCbThreads) {
        const uint4 d = dy[(size_t)t * hv + v];
        part += dot_bf16x8(d, ypool[(size_t)p * hv + v]);
        dypool[(size_t)p * hv + v] = scale_bf16x8(d, w);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (lane == 0) s_red[warp] = part;
      __syncthreads();
      if (tid == 0) {
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < kCbThreads / 32; ++i) sum += s_red[i];
        dw[f] = sum;
      }
      __syncthreads();
    }
    // every thread's dypool stores of the tile precede the barrier above
    if (tid == 0) red_release_gpu_add(flags + q, (uint32_t)tile);
  }
}

cudaError_t launch_combine_backward_tiles(const moe_shape &s, const void *dy, const void *ypool,
                                          const float *topk_w, const moe_plan_buffers &p,
                                          void *dypool, float *dw, int blocks, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  combine_backward_tiles_kernel<<<blocks, kCbThreads, 0, st>>>(
      static_cast<const uint4 *>(dy), static_cast<const uint4 *>(ypool), topk_w, p.row_src,
      p.meta, static_cast<uint4 *>(dypool), dw, p.tile_flags, s.k, s.H / 8, s.tile);
  return cudaGetLastError();
}

cudaError_t launch_combine_backward(const moe_shape &s, const void *dy, const void *ypool,
                                    const float *topk_w, const moe_plan_buffers &p,
                                    void *dypool, float *dw, int num_sms, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  int64_t grid = (int64_t)num_sms * 16;
  if (grid > s.T) grid = s.T;
  combine_backward_kernel<<<(int)grid, kCbThreads, 0, st>>>(
      static_cast<const uint4 *>(dy), static_cast<const uint4 *>(ypool), topk_w, p.pool_row,
      static_cast<uint4 *>(dypool), dw, s.T, s.k, s.H / 8);
  return cudaGetLastError();
}

}  // namespace moe
