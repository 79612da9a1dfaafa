// HBM rate probes: what a plain kernel of this library reaches when it only writes, or
// copies, a buffer far larger than L2. They give dispatch and combine the measured
// ceiling their rates are compared with (dispatch writes about nine bytes per byte it
// reads, so the write rate, not the copy rate, is the one that bounds it). Not part of the
// layer's method; the bench runs them beside the layer on the same GPU.
//   mode 0: write, 16-byte st.global.v4 stores, 8 per thread in flight, grid-stride
//   mode 1: write, cp.async.bulk stores of 16 KB from a zeroed shared-memory block (the
//           store form dispatch uses), one issuing lane per block, 4 groups in flight
//   mode 2: copy src -> dst, 16-byte loads and stores, 8 per thread in flight
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kVecThreads = 256;
constexpr int kUnroll = 8;
constexpr uint32_t kBulkBytes = 16384;

__global__ void __launch_bounds__(kVecThreads)
    probe_write_kernel(uint4 *__restrict__ dst, int64_t n_vec) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  const int64_t stride = (int64_t)gridDim.x * kVecThreads * kUnroll;
  for (int64_t base = (int64_t)blockIdx.x * kVecThreads * kUnroll + threadIdx.x; base < n_vec;
       base += stride) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kVecThreads;
      if (i < n_vec) dst[i] = z;
    }
  }
}

__global__ void __launch_bounds__(kVecThreads)
    probe_copy_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t n_vec) {
  const int64_t stride = (int64_t)gridDim.x * kVecThreads * kUnroll;
  for (int64_t base = (int64_t)blockIdx.x * kVecThreads * kUnroll + threadIdx.x; base < n_vec;
       base += stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kVecThreads;
      if (i < n_vec) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + (int64_t)u * kVecThreads;
      if (i < n_vec) dst[i] = v[u];
    }
  }
}

__global__ void __launch_bounds__(32)
    probe_bulk_write_kernel(uint8_t *__restrict__ dst, int64_t n_chunks) {
  __shared__ __align__(128) uint8_t zeros[kBulkBytes];
  for (uint32_t i = threadIdx.x * 16; i < kBulkBytes; i += 32 * 16)
    *reinterpret_cast<uint4 *>(zeros + i) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_shared();  // the zeros, written by threads, are read by the bulk copies
  __syncwarp();
  if (threadIdx.x != 0) return;
  int64_t issued = 0;
  for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     dst + (size_t)c * kBulkBytes),
                 "r"(smem_u32(zeros)), "r"(kBulkBytes)
                 : "memory");
    bulk_commit_group();
    // at most four 16 KB stores in flight per block
    if (++issued >= 4) asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
  }
  bulk_wait_group_all();
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_hbm_probe(void *dst, const void *src, size_t bytes, int32_t mode,
                             void *stream) {
  if (dst == nullptr || (mode == 2 && src == nullptr)) return MOE_ERR_INVALID_ARG;
  if (mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dst) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(src) & 15u) != 0)
    return MOE_ERR_MISALIGNED;
  if (bytes == 0) return MOE_OK;
  const size_t unit = mode == 1 ? kBulkBytes : 16;
  if (bytes % unit != 0) return MOE_ERR_INVALID_ARG;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode == 1) {
    // 12 one-warp blocks per SM, each with a 16 KB block of zeros and up to four 16 KB
    // stores in flight
    const int64_t n = (int64_t)(bytes / kBulkBytes);
    const int64_t grid = n < (int64_t)nsm * 12 ? n : (int64_t)nsm * 12;
    probe_bulk_write_kernel<<<(int)grid, 32, 0, st>>>(static_cast<uint8_t *>(dst), n);
  } else {
    const int64_t n = (int64_t)(bytes / 16);
    const int64_t per_block = (int64_t)kVecThreads * kUnroll;
    int64_t grid = (n + per_block - 1) / per_block;
    if (grid > (int64_t)nsm * 8) grid = (int64_t)nsm * 8;
    if (mode == 0)
      probe_write_kernel<<<(int)grid, kVecThreads, 0, st>>>(static_cast<uint4 *>(dst), n);
    else
      probe_copy_kernel<<<(int)grid, kVecThreads, 0, st>>>(static_cast<const uint4 *>(src),
                                                           static_cast<uint4 *>(dst), n);
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
