// Expert parallelism inside one node (StreamEP README: "intranode over NVLink"; "Pool-layout
// dispatch": routed pairs land directly in the expert-major, tile-padded pool of the rank
// that owns their expert). R ranks, one per GPU; rank d owns the E_r = E / R experts
// [d E_r, (d + 1) E_r). Every rank plans its own tokens over the E global experts (moe_plan);
// the per-expert counts of all ranks, C [R][E] (one all-gather of E integers per rank, made
// by the caller), fix every rank's pool: the rows of expert e come from rank 0's pairs, then
// rank 1's, ..., each in flat pair order, so rank d's pool is exactly the part of one
// dropless pool over all ranks' pairs that holds d's experts, re-based to row 0.
//
//   ep_prepare_kernel   C -> the workspaces of two plan scans (rows of each expert sent by
//                       each source rank): over all E experts (where each source writes)
//                       and over this rank's E_r experts (the grouped FFN's plan)
//   plan_scan_kernel    (plan.cu) twice: exclusive scans over the sources, padded offsets,
//                       the FFN's tile and row-chunk tables
//   ep_pad_kernel       zeroes this rank's padding rows (a block per row), counting each on
//                       its tile's flag
//   ep_dispatch_kernel  source side: x[t] staged once in shared memory, then stored (16-byte
//                       vectors, every lane) into the pool rows of its k pairs, on whichever
//                       rank owns each pair's expert (peer pointers); then each stored row is
//                       counted on its owner's tile flag (release at system scope), so a
//                       streaming grouped FFN on the owner takes a pool tile as soon as its
//                       rows from every rank and its padding have landed (flag = tile rows)
//   ep_combine_kernel   source side: out[t] = bf16(sum_j w[t, j] ypool_{owner}[row]) with the
//                       k rows gathered from their owners' ypools (peer loads), the same fp32
//                       FMA chain as combine.cu
// The grouped FFN in between is moe_grouped_ffn on each rank's own pool and plan. Peer
// pointers are plain device pointers of the other ranks' buffers (mapped for peer access by
// the caller); no TMA or multicast touches another GPU's memory.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kEpThreads = 256;

struct EpPeers {
  uint8_t *base[kMaxEpRanks];
};

struct EpFlags {
  uint32_t *base[kMaxEpRanks];   // each rank's pool tile flags (ep->local.tile_flags); or none
};

__global__ void __launch_bounds__(kEpThreads)
    ep_prepare_kernel(const int32_t *__restrict__ C, int32_t R, int32_t E, int32_t Er,
                      int32_t rank, int32_t *__restrict__ ws_g, int32_t *__restrict__ done_g,
                      int32_t *__restrict__ tiles_g, int64_t n_tiles_g,
                      int32_t *__restrict__ ws_l, int32_t *__restrict__ done_l,
                      int32_t *__restrict__ tiles_l, int64_t n_tiles_l, int32_t rank_pairs,
                      int32_t *__restrict__ status) {
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t gsz = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = gtid; i < (int64_t)E * R; i += gsz) {
    const int64_t e = i / R, s = i % R;
    int32_t c = C[s * E + e];
    // a rank sends at most its T k pairs: anything else cannot come from moe_plan, and is
    // clamped (so the scans stay in int32) and reported
    if (c < 0 || c > rank_pairs) {
      report(status, MOE_ERR_POOL_OVERFLOW, (int32_t)(s * E + e));
      c = c < 0 ? 0 : rank_pairs;
    }
    ws_g[i] = c;                                   // [e][s]
    if (e >= (int64_t)rank * Er && e < (int64_t)(rank + 1) * Er)
      ws_l[(e - (int64_t)rank * Er) * R + s] = c;  // [e - rank E_r][s]
  }
  for (int64_t i = gtid; i < n_tiles_g; i += gsz) tiles_g[i] = -1;
  for (int64_t i = gtid; i < n_tiles_l; i += gsz) tiles_l[i] = -1;
  if (gtid == 0) {
    *done_g = 0;
    *done_l = 0;
  }
}

// Padding rows of this rank's pool: [offsets[e] + counts[e], offsets[e + 1]) per local expert.
// Block (j, e) zeroes padding row j of expert e if it has one (16-byte stores; an expert has
// fewer than tile padding rows) and counts it on its tile's flag: every row in parallel.
__global__ void __launch_bounds__(kEpThreads)
    ep_pad_kernel(uint4 *__restrict__ pool, int32_t hv, const int32_t *__restrict__ counts,
                  const int32_t *__restrict__ offsets, uint32_t *__restrict__ flags,
                  int32_t tile) {
  const int e = blockIdx.y;
  const int64_t r = (int64_t)offsets[e] + counts[e] + blockIdx.x;
  if (r >= offsets[e + 1]) return;  // uniform across the block
  for (int i = threadIdx.x; i < hv; i += blockDim.x) pool[r * hv + i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (threadIdx.x == 0) red_release_sys_add(flags + r / tile, 1u);
}

// Row of pair f in its owner's pool, and the owner. own_*: the source's own plan over the
// E global experts; g_*: the plan over all ranks' pairs.
__device__ __forceinline__ int32_t ep_dest_row(int32_t f, int32_t src, int32_t R, int32_t Er,
                                               int32_t tile, const int32_t *own_pool_row,
                                               const int32_t *own_tile_expert,
                                               const int32_t *own_offsets,
                                               const int32_t *g_offsets,
                                               const int32_t *g_src_base, int64_t max_rows,
                                               int32_t *status, int32_t *owner) {
  const int32_t p = own_pool_row[f];
  if (p < 0) return -1;
  const int32_t e = own_tile_expert[p / tile];
  const int32_t d = e / Er;
  *owner = d;
  const int64_t row =
      (int64_t)g_offsets[e] - g_offsets[d * Er] + g_src_base[e * R + src] + (p - own_offsets[e]);
  // all_counts that disagree with a rank's own plan could place a row outside the owner's
  // pool: report it and skip the pair instead of touching memory past the pool
  if (row < 0 || row >= max_rows) {
    report(status, MOE_ERR_POOL_OVERFLOW, f);
    return -1;
  }
  return (int32_t)row;
}

__global__ void __launch_bounds__(kEpThreads)
    ep_dispatch_kernel(const uint4 *__restrict__ x, int32_t T, int32_t k, int32_t hv,
                       int32_t R, int32_t Er, int32_t tile, int32_t src,
                       const int32_t *__restrict__ own_pool_row,
                       const int32_t *__restrict__ own_tile_expert,
                       const int32_t *__restrict__ own_offsets,
                       const int32_t *__restrict__ g_offsets,
                       const int32_t *__restrict__ g_src_base, int64_t max_rows,
                       const int32_t *__restrict__ own_counts,
                       const int32_t *__restrict__ g_counts, int32_t *__restrict__ status,
                       const EpPeers pools, const EpFlags flags, bool signal) {
  extern __shared__ uint4 row[];  // [hv]: x[t]
  __shared__ int32_t s_row[kMaxTopK], s_dst[kMaxTopK];
  if (blockIdx.x == 0) {
    // this rank's row of all_counts, recovered from the scanned sources, must be its own
    // plan's counts; a mismatch means the caller's all_counts are not the ranks' plans
    const int32_t E = Er * R;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const int32_t next = src + 1 < R ? g_src_base[e * R + src + 1] : g_counts[e];
      if (next - g_src_base[e * R + src] != own_counts[e])
        report(status, MOE_ERR_POOL_OVERFLOW, e);
    }
  }
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    for (int i = threadIdx.x; i < hv; i += blockDim.x) row[i] = x[t * hv + i];
    if (threadIdx.x < k) {
      int32_t d = 0;
      s_row[threadIdx.x] = ep_dest_row((int32_t)(t * k + threadIdx.x), src, R, Er, tile,
                                       own_pool_row, own_tile_expert, own_offsets, g_offsets,
                                       g_src_base, max_rows, status, &d);
      s_dst[threadIdx.x] = d;
    }
    __syncthreads();
    for (int j = 0; j < k; ++j) {
      const int32_t r = s_row[j];
      if (r < 0) continue;  // uniform across the block
      uint4 *dst = reinterpret_cast<uint4 *>(pools.base[s_dst[j]]) + (size_t)r * hv;
      for (int i = threadIdx.x; i < hv; i += blockDim.x) dst[i] = row[i];
    }
    __syncthreads();
    // every thread's stores of the token's rows precede the barrier; the release at system
    // scope passes them on to the owner's acquire of the flag
    if (signal && threadIdx.x < k && s_row[threadIdx.x] >= 0)
      red_release_sys_add(flags.base[s_dst[threadIdx.x]] + s_row[threadIdx.x] / tile, 1u);
  }
}

__device__ __forceinline__ uint4 ld_nc_v4_ep(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kEpThreads)
    ep_combine_kernel(const float *__restrict__ topk_w, uint4 *__restrict__ out, int32_t T,
                      int32_t k, int32_t hv, int32_t R, int32_t Er, int32_t tile, int32_t src,
                      const int32_t *__restrict__ own_pool_row,
                      const int32_t *__restrict__ own_tile_expert,
                      const int32_t *__restrict__ own_offsets,
                      const int32_t *__restrict__ g_offsets,
                      const int32_t *__restrict__ g_src_base, int64_t max_rows,
                      int32_t *__restrict__ status, const EpPeers ypools) {
  __shared__ const uint4 *s_src[kMaxTopK];
  __shared__ float s_w[kMaxTopK];
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      int32_t d = 0;
      const int32_t r = ep_dest_row((int32_t)(t * k + threadIdx.x), src, R, Er, tile,
                                    own_pool_row, own_tile_expert, own_offsets, g_offsets,
                                    g_src_base, max_rows, status, &d);
      s_src[threadIdx.x] =
          r < 0 ? nullptr : reinterpret_cast<const uint4 *>(ypools.base[d]) + (size_t)r * hv;
      s_w[threadIdx.x] = topk_w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (int v = threadIdx.x; v < hv; v += blockDim.x) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      for (int j0 = 0; j0 < k; j0 += 8) {
        uint4 y[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (j0 + jj < k && s_src[j0 + jj] != nullptr) y[jj] = ld_nc_v4_ep(s_src[j0 + jj] + v);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (j0 + jj < k && s_src[j0 + jj] != nullptr) {
            const float w = s_w[j0 + jj];
            const uint32_t u[4] = {y[jj].x, y[jj].y, y[jj].z, y[jj].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
              acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
          }
      }
      out[t * hv + v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
    __syncthreads();
  }
}

EpPeers peers_of(void *const *ptrs, int32_t R) {
  EpPeers p{};
  for (int i = 0; i < R && i < kMaxEpRanks; ++i) p.base[i] = static_cast<uint8_t *>(ptrs[i]);
  return p;
}

EpFlags flags_of(uint32_t *const *ptrs, int32_t R) {
  EpFlags f{};
  for (int i = 0; ptrs != nullptr && i < R && i < kMaxEpRanks; ++i) f.base[i] = ptrs[i];
  return f;
}

}  // namespace

cudaError_t launch_ep_layout(const moe_shape &rank_shape, int32_t R, int32_t rank,
                             const int32_t *C, const moe_ep_plan &ep, void *pool,
                             int num_sms, cudaStream_t st) {
  const int32_t Er = rank_shape.E / R;
  const moe_shape gs = ep_global_shape(rank_shape, R), ls = ep_local_shape(rank_shape, R);
  const PlanGeom gg = plan_geom(gs), lg = plan_geom(ls);
  int32_t *done_g = ep.src_base + (size_t)rank_shape.E * R;
  int32_t *done_l = ep.local.workspace + (size_t)Er * R;
  const int grid = num_sms * 2;
  ep_prepare_kernel<<<grid, kEpThreads, 0, st>>>(C, R, rank_shape.E, Er, rank, ep.src_base,
                                                 done_g, ep.tile_expert, gg.n_tiles,
                                                 ep.local.workspace, done_l,
                                                 ep.local.tile_expert, lg.n_tiles,
                                                 rank_shape.T * rank_shape.k, ep.local.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_plan_scan_only(gs, R, ep.src_base, done_g, ep.counts, ep.offsets, ep.tile_expert,
                            ep.mblk, ep.meta, ep.local.status, st);
  if (e != cudaSuccess) return e;
  e = launch_plan_scan_only(ls, R, ep.local.workspace, done_l, ep.local.counts,
                            ep.local.offsets, ep.local.tile_expert, ep.local.mblk,
                            ep.local.meta, ep.local.status, st);
  if (e != cudaSuccess) return e;
  // the tile flags are not reset here: other ranks' dispatches may already be counting on
  // them; moe_ep_combine resets them after this rank's grouped FFN has used them
  ep_pad_kernel<<<dim3(rank_shape.tile - 1, Er), kEpThreads, 0, st>>>(
      static_cast<uint4 *>(pool), rank_shape.H / 8, ep.local.counts, ep.local.offsets,
      reinterpret_cast<uint32_t *>(ep.local.tile_flags), rank_shape.tile);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const moe_shape &rank_shape, int32_t R, int32_t rank,
                               const void *x, const moe_plan_buffers &own, const moe_ep_plan &ep,
                               void *const *pools, uint32_t *const *tile_flags, int num_sms,
                               cudaStream_t st) {
  if (rank_shape.T == 0) return cudaSuccess;
  const int hv = rank_shape.H / 8;
  const size_t smem = (size_t)hv * sizeof(uint4);  // one row of x (H <= 38,720 by check_shape)
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(ep_dispatch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return cudaErrorUnknown;
  // a block per token, every token of the rank in flight at once where they fit (8 blocks
  // of 256 threads per SM)
  int64_t grid = (int64_t)num_sms * 8;
  if (grid > rank_shape.T) grid = rank_shape.T;
  ep_dispatch_kernel<<<(int)grid, kEpThreads, smem, st>>>(
      static_cast<const uint4 *>(x), rank_shape.T, rank_shape.k, hv, R, rank_shape.E / R,
      rank_shape.tile, rank, own.pool_row, own.tile_expert, own.offsets, ep.offsets,
      ep.src_base, plan_geom(ep_local_shape(rank_shape, R)).pmax, own.counts, ep.counts,
      own.status, peers_of(pools, R), flags_of(tile_flags, R), tile_flags != nullptr);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const moe_shape &rank_shape, int32_t R, int32_t rank,
                              void *const *ypools, const float *topk_w,
                              const moe_plan_buffers &own, const moe_ep_plan &ep, void *out,
                              int num_sms, cudaStream_t st) {
  // this rank's pool tile flags, counted by every rank's dispatch and used by this rank's
  // grouped FFN, back to zero for the next layer call (also when this rank has no tokens)
  cudaError_t e = cudaMemsetAsync(
      ep.local.tile_flags, 0,
      sizeof(uint32_t) * (size_t)plan_geom(ep_local_shape(rank_shape, R)).n_tiles, st);
  if (e != cudaSuccess || rank_shape.T == 0) return e;
  int64_t grid = (int64_t)num_sms * 8;
  if (grid > rank_shape.T) grid = rank_shape.T;
  ep_combine_kernel<<<(int)grid, kEpThreads, 0, st>>>(
      topk_w, static_cast<uint4 *>(out), rank_shape.T, rank_shape.k, rank_shape.H / 8, R,
      rank_shape.E / R, rank_shape.tile, rank, own.pool_row, own.tile_expert, own.offsets,
      ep.offsets, ep.src_base, plan_geom(ep_local_shape(rank_shape, R)).pmax, own.status,
      peers_of(ypools, R));
  return cudaGetLastError();
}

}  // namespace moe
