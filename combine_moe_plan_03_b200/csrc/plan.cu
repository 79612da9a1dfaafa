// Routing plan: per-expert histogram, padded prefix offsets and a stable
// (token, k) -> pool-row map (StreamEP README, How it works, "Pool-layout
// dispatch": an expert-major, tile-padded pool).
//
// Three launches on the caller's stream:
//   plan_hist_kernel   one warp per 256-pair chunk counts its pairs per expert
//                      (shared-memory histogram), writes ws[e][chunk]; resets
//                      row_src, tile_expert, tile_flags and the finalize counter.
//   plan_scan_kernel   one block per expert: exclusive scan of ws[e][*] over the
//                      chunks (the chunk's base inside the expert), counts[e].
//                      The last block to finish pads the counts to the tile,
//                      scans them into offsets, and writes tile_expert, the GEMM
//                      row-chunk table and meta. An expert's live rows are cut into
//                      ceil(count/256) chunks of equal size (a multiple of 16), so
//                      the grouped GEMM's units of one expert run at the same pace
//                      and share each weight tile through L2.
//   plan_rank_kernel   each warp walks its chunk again 32 pairs at a time;
//                      __match_any_sync groups lanes with the same expert and the
//                      rank inside the group is the popcount of lower lanes, so
//                      pool_row[f] = offsets[e] + base[e][chunk] + running + rank
//                      is ordered by the flat pair id inside each expert.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

PlanGeom plan_geom(const moe_shape &s) {
  PlanGeom g;
  g.pairs = (int64_t)s.T * s.k;
  int64_t nonempty = g.pairs < s.E ? g.pairs : (int64_t)s.E;
  int64_t rows = g.pairs + nonempty * (s.tile - 1);
  g.pmax = (rows + s.tile - 1) / s.tile * s.tile;
  g.n_tiles = g.pmax / s.tile;
  g.n_chunks = (int32_t)((g.pairs + kPlanChunk - 1) / kPlanChunk);
  return g;
}

size_t plan_workspace_ints(const moe_shape &s) {
  PlanGeom g = plan_geom(s);
  return (size_t)s.E * (size_t)(g.n_chunks > 0 ? g.n_chunks : 1) + 8;
}

__global__ void __launch_bounds__(kPlanWarps * 32)
    plan_hist_kernel(const int32_t *__restrict__ idx, int64_t pairs, int32_t E, int32_t n_chunks,
                     int32_t *__restrict__ ws, int32_t *__restrict__ done_counter,
                     const PlanResets resets, int32_t *__restrict__ status) {
  extern __shared__ int32_t hist[];  // [kPlanWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kPlanWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int chunk = blockIdx.x * kPlanWarps + warp;
  if (chunk < n_chunks) {
    int32_t *h = hist + warp * E;
    const int64_t base = (int64_t)chunk * kPlanChunk;
#pragma unroll
    for (int r = 0; r < kPlanChunk / 32; ++r) {
      const int64_t f = base + r * 32 + lane;
      if (f < pairs) {
        const int32_t e = idx[f];
        if (e >= 0 && e < E)
          atomicAdd(&h[e], 1);
        else if (e != -1)
          report(status, MOE_ERR_BAD_INDEX, (int32_t)f);
      }
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) ws[(int64_t)e * n_chunks + chunk] = h[e];
  }
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t gsz = (int64_t)gridDim.x * blockDim.x;
  if (gtid == 0) *done_counter = 0;
  plan_reset_slice(resets, gtid, gsz);
}

PlanResets plan_resets(const moe_shape &s, const moe_plan_buffers &p) {
  const PlanGeom g = plan_geom(s);
  return PlanResets{p.row_src, g.pmax, p.tile_expert, p.tile_flags, g.n_tiles,
                    p.tok_pending, p.ready, (int64_t)s.T};
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, <= 1024).
// Returns the exclusive prefix; *total gets the block sum.
__device__ __forceinline__ int32_t block_excl_scan(int32_t v, int32_t *warp_sums, int32_t *total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t s = lane < nwarps ? warp_sums[lane] : 0;
    int32_t si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    if (lane < nwarps) warp_sums[lane] = si - s;  // exclusive warp prefix
    if (lane == 31) warp_sums[32] = si;
  }
  __syncthreads();
  const int32_t r = warp_sums[warp] + incl - v;
  *total = warp_sums[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256)
    plan_scan_kernel(int32_t *__restrict__ ws, int32_t n_chunks, int32_t E, int32_t tile,
                     int32_t *__restrict__ done_counter, int32_t *__restrict__ counts,
                     int32_t *__restrict__ offsets, int32_t *__restrict__ tile_expert,
                     int32_t *__restrict__ mblk, int32_t *__restrict__ meta, int64_t pmax,
                     int32_t *__restrict__ status) {
  __shared__ int32_t warp_sums[33];
  __shared__ int32_t s_last;
  const int e = blockIdx.x;
  int32_t *col = ws + (int64_t)e * n_chunks;
  int32_t carry = 0;
  for (int b = 0; b < n_chunks; b += blockDim.x) {
    const int i = b + threadIdx.x;
    const int32_t v = i < n_chunks ? col[i] : 0;
    int32_t tot;
    const int32_t ex = block_excl_scan(v, warp_sums, &tot);
    if (i < n_chunks) col[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) counts[e] = carry;

  // The last expert block to finish builds the offsets and the tile / row-block tables.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(done_counter, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  const int e1 = min(E, e0 + per);
  __shared__ unsigned long long s_rows;
  if (threadIdx.x == 0) s_rows = 0;
  __syncthreads();
  int64_t rows64 = 0;
  int32_t my_blk = 0;
  for (int x = e0; x < e1; ++x) {
    const int32_t c = __ldcg(counts + x);
    rows64 += ((int64_t)c + tile - 1) / tile * tile;
    const int32_t chunk = gemm_chunk_rows(c);
    if (c > 0) my_blk += (c + chunk - 1) / chunk;
  }
  // the block's total in 64 bits: a warp sum, then one shared atomic per warp
  unsigned long long wsum = (unsigned long long)rows64;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_rows, wsum);
  __syncthreads();
  // Counts beyond the dropless bound (only counts passed in by a caller, as in expert
  // parallelism, can do this): leave an empty plan, whose tables fit any arena, and report.
  if (s_rows > (unsigned long long)pmax) {
    for (int x = e0; x < e1; ++x) {
      counts[x] = 0;
      offsets[x] = 0;
    }
    if (threadIdx.x == 0) {
      offsets[E] = 0;
      for (int i = 0; i < 8; ++i) meta[i] = 0;
      report(status, MOE_ERR_POOL_OVERFLOW,
             s_rows > (unsigned long long)INT32_MAX ? INT32_MAX : (int32_t)s_rows);
    }
    return;
  }
  // the total is at most pmax (< 2^31), so the int32 scans below cannot overflow
  int32_t tot_rows, tot_blk;
  int32_t row = block_excl_scan((int32_t)rows64, warp_sums, &tot_rows);
  int32_t blk = block_excl_scan(my_blk, warp_sums, &tot_blk);
  for (int x = e0; x < e1; ++x) {
    const int32_t c = __ldcg(counts + x);
    const int32_t pad = (c + tile - 1) / tile * tile;
    offsets[x] = row;
    for (int32_t r = 0; r < pad; r += tile) tile_expert[(row + r) / tile] = x;
    const int32_t chunk = gemm_chunk_rows(c);
    const int32_t first = blk, n_ch = c > 0 ? (c + chunk - 1) / chunk : 0;
    for (int32_t r = 0; r < c; r += chunk) {  // live rows only: padding is not computed
      int32_t *m = mblk + (int64_t)kMblkInts * blk;
      m[0] = row + r;
      m[1] = x;
      m[2] = min(chunk, c - r);
      m[3] = first;
      m[4] = n_ch;
      ++blk;
    }
    row += pad;
  }
  if (threadIdx.x == 0) {
    offsets[E] = tot_rows;
    meta[0] = tot_rows / tile;
    meta[1] = tot_rows;
    meta[2] = tot_blk;
    meta[3] = 0;
    for (int i = 4; i < 8; ++i) meta[i] = 0;  // grouped-GEMM unit counters
  }
}

__global__ void __launch_bounds__(kPlanWarps * 32)
    plan_rank_kernel(const int32_t *__restrict__ idx, int64_t pairs, int32_t E, int32_t n_chunks,
                     const int32_t *__restrict__ ws, const int32_t *__restrict__ offsets,
                     int32_t *__restrict__ pool_row, int32_t *__restrict__ row_src) {
  extern __shared__ int32_t run[];  // [kPlanWarps][E]: next free row of expert e for this chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kPlanWarps + warp;
  if (chunk >= n_chunks) return;
  int32_t *r = run + warp * E;
  for (int e = lane; e < E; e += 32) r[e] = offsets[e] + ws[(int64_t)e * n_chunks + chunk];
  __syncwarp();
  const uint32_t lt = lanemask_lt();
  const int64_t base = (int64_t)chunk * kPlanChunk;
#pragma unroll 1
  for (int q = 0; q < kPlanChunk / 32; ++q) {
    const int64_t f = base + q * 32 + lane;
    const int32_t e = f < pairs ? idx[f] : -1;
    const bool live = e >= 0 && e < E;
    const int32_t key = live ? e : -1 - lane;  // dead lanes never match anyone
    const uint32_t same = __match_any_sync(0xffffffffu, key);
    const int32_t rank = __popc(same & lt);
    const int32_t row = live ? r[e] : 0;
    __syncwarp();
    if (live && rank == 0) r[e] = row + __popc(same);
    __syncwarp();
    if (f < pairs) {
      if (live) {
        pool_row[f] = row + rank;
        row_src[row + rank] = (int32_t)f;
      } else {
        pool_row[f] = -1;
      }
    }
  }
}

cudaError_t launch_plan(const moe_shape &s, const int32_t *topk_idx, const moe_plan_buffers &p,
                        cudaStream_t st) {
  const PlanGeom g = plan_geom(s);
  const size_t smem = sizeof(int32_t) * kPlanWarps * (size_t)s.E;
  int32_t *done = p.workspace + (size_t)s.E * (size_t)(g.n_chunks > 0 ? g.n_chunks : 1);
  const int nblk = g.n_chunks > 0 ? (g.n_chunks + kPlanWarps - 1) / kPlanWarps : 0;
  const int hist_blocks = nblk > 0 ? nblk : 1;
  plan_hist_kernel<<<hist_blocks, kPlanWarps * 32, smem, st>>>(
      topk_idx, g.pairs, s.E, g.n_chunks, p.workspace, done, plan_resets(s, p), p.status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_plan_scan_rank(s, topk_idx, p, st);
}

cudaError_t launch_plan_scan_only(const moe_shape &s, int32_t n_src, int32_t *ws, int32_t *done,
                                  int32_t *counts, int32_t *offsets, int32_t *tile_expert,
                                  int32_t *mblk, int32_t *meta, int32_t *status, cudaStream_t st) {
  plan_scan_kernel<<<s.E, 256, 0, st>>>(ws, n_src, s.E, s.tile, done, counts, offsets,
                                         tile_expert, mblk, meta, plan_geom(s).pmax, status);
  return cudaGetLastError();
}

cudaError_t launch_plan_scan_rank(const moe_shape &s, const int32_t *topk_idx,
                                  const moe_plan_buffers &p, cudaStream_t st) {
  const PlanGeom g = plan_geom(s);
  const size_t smem = sizeof(int32_t) * kPlanWarps * (size_t)s.E;
  int32_t *done = p.workspace + (size_t)s.E * (size_t)(g.n_chunks > 0 ? g.n_chunks : 1);
  const int nblk = g.n_chunks > 0 ? (g.n_chunks + kPlanWarps - 1) / kPlanWarps : 0;
  cudaError_t err;
  plan_scan_kernel<<<s.E, 256, 0, st>>>(p.workspace, g.n_chunks, s.E, s.tile, done, p.counts,
                                         p.offsets, p.tile_expert, p.mblk, p.meta, g.pmax,
                                         p.status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (nblk > 0) {
    plan_rank_kernel<<<nblk, kPlanWarps * 32, smem, st>>>(topk_idx, g.pairs, s.E, g.n_chunks,
                                                          p.workspace, p.offsets, p.pool_row,
                                                          p.row_src);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace moe
