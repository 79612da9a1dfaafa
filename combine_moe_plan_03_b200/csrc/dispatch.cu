// Dispatch (StreamEP README, How it works, "Pool-layout dispatch" and
// "Per-tile streaming"): every live (token, k) pair's row of x lands directly in
// its expert-major, tile-padded pool row, padding rows become zero, and each
// tile's flag counts the rows that have landed (release order), so the grouped
// GEMM can claim a tile as soon as its flag reaches the tile height.
//
// Rows move as whole-row bulk copies staged in shared memory: one bulk load of
// x[t] (H*2 bytes) into a shared buffer, then one bulk store of that buffer per
// pool row of the token; padding rows are bulk-stored from a zeroed shared row.
// Each block is one warp: lane j reads the token's j-th pool row id, lane 0 issues
// the copies; two staging buffers let the load of the block's next token overlap
// the stores of the current one.
// Work items, grid-stride over kPadPieces*E + T, each about one token's worth of stores:
//   item w < kPadPieces*E   padding rows 8q ... 8q + 7 (q = w % kPadPieces) of expert
//                           w / kPadPieces (all padding rows are in the expert's last tile)
//   item kPadPieces*E + t   token t
// HBM traffic per call: T*H*2 read + (live pairs + padding rows)*H*2 written.
// Armed for early combine, each token item also sets the token's count of expert-row stores
// that GEMM Y must make before the token can be combined, and a token without live pairs
// goes straight into the ready queue.
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kPadRowsPerItem = 8;
constexpr int kPadPieces = 128 / kPadRowsPerItem;  // covers the < tile <= 128 padding rows

__device__ __forceinline__ void bulk_load_row(void *dst_smem, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_store_row(void *dst, const void *src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src_smem)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// All but the newest `n` committed groups have finished reading their shared sources.
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

// All committed groups are complete (their global writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(32)
    dispatch_kernel(const uint8_t *__restrict__ x, const int32_t *__restrict__ pool_row,
                    const int32_t *__restrict__ offsets, const int32_t *__restrict__ counts,
                    uint8_t *__restrict__ pool, uint32_t *__restrict__ flags, int32_t T, int32_t k,
                    int32_t E, uint32_t row_bytes, int32_t tile, int32_t signal,
                    uint64_t timeout_ns, int32_t *__restrict__ status,
                    int32_t *__restrict__ tok_pending, int32_t *__restrict__ ready,
                    int32_t arrivals) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *zeros = sm + 2 * row_bytes;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 3 * row_bytes);
  int *never = reinterpret_cast<int *>(bar + 2);
  const int lane = threadIdx.x;

  for (uint32_t i = lane * 16; i < row_bytes; i += 32 * 16)
    *reinterpret_cast<uint4 *>(zeros + i) = make_uint4(0u, 0u, 0u, 0u);
  if (lane == 0) {
    mbar_init(bar + 0, 1);
    mbar_init(bar + 1, 1);
    *never = 0;
    fence_mbarrier_init();
  }
  fence_proxy_async_shared();  // the zeros and barriers, written by threads, are read by bulk copies
  __syncwarp();

  const int64_t n_pad_items = (int64_t)kPadPieces * E;
  const int64_t items = n_pad_items + T;
  const int64_t G = gridDim.x;
  // Lane 0 issues every copy. Token loads alternate between two staging buffers; the
  // load of the block's next token is issued before the current token's stores.
  uint32_t uses[2] = {0u, 0u};     // loads issued into each buffer so far
  uint32_t cur = 0;                // buffer holding the current token (if prefetched)
  bool have = false;               // the current token's load was already issued
  bool failed = false;
  for (int64_t w = blockIdx.x; w < items && !failed; w += G) {
    if (w < n_pad_items) {
      if (lane == 0) {
        const int e = (int)(w / kPadPieces);
        const int32_t start = offsets[e] + counts[e] + (int32_t)(w % kPadPieces) * kPadRowsPerItem;
        const int32_t end = min(offsets[e + 1], start + kPadRowsPerItem);
        if (end > start) {
          for (int32_t r = start; r < end; ++r)
            bulk_store_row(pool + (size_t)r * row_bytes, zeros, row_bytes);
          bulk_commit();
          if (signal) {
            bulk_wait_all();
            fence_proxy_async_global();
            red_release_gpu_add(flags + (end - 1) / tile, (uint32_t)(end - start));
          }
        }
      }
      continue;
    }
    const int64_t t = w - n_pad_items;
    const int32_t my_row = lane < k ? pool_row[t * k + lane] : -1;
    if (tok_pending != nullptr) {
      // early combine: GEMM Y makes `arrivals` row counts per live pair of the token
      const int live = __popc(__ballot_sync(0xffffffffu, my_row >= 0));
      if (lane == 0) {
        tok_pending[t] = live * arrivals;
        if (live == 0) {
          const int32_t pos = atomicAdd(ready + T + 1, 1);
          if (pos < T) st_release_gpu(ready + pos, (int32_t)t + 1);
        }
      }
    }
    if (lane == 0) {
      if (!have) {
        bulk_wait_read<0>();  // nothing may still read the buffer that is about to be filled
        mbar_arrive_expect_tx(bar + cur, row_bytes);
        bulk_load_row(sm + cur * row_bytes, x + (size_t)t * row_bytes, row_bytes, bar + cur);
        ++uses[cur];
      }
      const int64_t wn = w + G;
      const uint32_t nxt = cur ^ 1u;
      const bool prefetch = wn < items && wn >= n_pad_items;
      if (prefetch) {
        bulk_wait_read<0>();  // the previous token's stores have read the other buffer
        mbar_arrive_expect_tx(bar + nxt, row_bytes);
        bulk_load_row(sm + nxt * row_bytes, x + (size_t)(wn - n_pad_items) * row_bytes,
                      row_bytes, bar + nxt);
        ++uses[nxt];
      }
      if (!mbar_wait(bar + cur, (uses[cur] - 1u) & 1u, timeout_ns, never)) {
        report(status, MOE_ERR_PIPE_TIMEOUT, (int32_t)t);
        failed = true;
      }
      have = prefetch;
    }
    failed = __shfl_sync(0xffffffffu, failed ? 1 : 0, 0) != 0;
    if (failed) break;
    for (int j = 0; j < k; ++j) {
      const int32_t p = __shfl_sync(0xffffffffu, my_row, j);
      if (lane == 0 && p >= 0)
        bulk_store_row(pool + (size_t)p * row_bytes, sm + cur * row_bytes, row_bytes);
    }
    if (lane == 0) bulk_commit();
    if (signal) {
      // the rows must have landed before their tiles are counted (by the thread that
      // issued and waited for the writes)
      if (lane == 0) {
        bulk_wait_all();
        fence_proxy_async_global();
      }
      for (int j = 0; j < k; ++j) {
        const int32_t p = __shfl_sync(0xffffffffu, my_row, j);
        if (lane == 0 && p >= 0) red_release_gpu_add(flags + p / tile, 1u);
      }
    }
    cur ^= 1u;
  }
  if (lane == 0) {
    // a prefetched load that was never consumed must land before the block exits
    if (have) mbar_wait(bar + cur, (uses[cur] - 1u) & 1u, timeout_ns, never);
    bulk_wait_all();
  }
}

// Tile-ordered dispatch, for the streaming FFN: work item = one pool tile, taken in pool
// order (block b takes tiles b, b + G, ...), so tiles fill in the order in which GEMM A's
// unit tickets claim them. Each row of the tile is gathered through row_src: lane 0
// bulk-loads x[row_src[p] / k] into one of kTileBufs shared rows and bulk-stores it to
// pool[p] (padding rows from a zeroed row); loads run kTileBufs - 1 rows ahead of the
// stores. Once the tile's stores are complete the tile's flag is raised to the tile height
// (release). An x row is read once per pair here (k times per token, mostly from L2)
// instead of once per token: more reads, in exchange for tiles that fill in GEMM order.
constexpr int kTileBufs = 4;

__global__ void __launch_bounds__(32)
    dispatch_tiles_kernel(const uint8_t *__restrict__ x, const int32_t *__restrict__ row_src,
                          const int32_t *__restrict__ meta, uint8_t *__restrict__ pool,
                          uint32_t *__restrict__ flags, int32_t k, uint32_t row_bytes,
                          int32_t tile, uint64_t timeout_ns, int32_t *__restrict__ status,
                          int32_t *__restrict__ tok_pending, int32_t *__restrict__ ready,
                          int32_t arrivals, const int32_t *__restrict__ pool_row, int32_t T) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *zeros = sm + kTileBufs * row_bytes;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + (kTileBufs + 1) * row_bytes);
  int *never = reinterpret_cast<int *>(bar + kTileBufs);
  const int lane = threadIdx.x;
  for (uint32_t i = lane * 16; i < row_bytes; i += 32 * 16)
    *reinterpret_cast<uint4 *>(zeros + i) = make_uint4(0u, 0u, 0u, 0u);
  if (lane == 0) {
    for (int b = 0; b < kTileBufs; ++b) mbar_init(bar + b, 1);
    *never = 0;
    fence_mbarrier_init();
  }
  fence_proxy_async_shared();
  __syncwarp();

  // early combine: the token-major part (counts, tokens without a live pair) is small and
  // independent of the tiles: spread over the same blocks
  if (tok_pending != nullptr) {
    for (int64_t t = (int64_t)blockIdx.x * 32 + lane; t < T; t += (int64_t)gridDim.x * 32) {
      int live = 0;
      for (int j = 0; j < k; ++j) live += pool_row[t * k + j] >= 0 ? 1 : 0;
      tok_pending[t] = live * arrivals;
      if (live == 0) {
        const int32_t pos = atomicAdd(ready + T + 1, 1);
        if (pos < T) st_release_gpu(ready + pos, (int32_t)t + 1);
      }
    }
  }

  const int32_t n_tiles = meta[0];
  uint32_t uses[kTileBufs] = {};  // loads issued into each buffer (lane 0)
  bool failed = false;
  for (int32_t ti = blockIdx.x; ti < n_tiles && !failed; ti += gridDim.x) {
    const int32_t p0 = ti * tile;
    if (lane == 0) {
      // rows p0 + r; row r uses buffer r % kTileBufs; loads issued up to kTileBufs - 1 ahead
      int32_t issued = 0;
      auto issue = [&](int32_t r) {
        const int32_t src = row_src[p0 + r];
        if (src < 0) return;
        const int b = r % kTileBufs;
        mbar_arrive_expect_tx(bar + b, row_bytes);
        bulk_load_row(sm + b * row_bytes, x + (size_t)(src / k) * row_bytes, row_bytes, bar + b);
        ++uses[b];
      };
      for (; issued < kTileBufs - 1 && issued < tile; ++issued) issue(issued);
      for (int32_t r = 0; r < tile; ++r) {
        const int32_t src = row_src[p0 + r];
        const int b = r % kTileBufs;
        if (src >= 0) {
          if (!mbar_wait(bar + b, (uses[b] - 1u) & 1u, timeout_ns, never)) {
            report(status, MOE_ERR_PIPE_TIMEOUT, p0 + r);
            failed = true;
            break;
          }
          bulk_store_row(pool + (size_t)(p0 + r) * row_bytes, sm + b * row_bytes, row_bytes);
        } else {
          bulk_store_row(pool + (size_t)(p0 + r) * row_bytes, zeros, row_bytes);
        }
        bulk_commit();
        if (issued < tile) {
          // the buffer of row `issued` was last read by the store of row issued - kTileBufs
          // = r - 1, the group committed just before row r's
          bulk_wait_read<1>();
          issue(issued);
          ++issued;
        }
      }
      bulk_wait_all();
      if (!failed) {
        fence_proxy_async_global();
        red_release_gpu_add(flags + ti, (uint32_t)tile);
      }
    }
    failed = __shfl_sync(0xffffffffu, failed ? 1 : 0, 0) != 0;
  }
  if (lane == 0) {
    // loads issued for rows whose stores never came (after a failure) land before exit
    for (int b = 0; b < kTileBufs; ++b)
      if (uses[b] > 0) mbar_wait(bar + b, (uses[b] - 1u) & 1u, timeout_ns, never);
    bulk_wait_all();
  }
}

cudaError_t launch_dispatch(const moe_shape &s, const void *x, const moe_plan_buffers &p,
                            void *pool, int flags, int num_sms, cudaStream_t st) {
  const int signal = (flags & MOE_DISPATCH_SIGNAL_TILES) ? 1 : 0;
  const bool arm = (flags & MOE_DISPATCH_ARM_COMBINE) != 0;
  const uint32_t row_bytes = (uint32_t)s.H * 2;
  const size_t smem = dispatch_smem_bytes(s.H);
  if (smem > kMaxSmemPerBlock) return cudaErrorInvalidValue;  // refused by check_shape first
  // the kernel's shared-memory limit only grows, under a lock (host threads may launch
  // on the same device at once)
  static std::mutex mu;
  static size_t attr_smem[64] = {0};
  static size_t attr_smem_tiles[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // streaming: tiles in GEMM order, on the SMs the streaming FFN leaves free, when its
  // staging rows fit (else the token-order kernel, which raises the same flags)
  const size_t smem_tiles =
      (kTileBufs + 1) * (size_t)row_bytes + kTileBufs * sizeof(uint64_t) + 16;
  const bool tiles = signal && smem_tiles <= kMaxSmemPerBlock;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!tiles && attr_smem[dev] < smem) {
      cudaError_t e = cudaFuncSetAttribute(
          dispatch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr_smem[dev] = smem;
    }
    if (tiles && attr_smem_tiles[dev] < smem_tiles) {
      cudaError_t e = cudaFuncSetAttribute(dispatch_tiles_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem_tiles);
      if (e != cudaSuccess) return e;
      attr_smem_tiles[dev] = smem_tiles;
    }
  }
  if (tiles) {
    const PlanGeom g = plan_geom(s);
    const int per_sm = (int)(200 * 1024 / smem_tiles) > 0 ? (int)(200 * 1024 / smem_tiles) : 1;
    int64_t grid = (int64_t)kStreamDispatchSMs * per_sm;
    if (grid > g.n_tiles) grid = g.n_tiles;
    if (grid < 1) grid = 1;
    dispatch_tiles_kernel<<<(int)grid, 32, smem_tiles, st>>>(
        static_cast<const uint8_t *>(x), p.row_src, p.meta, static_cast<uint8_t *>(pool),
        p.tile_flags, s.k, row_bytes, s.tile, 2000000000ull, p.status,
        arm ? p.tok_pending : nullptr, arm ? p.ready : nullptr, early_combine_arrivals(s.H),
        p.pool_row, s.T);
    return cudaGetLastError();
  }
  const int per_sm = (int)(200 * 1024 / smem) > 0 ? (int)(200 * 1024 / smem) : 1;
  const int64_t items = (int64_t)kPadPieces * s.E + s.T;
  int64_t grid = (int64_t)num_sms * (per_sm < 16 ? per_sm : 16);
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  dispatch_kernel<<<(int)grid, 32, smem, st>>>(
      static_cast<const uint8_t *>(x), p.pool_row, p.offsets, p.counts,
      static_cast<uint8_t *>(pool), p.tile_flags, s.T, s.k, s.E, row_bytes, s.tile, signal,
      2000000000ull, p.status, arm ? p.tok_pending : nullptr, arm ? p.ready : nullptr,
      early_combine_arrivals(s.H));
  return cudaGetLastError();
}

}  // namespace moe
