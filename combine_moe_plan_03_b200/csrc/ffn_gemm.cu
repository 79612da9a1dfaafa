// Grouped SwiGLU FFN over the expert-major pool (StreamEP README, How it works,
// "CuTeDSL compute kernels": the forward grouped GEMMs A and Y), written for
// sm_100a tensor cores:
//   GEMM A: act[p, n]   = bf16( silu(pool[p] . W1[e][:, n]) * (pool[p] . W1[e][:, I + n]) )
//   GEMM Y: ypool[p, m] = bf16( act[p] . W2[e][:, m] )
// for the rows p of each 128-row block of expert e (the plan's row-block table).
//
// One persistent kernel per GEMM, one CTA per SM, 6 warps:
//   warp 0      TMA producer: per k-step, one 128x64 A box (K-major, 128-byte
//               swizzle) and N/64 B boxes of 64(k) x 64(n) (the weights stay in
//               their [K, N] layout: an MN-major operand) into a 4-stage ring.
//               In streaming mode it first waits (bounded, acquire) until the
//               tile flags of the block's pool rows are full.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=256 or 128, K=16; bf16 in, fp32 accumulate) into one of
//               two 256-column TMEM accumulators and commits the stage back to
//               the producer and the finished accumulator to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)...), SwiGLU (GEMM A) or plain conversion (GEMM Y), bf16
//               stores, then release the accumulator, so the epilogue of one
//               unit overlaps the main loop of the next.
// Work unit = (row block, N block); units are dealt round-robin over the CTAs,
// N block fastest, so the CTAs working at one time share the same A rows and the
// same expert's weights through L2.
//
// Every wait is bounded (global timer). The tile-flag wait, furthest upstream,
// gets the configured budget; the pipeline waits downstream of it get two (TMA
// producer, MMA) and three (epilogue) times as much, so the first wait to run
// out is the one that names the cause. A wait that runs out records
// MOE_ERR_PIPE_TIMEOUT / MOE_ERR_FLAG_TIMEOUT in the status word and raises a
// CTA-wide abort flag; the roles then leave their loops, the producer waits for
// the loads it has in flight, the MMA thread for its MMAs, and the TMEM is freed.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;        // 16 KB
constexpr int kChunkBytes = 64 * kBK * 2;     // 8 KB: 64 columns x 64 k-rows
constexpr int kBBytesMax = 4 * kChunkBytes;   // N <= 256
constexpr int kStageBytes = kABytes + kBBytesMax;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
constexpr int kThreads = 192;
constexpr int kBarrierBytes = 256;
constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;

struct FfnParams {
  const int32_t *mblk;     // row blocks {row_start, expert, rows}
  const int32_t *meta;     // meta[2] = number of row blocks
  const uint32_t *flags;   // pool tile flags (streaming)
  int32_t *status;
  uint16_t *out;           // act (GEMM A) or ypool (GEMM Y)
  int64_t out_ld;          // elements per row of out
  int32_t K;               // reduction length
  int32_t n_blocks;        // N blocks per row block
  int32_t bn;              // GEMM A: columns of act per block (gate and up each); GEMM Y: N
  int32_t k_rows;          // rows per expert in the B tensor map (H for W1, I for W2)
  int32_t up_col;          // GEMM A: first up column of W1 (= I)
  int32_t tile;            // pool tile rows
  int32_t streaming;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void raise_abort(volatile int *abort, int32_t *status, int32_t code,
                                            int32_t aux) {
  if (!*abort) report(status, code, aux);
  *abort = 1;
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b, const FfnParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *never = abort_flag + 1;  // stays 0: waits that must not be cut short by an abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = abort_flag;

  const int64_t n_units = (int64_t)prm.meta[2] * prm.n_blocks;
  const int mma_n = kMode == 0 ? 2 * prm.bn : prm.bn;
  const int n_chunks = mma_n / 64;
  const uint32_t stage_tx = (uint32_t)(kABytes + n_chunks * kChunkBytes);
  const int kb_count = prm.K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0, last_parity = 0;  // per stage: ever issued, parity of last issue
      for (int64_t u = blockIdx.x; u < n_units && !*abort; u += gridDim.x) {
        const int mb = (int)(u / prm.n_blocks);
        const int nb = (int)(u % prm.n_blocks);
        const int32_t row0 = prm.mblk[3 * mb + 0];
        const int32_t e = prm.mblk[3 * mb + 1];
        const int32_t rows = prm.mblk[3 * mb + 2];
        if (kMode == 0 && prm.streaming) {
          const int32_t t_end = (row0 + rows - 1) / prm.tile;
          for (int32_t t = row0 / prm.tile; t <= t_end && !*abort; ++t) {
            const uint64_t t0 = globaltimer_ns();
            uint32_t it = 0;
            while (ld_acquire_gpu(prm.flags + t) < (uint32_t)prm.tile) {
              if ((++it & 63u) == 0 && (*abort || globaltimer_ns() - t0 > prm.timeout_ns)) {
                raise_abort(abort, prm.status, MOE_ERR_FLAG_TIMEOUT, t);
                break;
              }
            }
          }
          fence_proxy_async_global();
          if (*abort) break;
        }
        const int32_t brow = e * prm.k_rows;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
            break;
          }
          uint8_t *sa = smem + stage * kStageBytes;
          uint8_t *sb = sa + kABytes;
          mbar_arrive_expect_tx(full + stage, stage_tx);
          tma_load_2d(sa, &tm_a, full + stage, kb * kBK, row0);
          const int32_t krow = brow + kb * kBK;
          if (kMode == 0) {
            const int half = n_chunks / 2;
            for (int c = 0; c < half; ++c)
              tma_load_2d(sb + c * kChunkBytes, &tm_b, full + stage, nb * prm.bn + c * 64, krow);
            for (int c = 0; c < half; ++c)
              tma_load_2d(sb + (half + c) * kChunkBytes, &tm_b, full + stage,
                          prm.up_col + nb * prm.bn + c * 64, krow);
          } else {
            for (int c = 0; c < n_chunks; ++c)
              tma_load_2d(sb + c * kChunkBytes, &tm_b, full + stage, nb * prm.bn + c * 64, krow);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort) {
        // Loads already issued land on their own; wait for them before the CTA exits.
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s))
            mbar_wait(full + s, (last_parity >> s) & 1u, prm.timeout_ns, never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kBM, (uint32_t)mma_n, true);
      uint32_t stage = 0, phase = 0, local = 0;
      for (int64_t u = blockIdx.x; u < n_units && !*abort; u += gridDim.x, ++local) {
        const uint32_t b = local & 1u;
        const uint32_t acc_phase = (local >> 1) & 1u;
        if (!mbar_wait(acc_empty + b, acc_phase ^ 1u, 2 * prm.timeout_ns, abort)) {
          raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kAccStride;
        bool ok = true;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(full + stage, phase, 2 * prm.timeout_ns, abort)) {
            raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major, 128-byte rows, 8-row groups 1024 B apart; +32 B per 16 k.
            const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
            // B: MN-major, 64-column chunks kChunkBytes apart, 8 k-rows per 1024 B; +2048 B per 16 k.
            const uint64_t bdesc = smem_desc_sw128(sb + kk * 2048, kChunkBytes, 1024);
            tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty + stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full + b);
      }
      // Wait for every MMA issued by this thread before the TMEM is released.
      tc_commit(drain);
      mbar_wait(drain, 0, prm.timeout_ns, never);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // accumulator row = TMEM lane
    uint32_t local = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
      const int mb = (int)(u / prm.n_blocks);
      const int nb = (int)(u % prm.n_blocks);
      const int32_t row0 = prm.mblk[3 * mb + 0];
      const int32_t rows = prm.mblk[3 * mb + 2];
      const uint32_t b = local & 1u;
      const uint32_t acc_phase = (local >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full + b, acc_phase, 3 * prm.timeout_ns, abort) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + b * kAccStride;
      const bool row_ok = r < rows;
      uint16_t *orow = prm.out + (size_t)(row0 + r) * prm.out_ld + (size_t)nb * prm.bn;
      if (kMode == 0) {
        for (int c = 0; c < prm.bn; c += 32) {
          uint32_t g[32], v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(taddr + c, g);
          tmem_ld_32x32b_x32(taddr + prm.bn + c, v);
          tmem_ld_wait();
          if (row_ok) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(v[2 * i]), u1 = __uint_as_float(v[2 * i + 1]);
              const float a0 = g0 / (1.0f + __expf(-g0)) * u0;
              const float a1 = g1 / (1.0f + __expf(-g1)) * u1;
              pk[i] = pack_bf16x2(a0, a1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else {
        for (int c = 0; c < prm.bn; c += 32) {
          uint32_t y[32];
          __syncwarp();
          tmem_ld_32x32b_x32(taddr + c, y);
          tmem_ld_wait();
          if (row_ok) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1]));
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + b);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- host side -------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [outer, inner] viewed as a 2-D tensor; box {64, box_outer},
// 128-byte swizzle (the canonical layout tcgen05 descriptors read).
static bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                      uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int kMode>
static cudaError_t launch_one(const CUtensorMap &ta, const CUtensorMap &tb, const FfnParams &prm,
                              int grid, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ffn_gemm_kernel<kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  ffn_gemm_kernel<kMode><<<grid, kThreads, kSmemBytes, st>>>(ta, tb, prm);
  return cudaGetLastError();
}

int launch_ffn(const moe_shape &s, const void *pool, const void *W1, const void *W2,
               const moe_plan_buffers &p, void *act, void *ypool, const moe_config &cfg,
               int num_sms, cudaStream_t st) {
  const PlanGeom g = plan_geom(s);
  if (g.pmax == 0) return MOE_OK;
  CUtensorMap ta_pool, tb_w1, ta_act, tb_w2;
  if (!make_tmap(&ta_pool, pool, (uint64_t)s.H, (uint64_t)g.pmax, kBM) ||
      !make_tmap(&tb_w1, W1, 2ull * s.I, (uint64_t)s.E * s.H, kBK) ||
      !make_tmap(&ta_act, act, (uint64_t)s.I, (uint64_t)g.pmax, kBM) ||
      !make_tmap(&tb_w2, W2, (uint64_t)s.H, (uint64_t)s.E * s.I, kBK))
    return MOE_ERR_CUDA;

  int grid = cfg.ffn_ctas > 0 ? cfg.ffn_ctas : (cfg.streaming ? num_sms - 16 : num_sms);
  if (grid < 1) grid = 1;
  const uint64_t timeout_ns =
      (uint64_t)(cfg.wait_timeout_us > 0 ? cfg.wait_timeout_us : 2000000) * 1000ull;

  FfnParams a{};
  a.mblk = p.mblk;
  a.meta = p.meta;
  a.flags = p.tile_flags;
  a.status = p.status;
  a.out = static_cast<uint16_t *>(act);
  a.out_ld = s.I;
  a.K = s.H;
  a.bn = (s.I % 128 == 0) ? 128 : 64;
  a.n_blocks = s.I / a.bn;
  a.k_rows = s.H;
  a.up_col = s.I;
  a.tile = s.tile;
  a.streaming = cfg.streaming;
  a.timeout_ns = timeout_ns;
  cudaEvent_t const *tev = reinterpret_cast<cudaEvent_t const *>(cfg.timing_events);
  if (tev != nullptr && cudaEventRecord(tev[3], st) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = launch_one<0>(ta_pool, tb_w1, a, grid, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[4], st) != cudaSuccess) return MOE_ERR_CUDA;

  FfnParams y = a;
  y.out = static_cast<uint16_t *>(ypool);
  y.out_ld = s.H;
  y.K = s.I;
  y.bn = (s.H % 256 == 0) ? 256 : ((s.H % 128 == 0) ? 128 : 64);
  y.n_blocks = s.H / y.bn;
  y.k_rows = s.I;
  y.up_col = 0;
  y.streaming = 0;
  e = launch_one<1>(ta_act, tb_w2, y, cfg.ffn_ctas > 0 ? cfg.ffn_ctas : num_sms, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[5], st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
