// Grouped SwiGLU FFN over the expert-major pool (StreamEP README, How it works,
// "CuTeDSL compute kernels": the forward grouped GEMMs A and Y), written for
// sm_100a tensor cores. This file holds the one-CTA-per-unit kernel (MOE_FFN_ONE_SM),
// the host side of both grouped-GEMM kernels (tensor maps, unit geometry, launches of
// the forward and of the backward's GEMMs) and the TMA tensor-map helpers; the SM-pair
// kernel, the default, is in ffn_gemm_pair.cu.
//   GEMM A: act[p, n]   = bf16( silu(pool[p] . W1[e][:, n]) * (pool[p] . W1[e][:, I + n]) )
//   GEMM Y: ypool[p, m] = bf16( act[p] . W2[e][:, m] )
// for the live rows p of expert e (pool rows past an expert's count are padding and
// are not computed; combine never reads them).
//
// Orientation: the weights are the MMA's M operand and the pool rows its N operand
// (D^T = W^T X^T). A work unit is (row chunk of one expert: up to 256 live rows,
// block of weight columns). Its N is the chunk's live rows rounded up to 16, so the
// tile padding of the pool costs (almost) no tensor work, and a chunk of 256 rows
// uses each weight tile it loads 256 times. Each unit has two 128-row weight tiles
// and two TMEM accumulators (128 lanes x N columns each):
//   GEMM A: tile 0 = 128 gate columns, tile 1 = the same 128 up columns, so lane f
//           of the epilogue holds gate and up of output column f for every row;
//   GEMM Y: tiles 0 and 1 = two adjacent blocks of 128 output columns.
//
// One persistent kernel per GEMM, one CTA per SM, 10 warps:
//   warp 0      TMA producer: per k-step two weight tiles of 128 columns x 64 k
//               (two 64x64 boxes each; weights stay in their [K, N] layout, read as
//               an MN-major operand, 128-byte swizzle) and ceil(N/32) boxes of
//               32 pool rows x 64 k (K-major, 128-byte swizzle), into a 3-stage
//               ring of 64 KB stages. In streaming mode it first waits (bounded,
//               acquire) until the tile flags of the chunk's pool rows are full.
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N<=256, K=16; bf16 in, fp32 accumulate), two per 16 k (one
//               per accumulator), commits each stage back to the producer and the
//               finished unit to the epilogue.
//   warps 2-9   epilogue: two warps per TMEM lane quadrant (warp w reads lanes
//               32*(w%4)... and every other group of 32 pool rows), tcgen05.ld,
//               SwiGLU (GEMM A) or conversion (GEMM Y) to bf16, a 32x32 turn in
//               shared memory, and 16-byte stores along the output rows.
// With prepacked weights (moe_pack_weights) each weight tile is one contiguous 16 KB
// box, so a unit streams contiguous HBM.
// Units are handed out in order (row chunk, then weight block) from a global ticket
// counter as CTAs free up, so the CTAs working at one time share the same pool rows
// and the same expert's weights through L2, and uneven units balance out. The
// producer takes the ticket and passes the unit id to the MMA thread and the
// epilogue through a 4-slot ring in shared memory.
//
// Every wait is bounded (global timer). The tile-flag wait, furthest upstream,
// gets the configured budget; the pipeline waits downstream of it get two (TMA
// producer, MMA) and three (epilogue) times as much, so the first wait to run
// out is the one that names the cause. A wait that runs out records
// MOE_ERR_PIPE_TIMEOUT / MOE_ERR_FLAG_TIMEOUT in the status word and raises a
// CTA-wide abort flag; the roles then leave their loops, the producer waits for
// the loads it has in flight, the MMA thread for its MMAs, and the TMEM is freed.
#include <mutex>
#include "ffn_gemm.cuh"

namespace moe {

constexpr int kBM = 128;                              // weight columns per tile (MMA M)
constexpr int kBK = 64;                               // k per stage
constexpr int kMaxN = kGemmBlockM;                    // pool rows per unit (MMA N <= 256)
constexpr int kStages = 3;
constexpr int kChunkBytes = 64 * kBK * 2;             // 8 KB: 64 weight columns x 64 k
constexpr int kWTileBytes = 2 * kChunkBytes;          // 16 KB: one 128-column weight tile
constexpr int kRowBox = 32;                           // pool rows per TMA box
constexpr int kRowBoxBytes = kRowBox * kBK * 2;       // 4 KB
constexpr int kStageBytes = 2 * kWTileBytes + kMaxN * kBK * 2;  // 64 KB
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr int kSchedSlots = 4;                        // unit ids in flight inside a CTA
constexpr int kBarrierBytes = 256;
constexpr int kXposeBytes = 32 * 32 * 2;              // per epilogue warp: 32 rows x 32 columns bf16
constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kEpiWarps * kXposeBytes + 1024;

__device__ __forceinline__ void raise_abort(volatile int *abort, int32_t *status, int32_t code,
                                            int32_t aux) {
  if (!*abort) report(status, code, aux);
  *abort = 1;
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_x, const FfnParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;  // the unit's accumulators are complete
  uint64_t *acc_empty = acc_full + 1;    // the epilogue has read them
  uint64_t *drain = acc_empty + 1;
  uint64_t *sched_full = drain + 1;          // [kSchedSlots] a unit id was written
  uint64_t *sched_empty = sched_full + kSchedSlots;  // [kSchedSlots] MMA + epilogue read it
  int32_t *sched = reinterpret_cast<int32_t *>(sched_empty + kSchedSlots);  // unit ids, -1 = end
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sched + kSchedSlots);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *never = abort_flag + 1;  // stays 0: waits that must not be cut short by an abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps * 32);
    mbar_init(drain, 1);
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(sched_full + i, 1);
      mbar_init(sched_empty + i, 1 + kEpiWarps);
    }
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
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

  const int32_t n_units = prm.meta[2] * prm.n_blocks;
  const int kb_count = prm.K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0, last_parity = 0;  // per stage: ever issued, parity of last issue
      uint32_t sslot = 0, sphase = 0;
      for (;;) {
        // take the next unit (tickets are handed out in unit order) and publish it
        if (!mbar_wait(sched_empty + sslot, sphase ^ 1u, 2 * prm.timeout_ns, abort)) {
          raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
          break;
        }
        const int32_t ticket = atomicAdd(prm.sched + 0, 1);
        const int64_t u = (ticket < n_units && !*abort) ? ticket : -1;
        sched[sslot] = (int32_t)u;
        mbar_arrive(sched_full + sslot);
        if (++sslot == kSchedSlots) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (u < 0) break;
        int32_t mb, nb;
        unit_coords(prm.mblk, u, prm.n_blocks, mb, nb);
        const int32_t row0 = prm.mblk[kMblkInts * mb + 0];
        const int32_t e = prm.mblk[kMblkInts * mb + 1];
        const int32_t rows = prm.mblk[kMblkInts * mb + 2];
        const int nbox = (rows + kRowBox - 1) / kRowBox;
        if (kMode == 0 && prm.streaming) {
          const int32_t t_end = (row0 + rows - 1) / prm.tile;
          for (int32_t t = row0 / prm.tile; t <= t_end && !*abort; ++t) {
            const uint64_t t0 = globaltimer_ns();
            uint32_t it = 0;
            while (ld_acquire_sys(prm.flags + t) < (uint32_t)prm.tile) {
              if ((++it & 63u) == 0 && (*abort || globaltimer_ns() - t0 > prm.timeout_ns)) {
                raise_abort(abort, prm.status, MOE_ERR_FLAG_TIMEOUT, t);
                break;
              }
            }
          }
          fence_proxy_async_global();
          if (*abort) break;
        }
        const int32_t wcol0 = nb * prm.col_step;
        const int32_t wcol1 = wcol0 + prm.col1_off;
        const uint32_t tx = (uint32_t)(2 * kWTileBytes + nbox * kRowBoxBytes);
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
            break;
          }
          uint8_t *sw0 = smem + stage * kStageBytes;
          uint8_t *sw1 = sw0 + kWTileBytes;
          uint8_t *sx = sw0 + 2 * kWTileBytes;
          const int32_t krow = e * prm.k_rows + kb * kBK;
          mbar_arrive_expect_tx(full + stage, tx);
          if (prm.packed) {
            const int32_t t0 = e * prm.pk_e + nb * prm.pk_nb + kb;
            tma_load_2d(sw0, &tm_w, full + stage, 0, t0 * 128);
            tma_load_2d(sw1, &tm_w, full + stage, 0, (t0 + prm.pk_j) * 128);
          } else {
            tma_load_2d(sw0, &tm_w, full + stage, wcol0, krow);
            tma_load_2d(sw0 + kChunkBytes, &tm_w, full + stage, wcol0 + 64, krow);
            tma_load_2d(sw1, &tm_w, full + stage, wcol1, krow);
            tma_load_2d(sw1 + kChunkBytes, &tm_w, full + stage, wcol1 + 64, krow);
          }
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(sx + i * kRowBoxBytes, &tm_x, full + stage, kb * kBK, row0 + i * kRowBox);
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
      // Every CTA has taken its last ticket (the end ticket, or the one before an abort)
      // before it counts itself done, so the last one may zero the counters for the next
      // launch, on the abort path too.
      __threadfence();
      const int group = prm.sched_group > 0 ? prm.sched_group : (int)gridDim.x;
      if (atomicAdd(prm.sched + 1, 1) == group - 1) {
        atomicExch(prm.sched + 0, 0);
        atomicExch(prm.sched + 1, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0, local = 0;
      uint32_t sslot = 0, sphase = 0;
      bool ok = true;
      for (;; ++local) {
        if (!mbar_wait(sched_full + sslot, sphase, 2 * prm.timeout_ns, abort)) {
          raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
          break;
        }
        const int32_t u = sched[sslot];
        mbar_arrive(sched_empty + sslot);
        if (++sslot == kSchedSlots) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (u < 0) break;
        int32_t mb, nb;
        unit_coords(prm.mblk, u, prm.n_blocks, mb, nb);
        const int32_t rows = prm.mblk[kMblkInts * mb + 2];
        const uint32_t n_mma = (uint32_t)((rows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32_ab(kBM, n_mma, /*a_mn=*/true, /*b_mn=*/false);
        // The accumulators may be overwritten once the epilogue read the previous unit
        // (parity of the previous unit; a fresh barrier passes parity 1).
        if (!mbar_wait(acc_empty, (local + 1u) & 1u, 2 * prm.timeout_ns, abort)) {
          raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(full + stage, phase, 2 * prm.timeout_ns, abort)) {
            raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sw0 = smem_u32(smem + stage * kStageBytes);
          const uint32_t sw1 = sw0 + kWTileBytes;
          const uint32_t sx = sw0 + 2 * kWTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // weights: MN-major, 64-column chunks kChunkBytes apart, 8 k-rows per 1024 B;
            // +2048 B per 16 k. Pool rows: K-major, 128-byte rows, 8-row groups 1024 B
            // apart; +32 B per 16 k.
            const uint64_t xdesc = smem_desc_sw128(sx + kk * 32, 16, 1024);
            const uint64_t w0 = smem_desc_sw128(sw0 + kk * 2048, kChunkBytes, 1024);
            const uint64_t w1 = smem_desc_sw128(sw1 + kk * 2048, kChunkBytes, 1024);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_bf16(tmem_base, w0, xdesc, idesc, acc);
            tc_mma_bf16(tmem_base + kAccStride, w1, xdesc, idesc, acc);
          }
          tc_commit(empty + stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      // Wait for every MMA issued by this thread before the TMEM is released.
      tc_commit(drain);
      mbar_wait(drain, 0, prm.timeout_ns, never);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Lane f of a warp holds output column f of its 32-column group for 32 pool rows
    // at a time; the warp turns that 32x32 block around in shared memory so that
    // every global store writes 16 contiguous bytes of one pool row.
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = (warp - 2) >> 2;          // which 32-row groups it takes
    const uint32_t tq = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint16_t *xp = reinterpret_cast<uint16_t *>(smem + kStages * kStageBytes + kBarrierBytes) +
                   (warp - 2) * (kXposeBytes / 2);
    uint32_t local = 0;
    uint32_t sslot = 0, sphase = 0;
    for (;; ++local) {
      int32_t u = -1;
      int got = 1;
      if (lane == 0) {
        got = mbar_wait_sleepy(sched_full + sslot, sphase, 3 * prm.timeout_ns, abort, 1024) ? 1 : 0;
        if (got) {
          u = sched[sslot];
          mbar_arrive(sched_empty + sslot);
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (++sslot == kSchedSlots) {
        sslot = 0;
        sphase ^= 1u;
      }
      if (!got) {
        if (lane == 0) raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
        break;
      }
      if (u < 0) break;
      int32_t mb, nb;
      unit_coords(prm.mblk, u, prm.n_blocks, mb, nb);
      const int32_t row0 = prm.mblk[kMblkInts * mb + 0];
      const int32_t rows = prm.mblk[kMblkInts * mb + 2];
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_sleepy(acc_full, local & 1u, 3 * prm.timeout_ns, abort, 1024) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort(abort, prm.status, MOE_ERR_PIPE_TIMEOUT, (int32_t)u);
        break;
      }
      tc_fence_after();
      // first output column of this warp's group for accumulator 0 / 1
      const int32_t cb0 = nb * prm.col_step + quad * 32;
      const int32_t cb1 = cb0 + prm.col1_off;
      const bool ok0 = cb0 < prm.n_out;
      const bool ok1 = kMode == 1 && cb1 < prm.n_out;
      for (int c = half * 32; c < rows; c += 64) {
        uint32_t a0[32], a1[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tq + c, a0);
        tmem_ld_32x32b_x32(tq + kAccStride + c, a1);
        tmem_ld_wait();
        const int lim = min(32, rows - c);
        for (int j = 0; j < (kMode == 0 ? 1 : 2); ++j) {
          if (!(j == 0 ? ok0 : ok1)) continue;  // uniform across the warp
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float v = kMode == 0
                                ? silu_mul(__uint_as_float(a0[i]), __uint_as_float(a1[i]))
                                : __uint_as_float(j == 0 ? a0[i] : a1[i]);
            xp[i * 32 + lane] = bf16_bits(v);
          }
          __syncwarp();
          const int32_t cb = j == 0 ? cb0 : cb1;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int v = lane + 32 * q;
            const int r = v >> 2;         // pool row inside the 32-row group
            const int part = v & 3;       // 8-column part of the 32 columns
            if (r < lim) {
              const uint4 val = *reinterpret_cast<const uint4 *>(xp + r * 32 + part * 8);
              *reinterpret_cast<uint4 *>(prm.out + (size_t)(row0 + c + r) * prm.out_ld + cb +
                                         part * 8) = val;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
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
  // looked up once (a function-local static is initialised once, thread-safely)
  static const EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

bool make_tmap_box(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, uint32_t swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                   : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                         : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
               uint32_t box_outer) {
  return make_tmap_box(m, base, inner, outer, 64, box_outer, 128);
}

template <int kMode>
static cudaError_t launch_one(const CUtensorMap &tw, const CUtensorMap &tx, const FfnParams &prm,
                              int grid, cudaStream_t st) {
  static bool attr_set[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::unique_lock<std::mutex> lock(mu);
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(ffn_gemm_kernel<kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  lock.unlock();
  ffn_gemm_kernel<kMode><<<grid, kThreads, kSmemBytes, st>>>(tw, tx, prm);
  return cudaGetLastError();
}

int launch_ffn(const moe_shape &s, const void *pool, const void *W1, const void *W2,
               const moe_plan_buffers &p, void *act, void *ypool, const float *topk_w,
               void *out, const moe_config &cfg, int num_sms, cudaStream_t st,
               cudaStream_t helper_stream, cudaEvent_t helper_done) {
  const bool early = cfg.early_combine != 0;
  // streaming with a helper stream: GEMM A runs on the SMs dispatch leaves free, and a second
  // launch of it, queued on the helper stream behind dispatch, takes the remaining SMs'
  // share of the same unit tickets once dispatch is done
  const bool helper = cfg.streaming && helper_stream != nullptr && helper_done != nullptr &&
                      cfg.ffn_ctas == 0;
  const PlanGeom g = plan_geom(s);
  if (g.pmax == 0) return MOE_OK;
  CUtensorMap tw1, tx_pool, tw2, tx_act;
  const PackGeom pg = pack_geom(s);
  bool ok;
  if (cfg.packed_weights) {
    // packed tiles: an array of 128-byte rows, one 128-row box per tile
    ok = make_tmap(&tw1, W1, 64, (uint64_t)pg.tiles1 * 128, 128) &&
         make_tmap(&tw2, W2, 64, (uint64_t)pg.tiles2 * 128, 128);
  } else {
    ok = make_tmap(&tw1, W1, 2ull * s.I, (uint64_t)s.E * s.H, kBK) &&
         make_tmap(&tw2, W2, (uint64_t)s.H, (uint64_t)s.E * s.I, kBK);
  }
  if (!ok || !make_tmap(&tx_pool, pool, (uint64_t)s.H, (uint64_t)g.pmax, kRowBox) ||
      !make_tmap(&tx_act, act, (uint64_t)s.I, (uint64_t)g.pmax, kRowBox))
    return MOE_ERR_CUDA;

  const bool pair = (cfg.ffn_kernel != 0 ? cfg.ffn_kernel : MOE_FFN_DEFAULT) == MOE_FFN_SM_PAIR;
  int grid = cfg.ffn_ctas > 0 ? cfg.ffn_ctas
                              : (cfg.streaming ? num_sms - kStreamDispatchSMs : num_sms);
  if (grid < 1) grid = 1;
  int grid_y = cfg.ffn_ctas > 0 ? cfg.ffn_ctas : num_sms;
  int grid_helper = helper ? num_sms - grid : 0;  // CTAs of the helper launch
  if (pair) {
    // clusters of two CTAs: as many as fit at once, at most half the requested CTAs
    const int fit0 = ffn_pair_max_clusters(0), fit1 = ffn_pair_max_clusters(1);
    if (fit0 < 1 || fit1 < 1) return MOE_ERR_CUDA;
    grid = grid / 2 < 1 ? 1 : (grid / 2 < fit0 ? grid / 2 : fit0);
    grid_y = grid_y / 2 < 1 ? 1 : (grid_y / 2 < fit1 ? grid_y / 2 : fit1);
    grid_helper = helper ? (fit0 - grid > 0 ? fit0 - grid : 0) : 0;
  }
  const bool use_helper = helper && grid_helper > 0;
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
  a.col_step = kBM;                       // 128 gate columns and the same 128 up columns
  a.col1_off = s.I;
  a.n_blocks = (s.I + kBM - 1) / kBM;
  a.n_out = s.I;
  a.n_out1 = s.I;
  a.k_rows = s.H;
  a.tile = s.tile;
  a.streaming = cfg.streaming;
  a.sched = p.meta + 4;
  a.packed = cfg.packed_weights ? 1 : 0;
  a.pk_e = 2 * pg.nb1 * pg.kb1;           // gate tiles of expert e, then its up tiles
  a.pk_j = pg.nb1 * pg.kb1;
  a.pk_nb = pg.kb1;
  a.pk_v = 0;
  if (pair) {                             // 256 gate and 256 up columns per unit
    a.col_step = 2 * kBM;
    a.n_blocks = (s.I + 2 * kBM - 1) / (2 * kBM);
    a.pk_nb = 2 * pg.kb1;
    a.pk_v = pg.kb1;
  }
  a.timeout_ns = timeout_ns;
  cudaEvent_t const *tev = reinterpret_cast<cudaEvent_t const *>(cfg.timing_events);
  if (tev != nullptr && cudaEventRecord(tev[3], st) != cudaSuccess) return MOE_ERR_CUDA;
  int a_mode = 0;
  if (cfg.gate_up != nullptr) {           // training step: also keep g | u for the backward
    a_mode = 3;
    a.out = static_cast<uint16_t *>(cfg.gate_up);
    a.out_ld = 2 * s.I;
    a.n_out1 = 2 * s.I;
    a.out2 = static_cast<uint16_t *>(act);
    a.out2_ld = s.I;
  }
  if (use_helper) a.sched_group = grid + grid_helper;  // both launches count themselves done
  cudaError_t e = pair ? launch_ffn_pair(a_mode, false, tw1, tx_pool, a, grid, st)
                       : launch_one<0>(tw1, tx_pool, a, grid, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (use_helper) {
    e = pair ? launch_ffn_pair(a_mode, false, tw1, tx_pool, a, grid_helper, helper_stream)
             : launch_one<0>(tw1, tx_pool, a, grid_helper, helper_stream);
    if (e != cudaSuccess || cudaEventRecord(helper_done, helper_stream) != cudaSuccess ||
        cudaStreamWaitEvent(st, helper_done, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // early combine counts GEMM Y's row chunks in the tile flags (GEMM A, the only reader of
  // the flags, is done; there are no more chunks than tiles): zero them first
  if (early && cudaMemsetAsync(p.tile_flags, 0, sizeof(uint32_t) * (size_t)g.n_tiles, st) !=
                   cudaSuccess)
    return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[4], st) != cudaSuccess) return MOE_ERR_CUDA;

  FfnParams y = a;
  y.sched_group = 0;
  y.out = static_cast<uint16_t *>(ypool);
  y.out_ld = s.H;
  y.K = s.I;
  y.col_step = 2 * kBM;                   // two adjacent 128-column blocks of W2
  y.col1_off = kBM;
  y.n_blocks = (s.H + 2 * kBM - 1) / (2 * kBM);
  y.n_out = s.H;
  y.n_out1 = s.H;
  y.k_rows = s.I;
  y.streaming = 0;
  y.sched = p.meta + 6;
  y.pk_e = pg.nb2 * pg.kb2;               // 128-column blocks of expert e, k fastest
  y.pk_j = pg.kb2;
  y.pk_nb = 2 * pg.kb2;
  if (pair) {                             // two adjacent blocks of 256 columns per unit
    y.col_step = 4 * kBM;
    y.col1_off = 2 * kBM;
    y.n_blocks = (s.H + 4 * kBM - 1) / (4 * kBM);
    y.pk_j = 2 * pg.kb2;
    y.pk_nb = 4 * pg.kb2;
    y.pk_v = pg.kb2;
  }
  if (early) {
    // GEMM Y combines every token once its k rows are stored (fused early combine)
    y.row_src = p.row_src;
    y.pool_row = p.pool_row;
    y.topk_w = topk_w;
    y.chunk_cnt = reinterpret_cast<int32_t *>(p.tile_flags);
    y.tok_pending = p.tok_pending;
    y.ready = p.ready;
    y.comb_out = static_cast<uint16_t *>(out);
    y.T = s.T;
    y.k = s.k;
  }
  e = pair ? launch_ffn_pair(1, false, tw2, tx_act, y, grid_y, st, early)
           : launch_one<1>(tw2, tx_act, y, grid_y, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[5], st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// The backward's three grouped GEMMs on SM pairs (backward.cu has the order and the
// formulas): gate / up recompute (W1 read MN-major, as in GEMM A), backward Y (W2 read
// K-major, SwiGLU backward in the epilogue), backward A (W1 read K-major). dypool_dpool
// holds dypool on entry and dpool on return.
int launch_ffn_backward(const moe_shape &s, const void *W1, const void *W2,
                        const moe_plan_buffers &p, const void *pool, void *act,
                        void *dypool_dpool, void *gu, void *dgu, void *dW1, void *dW2,
                        const moe_config &cfg, int num_sms, cudaStream_t st,
                        cudaEvent_t const *tev, void *early_dx, cudaEvent_t combine_done) {
  const PlanGeom g = plan_geom(s);
  if (g.pmax == 0) {
    // no rows at all (T = 0): the weight gradients are zero, the phases empty
    if (dW1 != nullptr &&
        cudaMemsetAsync(dW1, 0, (size_t)s.E * s.H * 2 * s.I * sizeof(uint16_t), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (dW2 != nullptr &&
        cudaMemsetAsync(dW2, 0, (size_t)s.E * s.I * s.H * sizeof(uint16_t), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (int i = 2; tev != nullptr && i <= 6; ++i)
      if (cudaEventRecord(tev[i], st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  CUtensorMap tw1_mn, tw2_k, tw1_k, tx_pool, tx_dy, tx_dgu;
  if (!make_tmap(&tw1_mn, W1, 2ull * s.I, (uint64_t)s.E * s.H, kBK) ||
      !make_tmap(&tw2_k, W2, (uint64_t)s.H, (uint64_t)s.E * s.I, 128) ||
      !make_tmap(&tw1_k, W1, 2ull * s.I, (uint64_t)s.E * s.H, 128) ||
      !make_tmap(&tx_pool, pool, (uint64_t)s.H, (uint64_t)g.pmax, kRowBox) ||
      !make_tmap(&tx_dy, dypool_dpool, (uint64_t)s.H, (uint64_t)g.pmax, kRowBox) ||
      !make_tmap(&tx_dgu, dgu, 2ull * s.I, (uint64_t)g.pmax, kRowBox))
    return MOE_ERR_CUDA;
  const int fit = ffn_pair_max_clusters(0);
  if (fit < 1) return MOE_ERR_CUDA;
  int clusters = (cfg.ffn_ctas > 0 ? cfg.ffn_ctas : num_sms) / 2;
  if (clusters < 1) clusters = 1;
  if (clusters > fit) clusters = fit;
  const uint64_t timeout_ns =
      (uint64_t)(cfg.wait_timeout_us > 0 ? cfg.wait_timeout_us : 2000000) * 1000ull;

  FfnParams b{};
  b.mblk = p.mblk;
  b.meta = p.meta;
  b.flags = p.tile_flags;
  b.status = p.status;
  b.tile = s.tile;
  b.streaming = 0;
  b.packed = 0;
  b.timeout_ns = timeout_ns;
  b.col_step = 2 * kBM;

  // gate / up recompute: gu[p] = [pool[p] . W1g | pool[p] . W1u], unless the forward kept them
  if (cfg.gate_up != nullptr) gu = cfg.gate_up;
  FfnParams r = b;
  r.out = static_cast<uint16_t *>(gu);
  r.out_ld = 2 * s.I;
  r.K = s.H;
  r.col1_off = s.I;
  r.n_blocks = (s.I + 2 * kBM - 1) / (2 * kBM);
  r.n_out = s.I;
  r.n_out1 = 2 * s.I;
  r.k_rows = s.H;
  r.sched = p.meta + 4;
  if (cfg.gate_up == nullptr && launch_ffn_pair(1, false, tw1_mn, tx_pool, r, clusters, st) !=
                                    cudaSuccess)
    return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[2], st) != cudaSuccess) return MOE_ERR_CUDA;

  // backward Y: da = dypool . W2^T (two 256-column blocks of da), SwiGLU backward -> dgu
  FfnParams y = b;
  y.out = static_cast<uint16_t *>(dgu);
  y.out_ld = 2 * s.I;
  y.K = s.H;
  y.col_step = 4 * kBM;
  y.col1_off = 2 * kBM;
  y.n_blocks = (s.I + 4 * kBM - 1) / (4 * kBM);
  y.n_out = s.I;
  y.n_out1 = s.I;
  y.k_rows = s.I;
  y.sched = p.meta + 6;
  y.aux = static_cast<const uint16_t *>(gu);
  y.aux_ld = 2 * s.I;
  y.aux_off = s.I;
  // streaming: the combine backward fills dypool tile by tile on the SMs backward Y leaves
  // free and raises the tiles' flags; backward Y takes a chunk once the flags of its tiles
  // are full. (Whether other blocks can sit beside the GEMM's CTAs is not relied on: with
  // the GEMM on every SM the combine backward it waits for could not start.)
  y.streaming = cfg.streaming;
  int clusters_y = clusters;
  if (cfg.streaming) {
    clusters_y = (num_sms - kStreamDispatchSMs) / 2;
    if (clusters_y > clusters) clusters_y = clusters;
    if (clusters_y < 1) clusters_y = 1;
  }
  if (launch_ffn_pair(2, true, tw2_k, tx_dy, y, clusters_y, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (combine_done != nullptr && cudaStreamWaitEvent(st, combine_done, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[3], st) != cudaSuccess) return MOE_ERR_CUDA;

  // dW2 = act^T . dypool per expert (before backward A overwrites dypool)
  if (dW2 != nullptr) {
    if (launch_zero_pad_rows(s, act, s.I, p, num_sms, st) != cudaSuccess ||
        launch_zero_pad_rows(s, dypool_dpool, s.H, p, num_sms, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int rc = launch_wgrad(s, act, s.I, dypool_dpool, s.H, dW2, p, p.meta + 6, cfg, num_sms, st);
    if (rc != MOE_OK) return rc;
  }
  if (tev != nullptr && cudaEventRecord(tev[4], st) != cudaSuccess) return MOE_ERR_CUDA;

  // backward A: dpool = dgu . W1^T (two 256-column blocks of dpool)
  FfnParams a = b;
  a.out = static_cast<uint16_t *>(dypool_dpool);
  a.out_ld = s.H;
  a.K = 2 * s.I;
  a.col_step = 4 * kBM;
  a.col1_off = 2 * kBM;
  a.n_blocks = (s.H + 4 * kBM - 1) / (4 * kBM);
  a.n_out = s.H;
  a.n_out1 = s.H;
  a.k_rows = s.H;
  a.sched = p.meta + 4;
  const bool early = early_dx != nullptr;
  if (early) {
    // dx[t] = bf16(sum_j dpool[pool_row[t, j]]) for each token as soon as its rows are
    // stored (unit weights: no topk_w), in the CTAs that finished their GEMM work
    a.row_src = p.row_src;
    a.pool_row = p.pool_row;
    a.topk_w = nullptr;
    a.chunk_cnt = reinterpret_cast<int32_t *>(p.tile_flags);
    a.tok_pending = p.tok_pending;
    a.ready = p.ready;
    a.comb_out = static_cast<uint16_t *>(early_dx);
    a.T = s.T;
    a.k = s.k;
  }
  // its row-chunk counters live in the tile flags (backward Y, their only other reader, is
  // done): zero them first
  if (early && cudaMemsetAsync(p.tile_flags, 0, sizeof(uint32_t) * (size_t)g.n_tiles, st) !=
                   cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_ffn_pair(1, true, tw1_k, tx_dgu, a, clusters, st, early) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[5], st) != cudaSuccess) return MOE_ERR_CUDA;

  // dW1 = pool^T . dgu per expert (the pool's padding rows are zero already)
  if (dW1 != nullptr) {
    if (launch_zero_pad_rows(s, dgu, 2 * s.I, p, num_sms, st) != cudaSuccess) return MOE_ERR_CUDA;
    const int rc = launch_wgrad(s, pool, s.H, dgu, 2 * s.I, dW1, p, p.meta + 4, cfg, num_sms, st);
    if (rc != MOE_OK) return rc;
  }
  if (tev != nullptr && cudaEventRecord(tev[6], st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
