// Grouped SwiGLU FFN on SM pairs: the same two GEMMs as ffn_gemm.cu (StreamEP README,
// How it works, "CuTeDSL compute kernels": grouped GEMM A then grouped GEMM Y), with
// each work unit computed by a cluster of two CTAs on two SMs through tcgen05's
// cta_group::2 MMA (M = 256):
//   GEMM A: act[p, n]   = bf16( silu(pool[p] . W1[e][:, n]) * (pool[p] . W1[e][:, I + n]) )
//   GEMM Y: ypool[p, m] = bf16( act[p] . W2[e][:, m] )
// for the live rows p of expert e.
//
// A unit is (row chunk of one expert: up to 256 live rows, block of weight columns).
// Weights are the MMA's M operand, the chunk's rows its N operand (N = live rows rounded
// up to 16). Each CTA of the pair holds 128 of the 256 weight columns of each MMA and
// half of the N pool rows; each CTA's TMEM receives the accumulator rows of its own
// 128 weight columns for all N pool rows. Two accumulators per unit:
//   GEMM A: 256 gate columns and the same 256 up columns (block of 256 act columns;
//           CTA r writes act columns 128 r ... 128 r + 127 of the block);
//   GEMM Y: two adjacent blocks of 256 output columns (block of 512 columns).
// Against one CTA per unit this halves each SM's share of the pool-row loads (per
// k-step a CTA loads 32 KB of weights and at most 16 KB of pool rows instead of 32 +
// 32 KB), so the 4-stage ring fits where the one-CTA kernel has 3 stages.
//
// Roles (10 warps per CTA, one CTA per SM):
//   warp 0  TMA producer (both CTAs): its CTA's two weight tiles and its half of the
//           pool rows per k-step. The first CTA's producer takes the unit tickets,
//           writes each unit id into both CTAs' 4-slot rings, and sets the expected
//           bytes of both CTAs' loads on its own full barrier, which the loads of
//           both CTAs complete (cta_group::2 form of the TMA load).
//   warp 1  both CTAs allocate 512 TMEM columns (cta_group::2). In the first CTA one
//           thread issues the MMAs and commits each stage to the empty barriers of
//           both CTAs and each finished unit to both CTAs' accumulator barriers.
//   2-9     epilogue (both CTAs), as in the one-CTA kernel, over the CTA's own TMEM;
//           a warp reports the accumulators read on the first CTA's barrier.
//   10      early combine only (GEMM Y with the combine fused in): a signal warp. For each
//           unit it waits until the CTA's epilogue warps have stored the unit's rows, then
//           counts each row against its token (tok_pending, acquire-release); the count
//           that reaches zero puts the token in the ready queue. After the GEMM work all
//           warps of the CTA pop tokens from that queue and combine them (the same fp32
//           FMA chain as combine.cu) while other CTAs still finish their last units.
// Every wait is bounded as in the one-CTA kernel (flag T, producer / MMA 2T,
// epilogue 3T); a wait that runs out raises the abort flag of both CTAs. Both CTAs
// leave through two cluster barriers (with a grace period between them after an
// abort, for loads still in flight) so that neither exits while the other may still
// write to its shared memory or barriers, and then free the TMEM.
#include <mutex>
#include "ffn_gemm.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;                              // weight columns per CTA per accumulator
constexpr int kBK = 64;                               // k per stage
constexpr int kStages = 4;
constexpr int kChunkBytes = 64 * kBK * 2;             // 8 KB: 64 weight columns x 64 k
constexpr int kWTileBytes = 2 * kChunkBytes;          // 16 KB: one 128-column weight tile
constexpr int kRowBox = 32;                           // pool rows per TMA box
constexpr int kRowBoxBytes = kRowBox * kBK * 2;       // 4 KB
constexpr int kHalfRows = kGemmBlockM / 2;            // pool rows per CTA (N / 2 <= 128)
constexpr int kStageBytes = 2 * kWTileBytes + kHalfRows * kBK * 2;  // 48 KB
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
// Epilogue warps per CTA (a multiple of 4: the warps of one TMEM lane quadrant split the
// unit's 32-row groups between them).
#ifndef MOE_PAIR_EPI_WARPS
#define MOE_PAIR_EPI_WARPS 8
#endif
constexpr int kEpiWarps = MOE_PAIR_EPI_WARPS;
static_assert(kEpiWarps % 4 == 0 && kEpiWarps >= 8 && kEpiWarps <= 16, "4 lane quadrants");
constexpr int kEpiParts = kEpiWarps / 4;              // warps per lane quadrant
// 32-row groups of a unit (<= 256 rows) per warp: warp part p takes groups p, p + kEpiParts, ...
constexpr int kGroupsPerWarp = (8 + kEpiParts - 1) / kEpiParts;
constexpr int kSignalWarp = 2 + kEpiWarps;            // early combine only
constexpr int threads_for(bool early) { return 64 + kEpiWarps * 32 + (early ? 32 : 0); }
constexpr int kSchedSlots = 4;
// readers of a unit id, all counted on the first CTA's sched_empty: its MMA thread and
// epilogue warps, the second CTA's producer and epilogue warps (and both signal warps)
constexpr int sched_readers(bool early) { return 1 + kEpiWarps + 1 + kEpiWarps + (early ? 2 : 0); }
constexpr int kBarrierBytes = 256;
constexpr int kXposeBytes = 32 * 32 * 2;
constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kEpiWarps * kXposeBytes + 1024;
constexpr uint64_t kAbortGraceNs = 1000000;           // after an abort: loads in flight land
constexpr uint32_t kParkNs = 20000;                   // epilogue waits: parked 20 us per try

__device__ __forceinline__ void raise_abort_pair(volatile int *abort, uint32_t peer_abort,
                                                 int32_t *status, int32_t code, int32_t aux) {
  if (!*abort) report(status, code, aux);
  *abort = 1;
  st_cluster_u32(peer_abort, 1u);
}

// SiLU and its derivative from one sigmoid: s = 1 / (1 + e^-g) as in silu_mul.
__device__ __forceinline__ void swiglu_backward(float da, float g, float u, float &dg, float &du) {
  const float s = recip_newton2(1.0f + ex2_approx(fminf(g * -1.4426950408889634f, 100.0f)));
  const float silu = g * s;
  du = da * silu;
  dg = da * u * (s * fmaf(g, 1.0f - s, 1.0f));
}

// 16-byte load through L2 only (rows that another SM wrote during this kernel).
__device__ __forceinline__ uint4 ld_cg_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ void fma_row8(float (&acc)[8], float w, const uint4 &v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
  }
}

// Early combine, after the CTA's GEMM work: each warp pops positions of the ready queue and
// combines their tokens, out[t] = bf16(sum_j w[t, j] ypool[pool_row[t, j]]) as an fp32 FMA
// chain over j ascending (combine.cu's arithmetic, so the result is bit-identical).
__device__ void early_combine_drain(const FfnParams &prm, int lane, uint64_t timeout_ns) {
  const int hv = prm.n_out / 8;  // 16-byte vectors per row
  const uint4 *yp = reinterpret_cast<const uint4 *>(prm.out);
  uint4 *op = reinterpret_cast<uint4 *>(prm.comb_out);
  for (;;) {
    int32_t pos = 0;
    if (lane == 0) pos = atomicAdd(prm.ready + prm.T, 1);
    pos = __shfl_sync(0xffffffffu, pos, 0);
    if (pos >= prm.T) break;
    int32_t v = 0;
    if (lane == 0) {
      v = ld_acquire_gpu_s32(prm.ready + pos);
      if (v == 0) {
        const uint64_t t0 = globaltimer_ns();
        uint32_t sleep_ns = 64;
        while ((v = ld_acquire_gpu_s32(prm.ready + pos)) == 0) {
          if (globaltimer_ns() - t0 > timeout_ns) break;
          __nanosleep(sleep_ns);
          if (sleep_ns < 2048) sleep_ns <<= 1;
        }
      }
      if (v == 0) report(prm.status, MOE_ERR_COMBINE_TIMEOUT, pos);
    }
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v == 0) break;
    __syncwarp();  // lane 0's acquire orders the other lanes' loads of the token's rows
    const int64_t t = v - 1;
    int32_t my_row = -1;
    float my_w = 0.0f;
    if (lane < prm.k) {
      my_row = prm.pool_row[t * prm.k + lane];
      my_w = prm.topk_w != nullptr ? prm.topk_w[t * prm.k + lane] : 1.0f;  // none: unit weights
    }
    // every lane runs every iteration (the shuffles below need the whole warp); a lane's
    // vectors past the row's end are masked
    for (int c0 = 0; c0 < hv; c0 += 64) {
      const int c = c0 + lane, c1 = c + 32;
      const bool v0 = c < hv, v1 = c1 < hv;
      float a0[8], a1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a0[i] = a1[i] = 0.0f;
      for (int j0 = 0; j0 < prm.k; j0 += 8) {
        uint4 y0[8], y1[8];
        int32_t rr[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          rr[jj] = __shfl_sync(0xffffffffu, my_row, (j0 + jj) & 31);
          if (j0 + jj < prm.k && rr[jj] >= 0) {
            if (v0) y0[jj] = ld_cg_v4(yp + (size_t)rr[jj] * hv + c);
            if (v1) y1[jj] = ld_cg_v4(yp + (size_t)rr[jj] * hv + c1);
          }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float w = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
          if (j0 + jj < prm.k && rr[jj] >= 0) {
            if (v0) fma_row8(a0, w, y0[jj]);
            if (v1) fma_row8(a1, w, y1[jj]);
          }
        }
      }
      if (v0)
        op[(size_t)t * hv + c] =
            make_uint4(pack_bf16x2(a0[0], a0[1]), pack_bf16x2(a0[2], a0[3]),
                       pack_bf16x2(a0[4], a0[5]), pack_bf16x2(a0[6], a0[7]));
      if (v1)
        op[(size_t)t * hv + c1] =
            make_uint4(pack_bf16x2(a1[0], a1[1]), pack_bf16x2(a1[2], a1[3]),
                       pack_bf16x2(a1[4], a1[5]), pack_bf16x2(a1[6], a1[7]));
    }
  }
}

template <int kMode, bool kAK, bool kEarly>
__global__ void __launch_bounds__(threads_for(kEarly), 1)
    ffn_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                         const __grid_constant__ CUtensorMap tm_x, const FfnParams prm) {
  static_assert(!kEarly || kMode == 1, "early combine folds into GEMM Y or backward A");
  constexpr int kSchedReaders = sched_readers(kEarly);
  extern __shared__ uint8_t smem_raw[];
  // The same offsets in both CTAs (the MMA reads both CTAs' operands at one address).
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;
  uint64_t *acc_empty = acc_full + 1;
  uint64_t *drain = acc_empty + 1;
  uint64_t *sched_full = drain + 1;
  uint64_t *sched_empty = sched_full + kSchedSlots;
  int32_t *sched = reinterpret_cast<int32_t *>(sched_empty + kSchedSlots);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sched + kSchedSlots);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *never = abort_flag + 1;
  // early combine: per sched slot, how many epilogue warps have stored their rows of the
  // slot's units so far (monotonic: unit `local` is stored when it reaches
  // kEpiWarps * (local / kSchedSlots + 1))
  uint32_t *stored = reinterpret_cast<uint32_t *>(never + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool lead = rank == 0;
  const uint32_t peer_abort = cluster_map(smem_u32(abort_flag), peer);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    mbar_init(drain, 1);
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(sched_full + i, 1);
      mbar_init(sched_empty + i, kSchedReaders);
      if (kEarly) stored[i] = 0;
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
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // Barriers of both CTAs are initialised and both TMEMs allocated before either CTA
  // touches the other's.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = abort_flag;

  const int32_t n_units = prm.meta[2] * prm.n_blocks;
  const int kb_count = prm.K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0, last_parity = 0;  // first CTA: stages whose bytes it expects
      uint32_t sslot = 0, sphase = 0;
      for (;;) {
        int32_t u;
        if (lead) {
          if (!mbar_wait<true>(sched_empty + sslot, sphase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
            break;
          }
          const int32_t ticket = atomicAdd(prm.sched + 0, 1);
          u = (ticket < n_units && !*abort) ? ticket : -1;
          sched[sslot] = u;
          st_cluster_u32(cluster_map(smem_u32(sched + sslot), peer), (uint32_t)u);
          mbar_arrive(sched_full + sslot);
          mbar_arrive_cluster(cluster_map(smem_u32(sched_full + sslot), peer));
        } else {
          if (!mbar_wait<true>(sched_full + sslot, sphase, 2 * prm.timeout_ns, abort)) {
            raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
            break;
          }
          u = sched[sslot];
          mbar_arrive_cluster(cluster_map(smem_u32(sched_empty + sslot), 0));
        }
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
        const int32_t half_rows = ((rows + 15) & ~15) >> 1;   // N / 2
        const int nbox = (half_rows + kRowBox - 1) / kRowBox;  // same in both CTAs
        const int32_t xrow0 = row0 + (int32_t)rank * half_rows;
        if ((kMode == 0 || kMode == 2 || kMode == 3) && prm.streaming) {
          const int32_t t_end = (row0 + rows - 1) / prm.tile;
          for (int32_t t = row0 / prm.tile; t <= t_end && !*abort; ++t) {
            const uint64_t t0 = globaltimer_ns();
            uint32_t it = 0;
            while (ld_acquire_sys(prm.flags + t) < (uint32_t)prm.tile) {
              if ((++it & 63u) == 0 && (*abort || globaltimer_ns() - t0 > prm.timeout_ns)) {
                raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_FLAG_TIMEOUT, t);
                break;
              }
            }
          }
          fence_proxy_async_global();
          if (*abort) break;
        }
        const int32_t wcol0 = nb * prm.col_step + (int32_t)rank * kBM;
        const int32_t wcol1 = wcol0 + prm.col1_off;
        const uint32_t tx = 2u * (uint32_t)(2 * kWTileBytes + nbox * kRowBoxBytes);
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
            break;
          }
          uint8_t *sw0 = smem + stage * kStageBytes;
          uint8_t *sw1 = sw0 + kWTileBytes;
          uint8_t *sx = sw0 + 2 * kWTileBytes;
          const uint32_t fb = cluster_map(smem_u32(full + stage), 0);
          if (lead) {
            mbar_arrive_expect_tx(full + stage, tx);
            issued |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (kAK) {
            // K-major weights: rows of the map are output columns, 64 k per 128-byte row
            const int32_t wrow = e * prm.k_rows + wcol0;
            tma_load_2d_pair(sw0, &tm_w, fb, kb * kBK, wrow);
            tma_load_2d_pair(sw1, &tm_w, fb, kb * kBK, wrow + prm.col1_off);
          } else if (prm.packed) {
            const int32_t t0 =
                e * prm.pk_e + nb * prm.pk_nb + (int32_t)rank * prm.pk_v + kb;
            tma_load_2d_pair(sw0, &tm_w, fb, 0, t0 * 128);
            tma_load_2d_pair(sw1, &tm_w, fb, 0, (t0 + prm.pk_j) * 128);
          } else {
            const int32_t krow = e * prm.k_rows + kb * kBK;
            tma_load_2d_pair(sw0, &tm_w, fb, wcol0, krow);
            tma_load_2d_pair(sw0 + kChunkBytes, &tm_w, fb, wcol0 + 64, krow);
            tma_load_2d_pair(sw1, &tm_w, fb, wcol1, krow);
            tma_load_2d_pair(sw1 + kChunkBytes, &tm_w, fb, wcol1 + 64, krow);
          }
          for (int i = 0; i < nbox; ++i)
            tma_load_2d_pair(sx + i * kRowBoxBytes, &tm_x, fb, kb * kBK, xrow0 + i * kRowBox);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort && lead)
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s))
            mbar_wait(full + s, (last_parity >> s) & 1u, prm.timeout_ns, never);
      if (lead) {
        // Every cluster has taken its last ticket (the end ticket, or the one before an
        // abort) before it counts itself done, so the last one may zero the counters for
        // the next launch, on the abort path too.
        __threadfence();
        const int group = prm.sched_group > 0 ? prm.sched_group : (int)(gridDim.x >> 1);
        if (atomicAdd(prm.sched + 1, 1) == group - 1) {
          atomicExch(prm.sched + 0, 0);
          atomicExch(prm.sched + 1, 0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0, local = 0;
      uint32_t sslot = 0, sphase = 0;
      bool ok = true;
      for (;; ++local) {
        if (!mbar_wait(sched_full + sslot, sphase, 2 * prm.timeout_ns, abort)) {
          raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
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
        const uint32_t idesc = idesc_bf16_f32_ab(2 * kBM, n_mma, /*a_mn=*/!kAK, /*b_mn=*/false);
        // Both CTAs' epilogues have read the previous unit's accumulators.
        if (!mbar_wait<true>(acc_empty, (local + 1u) & 1u, 2 * prm.timeout_ns, abort)) {
          raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait(full + stage, phase, 2 * prm.timeout_ns, abort)) {
            raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sw0 = smem_u32(smem + stage * kStageBytes);
          const uint32_t sw1 = sw0 + kWTileBytes;
          const uint32_t sx = sw0 + 2 * kWTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // weights: MN-major, 64-column chunks kChunkBytes apart, +2048 B per 16 k;
            // pool rows: K-major 128-byte rows, 8-row groups 1024 B apart, +32 B per 16 k
            // (K-major weights: the same form as the pool rows)
            const uint64_t xdesc = smem_desc_sw128(sx + kk * 32, 16, 1024);
            const uint64_t w0 = kAK ? smem_desc_sw128(sw0 + kk * 32, 16, 1024)
                                    : smem_desc_sw128(sw0 + kk * 2048, kChunkBytes, 1024);
            const uint64_t w1 = kAK ? smem_desc_sw128(sw1 + kk * 32, 16, 1024)
                                    : smem_desc_sw128(sw1 + kk * 2048, kChunkBytes, 1024);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_bf16_pair(tmem_base, w0, xdesc, idesc, acc);
            tc_mma_bf16_pair(tmem_base + kAccStride, w1, xdesc, idesc, acc);
          }
          tc_commit_pair_mc(empty + stage, 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(acc_full, 0x3);
      }
      // Wait for every MMA issued by this thread before either TMEM is released.
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait(drain, 0, prm.timeout_ns, never);
    }
  } else if (kEarly && warp == kSignalWarp) {
    // -------------------------------------------------------------- early-combine signals
    uint32_t sslot = 0, sphase = 0;
    for (uint32_t local = 0;; ++local) {
      int32_t u = -1;
      int got = 1;
      if (lane == 0) {
        got = mbar_wait_parked<true>(sched_full + sslot, sphase, 3 * prm.timeout_ns, abort,
                                     kParkNs)
                  ? 1
                  : 0;
        if (got) {
          u = sched[sslot];
          if (lead)
            mbar_arrive(sched_empty + sslot);
          else
            mbar_arrive_cluster(cluster_map(smem_u32(sched_empty + sslot), 0));
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (++sslot == kSchedSlots) {
        sslot = 0;
        sphase ^= 1u;
      }
      if (!got) {
        if (lane == 0) raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
        break;
      }
      if (u < 0) break;
      int ok = 1;
      if (lane == 0) {
        // all of this CTA's epilogue warps have stored the unit (bounded, sleeping poll)
        const uint32_t want = kEpiWarps * (local / kSchedSlots + 1);
        uint32_t *cnt = stored + (local % kSchedSlots);
        if (ld_acquire_cta_shared(cnt) < want) {
          const uint64_t t0 = globaltimer_ns();
          uint32_t sleep_ns = 64;
          while (ld_acquire_cta_shared(cnt) < want) {
            if (*abort || globaltimer_ns() - t0 > 3 * prm.timeout_ns) {
              ok = 0;
              break;
            }
            __nanosleep(sleep_ns);
            if (sleep_ns < 1024) sleep_ns <<= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
        break;
      }
      // this CTA's share of the unit is stored: count it on the row chunk (release: the
      // epilogue's stores before it; acquire: the other units' stores). The last of the
      // chunk's 2 x n_blocks counts drops each live row's token count by one, so a token's
      // count falls once per live pair instead of once per pair, column block and CTA.
      int32_t mb, nb;
      unit_coords(prm.mblk, u, prm.n_blocks, mb, nb);
      const int32_t row0 = prm.mblk[kMblkInts * mb + 0];
      const int32_t rows = prm.mblk[kMblkInts * mb + 2];
      int last = 0;
      if (lane == 0)
        last = atom_add_acq_rel_gpu(prm.chunk_cnt + mb, 1) == 2 * prm.n_blocks - 1 ? 1 : 0;
      last = __shfl_sync(0xffffffffu, last, 0);
      __syncwarp();  // lane 0's acquire orders the other lanes' releases below
      if (!last) continue;
      for (int r = lane; r < rows; r += 32) {
        const int32_t f = prm.row_src[row0 + r];
        if (f < 0) continue;
        const int32_t t = f / prm.k;
        if (atom_add_acq_rel_gpu(prm.tok_pending + t, -1) == 1) {
          const int32_t qpos = atomicAdd(prm.ready + prm.T + 1, 1);
          if (qpos < prm.T)
            st_release_gpu(prm.ready + qpos, t + 1);
          else  // more tokens completed than exist: counters armed twice for one plan
            report(prm.status, MOE_ERR_COMBINE_TIMEOUT, qpos);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;   // which of the quadrant's row-group parts
    const uint32_t tq = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint16_t *xp = reinterpret_cast<uint16_t *>(smem + kStages * kStageBytes + kBarrierBytes) +
                   (warp - 2) * (kXposeBytes / 2);
    const uint32_t acc_empty_lead = cluster_map(smem_u32(acc_empty), 0);
    uint32_t local = 0;
    uint32_t sslot = 0, sphase = 0;
    for (;; ++local) {
      int32_t u = -1;
      int got = 1;
      if (lane == 0) {
        got = mbar_wait_parked<true>(sched_full + sslot, sphase, 3 * prm.timeout_ns, abort,
                                     kParkNs)
                  ? 1
                  : 0;
        if (got) {
          u = sched[sslot];
          if (lead)
            mbar_arrive(sched_empty + sslot);
          else
            mbar_arrive_cluster(cluster_map(smem_u32(sched_empty + sslot), 0));
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (++sslot == kSchedSlots) {
        sslot = 0;
        sphase ^= 1u;
      }
      if (!got) {
        if (lane == 0) raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
        break;
      }
      if (u < 0) break;
      int32_t mb, nb;
      unit_coords(prm.mblk, u, prm.n_blocks, mb, nb);
      const int32_t row0 = prm.mblk[kMblkInts * mb + 0];
      const int32_t rows = prm.mblk[kMblkInts * mb + 2];
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_parked(acc_full, local & 1u, 3 * prm.timeout_ns, abort, kParkNs) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort_pair(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
        break;
      }
      tc_fence_after();
      const int32_t cb0 = nb * prm.col_step + (int32_t)rank * kBM + quad * 32;
      const int32_t cb1 = cb0 + prm.col1_off;
      const bool ok0 = cb0 < prm.n_out;
      const bool ok1 = kMode != 0 && cb1 < prm.n_out1;
      // First the warp's whole share of both accumulators (kGroupsPerWarp 32-row groups)
      // into registers as bf16 pairs (rows 2i, 2i+1 of a group in pk[.][i]), and the TMEM
      // back to the MMA thread; then the slower turn through shared memory and the
      // global stores, while the next unit's MMAs already run.
      constexpr int kOuts = kMode == 0 ? 1 : 2;  // output tiles per 32-row group
      uint32_t pk[kGroupsPerWarp * kOuts][16];
#pragma unroll
      for (int g = 0; g < kGroupsPerWarp; ++g) {
        const int c = part * 32 + g * 32 * kEpiParts;
        if (c < rows) {  // uniform across the warp
          __syncwarp();
          if (kMode == 0) {
            uint32_t a0[32], a1[32];
            tmem_ld_32x32b_x32(tq + c, a0);
            tmem_ld_32x32b_x32(tq + kAccStride + c, a1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[g][i] = pack_bf16x2(
                  silu_mul(__uint_as_float(a0[2 * i]), __uint_as_float(a1[2 * i])),
                  silu_mul(__uint_as_float(a0[2 * i + 1]), __uint_as_float(a1[2 * i + 1])));
          } else {
            // one accumulator at a time: 128 registers of pairs stay live at the end
#pragma unroll
            for (int j = 0; j < kOuts; ++j) {
              uint32_t a[32];
              tmem_ld_32x32b_x32(tq + j * kAccStride + c, a);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[kOuts * g + j][i] =
                    pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (lead)
          mbar_arrive_relaxed(acc_empty);
        else
          mbar_arrive_cluster_relaxed(acc_empty_lead);
      }
#pragma unroll
      for (int g = 0; g < kGroupsPerWarp; ++g) {
        const int c = part * 32 + g * 32 * kEpiParts;
        if (c < rows) {
          const int lim = min(32, rows - c);
#pragma unroll
          for (int j = 0; j < kOuts; ++j) {
            if (!(j == 0 ? ok0 : ok1)) continue;  // uniform across the warp
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t v = pk[kOuts * g + j][i];
              xp[(2 * i) * 32 + lane] = (uint16_t)(v & 0xFFFFu);
              xp[(2 * i + 1) * 32 + lane] = (uint16_t)(v >> 16);
            }
            __syncwarp();
            const int32_t cb = j == 0 ? cb0 : cb1;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int v = lane + 32 * q;
              const int r = v >> 2;
              const int part = v & 3;
              if (r < lim) {
                const uint4 val = *reinterpret_cast<const uint4 *>(xp + r * 32 + part * 8);
                if (kMode != 2) {
                  *reinterpret_cast<uint4 *>(prm.out + (size_t)(row0 + c + r) * prm.out_ld +
                                             cb + part * 8) = val;
                } else {
                  const size_t o = (size_t)(row0 + c + r) * prm.out_ld + cb + part * 8;
                  // 8 columns of one row: da from the turned block, g and u from the
                  // saved pre-activations, dg and du to the same columns of out
                  const size_t a = (size_t)(row0 + c + r) * prm.aux_ld + cb + part * 8;
                  const uint4 g8 = *reinterpret_cast<const uint4 *>(prm.aux + a);
                  const uint4 u8 = *reinterpret_cast<const uint4 *>(prm.aux + a + prm.aux_off);
                  const uint32_t dv[4] = {val.x, val.y, val.z, val.w};
                  const uint32_t gv[4] = {g8.x, g8.y, g8.z, g8.w};
                  const uint32_t uv[4] = {u8.x, u8.y, u8.z, u8.w};
                  uint32_t dgo[4], duo[4];
#pragma unroll
                  for (int h = 0; h < 4; ++h) {
                    float dg0, du0, dg1, du1;
                    swiglu_backward(__uint_as_float(dv[h] << 16), __uint_as_float(gv[h] << 16),
                                    __uint_as_float(uv[h] << 16), dg0, du0);
                    swiglu_backward(__uint_as_float(dv[h] & 0xFFFF0000u),
                                    __uint_as_float(gv[h] & 0xFFFF0000u),
                                    __uint_as_float(uv[h] & 0xFFFF0000u), dg1, du1);
                    dgo[h] = pack_bf16x2(dg0, dg1);
                    duo[h] = pack_bf16x2(du0, du1);
                  }
                  *reinterpret_cast<uint4 *>(prm.out + o) =
                      make_uint4(dgo[0], dgo[1], dgo[2], dgo[3]);
                  *reinterpret_cast<uint4 *>(prm.out + o + prm.aux_off) =
                      make_uint4(duo[0], duo[1], duo[2], duo[3]);
                }
              }
            }
          }
          if (kMode == 3 && ok0) {
            // act = bf16(silu(g) * u) from the bf16 g and u just stored, into out2; the
            // pairs of g are overwritten by the pairs of act
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t gp = pk[kOuts * g][i], up = pk[kOuts * g + 1][i];
              pk[kOuts * g][i] = pack_bf16x2(
                  silu_mul(__uint_as_float(gp << 16), __uint_as_float(up << 16)),
                  silu_mul(__uint_as_float(gp & 0xFFFF0000u), __uint_as_float(up & 0xFFFF0000u)));
              xp[(2 * i) * 32 + lane] = (uint16_t)(pk[kOuts * g][i] & 0xFFFFu);
              xp[(2 * i + 1) * 32 + lane] = (uint16_t)(pk[kOuts * g][i] >> 16);
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int v = lane + 32 * q;
              const int r = v >> 2;
              const int part = v & 3;
              if (r < lim)
                *reinterpret_cast<uint4 *>(prm.out2 + (size_t)(row0 + c + r) * prm.out2_ld +
                                           cb0 + part * 8) =
                    *reinterpret_cast<const uint4 *>(xp + r * 32 + part * 8);
            }
          }
        }
      }
      if (kEarly) {
        // the unit's rows of this warp are stored: counted on the slot's counter (the warp
        // barrier orders every lane's stores before lane 0's release; the signal warp's
        // acquire of the counter and its GPU-scope release of the token's count pass them
        // on to the combine, whose acquire reads the queue)
        __syncwarp();
        if (lane == 0) red_release_cta_shared_add(stored + (local % kSchedSlots), 1u);
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();
  // After an abort in either CTA, loads that one CTA issued may still be landing in its
  // shared memory and on the first CTA's barriers: give them time before both exit.
  if (threadIdx.x == 0 && (*abort || ld_cluster_u32(peer_abort) != 0u)) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kAbortGraceNs) __nanosleep(1000);
  }
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  if (kEarly && !*abort) early_combine_drain(prm, lane, 3 * prm.timeout_ns);
}

template <int kMode, bool kAK, bool kEarly = false>
cudaError_t launch_mode(const CUtensorMap &tw, const CUtensorMap &tx, const FfnParams &prm,
                        int clusters, cudaStream_t st) {
  static bool attr_set[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(ffn_gemm_pair_kernel<kMode, kAK, kEarly>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(2 * clusters, 1, 1);
  lc.blockDim = dim3(threads_for(kEarly), 1, 1);
  lc.dynamicSmemBytes = kSmemBytes;
  lc.stream = st;
  lc.attrs = at;
  lc.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&lc, ffn_gemm_pair_kernel<kMode, kAK, kEarly>, tw, tx, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int kMode, bool kAK, bool kEarly = false>
int max_clusters_mode() {
  static int cached[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    if (cudaFuncSetAttribute(ffn_gemm_pair_kernel<kMode, kAK, kEarly>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return 0;
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.gridDim = dim3(2, 1, 1);
    lc.blockDim = dim3(threads_for(kEarly), 1, 1);
    lc.dynamicSmemBytes = kSmemBytes;
    lc.attrs = at;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, ffn_gemm_pair_kernel<kMode, kAK, kEarly>, &lc) != cudaSuccess)
      return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace

cudaError_t launch_ffn_pair(int mode, bool a_kmajor, const CUtensorMap &tw,
                            const CUtensorMap &tx, const FfnParams &prm, int clusters,
                            cudaStream_t st, bool early) {
  if (early) {
    // GEMM Y (weights MN-major) or backward A (K-major) with the combine folded in
    if (mode != 1) return cudaErrorInvalidValue;
    // the extra signal warp: as many clusters as fit with it (at most those asked for)
    const int fit = a_kmajor ? max_clusters_mode<1, true, true>() : max_clusters_mode<1, false, true>();
    if (fit < 1) return cudaErrorInvalidConfiguration;
    const int c = clusters < fit ? clusters : fit;
    return a_kmajor ? launch_mode<1, true, true>(tw, tx, prm, c, st)
                    : launch_mode<1, false, true>(tw, tx, prm, c, st);
  }
  if (!a_kmajor)
    return mode == 0   ? launch_mode<0, false>(tw, tx, prm, clusters, st)
           : mode == 3 ? launch_mode<3, false>(tw, tx, prm, clusters, st)
                       : launch_mode<1, false>(tw, tx, prm, clusters, st);
  return mode == 2 ? launch_mode<2, true>(tw, tx, prm, clusters, st)
                   : launch_mode<1, true>(tw, tx, prm, clusters, st);
}

// All instantiations without early combine have the same block size and shared memory,
// hence the same count.
int ffn_pair_max_clusters(int) { return max_clusters_mode<0, false>(); }

}  // namespace moe
