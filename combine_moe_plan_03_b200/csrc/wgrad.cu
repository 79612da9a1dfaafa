// Weight gradients of the grouped FFN (the backward's weight GEMMs): for every expert e,
//   dW1[e] = pool_e^T . dgu_e      [H, 2I]      dgu = [dg | du] of the backward Y epilogue
//   dW2[e] = act_e^T  . dypool_e   [I, H]
// where X_e are the rows of expert e's pool segment. As one grouped GEMM:
//   D[e] [M, N] = sum over the segment's rows p of A[p, 0:M]^T (x) B[p, 0:N]
// with A, B row-major [P_max, M] / [P_max, N] activations and D [E, M, N] bf16.
//
// Design (tcgen05, SM pairs as in ffn_gemm_pair.cu): a work unit is (expert, 256 rows of D,
// 512 columns of D); one cta_group::2 MMA has M = 256 (128 rows of D per CTA) and N = 256
// (each CTA holds 128 of B's columns), K = 16, into one of two accumulators of 256 TMEM
// columns; the K loop runs over the expert's rows in steps of 64 (its live rows rounded up
// to 64: rows past the live ones must be zero, which zero_pad_rows_kernel ensures for the
// operands that are not zero there already). Both operands are read MN-major straight from
// the activations (for A the rows of D are contiguous in memory, for B its columns), TMA
// boxes of 64 columns x 64 rows: per stage and CTA two of A and four of B (48 KB), 4 stages.
// The epilogue hands the two accumulators back one at a time; the next unit's MMAs into the
// first are issued while the second is still being read. (The narrow tiling, 256 columns
// per unit with one accumulator in two buffers and 5 stages of 32 KB, is kept as the
// MOE_WGRAD_WIDE=0 build: it draws a third more operand bytes per flop.) In the epilogue
// each thread holds one row of D (its TMEM lane) and 32 consecutive columns per load; a
// warp's 32 x 64 share of a unit goes through shared memory as two 32 x 32 blocks (64-byte
// swizzled, 2 KB: small enough to leave room for the 4th stage) to two TMA stores (16
// epilogue warps; the gradients are 3·E·H·I bf16 values per call). An expert with no rows gets a zero
// gradient. Waits are bounded as in the forward kernels; a wait that runs out reports
// MOE_ERR_PIPE_TIMEOUT and raises both CTAs' abort flags.
#include <mutex>

#include "ffn_gemm.cuh"

namespace moe {

namespace {

constexpr int kBK = 64;
constexpr int kBoxBytes = 64 * kBK * 2;       // 8 KB: 64 columns x 64 rows
constexpr int kOpBytes = 2 * kBoxBytes;       // 16 KB: 128 columns of one operand
constexpr int kTmemCols = 512;
constexpr int kBufCols = 256;
constexpr int kEpiWarps = 16;                  // 4 per TMEM lane quadrant, 64 columns each
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr int kSchedSlots = 4;
constexpr int kSchedReaders = 1 + kEpiWarps + 1 + kEpiWarps;
constexpr int kBarrierBytes = 256;
constexpr int kStageOutBytes = 32 * 32 * 2;    // a warp's 32 rows x 32 columns of D
constexpr int kOutBytes = kEpiWarps * kStageOutBytes;

// Two tilings of D. Narrow: a unit is 256 x 256 of D, one accumulator of 256 TMEM columns in
// two buffers (the epilogue of one unit overlaps the MMAs of the next), stages of A and one
// B half (32 KB), 5 stages. Wide: a unit is 256 x 512 of D, two accumulators (all 512 TMEM
// columns), stages of A and two B halves (48 KB), 4 stages: each A tile serves twice the
// MMA work, so the SMs draw 25% fewer operand bytes per flop from L2; the accumulators are
// handed back one at a time and the next unit's MMAs into the first start meanwhile.
template <bool kWide>
struct WgradGeom {
  static constexpr int kAccs = kWide ? 2 : 1;               // accumulators per unit
  static constexpr int kUnitCols = 256 * kAccs;             // columns of D per unit
  static constexpr int kStageBytes = kOpBytes * (1 + kAccs);
  static constexpr int kStages = kWide ? 4 : 5;
  static constexpr int kRingBytes = kStages * kStageBytes;  // 192 KB / 160 KB
  // shared memory: stage ring, then the epilogue's blocks (1024-byte aligned, more than the
  // 64-byte swizzle of their TMA stores wants), then the barriers
  static constexpr int kSmemBytes = kRingBytes + kOutBytes + kBarrierBytes + 1024;
};
static_assert(WgradGeom<true>::kSmemBytes <= 227 * 1024, "shared memory");
static_assert(WgradGeom<false>::kSmemBytes <= 227 * 1024, "shared memory");
constexpr uint64_t kAbortGraceNs = 1000000;
constexpr uint32_t kParkNs = 20000;

struct WgradParams {
  const int32_t *offsets;   // [E + 1] expert segment starts (rows)
  const int32_t *counts;    // [E] live rows per expert
  int32_t *status;
  uint16_t *out;            // D [E, M, N]
  int32_t E, M, N;
  int32_t mb_count, nb_count;  // blocks of 256 rows / of the unit's columns of D
  int32_t *sched;           // {ticket, clusters done}
  uint64_t timeout_ns;
};

__device__ __forceinline__ void raise_abort_w(volatile int *abort, uint32_t peer_abort,
                                              int32_t *status, int32_t code, int32_t aux) {
  if (!*abort) report(status, code, aux);
  *abort = 1;
  st_cluster_u32(peer_abort, 1u);
}

__device__ __forceinline__ int32_t k_steps(const WgradParams &prm, int32_t e) {
  return (prm.counts[e] + kBK - 1) / kBK;
}

template <bool kWide>
__global__ void __launch_bounds__(kThreads, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_d, const WgradParams prm) {
  using G = WgradGeom<kWide>;
  constexpr int kStages = G::kStages;
  constexpr int kStageBytes = G::kStageBytes;
  constexpr int kRingBytes = G::kRingBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRingBytes + kOutBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;    // [2]: buffers (narrow) / one per unit (wide)
  uint64_t *acc_empty = acc_full + 2;      // [2]: buffers (narrow) / accumulators (wide)
  uint64_t *drain = acc_empty + 2;
  uint64_t *sched_full = drain + 1;
  uint64_t *sched_empty = sched_full + kSchedSlots;
  int32_t *sched = reinterpret_cast<int32_t *>(sched_empty + kSchedSlots);
  int32_t *sched_k = sched + kSchedSlots;   // the unit's k-steps, published with its id
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sched_k + kSchedSlots);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *never = abort_flag + 1;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(sched_full + i, 1);
      mbar_init(sched_empty + i, kSchedReaders);
    }
    *abort_flag = 0;
    *never = 0;
    fence_mbarrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 2 && lane == 0) tma_prefetch_desc(&tm_d);
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int *abort = abort_flag;
  const int32_t units_per_e = prm.mb_count * prm.nb_count;
  const int32_t n_units = prm.E * units_per_e;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0, issued = 0, last_parity = 0;
      uint32_t sslot = 0, sphase = 0;
      // the first CTA asks for the next ticket one unit ahead, so the atomic's round trip
      // overlaps the loads of the current unit (the units are short: a few k-steps)
      int32_t next_ticket = lead ? atomicAdd(prm.sched + 0, 1) : 0;
      for (;;) {
        int32_t u, kpeer = 0;
        if (lead) {
          if (!mbar_wait<true>(sched_empty + sslot, sphase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
            break;
          }
          const int32_t ticket = next_ticket;
          if (ticket < n_units) next_ticket = atomicAdd(prm.sched + 0, 1);
          u = (ticket < n_units && !*abort) ? ticket : -1;
          const int32_t kc = u >= 0 ? k_steps(prm, u / units_per_e) : 0;
          sched[sslot] = u;
          sched_k[sslot] = kc;
          st_cluster_u32(cluster_map(smem_u32(sched + sslot), peer), (uint32_t)u);
          st_cluster_u32(cluster_map(smem_u32(sched_k + sslot), peer), (uint32_t)kc);
          mbar_arrive(sched_full + sslot);
          mbar_arrive_cluster(cluster_map(smem_u32(sched_full + sslot), peer));
        } else {
          if (!mbar_wait<true>(sched_full + sslot, sphase, 2 * prm.timeout_ns, abort)) {
            raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
            break;
          }
          u = sched[sslot];
          kpeer = sched_k[sslot];
          if (u >= -1 && kpeer >= 0)   // issued once both reads have returned
            mbar_arrive_cluster_relaxed(cluster_map(smem_u32(sched_empty + sslot), 0));
        }
        const int32_t kcount = lead ? sched_k[sslot] : kpeer;
        if (++sslot == kSchedSlots) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (u < 0) break;
        const int32_t e = u / units_per_e;
        const int32_t rest = u % units_per_e;
        const int32_t mb = rest / prm.nb_count;
        const int32_t nb = rest % prm.nb_count;
        const int32_t row0 = prm.offsets[e];
        const int32_t acol = mb * 256 + (int32_t)rank * 128;
        const int32_t bcol = nb * G::kUnitCols + (int32_t)rank * 128;
        for (int32_t kb = 0; kb < kcount; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, 2 * prm.timeout_ns, abort)) {
            raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
            break;
          }
          uint8_t *sa = smem + stage * kStageBytes;
          uint8_t *sb = sa + kOpBytes;
          const uint32_t fb = cluster_map(smem_u32(full + stage), 0);
          if (lead) {
            mbar_arrive_expect_tx(full + stage, 2u * kStageBytes);
            issued |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          const int32_t r = row0 + kb * kBK;
          tma_load_2d_pair(sa, &tm_a, fb, acol, r);
          tma_load_2d_pair(sa + kBoxBytes, &tm_a, fb, acol + 64, r);
          tma_load_2d_pair(sb, &tm_b, fb, bcol, r);
          tma_load_2d_pair(sb + kBoxBytes, &tm_b, fb, bcol + 64, r);
          if (kWide) {  // the second accumulator's B half: 256 columns further
            tma_load_2d_pair(sb + kOpBytes, &tm_b, fb, bcol + 256, r);
            tma_load_2d_pair(sb + kOpBytes + kBoxBytes, &tm_b, fb, bcol + 320, r);
          }
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
        // counted done on the abort path too (its last ticket is taken), so the last
        // cluster zeroes the counters for the next launch in every case
        __threadfence();
        if (atomicAdd(prm.sched + 1, 1) == (int)(gridDim.x >> 1) - 1) {
          atomicExch(prm.sched + 0, 0);
          atomicExch(prm.sched + 1, 0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0, local = 0, sslot = 0, sphase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32_ab(256, 256, /*a_mn=*/true, /*b_mn=*/true);
      for (;; ++local) {
        if (!mbar_wait(sched_full + sslot, sphase, 2 * prm.timeout_ns, abort)) {
          raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
          break;
        }
        const int32_t u = sched[sslot];
        const int32_t kcount = sched_k[sslot];
        if (u >= -1 && kcount >= 0) mbar_arrive_relaxed(sched_empty + sslot);
        if (++sslot == kSchedSlots) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (u < 0) break;
        // narrow: the unit's accumulator is buffer local % 2, in its (local / 2)-th use;
        // wide: accumulators 0 and 1 (TMEM columns 0 and 256), each in its local-th use
        const uint32_t buf = kWide ? 0u : (local & 1u);
        const uint32_t empty_parity = kWide ? ((local + 1u) & 1u) : (((local >> 1) + 1u) & 1u);
        if (!mbar_wait<true>(acc_empty + buf, empty_parity, 2 * prm.timeout_ns, abort)) {
          raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * kBufCols;
        bool need1 = kWide;  // the second accumulator not yet handed back for this unit
        for (int32_t kb = 0; kb < kcount; ++kb) {
          if (!mbar_wait(full + stage, phase, 2 * prm.timeout_ns, abort)) {
            raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t sb = sa + kOpBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // both MN-major: 64-column chunks kBoxBytes apart, 8 rows per 1024 B, +2048 B
            // per 16 rows of K
            const uint64_t ad = smem_desc_sw128(sa + kk * 2048, kBoxBytes, 1024);
            const uint64_t bd = smem_desc_sw128(sb + kk * 2048, kBoxBytes, 1024);
            tc_mma_bf16_pair(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if (kWide) {
            if (need1) {
              // the first accumulator's MMAs of this k-step are queued; now the second
              // accumulator must have been read by both CTAs' epilogues
              if (!mbar_wait<true>(acc_empty + 1, empty_parity, 2 * prm.timeout_ns, abort)) {
                raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
                ok = false;
                break;
              }
              tc_fence_after();
              need1 = false;
            }
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(sa + kk * 2048, kBoxBytes, 1024);
              const uint64_t bd = smem_desc_sw128(sb + kOpBytes + kk * 2048, kBoxBytes, 1024);
              tc_mma_bf16_pair(d + kBufCols, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit_pair_mc(empty + stage, 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (need1) {  // a unit without rows: still one use of the second accumulator
          if (!mbar_wait<true>(acc_empty + 1, empty_parity, 2 * prm.timeout_ns, abort)) {
            raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
            break;
          }
          tc_fence_after();
        }
        tc_commit_pair_mc(acc_full + buf, 0x3);
      }
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait(drain, 0, prm.timeout_ns, never);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // warp w reads TMEM lanes 32 (w % 4) ... (32 rows of D) and columns 64 h ... 64 h + 63,
    // h = (w - 2) / 4, of the unit's 256 columns, 32 at a time: each thread puts its row's
    // 64 columns, 32 at a time, into the warp's 32 x 32 block in shared memory, in the
    // 64-byte swizzled order (16-byte chunk c of row r at c ^ ((r / 2) % 4), so each group
    // of 8 lanes hits every bank once), and one thread writes the block to D with a TMA
    // store.
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;
    const uint32_t tq = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint8_t *stg = smem + kRingBytes + (warp - 2) * kStageOutBytes;
    uint32_t local = 0, sslot = 0, sphase = 0;
    for (;; ++local) {
      int32_t u = -1, kc = 0;
      int got = 1;
      if (lane == 0) {
        got = mbar_wait_parked<true>(sched_full + sslot, sphase, 3 * prm.timeout_ns, abort,
                                     kParkNs)
                  ? 1
                  : 0;
        if (got) {
          u = sched[sslot];
          kc = sched_k[sslot];
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      kc = __shfl_sync(0xffffffffu, kc, 0);
      if (lane == 0 && got) {   // after the shuffles: the slot's values are in registers
        if (lead)
          mbar_arrive_relaxed(sched_empty + sslot);
        else
          mbar_arrive_cluster_relaxed(cluster_map(smem_u32(sched_empty + sslot), 0));
      }
      if (++sslot == kSchedSlots) {
        sslot = 0;
        sphase ^= 1u;
      }
      if (!got) {
        if (lane == 0) raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, -1);
        break;
      }
      if (u < 0) break;
      const int32_t e = u / units_per_e;
      const int32_t rest = u % units_per_e;
      const int32_t mb = rest / prm.nb_count;
      const int32_t nb = rest % prm.nb_count;
      const bool live = kc > 0;
      const uint32_t buf = kWide ? 0u : (local & 1u);
      const uint32_t full_parity = kWide ? (local & 1u) : ((local >> 1) & 1u);
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_parked(acc_full + buf, full_parity, 3 * prm.timeout_ns, abort, kParkNs)
                 ? 1
                 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort_w(abort, peer_abort, prm.status, MOE_ERR_PIPE_TIMEOUT, u);
        break;
      }
      tc_fence_after();
      const int32_t m0 = mb * 256 + (int32_t)rank * 128 + quad * 32;  // first row of D here
#pragma unroll
      for (int j = 0; j < G::kAccs; ++j) {
        const uint32_t acc = kWide ? (uint32_t)j : buf;                 // TMEM buffer / barrier
        const int32_t ncol0 = nb * G::kUnitCols + j * 256 + part * 64;  // first column of D here
        const bool store = m0 < prm.M && ncol0 < prm.N;                 // uniform across the warp
        // the warp's 64 columns into registers as bf16 pairs, then the accumulator goes back
        // to the MMA thread before the (possibly waiting) staging and store
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t a[32];
          __syncwarp();
          if (live) {
            tmem_ld_32x32b_x32(tq + acc * kBufCols + part * 64 + q * 32, a);
            tmem_ld_wait();
          }
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[16 * q + i] =
                live ? pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])) : 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (lead)
            mbar_arrive_relaxed(acc_empty + acc);
          else
            mbar_arrive_cluster_relaxed(cluster_map(smem_u32(acc_empty + acc), 0));
        }
        if (store) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {   // the warp's 64 columns as two 32 x 32 blocks
            if (lane == 0) bulk_wait_group_read<0>();   // the previous store has read the block
            __syncwarp();
            uint4 *row = reinterpret_cast<uint4 *>(stg + lane * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              row[c ^ ((lane >> 1) & 3)] =
                  make_uint4(pk[16 * h + 4 * c], pk[16 * h + 4 * c + 1], pk[16 * h + 4 * c + 2],
                             pk[16 * h + 4 * c + 3]);
            fence_proxy_async_shared();   // the block, written by threads, is read by the TMA
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_d, stg, ncol0 + 32 * h, e * prm.M + m0);
              bulk_commit_group();
            }
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();   // every block written before the CTA exits
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (threadIdx.x == 0 && (*abort || ld_cluster_u32(peer_abort) != 0u)) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kAbortGraceNs) __nanosleep(1000);
  }
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Rows [offsets[e] + counts[e], offsets[e] + roundup(counts[e], 64)) of a [P, width] bf16
// buffer set to zero: the rows the weight-gradient GEMMs read past an expert's live rows.
// One block per expert, 16-byte stores.
__global__ void __launch_bounds__(256)
    zero_pad_rows_kernel(uint16_t *__restrict__ buf, int32_t width, const int32_t *__restrict__ offsets,
                         const int32_t *__restrict__ counts, int32_t E) {
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int32_t c = counts[e];
    const int32_t r0 = offsets[e] + c;
    const int32_t r1 = offsets[e] + ((c + kBK - 1) / kBK) * kBK;
    const int32_t vpr = width / 8;
    const int64_t n = (int64_t)(r1 - r0) * vpr;
    uint4 *base = reinterpret_cast<uint4 *>(buf + (size_t)r0 * width);
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) base[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

cudaError_t launch_zero_pad_rows(const moe_shape &s, void *buf, int32_t width,
                                 const moe_plan_buffers &p, int num_sms, cudaStream_t st) {
  const int grid = s.E < num_sms * 4 ? s.E : num_sms * 4;
  zero_pad_rows_kernel<<<grid, 256, 0, st>>>(static_cast<uint16_t *>(buf), width, p.offsets,
                                            p.counts, s.E);
  return cudaGetLastError();
}

// Cluster fit of one kernel variant per device, found once (under a lock: host threads may
// launch at the same time). Internal linkage: the static locals of a function template with
// external linkage are one object per process, shared by every copy of this library that is
// loaded, and another copy's cache would skip this copy's shared-memory attribute.
template <bool kWide>
static int wgrad_fit(int dev, cudaLaunchConfig_t lc) {
  static std::mutex mu;
  static int fit[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (fit[dev] == 0) {
    if (cudaFuncSetAttribute(wgrad_pair_kernel<kWide>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             WgradGeom<kWide>::kSmemBytes) != cudaSuccess)
      return 0;
    lc.gridDim = dim3(2, 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, wgrad_pair_kernel<kWide>, &lc) != cudaSuccess || n < 1)
      return 0;
    fit[dev] = n;
  }
  return fit[dev];
}

template <bool kWide>
static int launch_wgrad_t(const moe_shape &s, const CUtensorMap &ta, const CUtensorMap &tb,
                   const CUtensorMap &td, int32_t M, int32_t N, void *D,
                   const moe_plan_buffers &p, int32_t *sched, const moe_config &cfg, int num_sms,
                   cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = WgradGeom<kWide>::kSmemBytes;
  lc.attrs = at;
  lc.numAttrs = 1;
  const int fit = wgrad_fit<kWide>(dev, lc);
  if (fit < 1) return MOE_ERR_CUDA;
  int clusters = (cfg.ffn_ctas > 0 ? cfg.ffn_ctas : num_sms) / 2;
  if (clusters < 1) clusters = 1;
  if (clusters > fit) clusters = fit;
  WgradParams prm{};
  prm.offsets = p.offsets;
  prm.counts = p.counts;
  prm.status = p.status;
  prm.out = static_cast<uint16_t *>(D);
  prm.E = s.E;
  prm.M = M;
  prm.N = N;
  prm.mb_count = (M + 255) / 256;
  prm.nb_count = (N + WgradGeom<kWide>::kUnitCols - 1) / WgradGeom<kWide>::kUnitCols;
  prm.sched = sched;
  prm.timeout_ns = (uint64_t)(cfg.wait_timeout_us > 0 ? cfg.wait_timeout_us : 2000000) * 1000ull;
  lc.gridDim = dim3(2 * clusters, 1, 1);
  lc.stream = st;
  if (cudaLaunchKernelEx(&lc, wgrad_pair_kernel<kWide>, ta, tb, td, prm) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

#ifndef MOE_WGRAD_WIDE
#define MOE_WGRAD_WIDE 1
#endif

// D [E, M, N] = per expert A_e^T B_e over the expert's segment; A [P_max, M], B [P_max, N].
int launch_wgrad(const moe_shape &s, const void *A, int32_t M, const void *B, int32_t N,
                 void *D, const moe_plan_buffers &p, int32_t *sched, const moe_config &cfg,
                 int num_sms, cudaStream_t st) {
  const PlanGeom g = plan_geom(s);
  CUtensorMap ta, tb, td;
  const uint64_t rows = g.pmax > 0 ? (uint64_t)g.pmax : 1;
  if (!make_tmap(&ta, A, (uint64_t)M, rows, kBK) || !make_tmap(&tb, B, (uint64_t)N, rows, kBK) ||
      !make_tmap_box(&td, D, (uint64_t)N, (uint64_t)s.E * M, 32, 32, 64))
    return MOE_ERR_CUDA;
  if (MOE_WGRAD_WIDE)
    return launch_wgrad_t<true>(s, ta, tb, td, M, N, D, p, sched, cfg, num_sms, st);
  return launch_wgrad_t<false>(s, ta, tb, td, M, N, D, p, sched, cfg, num_sms, st);
}

}  // namespace moe
