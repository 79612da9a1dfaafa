// Launchers shared between the kernel files and the C ABI (moe_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Pairs per plan chunk (one warp counts and ranks one chunk) and warps per block.
constexpr int kPlanChunk = 256;
constexpr int kPlanWarps = 8;
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kGemmBlockM = 256;  // most live rows of one expert in one grouped-GEMM unit
// GEMM row-chunk table entry: {first row, expert, live rows, expert's first chunk, expert's
// chunk count}
constexpr int kMblkInts = 5;
constexpr size_t kMaxSmemPerBlock = 232448;  // opt-in dynamic shared memory per block (227 KB)
constexpr int kMaxEpRanks = MOE_EP_MAX_RANKS;  // expert-parallel ranks (GPUs of one node)

// Expert parallelism: the shapes of the plan over all ranks' pairs (E global experts) and of
// one rank's pool (its E / R experts), for R ranks of T tokens each.
inline moe_shape ep_global_shape(const moe_shape &s, int32_t R) {
  return moe_shape{s.T * R, s.H, s.I, s.E, s.k, s.tile};
}
inline moe_shape ep_local_shape(const moe_shape &s, int32_t R) {
  return moe_shape{s.T * R, s.H, s.I, s.E / R, s.k, s.tile};
}

// Streaming (moe_config.streaming): SMs left to the tile-ordered dispatch while GEMM A
// claims tiles on the others.
constexpr int kStreamDispatchSMs = 16;

// Dynamic shared memory of the dispatch kernel: two staging rows of x, one row of zeros
// (H bf16 each) and its barriers. Shapes whose rows do not fit are refused on the host.
inline size_t dispatch_smem_bytes(int32_t H) {
  return 3 * (size_t)H * 2 + 2 * sizeof(uint64_t) + 16;
}

// Rows per grouped-GEMM chunk for an expert with c live rows: the rows are cut into
// ceil(c / 256) chunks of equal size, rounded up to a multiple of 16 (the MMA's N step).
__host__ __device__ inline int32_t gemm_chunk_rows(int32_t c) {
  if (c <= 0) return kGemmBlockM;
  const int32_t n = (c + kGemmBlockM - 1) / kGemmBlockM;
  return ((c + n - 1) / n + 15) & ~15;
}

struct PlanGeom {
  int64_t pairs;     // T * k
  int64_t pmax;      // dropless pool bound
  int64_t n_tiles;   // pmax / tile
  int32_t n_chunks;  // ceil(pairs / kPlanChunk)
};

PlanGeom plan_geom(const moe_shape &s);

// Prepacked weight tiles (pack.cu): 128 rows of 64 bf16 (16 KB) per tile.
struct PackGeom {
  int32_t nb1, kb1;  // W1: 128-column blocks of each of gate / up, 64-row k blocks
  int32_t nb2, kb2;  // W2: 128-column blocks (even count), 64-row k blocks
  int64_t tiles1, tiles2;
};
PackGeom pack_geom(const moe_shape &s);
cudaError_t launch_pack(const moe_shape &s, const void *W1, const void *W2, void *W1p, void *W2p,
                        int num_sms, cudaStream_t st);
size_t plan_workspace_ints(const moe_shape &s);
struct PlanResets;
// What the plan's first kernel resets (row_src, tile tables, flags, early-combine counters).
PlanResets plan_resets(const moe_shape &s, const moe_plan_buffers &p);

cudaError_t launch_plan(const moe_shape &s, const int32_t *topk_idx, const moe_plan_buffers &p,
                        cudaStream_t st);
// The plan's per-expert scan over n_src sources (ws [E][n_src] of counts, scanned in place;
// *done zero) and the tables it builds: counts, offsets, tile table, row-chunk table, meta.
cudaError_t launch_plan_scan_only(const moe_shape &s, int32_t n_src, int32_t *ws, int32_t *done,
                                  int32_t *counts, int32_t *offsets, int32_t *tile_expert,
                                  int32_t *mblk, int32_t *meta, int32_t *status, cudaStream_t st);
// ep.cu: expert parallelism (layout from all ranks' counts, dispatch into the owners' pools,
// combine from the owners' ypools).
cudaError_t launch_ep_layout(const moe_shape &rank_shape, int32_t R, int32_t rank,
                             const int32_t *C, const moe_ep_plan &ep, void *pool,
                             int num_sms, cudaStream_t st);
cudaError_t launch_ep_dispatch(const moe_shape &rank_shape, int32_t R, int32_t rank,
                               const void *x, const moe_plan_buffers &own, const moe_ep_plan &ep,
                               void *const *pools, uint32_t *const *tile_flags, int num_sms,
                               cudaStream_t st);
cudaError_t launch_ep_combine(const moe_shape &rank_shape, int32_t R, int32_t rank,
                              void *const *ypools, const float *topk_w,
                              const moe_plan_buffers &own, const moe_ep_plan &ep, void *out,
                              int num_sms, cudaStream_t st);
// The plan's second and third launches (per-expert scan + tables, stable rank), after
// ws[e][chunk] holds the per-chunk counts (written by plan_hist_kernel or the router).
cudaError_t launch_plan_scan_rank(const moe_shape &s, const int32_t *topk_idx,
                                  const moe_plan_buffers &p, cudaStream_t st);
cudaError_t launch_route(const moe_shape &s, const float *logits, const float *bias,
                         int32_t *topk_idx, float *topk_w, const moe_plan_buffers *p,
                         int num_sms, cudaStream_t st);
// flags: MOE_DISPATCH_SIGNAL_TILES | MOE_DISPATCH_ARM_COMBINE
cudaError_t launch_dispatch(const moe_shape &s, const void *x, const moe_plan_buffers &p,
                            void *pool, int flags, int num_sms, cudaStream_t st);
cudaError_t launch_combine(const moe_shape &s, const void *ypool, const float *topk_w,
                           const moe_plan_buffers &p, void *out, int num_sms, cudaStream_t st);
cudaError_t launch_arm_tokens(const moe_shape &s, const moe_plan_buffers &p, int num_sms,
                              cudaStream_t st);
cudaError_t launch_combine_backward_tiles(const moe_shape &s, const void *dy, const void *ypool,
                                          const float *topk_w, const moe_plan_buffers &p,
                                          void *dypool, float *dw, int blocks, cudaStream_t st);
cudaError_t launch_combine_backward(const moe_shape &s, const void *dy, const void *ypool,
                                    const float *topk_w, const moe_plan_buffers &p,
                                    void *dypool, float *dw, int num_sms, cudaStream_t st);
// Returns MOE_OK or a MOE_ERR_* code. With dW1 / dW2 (and act) also the weight gradients.
// early_dx: with cfg.early_combine, backward A also writes the dispatch backward into it
// (the token counters armed by launch_arm_tokens first); nullptr: backward A alone.
// combine_done: with cfg.streaming, the event after the tile-ordered combine backward on the
// other stream; st waits for it once backward Y is queued (dW2 and the caller need all of
// dypool and dw).
int launch_ffn_backward(const moe_shape &s, const void *W1, const void *W2,
                        const moe_plan_buffers &p, const void *pool, void *act,
                        void *dypool_dpool, void *gu, void *dgu, void *dW1, void *dW2,
                        const moe_config &cfg, int num_sms, cudaStream_t st,
                        cudaEvent_t const *tev, void *early_dx = nullptr,
                        cudaEvent_t combine_done = nullptr);
// wgrad.cu: D [E, M, N] = per expert A_e^T B_e over its pool segment (rows past the live
// ones must be zero in A and B); and the kernel that zeroes those rows of a buffer.
int launch_wgrad(const moe_shape &s, const void *A, int32_t M, const void *B, int32_t N,
                 void *D, const moe_plan_buffers &p, int32_t *sched, const moe_config &cfg,
                 int num_sms, cudaStream_t st);
cudaError_t launch_zero_pad_rows(const moe_shape &s, void *buf, int32_t width,
                                 const moe_plan_buffers &p, int num_sms, cudaStream_t st);
// Returns MOE_OK or a MOE_ERR_* code. With topk_w / out (cfg.early_combine) GEMM Y also
// combines the tokens into out as their rows complete.
// With cfg.streaming, helper_stream / helper_done (both or neither) let a second launch of
// GEMM A, queued on helper_stream after dispatch, join the first one's unit tickets on the
// SMs dispatch used; st waits for helper_done (recorded after it) before GEMM Y.
int launch_ffn(const moe_shape &s, const void *pool, const void *W1, const void *W2,
               const moe_plan_buffers &p, void *act, void *ypool, const float *topk_w,
               void *out, const moe_config &cfg, int num_sms, cudaStream_t st,
               cudaStream_t helper_stream = nullptr, cudaEvent_t helper_done = nullptr);

// Early combine: a row chunk counts once per token row when all its units (every column
// block, both CTAs of a pair) are stored, so a token with n live pairs waits for
// n * early_combine_arrivals(H) = n counts.
__host__ __device__ inline int32_t early_combine_arrivals(int32_t) {
  return 1;
}

}  // namespace moe
