// C ABI of libmoe.so (declared in include/moe.h): argument checks, plan arena
// layout, and the ordering of the layer's kernels on the caller's communicate
// and compute streams (StreamEP README, How it works, "Caller-owned streams").
#include <mutex>
#include <string.h>

#include "moe_common.cuh"
#include "moe_internal.h"

using namespace moe;

namespace {

int sm_count_cached(int *out) {
  static int counts[64] = {0};
  static int ok[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!ok[dev]) {
    int major = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (major != 10) return MOE_ERR_NO_DEVICE;
    counts[dev] = n;
    ok[dev] = 1;
  }
  *out = counts[dev];
  return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const moe_shape *s, bool need_ffn) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E <= 0 || s->k <= 0) return MOE_ERR_INVALID_ARG;
  if (s->k > kMaxTopK || s->E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (s->tile != 64 && s->tile != 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->H % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (dispatch_smem_bytes(s->H) > kMaxSmemPerBlock) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (need_ffn && (s->I <= 0 || s->I % 64 != 0)) return MOE_ERR_UNSUPPORTED_SHAPE;
  const PlanGeom g = plan_geom(*s);
  if (g.pairs > INT32_MAX || g.pmax > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if ((int64_t)s->E * s->H > INT32_MAX || (int64_t)s->E * (s->I > 0 ? s->I : 0) > INT32_MAX)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int check_plan(const moe_plan_buffers *p) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (!p->counts || !p->offsets || !p->pool_row || !p->row_src || !p->tile_expert || !p->mblk ||
      !p->meta || !p->tile_flags || !p->workspace || !p->status)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int check_config(const moe_config &c) {
  if (c.ffn_kernel != 0 && c.ffn_kernel != MOE_FFN_ONE_SM && c.ffn_kernel != MOE_FFN_SM_PAIR)
    return MOE_ERR_INVALID_ARG;
  if (c.ffn_ctas < 0 || c.wait_timeout_us < 0) return MOE_ERR_INVALID_ARG;
  if (c.gate_up != nullptr && (c.ffn_kernel == MOE_FFN_ONE_SM ||
                               (MOE_FFN_DEFAULT == MOE_FFN_ONE_SM && c.ffn_kernel == 0)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(c.gate_up)) return MOE_ERR_MISALIGNED;
  if (c.early_combine != 0 && c.early_combine != 1) return MOE_ERR_INVALID_ARG;
  if (c.early_combine && (c.ffn_kernel == MOE_FFN_ONE_SM ||
                          (MOE_FFN_DEFAULT == MOE_FFN_ONE_SM && c.ffn_kernel == 0)))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

constexpr int kPlanFields = 12;

// Sizes (in 4-byte words) of the plan buffers, in moe_plan_buffers field order.
void plan_sizes(const moe_shape &s, size_t words[kPlanFields]) {
  const PlanGeom g = plan_geom(s);
  words[0] = (size_t)s.E;
  words[1] = (size_t)s.E + 1;
  words[2] = (size_t)g.pairs;
  words[3] = (size_t)g.pmax;
  words[4] = (size_t)g.n_tiles;
  words[5] = kMblkInts * (size_t)g.n_tiles;
  words[6] = 8;
  words[7] = (size_t)g.n_tiles;
  words[8] = plan_workspace_ints(s);
  words[9] = 4;
  words[10] = (size_t)s.T;
  words[11] = (size_t)s.T + 4;
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Expert parallelism: rank shape checks, and the EP plan arena (the all-expert prefix, then
// the rank's pool plan, whose scratch must also hold the per-source counts of its experts).
int check_ep(const moe_shape *s, int32_t R) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if (R < 1 || R > kMaxEpRanks || s->E % R != 0) return MOE_ERR_INVALID_ARG;
  if ((int64_t)s->T * R > INT32_MAX) return MOE_ERR_INVALID_ARG;
  const moe_shape g = ep_global_shape(*s, R);
  return check_shape(&g, false);
}

constexpr int kEpFields = 6;
void ep_sizes(const moe_shape &s, int32_t R, size_t words[kEpFields + kPlanFields]) {
  const moe_shape g = ep_global_shape(s, R), l = ep_local_shape(s, R);
  const PlanGeom gg = plan_geom(g);
  words[0] = (size_t)s.E;
  words[1] = (size_t)s.E + 1;
  words[2] = (size_t)s.E * R + 8;
  words[3] = (size_t)gg.n_tiles;
  words[4] = kMblkInts * (size_t)gg.n_tiles;
  words[5] = 8;
  plan_sizes(l, words + kEpFields);
  const size_t need = (size_t)(s.E / R) * R + 8;
  if (words[kEpFields + 8] < need) words[kEpFields + 8] = need;
}

// The grouped FFN's host checks and launch, for moe_grouped_ffn (topk_w / out NULL),
// moe_grouped_ffn_combine (both set) and moe_forward (which may pass a helper stream and
// event for the streaming layer's second GEMM A launch).
int grouped_ffn_entry(const moe_shape *s, const void *pool, const void *W1, const void *W2,
                      const moe_plan_buffers *p, void *act, void *ypool, const float *topk_w,
                      void *out, const moe_config *cfg, bool combine, cudaStream_t st,
                      cudaStream_t helper_stream, cudaEvent_t helper_done) {
  int rc = check_shape(s, true);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (!pool || !W1 || !W2 || !act || !ypool) return MOE_ERR_INVALID_ARG;
  if (combine && (!p->tok_pending || !p->ready)) return MOE_ERR_INVALID_ARG;
  if (combine && s->T > 0 && (!topk_w || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(pool) || !aligned16(W1) || !aligned16(W2) || !aligned16(act) ||
      !aligned16(ypool) || !aligned16(out))
    return MOE_ERR_MISALIGNED;
  moe_config c{};
  if (cfg != nullptr) c = *cfg;
  if ((rc = check_config(c)) != MOE_OK) return rc;
  if ((c.early_combine != 0) != combine) return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  return launch_ffn(*s, pool, W1, W2, *p, act, ypool, combine ? topk_w : nullptr,
                    combine ? out : nullptr, c, nsm, st, helper_stream, helper_done);
}

}  // namespace

extern "C" {

int moe_packed_weight_bytes(const moe_shape *s, size_t *w1p_bytes, size_t *w2p_bytes) {
  int rc = check_shape(s, true);
  if (rc != MOE_OK) return rc;
  if (w1p_bytes == nullptr || w2p_bytes == nullptr) return MOE_ERR_INVALID_ARG;
  const PackGeom g = pack_geom(*s);
  *w1p_bytes = (size_t)g.tiles1 * 128 * 64 * 2;
  *w2p_bytes = (size_t)g.tiles2 * 128 * 64 * 2;
  return MOE_OK;
}

int moe_pack_weights(const moe_shape *s, const void *W1, const void *W2, void *W1p, void *W2p,
                     void *stream) {
  int rc = check_shape(s, true);
  if (rc != MOE_OK) return rc;
  if (!W1 || !W2 || !W1p || !W2p) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W1) || !aligned16(W2) || !aligned16(W1p) || !aligned16(W2p))
    return MOE_ERR_MISALIGNED;
  const PackGeom g = pack_geom(*s);
  if ((g.tiles1 + g.tiles2) * 128 > INT32_MAX) return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_pack(*s, W1, W2, W1p, W2p, nsm, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_pool_rows_max(const moe_shape *s, int64_t *rows_out) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if (rows_out == nullptr) return MOE_ERR_INVALID_ARG;
  *rows_out = plan_geom(*s).pmax;
  return MOE_OK;
}

int moe_plan_arena_bytes(const moe_shape *s, size_t *bytes_out) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if (bytes_out == nullptr) return MOE_ERR_INVALID_ARG;
  size_t w[kPlanFields];
  plan_sizes(*s, w);
  size_t total = 0;
  for (int i = 0; i < kPlanFields; ++i) total += round256(w[i] * 4);
  *bytes_out = total;
  return MOE_OK;
}

int moe_plan_bind(const moe_shape *s, void *arena, moe_plan_buffers *out) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if (arena == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(arena) & 255u) != 0) return MOE_ERR_MISALIGNED;
  size_t w[kPlanFields];
  plan_sizes(*s, w);
  char *base = static_cast<char *>(arena);
  void *ptrs[kPlanFields];
  for (int i = 0; i < kPlanFields; ++i) {
    ptrs[i] = base;
    base += round256(w[i] * 4);
  }
  out->counts = static_cast<int32_t *>(ptrs[0]);
  out->offsets = static_cast<int32_t *>(ptrs[1]);
  out->pool_row = static_cast<int32_t *>(ptrs[2]);
  out->row_src = static_cast<int32_t *>(ptrs[3]);
  out->tile_expert = static_cast<int32_t *>(ptrs[4]);
  out->mblk = static_cast<int32_t *>(ptrs[5]);
  out->meta = static_cast<int32_t *>(ptrs[6]);
  out->tile_flags = static_cast<uint32_t *>(ptrs[7]);
  out->workspace = static_cast<int32_t *>(ptrs[8]);
  out->status = static_cast<int32_t *>(ptrs[9]);
  out->tok_pending = static_cast<int32_t *>(ptrs[10]);
  out->ready = static_cast<int32_t *>(ptrs[11]);
  return MOE_OK;
}

int moe_plan(const moe_shape *s, const int32_t *topk_idx, const moe_plan_buffers *p,
             int32_t *host_P, void *stream) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (topk_idx == nullptr && s->T > 0) return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_plan(*s, topk_idx, *p, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (host_P != nullptr) {
    if (cudaMemcpyAsync(host_P, p->meta + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_route(const moe_shape *s, const float *logits, const float *bias, int32_t *topk_idx,
              float *topk_w, void *stream) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if (s->k > s->E) return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_route(*s, logits, bias, topk_idx, topk_w, nullptr, nsm,
                   static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_route_plan(const moe_shape *s, const float *logits, const float *bias, int32_t *topk_idx,
                   float *topk_w, const moe_plan_buffers *p, int32_t *host_P, void *stream) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (s->k > s->E) return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_route(*s, logits, bias, topk_idx, topk_w, p, nsm, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (host_P != nullptr &&
      cudaMemcpyAsync(host_P, p->meta + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_dispatch(const moe_shape *s, const void *x, const moe_plan_buffers *p, void *pool,
                 int32_t signal_flags, void *stream) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if ((x == nullptr && s->T > 0) || pool == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(pool)) return MOE_ERR_MISALIGNED;
  // a mask of MOE_DISPATCH_SIGNAL_TILES and MOE_DISPATCH_ARM_COMBINE; any other non-zero
  // value keeps its old meaning (tile flags only)
  int flags = signal_flags;
  if (flags & ~(MOE_DISPATCH_SIGNAL_TILES | MOE_DISPATCH_ARM_COMBINE))
    flags = MOE_DISPATCH_SIGNAL_TILES;
  if ((flags & MOE_DISPATCH_ARM_COMBINE) && (!p->tok_pending || !p->ready))
    return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_dispatch(*s, x, *p, pool, flags, nsm, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_grouped_ffn(const moe_shape *s, const void *pool, const void *W1, const void *W2,
                    const moe_plan_buffers *p, void *act, void *ypool, const moe_config *cfg,
                    void *stream) {
  // early combine is moe_grouped_ffn_combine's
  return grouped_ffn_entry(s, pool, W1, W2, p, act, ypool, nullptr, nullptr, cfg, false,
                           static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int moe_grouped_ffn_combine(const moe_shape *s, const void *pool, const void *W1, const void *W2,
                            const moe_plan_buffers *p, void *act, void *ypool,
                            const float *topk_w, void *out, const moe_config *cfg,
                            void *stream) {
  return grouped_ffn_entry(s, pool, W1, W2, p, act, ypool, topk_w, out, cfg, true,
                           static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int moe_combine(const moe_shape *s, const void *ypool, const float *topk_w,
                const moe_plan_buffers *p, void *out, void *stream) {
  int rc = check_shape(s, false);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (s->T > 0 && (!ypool || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ypool) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_combine(*s, ypool, topk_w, *p, out, nsm, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"

namespace {

// The backward on one stream (comm == compute, no events) or, with cfg->streaming, with the
// combine backward on comm in pool-tile order while backward Y on compute takes the tiles
// as their flags fill (the mirror of the streaming forward).
int backward_entry(const moe_shape *s, const void *dy, const float *topk_w, const void *W1,
                   const void *W2, const moe_plan_buffers *p, const void *pool, void *act,
                   const void *ypool, void *gu, void *dgu, void *dpool, void *dx, float *dw,
                   void *dW1, void *dW2, const moe_config *cfg, cudaStream_t comm,
                   cudaStream_t st, cudaEvent_t ev_a, cudaEvent_t ev_b) {
  int rc = check_shape(s, true);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (!W1 || !W2 || !pool || !ypool || !dgu || !dpool) return MOE_ERR_INVALID_ARG;
  if (!gu && !(cfg != nullptr && cfg->gate_up != nullptr)) return MOE_ERR_INVALID_ARG;
  if (s->T > 0 && (!dy || !topk_w || !dx || !dw)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(W1) || !aligned16(W2) || !aligned16(pool) ||
      !aligned16(ypool) || !aligned16(gu) || !aligned16(dgu) || !aligned16(dpool) ||
      !aligned16(dx) || !aligned16(act) || !aligned16(dW1) || !aligned16(dW2))
    return MOE_ERR_MISALIGNED;
  if (dW2 != nullptr && act == nullptr) return MOE_ERR_INVALID_ARG;
  moe_config c{};
  if (cfg != nullptr) c = *cfg;
  if ((rc = check_config(c)) != MOE_OK) return rc;
  if (c.packed_weights || c.ffn_kernel == MOE_FFN_ONE_SM) return MOE_ERR_INVALID_ARG;
  const bool streaming = c.streaming && s->T > 0;
  if (c.streaming && (comm == st || ev_a == nullptr || ev_b == nullptr))
    return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  cudaEvent_t const *tev = reinterpret_cast<cudaEvent_t const *>(c.timing_events);
  if (tev != nullptr && cudaEventRecord(tev[0], st) != cudaSuccess) return MOE_ERR_CUDA;
  // early_combine: the dispatch backward folds into backward A (the mirror of early combine)
  const bool early = c.early_combine && s->T > 0;
  if (early && (!p->tok_pending || !p->ready)) return MOE_ERR_INVALID_ARG;
  if (early && launch_arm_tokens(*s, *p, nsm, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (streaming) {
    // flags and dw cleared in stream order before either stream starts on them
    const PlanGeom g = plan_geom(*s);
    if (cudaMemsetAsync(p->tile_flags, 0, sizeof(uint32_t) * (size_t)g.n_tiles, st) !=
            cudaSuccess ||
        cudaMemsetAsync(dw, 0, sizeof(float) * (size_t)s->T * s->k, st) != cudaSuccess ||
        cudaEventRecord(ev_a, st) != cudaSuccess || cudaStreamWaitEvent(comm, ev_a, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    // 8 blocks of 128 threads for each of the SMs that backward Y leaves free: the combine
    // backward never depends on finding room beside backward Y's CTAs (which wait for it)
    if (launch_combine_backward_tiles(*s, dy, ypool, topk_w, *p, dpool, dw,
                                      kStreamDispatchSMs * 8, comm) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (tev != nullptr && cudaEventRecord(tev[1], comm) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventRecord(ev_b, comm) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    if (launch_combine_backward(*s, dy, ypool, topk_w, *p, dpool, dw, nsm, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (tev != nullptr && cudaEventRecord(tev[1], st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if ((rc = launch_ffn_backward(*s, W1, W2, *p, pool, act, dpool, gu, dgu, dW1, dW2, c, nsm, st,
                                tev, early ? dx : nullptr, streaming ? ev_b : nullptr)) != MOE_OK)
    return rc;
  if (!early && launch_combine(*s, dpool, nullptr, *p, dx, nsm, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[7], st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_backward(const moe_shape *s, const void *dy, const float *topk_w, const void *W1,
                 const void *W2, const moe_plan_buffers *p, const void *pool, void *act,
                 const void *ypool, void *gu, void *dgu, void *dpool, void *dx, float *dw,
                 void *dW1, void *dW2, const moe_config *cfg, void *stream) {
  if (cfg != nullptr && cfg->streaming) return MOE_ERR_INVALID_ARG;  // needs two streams
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return backward_entry(s, dy, topk_w, W1, W2, p, pool, act, ypool, gu, dgu, dpool, dx, dw, dW1,
                        dW2, cfg, st, st, nullptr, nullptr);
}

int moe_backward_streams(const moe_shape *s, const void *dy, const float *topk_w, const void *W1,
                         const void *W2, const moe_plan_buffers *p, const void *pool, void *act,
                         const void *ypool, void *gu, void *dgu, void *dpool, void *dx, float *dw,
                         void *dW1, void *dW2, const moe_config *cfg, void *comm_stream,
                         void *compute_stream, void *ev_a, void *ev_b) {
  return backward_entry(s, dy, topk_w, W1, W2, p, pool, act, ypool, gu, dgu, dpool, dx, dw, dW1,
                        dW2, cfg, static_cast<cudaStream_t>(comm_stream),
                        static_cast<cudaStream_t>(compute_stream),
                        static_cast<cudaEvent_t>(ev_a), static_cast<cudaEvent_t>(ev_b));
}

int moe_forward(const moe_shape *s, const void *x, const int32_t *topk_idx, const float *topk_w,
                const void *W1, const void *W2, const moe_plan_buffers *p, void *pool, void *act,
                void *ypool, void *out, const moe_config *cfg, void *comm_stream,
                void *compute_stream, void *ev_plan, void *ev_dispatch) {
  const bool identity = (W1 == nullptr && W2 == nullptr);
  int rc = check_shape(s, !identity);
  if (rc != MOE_OK) return rc;
  if ((rc = check_plan(p)) != MOE_OK) return rc;
  if (ev_plan == nullptr || ev_dispatch == nullptr) return MOE_ERR_INVALID_ARG;
  if ((W1 == nullptr) != (W2 == nullptr)) return MOE_ERR_INVALID_ARG;
  moe_config c{};
  if (cfg != nullptr) c = *cfg;
  if ((rc = check_config(c)) != MOE_OK) return rc;
  cudaStream_t comm = static_cast<cudaStream_t>(comm_stream);
  cudaStream_t comp = static_cast<cudaStream_t>(compute_stream);
  cudaEvent_t evp = static_cast<cudaEvent_t>(ev_plan);
  cudaEvent_t evd = static_cast<cudaEvent_t>(ev_dispatch);
  // The plan buffers and the pool are reused: wait for the previous call's compute work.
  if (comm != comp) {
    if (cudaEventRecord(evd, comp) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(comm, evd, 0) != cudaSuccess) return MOE_ERR_CUDA;
  }
  cudaEvent_t const *tev = reinterpret_cast<cudaEvent_t const *>(c.timing_events);
  if (tev != nullptr && cudaEventRecord(tev[0], comm) != cudaSuccess) return MOE_ERR_CUDA;
  if ((rc = moe_plan(s, topk_idx, p, nullptr, comm)) != MOE_OK) return rc;
  if (cudaEventRecord(evp, comm) != cudaSuccess) return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[1], comm) != cudaSuccess) return MOE_ERR_CUDA;
  const bool early = !identity && c.early_combine;
  const int signal = ((!identity && c.streaming) ? MOE_DISPATCH_SIGNAL_TILES : 0) |
                     (early ? MOE_DISPATCH_ARM_COMBINE : 0);
  if ((rc = moe_dispatch(s, x, p, pool, signal, comm)) != MOE_OK) return rc;
  if (cudaEventRecord(evd, comm) != cudaSuccess) return MOE_ERR_CUDA;
  if (tev != nullptr && cudaEventRecord(tev[2], comm) != cudaSuccess) return MOE_ERR_CUDA;
  if (!identity) {
    if (cudaStreamWaitEvent(comp, c.streaming ? evp : evd, 0) != cudaSuccess) return MOE_ERR_CUDA;
    // streaming: the FFN's second GEMM A launch goes on the communicate stream behind
    // dispatch; evp, already waited for above, is recorded again after it
    if ((rc = grouped_ffn_entry(s, pool, W1, W2, p, act, ypool, topk_w, out, &c, early, comp,
                                c.streaming ? comm : nullptr, c.streaming ? evp : nullptr)) !=
        MOE_OK)
      return rc;
  }
  if (early) {
    // GEMM Y combined each token as its rows completed; no separate combine launch
    if (cudaStreamWaitEvent(comp, evd, 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (tev != nullptr && cudaEventRecord(tev[6], comp) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (cudaStreamWaitEvent(comp, evd, 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (identity && tev != nullptr) {
    for (int i = 3; i < 6; ++i)
      if (cudaEventRecord(tev[i], comp) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if ((rc = moe_combine(s, identity ? pool : ypool, topk_w, p, out, comp)) != MOE_OK) return rc;
  if (tev != nullptr && cudaEventRecord(tev[6], comp) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_events_create(void **events, int32_t n) {
  if (events == nullptr || n < 0) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    events[i] = e;
  }
  return MOE_OK;
}

int moe_timing_events_create(void **events, int32_t n) {
  if (events == nullptr || n < 0) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
    events[i] = e;
  }
  return MOE_OK;
}

int moe_event_elapsed_ms(void *start, void *end, float *ms) {
  if (start == nullptr || end == nullptr || ms == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaEventElapsedTime(ms, static_cast<cudaEvent_t>(start), static_cast<cudaEvent_t>(end)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_events_destroy(void **events, int32_t n) {
  if (events == nullptr || n < 0) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (events[i] != nullptr) cudaEventDestroy(static_cast<cudaEvent_t>(events[i]));
  return MOE_OK;
}

int moe_get_status(const moe_plan_buffers *p, int32_t *code, int32_t *aux) {
  if (p == nullptr || p->status == nullptr || code == nullptr) return MOE_ERR_INVALID_ARG;
  int32_t h[2] = {0, 0};
  if (cudaMemcpy(h, p->status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  *code = h[0];
  if (aux != nullptr) *aux = h[1];
  return MOE_OK;
}

int moe_clear_status(const moe_plan_buffers *p, void *stream) {
  if (p == nullptr || p->status == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p->status, 0, 4 * sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  // the grouped GEMMs' unit counters (meta[4..7]), so that a GEMM run again on the same
  // plan after a failed one starts from its first unit
  if (p->meta != nullptr &&
      cudaMemsetAsync(p->meta + 4, 0, 4 * sizeof(int32_t), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

const char *moe_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (H, I multiples of 64; tile 64 or 128)";
    case MOE_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_NO_DEVICE: return "current device is not sm_100";
    case MOE_ERR_SCRATCH_LIMIT:
      return "shape needs more plan scratch than moe_plan_noalloc's static buffer holds";
    case MOE_ERR_BAD_INDEX: return "topk_idx value outside [-1, E)";
    case MOE_ERR_FLAG_TIMEOUT: return "streaming FFN timed out waiting for a pool tile";
    case MOE_ERR_POOL_OVERFLOW: return "pool rows exceeded the dropless bound";
    case MOE_ERR_PIPE_TIMEOUT: return "FFN pipeline wait timed out";
    case MOE_ERR_COMBINE_TIMEOUT: return "early combine timed out waiting for a token's rows";
    default: return "unknown error";
  }
}

int moe_ep_local_shape(const moe_shape *s, int32_t R, moe_shape *out) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = ep_local_shape(*s, R);
  return MOE_OK;
}

int moe_ep_pool_rows(const moe_shape *s, int32_t R, int64_t *rows_out) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (rows_out == nullptr) return MOE_ERR_INVALID_ARG;
  *rows_out = plan_geom(ep_local_shape(*s, R)).pmax;
  return MOE_OK;
}

int moe_ep_arena_bytes(const moe_shape *s, int32_t R, size_t *bytes_out) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (bytes_out == nullptr) return MOE_ERR_INVALID_ARG;
  size_t w[kEpFields + kPlanFields];
  ep_sizes(*s, R, w);
  size_t total = 0;
  for (int i = 0; i < kEpFields + kPlanFields; ++i) total += round256(w[i] * 4);
  *bytes_out = total;
  return MOE_OK;
}

int moe_ep_bind(const moe_shape *s, int32_t R, void *arena, moe_ep_plan *out) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (arena == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(arena) & 255u) != 0) return MOE_ERR_MISALIGNED;
  size_t w[kEpFields + kPlanFields];
  ep_sizes(*s, R, w);
  char *base = static_cast<char *>(arena);
  int32_t *ptrs[kEpFields + kPlanFields];
  for (int i = 0; i < kEpFields + kPlanFields; ++i) {
    ptrs[i] = reinterpret_cast<int32_t *>(base);
    base += round256(w[i] * 4);
  }
  out->counts = ptrs[0];
  out->offsets = ptrs[1];
  out->src_base = ptrs[2];
  out->tile_expert = ptrs[3];
  out->mblk = ptrs[4];
  out->meta = ptrs[5];
  int32_t *const *q = ptrs + kEpFields;
  moe_plan_buffers &l = out->local;
  l.counts = q[0];
  l.offsets = q[1];
  l.pool_row = q[2];
  l.row_src = q[3];
  l.tile_expert = q[4];
  l.mblk = q[5];
  l.meta = q[6];
  l.tile_flags = reinterpret_cast<uint32_t *>(q[7]);
  l.workspace = q[8];
  l.status = q[9];
  l.tok_pending = q[10];
  l.ready = q[11];
  return MOE_OK;
}

int moe_ep_layout(const moe_shape *s, int32_t R, int32_t rank, const int32_t *all_counts,
                  const moe_ep_plan *ep, void *pool, void *stream) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (rank < 0 || rank >= R || all_counts == nullptr || ep == nullptr || pool == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((rc = check_plan(&ep->local)) != MOE_OK) return rc;
  if (!ep->counts || !ep->offsets || !ep->src_base || !ep->tile_expert || !ep->mblk || !ep->meta)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(pool)) return MOE_ERR_MISALIGNED;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_ep_layout(*s, R, rank, all_counts, *ep, pool, nsm,
                       static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

namespace {
int check_ep_call(const moe_shape *s, int32_t R, int32_t rank, const moe_plan_buffers *own,
                  const moe_ep_plan *ep, void *const *peers) {
  int rc = check_ep(s, R);
  if (rc != MOE_OK) return rc;
  if (rank < 0 || rank >= R || own == nullptr || ep == nullptr || peers == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((rc = check_plan(own)) != MOE_OK) return rc;
  if (!ep->offsets || !ep->src_base) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < R; ++i) {
    if (peers[i] == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(peers[i])) return MOE_ERR_MISALIGNED;
  }
  return MOE_OK;
}
}  // namespace

int moe_ep_dispatch(const moe_shape *s, int32_t R, int32_t rank, const void *x,
                    const moe_plan_buffers *own, const moe_ep_plan *ep, void *const *pools,
                    uint32_t *const *tile_flags, void *stream) {
  int rc = check_ep_call(s, R, rank, own, ep, pools);
  if (rc != MOE_OK) return rc;
  if (x == nullptr && s->T > 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x)) return MOE_ERR_MISALIGNED;
  if (tile_flags != nullptr)
    for (int i = 0; i < R; ++i)
      if (tile_flags[i] == nullptr || (reinterpret_cast<uintptr_t>(tile_flags[i]) & 3u) != 0)
        return MOE_ERR_INVALID_ARG;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_ep_dispatch(*s, R, rank, x, *own, *ep, pools, tile_flags, nsm,
                         static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_ep_combine(const moe_shape *s, int32_t R, int32_t rank, void *const *ypools,
                   const float *topk_w, const moe_plan_buffers *own, const moe_ep_plan *ep,
                   void *out, void *stream) {
  int rc = check_ep_call(s, R, rank, own, ep, ypools);
  if (rc != MOE_OK) return rc;
  if (s->T > 0 && (topk_w == nullptr || out == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out)) return MOE_ERR_MISALIGNED;
  int nsm;
  if ((rc = sm_count_cached(&nsm)) != MOE_OK) return rc;
  if (launch_ep_combine(*s, R, rank, ypools, topk_w, *own, *ep, out, nsm,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

const char *moe_version(void) { return "moe-b200 0.2 (sm_100a)"; }

}  // extern "C"
