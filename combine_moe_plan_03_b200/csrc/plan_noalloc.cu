// moe_plan_noalloc: the routing plan with its scratch in a static device buffer
// owned by this library, for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host framework that owns the whole
// device-memory budget and hands its extensions no allocator (an inference
// engine's plugin hook, for instance), and latency-critical loops where a
// cudaMalloc (which may synchronise the device, and may fail once a fixed
// memory budget is spent) is not acceptable. moe_plan needs a caller-sized
// workspace (per-expert counts for every 256-pair chunk plus one counter);
// this variant keeps that workspace in g_plan_scratch below instead, so the
// caller only passes the inputs and the plan outputs.
//
// Limits and rules:
//   - g_plan_scratch holds kNoallocScratchInts int32 (2 MiB + 256 B). A shape
//     needs E * max(1, ceil(T*k / 256)) + 8 of them; larger shapes are rejected
//     with MOE_ERR_SCRATCH_LIMIT before anything is launched. Every GPU that
//     loads the library keeps this buffer until the process exits.
//   - All calls on a device share the one buffer, and it keeps whatever the last
//     call left there. The first kernel of each call overwrites every count it
//     reads and zeroes the finalize counter, so no state leaks between calls
//     that run one after the other; calls that overlap on the GPU (concurrent
//     streams) race on the buffer and must not be issued.
//   - The device address of the buffer is looked up once per device, on the first
//     call made with that device current (cudaGetSymbolAddress). Make that first
//     call before any stream capture.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr size_t kNoallocScratchInts = (size_t(1) << 19) + 64;

static __device__ __align__(256) int32_t g_plan_scratch[kNoallocScratchInts];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
int32_t *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_plan_scratch on the current device (looked up once per device).
int scratch_for_current_device(int32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_plan_scratch) != cudaSuccess || ptr == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t *>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_plan_noalloc(const moe_shape *s, const int32_t *topk_idx,
                                const moe_plan_buffers *p, int32_t *host_P, void *stream) {
  if (s == nullptr || p == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E <= 0 || s->k <= 0 || s->k > kMaxTopK ||
      s->E > kMaxExperts)
    return MOE_ERR_INVALID_ARG;
  if (s->tile != 64 && s->tile != 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->H % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const PlanGeom g = plan_geom(*s);
  if (g.pairs > INT32_MAX || g.pmax > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (plan_workspace_ints(*s) > kNoallocScratchInts) return MOE_ERR_SCRATCH_LIMIT;
  if (!p->counts || !p->offsets || !p->pool_row || !p->row_src || !p->tile_expert || !p->mblk ||
      !p->meta || !p->tile_flags || !p->status)
    return MOE_ERR_INVALID_ARG;
  if (topk_idx == nullptr && s->T > 0) return MOE_ERR_INVALID_ARG;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_NO_DEVICE;
  int32_t *scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  moe_plan_buffers q = *p;
  q.workspace = scratch;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_plan(*s, topk_idx, q, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (host_P != nullptr &&
      cudaMemcpyAsync(host_P, p->meta + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
