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
//   - The device address of the buffer is looked up once per device context, on the
//     first call made with that device current (cudaGetSymbolAddress). Make that first
//     call before any stream capture. The address is cached per CUDA context, so a
//     call after cudaDeviceReset (which gives the device a new context and reloads the
//     module) looks it up again instead of reusing a stale one.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr size_t kNoallocScratchInts = (size_t(1) << 19) + 64;

static __device__ __align__(256) int32_t g_plan_scratch[kNoallocScratchInts];

namespace {

// Cached addresses, one per CUDA context, keyed by the context's process-unique id (a
// device's primary context gets a new id when a device reset re-creates it); the oldest
// entry is replaced when the table is full.
constexpr int kCacheSlots = 64;
struct ScratchSlot {
  unsigned long long ctx_id;
  int32_t *ptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch_cache[kCacheSlots] = {};
int g_scratch_next = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

void *driver_entry(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// Id of the context the runtime uses on the current device.
int current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_ctx == nullptr) get_ctx = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
  if (get_id == nullptr) get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  if (get_ctx == nullptr || get_id == nullptr) return MOE_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  if (ctx == nullptr) {
    // no context current yet: cudaSetDevice makes the device's primary context current
    // (it allocates nothing)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOE_ERR_CUDA;
  }
  return get_id(ctx, id) == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Device address of g_plan_scratch in the current context (looked up once per context).
int scratch_for_current_device(int32_t **out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  int rc = current_context_id(&id);
  if (rc != MOE_OK) return rc;
  for (int i = 0; i < kCacheSlots; ++i)
    if (g_scratch_cache[i].ptr != nullptr && g_scratch_cache[i].ctx_id == id) {
      *out = g_scratch_cache[i].ptr;
      return MOE_OK;
    }
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_plan_scratch) != cudaSuccess || ptr == nullptr)
    return MOE_ERR_CUDA;
  g_scratch_cache[g_scratch_next] = ScratchSlot{id, static_cast<int32_t *>(ptr)};
  g_scratch_next = (g_scratch_next + 1) % kCacheSlots;
  *out = static_cast<int32_t *>(ptr);
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
