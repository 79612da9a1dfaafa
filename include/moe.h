/*
 * moe.h - C ABI of libmoe.so: the Mixture-of-Experts layer's plan, dispatch,
 * grouped SwiGLU FFN and combine on one NVIDIA B200 (sm_100a).
 *
 * The operations follow the StreamEP README, section "How it works":
 *   - "Pool-layout dispatch": routed (token, k) pairs land directly in an
 *     expert-major, tile-padded pool, so dispatch's output is the grouped GEMM's
 *     input with no separate permute            -> moe_plan, moe_dispatch
 *   - "Per-tile streaming": dispatch signals each pool tile as it fills and the
 *     compute kernels claim ready tiles while later tokens are still arriving;
 *     combine handles a token once its compute is done
 *                                                -> tile flags, moe_grouped_ffn
 *                                                   (streaming), moe_combine
 *   - "Caller-owned streams": the layer runs on a compute stream and a
 *     communicate stream that the caller supplies; the only host sync is one
 *     poll that sizes the dropless pool          -> every call takes the stream;
 *                                                   moe_plan's optional host_P
 *   - "CuTeDSL compute kernels": the forward grouped GEMMs A (gate/up) and
 *     Y (down)                                   -> moe_grouped_ffn
 *     and the backward grouped GEMMs A and Y, with the backward pass mirroring
 *     dispatch and combine                        -> moe_backward (plus the weight
 *                                                   gradients)
 * and the StreamEP call stream_moe_func(buffer, x, topk_idx, topk_weights, ...,
 * w1_local, w2_local, streams=...) shown there            -> moe_forward.
 * The router's softmax / top-k, which StreamEP takes as inputs, is here too
 *                                                -> moe_route, moe_route_plan.
 *
 * Conventions (all entry points):
 *   - Every pointer argument named as a tensor is a DEVICE pointer owned by the
 *     caller (for example a torch tensor's data_ptr()); the library never
 *     allocates, frees or keeps device memory, and never synchronises the device
 *     except in moe_get_status.
 *   - Streams and events are passed as void* holding a cudaStream_t /
 *     cudaEvent_t (0 = the legacy default stream). Work is enqueued on the
 *     given stream; calls return once it is enqueued.
 *   - Layouts are row-major and dense:
 *       x       [T, H]      bf16     token activations
 *       topk_idx[T, k]      int32    expert of pair f = t*k + j; -1 = dropped pair
 *       topk_w  [T, k]      fp32     routing weight of pair f
 *       W1      [E, H, 2I]  bf16     per expert: columns [0, I) gate, [I, 2I) up
 *       W2      [E, I, H]   bf16     per expert down projection
 *       pool    [P_max, H]  bf16     expert-major, tile-padded dispatched rows
 *       act     [P_max, I]  bf16     silu(pool W1_gate) * (pool W1_up), per row
 *       ypool   [P_max, H]  bf16     act W2, per row
 *       out     [T, H]      bf16     out[t] = sum_j topk_w[t,j] * ypool[pool_row[t,j]]
 *     with P_max = moe_pool_rows_max(shape). bf16 buffers must be 16-byte
 *     aligned; H and I must be multiples of 64 (I a multiple of 128 is fastest).
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code, checked on the
 *     host before anything is launched. Errors found on the device (an expert
 *     index out of range, a wait that ran out of time) never trap: the first
 *     one is written to the plan's status word and read with moe_get_status.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ------------------------------------------------------------------- */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)       /* null pointer, negative size, k > 32, E > 1024 ... */
#define MOE_ERR_UNSUPPORTED_SHAPE (-2) /* H or I not a multiple of 64, tile not 64 or 128,
                                          H above 38,720 (3 rows of x must fit in the 227 KB
                                          of shared memory of one dispatch block) */
#define MOE_ERR_MISALIGNED (-3)        /* a tensor pointer not 16-byte aligned */
#define MOE_ERR_CUDA (-4)              /* a CUDA runtime / driver call failed */
#define MOE_ERR_NO_DEVICE (-5)         /* current device is not sm_100 */
#define MOE_ERR_SCRATCH_LIMIT (-6)     /* moe_plan_noalloc: shape needs more than its static scratch */
/* device-side errors, reported through the status word (moe_get_status) */
#define MOE_ERR_BAD_INDEX (-10)     /* topk_idx value outside [-1, E); aux = pair id */
#define MOE_ERR_FLAG_TIMEOUT (-11)  /* streaming FFN gave up waiting on a tile flag; aux = tile */
#define MOE_ERR_POOL_OVERFLOW (-12) /* plan produced more rows than P_max (cannot happen for valid input) */
#define MOE_ERR_PIPE_TIMEOUT (-13)  /* an FFN pipeline barrier wait ran out of time; aux = unit */
#define MOE_ERR_COMBINE_TIMEOUT (-14) /* early combine gave up waiting for a token's expert rows;
                                         aux = position in the ready queue */

/* Layer shape. T tokens, hidden H, expert intermediate I, E experts, top-k,
 * pool tile rows (64 or 128). */
typedef struct moe_shape {
  int32_t T, H, I, E, k, tile;
} moe_shape;

/* Routing plan buffers (device). Carve them from one caller-allocated arena with
 * moe_plan_bind, or point each field at a buffer of the size moe_plan_bind uses. */
typedef struct moe_plan_buffers {
  int32_t *counts;      /* [E]          pairs routed to each expert */
  int32_t *offsets;     /* [E + 1]      start row of each expert's pool segment; offsets[E] = P */
  int32_t *pool_row;    /* [T * k]      pool row of pair f, -1 for a dropped pair */
  int32_t *row_src;     /* [P_max]      pair id of pool row p, -1 for padding */
  int32_t *tile_expert; /* [P_max/tile] expert of pool tile i, -1 past P/tile */
  int32_t *mblk;        /* [5 * P_max/tile] GEMM row chunks: {row_start, expert, live rows <= 256,
                                        the expert's first chunk, its number of chunks} */
  int32_t *meta;        /* [8]          num_tiles, P, number of row chunks, 0, and four
                                        grouped-GEMM unit counters (zeroed by moe_plan) */
  uint32_t *tile_flags; /* [P_max/tile] rows landed per tile (streaming) */
  int32_t *workspace;   /* plan scratch: per-(expert, 256-pair chunk) counts + 1 counter */
  int32_t *status;      /* [4]          code, aux, 0, 0 (first device error wins) */
  /* early combine (moe_config.early_combine); may be NULL otherwise. moe_plan zeroes both. */
  int32_t *tok_pending; /* [T]          live pairs per token whose GEMM Y row chunk is not
                                        complete yet */
  int32_t *ready;       /* [T + 4]      queue of finished tokens (t + 1; 0 = not yet), then
                                        its head and tail counters */
} moe_plan_buffers;

#define MOE_FFN_ONE_SM 1
#define MOE_FFN_SM_PAIR 2
#define MOE_FFN_DEFAULT MOE_FFN_SM_PAIR /* the kernel that moe_config.ffn_kernel = 0 selects */

/* FFN launch options (all fields 0 = defaults). */
typedef struct moe_config {
  int32_t streaming;       /* 1: the FFN claims pool tiles as their flags fill (dispatch may
                              still be running on the communicate stream); 0: the caller
                              orders the FFN after dispatch. */
  int32_t ffn_ctas;        /* persistent FFN CTAs; 0 = number of SMs (streaming: SMs - 16) */
  int32_t wait_timeout_us; /* bound on every device-side wait; 0 = 2,000,000 us */
  int32_t packed_weights;  /* 1: W1 / W2 passed to moe_grouped_ffn / moe_forward are the
                              tiles written by moe_pack_weights, not [E,H,2I] / [E,I,H] */
  int32_t ffn_kernel;      /* grouped-GEMM kernel: MOE_FFN_ONE_SM (one CTA per work unit,
                              MMA M = 128) or MOE_FFN_SM_PAIR (a cluster of two CTAs on two
                              SMs per unit, cta_group::2 MMA with M = 256); 0 = default */
  /* NULL, or 7 cudaEvent_t (8 for moe_backward) that moe_forward records at the phase
     boundaries, each on
     the stream of the kernels around it: [0] comm before plan, [1] comm after plan,
     [2] comm after dispatch, [3] compute before the FFN, [4] compute after GEMM A,
     [5] compute after GEMM Y, [6] compute after combine. moe_grouped_ffn records
     [3], [4], [5]. For per-kernel timing with cudaEventElapsedTime. */
  void *const *timing_events;
  /* NULL, or a device buffer [P_max, 2I] bf16 (16-byte aligned) for the gate / up values of
     a training step, SM-pair kernels only. moe_forward / moe_grouped_ffn: GEMM A also stores
     [g | u] = bf16([pool W1_gate | pool W1_up]) of every live row there, and computes
     act = bf16(silu(g) * u) from those bf16 values. moe_backward: g and u are read from
     there (from the forward call made with the same buffer) instead of being recomputed. */
  void *gate_up;
  /* 1: early combine ("Per-tile streaming": combine handles a token as soon as its compute is
     done), SM-pair kernels only. GEMM Y counts, per token, the expert rows it has stored;
     the store that completes a token puts the token in a ready queue (p->ready), and the
     GEMM's CTAs, once they run out of GEMM work, combine the queued tokens into out while
     the last GEMM units still run. Needs p->tok_pending and p->ready, and moe_dispatch with
     MOE_DISPATCH_ARM_COMBINE (moe_forward does both); out is bit-identical to moe_combine's. */
  int32_t early_combine;
} moe_config;

/*
 * Weight prepack (a layout copy made once, e.g. when the model is loaded; not part of
 * the pages' method). The grouped GEMMs read each expert's weights as tiles of 64 k-rows
 * x 128 columns; from [E,H,2I] / [E,I,H] every such tile is 64 pieces of 128 bytes at the
 * matrix's row pitch. moe_pack_weights stores each tile as one contiguous 16 KB block in
 * the order the GEMM's shared-memory tile takes, so the weight stream reads contiguous
 * HBM. Packed sizes (bytes) from moe_packed_weight_bytes; columns past I / H are zero.
 * W1p and W2p are caller-owned device buffers, 16-byte aligned; the copy runs on `stream`.
 */
int moe_packed_weight_bytes(const moe_shape *s, size_t *w1p_bytes, size_t *w2p_bytes);
int moe_pack_weights(const moe_shape *s, const void *W1, const void *W2, void *W1p, void *W2p,
                     void *stream);

/* Dropless pool bound: T*k + min(E, T*k)*(tile-1), rounded up to a multiple of tile. */
int moe_pool_rows_max(const moe_shape *s, int64_t *rows_out);

/* Bytes of the plan arena for this shape (one device allocation, 256-byte aligned). */
int moe_plan_arena_bytes(const moe_shape *s, size_t *bytes_out);

/* Point the fields of *out into a caller-owned device arena of moe_plan_arena_bytes
 * bytes. Host-only, no device work. The arena's status word must be zeroed once
 * by the caller (or with moe_clear_status) before first use. */
int moe_plan_bind(const moe_shape *s, void *arena, moe_plan_buffers *out);

/*
 * Routing plan (StreamEP README, How it works, "Pool-layout dispatch").
 * From topk_idx [T, k] (device int32) computes, on `stream`:
 *   counts[e], offsets (exclusive prefix of counts padded up to the tile), P,
 *   pool_row[f] = offsets[e] + rank of f among the pairs of expert e (flat pair id
 *   ascending: a stable map), row_src (inverse map, -1 for padding), tile_expert,
 *   the GEMM row-block table mblk, meta, and resets tile_flags to 0.
 * If host_P is not NULL (pinned host memory), P is copied there asynchronously:
 * the one poll that sizes the dropless pool. Values outside [-1, E) in topk_idx
 * give MOE_ERR_BAD_INDEX in the status word and those pairs are dropped.
 */
int moe_plan(const moe_shape *s, const int32_t *topk_idx, const moe_plan_buffers *p,
             int32_t *host_P, void *stream);

/*
 * Router on the device (the topk_idx / topk_weights inputs of the StreamEP call: the
 * gate's softmax, top-k, renormalised). For each token t of fp32 logits [T, E] and an
 * optional fp32 bias [E] (NULL for none): scores v = logit + bias (fp32); the k largest
 * scores, largest first, equal scores by lower expert index, go to topk_idx [T, k];
 * topk_w [T, k] = their softmax probabilities renormalised over the k chosen (fp32,
 * expf). Requires k <= E. Logits must be finite.
 */
int moe_route(const moe_shape *s, const float *logits, const float *bias, int32_t *topk_idx,
              float *topk_w, void *stream);

/*
 * moe_route followed by moe_plan, with the router and the plan's per-expert histogram
 * in one kernel when k divides 256 (each block routes one 256-pair plan chunk); same
 * outputs as the two calls. host_P as in moe_plan.
 */
int moe_route_plan(const moe_shape *s, const float *logits, const float *bias, int32_t *topk_idx,
                   float *topk_w, const moe_plan_buffers *p, int32_t *host_P, void *stream);

/*
 * Dispatch (StreamEP README, How it works, "Pool-layout dispatch" and "Per-tile
 * streaming"): pool[pool_row[t*k+j]] = x[t] for every live pair, padding rows of
 * each expert's segment set to zero, and (signal_flags != 0) tile_flags[p / tile]
 * incremented with release order once row p has landed. Reads x [T, H], writes
 * pool [P_max, H] (rows >= P are not touched). Runs after moe_plan on `stream`.
 * signal_flags is a mask of MOE_DISPATCH_SIGNAL_TILES and MOE_DISPATCH_ARM_COMBINE (any
 * other non-zero value counts as MOE_DISPATCH_SIGNAL_TILES alone).
 */
#define MOE_DISPATCH_SIGNAL_TILES 1  /* count landed rows in tile_flags (streaming FFN) */
#define MOE_DISPATCH_ARM_COMBINE 2   /* set p->tok_pending for early combine, queue the tokens
                                        that have no live pair */
int moe_dispatch(const moe_shape *s, const void *x, const moe_plan_buffers *p, void *pool,
                 int32_t signal_flags, void *stream);

/*
 * Grouped SwiGLU FFN over the pool (StreamEP README, How it works, "CuTeDSL
 * compute kernels": grouped GEMM A then grouped GEMM Y), tcgen05 tensor cores:
 *   act[p]   = bf16( silu(pool[p] W1[e]_gate) * (pool[p] W1[e]_up) )   (fp32 accumulate)
 *   ypool[p] = bf16( act[p] W2[e] )                                     (fp32 accumulate)
 * for every live row p (a row that holds a routed pair), e = the expert of p's
 * segment. Padding rows of act and ypool are not written (combine never reads them).
 * With cfg->streaming the first GEMM waits (bounded) until tile_flags[tile] == tile
 * for each tile it reads, so it may be launched while moe_dispatch is still running
 * on another stream; otherwise it must be ordered after moe_dispatch.
 */
int moe_grouped_ffn(const moe_shape *s, const void *pool, const void *W1, const void *W2,
                    const moe_plan_buffers *p, void *act, void *ypool, const moe_config *cfg,
                    void *stream);

/*
 * moe_grouped_ffn with the combine fused in (early combine; StreamEP README, How it works,
 * "Per-tile streaming": combine starts on a token as soon as its compute is done). The same
 * GEMMs A and Y, and out[t] = bf16(sum_j topk_w[t,j] * ypool[pool_row[t,j]]) exactly as
 * moe_combine computes it (fp32 FMA chain, j ascending), each token combined by the GEMM Y
 * kernel's CTAs as soon as its k rows are stored. Needs cfg->early_combine = 1, the SM-pair
 * kernel, p->tok_pending / p->ready, and moe_dispatch run with MOE_DISPATCH_ARM_COMBINE
 * after this call's moe_plan. GEMM Y counts its finished units per row chunk in
 * p->tile_flags (zeroed after GEMM A, their streaming reader, is done). A token whose rows
 * never arrive (the counters were not armed) gives MOE_ERR_COMBINE_TIMEOUT in the status
 * word after cfg->wait_timeout_us.
 */
int moe_grouped_ffn_combine(const moe_shape *s, const void *pool, const void *W1, const void *W2,
                            const moe_plan_buffers *p, void *act, void *ypool,
                            const float *topk_w, void *out, const moe_config *cfg,
                            void *stream);

/*
 * Combine (StreamEP README, How it works, "Per-tile streaming": combine of a token
 * once its compute is done): out[t] = bf16( sum_j topk_w[t,j] * ypool[pool_row[t,j]] ),
 * an fp32 fused multiply-add chain over j ascending; dropped pairs add nothing.
 * Pass the pool itself as ypool for identity experts.
 */
int moe_combine(const moe_shape *s, const void *ypool, const float *topk_w,
                const moe_plan_buffers *p, void *out, void *stream);

/*
 * The whole layer (the StreamEP stream_moe_func call): plan and dispatch on
 * comm_stream, grouped FFN and combine on compute_stream, ordered with the two
 * caller-owned events (ev_plan, ev_dispatch; create them with moe_events_create).
 * W1 == NULL and W2 == NULL selects identity experts (combine reads the pool;
 * act and ypool are not used). compute_stream waits for the previous work on
 * comm_stream, and comm_stream for the previous work on compute_stream, so calls
 * may be issued back to back with the same buffers.
 */
int moe_forward(const moe_shape *s, const void *x, const int32_t *topk_idx, const float *topk_w,
                const void *W1, const void *W2, const moe_plan_buffers *p, void *pool, void *act,
                void *ypool, void *out, const moe_config *cfg, void *comm_stream,
                void *compute_stream, void *ev_plan, void *ev_dispatch);

/*
 * Backward of the layer's activation path (StreamEP README, How it works: the backward
 * grouped GEMMs A and Y of "CuTeDSL compute kernels", and the backward pass that mirrors
 * dispatch and combine, "Per-tile streaming"), on one stream. Given
 *   dy [T, H] bf16        the gradient of the loss with respect to moe_forward's out,
 *   topk_w [T, k] fp32    the routing weights of that forward call,
 *   W1, W2                the weights in their given layout [E,H,2I] / [E,I,H] (read
 *                         K-major here; prepacked tiles are not accepted),
 *   p, pool, ypool        the plan buffers, pool and ypool of that forward call (it must
 *                         have run with weights, not identity experts),
 * it computes, with e the expert of pool row p = pool_row[t,j]:
 *   dw[t,j]  = sum_h dy[t,h] * ypool[p,h]                       (fp32; 0 for a dropped pair)
 *   dypool[p] = bf16(topk_w[t,j] * dy[t])                        (into dpool)
 *   gu[p]    = bf16([pool[p] W1[e]_gate | pool[p] W1[e]_up])    (gate / up recompute)
 *   dgu[p]   = bf16([da * u * silu'(g) | da * silu(g)]),  da = dypool[p] W2[e]^T (fp32)
 *   dpool[p] = bf16(dgu[p] W1[e]^T)                              (overwrites dypool)
 *   dx[t]    = bf16(sum_j dpool[pool_row[t,j]])                  (fp32 sum in j order)
 * and, when dW2 / dW1 are not NULL, the weight gradients (fp32 sums, bf16 results; an expert
 * with no rows gets zeros):
 *   dW2[e] = sum over e's rows p of act[p]^T dypool[p]           [E, I, H]
 *   dW1[e] = sum over e's rows p of pool[p]^T dgu[p]             [E, H, 2I]
 * act is the forward call's act buffer (needed for dW2; its padding rows are set to zero).
 * Work buffers (device, caller-owned, 16-byte aligned): gu and dgu [P_max, 2I] bf16,
 * dpool [P_max, H] bf16. Outputs: dx [T, H] bf16, dw [T, k] fp32, dW1, dW2 bf16. The grouped
 * GEMMs run on SM pairs (cfg->ffn_kernel must be 0 or MOE_FFN_SM_PAIR; cfg->packed_weights
 * and cfg->streaming must be 0: streaming needs moe_backward_streams). cfg->early_combine = 1
 * mirrors early combine: the dispatch
 * backward is folded into backward A, whose CTAs sum each token's k dpool rows as soon as
 * they are stored (p's tok_pending and ready are re-armed first; dx is bit-identical);
 * cfg->wait_timeout_us bounds that wait too (MOE_ERR_COMBINE_TIMEOUT). cfg->timing_events,
 * if set, holds 8 events recorded on `stream`: [0] before, [1] after the combine backward,
 * [2] after the recompute, [3] after backward Y, [4] after dW2, [5] after backward A, [6]
 * after dW1, [7] after the dispatch backward (with early_combine: after dW1 as well).
 */
int moe_backward(const moe_shape *s, const void *dy, const float *topk_w, const void *W1,
                 const void *W2, const moe_plan_buffers *p, const void *pool, void *act,
                 const void *ypool, void *gu, void *dgu, void *dpool, void *dx, float *dw,
                 void *dW1, void *dW2, const moe_config *cfg, void *stream);

/*
 * moe_backward on the caller's two streams (the layer's communicate and compute streams, as
 * in moe_forward), which also accepts cfg->streaming = 1: the mirror of the streaming
 * forward. The combine backward then runs in pool-tile order on comm_stream (on the 16 SMs
 * backward Y leaves free), raising each pool tile's flag once its dypool rows and dw are
 * written (dw is
 * zeroed first, so dropped pairs keep 0), while backward Y on compute_stream takes each row
 * chunk as soon as the flags of its tiles are full (bounded wait: MOE_ERR_FLAG_TIMEOUT);
 * everything else runs on compute_stream, which waits for the combine backward before the
 * weight gradients. Results are bit-identical to moe_backward's. ev_a / ev_b: two events
 * (moe_events_create) for the ordering; comm_stream must differ from compute_stream when
 * streaming. With cfg->streaming = 0 it is moe_backward on compute_stream.
 */
int moe_backward_streams(const moe_shape *s, const void *dy, const float *topk_w, const void *W1,
                         const void *W2, const moe_plan_buffers *p, const void *pool, void *act,
                         const void *ypool, void *gu, void *dgu, void *dpool, void *dx, float *dw,
                         void *dW1, void *dW2, const moe_config *cfg, void *comm_stream,
                         void *compute_stream, void *ev_a, void *ev_b);

/* Create / destroy n cudaEvent_t (timing disabled) for moe_forward's ordering. */
int moe_events_create(void **events, int32_t n);
int moe_events_destroy(void **events, int32_t n);

/* Create n cudaEvent_t with timing enabled (for moe_config.timing_events); destroy
 * them with moe_events_destroy. */
int moe_timing_events_create(void **events, int32_t n);

/* Milliseconds between two recorded timing events (cudaEventElapsedTime; the end
 * event must have completed, else MOE_ERR_CUDA). */
int moe_event_elapsed_ms(void *start, void *end, float *ms);

/* Read the status word (synchronous: waits for work already queued that writes it). */
int moe_get_status(const moe_plan_buffers *p, int32_t *code, int32_t *aux);

/* Zero the status word on `stream`, and (when p->meta is set) the grouped GEMMs' unit
 * counters meta[4..7], so that an FFN re-run on the same plan after a device error starts
 * from its first unit. Call it while no layer call that uses these plan buffers is in
 * flight. */
int moe_clear_status(const moe_plan_buffers *p, void *stream);

/* Text for an error code. */
const char *moe_strerror(int code);

/*
 * moe_plan_noalloc - moe_plan for callers that cannot allocate device memory.
 * The paper has no counterpart; this is a convenience of this library.
 *
 * Same inputs, outputs and results as moe_plan (bit for bit), but the plan's
 * scratch lives in a static device buffer inside the library, so p->workspace is
 * ignored (it may be NULL) and the caller never sizes or allocates scratch. Meant
 * for code whose host framework owns all device memory and gives it no allocator
 * (an inference engine's plugin hook, for instance), or loops that cannot afford
 * a cudaMalloc's device synchronisation or its failure under a fixed budget.
 *   - Maximum: E * max(1, ceil(T*k/256)) + 8 <= MOE_PLAN_NOALLOC_SCRATCH_INTS
 *     (2 MiB + 256 B of int32; e.g. E = 256 with up to 524,288 pairs). Larger
 *     shapes return MOE_ERR_SCRATCH_LIMIT and launch nothing. Every GPU that loads
 *     the library holds this buffer until the process exits.
 *   - All calls on a device share the buffer and it keeps the last call's
 *     contents; each call rewrites what it reads and zeroes its counter first, so
 *     back-to-back calls are independent, but calls that overlap on the GPU
 *     (issued on concurrent streams) race on it.
 *   - The first call on a device (with that device current) looks up the
 *     buffer's device address; make it before any stream capture. The address
 *     is kept per CUDA context: after a device reset the next call looks it up
 *     again.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define MOE_PLAN_NOALLOC_SCRATCH_INTS ((1 << 19) + 64)
int moe_plan_noalloc(const moe_shape *s, const int32_t *topk_idx, const moe_plan_buffers *p,
                     int32_t *host_P, void *stream);

/*
 * HBM rate probe (a measurement aid, not part of the pages' method): one launch on `stream`
 * that only writes `bytes` of zeros to dst (mode 0: 16-byte vector stores; mode 1:
 * cp.async.bulk stores of 16 KB blocks from shared memory, the store form of moe_dispatch;
 * bytes a multiple of 16 KB), or copies src to dst (mode 2: 16-byte vector loads and
 * stores). Timed with events around it on a buffer far larger than L2 it gives the write and
 * copy rates this library's own kernels reach, the ceilings dispatch and combine are
 * compared with. dst (and src) are caller-owned device buffers, 16-byte aligned; bytes a
 * multiple of 16. Errors: MOE_ERR_INVALID_ARG, MOE_ERR_MISALIGNED, MOE_ERR_CUDA.
 */
int moe_hbm_probe(void *dst, const void *src, size_t bytes, int32_t mode, void *stream);

/*
 * Expert parallelism inside one node (StreamEP README: dispatch and combine "intranode over
 * NVLink"; "Pool-layout dispatch"). R ranks (one per GPU, R <= MOE_EP_MAX_RANKS, E a
 * multiple of R); rank d owns experts [d E/R, (d+1) E/R). Shapes below are per rank:
 * rank_shape = {T tokens of this rank, H, I, E global experts, k, tile}. A layer call on
 * rank r:
 *   1. moe_plan(rank_shape, topk_idx, own)        this rank's pairs over the E experts
 *   2. all-gather own.counts ([E] int32) over the ranks into all_counts [R][E] (device; by the
 *      caller, e.g. one NCCL all-gather); it orders this step after every rank's previous
 *      use of its pool
 *   3. moe_ep_layout(rank_shape, R, r, all_counts, ep, pool)   every rank's pool layout, this
 *      rank's pool plan (ep->local) and zero padding rows
 *   4. moe_ep_dispatch(..., pools, tile_flags)     x rows into their owners' pools, each row
 *      counted on its owner's tile flag
 *   5. a barrier over the ranks (every rank's dispatch done); or none, with a streaming FFN
 *      (moe_config.streaming = 1) that takes each pool tile once its flag is full
 *   6. moe_grouped_ffn(local_shape, pool, W1 / W2 of this rank's experts, &ep->local, ...)
 *      with local_shape from moe_ep_local_shape (T = R * rank T, E = E / R)
 *   7. a barrier (every rank's FFN done)
 *   8. moe_ep_combine(..., ypools, topk_w, own, ep, out)   out[t] from the owners' ypools
 * The pool of rank d holds the rows of d's experts from rank 0's pairs, then rank 1's, ...,
 * each in flat pair order, padded per expert to the tile: the part of one dropless pool over
 * all ranks' pairs that holds d's experts. pools / ypools: host arrays of R device pointers
 * (every rank's pool [moe_ep_pool_rows, H] / ypool, mapped for peer access); x rows are
 * stored into peers' pools and ypool rows loaded from peers' ypools with plain 16-byte
 * accesses. No collective is issued by the library.
 */
#define MOE_EP_MAX_RANKS 8
typedef struct moe_ep_plan {
  moe_plan_buffers local; /* this rank's pool: the grouped FFN's plan (local shape) */
  int32_t *counts;        /* [E]       pairs of all ranks per expert */
  int32_t *offsets;       /* [E + 1]   padded prefix over all experts (rank d's pool starts at
                                       offsets[d E / R]) */
  int32_t *src_base;      /* [E * R + 8] rows of expert e from ranks before s: [e * R + s] */
  int32_t *tile_expert;   /* tile and row-chunk tables and meta of the all-expert prefix */
  int32_t *mblk;
  int32_t *meta;
} moe_ep_plan;

/* Local shape {R * T, H, I, E / R, k, tile} of a rank's pool; pool rows (dropless bound for
 * all ranks' pairs on E / R experts); bytes of the EP plan arena; binding the arena (host
 * only: 256-byte aligned slices of the caller's device arena, which must be zeroed once
 * before the first layer call: its status word and pool tile flags start at zero).
 * Errors: MOE_ERR_INVALID_ARG (R outside [1, MOE_EP_MAX_RANKS], E not a multiple of R, a
 * shape that check fails, NULL pointers), MOE_ERR_UNSUPPORTED_SHAPE. */
int moe_ep_local_shape(const moe_shape *rank_shape, int32_t R, moe_shape *out);
int moe_ep_pool_rows(const moe_shape *rank_shape, int32_t R, int64_t *rows_out);
int moe_ep_arena_bytes(const moe_shape *rank_shape, int32_t R, size_t *bytes_out);
int moe_ep_bind(const moe_shape *rank_shape, int32_t R, void *arena, moe_ep_plan *out);

/* Step 3: from all_counts [R][E] (device int32), the layout of every rank's pool, this rank's
 * pool plan ep->local (reset and built; its status word is the layer's) and zeroed padding
 * rows in this rank's pool. A count outside [0, T k], or totals beyond the pool, give
 * MOE_ERR_POOL_OVERFLOW in ep->local's status word and an empty pool plan. */
int moe_ep_layout(const moe_shape *rank_shape, int32_t R, int32_t rank,
                  const int32_t *all_counts, const moe_ep_plan *ep, void *pool, void *stream);

/* Step 4: pool_{owner(e)}[row of pair f] = x[t] for every live pair f = t*k + j of this rank
 * (own: this rank's moe_plan). tile_flags: NULL, or a host array of R device pointers, each
 * rank's ep->local.tile_flags (mapped for peer access); then every stored row adds one to
 * its owner's tile flag (release at system scope) after the row's stores, and the owner's
 * moe_ep_layout adds one per padding row, so a tile's flag reaches the tile height when all
 * its rows have landed: a grouped FFN with moe_config.streaming = 1 on the owner takes each
 * tile then (its waits acquire at system scope). The flags must be zero before the first
 * call (a zeroed arena); moe_ep_combine zeroes the rank's own flags again after its FFN has
 * used them, so no reset races with the next call's dispatches from other ranks (which
 * follow the next count exchange). This rank's row of all_counts must equal own's counts, else
 * MOE_ERR_POOL_OVERFLOW (aux = expert) in own's status word. A row that all_counts would
 * place outside the owner's pool is skipped and reported the same way (aux = pair id);
 * moe_ep_combine checks rows the same way. */
int moe_ep_dispatch(const moe_shape *rank_shape, int32_t R, int32_t rank, const void *x,
                    const moe_plan_buffers *own, const moe_ep_plan *ep, void *const *pools,
                    uint32_t *const *tile_flags, void *stream);

/* Step 8: out[t] = bf16(sum_j topk_w[t,j] * ypool_{owner}[row of pair t*k + j]), fp32 FMA
 * chain over j ascending (moe_combine's arithmetic); dropped pairs add nothing. */
int moe_ep_combine(const moe_shape *rank_shape, int32_t R, int32_t rank, void *const *ypools,
                   const float *topk_w, const moe_plan_buffers *own, const moe_ep_plan *ep,
                   void *out, void *stream);

/* Library version string. */
const char *moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
