"""B200 (sm_100a) MoE layer hot path: plan -> dispatch -> grouped SwiGLU FFN -> combine.

Thin ctypes binding of ``libmoe.so`` (declared in ``include/moe.h``). Every
function here only marshals arguments; all of the layer's work runs in the CUDA
kernels of ``csrc/``. Tensor arguments are device pointers (ints, e.g.
``tensor.data_ptr()``) and streams/events are raw handles (``stream.cuda_stream``).
Importing fails loudly when the library has not been built: there is no
fallback path.

Method: StreamEP README, "How it works" (pool-layout dispatch into an
expert-major tile-padded pool, per-tile streaming flags, caller-owned compute and
communicate streams, grouped GEMMs A / Y).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_MISALIGNED = -3
MOE_ERR_CUDA = -4
MOE_ERR_NO_DEVICE = -5
MOE_ERR_SCRATCH_LIMIT = -6
MOE_PLAN_NOALLOC_SCRATCH_INTS = (1 << 19) + 64
MOE_ERR_BAD_INDEX = -10
MOE_ERR_FLAG_TIMEOUT = -11
MOE_ERR_POOL_OVERFLOW = -12
MOE_ERR_PIPE_TIMEOUT = -13
MOE_ERR_COMBINE_TIMEOUT = -14
MOE_DISPATCH_SIGNAL_TILES = 1
MOE_DISPATCH_ARM_COMBINE = 2


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("tile", ctypes.c_int32)]


class moe_plan_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "counts", "offsets", "pool_row", "row_src", "tile_expert", "mblk", "meta",
        "tile_flags", "workspace", "status", "tok_pending", "ready")]


class moe_config(ctypes.Structure):
    _fields_ = [("streaming", ctypes.c_int32), ("ffn_ctas", ctypes.c_int32),
                ("wait_timeout_us", ctypes.c_int32), ("packed_weights", ctypes.c_int32),
                ("ffn_kernel", ctypes.c_int32), ("timing_events", ctypes.c_void_p),
                ("gate_up", ctypes.c_void_p), ("early_combine", ctypes.c_int32)]


MOE_EP_MAX_RANKS = 8


class moe_ep_plan(ctypes.Structure):
    _fields_ = [("local", moe_plan_buffers)] + [(n, ctypes.c_void_p) for n in (
        "counts", "offsets", "src_base", "tile_expert", "mblk", "meta")]


MOE_FFN_ONE_SM = 1
MOE_FFN_SM_PAIR = 2
MOE_FFN_DEFAULT = MOE_FFN_SM_PAIR      # moe.h: the kernel that ffn_kernel = 0 selects


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {moe_strerror(code)} ({code})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libmoe.so is not built ({LIB_PATH}); run combine_moe_plan_03_b200/build.py "
            "or __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    sig = {
        "moe_pool_rows_max": [P(moe_shape), P(ctypes.c_int64)],
        "moe_plan_arena_bytes": [P(moe_shape), P(ctypes.c_size_t)],
        "moe_plan_bind": [P(moe_shape), vp, P(moe_plan_buffers)],
        "moe_plan": [P(moe_shape), vp, P(moe_plan_buffers), vp, vp],
        "moe_dispatch": [P(moe_shape), vp, P(moe_plan_buffers), vp, i32, vp],
        "moe_grouped_ffn": [P(moe_shape), vp, vp, vp, P(moe_plan_buffers), vp, vp,
                            P(moe_config), vp],
        "moe_combine": [P(moe_shape), vp, vp, P(moe_plan_buffers), vp, vp],
        "moe_grouped_ffn_combine": [P(moe_shape), vp, vp, vp, P(moe_plan_buffers), vp, vp, vp,
                                    vp, P(moe_config), vp],
        "moe_forward": [P(moe_shape), vp, vp, vp, vp, vp, P(moe_plan_buffers), vp, vp, vp, vp,
                        P(moe_config), vp, vp, vp, vp],
        "moe_backward": [P(moe_shape), vp, vp, vp, vp, P(moe_plan_buffers), vp, vp, vp, vp, vp,
                         vp, vp, vp, vp, vp, P(moe_config), vp],
        "moe_backward_streams": [P(moe_shape), vp, vp, vp, vp, P(moe_plan_buffers), vp, vp, vp,
                                 vp, vp, vp, vp, vp, vp, vp, P(moe_config), vp, vp, vp, vp],
        "moe_events_create": [P(vp), i32],
        "moe_timing_events_create": [P(vp), i32],
        "moe_event_elapsed_ms": [vp, vp, P(ctypes.c_float)],
        "moe_events_destroy": [P(vp), i32],
        "moe_get_status": [P(moe_plan_buffers), P(i32), P(i32)],
        "moe_clear_status": [P(moe_plan_buffers), vp],
        "moe_plan_noalloc": [P(moe_shape), vp, P(moe_plan_buffers), vp, vp],
        "moe_route": [P(moe_shape), vp, vp, vp, vp, vp],
        "moe_route_plan": [P(moe_shape), vp, vp, vp, vp, P(moe_plan_buffers), vp, vp],
        "moe_packed_weight_bytes": [P(moe_shape), P(ctypes.c_size_t), P(ctypes.c_size_t)],
        "moe_pack_weights": [P(moe_shape), vp, vp, vp, vp, vp],
        "moe_hbm_probe": [vp, vp, ctypes.c_size_t, i32, vp],
        "moe_ep_local_shape": [P(moe_shape), i32, P(moe_shape)],
        "moe_ep_pool_rows": [P(moe_shape), i32, P(ctypes.c_int64)],
        "moe_ep_arena_bytes": [P(moe_shape), i32, P(ctypes.c_size_t)],
        "moe_ep_bind": [P(moe_shape), i32, vp, P(moe_ep_plan)],
        "moe_ep_layout": [P(moe_shape), i32, i32, vp, P(moe_ep_plan), vp, vp],
        "moe_ep_dispatch": [P(moe_shape), i32, i32, vp, P(moe_plan_buffers), P(moe_ep_plan),
                            P(vp), P(vp), vp],
        "moe_ep_combine": [P(moe_shape), i32, i32, P(vp), vp, P(moe_plan_buffers),
                           P(moe_ep_plan), vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.moe_strerror.argtypes = [ctypes.c_int]
    L.moe_strerror.restype = ctypes.c_char_p
    L.moe_version.argtypes = []
    L.moe_version.restype = ctypes.c_char_p
    return L


_lib = _load()

# Names exported by include/moe.h, in declaration order.
EXPORTS = ["moe_route", "moe_route_plan", "moe_packed_weight_bytes", "moe_pack_weights", "moe_pool_rows_max", "moe_plan_arena_bytes", "moe_plan_bind", "moe_plan",
           "moe_dispatch", "moe_grouped_ffn", "moe_grouped_ffn_combine", "moe_combine",
           "moe_forward", "moe_backward", "moe_backward_streams",
           "moe_events_create",
           "moe_events_destroy", "moe_timing_events_create", "moe_event_elapsed_ms",
           "moe_get_status", "moe_clear_status", "moe_strerror", "moe_plan_noalloc",
           "moe_hbm_probe", "moe_ep_local_shape", "moe_ep_pool_rows", "moe_ep_arena_bytes",
           "moe_ep_bind", "moe_ep_layout", "moe_ep_dispatch", "moe_ep_combine", "moe_version"]


def lib():
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoEError(fn, rc)


def _shape(s) -> moe_shape:
    if isinstance(s, moe_shape):
        return s
    return moe_shape(int(s.T), int(s.H), int(s.I), int(s.E), int(s.k), int(s.tile))


def moe_strerror(code: int) -> str:
    return _lib.moe_strerror(int(code)).decode()


def moe_version() -> str:
    return _lib.moe_version().decode()


def moe_packed_weight_bytes(shape) -> tuple[int, int]:
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("moe_packed_weight_bytes", _lib.moe_packed_weight_bytes(ctypes.byref(_shape(shape)),
                                                                   ctypes.byref(a), ctypes.byref(b)))
    return int(a.value), int(b.value)


def moe_pack_weights(shape, w1_ptr: int, w2_ptr: int, w1p_ptr: int, w2p_ptr: int,
                     stream: int = 0) -> None:
    _check("moe_pack_weights", _lib.moe_pack_weights(ctypes.byref(_shape(shape)), w1_ptr, w2_ptr,
                                                     w1p_ptr, w2p_ptr, stream or None))


def moe_hbm_probe(dst_ptr: int, src_ptr: int, nbytes: int, mode: int, stream: int = 0) -> None:
    """One write-only (mode 0: 16-byte stores, 1: 16 KB bulk stores) or copy (mode 2) pass
    over nbytes of device memory: the HBM rates the layer's copy kernels are compared with."""
    _check("moe_hbm_probe", _lib.moe_hbm_probe(dst_ptr, src_ptr or None, nbytes, mode,
                                               stream or None))


# ---- expert parallelism inside one node (R ranks; shapes are per rank) --------------------

def moe_ep_local_shape(shape, R: int) -> moe_shape:
    out = moe_shape()
    _check("moe_ep_local_shape", _lib.moe_ep_local_shape(ctypes.byref(_shape(shape)), R,
                                                         ctypes.byref(out)))
    return out


def moe_ep_pool_rows(shape, R: int) -> int:
    out = ctypes.c_int64(0)
    _check("moe_ep_pool_rows", _lib.moe_ep_pool_rows(ctypes.byref(_shape(shape)), R,
                                                     ctypes.byref(out)))
    return int(out.value)


def moe_ep_arena_bytes(shape, R: int) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_ep_arena_bytes", _lib.moe_ep_arena_bytes(ctypes.byref(_shape(shape)), R,
                                                         ctypes.byref(out)))
    return int(out.value)


def moe_ep_bind(shape, R: int, arena_ptr: int) -> moe_ep_plan:
    out = moe_ep_plan()
    _check("moe_ep_bind", _lib.moe_ep_bind(ctypes.byref(_shape(shape)), R, arena_ptr,
                                           ctypes.byref(out)))
    return out


def _ptr_array(ptrs):
    return (ctypes.c_void_p * len(ptrs))(*ptrs)


def moe_ep_layout(shape, R: int, rank: int, all_counts_ptr: int, ep: moe_ep_plan,
                  pool_ptr: int, stream: int = 0) -> None:
    _check("moe_ep_layout", _lib.moe_ep_layout(ctypes.byref(_shape(shape)), R, rank,
                                               all_counts_ptr, ctypes.byref(ep), pool_ptr,
                                               stream or None))


def moe_ep_dispatch(shape, R: int, rank: int, x_ptr: int, own: moe_plan_buffers,
                    ep: moe_ep_plan, pool_ptrs, stream: int = 0, flag_ptrs=None) -> None:
    flags = _ptr_array(flag_ptrs) if flag_ptrs is not None else None
    _check("moe_ep_dispatch", _lib.moe_ep_dispatch(ctypes.byref(_shape(shape)), R, rank, x_ptr,
                                                   ctypes.byref(own), ctypes.byref(ep),
                                                   _ptr_array(pool_ptrs), flags, stream or None))


def moe_ep_combine(shape, R: int, rank: int, ypool_ptrs, topk_w_ptr: int,
                   own: moe_plan_buffers, ep: moe_ep_plan, out_ptr: int, stream: int = 0) -> None:
    _check("moe_ep_combine", _lib.moe_ep_combine(ctypes.byref(_shape(shape)), R, rank,
                                                 _ptr_array(ypool_ptrs), topk_w_ptr,
                                                 ctypes.byref(own), ctypes.byref(ep), out_ptr,
                                                 stream or None))


def moe_pool_rows_max(shape) -> int:
    out = ctypes.c_int64(0)
    _check("moe_pool_rows_max", _lib.moe_pool_rows_max(ctypes.byref(_shape(shape)),
                                                       ctypes.byref(out)))
    return int(out.value)


def moe_plan_arena_bytes(shape) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_plan_arena_bytes", _lib.moe_plan_arena_bytes(ctypes.byref(_shape(shape)),
                                                             ctypes.byref(out)))
    return int(out.value)


def moe_plan_bind(shape, arena_ptr: int) -> moe_plan_buffers:
    p = moe_plan_buffers()
    _check("moe_plan_bind", _lib.moe_plan_bind(ctypes.byref(_shape(shape)), arena_ptr,
                                               ctypes.byref(p)))
    return p


def moe_plan(shape, topk_idx_ptr: int, plan: moe_plan_buffers, host_P_ptr: int = 0,
             stream: int = 0) -> None:
    _check("moe_plan", _lib.moe_plan(ctypes.byref(_shape(shape)), topk_idx_ptr,
                                     ctypes.byref(plan), host_P_ptr or None, stream or None))


def moe_plan_noalloc(shape, topk_idx_ptr: int, plan: moe_plan_buffers, host_P_ptr: int = 0,
                     stream: int = 0) -> None:
    """moe_plan without caller-provided scratch (for callers that cannot allocate device
    memory): the library's static 2 MiB device buffer holds it, plan.workspace is ignored."""
    _check("moe_plan_noalloc", _lib.moe_plan_noalloc(ctypes.byref(_shape(shape)), topk_idx_ptr,
                                                     ctypes.byref(plan), host_P_ptr or None,
                                                     stream or None))


def moe_route(shape, logits_ptr: int, bias_ptr: int, topk_idx_ptr: int, topk_w_ptr: int,
              stream: int = 0) -> None:
    _check("moe_route", _lib.moe_route(ctypes.byref(_shape(shape)), logits_ptr, bias_ptr or None,
                                       topk_idx_ptr, topk_w_ptr, stream or None))


def moe_route_plan(shape, logits_ptr: int, bias_ptr: int, topk_idx_ptr: int, topk_w_ptr: int,
                   plan: moe_plan_buffers, host_P_ptr: int = 0, stream: int = 0) -> None:
    _check("moe_route_plan", _lib.moe_route_plan(ctypes.byref(_shape(shape)), logits_ptr,
                                                 bias_ptr or None, topk_idx_ptr, topk_w_ptr,
                                                 ctypes.byref(plan), host_P_ptr or None,
                                                 stream or None))


def moe_dispatch(shape, x_ptr: int, plan: moe_plan_buffers, pool_ptr: int,
                 signal_flags: int = 0, stream: int = 0) -> None:
    _check("moe_dispatch", _lib.moe_dispatch(ctypes.byref(_shape(shape)), x_ptr,
                                             ctypes.byref(plan), pool_ptr, int(signal_flags),
                                             stream or None))


def moe_grouped_ffn(shape, pool_ptr: int, w1_ptr: int, w2_ptr: int, plan: moe_plan_buffers,
                    act_ptr: int, ypool_ptr: int, cfg: moe_config | None = None,
                    stream: int = 0) -> None:
    cfg = cfg or moe_config()
    _check("moe_grouped_ffn", _lib.moe_grouped_ffn(ctypes.byref(_shape(shape)), pool_ptr, w1_ptr,
                                                   w2_ptr, ctypes.byref(plan), act_ptr, ypool_ptr,
                                                   ctypes.byref(cfg), stream or None))


def moe_grouped_ffn_combine(shape, pool_ptr: int, w1_ptr: int, w2_ptr: int,
                            plan: moe_plan_buffers, act_ptr: int, ypool_ptr: int, topk_w_ptr: int,
                            out_ptr: int, cfg: moe_config | None = None, stream: int = 0) -> None:
    """Grouped FFN with the combine fused into GEMM Y (cfg.early_combine must be 1; the
    plan's counters armed by moe_dispatch with MOE_DISPATCH_ARM_COMBINE)."""
    cfg = cfg or moe_config(early_combine=1)
    _check("moe_grouped_ffn_combine", _lib.moe_grouped_ffn_combine(
        ctypes.byref(_shape(shape)), pool_ptr, w1_ptr, w2_ptr, ctypes.byref(plan), act_ptr,
        ypool_ptr, topk_w_ptr or None, out_ptr or None, ctypes.byref(cfg), stream or None))


def moe_combine(shape, ypool_ptr: int, topk_w_ptr: int, plan: moe_plan_buffers, out_ptr: int,
                stream: int = 0) -> None:
    _check("moe_combine", _lib.moe_combine(ctypes.byref(_shape(shape)), ypool_ptr, topk_w_ptr,
                                           ctypes.byref(plan), out_ptr, stream or None))


def moe_forward(shape, x_ptr: int, topk_idx_ptr: int, topk_w_ptr: int, w1_ptr: int, w2_ptr: int,
                plan: moe_plan_buffers, pool_ptr: int, act_ptr: int, ypool_ptr: int, out_ptr: int,
                cfg: moe_config | None, comm_stream: int, compute_stream: int, ev_plan: int,
                ev_dispatch: int) -> None:
    cfg = cfg or moe_config()
    _check("moe_forward", _lib.moe_forward(
        ctypes.byref(_shape(shape)), x_ptr, topk_idx_ptr, topk_w_ptr, w1_ptr or None,
        w2_ptr or None, ctypes.byref(plan), pool_ptr, act_ptr or None, ypool_ptr or None, out_ptr,
        ctypes.byref(cfg), comm_stream or None, compute_stream or None, ev_plan, ev_dispatch))


def moe_backward(shape, dy_ptr: int, topk_w_ptr: int, w1_ptr: int, w2_ptr: int,
                 plan: moe_plan_buffers, pool_ptr: int, act_ptr: int, ypool_ptr: int, gu_ptr: int,
                 dgu_ptr: int, dpool_ptr: int, dx_ptr: int, dw_ptr: int, dw1_ptr: int,
                 dw2_ptr: int, cfg: moe_config | None, stream: int) -> None:
    cfg = cfg or moe_config()
    _check("moe_backward", _lib.moe_backward(
        ctypes.byref(_shape(shape)), dy_ptr or None, topk_w_ptr or None, w1_ptr or None,
        w2_ptr or None, ctypes.byref(plan), pool_ptr or None, act_ptr or None, ypool_ptr or None,
        gu_ptr or None, dgu_ptr or None, dpool_ptr or None, dx_ptr or None, dw_ptr or None,
        dw1_ptr or None, dw2_ptr or None, ctypes.byref(cfg), stream or None))


def moe_backward_streams(shape, dy_ptr: int, topk_w_ptr: int, w1_ptr: int, w2_ptr: int,
                         plan: moe_plan_buffers, pool_ptr: int, act_ptr: int, ypool_ptr: int,
                         gu_ptr: int, dgu_ptr: int, dpool_ptr: int, dx_ptr: int, dw_ptr: int,
                         dw1_ptr: int, dw2_ptr: int, cfg: moe_config | None, comm_stream: int,
                         compute_stream: int, ev_a: int, ev_b: int) -> None:
    cfg = cfg or moe_config()
    _check("moe_backward_streams", _lib.moe_backward_streams(
        ctypes.byref(_shape(shape)), dy_ptr or None, topk_w_ptr or None, w1_ptr or None,
        w2_ptr or None, ctypes.byref(plan), pool_ptr or None, act_ptr or None, ypool_ptr or None,
        gu_ptr or None, dgu_ptr or None, dpool_ptr or None, dx_ptr or None, dw_ptr or None,
        dw1_ptr or None, dw2_ptr or None, ctypes.byref(cfg), comm_stream or None,
        compute_stream or None, ev_a or None, ev_b or None))


def moe_events_create(n: int) -> list[int]:
    arr = (ctypes.c_void_p * n)()
    _check("moe_events_create", _lib.moe_events_create(arr, n))
    return [int(a) for a in arr]


def moe_timing_events_create(n: int) -> list[int]:
    arr = (ctypes.c_void_p * n)()
    _check("moe_timing_events_create", _lib.moe_timing_events_create(arr, n))
    return [int(a) for a in arr]


def moe_event_elapsed_ms(start: int, end: int) -> float:
    ms = ctypes.c_float(0)
    _check("moe_event_elapsed_ms", _lib.moe_event_elapsed_ms(start, end, ctypes.byref(ms)))
    return float(ms.value)


def moe_events_destroy(events: list[int]) -> None:
    arr = (ctypes.c_void_p * len(events))(*events)
    _check("moe_events_destroy", _lib.moe_events_destroy(arr, len(events)))


def moe_get_status(plan: moe_plan_buffers) -> tuple[int, int]:
    code, aux = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("moe_get_status", _lib.moe_get_status(ctypes.byref(plan), ctypes.byref(code),
                                                 ctypes.byref(aux)))
    return int(code.value), int(aux.value)


def moe_clear_status(plan: moe_plan_buffers, stream: int = 0) -> None:
    _check("moe_clear_status", _lib.moe_clear_status(ctypes.byref(plan), stream or None))


from .layer import MoELayerBuffers  # noqa: E402  (torch-allocated buffers for one shape)
