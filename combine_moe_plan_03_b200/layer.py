"""Device buffers for one MoE layer shape, allocated with torch, used through the C ABI.

PyTorch only provides device memory, streams and events here; every step of the
layer runs in libmoe's kernels. ``forward`` is the StreamEP ``stream_moe_func``
call shape (x, topk_idx, topk_weights, w1, w2, streams) on one GPU.
"""
from __future__ import annotations

import ctypes

import torch

from . import (moe_backward, moe_backward_streams, moe_config, moe_events_create,
               moe_events_destroy, moe_forward, moe_pack_weights, moe_packed_weight_bytes,
               moe_plan_arena_bytes, moe_plan_bind, moe_pool_rows_max, moe_shape)


def ctypes_copy(dst: ctypes.Structure, src: ctypes.Structure) -> None:
    ctypes.memmove(ctypes.addressof(dst), ctypes.addressof(src), ctypes.sizeof(dst))


_PLAN_FIELDS = ("counts", "offsets", "pool_row", "row_src", "tile_expert", "mblk", "meta",
                "tile_flags", "workspace", "status", "tok_pending", "ready")


class MoELayerBuffers:
    """Plan arena, pool, act, ypool and out for shape (T, H, I, E, k, tile), plus the
    caller-owned communicate / compute streams and the two ordering events."""

    def __init__(self, T: int, H: int, I: int, E: int, k: int, tile: int,
                 device: str | torch.device = "cuda", identity: bool = False,
                 streams: tuple[torch.cuda.Stream, torch.cuda.Stream] | None = None):
        self.shape = moe_shape(T, H, I, E, k, tile)
        self.device = torch.device(device)
        self.identity = identity
        self.P_max = moe_pool_rows_max(self.shape)
        nbytes = moe_plan_arena_bytes(self.shape)
        self.arena = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        self.plan = moe_plan_bind(self.shape, self.arena.data_ptr())
        bf = torch.bfloat16
        self.pool = torch.empty((max(self.P_max, 1), H), dtype=bf, device=self.device)
        if identity:
            self.act = None
            self.ypool = None
        else:
            self.act = torch.empty((max(self.P_max, 1), I), dtype=bf, device=self.device)
            self.ypool = torch.empty((max(self.P_max, 1), H), dtype=bf, device=self.device)
        self.out = torch.empty((max(T, 1), H), dtype=bf, device=self.device)
        if streams is None:
            streams = (torch.cuda.Stream(self.device), torch.cuda.Stream(self.device))
        self.comm, self.compute = streams
        self.events = moe_events_create(2)
        self.gu = self.dgu = self.dpool = None      # backward work buffers, on first use

    def close(self):
        if self.events:
            moe_events_destroy(self.events)
            self.events = []

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def plan_view(self, name: str) -> torch.Tensor:
        """int32 view of one plan buffer inside the arena (for inspection and tests)."""
        ptr = getattr(self.plan, name)
        off = ptr - self.arena.data_ptr()
        i = _PLAN_FIELDS.index(name)
        end = (getattr(self.plan, _PLAN_FIELDS[i + 1]) - self.arena.data_ptr()
               if i + 1 < len(_PLAN_FIELDS) else self.arena.numel())
        return self.arena[off:end].view(torch.int32)

    def pack_weights(self, W1: torch.Tensor, W2: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
        """One-time prepack of W1 [E,H,2I] / W2 [E,I,H] into the GEMMs' tile layout
        (moe_pack_weights). Use the results with ``moe_config(packed_weights=1)``."""
        s = self.shape
        assert tuple(W1.shape) == (s.E, s.H, 2 * s.I) and W1.dtype == torch.bfloat16
        assert tuple(W2.shape) == (s.E, s.I, s.H) and W2.dtype == torch.bfloat16
        b1, b2 = moe_packed_weight_bytes(s)
        W1p = torch.empty(b1 // 2, dtype=torch.bfloat16, device=self.device)
        W2p = torch.empty(b2 // 2, dtype=torch.bfloat16, device=self.device)
        cur = self._enter()
        moe_pack_weights(s, W1.data_ptr(), W2.data_ptr(), W1p.data_ptr(), W2p.data_ptr(),
                         self.compute.cuda_stream)
        self._leave(cur)
        self.compute.synchronize()
        return W1p, W2p

    def _backward_buffers(self):
        s = self.shape
        if self.gu is None:
            rows, bf = max(self.P_max, 1), torch.bfloat16
            self.gu = torch.empty((rows, 2 * s.I), dtype=bf, device=self.device)
            self.dgu = torch.empty((rows, 2 * s.I), dtype=bf, device=self.device)
            self.dpool = torch.empty((rows, s.H), dtype=bf, device=self.device)

    def forward(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                W1: torch.Tensor | None, W2: torch.Tensor | None,
                cfg: moe_config | None = None, out: torch.Tensor | None = None,
                save_for_backward: bool = False) -> torch.Tensor:
        """Enqueue the layer (plan + dispatch on comm, FFN + combine on compute).
        Writes ``out`` [T, H] bf16 (default: this object's own buffer) and returns it; it is
        ready once the compute stream reaches this point. With ``save_for_backward`` GEMM A
        also keeps the gate / up values (``moe_config.gate_up``), so that ``backward`` need
        not recompute them."""
        s = self.shape
        if save_for_backward and not self.identity:
            self._backward_buffers()
            c = moe_config()
            if cfg is not None:
                ctypes_copy(c, cfg)
            c.gate_up = self.gu.data_ptr()
            cfg = c
        self._gu_saved = bool(save_for_backward and not self.identity)
        if out is None:
            out = self.out[: s.T]
        assert out.dtype == torch.bfloat16 and tuple(out.shape) == (s.T, s.H) and out.is_contiguous()
        assert x.dtype == torch.bfloat16 and tuple(x.shape) == (s.T, s.H) and x.is_contiguous()
        assert topk_idx.dtype == torch.int32 and tuple(topk_idx.shape) == (s.T, s.k)
        assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (s.T, s.k)
        w1 = w2 = act = ypool = 0
        if not self.identity:
            assert W1 is not None and W2 is not None
            assert W1.dtype == torch.bfloat16 and W2.dtype == torch.bfloat16
            if cfg is not None and cfg.packed_weights:
                b1, b2 = moe_packed_weight_bytes(s)
                assert W1.numel() * 2 >= b1 and W2.numel() * 2 >= b2
            else:
                assert tuple(W1.shape) == (s.E, s.H, 2 * s.I)
                assert tuple(W2.shape) == (s.E, s.I, s.H)
            w1, w2 = W1.data_ptr(), W2.data_ptr()
            act, ypool = self.act.data_ptr(), self.ypool.data_ptr()
        cur = self._enter()
        moe_forward(s, x.data_ptr(), topk_idx.data_ptr(), topk_w.data_ptr(), w1, w2, self.plan,
                    self.pool.data_ptr(), act, ypool, out.data_ptr(), cfg,
                    self.comm.cuda_stream, self.compute.cuda_stream, self.events[0],
                    self.events[1])
        self._leave(cur)
        return out

    def _enter(self) -> torch.cuda.Stream:
        # the layer's streams start after the caller's work so far on its current stream
        # (inputs made there are complete) ...
        cur = torch.cuda.current_stream(self.device)
        self.comm.wait_stream(cur)
        self.compute.wait_stream(cur)
        return cur

    def _leave(self, cur: torch.cuda.Stream) -> None:
        # ... and the caller's stream continues after the layer: the outputs are ready in its
        # stream order, and memory of its tensors that it frees (temporaries passed in) is
        # reused only by work that runs after the layer's kernels
        cur.wait_stream(self.compute)

    def backward(self, dy: torch.Tensor, topk_w: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor,
                 cfg: moe_config | None = None, dx: torch.Tensor | None = None,
                 dw: torch.Tensor | None = None, dW1: torch.Tensor | None = None,
                 dW2: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
        """Backward of the last ``forward`` call on these buffers (its plan, pool, act and
        ypool), on the compute stream: returns (dx [T, H] bf16, dw [T, k] fp32) for the
        upstream gradient dy [T, H] bf16 (moe_backward), and fills the weight gradients
        dW1 [E, H, 2I] / dW2 [E, I, H] (bf16) when they are given. W1 / W2 in their given
        layout."""
        s = self.shape
        assert not self.identity
        assert dy.dtype == torch.bfloat16 and tuple(dy.shape) == (s.T, s.H) and dy.is_contiguous()
        assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (s.T, s.k)
        assert tuple(W1.shape) == (s.E, s.H, 2 * s.I) and tuple(W2.shape) == (s.E, s.I, s.H)
        bf = torch.bfloat16
        self._backward_buffers()
        c = moe_config()
        if cfg is not None:
            ctypes_copy(c, cfg)
        # the gate / up values kept by a forward(save_for_backward=True) replace the recompute
        c.gate_up = self.gu.data_ptr() if getattr(self, "_gu_saved", False) else None
        cfg = c
        if dx is None:
            dx = torch.empty((max(s.T, 1), s.H), dtype=bf, device=self.device)[: s.T]
        if dw is None:
            dw = torch.empty((max(s.T, 1), s.k), dtype=torch.float32, device=self.device)[: s.T]
        for t, shp in ((dW1, (s.E, s.H, 2 * s.I)), (dW2, (s.E, s.I, s.H))):
            assert t is None or (t.dtype == bf and tuple(t.shape) == shp and t.is_contiguous())
        args = (s, dy.data_ptr(), topk_w.data_ptr(), W1.data_ptr(), W2.data_ptr(), self.plan,
                self.pool.data_ptr(), self.act.data_ptr(), self.ypool.data_ptr(),
                self.gu.data_ptr(), self.dgu.data_ptr(), self.dpool.data_ptr(),
                dx.data_ptr(), dw.data_ptr(), dW1.data_ptr() if dW1 is not None else 0,
                dW2.data_ptr() if dW2 is not None else 0, cfg)
        cur = self._enter()
        if cfg.streaming:
            # the combine backward in tile order on the communicate stream, backward Y
            # taking tiles on the compute stream (moe_backward_streams)
            moe_backward_streams(*args, self.comm.cuda_stream, self.compute.cuda_stream,
                                 self.events[0], self.events[1])
        else:
            moe_backward(*args, self.compute.cuda_stream)
        self._leave(cur)
        return dx, dw
