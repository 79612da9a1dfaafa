"""Expert parallelism inside one node over a torch.distributed process group (one rank per
GPU), on top of the C ABI's moe_ep_* calls (StreamEP README: dispatch and combine
"intranode over NVLink"; "Pool-layout dispatch").

Each rank owns E / R experts. Its pool, ypool and EP plan arena are separate device
allocations whose CUDA IPC handles are exchanged once, so every rank holds every peer's
pool / ypool / tile-flag pointers; the kernels then store into and load from peers' memory
with plain 16-byte accesses and system-scope flag atomics (no multicast). One layer call:

    moe_plan -> all-gather of the E per-expert counts (NCCL) -> moe_ep_layout ->
    moe_ep_dispatch (rows into their owners' pools, counted on the owners' tile flags) ->
    barrier (or a streaming FFN that takes tiles by their flags) -> moe_grouped_ffn on this
    rank's experts -> barrier -> moe_ep_combine (rows back from the owners' ypools)

All of it runs in the stream order of the caller's current stream; the barriers are NCCL
all-reduces of one word, which complete on a rank only after every rank has enqueued them
behind its own kernels. With one rank the peers are this rank's own buffers.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (moe_config, moe_ep_arena_bytes, moe_ep_bind, moe_ep_combine, moe_ep_dispatch,
               moe_ep_layout, moe_ep_local_shape, moe_ep_pool_rows, moe_get_status,
               moe_grouped_ffn, moe_plan, moe_plan_arena_bytes, moe_plan_bind, moe_shape)


def _rt():
    from cuda.bindings import runtime
    return runtime


def _ok(res):
    err = res[0] if isinstance(res, tuple) else res
    if int(err) != 0:
        raise RuntimeError(f"CUDA runtime call failed: {err}")
    return res[1] if isinstance(res, tuple) and len(res) > 1 else None


def exchange(obj, group=None) -> list:
    """Every rank's `obj` in rank order (all_gather_object over the group; one rank: [obj])."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return [obj]
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


class EPLayer:
    """One rank's share of the expert-parallel layer: T tokens of this rank, E global experts
    (this rank owns experts [rank E/R, (rank+1) E/R)), top-k routing, tile-padded pools."""

    def __init__(self, T: int, H: int, I: int, E: int, k: int, tile: int, group=None):
        rt = _rt()
        self.group = group
        self.R = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.rs = moe_shape(T, H, I, E, k, tile)
        self.ls = moe_ep_local_shape(self.rs, self.R)
        self.rows = moe_ep_pool_rows(self.rs, self.R)
        bf = torch.bfloat16
        # this rank's own plan of its tokens over the E experts, and its outputs
        self.plan_arena = torch.zeros(moe_plan_arena_bytes(self.rs), dtype=torch.uint8,
                                      device=self.device)
        self.own = moe_plan_bind(self.rs, self.plan_arena.data_ptr())
        off = self.own.counts - self.plan_arena.data_ptr()
        self.own_counts = self.plan_arena[off:off + 4 * E].view(torch.int32)
        self.counts_all = torch.zeros((self.R, E), dtype=torch.int32, device=self.device)
        self.act = torch.empty((self.rows, I), dtype=bf, device=self.device)
        self.out = torch.empty((max(T, 1), H), dtype=bf, device=self.device)
        self.word = torch.zeros(1, dtype=torch.int32, device=self.device)
        # the memory peers reach: separate allocations, so IPC handles cover them exactly
        self._owned = []
        self.ep_bytes = moe_ep_arena_bytes(self.rs, self.R)
        self.pool_ptr = self._alloc(self.rows * H * 2)
        self.ypool_ptr = self._alloc(self.rows * H * 2)
        self.ep_ptr = self._alloc(self.ep_bytes)
        _ok(rt.cudaMemset(self.ep_ptr, 0, self.ep_bytes))   # status word and tile flags
        self.ep = moe_ep_bind(self.rs, self.R, self.ep_ptr)
        flags_off = self.ep.local.tile_flags - self.ep_ptr
        # every rank's pool / ypool / EP arena, opened through CUDA IPC (own: as is)
        handles = [] if self.R == 1 else [bytes(_ok(rt.cudaIpcGetMemHandle(p)).reserved)
                                          for p in (self.pool_ptr, self.ypool_ptr, self.ep_ptr)]
        peers = exchange((self.rank, handles, flags_off), group)
        self._opened = []
        self.pool_ptrs, self.ypool_ptrs, self.flag_ptrs = [], [], []
        for r, hs, foff in peers:
            if r == self.rank:
                ptrs = [self.pool_ptr, self.ypool_ptr, self.ep_ptr]
            else:
                ptrs = []
                for raw in hs:
                    h = rt.cudaIpcMemHandle_t()
                    h.reserved = raw
                    p = int(_ok(rt.cudaIpcOpenMemHandle(h, rt.cudaIpcMemLazyEnablePeerAccess)))
                    self._opened.append(p)
                    ptrs.append(p)
            self.pool_ptrs.append(ptrs[0])
            self.ypool_ptrs.append(ptrs[1])
            self.flag_ptrs.append(ptrs[2] + foff)

    def _alloc(self, nbytes: int) -> int:
        p = int(_ok(_rt().cudaMalloc(max(int(nbytes), 256))))
        self._owned.append(p)
        return p

    def _barrier(self):
        # completes on this rank only after every rank enqueued it behind its own kernels
        if self.R > 1:
            dist.all_reduce(self.word, group=self.group)

    def forward(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                W1_local: torch.Tensor, W2_local: torch.Tensor,
                cfg: moe_config | None = None) -> torch.Tensor:
        """out [T, H] bf16 for this rank's tokens; W1_local / W2_local: this rank's E/R
        experts (given layout, or prepacked with cfg.packed_weights). With cfg.streaming the
        FFN takes pool tiles by their flags and the barrier before it is left out."""
        cfg = cfg or moe_config()
        st = torch.cuda.current_stream(self.device).cuda_stream
        s, R, r = self.rs, self.R, self.rank
        moe_plan(s, topk_idx.data_ptr(), self.own, 0, st)
        if R > 1:
            dist.all_gather_into_tensor(self.counts_all, self.own_counts, group=self.group)
        else:
            self.counts_all[0].copy_(self.own_counts)
        moe_ep_layout(s, R, r, self.counts_all.data_ptr(), self.ep, self.pool_ptr, st)
        moe_ep_dispatch(s, R, r, x.data_ptr(), self.own, self.ep, self.pool_ptrs, st,
                        self.flag_ptrs)
        if not cfg.streaming:
            self._barrier()
        moe_grouped_ffn(self.ls, self.pool_ptr, W1_local.data_ptr(), W2_local.data_ptr(),
                        self.ep.local, self.act.data_ptr(), self.ypool_ptr, cfg, st)
        self._barrier()
        out = self.out[: s.T]
        moe_ep_combine(s, R, r, self.ypool_ptrs, topk_w.data_ptr(), self.own, self.ep,
                       out.data_ptr(), st)
        return out

    def status(self) -> tuple[int, int]:
        """First device error of this rank's calls (its plan's word, else its pool plan's)."""
        code = moe_get_status(self.own)
        return code if code[0] != 0 else moe_get_status(self.ep.local)

    def close(self):
        rt = _rt()
        torch.cuda.synchronize(self.device)
        for p in self._opened:
            rt.cudaIpcCloseMemHandle(p)
        for p in self._owned:
            rt.cudaFree(p)
        self._opened, self._owned = [], []
