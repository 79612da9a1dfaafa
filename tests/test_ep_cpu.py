"""Expert parallelism, host side (no GPU): the EP sizes and arena binding, argument checks, and
the one exchange step of the layer (the all-gather of every rank's per-expert counts) over two
gloo ranks, with the pool layout it implies checked against the oracle's plan of all ranks'
pairs."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth_inputs as si


def test_ep_sizes_and_bind_are_host_only():
    import combine_moe_plan_03_b200 as moe
    rs = moe.moe_shape(256, 7168, 2048, 256, 8, 128)
    for R in (1, 2, 4, 8):
        ls = moe.moe_ep_local_shape(rs, R)
        assert (ls.T, ls.H, ls.I, ls.E, ls.k, ls.tile) == (256 * R, 7168, 2048, 256 // R, 8, 128)
        rows = moe.moe_ep_pool_rows(rs, R)
        pairs = 256 * R * 8
        assert rows == -(-(pairs + min(256 // R, pairs) * 127) // 128) * 128
        assert rows == moe.moe_pool_rows_max(ls)
        nbytes = moe.moe_ep_arena_bytes(rs, R)
        ep = moe.moe_ep_bind(rs, R, 1 << 20)
        fields = [ep.counts, ep.offsets, ep.src_base, ep.tile_expert, ep.mblk, ep.meta] + \
                 [getattr(ep.local, f) for f, _ in moe.moe_plan_buffers._fields_]
        assert all(f % 256 == 0 for f in fields)
        assert fields == sorted(fields) and fields[-1] < (1 << 20) + nbytes
        # the pool plan's scratch holds the per-source counts of the rank's experts
        assert ep.local.status - ep.local.workspace >= 4 * ((256 // R) * R + 8)


@pytest.mark.parametrize("R,E", [(0, 8), (9, 72), (3, 8), (-1, 8)])
def test_ep_rejects_bad_rank_counts(R, E):
    import combine_moe_plan_03_b200 as moe
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_ep_arena_bytes(moe.moe_shape(64, 128, 128, E, 2, 64), R)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG


def test_ep_calls_check_ranks_and_pointers_on_the_host():
    import combine_moe_plan_03_b200 as moe
    rs = moe.moe_shape(64, 128, 128, 8, 2, 64)
    ep = moe.moe_ep_bind(rs, 2, 1 << 20)
    own = moe.moe_plan_bind(rs, 1 << 24)
    with pytest.raises(moe.MoEError) as ei:              # rank outside [0, R)
        moe.moe_ep_layout(rs, 2, 2, 1 << 26, ep, 1 << 27)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:              # a missing peer pool
        moe.moe_ep_dispatch(rs, 2, 0, 1 << 26, own, ep, [1 << 27, 0])
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:              # a misaligned tile-flag pointer
        moe.moe_ep_dispatch(rs, 2, 0, 1 << 26, own, ep, [1 << 27, 1 << 28], 0, [1 << 20, 2])
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:              # a misaligned peer ypool
        moe.moe_ep_combine(rs, 2, 1, [1 << 27, (1 << 28) + 8], 1 << 26, own, ep, 1 << 25)
    assert ei.value.code == moe.MOE_ERR_MISALIGNED


def _layout_rows(C, own_idx, rank, E, tile):
    """Where the pairs of `rank` go: (owner, row) per pair, from the gathered counts C [R][E]
    and the rank's own stable order, by the layout rule (owner d of expert e = e // (E/R);
    rows of e from ranks 0, 1, ... in turn, each in flat pair order; experts padded to the
    tile; each owner's pool starts at its first expert)."""
    R = C.shape[0]
    Er = E // R
    tot = C.sum(0)
    padded = -(-tot // tile) * tile
    off = np.concatenate([[0], np.cumsum(padded)])
    before = np.cumsum(C, 0) - C                       # rows of e from ranks before s
    seen = np.zeros(E, np.int64)
    out = []
    for e in own_idx.reshape(-1):
        if e < 0:
            out.append((-1, -1))
            continue
        d = e // Er
        out.append((d, off[e] - off[d * Er] + before[rank, e] + seen[e]))
        seen[e] += 1
    return out


def _ep_rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    cfg = si.custom("ep-cpu", T=96, H=64, I=64, E=8, k=3, tile=64, seed=17)
    idx, _ = si.make_routing(cfg, rank)
    counts = torch.from_numpy(np.bincount(idx[idx >= 0], minlength=cfg.E).astype(np.int32))
    gathered = [torch.zeros_like(counts) for _ in range(world)]
    dist.all_gather(gathered, counts)                   # the layer's one exchange step
    C = torch.stack(gathered).numpy()
    q.put((rank, C, _layout_rows(C, idx, rank, cfg.E, cfg.tile)))
    dist.destroy_process_group()


def test_ep_count_exchange_over_two_gloo_ranks_and_layout_against_the_oracle():
    import oracle
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {r: (C, rows) for r, C, rows in results}
    cfg = si.custom("ep-cpu", T=96, H=64, I=64, E=8, k=3, tile=64, seed=17)
    idx_all = np.concatenate([si.make_routing(cfg, r)[0] for r in range(2)])
    np.testing.assert_array_equal(by_rank[0][0], by_rank[1][0])   # both ranks see the same C
    # the oracle's plan of all ranks' pairs: owner d's pool is its experts' part, re-based
    ref = oracle.get().plan(idx_all, cfg.E, cfg.tile)
    Er = cfg.E // 2
    pairs = cfg.T * cfg.k
    for r in range(2):
        for f, (d, row) in enumerate(by_rank[r][1]):
            g = ref["pool_row"].reshape(-1)[r * pairs + f]
            if g < 0:
                assert (d, row) == (-1, -1)
                continue
            assert row == g - ref["offsets"][d * Er]


def test_backward_streaming_needs_two_streams_and_events():
    """Host checks only (no launch): moe_backward refuses cfg.streaming (it has one stream);
    moe_backward_streams refuses it with one stream for both roles or without events."""
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(64, 128, 128, 4, 2, 64)
    plan = moe.moe_plan_bind(s, 1 << 24)
    a = [1 << 28] * 12
    cfg = moe.moe_config(streaming=1)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_backward(s, *a[:4], plan, *a[4:], 0, 0, cfg, 0)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    for comm, comp, ea, eb in ((1 << 12, 1 << 12, 1 << 13, 1 << 14), (1 << 12, 1 << 15, 0, 1 << 14)):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_backward_streams(s, *a[:4], plan, *a[4:], 0, 0, cfg, comm, comp, ea, eb)
        assert ei.value.code == moe.MOE_ERR_INVALID_ARG


def _exchange_rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from combine_moe_plan_03_b200.ep import exchange
    got = exchange((rank, [bytes([rank] * 64), bytes([rank + 1] * 64)], 256 * (rank + 1)))
    q.put((rank, got))
    dist.destroy_process_group()


def test_ep_layer_handle_exchange_over_two_gloo_ranks():
    """EPLayer's one host-side exchange (each rank's IPC handles and flag offset, gathered in
    rank order), over two gloo ranks on the CPU."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(2):
        assert [g[0] for g in res[rank]] == [0, 1]
        assert res[rank][1][1][0] == bytes([1] * 64) and res[rank][0][2] == 256
