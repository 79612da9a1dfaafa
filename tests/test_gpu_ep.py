"""Expert parallelism inside one node (StreamEP README: dispatch and combine intranode over
NVLink), with R ranks emulated on one GPU: every rank's buffers live on the same device and
the "peer" pointers are plain pointers, which is what the kernels see on several GPUs too.
Each rank's pool must be bit for bit the part of one dropless pool over all ranks' pairs
that holds the rank's experts, and each rank's output must be bit for bit the single-GPU
layer's output for its tokens (the GEMMs compute each row independently of the others in
its chunk, and combine keeps the same FMA chain), and within the layer's tolerance of the
oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def _run_ep(cfg, R, drop=0.0, check_pools=True, streaming=0, calls=1):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import DEV, bf16_dev, bf16_host, f32_dev, i32_dev, weights_dev
    W1, W2 = weights_dev(cfg)
    rs = moe.moe_shape(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    ls = moe.moe_ep_local_shape(rs, R)
    Er = cfg.E // R
    rows = moe.moe_ep_pool_rows(rs, R)
    xs, idxs, ws = [], [], []
    for r in range(R):
        x = si.make_x(cfg, r)
        idx, w = si.make_routing(cfg, r)
        if drop > 0:
            idx = idx.copy()
            idx[np.random.default_rng(r).random(idx.shape) < drop] = -1
        xs.append(x), idxs.append(idx), ws.append(w)
    own = [moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile, identity=True)
           for _ in range(R)]
    ep_arena = [torch.zeros(moe.moe_ep_arena_bytes(rs, R), dtype=torch.uint8, device=DEV)
                for _ in range(R)]
    ep = [moe.moe_ep_bind(rs, R, a.data_ptr()) for a in ep_arena]
    pools = [torch.full((rows, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
             for _ in range(R)]
    acts = [torch.empty((rows, cfg.I), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    ypools = [torch.empty((rows, cfg.H), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    outs = [torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
            for _ in range(R)]
    dx = [bf16_dev(x) for x in xs]
    dw = [f32_dev(w) for w in ws]
    pool_ptrs = [p.data_ptr() for p in pools]
    ypool_ptrs = [p.data_ptr() for p in ypools]
    # with streaming, every stored row is counted on its owner's tile flag and each rank's
    # GEMM A takes a tile once its flag is full (here all dispatches precede the FFNs in
    # stream order, so the flags are full when it looks)
    flag_ptrs = [e_.local.tile_flags for e_ in ep] if streaming else None
    w1s = [W1[r * Er:(r + 1) * Er].contiguous() for r in range(R)]
    w2s = [W2[r * Er:(r + 1) * Er].contiguous() for r in range(R)]
    for _ in range(calls):
        # 1. each rank's own plan over the E global experts
        for r in range(R):
            moe.moe_plan(rs, i32_dev(idxs[r]).data_ptr(), own[r].plan, 0, 0)
        # 2. the all-gather of the counts (here: stacking the ranks' rows)
        C = torch.stack([own[r].plan_view("counts")[: cfg.E] for r in range(R)]).contiguous()
        # 3.-8. layout, dispatch into the owners' pools, each rank's FFN, combine from the owners
        for r in range(R):
            moe.moe_ep_layout(rs, R, r, C.data_ptr(), ep[r], pools[r].data_ptr(), 0)
        for r in range(R):
            moe.moe_ep_dispatch(rs, R, r, dx[r].data_ptr(), own[r].plan, ep[r], pool_ptrs, 0,
                                flag_ptrs)
        for r in range(R):
            moe.moe_grouped_ffn(ls, pools[r].data_ptr(), w1s[r].data_ptr(), w2s[r].data_ptr(),
                                ep[r].local, acts[r].data_ptr(), ypools[r].data_ptr(),
                                moe.moe_config(streaming=streaming), 0)
        for r in range(R):
            moe.moe_ep_combine(rs, R, r, ypool_ptrs, dw[r].data_ptr(), own[r].plan, ep[r],
                               outs[r].data_ptr(), 0)
    torch.cuda.synchronize()
    for r in range(R):   # moe_ep_combine leaves the rank's tile flags at zero for the next call
        n_tiles = rows // cfg.tile
        off = ep[r].local.tile_flags - ep_arena[r].data_ptr()
        assert not ep_arena[r][off:off + 4 * n_tiles].any(), f"rank {r} flags"
    for r in range(R):
        assert moe.moe_get_status(own[r].plan)[0] == 0
        assert moe.moe_get_status(ep[r].local)[0] == 0
    if check_pools:
        # every rank's pool = its experts' part of one pool over all ranks' pairs
        idx_all = np.concatenate(idxs)
        x_all = np.concatenate(xs)
        ref = oracle.get().plan(idx_all, cfg.E, cfg.tile)
        pool_all = oracle.get().pool(ref["row_src"], ref["P"], x_all, cfg.k)
        for r in range(R):
            a, b = int(ref["offsets"][r * Er]), int(ref["offsets"][(r + 1) * Er])
            np.testing.assert_array_equal(bf16_host(pools[r][: b - a]), pool_all[a:b],
                                          err_msg=f"rank {r} pool")
    res = []
    for r in range(R):
        # the single-GPU layer on the same tokens and all experts
        single = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
        o = single.forward(dx[r], i32_dev(idxs[r]), dw[r], W1, W2, moe.moe_config())
        torch.cuda.synchronize()
        res.append((outs[r], o.clone()))
        single.close()
    for b in own:
        b.close()
    return xs, idxs, ws, res


EP_SHAPES = [
    # name, T per rank, H, I, E, k, tile, R
    ("R2", 200, 256, 256, 8, 2, 64, 2),
    ("R4-tile128", 150, 384, 128, 16, 3, 128, 4),
    ("R8-k8", 96, 256, 192, 32, 8, 64, 8),
]


@pytest.mark.parametrize("streaming", [0, 1])
@pytest.mark.parametrize("shape", EP_SHAPES, ids=[s[0] for s in EP_SHAPES])
@pytest.mark.parametrize("drop", [0.0, 0.2])
def test_ep_emulated_ranks_match_single_gpu_and_oracle(shape, drop, streaming):
    from gpu_helpers import assert_layer_close, to_f64
    name, T, H, I, E, k, tile, R = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=555 + T)
    xs, idxs, ws, res = _run_ep(cfg, R, drop=drop, streaming=streaming, calls=1 + streaming)
    W1h = [si.make_w1_expert(cfg, e) for e in range(E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(E)]
    for r, (ep_out, single_out) in enumerate(res):
        assert torch.equal(ep_out.view(torch.int16), single_out.view(torch.int16)), f"rank {r}"
        ref = oracle.get().moe_forward(xs[r], idxs[r], ws[r], W1h, W2h)
        assert_layer_close(to_f64(ep_out), ref, f"{name} rank {r}")


def test_ep_deepseek_shape_eight_ranks():
    """Eight emulated ranks of the DeepSeek-V3 expert shape (H=7168, I=2048, 256 experts,
    top-8) with 256 tokens each: outputs bit for bit the single-GPU layer's, sampled tokens
    against the oracle."""
    from gpu_helpers import assert_layer_close, sample_tokens, to_f64
    base = si.CONFIGS["deepseek_v3"]
    cfg = si.custom("ep-ds", T=256, H=base.H, I=base.I, E=base.E, k=base.k, tile=base.tile,
                    seed=base.seed, routing=base.routing, bias_sigma=base.bias_sigma)
    xs, idxs, ws, res = _run_ep(cfg, 8, check_pools=False)
    for r, (ep_out, single_out) in enumerate(res):
        assert torch.equal(ep_out.view(torch.int16), single_out.view(torch.int16)), f"rank {r}"
    tok = sample_tokens(cfg.T, 8, seed=3)
    W1h = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    ref = oracle.get().moe_forward(xs[0][tok], idxs[0][tok], ws[0][tok], W1h, W2h)
    assert_layer_close(to_f64(res[0][0][torch.from_numpy(tok).to(res[0][0].device)]), ref,
                       "deepseek-shaped EP rank 0")


@pytest.mark.parametrize("bad", ["huge", "negative", "too_many_rows"])
def test_ep_counts_that_disagree_with_the_plans_are_reported_not_followed(bad):
    """A host-made failure: all_counts that no set of moe_plan calls can produce. The layout
    clamps them and reports MOE_ERR_POOL_OVERFLOW; dispatch and combine place no row outside
    a pool (guard rows after each pool stay untouched) and the context stays usable."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import DEV, bf16_dev, f32_dev, i32_dev
    R = 2
    cfg = si.custom("ep-bad", T=64, H=128, I=128, E=4, k=2, tile=64, seed=31)
    rs = moe.moe_shape(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    rows = moe.moe_ep_pool_rows(rs, R)
    guard = 64
    own = [moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile, identity=True)
           for _ in range(R)]
    arenas = [torch.zeros(moe.moe_ep_arena_bytes(rs, R), dtype=torch.uint8, device=DEV)
              for _ in range(R)]
    ep = [moe.moe_ep_bind(rs, R, a.data_ptr()) for a in arenas]
    pools = [torch.full((rows + guard, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
             for _ in range(R)]
    ypools = [torch.zeros((rows + guard, cfg.H), dtype=torch.bfloat16, device=DEV)
              for _ in range(R)]
    outs = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    xs = [bf16_dev(si.make_x(cfg, r)) for r in range(R)]
    routs = [si.make_routing(cfg, r) for r in range(R)]
    for r in range(R):
        moe.moe_plan(rs, i32_dev(routs[r][0]).data_ptr(), own[r].plan, 0, 0)
    C = torch.stack([own[r].plan_view("counts")[: cfg.E] for r in range(R)]).contiguous()
    if bad == "huge":
        C[0, 1] = 1 << 30
    elif bad == "negative":
        C[1, 2] = -5
    else:                      # within [0, T k] each, but moving rank 0's rows down
        C[0, 0] = cfg.T * cfg.k
    for r in range(R):
        moe.moe_ep_layout(rs, R, r, C.data_ptr(), ep[r], pools[r].data_ptr(), 0)
    for r in range(R):
        moe.moe_ep_dispatch(rs, R, r, xs[r].data_ptr(), own[r].plan, ep[r],
                            [p.data_ptr() for p in pools], 0,
                            [e_.local.tile_flags for e_ in ep])
    for r in range(R):
        moe.moe_ep_combine(rs, R, r, [p.data_ptr() for p in ypools],
                           f32_dev(routs[r][1]).data_ptr(), own[r].plan, ep[r],
                           outs[r].data_ptr(), 0)
    torch.cuda.synchronize()
    codes = [moe.moe_get_status(ep[r].local)[0] for r in range(R)] + \
            [moe.moe_get_status(own[r].plan)[0] for r in range(R)]
    assert moe.MOE_ERR_POOL_OVERFLOW in codes, codes
    assert set(codes) <= {0, moe.MOE_ERR_POOL_OVERFLOW}, codes
    for r in range(R):
        assert torch.isnan(pools[r][rows:].float()).all(), f"rank {r} guard rows written"
    # the context still works: a clean single-GPU layer call
    single = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    from gpu_helpers import weights_dev
    W1, W2 = weights_dev(cfg)
    single.forward(xs[0], i32_dev(routs[0][0]), f32_dev(routs[0][1]), W1, W2, moe.moe_config())
    torch.cuda.synchronize()
    assert moe.moe_get_status(single.plan)[0] == 0
    single.close()
    for b in own:
        b.close()


def test_bench_ep_section_matches_single_gpu_layer():
    """bench.py's expert-parallel timing section on a small workload, with prepacked weights
    sliced per rank: its output equals the single-GPU layer's bit for bit and its rates are
    positive."""
    import bench
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import DEV, bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("ep-bench", T=512, H=512, I=256, E=16, k=4, tile=128, seed=91)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    W1p, W2p = buf.pack_weights(W1, W2)
    x = bf16_dev(si.make_x(cfg))
    idx, w = si.make_routing(cfg)
    di, dw = i32_dev(idx), f32_dev(w)
    single = buf.forward(x, di, dw, W1p, W2p, moe.moe_config(packed_weights=1))
    torch.cuda.synchronize()
    single = single.clone()
    peaks, _ = bench.load_peaks()
    res = bench.time_ep(moe, cfg, DEV, x, di, dw, W1p, W2p, 1, 4, single, peaks, reps=2)
    assert res["matches_single_gpu_layer"]
    assert res["ms_per_layer_call"] > 0 and res["dispatch_gbs"] > 0 and res["combine_gbs"] > 0
    assert res["nvlink"]["remote_pairs_per_rank_max"] <= cfg.T // 4 * cfg.k
    buf.close()


def test_ep_streaming_ffn_times_out_without_the_dispatch_flags():
    """A host-made failure: dispatch without tile flags, then a streaming grouped FFN on the
    owner: its pool tiles never fill (only the padding rows were counted), GEMM A's bounded
    wait reports MOE_ERR_FLAG_TIMEOUT, and after moe_clear_status a non-streaming FFN on the
    same context is correct."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import DEV, bf16_dev, i32_dev, weights_dev
    R = 2
    cfg = si.custom("ep-to", T=128, H=256, I=128, E=4, k=2, tile=64, seed=5)
    W1, W2 = weights_dev(cfg)
    rs = moe.moe_shape(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    ls = moe.moe_ep_local_shape(rs, R)
    rows = moe.moe_ep_pool_rows(rs, R)
    own = [moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile, identity=True)
           for _ in range(R)]
    arenas = [torch.zeros(moe.moe_ep_arena_bytes(rs, R), dtype=torch.uint8, device=DEV)
              for _ in range(R)]
    ep = [moe.moe_ep_bind(rs, R, a.data_ptr()) for a in arenas]
    pools = [torch.empty((rows, cfg.H), dtype=torch.bfloat16, device=DEV) for _ in range(R)]
    act = torch.empty((rows, cfg.I), dtype=torch.bfloat16, device=DEV)
    ypool = torch.empty((rows, cfg.H), dtype=torch.bfloat16, device=DEV)
    xs = [bf16_dev(si.make_x(cfg, r)) for r in range(R)]
    for r in range(R):
        moe.moe_plan(rs, i32_dev(si.make_routing(cfg, r)[0]).data_ptr(), own[r].plan, 0, 0)
    C = torch.stack([own[r].plan_view("counts")[: cfg.E] for r in range(R)]).contiguous()
    for r in range(R):
        moe.moe_ep_layout(rs, R, r, C.data_ptr(), ep[r], pools[r].data_ptr(), 0)
    for r in range(R):
        moe.moe_ep_dispatch(rs, R, r, xs[r].data_ptr(), own[r].plan, ep[r],
                            [p.data_ptr() for p in pools], 0)        # no flags
    Er = cfg.E // R
    w1, w2 = W1[:Er].contiguous(), W2[:Er].contiguous()
    moe.moe_grouped_ffn(ls, pools[0].data_ptr(), w1.data_ptr(), w2.data_ptr(), ep[0].local,
                        act.data_ptr(), ypool.data_ptr(),
                        moe.moe_config(streaming=1, wait_timeout_us=2000), 0)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(ep[0].local)
    assert code == moe.MOE_ERR_FLAG_TIMEOUT, (moe.moe_strerror(code), aux)
    moe.moe_clear_status(ep[0].local, 0)
    moe.moe_grouped_ffn(ls, pools[0].data_ptr(), w1.data_ptr(), w2.data_ptr(), ep[0].local,
                        act.data_ptr(), ypool.data_ptr(), moe.moe_config(), 0)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ep[0].local)[0] == 0
    for b in own:
        b.close()


@pytest.mark.parametrize("streaming", [0, 1])
def test_ep_layer_one_rank_matches_single_gpu(streaming):
    """EPLayer (the process-group runner of the EP calls) with one rank: its peer pointers are
    its own buffers; two calls in a row equal the single-GPU layer bit for bit."""
    import combine_moe_plan_03_b200 as moe
    from combine_moe_plan_03_b200.ep import EPLayer
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("ep-layer", T=300, H=384, I=256, E=6, k=2, tile=64, seed=71)
    W1, W2 = weights_dev(cfg)
    layer = EPLayer(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    single = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    for mb in range(2):
        x, di, dw = bf16_dev(si.make_x(cfg, mb)), None, None
        idx, w = si.make_routing(cfg, mb)
        di, dw = i32_dev(idx), f32_dev(w)
        torch.cuda.synchronize()
        out = layer.forward(x, di, dw, W1, W2, moe.moe_config(streaming=streaming))
        ref = single.forward(x, di, dw, W1, W2)
        torch.cuda.synchronize()
        assert layer.status()[0] == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), mb
    layer.close()
    single.close()
