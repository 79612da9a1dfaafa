"""Device-side error reporting without faults or hangs: bad expert index, a streaming FFN
whose tiles never fill (bounded wait), and a usable context afterwards."""
import numpy as np
import pytest
import torch

import synth_inputs as si

pytestmark = pytest.mark.gpu


def test_bad_index_reported_and_pair_dropped():
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import i32_dev
    T, E, k = 64, 8, 2
    idx = np.random.default_rng(0).integers(0, E, size=(T, k)).astype(np.int32)
    idx[10, 1] = 8
    idx[20, 0] = -5
    buf = moe.MoELayerBuffers(T, 64, 64, E, k, 64, identity=True)
    moe.moe_plan(buf.shape, i32_dev(idx).data_ptr(), buf.plan, 0, 0)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == moe.MOE_ERR_BAD_INDEX and aux in (21, 40)
    pr = buf.plan_view("pool_row")[: T * k].cpu().numpy()
    assert pr[21] == -1 and pr[40] == -1
    moe.moe_clear_status(buf.plan, 0)
    assert moe.moe_get_status(buf.plan)[0] == 0
    buf.close()


@pytest.mark.parametrize("ffn_kernel", [1, 2], ids=["one_sm", "sm_pair"])
def test_streaming_wait_times_out_then_context_is_usable(ffn_kernel):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("to", T=128, H=128, I=128, E=4, k=2, tile=64, seed=3)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    moe.moe_plan(buf.shape, i32_dev(idx).data_ptr(), buf.plan, 0, 0)
    # no dispatch: the tile flags stay 0, the streaming FFN must give up after ~1 ms
    moe.moe_grouped_ffn(buf.shape, buf.pool.data_ptr(), W1.data_ptr(), W2.data_ptr(), buf.plan,
                        buf.act.data_ptr(), buf.ypool.data_ptr(),
                        moe.moe_config(1, 0, 1000, 0, ffn_kernel), 0)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == moe.MOE_ERR_FLAG_TIMEOUT and aux >= 0
    # the context still works: a full layer afterwards is correct
    moe.moe_clear_status(buf.plan, 0)
    out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2,
                      moe.moe_config(0, 0, 0, 0, ffn_kernel))
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    assert torch.isfinite(out.float()).all()
    buf.close()


@pytest.mark.parametrize("ffn_kernel", [1, 2], ids=["one_sm", "sm_pair"])
def test_ffn_rerun_on_same_plan_after_timeout(ffn_kernel):
    """A grouped FFN that gave up (its tile flags never filled) leaves the unit counters
    ready for the next launch: after moe_clear_status the FFN runs again on the same plan,
    without a new moe_plan, and the layer matches the oracle on every token."""
    import combine_moe_plan_03_b200 as moe
    import oracle
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("rerun", T=192, H=128, I=256, E=4, k=2, tile=64, seed=21)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    shape = buf.shape
    d_idx, d_w, d_x = i32_dev(idx), f32_dev(w), bf16_dev(x)
    moe.moe_plan(shape, d_idx.data_ptr(), buf.plan, 0, 0)
    ffn = lambda c: moe.moe_grouped_ffn(shape, buf.pool.data_ptr(), W1.data_ptr(),  # noqa: E731
                                        W2.data_ptr(), buf.plan, buf.act.data_ptr(),
                                        buf.ypool.data_ptr(), c, 0)
    ffn(moe.moe_config(1, 0, 1000, 0, ffn_kernel))      # flags never fill: gives up after 1 ms
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == moe.MOE_ERR_FLAG_TIMEOUT
    moe.moe_clear_status(buf.plan, 0)
    buf.ypool.view(torch.int16).fill_(0x7FC0)            # poisoned: every live row is rewritten
    moe.moe_dispatch(shape, d_x.data_ptr(), buf.plan, buf.pool.data_ptr(), False, 0)
    ffn(moe.moe_config(0, 0, 0, 0, ffn_kernel))          # same plan, no moe_plan in between
    moe.moe_combine(shape, buf.ypool.data_ptr(), d_w.data_ptr(), buf.plan, buf.out.data_ptr(), 0)
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    W1h = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    ref = oracle.get().moe_forward(x, idx, w, W1h, W2h)
    assert_layer_close(to_f64(buf.out), ref, "re-run after a timeout")
    buf.close()
