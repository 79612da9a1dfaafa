"""Early combine (StreamEP README, How it works, "Per-tile streaming": combine starts on a
token as soon as its compute is done): GEMM Y counts each token's stored expert rows and the
GEMM's CTAs combine ready tokens while the last units still run. Its output must equal the
serial combine's bit for bit (the same fp32 FMA chain), and the layer must match the oracle
within the layer's tolerance; a token whose rows never arrive ends in a bounded wait."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu

SHAPES = [
    # name, T, H, I, E, k, tile
    ("tiny-like", 256, 256, 512, 8, 2, 64),
    ("ragged-H", 300, 320, 256, 4, 2, 128),      # GEMM Y's one 512-column block half empty
    ("wide-H", 150, 1088, 128, 5, 3, 64),        # three column blocks, the last ragged
    ("one-expert", 130, 320, 384, 1, 1, 128),
    ("k8", 96, 512, 256, 16, 8, 64),
]


def _layer(cfg, early, streaming=0, drop=0.0, W=None):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    if drop > 0:
        rng = np.random.default_rng(5)
        idx = idx.copy()
        idx[rng.random(idx.shape) < drop] = -1
        idx[: 3] = -1                                           # tokens with no live pair
    W1, W2 = W if W is not None else weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    for t in (buf.pool, buf.act, buf.ypool, buf.out):
        t.view(torch.int16).fill_(0x7FC0)                       # poisoned storage
    out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2,
                      moe.moe_config(streaming=streaming, early_combine=early))
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    return buf, out.clone(), x, idx, w, (W1, W2)


@pytest.mark.parametrize("streaming", [0, 1])
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_early_combine_equals_serial_combine_and_oracle(shape, streaming):
    from gpu_helpers import assert_layer_close, to_f64
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=4321 + T)
    b0, serial, x, idx, w, W = _layer(cfg, early=0, streaming=streaming, drop=0.1)
    b1, early, *_ = _layer(cfg, early=1, streaming=streaming, drop=0.1, W=W)
    assert torch.equal(early.view(torch.int16), serial.view(torch.int16))
    W1h = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    ref = oracle.get().moe_forward(x, idx, w, W1h, W2h)
    assert_layer_close(to_f64(early), ref, f"{name} early combine")
    assert not to_f64(early)[:3].any()                          # no live pair: zero output
    b0.close()
    b1.close()


def test_early_combine_repeated_calls_on_one_plan_buffer():
    """Back-to-back layer calls with early combine reuse the counters and the queue: the
    plan resets them every call."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("rep", T=200, H=256, I=256, E=6, k=2, tile=64, seed=77)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    outs = []
    for mb in range(3):
        x = si.make_x(cfg, mb)
        idx, w = si.make_routing(cfg, mb)
        args = (bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2)
        # out is ready once the layer's compute stream reaches it: synchronise before copying
        a = buf.forward(*args, moe.moe_config())
        torch.cuda.synchronize()
        a = a.clone()
        b = buf.forward(*args, moe.moe_config(early_combine=1))
        torch.cuda.synchronize()
        b = b.clone()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), mb
        outs.append(b)
    assert moe.moe_get_status(buf.plan)[0] == 0
    assert not torch.equal(outs[0], outs[1])
    buf.close()


def test_early_combine_entry_point_through_the_c_abi():
    """moe_plan, moe_dispatch armed for early combine, moe_grouped_ffn_combine: out equals
    moe_grouped_ffn followed by moe_combine, bit for bit."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("abi", T=333, H=384, I=192, E=7, k=3, tile=64, seed=99)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    s = buf.shape
    dx, di, dw = bf16_dev(x), i32_dev(idx), f32_dev(w)
    moe.moe_plan(s, di.data_ptr(), buf.plan, 0, 0)
    moe.moe_dispatch(s, dx.data_ptr(), buf.plan, buf.pool.data_ptr(), 0, 0)
    moe.moe_grouped_ffn(s, buf.pool.data_ptr(), W1.data_ptr(), W2.data_ptr(), buf.plan,
                        buf.act.data_ptr(), buf.ypool.data_ptr(), moe.moe_config(), 0)
    ref = torch.empty_like(buf.out)
    moe.moe_combine(s, buf.ypool.data_ptr(), dw.data_ptr(), buf.plan, ref.data_ptr(), 0)
    got = torch.full_like(buf.out, float("nan"))
    moe.moe_plan(s, di.data_ptr(), buf.plan, 0, 0)
    moe.moe_dispatch(s, dx.data_ptr(), buf.plan, buf.pool.data_ptr(),
                     moe.MOE_DISPATCH_ARM_COMBINE, 0)
    moe.moe_grouped_ffn_combine(s, buf.pool.data_ptr(), W1.data_ptr(), W2.data_ptr(), buf.plan,
                                buf.act.data_ptr(), buf.ypool.data_ptr(), dw.data_ptr(),
                                got.data_ptr(), moe.moe_config(early_combine=1), 0)
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    # every queue position was taken exactly once: head passed T, tail == T
    ready = buf.plan_view("ready")[: cfg.T + 4].cpu().numpy()
    assert ready[cfg.T + 1] == cfg.T and ready[cfg.T] >= cfg.T
    assert sorted(ready[: cfg.T] - 1) == list(range(cfg.T))
    buf.close()


def test_early_combine_times_out_when_the_counters_are_not_armed():
    """A host-made failure: dispatch without MOE_DISPATCH_ARM_COMBINE leaves every token's
    count at zero, so no token is ever queued; the combine's bounded wait (1 ms) reports
    MOE_ERR_COMBINE_TIMEOUT and the context stays usable."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("to-ec", T=128, H=256, I=128, E=4, k=2, tile=64, seed=8)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    s = buf.shape
    dx, di, dw = bf16_dev(x), i32_dev(idx), f32_dev(w)
    moe.moe_plan(s, di.data_ptr(), buf.plan, 0, 0)
    moe.moe_dispatch(s, dx.data_ptr(), buf.plan, buf.pool.data_ptr(), 0, 0)   # not armed
    moe.moe_grouped_ffn_combine(s, buf.pool.data_ptr(), W1.data_ptr(), W2.data_ptr(), buf.plan,
                                buf.act.data_ptr(), buf.ypool.data_ptr(), dw.data_ptr(),
                                buf.out.data_ptr(), moe.moe_config(wait_timeout_us=1000,
                                                                   early_combine=1), 0)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == moe.MOE_ERR_COMBINE_TIMEOUT and 0 <= aux < cfg.T
    moe.moe_clear_status(buf.plan, 0)
    out = buf.forward(dx, di, dw, W1, W2, moe.moe_config(early_combine=1))
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    W1h = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    assert_layer_close(to_f64(out), oracle.get().moe_forward(x, idx, w, W1h, W2h), "after")
    buf.close()
