"""moe_dispatch (bit-exact pool, zero padding, tile flags) and moe_combine (identity experts)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def _layer(cfg, mb=0):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev
    x = si.make_x(cfg, mb)
    idx, w = si.make_routing(cfg, mb)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, max(cfg.I, 64), cfg.E, cfg.k, cfg.tile, identity=True)
    return buf, x, idx, w, bf16_dev(x), i32_dev(idx), f32_dev(w)


@pytest.mark.parametrize("name,signal", [
    ("tiny", 0), ("tiny", 1), ("qwen3_235b_a22b", 0), ("qwen3_235b_a22b", 1),
    ("dc_sweep_T4096_zipf", 0), ("dc_sweep_T4096_zipf", 1), ("deepseek_v3", 1)])
def test_dispatch_pool_exact(name, signal):
    """signal = 0: the token-order dispatch; 1: the tile-order dispatch of the streaming
    layer (tiles gathered through row_src in pool order, each tile's flag raised once)."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_host
    cfg = si.CONFIGS[name]
    buf, x, idx, w, dx, didx, dw = _layer(cfg)
    buf.pool.view(torch.int16).fill_(0x7FC0)                  # poison: NaN pattern
    moe.moe_plan(buf.shape, didx.data_ptr(), buf.plan, 0, 0)
    moe.moe_dispatch(buf.shape, dx.data_ptr(), buf.plan, buf.pool.data_ptr(), signal, 0)
    torch.cuda.synchronize()
    ref = oracle.get().plan(idx, cfg.E, cfg.tile)
    P = ref["P"]
    want = oracle.get().pool(ref["row_src"], P, x, cfg.k)
    got = bf16_host(buf.pool[:P])
    np.testing.assert_array_equal(got, want)
    flags = buf.plan_view("tile_flags")[: P // cfg.tile].cpu().numpy().view(np.uint32)
    assert np.all(flags == (cfg.tile if signal else 0))       # every tile fully landed
    assert moe.moe_get_status(buf.plan)[0] == 0
    buf.close()


def _combine_bound(x, idx, w, ref):
    """fp32 FMA chain over k terms then one bf16 rounding:
    |out - y| <= 2^-8 |y| + k * 2^-23 * sum_j |w_j x| (elementwise)."""
    xf = si.bf16_to_f64(x)
    aw = np.where(idx >= 0, np.abs(w.astype(np.float64)), 0.0).sum(1)
    return 2.0 ** -8 * np.abs(ref) + idx.shape[1] * 2.0 ** -23 * aw[:, None] * np.abs(xf) + 1e-30


@pytest.mark.parametrize("name", ["tiny", "dc_sweep_T1024_uniform", "dc_sweep_T4096_zipf"])
def test_identity_layer_elementwise(name):
    """Identity experts through the whole layer (plan, dispatch, combine on two streams)."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_host
    cfg = si.CONFIGS[name]
    buf, x, idx, w, dx, didx, dw = _layer(cfg)
    buf.out.view(torch.int16).fill_(0x7FC0)
    out = buf.forward(dx, didx, dw, None, None)
    torch.cuda.synchronize()
    got = si.bf16_to_f64(bf16_host(out))
    ref = oracle.get().moe_forward_identity(x, idx, w)
    assert np.all(np.abs(got - ref) <= _combine_bound(x, idx, w, ref))
    # closed form: y = x * sum_j w_j (sum of weights ~ 1)
    np.testing.assert_allclose(got, si.bf16_to_f64(x) * w.sum(1, dtype=np.float64)[:, None],
                               rtol=1e-2, atol=1e-2)
    assert moe.moe_get_status(buf.plan)[0] == 0
    buf.close()


def test_combine_random_pool_with_dropped_pairs_and_special_values():
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, bf16_host, f32_dev, i32_dev
    rng = np.random.default_rng(11)
    T, H, E, k, tile = 333, 192, 12, 5, 64
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    w = rng.standard_normal((T, k)).astype(np.float32)
    w[::7, 0] = 0.0
    buf = moe.MoELayerBuffers(T, H, 64, E, k, tile, identity=True)
    moe.moe_plan(buf.shape, i32_dev(idx).data_ptr(), buf.plan, 0, 0)
    ref_plan = oracle.get().plan(idx, E, tile)
    yp = si.f32_to_bf16_bits(rng.standard_normal((buf.P_max, H)).astype(np.float32) * 3)
    yp[5, :8] = si.f32_to_bf16_bits(np.array([0, -0.0, 1e30, -1e30, 3e38, -3e38, 1e-30, 7],
                                             np.float32))
    dyp = bf16_dev(yp)
    moe.moe_combine(buf.shape, dyp.data_ptr(), f32_dev(w).data_ptr(), buf.plan,
                    buf.out.data_ptr(), 0)
    torch.cuda.synchronize()
    got = si.bf16_to_f64(bf16_host(buf.out[:T]))
    ref = oracle.get().combine(ref_plan["pool_row"], w, yp[: ref_plan["P"]])
    fin = np.isfinite(got) & np.isfinite(ref) & (np.abs(ref) < 3e38)
    ypf = si.bf16_to_f64(yp)
    aw = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            p = ref_plan["pool_row"][t, j]
            if p >= 0:
                aw[t] += abs(float(w[t, j])) * np.abs(ypf[p])
    bound = 2.0 ** -8 * np.abs(ref) + k * 2.0 ** -23 * aw + 1e-30
    assert np.all(np.abs(got - ref)[fin] <= bound[fin])
    buf.close()
