"""The router on the device (softmax top-k, renormalised) and the router fused with the
plan, against the oracle: the chosen experts exactly, the weights within fp32 rounding
(expf and one division: relative 2e-6), the plan maps bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def _logits(cfg, T=None):
    T = cfg.T if T is None else T
    lg = si.normal_f32(cfg.seed, si.STREAM_LOGITS, 0, T * cfg.E).reshape(T, cfg.E)
    bias = si.normal_f32(cfg.seed, si.STREAM_BIAS, 0, cfg.E, cfg.bias_sigma) \
        if cfg.routing == "softmax_bias" else None
    return lg, bias


def _route_gpu(T, E, k, lg, bias, fused=False, tile=128):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import f32_dev
    dl = f32_dev(lg)
    db = f32_dev(bias) if bias is not None else None
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    buf = None
    if fused:
        buf = moe.MoELayerBuffers(T, 64, 64, E, k, tile, identity=True)
        moe.moe_route_plan(buf.shape, dl.data_ptr(), db.data_ptr() if db is not None else 0,
                           idx.data_ptr(), w.data_ptr(), buf.plan, 0, 0)
    else:
        moe.moe_route(moe.moe_shape(T, 64, 64, E, k, tile), dl.data_ptr(),
                      db.data_ptr() if db is not None else 0, idx.data_ptr(), w.data_ptr(), 0)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), buf


def _check(idx, w, ridx, rw):
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w.astype(np.float64), rw, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["tiny", "qwen3_235b_a22b", "deepseek_v3"])
def test_route_workload_logits(name):
    cfg = si.CONFIGS[name]
    lg, bias = _logits(cfg)
    idx, w, _ = _route_gpu(cfg.T, cfg.E, cfg.k, lg, bias)
    ridx, rw = oracle.get().route(lg, cfg.k, bias)
    _check(idx, w, ridx, rw)
    gidx, _ = si.make_routing(cfg)            # the input generator makes the same choice
    np.testing.assert_array_equal(idx, gidx)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (77, 5, 5), (300, 1024, 32), (64, 33, 1),
                                   (129, 256, 8)])
def test_route_shapes(T, E, k):
    rng = np.random.default_rng(T + E + k)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.5).astype(np.float32) if E > 1 else None
    idx, w, _ = _route_gpu(T, E, k, lg, bias)
    _check(idx, w, *oracle.get().route(lg, k, bias))


def test_route_exact_ties():
    T, E, k = 40, 64, 8
    rng = np.random.default_rng(3)
    lg = np.round(rng.standard_normal((T, E)) * 2).astype(np.float32)   # many equal scores
    lg[5] = 0.0                                                          # all equal
    idx, w, _ = _route_gpu(T, E, k, lg, None)
    _check(idx, w, *oracle.get().route(lg, k))
    assert idx[5].tolist() == list(range(8))


@pytest.mark.parametrize("k,tile", [(8, 128), (2, 64), (3, 128), (6, 64)])
def test_route_plan_maps_exact(k, tile):
    from gpu_helpers import check_plan_exact
    cfg = si.CONFIGS["deepseek_v3"]
    T = 1500
    lg, bias = _logits(cfg, T)
    idx, w, buf = _route_gpu(T, cfg.E, k, lg, bias, fused=True, tile=tile)
    ridx, rw = oracle.get().route(lg, k, bias)
    _check(idx, w, ridx, rw)
    check_plan_exact(buf, oracle.get().plan(ridx, cfg.E, tile), T, k)
    import combine_moe_plan_03_b200 as moe
    assert moe.moe_get_status(buf.plan)[0] == 0
    buf.close()
