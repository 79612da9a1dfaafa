"""The backward's mirrored overlaps (StreamEP README, How it works, "Per-tile streaming": the
backward pass mirrors both of the forward's overlaps). Early dispatch backward: with
moe_config.early_combine = 1, backward A's CTAs sum each token's k dpool rows as soon as they
are stored (the dispatch backward folded in, as early combine folds the combine into GEMM
Y). Every output must equal the serial backward's bit for bit (the same fp32 sum in j order),
and stay within the layer's tolerance of the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu

SHAPES = [
    # name, T, H, I, E, k, tile, dropped fraction
    ("tiny-like", 256, 256, 512, 8, 2, 64, 0.0),
    ("ragged-H", 300, 320, 256, 4, 2, 128, 0.1),      # backward A's 512-column block half empty
    ("wide-H", 150, 1088, 128, 5, 3, 64, 0.1),        # three column blocks, the last ragged
    ("k8", 96, 512, 256, 16, 8, 64, 0.2),
    ("half-dropped", 90, 128, 128, 4, 2, 64, 0.5),
    ("E1-k1", 100, 128, 192, 1, 1, 128, 0.0),         # one expert, one pair per token
    ("k16", 64, 128, 128, 32, 16, 64, 0.1),           # two groups of 8 pairs per token
]


def _backward(cfg, W1, W2, x, idx, w, dy, early, weight_grads=True):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    dw_dev = f32_dev(w)
    buf.forward(bf16_dev(x), i32_dev(idx), dw_dev, W1, W2, save_for_backward=True)
    gW = None
    if weight_grads:
        gW = (torch.full((cfg.E, cfg.H, 2 * cfg.I), float("nan"), dtype=torch.bfloat16,
                         device=W1.device),
              torch.full((cfg.E, cfg.I, cfg.H), float("nan"), dtype=torch.bfloat16,
                         device=W1.device))
    dx = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device=W1.device)
    # the poisoned outputs are filled on the default stream; the backward runs on the
    # layer's compute stream: the fills must be done before it writes
    torch.cuda.synchronize()
    dx, dwg = buf.backward(bf16_dev(dy), dw_dev, W1, W2, moe.moe_config(early_combine=early),
                           dx=dx, dW1=gW[0] if gW else None, dW2=gW[1] if gW else None)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    out = (dx.clone(), dwg.clone()) + ((gW[0].clone(), gW[1].clone()) if gW else ())
    buf.close()
    return out


def _same(a, b, what):
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    assert torch.equal(a, b), what


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_early_dispatch_backward_equals_serial_and_oracle(shape):
    from gpu_helpers import to_f64, weights_dev
    name, T, H, I, E, k, tile, drop = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=777 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    if drop > 0:
        idx = idx.copy()
        idx[np.random.default_rng(3).random(idx.shape) < drop] = -1
        idx[:2] = -1                                  # tokens without a live pair: dx = 0
    dy = si.make_dy(cfg)
    serial = _backward(cfg, W1, W2, x, idx, w, dy, early=0)
    early = _backward(cfg, W1, W2, x, idx, w, dy, early=1)
    for a, b, what in zip(early, serial, ("dx", "dw", "dW1", "dW2")):
        _same(a, b, f"{name} {what}")
    rdx, rdw = oracle.get().moe_backward(x, idx, w, [si.make_w1_expert(cfg, e) for e in range(E)],
                                         [si.make_w2_expert(cfg, e) for e in range(E)], dy)
    scale = np.abs(rdx).max()
    assert np.abs(to_f64(early[0]) - rdx).max() <= 2e-2 * scale
    if drop > 0:
        assert not to_f64(early[0])[:2].any()


def test_early_dispatch_backward_full_deepseek():
    """The DeepSeek-V3-shaped layer at full size: the early dispatch backward's dx equals the
    serial one bit for bit (every token)."""
    from test_gpu_full import _weights
    cfg = si.CONFIGS["deepseek_v3"]
    _, _, W1, W2 = _weights(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    dy = si.make_dy(cfg)
    serial = _backward(cfg, W1, W2, x, idx, w, dy, early=0, weight_grads=False)
    early = _backward(cfg, W1, W2, x, idx, w, dy, early=1, weight_grads=False)
    _same(early[0], serial[0], "dx")
    _same(early[1], serial[1], "dw")


@pytest.mark.parametrize("shape", SHAPES[:4], ids=[s[0] for s in SHAPES[:4]])
@pytest.mark.parametrize("early", [0, 1])
def test_streaming_backward_equals_serial(shape, early):
    """The streaming backward (moe_backward_streams): the combine backward in pool-tile order
    on the communicate stream raising tile flags, backward Y taking tiles on the compute
    stream; every output bit-identical to the serial backward's (dw of dropped pairs 0)."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import weights_dev
    name, T, H, I, E, k, tile, drop = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=991 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    if drop > 0:
        idx = idx.copy()
        idx[np.random.default_rng(4).random(idx.shape) < drop] = -1
    dy = si.make_dy(cfg)
    serial = _backward(cfg, W1, W2, x, idx, w, dy, early=0)
    got = _backward_cfg(cfg, W1, W2, x, idx, w, dy, moe.moe_config(streaming=1, early_combine=early))
    for a, b, what in zip(got, serial, ("dx", "dw", "dW1", "dW2")):
        _same(a, b, f"{name} {what}")


def _backward_cfg(cfg, W1, W2, x, idx, w, dy, mcfg):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    dw_dev = f32_dev(w)
    buf.forward(bf16_dev(x), i32_dev(idx), dw_dev, W1, W2, save_for_backward=True)
    gW = (torch.full((cfg.E, cfg.H, 2 * cfg.I), float("nan"), dtype=torch.bfloat16,
                     device=W1.device),
          torch.full((cfg.E, cfg.I, cfg.H), float("nan"), dtype=torch.bfloat16, device=W1.device))
    dw_out = torch.full((cfg.T, cfg.k), float("nan"), dtype=torch.float32, device=W1.device)
    torch.cuda.synchronize()   # fills (default stream) before the backward (compute stream)
    dx, dwg = buf.backward(bf16_dev(dy), dw_dev, W1, W2, mcfg, dw=dw_out, dW1=gW[0], dW2=gW[1])
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    out = (dx.clone(), dwg.clone(), gW[0].clone(), gW[1].clone())
    buf.close()
    return out

