"""moe_pack_weights: the packed tile layout, bit for bit, against a numpy restatement of it,
and the layer with packed weights against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def pack_ref(W: np.ndarray, groups: int, group_cols: int, nb: int, kb: int) -> np.ndarray:
    """tiles [E, groups, nb, kb] of 128 rows x 64: row c*64+kr = W[e, kb*64+kr,
    g*group_cols + nb*128 + c*64 : +64], zero past group_cols."""
    E, K, _ = W.shape
    out = np.zeros((E, groups, nb, kb, 2, 64, 64), np.uint16)
    for g in range(groups):
        for n in range(nb):
            for c in range(2):
                col = n * 128 + c * 64
                if col >= group_cols:
                    continue
                blk = W[:, :, g * group_cols + col: g * group_cols + col + 64]   # [E, K, 64]
                out[:, g, n, :, c] = blk.reshape(E, kb, 64, 64)
    return out.reshape(-1)


@pytest.mark.parametrize("H,I,E", [(256, 512, 3), (192, 64, 2), (320, 192, 2), (128, 128, 1)])
def test_pack_layout_exact(H, I, E):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, bf16_host
    cfg = si.custom("pack", T=64, H=H, I=I, E=E, k=1, tile=64, seed=17 + H + I)
    W1 = si.make_w1(cfg)
    W2 = si.make_w2(cfg)
    buf = moe.MoELayerBuffers(cfg.T, H, I, E, 1, 64)
    W1p, W2p = buf.pack_weights(bf16_dev(W1), bf16_dev(W2))
    nb1, kb1 = -(-I // 128), H // 64
    nb2, kb2 = 2 * -(-H // 256), I // 64
    np.testing.assert_array_equal(bf16_host(W1p), pack_ref(W1, 2, I, nb1, kb1))
    np.testing.assert_array_equal(bf16_host(W2p), pack_ref(W2, 1, H, nb2, kb2))
    buf.close()


SHAPES = [("tiny-like", 256, 256, 512, 8, 2, 64), ("ragged", 200, 192, 64, 3, 2, 64),
          ("H320-I192", 150, 320, 192, 5, 3, 128), ("big-chunks", 700, 256, 128, 3, 2, 128)]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_layer_with_packed_weights(shape):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=99 + T)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    W1, W2 = si.make_w1(cfg), si.make_w2(cfg)
    buf = moe.MoELayerBuffers(T, H, I, E, k, tile)
    W1p, W2p = buf.pack_weights(bf16_dev(W1), bf16_dev(W2))
    for st in (0, 1):
        buf.act.view(torch.int16).fill_(0x7FC0)
        out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1p, W2p,
                          moe.moe_config(st, 0, 0, 1, 0, None))
        torch.cuda.synchronize()
        assert moe.moe_get_status(buf.plan)[0] == 0
        ref = oracle.get().moe_forward(x, idx, w, list(W1), list(W2))
        assert_layer_close(to_f64(out), ref, f"{name} streaming={st}")
    buf.close()
