"""The whole layer captured once in a CUDA graph (plan and dispatch on the communicate
stream, FFN and combine on the compute stream, no host sync inside) and replayed with new
inputs copied into the captured buffers: every replay's routing maps are exact and its
output is within the layer's bound. Storage is reused across replays."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def test_graph_capture_and_replay_with_changing_routing():
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("graph", T=192, H=256, I=256, E=6, k=2, tile=64, seed=4242, micro_batches=4)
    W1, W2 = weights_dev(cfg)
    W1h = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2h = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    inputs = []
    for mb in range(cfg.micro_batches):
        x = si.make_x(cfg, mb)
        idx, w = si.make_routing(cfg, mb)
        if mb == 3:
            idx[::5, 1] = -1                       # dropped pairs in one of the batches
        inputs.append((x, idx, w, oracle.get().moe_forward(x, idx, w, W1h, W2h),
                       oracle.get().plan(idx, cfg.E, cfg.tile)))
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    dx = bf16_dev(inputs[0][0])
    didx = i32_dev(inputs[0][1])
    dw = f32_dev(inputs[0][2])
    buf.forward(dx, didx, dw, W1, W2)             # eager call first (one-time set-up)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        fork = torch.cuda.Event()
        fork.record(cap)
        buf.comm.wait_event(fork)
        buf.compute.wait_event(fork)
        out = buf.forward(dx, didx, dw, W1, W2)
        j1, j2 = torch.cuda.Event(), torch.cuda.Event()
        j1.record(buf.compute)
        j2.record(buf.comm)
        cap.wait_event(j1)
        cap.wait_event(j2)
    torch.cuda.synchronize()

    for it in range(20):
        x, idx, w, ref, ref_plan = inputs[(it * 3 + 1) % cfg.micro_batches]
        dx.copy_(bf16_dev(x))
        didx.copy_(i32_dev(idx))
        dw.copy_(f32_dev(w))
        out.view(torch.int16).fill_(0x7FC0)       # poison the output between replays
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_status(buf.plan)[0] == 0
        np.testing.assert_array_equal(buf.plan_view("pool_row")[: cfg.T * cfg.k].cpu().numpy(),
                                      ref_plan["pool_row"].reshape(-1))
        assert_layer_close(to_f64(out), ref, f"replay {it}")
    del g
    buf.close()
