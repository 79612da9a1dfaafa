"""Full-size workloads in the launch configuration the benchmark times (moe_forward on two
streams): every routing map bit-exact, outputs checked against the oracle on sampled tokens
(first, last and a seeded random set), pool padding zero, no device error."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu

N_SAMPLE = 40


def _weights(cfg):
    from gpu_helpers import DEV
    h1, h2 = si.make_w1(cfg), si.make_w2(cfg)
    W1 = torch.from_numpy(h1.view(np.int16)).to(DEV).view(torch.bfloat16)
    W2 = torch.from_numpy(h2.view(np.int16)).to(DEV).view(torch.bfloat16)
    return h1, h2, W1, W2


# (workload, streaming, packed weights, grouped-GEMM kernel: 1 one SM, 2 SM pair)
@pytest.mark.parametrize("name,streaming,packed,ffn_kernel", [
    ("qwen3_235b_a22b", 0, 0, 1), ("qwen3_235b_a22b", 1, 1, 1), ("qwen3_235b_a22b", 0, 1, 2),
    ("deepseek_v3", 0, 1, 1), ("deepseek_v3", 1, 0, 1), ("deepseek_v3", 0, 1, 2),
    ("deepseek_v3", 1, 0, 2), ("decode_microbatch", 1, 1, 1), ("decode_microbatch", 0, 1, 2)])
def test_full_layer(name, streaming, packed, ffn_kernel):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import (assert_layer_close, bf16_dev, check_plan_exact, f32_dev, i32_dev,
                             sample_tokens, to_f64)
    cfg = si.CONFIGS[name]
    h1, h2, W1, W2 = _weights(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    buf.pool.view(torch.int16).fill_(0x7FC0)
    if packed:                                   # the layout the benchmark times
        W1, W2 = buf.pack_weights(W1, W2)
    W1l = [h1[e] for e in range(cfg.E)]
    W2l = [h2[e] for e in range(cfg.E)]
    for mb in range(cfg.micro_batches):
        x = si.make_x(cfg, mb)
        idx, w = si.make_routing(cfg, mb)
        out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2,
                          moe.moe_config(streaming, 0, 0, packed, ffn_kernel, None))
        torch.cuda.synchronize()
        code, aux = moe.moe_get_status(buf.plan)
        assert code == 0, (moe.moe_strerror(code), aux)
        ref_plan = oracle.get().plan(idx, cfg.E, cfg.tile)
        check_plan_exact(buf, ref_plan, cfg.T, cfg.k)
        pad = np.nonzero(ref_plan["row_src"][: ref_plan["P"]] < 0)[0]
        if pad.size:
            sel = torch.from_numpy(pad[:: max(1, pad.size // 512)]).to(buf.pool.device)
            assert int(buf.pool[sel].view(torch.int16).abs().sum()) == 0
        tok = sample_tokens(cfg.T, N_SAMPLE, seed=mb)
        ref = oracle.get().moe_forward(x[tok], idx[tok], w[tok], W1l, W2l)
        got = to_f64(out[torch.from_numpy(tok).to(out.device)])
        assert_layer_close(got, ref, f"{name} mb{mb}")
    buf.close()


@pytest.mark.parametrize("T", [1024, 4096, 16384, 65536])
@pytest.mark.parametrize("routing", ["uniform", "zipf"])
def test_dc_sweep_identity(T, routing):
    """Dispatch/combine sweep with identity experts: out = sum_j w_j x_t, checked on every
    element against the oracle with the fp32-FMA-then-bf16 bound."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, bf16_host, check_plan_exact, f32_dev, i32_dev
    cfg = si.CONFIGS[f"dc_sweep_T{T}_{routing}"]
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, 64, cfg.E, cfg.k, cfg.tile, identity=True)
    out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), None, None)
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    check_plan_exact(buf, oracle.get().plan(idx, cfg.E, cfg.tile), cfg.T, cfg.k)
    got = si.bf16_to_f64(bf16_host(out))
    step = max(1, cfg.T // 2048)                     # every element of a strided token subset
    rows = np.arange(0, cfg.T, step)
    ref = oracle.get().moe_forward_identity(x[rows], idx[rows], w[rows])
    xf = si.bf16_to_f64(x[rows])
    aw = np.abs(w[rows].astype(np.float64)).sum(1)
    bound = 2.0 ** -8 * np.abs(ref) + cfg.k * 2.0 ** -23 * aw[:, None] * np.abs(xf) + 1e-30
    assert np.all(np.abs(got[rows] - ref) <= bound)
    buf.close()


@pytest.mark.parametrize("name,streaming", [("deepseek_v3", 0), ("deepseek_v3", 1),
                                            ("qwen3_235b_a22b", 0), ("decode_microbatch", 0)])
def test_full_layer_early_combine(name, streaming):
    """Early combine (fused into GEMM Y) at full size in the benchmark's launch configuration
    (prepacked weights): every token's output equal to the serial combine's bit for bit, and
    sampled tokens within the layer's tolerance of the oracle."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, sample_tokens, to_f64
    cfg = si.CONFIGS[name]
    h1, h2, W1, W2 = _weights(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    W1, W2 = buf.pack_weights(W1, W2)
    W1l = [h1[e] for e in range(cfg.E)]
    W2l = [h2[e] for e in range(cfg.E)]
    for mb in range(cfg.micro_batches):
        x = si.make_x(cfg, mb)
        idx, w = si.make_routing(cfg, mb)
        args = (bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2)
        serial = buf.forward(*args, moe.moe_config(streaming=streaming, packed_weights=1))
        torch.cuda.synchronize()               # out is the layer's compute stream's result
        serial = serial.clone()
        buf.out.view(torch.int16).fill_(0x7FC0)
        early = buf.forward(*args, moe.moe_config(streaming=streaming, packed_weights=1,
                                                  early_combine=1))
        torch.cuda.synchronize()
        code, aux = moe.moe_get_status(buf.plan)
        assert code == 0, (moe.moe_strerror(code), aux)
        assert torch.equal(early.view(torch.int16), serial.view(torch.int16)), f"{name} mb{mb}"
        tok = sample_tokens(cfg.T, N_SAMPLE, seed=100 + mb)
        ref = oracle.get().moe_forward(x[tok], idx[tok], w[tok], W1l, W2l)
        got = to_f64(early[torch.from_numpy(tok).to(early.device)])
        assert_layer_close(got, ref, f"{name} mb{mb} early combine")
    buf.close()
