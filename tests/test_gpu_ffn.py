"""The grouped SwiGLU FFN (tcgen05) and the whole layer vs the oracle, on small shapes that
still span several tiles, both N-block widths and a ragged tail."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def run_layer(cfg, streaming=0, mb=0, W=None, ffn_kernel=0):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    x = si.make_x(cfg, mb)
    idx, w = si.make_routing(cfg, mb)
    W1, W2 = W if W is not None else weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    for t in (buf.pool, buf.act, buf.ypool, buf.out):
        t.view(torch.int16).fill_(0x7FC0)                     # poisoned storage
    out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2,
                      moe.moe_config(streaming, 0, 0, 0, ffn_kernel))
    torch.cuda.synchronize()
    return buf, x, idx, w, W1, W2, out


def oracle_rows(cfg, x, idx, w, tokens):
    W1 = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2 = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    return oracle.get().moe_forward(x[tokens], idx[tokens], w[tokens], W1, W2)


SHAPES = [
    # name, T, H, I, E, k, tile
    ("tiny-like", 256, 256, 512, 8, 2, 64),
    ("tile128", 300, 256, 256, 4, 2, 128),
    ("I64-H192", 200, 192, 64, 3, 2, 64),       # GEMM A half width 64, GEMM Y N=64
    ("H128-I192", 150, 128, 192, 5, 3, 128),    # GEMM Y N=128, GEMM A half width 64
    ("one-expert", 130, 320, 384, 1, 1, 128),
    ("deep-K", 64, 1024, 256, 2, 2, 64),
    ("pairs-tile64", 500, 128, 128, 3, 2, 64),     # 256-row units plus 64/128/192-row tails
    ("pairs-tile128", 700, 256, 128, 3, 2, 128),   # pair units and single 128-row units
]


KERNELS = [1, 2]   # MOE_FFN_ONE_SM, MOE_FFN_SM_PAIR


@pytest.mark.parametrize("ffn_kernel", KERNELS, ids=["one_sm", "sm_pair"])
@pytest.mark.parametrize("streaming", [0, 1])
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_layer_small_shapes(shape, streaming, ffn_kernel):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, to_f64, check_plan_exact
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=1234 + T)
    buf, x, idx, w, W1, W2, out = run_layer(cfg, streaming, ffn_kernel=ffn_kernel)
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    check_plan_exact(buf, oracle.get().plan(idx, E, tile), T, k)
    ref = oracle_rows(cfg, x, idx, w, np.arange(T))
    assert_layer_close(to_f64(out), ref, name)
    buf.close()


def test_tiny_config_all_tokens_and_act():
    """The tiny config end to end, plus GEMM A's act rows against the oracle's a = silu(g)*u."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, to_f64
    cfg = si.CONFIGS["tiny"]
    buf, x, idx, w, W1, W2, out = run_layer(cfg)
    assert moe.moe_get_status(buf.plan)[0] == 0
    ref = oracle_rows(cfg, x, idx, w, np.arange(cfg.T))
    assert_layer_close(to_f64(out), ref, "tiny")
    plan = oracle.get().plan(idx, cfg.E, cfg.tile)
    act = to_f64(buf.act[: plan["P"]])
    for f in (0, 1, 77, 300, cfg.T * cfg.k - 1):
        t, j = divmod(f, cfg.k)
        e = idx[t, j]
        g, u, a, z = oracle.get().expert_ffn(x[t], si.make_w1_expert(cfg, e),
                                             si.make_w2_expert(cfg, e))
        p = plan["pool_row"][t, j]
        assert np.abs(act[p] - a).max() <= 2e-2 * np.abs(a).max()
    # every live row of act is finite (padding rows are not computed)
    live = plan["row_src"][: plan["P"]] >= 0
    assert np.isfinite(act[live]).all()
    buf.close()


def test_back_to_back_layers_reuse_flags():
    """Three layer calls in a row on the same buffers (flags reset by each plan)."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("b2b", T=384, H=256, I=256, E=6, k=2, tile=64, seed=99, micro_batches=3)
    W1, W2 = weights_dev(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    outs, ins = [], []
    for mb in range(3):
        x = si.make_x(cfg, mb)
        idx, w = si.make_routing(cfg, mb)
        ins.append((x, idx, w, bf16_dev(x), i32_dev(idx), f32_dev(w)))
    for mb in range(3):
        x, idx, w, dx, di, dw = ins[mb]
        o = buf.forward(dx, di, dw, W1, W2, moe.moe_config(1, 0, 0, 0, 0))
        with torch.cuda.stream(buf.compute):
            outs.append(o.clone())
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    for mb in range(3):
        x, idx, w = ins[mb][:3]
        ref = oracle_rows(cfg, x, idx, w, np.arange(cfg.T))
        assert_layer_close(to_f64(outs[mb]), ref, f"mb{mb}")
    buf.close()


@pytest.mark.parametrize("ffn_kernel", KERNELS, ids=["one_sm", "sm_pair"])
def test_act_every_live_row_within_one_bf16_ulp(ffn_kernel):
    """GEMM A's SwiGLU output (act) on every live pool row against the oracle's
    a = silu(g) * u in fp64, element by element: at most one bf16 ulp apart (the GPU's fp32
    sums and its exponential / reciprocal move a by about 1e-5 relative before the final
    rounding; near a = 0 the bound adds 1e-5 of the row's largest |a|). W1 is scaled by 4 (exact in bf16) so that g spans about [-16, 16]."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, to_f64
    cfg = si.custom("actulp", T=256, H=256, I=512, E=8, k=2, tile=64, seed=4242)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    # x4 only moves the exponent: the bf16 -> float32 -> bf16 round trip is exact
    w1_bits = [torch.from_numpy(si.bf16_to_f64(si.make_w1_expert(cfg, e)).astype(np.float32) * 4)
               .to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
               for e in range(cfg.E)]
    w2_bits = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    W1 = bf16_dev(np.stack(w1_bits))
    W2 = bf16_dev(np.stack(w2_bits))
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2,
                moe.moe_config(0, 0, 0, 0, ffn_kernel))
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0
    plan = oracle.get().plan(idx, cfg.E, cfg.tile)
    act = to_f64(buf.act[: plan["P"]])
    gmax = 0.0
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = idx[t, j]
            g, u, a, _ = oracle.get().expert_ffn(x[t], w1_bits[e], w2_bits[e])
            gmax = max(gmax, float(np.abs(g).max()))
            got = act[plan["pool_row"][t, j]]
            # one bf16 ulp of a, plus the fp32 summation error of g and u (~1e-7 of the
            # row's scale) where a itself is near zero
            bound = 2.0 ** -7 * np.abs(a) + 1e-5 * np.abs(a).max()
            assert np.all(np.abs(got - a) <= bound), (t, j, float((np.abs(got - a) / bound).max()))
    assert gmax > 10.0                      # the scaled weights reach the tails of silu
    buf.close()


@pytest.mark.parametrize("ffn_ctas", [2, 3, 6], ids=["1cluster", "odd3", "3clusters"])
def test_pair_kernel_few_clusters_many_units(ffn_ctas):
    """The SM-pair kernel with 1 or 3 clusters (an odd CTA count rounds down to whole pairs):
    every cluster runs many units in a row through the ticket ring, and the ticket
    counters reset themselves for the next launch (two layer calls on the same plan)."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("fewcl", T=700, H=256, I=384, E=5, k=2, tile=128, seed=777)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    c = moe.moe_config(0, ffn_ctas, 0, 0, moe.MOE_FFN_SM_PAIR)
    ref = oracle_rows(cfg, x, idx, w, np.arange(cfg.T))
    for call in range(2):
        out = buf.forward(bf16_dev(x), i32_dev(idx), f32_dev(w), W1, W2, c)
        torch.cuda.synchronize()
        code, aux = moe.moe_get_status(buf.plan)
        assert code == 0, (moe.moe_strerror(code), aux)
        assert_layer_close(to_f64(out), ref, f"fewcl call{call}")
        # both GEMMs' ticket / done counters are back to zero after each launch
        meta = buf.plan_view("meta").cpu().numpy()
        assert (meta[4:8] == 0).all(), meta
    buf.close()
