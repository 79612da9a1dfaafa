"""Backward of the layer's activation path (moe_backward: combine backward, gate / up
recompute, backward Y with the SwiGLU backward, backward A, dispatch backward) against the
oracle's fp64 gradients: dx on every token of small shapes that span several tiles and
ragged chunks, and on sampled tokens of the full DeepSeek-V3-shaped layer; dw likewise."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu

TOL = 2e-2   # max |err| <= TOL * max |ref|, as for the forward


def _close(got, ref, what):
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= TOL * scale, f"{what}: max err {err:.3e} vs {TOL} * {scale:.3e}"


def _run(cfg, W1, W2, x, idx, w, dy, weight_grads=False):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    dw_dev = f32_dev(w)
    buf.forward(bf16_dev(x), i32_dev(idx), dw_dev, W1, W2)
    gW = None
    if weight_grads:
        gW = (torch.full((cfg.E, cfg.H, 2 * cfg.I), float("nan"), dtype=torch.bfloat16,
                         device=W1.device),
              torch.full((cfg.E, cfg.I, cfg.H), float("nan"), dtype=torch.bfloat16,
                         device=W1.device))
    torch.cuda.synchronize()   # the fills (default stream) before the backward (compute stream)
    dx, dwg = buf.backward(bf16_dev(dy), dw_dev, W1, W2, dW1=gW[0] if gW else None,
                           dW2=gW[1] if gW else None)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    if weight_grads:
        return buf, dx, dwg, gW
    return buf, dx, dwg


SHAPES = [
    # name, T, H, I, E, k, tile
    ("tiny-like", 256, 256, 512, 8, 2, 64),
    ("tile128-ragged", 300, 256, 256, 4, 2, 128),
    ("I64-H192", 200, 192, 64, 3, 2, 64),
    ("H640-I384", 150, 640, 384, 5, 3, 128),
    ("pairs-tile64", 500, 128, 128, 3, 2, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_backward_small_shapes_all_tokens(shape):
    from gpu_helpers import to_f64, weights_dev
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=4321 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    idx[3, 0] = -1                                   # a dropped pair
    dy = si.make_dy(cfg)
    buf, dx, dw = _run(cfg, W1, W2, x, idx, w, dy)
    W1l = [si.make_w1_expert(cfg, e) for e in range(E)]
    W2l = [si.make_w2_expert(cfg, e) for e in range(E)]
    rdx, rdw = oracle.get().moe_backward(x, idx, w, W1l, W2l, dy)
    _close(to_f64(dx), rdx, f"{name} dx")
    _close(dw.cpu().numpy().astype(np.float64), rdw, f"{name} dw")
    assert float(dw[3, 0]) == 0.0
    buf.close()


def test_backward_full_deepseek_sampled_tokens():
    """The DeepSeek-V3-shaped layer at full size: dx and dw on 24 sampled tokens."""
    from gpu_helpers import sample_tokens, to_f64
    from test_gpu_full import _weights
    cfg = si.CONFIGS["deepseek_v3"]
    h1, h2, W1, W2 = _weights(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    dy = si.make_dy(cfg)
    buf, dx, dw = _run(cfg, W1, W2, x, idx, w, dy)
    tok = sample_tokens(cfg.T, 24, seed=5)
    rdx, rdw = oracle.get().moe_backward(x[tok], idx[tok], w[tok], [h1[e] for e in range(cfg.E)],
                                         [h2[e] for e in range(cfg.E)], dy[tok])
    sel = torch.from_numpy(tok).to(dx.device)
    _close(to_f64(dx[sel]), rdx, "deepseek dx")
    _close(dw[sel].cpu().numpy().astype(np.float64), rdw, "deepseek dw")
    buf.close()


@pytest.mark.parametrize("shape", SHAPES[:3], ids=[s[0] for s in SHAPES[:3]])
def test_forward_saving_gate_up_then_backward(shape):
    """A training step: forward with save_for_backward (GEMM A also stores g | u and makes
    act from them), then the backward without the recompute. The forward output, the saved
    g and u, dx and dw all against the oracle."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=999 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    dy = si.make_dy(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    wd = f32_dev(w)
    out = buf.forward(bf16_dev(x), i32_dev(idx), wd, W1, W2, save_for_backward=True)
    dx, dw = buf.backward(bf16_dev(dy), wd, W1, W2)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    W1l = [si.make_w1_expert(cfg, e) for e in range(E)]
    W2l = [si.make_w2_expert(cfg, e) for e in range(E)]
    ref = oracle.get().moe_forward(x, idx, w, W1l, W2l)
    assert_layer_close(to_f64(out), ref, f"{name} forward")
    plan = oracle.get().plan(idx, E, tile)
    gu = to_f64(buf.gu[: plan["P"]])
    for f in (0, 7, T * k - 1):
        t, j = divmod(f, k)
        if idx[t, j] < 0:
            continue
        g, u, _, _ = oracle.get().expert_ffn(x[t], W1l[idx[t, j]], W2l[idx[t, j]])
        row = gu[plan["pool_row"][t, j]]
        for got, want in ((row[:I], g), (row[I:], u)):
            assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-5 * np.abs(want).max())
    rdx, rdw = oracle.get().moe_backward(x, idx, w, W1l, W2l, dy)
    _close(to_f64(dx), rdx, f"{name} dx")
    _close(dw.cpu().numpy().astype(np.float64), rdw, f"{name} dw")
    buf.close()


EDGE = [
    # name, T, H, I, E, k, tile, drop (fraction of pairs set to -1)
    ("k16", 64, 128, 128, 32, 16, 64, 0.0),         # two groups of 8 pairs per token
    ("E1-k1", 100, 128, 192, 1, 1, 128, 0.0),       # one expert: a dense SwiGLU FFN
    ("half-dropped", 90, 128, 128, 4, 2, 64, 0.5),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_backward_edge_cases(case):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import to_f64, weights_dev
    name, T, H, I, E, k, tile, drop = case
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=2024 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    if drop:
        rng = np.random.default_rng(7)
        idx[rng.random(idx.shape) < drop] = -1
    dy = si.make_dy(cfg)
    buf, dx, dw = _run(cfg, W1, W2, x, idx, w, dy)
    W1l = [si.make_w1_expert(cfg, e) for e in range(E)]
    W2l = [si.make_w2_expert(cfg, e) for e in range(E)]
    rdx, rdw = oracle.get().moe_backward(x, idx, w, W1l, W2l, dy)
    _close(to_f64(dx), rdx, f"{name} dx")
    _close(dw.cpu().numpy().astype(np.float64), rdw, f"{name} dw")
    assert np.all(dw.cpu().numpy()[idx < 0] == 0.0)
    buf.close()


def test_backward_no_live_pairs_and_no_tokens():
    """Every pair dropped: dx = 0 and dw = 0 with no device error. T = 0: no rows, so the
    weight gradients are exactly zero."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import bf16_dev, f32_dev, i32_dev, weights_dev
    cfg = si.custom("alldrop", T=40, H=128, I=128, E=4, k=2, tile=64, seed=5)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    idx[:] = -1
    buf, dx, dw = _run(cfg, W1, W2, x, idx, w, si.make_dy(cfg))
    assert not dx.float().abs().sum().item() and not dw.abs().sum().item()
    buf.close()
    buf = moe.MoELayerBuffers(0, 128, 128, 4, 2, 64)
    e = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    ei = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    ew = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    buf.forward(e, ei, ew, W1, W2)
    gW1 = torch.full((4, 128, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    gW2 = torch.full((4, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()   # the fills (default stream) before the backward (compute stream)
    dx, dw = buf.backward(e, ew, W1, W2, dW1=gW1, dW2=gW2)
    torch.cuda.synchronize()
    assert moe.moe_get_status(buf.plan)[0] == 0 and dx.numel() == 0 and dw.numel() == 0
    assert not gW1.float().abs().sum().item() and not gW2.float().abs().sum().item()
    buf.close()


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_weight_gradients_small_shapes_every_expert(shape):
    """dW1 and dW2 of every expert against the oracle (expert 0 is left without rows, so its
    gradients must be exactly zero); dx and dw of the same call too."""
    from gpu_helpers import to_f64, weights_dev
    name, T, H, I, E, k, tile = shape
    cfg = si.custom(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=777 + T)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    if E > k:
        idx[idx == 0] = -1                           # expert 0 gets no rows
    dy = si.make_dy(cfg)
    buf, dx, dw, (gW1, gW2) = _run(cfg, W1, W2, x, idx, w, dy, weight_grads=True)
    W1l = [si.make_w1_expert(cfg, e) for e in range(E)]
    W2l = [si.make_w2_expert(cfg, e) for e in range(E)]
    for e in range(E):
        r1, r2 = oracle.get().expert_weight_grads(x, idx, w, W1l[e], W2l[e], e, dy)
        g1, g2 = to_f64(gW1[e]), to_f64(gW2[e])
        if not (idx == e).any():
            assert not np.any(g1) and not np.any(g2), f"{name} expert {e} without rows"
            continue
        _close(g1, r1, f"{name} dW1[{e}]")
        _close(g2, r2, f"{name} dW2[{e}]")
    rdx, rdw = oracle.get().moe_backward(x, idx, w, W1l, W2l, dy)
    _close(to_f64(dx), rdx, f"{name} dx")
    _close(dw.cpu().numpy().astype(np.float64), rdw, f"{name} dw")
    buf.close()


def test_weight_gradients_every_row_residue():
    """Experts whose row counts fall in every residue class of the weight-gradient K loop
    (steps of 64 rows, MMAs of 16): 1, 15, 16, 17, 31, ..., 129 rows, one expert each, and
    one expert without rows; dW1 and dW2 of each against the oracle."""
    from gpu_helpers import to_f64, weights_dev
    counts = [1, 15, 16, 17, 31, 32, 33, 47, 48, 49, 63, 64, 65, 80, 127, 128, 129, 0]
    E, T = len(counts), sum(counts)
    cfg = si.custom("row-residues", T=T, H=256, I=128, E=E, k=1, tile=64, seed=4242)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    _, w = si.make_routing(cfg)
    order = np.random.default_rng(4242).permutation(T)
    idx = np.repeat(np.arange(E, dtype=np.int32), counts)[order].reshape(T, 1)
    dy = si.make_dy(cfg)
    buf, dx, dw, (gW1, gW2) = _run(cfg, W1, W2, x, idx, w, dy, weight_grads=True)
    for e in range(E):
        g1, g2 = to_f64(gW1[e]), to_f64(gW2[e])
        if counts[e] == 0:
            assert not np.any(g1) and not np.any(g2), f"expert {e} without rows"
            continue
        r1, r2 = oracle.get().expert_weight_grads(x, idx, w, si.make_w1_expert(cfg, e),
                                                  si.make_w2_expert(cfg, e), e, dy)
        _close(g1, r1, f"dW1[{e}] ({counts[e]} rows)")
        _close(g2, r2, f"dW2[{e}] ({counts[e]} rows)")
    buf.close()


def _oracle_weight_grads_threaded(x, idx, w, W1e, W2e, e, dy, threads=8):
    """The oracle's weight gradients of expert e, with the expert's tokens split into
    `threads` contiguous slices computed at once (the oracle releases the GIL) and the
    slices' sums added: the same products, summed in fp64 in slices."""
    import concurrent.futures as cf
    tok = np.nonzero((idx == e).any(1))[0]
    parts = [p for p in np.array_split(tok, threads) if p.size]
    orc = oracle.get()

    def one(p):
        return orc.expert_weight_grads(x[p], idx[p], w[p], W1e, W2e, e, dy[p])
    with cf.ThreadPoolExecutor(len(parts)) as ex:
        res = list(ex.map(one, parts))
    return sum(r[0] for r in res), sum(r[1] for r in res)


def test_weight_gradients_full_deepseek_two_experts():
    """The DeepSeek-V3-shaped layer at full size: dW1 and dW2 of the two experts with the
    fewest (non-zero) rows and of the expert with the most rows (the longest fp32
    accumulation, up to ~2,400 rows), element by element against the oracle."""
    from gpu_helpers import to_f64
    from test_gpu_full import _weights
    cfg = si.CONFIGS["deepseek_v3"]
    h1, h2, W1, W2 = _weights(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    dy = si.make_dy(cfg)
    buf, dx, dw, (gW1, gW2) = _run(cfg, W1, W2, x, idx, w, dy, weight_grads=True)
    cnt = np.bincount(idx[idx >= 0].reshape(-1), minlength=cfg.E)
    order = [int(e) for e in np.argsort(cnt, kind="stable") if cnt[e] > 0]
    for e in order[:2] + order[-1:]:
        r1, r2 = _oracle_weight_grads_threaded(x, idx, w, h1[e], h2[e], e, dy)
        _close(to_f64(gW1[e]), r1, f"deepseek dW1[{e}] ({cnt[e]} rows)")
        _close(to_f64(gW2[e]), r2, f"deepseek dW2[{e}] ({cnt[e]} rows)")
    assert cnt[order[-1]] > 1000                  # the most-loaded expert: a long K loop
    buf.close()


def test_packed_forward_saving_gate_up_then_backward():
    """The training step as the benchmark runs it: the forward with prepacked weights keeping
    g | u, the backward reading the weights in their given layout; output, saved g / u and
    gradients against the oracle."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import assert_layer_close, bf16_dev, f32_dev, i32_dev, to_f64, weights_dev
    cfg = si.custom("packed-train", T=300, H=256, I=384, E=4, k=2, tile=128, seed=31337)
    W1, W2 = weights_dev(cfg)
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    dy = si.make_dy(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile)
    W1p, W2p = buf.pack_weights(W1, W2)
    wd = f32_dev(w)
    out = buf.forward(bf16_dev(x), i32_dev(idx), wd, W1p, W2p, moe.moe_config(packed_weights=1),
                      save_for_backward=True)
    gW1 = torch.empty((cfg.E, cfg.H, 2 * cfg.I), dtype=torch.bfloat16, device=W1.device)
    gW2 = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=W1.device)
    dx, dw = buf.backward(bf16_dev(dy), wd, W1, W2, dW1=gW1, dW2=gW2)
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    assert code == 0, (moe.moe_strerror(code), aux)
    W1l = [si.make_w1_expert(cfg, e) for e in range(cfg.E)]
    W2l = [si.make_w2_expert(cfg, e) for e in range(cfg.E)]
    assert_layer_close(to_f64(out), oracle.get().moe_forward(x, idx, w, W1l, W2l), "packed forward")
    rdx, rdw = oracle.get().moe_backward(x, idx, w, W1l, W2l, dy)
    _close(to_f64(dx), rdx, "packed dx")
    _close(dw.cpu().numpy().astype(np.float64), rdw, "packed dw")
    for e in range(cfg.E):
        r1, r2 = oracle.get().expert_weight_grads(x, idx, w, W1l[e], W2l[e], e, dy)
        _close(to_f64(gW1[e]), r1, f"packed dW1[{e}]")
        _close(to_f64(gW2[e]), r2, f"packed dW2[{e}]")
    buf.close()
