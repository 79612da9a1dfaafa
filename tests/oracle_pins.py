"""Pins that tie the CPU oracle to something other than itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with: a hand-worked example (tests/golden), a brute force written a
different way (stable sort; dense all-experts einsum), a library routine on a
textbook special case (torch float64 matmuls), a closed form, or an invariant.
``test_oracle_pins`` runs them on the real oracle; ``test_oracle_mutants`` builds
copies of the oracle with planted mistakes and checks that some pin fails.
"""
from __future__ import annotations

import json
import os

import numpy as np

import synth_inputs as si

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def bf16(a) -> np.ndarray:
    return si.f32_to_bf16_bits(np.asarray(a, np.float32))


def f64(b) -> np.ndarray:
    return si.bf16_to_f64(np.asarray(b, np.uint16))


def silu_np(v):
    return v / (1.0 + np.exp(-v))


# ---------------------------------------------------------------- plan ----------------

def pin_plan_worked(orc):
    cases = json.load(open(os.path.join(GOLDEN, "worked_plan.json")))["cases"]
    for c in cases:
        idx = np.array(c["topk_idx"], np.int32)
        r = orc.plan(idx, c["E"], c["tile"])
        assert r["P"] == c["P"], c["name"]
        assert r["P_max"] == c["P_max"], c["name"]
        np.testing.assert_array_equal(r["counts"], c["counts"])
        np.testing.assert_array_equal(r["offsets"], c["offsets"])
        np.testing.assert_array_equal(r["pool_row"], np.array(c["pool_row"]))
        np.testing.assert_array_equal(r["row_src"], c["row_src"])
        np.testing.assert_array_equal(r["tile_expert"], c["tile_expert"])


def plan_bruteforce(idx: np.ndarray, E: int, tile: int):
    """Stable sort of the flat pair ids by expert, then pad each expert's run to the tile."""
    flat = idx.reshape(-1)
    live = [f for f in range(flat.size) if flat[f] >= 0]
    order = sorted(live, key=lambda f: flat[f])          # Python's sort is stable
    pool_row = -np.ones(flat.size, np.int64)
    row = 0
    counts = np.zeros(E, np.int64)
    offsets = [0]
    pos = 0
    for e in range(E):
        run = [f for f in order[pos:] if flat[f] == e]
        pos += len(run)
        counts[e] = len(run)
        for i, f in enumerate(run):
            pool_row[f] = row + i
        row += -(-len(run) // tile) * tile
        offsets.append(row)
    return counts, np.array(offsets), pool_row.reshape(idx.shape), row


def pin_plan_bruteforce(orc):
    rng = _rng(1)
    for (T, k, E, tile) in [(1, 1, 1, 4), (7, 2, 3, 4), (33, 3, 5, 8), (64, 8, 16, 16),
                            (100, 4, 40, 64), (5, 6, 9, 128)]:
        idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
        r = orc.plan(idx, E, tile)
        counts, offsets, pool_row, P = plan_bruteforce(idx, E, tile)
        np.testing.assert_array_equal(r["counts"], counts)
        np.testing.assert_array_equal(r["offsets"], offsets)
        np.testing.assert_array_equal(r["pool_row"], pool_row)
        assert r["P"] == P


def check_plan_invariants(r, idx: np.ndarray, E: int, tile: int):
    flat = idx.reshape(-1)
    live = flat >= 0
    assert int(r["counts"].sum()) == int(live.sum())
    assert np.all(r["offsets"] % tile == 0)
    assert np.all(np.diff(r["offsets"]) >= r["counts"])
    assert np.all(np.diff(r["offsets"]) - r["counts"] < tile)
    assert r["P"] == r["offsets"][-1] <= r["P_max"]
    pr = r["pool_row"].reshape(-1)
    assert np.all(pr[~live] == -1)
    rows = pr[live]
    assert len(np.unique(rows)) == rows.size                    # injective
    rs = r["row_src"]
    assert np.all(rs[rows] == np.nonzero(live)[0])               # inverse map
    assert int((rs >= 0).sum()) == rows.size                     # the rest is padding
    for e in range(E):                                           # expert-major, stable
        fs = np.nonzero(flat == e)[0]
        pe = pr[fs]
        assert np.all(pe >= r["offsets"][e]) and np.all(pe < r["offsets"][e + 1])
        assert np.all(np.diff(pe) == 1)
        if fs.size:
            assert pe[0] == r["offsets"][e]
    te = r["tile_expert"]
    for e in range(E):
        a, b = r["offsets"][e] // tile, r["offsets"][e + 1] // tile
        assert np.all(te[a:b] == e)
    assert np.all(te[r["P"] // tile:] == -1)


def pin_plan_invariants(orc):
    rng = _rng(2)
    for (T, k, E, tile) in [(300, 2, 8, 64), (1000, 8, 256, 128), (17, 8, 256, 128)]:
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        idx[rng.random(idx.shape) < 0.05] = -1
        r = orc.plan(idx, E, tile)
        check_plan_invariants(r, idx, E, tile)


def pin_plan_bad_index(orc):
    import oracle
    for bad in (-2, 8, 1 << 20):
        idx = np.zeros((4, 2), np.int32)
        idx[2, 1] = bad
        try:
            orc.plan(idx, 8, 64)
        except oracle.OracleError as e:
            assert e.code == oracle.ERR_BAD_INDEX
        else:
            raise AssertionError("bad index accepted")


# ---------------------------------------------------------------- pool ----------------

def pin_pool_gather(orc):
    rng = _rng(3)
    T, k, E, tile, H = 50, 3, 6, 8, 24
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    x = rng.integers(0, 1 << 16, size=(T, H)).astype(np.uint16)
    r = orc.plan(idx, E, tile)
    pool = orc.pool(r["row_src"], r["P"], x, k)
    expect = np.zeros((r["P"], H), np.uint16)
    for t in range(T):
        for j in range(k):
            if idx[t, j] >= 0:
                expect[r["pool_row"][t, j]] = x[t]
    np.testing.assert_array_equal(pool, expect)
    pad = r["row_src"][: r["P"]] < 0
    assert np.all(pool[pad] == 0)


# ---------------------------------------------------------------- FFN ------------------

def pin_ffn_worked(orc):
    c = json.load(open(os.path.join(GOLDEN, "worked_ffn.json")))
    x = bf16(c["x"])
    W1 = [bf16(w) for w in c["W1"]]
    W2 = [bf16(w) for w in c["W2"]]
    idx = np.array(c["topk_idx"], np.int32)
    w = np.array(c["topk_w"], np.float32)
    _, _, _, z00 = orc.expert_ffn(x[0], W1[0], W2[0])
    _, _, _, z01 = orc.expert_ffn(x[0], W1[1], W2[1])
    np.testing.assert_allclose(z00, c["z_token0_expert0"], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(z01, c["z_token0_expert1"], rtol=1e-14, atol=1e-15)
    y = orc.moe_forward(x, idx, w, W1, W2, n_threads=1)
    np.testing.assert_allclose(y, c["y"], rtol=1e-14, atol=1e-15)


def _rand_layer(rng, T, H, I, E, k, drop=0.0):
    x = bf16(rng.standard_normal((T, H)))
    W1 = bf16(rng.standard_normal((E, H, 2 * I)) / np.sqrt(H))
    W2 = bf16(rng.standard_normal((E, I, H)) / np.sqrt(I))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx[rng.random(idx.shape) < drop] = -1
    w = rng.random((T, k)).astype(np.float32)
    return x, W1, W2, idx, w


def dense_bruteforce(x, W1, W2, idx, w):
    """Every token through every expert (einsum), masked by a dense [T, E] routing matrix."""
    xf, W1f, W2f = f64(x), f64(W1), f64(W2)
    T, E = x.shape[0], W1.shape[0]
    I = W2.shape[1]
    R = np.zeros((T, E))
    for t in range(T):
        for j in range(idx.shape[1]):
            if idx[t, j] >= 0:
                R[t, idx[t, j]] += float(w[t, j])
    gate = np.einsum("th,ehn->ten", xf, W1f[:, :, :I])
    up = np.einsum("th,ehn->ten", xf, W1f[:, :, I:])
    Z = np.einsum("ten,enm->tem", silu_np(gate) * up, W2f)
    return np.einsum("te,tem->tm", R, Z)


def pin_ffn_dense_bruteforce(orc):
    rng = _rng(4)
    for (T, H, I, E, k, drop) in [(16, 64, 64, 4, 2, 0.1), (5, 16, 8, 3, 3, 0.0),
                                  (9, 32, 48, 4, 1, 0.0), (3, 8, 16, 2, 2, 0.3)]:
        x, W1, W2, idx, w = _rand_layer(rng, T, H, I, E, k, drop)
        y = orc.moe_forward(x, idx, w, list(W1), list(W2), n_threads=2)
        ref = dense_bruteforce(x, W1, W2, idx, w)
        np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def pin_ffn_textbook_torch(orc):
    """E=1, k=1, w=1: a plain dense SwiGLU FFN, computed with torch float64 matmuls."""
    import torch
    rng = _rng(5)
    T, H, I = 12, 40, 24
    x, W1, W2, _, _ = _rand_layer(rng, T, H, I, 1, 1)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    y = orc.moe_forward(x, idx, w, [W1[0]], [W2[0]], n_threads=1)
    X = torch.from_numpy(f64(x))
    Wg = torch.from_numpy(f64(W1[0][:, :I]))
    Wu = torch.from_numpy(f64(W1[0][:, I:]))
    Wd = torch.from_numpy(f64(W2[0]))
    ref = (torch.nn.functional.silu(X @ Wg) * (X @ Wu)) @ Wd
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)


def pin_ffn_closed_form(orc):
    """H = I, W1 = [alpha*Id | beta*Id], W2 = Id: y[t] = w * silu(alpha x) * (beta x) elementwise."""
    rng = _rng(6)
    T, H = 10, 16
    alpha, beta = 0.5, -2.0
    x = bf16(rng.standard_normal((T, H)))
    Id = np.eye(H)
    W1 = bf16(np.concatenate([alpha * Id, beta * Id], axis=1))[None]
    W2 = bf16(Id)[None]
    idx = np.zeros((T, 1), np.int32)
    w = rng.random((T, 1)).astype(np.float32)
    y = orc.moe_forward(x, idx, w, [W1[0]], [W2[0]], n_threads=1)
    xf = f64(x)
    expect = w.astype(np.float64) * silu_np(alpha * xf) * (beta * xf)
    np.testing.assert_allclose(y, expect, rtol=1e-14, atol=1e-300)


def pin_ffn_linearity(orc):
    rng = _rng(7)
    x, W1, W2, idx, w = _rand_layer(rng, 6, 32, 16, 3, 2)
    y1 = orc.moe_forward(x, idx, w, list(W1), list(W2), n_threads=1)
    y2 = orc.moe_forward(x, idx, 2 * w, list(W1), list(W2), n_threads=1)
    np.testing.assert_array_equal(y2, 2 * y1)                  # scaling by 2 is exact
    y0 = orc.moe_forward(x, idx, w, list(W1), list(np.zeros_like(W2)), n_threads=1)
    assert np.all(y0 == 0)
    yz = orc.moe_forward(x, idx, np.zeros_like(w), list(W1), list(W2), n_threads=1)
    assert np.all(yz == 0)


def pin_ffn_permutation(orc):
    rng = _rng(8)
    x, W1, W2, idx, w = _rand_layer(rng, 9, 16, 16, 4, 2)
    perm = rng.permutation(9)
    y = orc.moe_forward(x, idx, w, list(W1), list(W2), n_threads=1)
    yp = orc.moe_forward(x[perm], idx[perm], w[perm], list(W1), list(W2), n_threads=1)
    np.testing.assert_array_equal(yp, y[perm])
    # the plan moves pairs the way the stable rule predicts
    r = orc.plan(idx[perm], 4, 8)
    _, _, pr, _ = plan_bruteforce(idx[perm], 4, 8)
    np.testing.assert_array_equal(r["pool_row"], pr)


# ---------------------------------------------------------------- combine --------------

def pin_identity_closed_form(orc):
    """Identity experts: y[t] = x[t] * (sum of t's live routing weights)."""
    rng = _rng(9)
    T, H, k, E = 20, 24, 4, 10
    x = bf16(rng.standard_normal((T, H)))
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    y = orc.moe_forward_identity(x, idx, w)
    s = np.where(idx >= 0, w.astype(np.float64), 0.0).sum(axis=1)
    np.testing.assert_allclose(y, f64(x) * s[:, None], rtol=1e-15, atol=0)


def pin_combine_gather(orc):
    rng = _rng(10)
    T, k, E, tile, H = 30, 3, 5, 4, 12
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    w = rng.standard_normal((T, k)).astype(np.float32)
    r = orc.plan(idx, E, tile)
    ypool = bf16(rng.standard_normal((r["P"], H)))
    y = orc.combine(r["pool_row"], w, ypool)
    yp = f64(ypool)
    expect = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            p = r["pool_row"][t, j]
            if p >= 0:
                expect[t] += float(w[t, j]) * yp[p]
    np.testing.assert_allclose(y, expect, rtol=1e-15, atol=1e-300)
    # combine over the dispatched pool equals the identity-experts layer
    x = bf16(rng.standard_normal((T, H)))
    pool = orc.pool(r["row_src"], r["P"], x, k)
    np.testing.assert_allclose(orc.combine(r["pool_row"], w, pool),
                               orc.moe_forward_identity(x, idx, w), rtol=1e-15, atol=0)


# ---------------------------------------------------------------- router ---------------

def route_bruteforce(logits, k, bias=None):
    """np.lexsort on (-score, index) of the fp32 scores; softmax over all experts in double,
    renormalised over the chosen ones."""
    v = logits.astype(np.float32) + (bias.astype(np.float32) if bias is not None else np.float32(0))
    T, E = v.shape
    idx = np.empty((T, k), np.int64)
    w = np.empty((T, k))
    for t in range(T):
        order = np.lexsort((np.arange(E), -v[t].astype(np.float64)))
        idx[t] = order[:k]
        p = np.exp(v[t].astype(np.float64) - v[t].max())
        p /= p.sum()
        w[t] = p[order[:k]] / p[order[:k]].sum()
    return idx, w


def pin_route_bruteforce(orc):
    rng = _rng(11)
    for (T, E, k, with_bias) in [(50, 8, 2, False), (40, 64, 8, True), (10, 256, 8, True),
                                 (7, 5, 5, False), (9, 33, 1, True)]:
        lg = rng.standard_normal((T, E)).astype(np.float32)
        b = (rng.standard_normal(E) * 0.5).astype(np.float32) if with_bias else None
        idx, w = orc.route(lg, k, b)
        ridx, rw = route_bruteforce(lg, k, b)
        np.testing.assert_array_equal(idx, ridx)
        np.testing.assert_allclose(w, rw, rtol=1e-12, atol=0)


def pin_route_special_cases(orc):
    rng = _rng(12)
    lg = rng.standard_normal((6, 16)).astype(np.float32)
    idx, w = orc.route(lg, 1)
    np.testing.assert_array_equal(idx[:, 0], np.argmax(lg, axis=1))
    assert np.all(w == 1.0)                                       # k = 1: weight exactly 1
    idx, w = orc.route(lg, 16)                                    # k = E: the full softmax
    sm = np.exp(lg.astype(np.float64) - lg.max(1, keepdims=True))
    sm /= sm.sum(1, keepdims=True)
    np.testing.assert_allclose(w, np.take_along_axis(sm, idx.astype(np.int64), 1), rtol=1e-12)
    tie = np.zeros((1, 6), np.float32)
    tie[0, [1, 4]] = 2.0                                          # exact tie: lower index first
    idx, w = orc.route(tie, 3)
    assert idx.tolist() == [[1, 4, 0]]
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-15)


def _bf16_neighbours(b: int):
    """The bf16 values just below and just above the bf16 pattern b (b not +-0)."""
    if b & 0x8000:          # negative: a larger pattern is more negative
        return b + 1, b - 1
    return b - 1, b + 1


def pin_backward_finite_differences(orc):
    """dx and dw against central differences of the forward oracle's L = sum(dy * y).
    x moves to its neighbouring bf16 values (the inputs stay exact bf16); y is linear in
    w, so the difference quotient in w is exact up to rounding."""
    rng = _rng(11)
    T, H, I, E, k = 3, 16, 8, 3, 2
    x, W1, W2, idx, w = _rand_layer(rng, T, H, I, E, k)
    idx[1, 1] = -1                                   # one dropped pair
    dy = bf16(rng.standard_normal((T, H)))
    W1l, W2l = list(W1), list(W2)
    dx, dw = orc.moe_backward(x, idx, w, W1l, W2l, dy, n_threads=1)
    dyf = f64(dy)

    def loss(xx, ww):
        return float((orc.moe_forward(xx, idx, ww, W1l, W2l, n_threads=1) * dyf).sum())

    fd = np.zeros_like(dx)
    for t in range(T):
        for h in range(H):
            lo, hi = _bf16_neighbours(int(x[t, h]))
            xl, xh = x.copy(), x.copy()
            xl[t, h], xh[t, h] = lo, hi
            step = float(f64(np.array([hi], np.uint16))[0] - f64(np.array([lo], np.uint16))[0])
            fd[t, h] = (loss(xh, w) - loss(xl, w)) / step
    np.testing.assert_allclose(dx, fd, rtol=0, atol=2e-3 * np.abs(fd).max())
    for t in range(T):
        for j in range(k):
            d = np.float32(2.0 ** -8) * max(abs(w[t, j]), np.float32(1e-3))
            wl, wh = w.copy(), w.copy()
            wl[t, j] -= d
            wh[t, j] += d
            q = (loss(x, wh) - loss(x, wl)) / (float(wh[t, j]) - float(wl[t, j]))
            assert abs(dw[t, j] - q) <= 1e-9 * max(1.0, abs(q)), (t, j, dw[t, j], q)
    assert dw[1, 1] == 0.0                           # the dropped pair


def pin_backward_textbook_torch(orc):
    """E=1, k=1, w=1: the gradient of sum(dy * FFN(x)) for a dense SwiGLU FFN by torch
    float64 autograd; dw is sum(dy * FFN(x)) per token."""
    import torch
    rng = _rng(12)
    T, H, I = 6, 24, 16
    x, W1, W2, _, _ = _rand_layer(rng, T, H, I, 1, 1)
    dy = bf16(rng.standard_normal((T, H)))
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    dx, dw = orc.moe_backward(x, idx, w, [W1[0]], [W2[0]], dy, n_threads=1)
    X = torch.from_numpy(f64(x)).requires_grad_(True)
    Wg = torch.from_numpy(f64(W1[0][:, :I]))
    Wu = torch.from_numpy(f64(W1[0][:, I:]))
    Wd = torch.from_numpy(f64(W2[0]))
    Y = (torch.nn.functional.silu(X @ Wg) * (X @ Wu)) @ Wd
    D = torch.from_numpy(f64(dy))
    (Y * D).sum().backward()
    np.testing.assert_allclose(dx, X.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw[:, 0], (Y * D).sum(1).detach().numpy(), rtol=1e-10,
                               atol=1e-12)


def pin_backward_linear_in_dy(orc):
    """Doubling dy doubles dx and dw exactly (every operation is linear in dy and scaling
    by 2 is exact in double); dy = 0 gives zeros."""
    rng = _rng(13)
    x, W1, W2, idx, w = _rand_layer(rng, 4, 16, 8, 3, 2, drop=0.25)
    dy = bf16(rng.standard_normal((4, 16)))
    dy2 = bf16(2.0 * f64(dy))
    a = orc.moe_backward(x, idx, w, list(W1), list(W2), dy, n_threads=1)
    b = orc.moe_backward(x, idx, w, list(W1), list(W2), dy2, n_threads=1)
    assert np.array_equal(2.0 * a[0], b[0]) and np.array_equal(2.0 * a[1], b[1])
    z = orc.moe_backward(x, idx, w, list(W1), list(W2), np.zeros_like(dy), n_threads=1)
    assert not z[0].any() and not z[1].any()


def pin_weight_grads_finite_differences(orc):
    """dW1 and dW2 of one expert against central differences of the forward oracle's
    L = sum(dy * y), each weight moved to its neighbouring bf16 values."""
    rng = _rng(14)
    T, H, I, E, k = 5, 8, 4, 3, 2
    x, W1, W2, idx, w = _rand_layer(rng, T, H, I, E, k)
    idx[2, 1] = -1
    e = int(idx[0, 0])
    dy = bf16(rng.standard_normal((T, H)))
    dW1, dW2 = orc.expert_weight_grads(x, idx, w, W1[e], W2[e], e, dy)
    dyf = f64(dy)

    def loss(W1m, W2m):
        return float((orc.moe_forward(x, idx, w, list(W1m), list(W2m), n_threads=1) * dyf).sum())

    for name, W, dW in (("W1", W1, dW1), ("W2", W2, dW2)):
        fd = np.zeros_like(dW)
        for pos in np.ndindex(*dW.shape):
            lo, hi = _bf16_neighbours(int(W[e][pos]))
            Wl, Wh = W.copy(), W.copy()
            Wl[e][pos], Wh[e][pos] = lo, hi
            step = float(f64(np.array([hi], np.uint16))[0] - f64(np.array([lo], np.uint16))[0])
            if name == "W1":
                fd[pos] = (loss(Wh, W2) - loss(Wl, W2)) / step
            else:
                fd[pos] = (loss(W1, Wh) - loss(W1, Wl)) / step
        np.testing.assert_allclose(dW, fd, rtol=0, atol=2e-3 * np.abs(fd).max(), err_msg=name)


def pin_weight_grads_textbook_torch(orc):
    """E=1, k=1, w=1: dW1 and dW2 of a dense SwiGLU FFN by torch float64 autograd."""
    import torch
    rng = _rng(15)
    T, H, I = 7, 16, 12
    x, W1, W2, _, _ = _rand_layer(rng, T, H, I, 1, 1)
    dy = bf16(rng.standard_normal((T, H)))
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    dW1, dW2 = orc.expert_weight_grads(x, idx, w, W1[0], W2[0], 0, dy)
    X = torch.from_numpy(f64(x))
    A = torch.from_numpy(f64(W1[0])).requires_grad_(True)
    B = torch.from_numpy(f64(W2[0])).requires_grad_(True)
    Y = (torch.nn.functional.silu(X @ A[:, :I]) * (X @ A[:, I:])) @ B
    (Y * torch.from_numpy(f64(dy))).sum().backward()
    np.testing.assert_allclose(dW1, A.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dW2, B.grad.numpy(), rtol=1e-10, atol=1e-12)


ALL_PINS = [
    pin_plan_worked, pin_plan_bruteforce, pin_plan_invariants, pin_plan_bad_index,
    pin_pool_gather, pin_ffn_worked, pin_ffn_dense_bruteforce, pin_ffn_textbook_torch,
    pin_ffn_closed_form, pin_ffn_linearity, pin_ffn_permutation, pin_identity_closed_form,
    pin_combine_gather, pin_route_bruteforce, pin_route_special_cases,
    pin_backward_finite_differences, pin_backward_textbook_torch, pin_backward_linear_in_dy,
    pin_weight_grads_finite_differences, pin_weight_grads_textbook_torch,
]
