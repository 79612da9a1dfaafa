"""Shared helpers for the GPU parity tests (inputs from synth_inputs, expectations from oracle)."""
from __future__ import annotations

import numpy as np
import torch

import synth_inputs as si

DEV = torch.device("cuda:0")


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 device tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return si.bf16_to_f64(bf16_host(t))


def i32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(DEV)


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


def weights_dev(cfg) -> tuple[torch.Tensor, torch.Tensor]:
    """W1 [E,H,2I], W2 [E,I,H] generated expert by expert on the host and copied to the device."""
    W1 = torch.empty((cfg.E, cfg.H, 2 * cfg.I), dtype=torch.bfloat16, device=DEV)
    W2 = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=DEV)
    step = max(1, (1 << 27) // (cfg.H * 2 * cfg.I))   # ~256 MB of host buffer per copy
    for e0 in range(0, cfg.E, step):
        e1 = min(cfg.E, e0 + step)
        n1 = cfg.H * 2 * cfg.I
        h1 = si.normal_bf16(cfg.seed, si.STREAM_W1, e0 * n1, (e1 - e0) * n1, cfg.w1_sigma())
        W1[e0:e1].copy_(torch.from_numpy(h1.view(np.int16)).view(torch.bfloat16)
                        .view(e1 - e0, cfg.H, 2 * cfg.I))
        n2 = cfg.I * cfg.H
        h2 = si.normal_bf16(cfg.seed, si.STREAM_W2, e0 * n2, (e1 - e0) * n2, cfg.w2_sigma())
        W2[e0:e1].copy_(torch.from_numpy(h2.view(np.int16)).view(torch.bfloat16)
                        .view(e1 - e0, cfg.I, cfg.H))
    return W1, W2


def check_plan_exact(buf, ref, T, k):
    """Bit-exact comparison of every plan output with the oracle's plan."""
    P = ref["P"]
    E = len(ref["counts"])
    np.testing.assert_array_equal(buf.plan_view("counts")[:E].cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(buf.plan_view("offsets")[:E + 1].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(buf.plan_view("pool_row")[:T * k].cpu().numpy(),
                                  ref["pool_row"].reshape(-1))
    np.testing.assert_array_equal(buf.plan_view("row_src")[:ref["P_max"]].cpu().numpy(),
                                  ref["row_src"])
    nt = ref["P_max"] // buf.shape.tile
    np.testing.assert_array_equal(buf.plan_view("tile_expert")[:nt].cpu().numpy(),
                                  ref["tile_expert"])
    meta = buf.plan_view("meta")[:4].cpu().numpy()
    assert meta[0] == P // buf.shape.tile and meta[1] == P
    # GEMM row chunks: an expert's live rows in ceil(c/256) equal chunks (multiples of 16),
    # each entry {first row, expert, rows, the expert's first chunk, its chunk count}
    mb = buf.plan_view("mblk")[: 5 * meta[2]].cpu().numpy().reshape(-1, 5)
    want = []
    for e in range(E):
        a, c = int(ref["offsets"][e]), int(ref["counts"][e])
        if c == 0:
            continue
        n = -(-c // 256)
        step = (-(-c // n) + 15) // 16 * 16
        first = len(want)
        for r in range(a, a + c, step):
            want.append((r, e, min(step, a + c - r), first, -(-c // step)))
    np.testing.assert_array_equal(mb, np.array(want, np.int64).reshape(-1, 5))


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if T <= n:
        return np.arange(T)
    s = set(rng.choice(T, size=n - 2, replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s))


def assert_layer_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = ""):
    """The layer's acceptance bound: max |err| <= 2e-2 * max |y_ref| (bf16 in, fp32 accumulate)."""
    err = np.abs(y_gpu - y_ref).max()
    tol = 2e-2 * np.abs(y_ref).max()
    assert np.isfinite(y_gpu).all(), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max|err| {err:.4e} > {tol:.4e}"
    return err, tol
