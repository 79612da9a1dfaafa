"""CPU oracle for the MoE layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The product package (``combine_moe_plan_03_b200``) never
imports it and shares no code with it. The arithmetic lives in ``oracle.c``
(plain C, double precision); this module compiles it with gcc and marshals
numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")

ERR_ARG = -1
ERR_MISSING_EXPERT = -2
ERR_BAD_INDEX = -10

CFLAGS = ["-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-std=c11"]


def build(src: str = SRC, out: str = LIB_PATH, verbose: bool = False) -> str:
    """Compile the oracle (gcc, strict IEEE double: no fast-math, no FMA contraction)."""
    # written under a name of this process, then renamed into place: another process never
    # loads a half-written library, and two builds at once do not mix their output
    tmp = f"{out}.tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, "-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes view of one compiled oracle library (the real one, or a test variant)."""

    def __init__(self, path: str = LIB_PATH):
        if path == LIB_PATH and not os.path.exists(path):
            build()
        L = ctypes.CDLL(path)
        i32, i64, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
        L.oracle_pool_rows_max.argtypes = [i64, i32, i32, i32]
        L.oracle_pool_rows_max.restype = i64
        L.oracle_plan.argtypes = [i64, i32, i32, i32, vp, vp, vp, vp, vp, i64, vp, i64, vp]
        L.oracle_plan.restype = ctypes.c_int
        L.oracle_pool.argtypes = [i64, i32, i32, vp, vp, vp]
        L.oracle_expert_ffn.argtypes = [i32, i32, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_forward.argtypes = [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                         ctypes.c_int]
        L.oracle_moe_forward.restype = ctypes.c_int
        L.oracle_moe_forward_identity.argtypes = [i64, i32, i32, vp, vp, vp, vp]
        L.oracle_moe_forward_identity.restype = ctypes.c_int
        L.oracle_combine.argtypes = [i64, i32, i32, vp, vp, vp, vp]
        L.oracle_combine.restype = ctypes.c_int
        L.oracle_route.argtypes = [i64, i32, i32, vp, vp, vp, vp]
        L.oracle_route.restype = ctypes.c_int
        L.oracle_moe_backward.argtypes = [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                          vp, ctypes.c_int]
        L.oracle_moe_backward.restype = ctypes.c_int
        L.oracle_expert_weight_grads.argtypes = [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp,
                                                 i32, vp, vp, vp]
        L.oracle_expert_weight_grads.restype = ctypes.c_int
        self.L = L

    # ---- plan -------------------------------------------------------------------------
    def pool_rows_max(self, T: int, k: int, E: int, tile: int) -> int:
        return int(self.L.oracle_pool_rows_max(T, k, E, tile))

    def plan(self, topk_idx: np.ndarray, E: int, tile: int):
        """Returns dict(counts, offsets, pool_row, row_src, tile_expert, P) or raises on error."""
        idx = np.ascontiguousarray(topk_idx, np.int32)
        T, k = idx.shape
        pmax = self.pool_rows_max(T, k, E, tile)
        counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        pool_row = np.empty(T * k, np.int32)
        row_src = np.empty(pmax, np.int32)
        tile_expert = np.empty(max(pmax // tile, 1), np.int32)
        P = ctypes.c_int64(0)
        rc = self.L.oracle_plan(T, k, E, tile, _p(idx), _p(counts), _p(offsets), _p(pool_row),
                                _p(row_src), pmax, _p(tile_expert), tile_expert.size,
                                ctypes.addressof(P))
        if rc != 0:
            raise OracleError(rc)
        return dict(counts=counts, offsets=offsets, pool_row=pool_row.reshape(T, k),
                    row_src=row_src, tile_expert=tile_expert[: pmax // tile], P=int(P.value),
                    P_max=pmax)

    def pool(self, row_src: np.ndarray, P: int, x: np.ndarray, k: int) -> np.ndarray:
        x = np.ascontiguousarray(x, np.uint16)
        rs = np.ascontiguousarray(row_src, np.int32)
        H = x.shape[1]
        out = np.empty((P, H), np.uint16)
        self.L.oracle_pool(P, H, k, _p(rs), _p(x), _p(out))
        return out

    # ---- FFN / layer ------------------------------------------------------------------
    def expert_ffn(self, x_row: np.ndarray, W1e: np.ndarray, W2e: np.ndarray):
        """Returns (g, u, a, z) in float64 for one token row through one expert."""
        H = x_row.shape[0]
        I = W2e.shape[0]
        x_row = np.ascontiguousarray(x_row, np.uint16)
        W1e = np.ascontiguousarray(W1e, np.uint16)
        W2e = np.ascontiguousarray(W2e, np.uint16)
        g, u, a = (np.empty(I, np.float64) for _ in range(3))
        z = np.empty(H, np.float64)
        self.L.oracle_expert_ffn(H, I, _p(x_row), _p(W1e), _p(W2e), _p(g), _p(u), _p(a), _p(z))
        return g, u, a, z

    def moe_forward(self, x_rows: np.ndarray, idx_rows: np.ndarray, w_rows: np.ndarray,
                    W1: Sequence[Optional[np.ndarray]], W2: Sequence[Optional[np.ndarray]],
                    n_threads: int = 0) -> np.ndarray:
        """y [n, H] float64 for the given token rows. W1/W2: one array (or None) per expert."""
        x_rows = np.ascontiguousarray(x_rows, np.uint16)
        idx_rows = np.ascontiguousarray(idx_rows, np.int32)
        w_rows = np.ascontiguousarray(w_rows, np.float32)
        n, H = x_rows.shape
        k = idx_rows.shape[1]
        E = len(W1)
        I = next(w.shape[0] for w in W2 if w is not None)
        keep = []
        p1 = (ctypes.c_void_p * E)()
        p2 = (ctypes.c_void_p * E)()
        for e in range(E):
            if W1[e] is not None:
                a1 = np.ascontiguousarray(W1[e], np.uint16)
                a2 = np.ascontiguousarray(W2[e], np.uint16)
                keep += [a1, a2]
                p1[e] = a1.ctypes.data
                p2[e] = a2.ctypes.data
        y = np.empty((n, H), np.float64)
        if n_threads <= 0:
            n_threads = os.cpu_count() or 1
        rc = self.L.oracle_moe_forward(n, H, I, E, k, _p(x_rows), _p(idx_rows), _p(w_rows),
                                       p1, p2, _p(y), n_threads)
        if rc != 0:
            raise OracleError(rc)
        return y

    def moe_backward(self, x_rows: np.ndarray, idx_rows: np.ndarray, w_rows: np.ndarray,
                     W1: Sequence[Optional[np.ndarray]], W2: Sequence[Optional[np.ndarray]],
                     dy_rows: np.ndarray, n_threads: int = 0):
        """(dx [n, H], dw [n, k]) in float64: gradients of sum(dy * y) for the given tokens."""
        x_rows = np.ascontiguousarray(x_rows, np.uint16)
        idx_rows = np.ascontiguousarray(idx_rows, np.int32)
        w_rows = np.ascontiguousarray(w_rows, np.float32)
        dy_rows = np.ascontiguousarray(dy_rows, np.uint16)
        n, H = x_rows.shape
        k = idx_rows.shape[1]
        E = len(W1)
        I = next(w.shape[0] for w in W2 if w is not None)
        keep = []
        p1 = (ctypes.c_void_p * E)()
        p2 = (ctypes.c_void_p * E)()
        for e in range(E):
            if W1[e] is not None:
                a1 = np.ascontiguousarray(W1[e], np.uint16)
                a2 = np.ascontiguousarray(W2[e], np.uint16)
                keep += [a1, a2]
                p1[e] = a1.ctypes.data
                p2[e] = a2.ctypes.data
        dx = np.empty((n, H), np.float64)
        dw = np.empty((n, k), np.float64)
        if n_threads <= 0:
            n_threads = os.cpu_count() or 1
        rc = self.L.oracle_moe_backward(n, H, I, E, k, _p(x_rows), _p(idx_rows), _p(w_rows),
                                        p1, p2, _p(dy_rows), _p(dx), _p(dw), n_threads)
        if rc != 0:
            raise OracleError(rc)
        return dx, dw

    def expert_weight_grads(self, x: np.ndarray, topk_idx: np.ndarray, topk_w: np.ndarray,
                            W1e: np.ndarray, W2e: np.ndarray, e: int, dy: np.ndarray):
        """(dW1 [H, 2I], dW2 [I, H]) in float64 for expert e, over all tokens of the call."""
        x = np.ascontiguousarray(x, np.uint16)
        idx = np.ascontiguousarray(topk_idx, np.int32)
        w = np.ascontiguousarray(topk_w, np.float32)
        W1e = np.ascontiguousarray(W1e, np.uint16)
        W2e = np.ascontiguousarray(W2e, np.uint16)
        dy = np.ascontiguousarray(dy, np.uint16)
        T, H = x.shape
        k = idx.shape[1]
        I = W2e.shape[0]
        dW1 = np.empty((H, 2 * I), np.float64)
        dW2 = np.empty((I, H), np.float64)
        E = int(max(idx.max(initial=0), e)) + 1
        rc = self.L.oracle_expert_weight_grads(T, H, I, E, k, _p(x), _p(idx), _p(w), _p(W1e),
                                               _p(W2e), e, _p(dy), _p(dW1), _p(dW2))
        if rc != 0:
            raise OracleError(rc)
        return dW1, dW2

    def moe_forward_identity(self, x: np.ndarray, topk_idx: np.ndarray,
                             topk_w: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, np.uint16)
        idx = np.ascontiguousarray(topk_idx, np.int32)
        w = np.ascontiguousarray(topk_w, np.float32)
        T, H = x.shape
        y = np.empty((T, H), np.float64)
        rc = self.L.oracle_moe_forward_identity(T, H, idx.shape[1], _p(x), _p(idx), _p(w), _p(y))
        if rc != 0:
            raise OracleError(rc)
        return y

    def combine(self, pool_row: np.ndarray, topk_w: np.ndarray, ypool: np.ndarray) -> np.ndarray:
        pr = np.ascontiguousarray(pool_row, np.int32)
        w = np.ascontiguousarray(topk_w, np.float32)
        yp = np.ascontiguousarray(ypool, np.uint16)
        T, k = pr.shape
        H = yp.shape[1]
        y = np.empty((T, H), np.float64)
        rc = self.L.oracle_combine(T, H, k, _p(pr), _p(w), _p(yp), _p(y))
        if rc != 0:
            raise OracleError(rc)
        return y


    def route(self, logits: np.ndarray, k: int, bias: Optional[np.ndarray] = None):
        """Router: (topk_idx [T, k] int32, topk_w [T, k] float64) from fp32 logits [T, E]."""
        lg = np.ascontiguousarray(logits, np.float32)
        T, E = lg.shape
        b = None if bias is None else np.ascontiguousarray(bias, np.float32)
        idx = np.empty((T, k), np.int32)
        w = np.empty((T, k), np.float64)
        rc = self.L.oracle_route(T, E, k, _p(lg), 0 if b is None else _p(b), _p(idx), _p(w))
        if rc != 0:
            raise OracleError(rc)
        return idx, w


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle error {code}")
        self.code = code


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
