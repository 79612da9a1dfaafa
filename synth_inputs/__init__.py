"""Seeded synthetic inputs for the MoE layer (shared by the CUDA path's tests/bench and the oracle).

Holds no arithmetic of the layer itself: it draws x, W1, W2 and the router's
top-k choice with a counter-based generator (SplitMix64 + Box-Muller, defined in
``gen.c``) so that any slice can be regenerated on its own, bit for bit.

Workloads (shapes and distributions of the StreamEP pool-layout MoE layer that the
pages describe; the sizes follow the DeepSeek-V3 / Qwen3-235B-A22B families and the
3 x 128-token decode micro-batches of attention/FFN disaggregation):

  tiny              T=256,  H=256,  I=512,  E=8,   k=2, tile=64,  softmax top-k
  qwen3_235b_a22b   T=4096, H=4096, I=1536, E=128, k=8, tile=128, softmax top-k
  deepseek_v3       T=8192, H=7168, I=2048, E=256, k=8, tile=128, softmax top-k with
                    a per-expert N(0, 0.5) bias added to the logits
  decode_microbatch 3 x T=128, H=7168, I=2048, E=256, k=8, tile=128, Zipf(1.2) routing
  dc_sweep_T{1024,4096,16384,65536}_{uniform,zipf}
                    H=7168, E=256, k=8, tile=128, identity experts
  deepseek_v3_e32   T=1024, H=7168, I=2048, E=32, k=8, tile=128 (profiling size)
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

# Stream ids of the counter-based generator.
STREAM_X = 1
STREAM_W1 = 2
STREAM_W2 = 3
STREAM_LOGITS = 4
STREAM_BIAS = 5
STREAM_PERM = 6
STREAM_DRAW = 7
STREAM_ZLOGITS = 8
STREAM_DY = 9        # upstream gradient of the layer output (backward)

SEED_BASE = 0x5EED0000


def build(verbose: bool = False) -> str:
    """Compile ``gen.c`` into ``libsynth.so`` next to it (gcc, OpenMP, no fast-math)."""
    import subprocess

    src = os.path.join(_HERE, "gen.c")
    # written under a name of this process, then renamed into place: another process never
    # loads a half-written library, and two builds at once do not mix their output
    tmp = f"{_LIB_PATH}.tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i64, f64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.gen_bits.argtypes = [u64, u64, u64, i64, vp]
        L.gen_uniform_f64.argtypes = [u64, u64, u64, i64, vp]
        L.gen_normal_f64.argtypes = [u64, u64, u64, i64, f64, vp]
        L.gen_normal_f32.argtypes = [u64, u64, u64, i64, f64, vp]
        L.gen_normal_bf16.argtypes = [u64, u64, u64, i64, f64, vp]
        L.gen_router_softmax_topk.argtypes = [i64, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.gen_router_softmax_topk.restype = ctypes.c_int
        L.gen_router_zipf.argtypes = [i64, i64, ctypes.c_int, ctypes.c_int, f64, u64, u64, u64, u64,
                                      vp, vp]
        L.gen_router_zipf.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def bits(seed: int, stream: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint64)
    lib().gen_bits(seed, stream, first, n, _ptr(out))
    return out


def uniform(seed: int, stream: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().gen_uniform_f64(seed, stream, first, n, _ptr(out))
    return out


def normal_f64(seed: int, stream: int, first: int, n: int, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(n, np.float64)
    lib().gen_normal_f64(seed, stream, first, n, sigma, _ptr(out))
    return out


def normal_f32(seed: int, stream: int, first: int, n: int, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().gen_normal_f32(seed, stream, first, n, sigma, _ptr(out))
    return out


def normal_bf16(seed: int, stream: int, first: int, n: int, sigma: float = 1.0,
                out: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bit patterns (uint16) of sigma * N(0,1), elements [first, first + n) of a stream."""
    if out is None:
        out = np.empty(n, np.uint16)
    assert out.dtype == np.uint16 and out.size == n
    lib().gen_normal_bf16(seed, stream, first, n, sigma, _ptr(out))
    return out


def normal_bf16_into(addr: int, seed: int, stream: int, first: int, n: int, sigma: float) -> None:
    """Same as :func:`normal_bf16`, written to raw host memory at ``addr`` (e.g. pinned memory)."""
    lib().gen_normal_bf16(seed, stream, first, n, sigma, addr)


def router_softmax_topk(logits: np.ndarray, k: int, bias: Optional[np.ndarray] = None):
    T, E = logits.shape
    logits = np.ascontiguousarray(logits, np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    b = 0
    if bias is not None:
        bias = np.ascontiguousarray(bias, np.float32)
        b = _ptr(bias)
    rc = lib().gen_router_softmax_topk(T, E, k, _ptr(logits), b, _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("router_softmax_topk: bad sizes")
    return idx, w


def router_zipf(T: int, t0: int, E: int, k: int, alpha: float, seed: int):
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    rc = lib().gen_router_zipf(T, t0, E, k, alpha, seed, STREAM_PERM, STREAM_DRAW, STREAM_ZLOGITS,
                               _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError("router_zipf: bad sizes")
    return idx, w


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens per layer call (per micro-batch for decode)
    H: int                 # hidden size
    I: int                 # expert intermediate size
    E: int                 # experts
    k: int                 # top-k
    tile: int              # pool tile rows
    seed: int
    routing: str = "softmax"     # "softmax" | "softmax_bias" | "zipf"
    alpha: float = 1.2           # Zipf exponent
    bias_sigma: float = 0.5      # std of the per-expert router bias (softmax_bias)
    micro_batches: int = 1       # independent layer calls, T tokens each
    identity: bool = False       # identity experts: no FFN, combine reads the pool

    @property
    def total_tokens(self) -> int:
        return self.T * self.micro_batches

    @property
    def pairs(self) -> int:
        return self.T * self.k

    def pool_rows_max(self) -> int:
        """Dropless pool bound: T*k real rows + at most (tile - 1) padding rows per non-empty expert."""
        n = self.T * self.k
        rows = n + min(self.E, n) * (self.tile - 1)
        return (rows + self.tile - 1) // self.tile * self.tile

    def w1_sigma(self) -> float:
        return 1.0 / math.sqrt(self.H)

    def w2_sigma(self) -> float:
        return 1.0 / math.sqrt(self.I)


def _cfg_list():
    out = {}
    out["tiny"] = MoEConfig("tiny", T=256, H=256, I=512, E=8, k=2, tile=64, seed=SEED_BASE + 0)
    out["qwen3_235b_a22b"] = MoEConfig("qwen3_235b_a22b", T=4096, H=4096, I=1536, E=128, k=8,
                                       tile=128, seed=SEED_BASE + 1)
    out["deepseek_v3"] = MoEConfig("deepseek_v3", T=8192, H=7168, I=2048, E=256, k=8, tile=128,
                                   seed=SEED_BASE + 2, routing="softmax_bias", bias_sigma=0.5)
    out["decode_microbatch"] = MoEConfig("decode_microbatch", T=128, H=7168, I=2048, E=256, k=8,
                                         tile=128, seed=SEED_BASE + 3, routing="zipf", alpha=1.2,
                                         micro_batches=3)
    # the DeepSeek-V3 expert shape at 32 experts: ~256 rows per expert like the full layer,
    # about 3 GB on the device (for detailed kernel profiles)
    out["deepseek_v3_e32"] = MoEConfig("deepseek_v3_e32", T=1024, H=7168, I=2048, E=32, k=8,
                                       tile=128, seed=SEED_BASE + 5, routing="softmax_bias",
                                       bias_sigma=0.5)
    for T in (1024, 4096, 16384, 65536):
        for r in ("uniform", "zipf"):
            nm = f"dc_sweep_T{T}_{r}"
            out[nm] = MoEConfig(nm, T=T, H=7168, I=0, E=256, k=8, tile=128, seed=SEED_BASE + 4,
                                routing="softmax" if r == "uniform" else "zipf", alpha=1.2,
                                identity=True)
    return out


CONFIGS = _cfg_list()


def custom(name: str, T: int, H: int, I: int, E: int, k: int, tile: int, seed: int,
           routing: str = "softmax", **kw) -> MoEConfig:
    """A config of any shape with the same recipe (used for edge cases and small tests)."""
    return MoEConfig(name, T=T, H=H, I=I, E=E, k=k, tile=tile, seed=seed, routing=routing, **kw)


def make_routing(cfg: MoEConfig, micro_batch: int = 0):
    """topk_idx [T, k] int32 and topk_w [T, k] fp32 for one layer call."""
    t0 = micro_batch * cfg.T
    if cfg.routing == "zipf":
        return router_zipf(cfg.T, t0, cfg.E, cfg.k, cfg.alpha, cfg.seed)
    logits = normal_f32(cfg.seed, STREAM_LOGITS, t0 * cfg.E, cfg.T * cfg.E).reshape(cfg.T, cfg.E)
    bias = None
    if cfg.routing == "softmax_bias":
        bias = normal_f32(cfg.seed, STREAM_BIAS, 0, cfg.E, cfg.bias_sigma)
    return router_softmax_topk(logits, cfg.k, bias)


def make_x(cfg: MoEConfig, micro_batch: int = 0) -> np.ndarray:
    """x [T, H] bf16 bit patterns, N(0,1)."""
    t0 = micro_batch * cfg.T
    return normal_bf16(cfg.seed, STREAM_X, t0 * cfg.H, cfg.T * cfg.H).reshape(cfg.T, cfg.H)



def make_dy(cfg: MoEConfig, mb: int = 0) -> np.ndarray:
    """dy [T, H] bf16 ~ N(0, 1): the gradient of a loss with respect to the layer output,
    for the backward (micro-batch mb)."""
    n = cfg.T * cfg.H
    return normal_bf16(cfg.seed, STREAM_DY, mb * n, n, 1.0).reshape(cfg.T, cfg.H)

def make_x_rows(cfg: MoEConfig, tokens: np.ndarray, micro_batch: int = 0) -> np.ndarray:
    """Selected rows of x (global regeneration of single rows)."""
    t0 = micro_batch * cfg.T
    out = np.empty((len(tokens), cfg.H), np.uint16)
    for i, t in enumerate(tokens):
        normal_bf16(cfg.seed, STREAM_X, (t0 + int(t)) * cfg.H, cfg.H, 1.0, out[i])
    return out


def make_w1_expert(cfg: MoEConfig, e: int) -> np.ndarray:
    """W1[e] [H, 2I] bf16 bits; columns [0, I) are the gate projection, [I, 2I) the up projection."""
    n = cfg.H * 2 * cfg.I
    return normal_bf16(cfg.seed, STREAM_W1, e * n, n, cfg.w1_sigma()).reshape(cfg.H, 2 * cfg.I)


def make_w2_expert(cfg: MoEConfig, e: int) -> np.ndarray:
    """W2[e] [I, H] bf16 bits."""
    n = cfg.I * cfg.H
    return normal_bf16(cfg.seed, STREAM_W2, e * n, n, cfg.w2_sigma()).reshape(cfg.I, cfg.H)


def make_w1(cfg: MoEConfig) -> np.ndarray:
    n = cfg.E * cfg.H * 2 * cfg.I
    return normal_bf16(cfg.seed, STREAM_W1, 0, n, cfg.w1_sigma()).reshape(cfg.E, cfg.H, 2 * cfg.I)


def make_w2(cfg: MoEConfig) -> np.ndarray:
    n = cfg.E * cfg.I * cfg.H
    return normal_bf16(cfg.seed, STREAM_W2, 0, n, cfg.w2_sigma()).reshape(cfg.E, cfg.I, cfg.H)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 bit patterns (nearest-even), for building test inputs."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r
