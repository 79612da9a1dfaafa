"""The SwiGLU epilogue's reciprocal (magic-constant estimate + two Newton-Raphson steps,
csrc/ffn_gemm.cuh) emulated in float32 on the host: its error bound over the whole range
it is used on, so that a change of the constant or of the step count is caught without
a GPU. The device results themselves are checked element by element against the oracle
in tests/test_gpu_ffn.py."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _device_constant():
    src = open(os.path.join(ROOT, "combine_moe_plan_03_b200", "csrc", "ffn_gemm.cuh")).read()
    k = int(re.search(r"kRecipMagic = (0x[0-9A-Fa-f]+);", src).group(1), 16)
    steps = len(re.findall(r"y = y \* fmaf\(-d, y, 2\.0f\);",
                           src[src.index("recip_newton2"):src.index("silu_mul")]))
    return k, steps


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 a, b; one rounding of the sum to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c).astype(np.float32)


def test_reciprocal_error_bound_over_its_range():
    k, steps = _device_constant()
    assert steps == 2
    d = np.concatenate([np.linspace(1, 2, 100001, dtype=np.float32),
                        (2.0 ** np.linspace(0, 100, 100001)).astype(np.float32)])
    y = (np.int64(k) - d.view(np.int32).astype(np.int64)).astype(np.int32).view(np.float32)
    first = np.abs(y.astype(np.float64) * d - 1).max()
    assert first < 0.052                     # first estimate within 5.1%
    for _ in range(steps):
        y = (y * _fma32(-d, y, 2.0)).astype(np.float32)
    rel = np.abs(y.astype(np.float64) * d - 1).max()
    assert rel < 1e-5                        # well under a bf16 ulp (2^-8 relative)


def test_silu_emulation_matches_definition():
    """silu(g)*u through the emulated reciprocal agrees with the textbook formula in
    float64 to 2e-5 relative over g in [-60, 60] (exp taken exactly here: the device's
    ex2.approx adds about 2^-22)."""
    k, _ = _device_constant()
    g = np.linspace(-60, 60, 200001).astype(np.float32)
    u = np.float32(1.25)
    e = np.minimum(np.exp2(np.minimum(g.astype(np.float64) * -1.4426950408889634, 100.0)),
                   np.finfo(np.float32).max).astype(np.float32)
    d = (np.float32(1.0) + e).astype(np.float32)
    y = (np.int64(k) - d.view(np.int32).astype(np.int64)).astype(np.int32).view(np.float32)
    for _ in range(2):
        y = (y * _fma32(-d, y, 2.0)).astype(np.float32)
    got = g.astype(np.float64) * u * y
    ref = g.astype(np.float64) * u / (1.0 + np.exp(-g.astype(np.float64)))
    assert np.all(np.abs(got - ref) <= 2e-5 * np.abs(ref) + 1e-30)


def test_reciprocal_magic_constant_is_the_minimax_first_estimate():
    """The reciprocal's first estimate takes the bit pattern M - bits(d). Over one binade
    of d (the error repeats in every binade) the best M is the one whose largest relative
    error is smallest; a scan finds it, and the constant in the kernels' header must be
    within 1e-6 of that optimum (and its two Newton steps below 1e-5)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "combine_moe_plan_03_b200", "csrc",
                            "ffn_gemm.cuh")).read()
    M_hdr = int(re.search(r"constexpr int32_t kRecipMagic = (0x[0-9A-Fa-f]+);", src).group(1), 16)
    d = np.linspace(1.0, 2.0, 400_001).astype(np.float32)
    db = d.view(np.int32).astype(np.int64)
    dd = d.astype(np.float64)

    def first(M):
        return (np.int64(M) - db).astype(np.int32).view(np.float32).astype(np.float64)

    def err(M):
        return np.abs(first(M) * dd - 1.0).max()

    coarse = min(range(0x7EF00000, 0x7EF60000, 0x100), key=err)
    best = min(range(coarse - 0x100, coarse + 0x100), key=err)
    assert err(M_hdr) - err(best) < 1e-6
    y = first(M_hdr)
    for _ in range(2):
        y = y * (2.0 - dd * y)
    assert np.abs(y * dd - 1.0).max() < 1e-5
