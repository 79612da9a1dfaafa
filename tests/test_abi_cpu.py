"""The C-ABI library without a GPU: it loads, exports every declared symbol, and rejects
bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"^(?:int|const char \*)\s*(moe_\w+)\(", src, re.M)))


def test_library_loads_and_exports_every_declared_symbol():
    import combine_moe_plan_03_b200 as moe
    L = ctypes.CDLL(moe.LIB_PATH)
    syms = declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(L, s), f"{s} declared in include/moe.h but not exported"
    assert sorted(moe.EXPORTS) == syms


def test_sizes_and_bind_are_host_only():
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(8192, 7168, 2048, 256, 8, 128)
    assert moe.moe_pool_rows_max(s) == 65536 + 256 * 127
    nbytes = moe.moe_plan_arena_bytes(s)
    assert nbytes > 0 and nbytes % 256 == 0
    p = moe.moe_plan_bind(s, 1 << 20)
    ptrs = [getattr(p, f) for f, _ in moe.moe_plan_buffers._fields_]
    assert ptrs == sorted(ptrs) and all(q % 256 == 0 for q in ptrs)
    assert ptrs[-1] < (1 << 20) + nbytes


@pytest.mark.parametrize("shape,code", [
    ((16, 100, 128, 8, 2, 64), -2),     # H not a multiple of 64
    ((16, 128, 128, 8, 2, 32), -2),     # tile not 64/128
    ((16, 128, 128, 8, 33, 64), -1),    # k > 32
    ((16, 128, 128, 2000, 2, 64), -1),  # E > 1024
    ((-1, 128, 128, 8, 2, 64), -1),
    ((16, 38784, 128, 8, 2, 64), -2),   # 3 rows of x exceed a dispatch block's shared memory
])
def test_bad_shapes_rejected(shape, code):
    import combine_moe_plan_03_b200 as moe
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_pool_rows_max(moe.moe_shape(*shape))
    assert ei.value.code == code


def test_misaligned_and_null_rejected_without_device():
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(16, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch(s, (1 << 20) + 8, p, 1 << 24)
    assert ei.value.code == moe.MOE_ERR_MISALIGNED
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_grouped_ffn(s, 1 << 20, 1 << 21, 0, p, 1 << 22, 1 << 23)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    bad = moe.moe_plan_buffers()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_combine(s, 1 << 20, 1 << 21, bad, 1 << 22)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_strerror(-11).startswith("streaming FFN")


def test_ffn_kernel_constants_and_config_layout():
    """The binding's constants and moe_config layout match include/moe.h; an unknown
    grouped-GEMM kernel is rejected on the host."""
    import combine_moe_plan_03_b200 as moe
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    defs = dict(re.findall(r"^#define (MOE_FFN_\w+) (\w+)", src, re.M))
    assert int(defs["MOE_FFN_ONE_SM"]) == moe.MOE_FFN_ONE_SM
    assert int(defs["MOE_FFN_SM_PAIR"]) == moe.MOE_FFN_SM_PAIR
    assert getattr(moe, defs["MOE_FFN_DEFAULT"]) == moe.MOE_FFN_DEFAULT
    body = re.search(r"typedef struct moe_config \{(.*?)\} moe_config;", src, re.S).group(1)
    fields = re.findall(r"^\s*(?:int32_t|void \*const \*|void \*)\s*(\w+);", body, re.M)
    assert fields == [f for f, _ in moe.moe_config._fields_]
    assert moe.moe_config.timing_events.offset == 24 and moe.moe_config.gate_up.offset == 32
    assert moe.moe_config.early_combine.offset == 40 and ctypes.sizeof(moe.moe_config) == 48
    s = moe.moe_shape(16, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    for bad in (3, -1):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_grouped_ffn(s, 1 << 20, 1 << 21, 1 << 21, p, 1 << 22, 1 << 23,
                                moe.moe_config(0, 0, 0, 0, bad))
        assert ei.value.code == moe.MOE_ERR_INVALID_ARG


def test_backward_rejects_unsupported_configs_on_the_host():
    """moe_backward needs the weights in their given layout, no streaming, the SM-pair
    kernels and every buffer; each violation is refused before any device work."""
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(16, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    q = [(1 << 21) + i * (1 << 16) for i in range(14)]

    def call(cfg, **over):
        a = dict(dy=q[0], tw=q[1], w1=q[2], w2=q[3], pool=q[4], act=q[5], ypool=q[6], gu=q[7],
                 dgu=q[8], dpool=q[9], dx=q[10], dw=q[11], dW1=q[12], dW2=q[13])
        a.update(over)
        moe.moe_backward(s, a["dy"], a["tw"], a["w1"], a["w2"], p, a["pool"], a["act"],
                         a["ypool"], a["gu"], a["dgu"], a["dpool"], a["dx"], a["dw"], a["dW1"],
                         a["dW2"], cfg, 0)

    for cfg in (moe.moe_config(0, 0, 0, 1, 0), moe.moe_config(1, 0, 0, 0, 0),
                moe.moe_config(0, 0, 0, 0, moe.MOE_FFN_ONE_SM), moe.moe_config(0, 0, 0, 0, 9)):
        with pytest.raises(moe.MoEError) as ei:
            call(cfg)
        assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    for over, code in (({"gu": 0}, moe.MOE_ERR_INVALID_ARG),          # a missing work buffer
                       ({"act": 0}, moe.MOE_ERR_INVALID_ARG),         # dW2 needs act
                       ({"dx": q[10] + 4}, moe.MOE_ERR_MISALIGNED),
                       ({"dW1": q[12] + 8}, moe.MOE_ERR_MISALIGNED)):
        with pytest.raises(moe.MoEError) as ei:
            call(None, **over)
        assert ei.value.code == code, over


def test_gate_up_needs_the_pair_kernel_and_alignment():
    """moe_config.gate_up (the training step's saved gate / up values) is refused with the
    one-CTA kernel and when misaligned, on the host."""
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(16, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    for cfg, code in ((moe.moe_config(0, 0, 0, 0, moe.MOE_FFN_ONE_SM, None, 1 << 24),
                       moe.MOE_ERR_INVALID_ARG),
                      (moe.moe_config(0, 0, 0, 0, 0, None, (1 << 24) + 8), moe.MOE_ERR_MISALIGNED)):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_grouped_ffn(s, 1 << 20, 1 << 21, 1 << 21, p, 1 << 22, 1 << 23, cfg)
        assert ei.value.code == code


def test_plan_struct_layout_matches_the_header():
    """moe_plan_buffers' fields in include/moe.h, in order, are the binding's; the arena
    gives the early-combine counters T and T + 4 ints after the status word."""
    import combine_moe_plan_03_b200 as moe
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    body = re.search(r"typedef struct moe_plan_buffers \{(.*?)\} moe_plan_buffers;", src,
                     re.S).group(1)
    fields = re.findall(r"^\s*u?int32_t \*(\w+);", body, re.M)
    assert fields == [f for f, _ in moe.moe_plan_buffers._fields_]
    s = moe.moe_shape(1000, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    assert p.tok_pending - p.status == 256                       # [4] status, 256-B aligned
    assert p.ready - p.tok_pending == (1000 * 4 + 255) // 256 * 256
    assert moe.moe_plan_arena_bytes(s) == p.ready + (1004 * 4 + 255) // 256 * 256 - (1 << 20)


def test_early_combine_is_refused_where_it_does_not_apply():
    """Early combine needs the SM-pair kernel, its own entry point (moe_grouped_ffn refuses
    it, moe_grouped_ffn_combine requires it) and the plan's counters; dispatch cannot arm
    counters that are not there. All checked on the host."""
    import combine_moe_plan_03_b200 as moe
    s = moe.moe_shape(16, 128, 128, 8, 2, 64)
    p = moe.moe_plan_bind(s, 1 << 20)
    args = (s, 1 << 22, 1 << 23, 1 << 23, p, 1 << 24, 1 << 25)
    cases = (
        (lambda: moe.moe_grouped_ffn(*args, moe.moe_config(early_combine=1))),
        (lambda: moe.moe_grouped_ffn_combine(*args, 1 << 26, 1 << 27, moe.moe_config())),
        (lambda: moe.moe_grouped_ffn_combine(
            *args, 1 << 26, 1 << 27, moe.moe_config(ffn_kernel=moe.MOE_FFN_ONE_SM,
                                                    early_combine=1))),
        (lambda: moe.moe_grouped_ffn_combine(*args, 1 << 26, 1 << 27,
                                             moe.moe_config(early_combine=2))),
    )
    for c in cases:
        with pytest.raises(moe.MoEError) as ei:
            c()
        assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    q = moe.moe_plan_buffers.from_buffer_copy(p)
    q.tok_pending = None
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_grouped_ffn_combine(s, 1 << 22, 1 << 23, 1 << 23, q, 1 << 24, 1 << 25, 1 << 26,
                                    1 << 27, moe.moe_config(early_combine=1))
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch(s, 1 << 22, q, 1 << 23, moe.MOE_DISPATCH_ARM_COMBINE)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:                      # out misaligned
        moe.moe_grouped_ffn_combine(*args, 1 << 26, (1 << 27) + 2, moe.moe_config(early_combine=1))
    assert ei.value.code == moe.MOE_ERR_MISALIGNED
    assert "early combine" in moe.moe_strerror(moe.MOE_ERR_COMBINE_TIMEOUT)
