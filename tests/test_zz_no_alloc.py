"""moe_plan_noalloc, the plan for callers that cannot allocate device memory, against moe_plan.

Some callers run inside a framework that owns every byte of device memory and gives
extensions no allocator, or in loops that cannot afford a cudaMalloc. For them the
library keeps the plan's scratch in its own static device buffer. This file checks,
through the C ABI, that the no-allocation variant produces exactly what moe_plan
produces (integer maps: bit for bit), on two calls in a row so that scratch left
behind by the first call cannot leak into the second, and that a shape too big for
the static buffer is refused before anything runs. It is named to be collected last.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si

pytestmark = pytest.mark.gpu

FIELDS = ("counts", "offsets", "pool_row", "row_src", "tile_expert", "mblk", "meta",
          "tile_flags")


def _plan_outputs(buf, fields=FIELDS):
    return {f: buf.plan_view(f).cpu().numpy().copy() for f in fields}


def _routing(case):
    if case == "deepseek_v3":
        cfg = si.CONFIGS["deepseek_v3"]
        idx, _ = si.make_routing(cfg)
        return cfg.T, cfg.E, cfg.k, cfg.tile, idx
    if case == "largest_accepted":
        # E = 256 experts and 524,288 pairs: 256 * 2048 chunk counts + 8 = 524,296 of the
        # buffer's 524,352 ints, the largest shape of this E that fits
        rng = np.random.default_rng(11)
        T, E, k, tile = 65536, 256, 8, 128
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
        return T, E, k, tile, idx
    rng = np.random.default_rng(7)
    T, E, k, tile = 3000, 40, 6, 64
    idx = rng.integers(0, 5, size=(T, k)).astype(np.int32)   # skewed: 5 hot experts
    idx[rng.random(idx.shape) < 0.1] = -1                    # dropped pairs
    return T, E, k, tile, idx


def test_noalloc_plan_matches_moe_plan_two_calls_in_a_row():
    import combine_moe_plan_03_b200 as moe
    for case in ("deepseek_v3", "skewed_with_drops", "largest_accepted"):  # calls in a row
        T, E, k, tile, idx = _routing(case)
        d_idx = torch.from_numpy(idx).cuda()
        ref = moe.MoELayerBuffers(T, 64, 64, E, k, tile, identity=True)
        moe.moe_plan(ref.shape, d_idx.data_ptr(), ref.plan, 0, 0)
        got = moe.MoELayerBuffers(T, 64, 64, E, k, tile, identity=True)
        got.arena.fill_(0xA5)                                # poisoned outputs
        noalloc_plan = moe.moe_plan_buffers.from_buffer_copy(got.plan)
        noalloc_plan.workspace = None                        # not used by the variant
        moe.moe_clear_status(noalloc_plan, 0)
        moe.moe_plan_noalloc(got.shape, d_idx.data_ptr(), noalloc_plan, 0, 0)
        torch.cuda.synchronize()
        assert moe.moe_get_status(ref.plan)[0] == 0
        assert moe.moe_get_status(noalloc_plan)[0] == 0
        a, b = _plan_outputs(ref), _plan_outputs(got)
        n = {"counts": E, "offsets": E + 1, "pool_row": T * k, "row_src": ref.P_max,
             "tile_expert": ref.P_max // tile, "meta": 4, "tile_flags": ref.P_max // tile}
        for f in FIELDS:
            m = 5 * int(a["meta"][2]) if f == "mblk" else n[f]
            np.testing.assert_array_equal(b[f][:m], a[f][:m], err_msg=f"{case}: {f}")
        ref.close()
        got.close()


def test_noalloc_plan_rejects_shapes_beyond_its_scratch():
    import combine_moe_plan_03_b200 as moe
    p = moe.moe_plan_buffers(*([1 << 20] * 12))
    # E=1024 experts with 1M pairs needs 1024 * 4096 + 8 ints > 2^19 + 64;
    # one 256-pair chunk past the largest accepted E=256 shape needs 256 * 2049 + 8;
    # one expert more than that shape needs 257 * 2048 + 8
    for s in (moe.moe_shape(131072, 64, 64, 1024, 8, 128),
              moe.moe_shape(65536 + 32, 64, 64, 256, 8, 128),
              moe.moe_shape(65536, 64, 64, 257, 8, 128)):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_plan_noalloc(s, 1 << 20, p, 0, 0)
        assert ei.value.code == moe.MOE_ERR_SCRATCH_LIMIT
