"""moe_plan on the GPU vs the oracle's plan: bit-exact on every routing map."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def _run(T, H, E, k, tile, idx):
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import i32_dev
    buf = moe.MoELayerBuffers(T, H, 64, E, k, tile, identity=True)
    d_idx = i32_dev(idx.reshape(T, k)) if T > 0 else torch.zeros(1, dtype=torch.int32,
                                                                 device="cuda")
    moe.moe_plan(buf.shape, d_idx.data_ptr(), buf.plan, 0, buf.comm.cuda_stream)
    torch.cuda.synchronize()
    return buf


@pytest.mark.parametrize("name", ["tiny", "qwen3_235b_a22b", "deepseek_v3", "decode_microbatch",
                                  "dc_sweep_T65536_uniform", "dc_sweep_T65536_zipf",
                                  "dc_sweep_T1024_zipf"])
def test_plan_configs_exact(name):
    from gpu_helpers import check_plan_exact
    import combine_moe_plan_03_b200 as moe
    cfg = si.CONFIGS[name]
    for mb in range(cfg.micro_batches):
        idx, _ = si.make_routing(cfg, mb)
        buf = _run(cfg.T, cfg.H, cfg.E, cfg.k, cfg.tile, idx)
        ref = oracle.get().plan(idx, cfg.E, cfg.tile)
        check_plan_exact(buf, ref, cfg.T, cfg.k)
        assert moe.moe_get_status(buf.plan)[0] == 0
        buf.close()


EDGE = [
    # T, E, k, tile, description
    (1, 1, 1, 64, "one pair"),
    (1, 256, 8, 128, "one token, k=8"),
    (257, 3, 2, 64, "ragged chunk tail"),
    (1000, 1, 4, 128, "every pair to the single expert"),
    (513, 1024, 8, 64, "E at the maximum"),
    (300, 7, 32, 128, "k at the maximum"),
]


@pytest.mark.parametrize("T,E,k,tile,desc", EDGE, ids=[e[-1] for e in EDGE])
def test_plan_edge_exact(T, E, k, tile, desc):
    from gpu_helpers import check_plan_exact
    rng = np.random.default_rng(T * 7 + E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    buf = _run(T, 64, E, k, tile, idx)
    check_plan_exact(buf, oracle.get().plan(idx, E, tile), T, k)
    buf.close()


def test_plan_dropped_pairs_and_skew():
    from gpu_helpers import check_plan_exact
    rng = np.random.default_rng(5)
    T, E, k, tile = 2000, 64, 6, 128
    idx = rng.integers(0, 4, size=(T, k)).astype(np.int32)      # 4 hot experts, 60 empty
    idx[rng.random(idx.shape) < 0.2] = -1                       # dropped pairs
    buf = _run(T, 64, E, k, tile, idx)
    check_plan_exact(buf, oracle.get().plan(idx, E, tile), T, k)
    buf.close()


def test_plan_empty_batch():
    import combine_moe_plan_03_b200 as moe
    buf = _run(0, 64, 8, 2, 64, np.zeros((0, 2), np.int32))
    assert buf.plan_view("counts")[:8].sum().item() == 0
    assert buf.plan_view("meta")[:3].tolist() == [0, 0, 0]
    assert moe.moe_get_status(buf.plan)[0] == 0
    buf.close()


def test_plan_repeated_calls_reuse_buffers():
    """Plan buffers (and the finalize counter) are reused call after call."""
    from gpu_helpers import check_plan_exact
    import combine_moe_plan_03_b200 as moe
    T, E, k, tile = 700, 16, 4, 64
    buf = moe.MoELayerBuffers(T, 64, 64, E, k, tile, identity=True)
    from gpu_helpers import i32_dev
    for it in range(4):
        idx = np.random.default_rng(it).integers(0, E, size=(T, k)).astype(np.int32)
        d = i32_dev(idx)
        moe.moe_plan(buf.shape, d.data_ptr(), buf.plan, 0, 0)
        torch.cuda.synchronize()
        check_plan_exact(buf, oracle.get().plan(idx, E, tile), T, k)
    buf.close()


def test_plan_host_poll():
    """The one host poll: P copied to pinned host memory on the stream."""
    import combine_moe_plan_03_b200 as moe
    from gpu_helpers import i32_dev
    cfg = si.CONFIGS["qwen3_235b_a22b"]
    idx, _ = si.make_routing(cfg)
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.tile, identity=True)
    host = torch.zeros(1, dtype=torch.int32).pin_memory()
    d = i32_dev(idx)
    moe.moe_plan(buf.shape, d.data_ptr(), buf.plan, host.data_ptr(), buf.comm.cuda_stream)
    buf.comm.synchronize()
    assert int(host[0]) == oracle.get().plan(idx, cfg.E, cfg.tile)["P"]
    buf.close()
