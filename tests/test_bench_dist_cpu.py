"""bench.py's multi-rank host logic on CPU with gloo (world size 2): max-over-ranks timing,
the whole-job value, and the reference arm running on rank 0 only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (10 + r) ms for the timed region and 2 + 3r ms for one phase
        red = bench.reduce_max([10.0 + rank, 2.0 + 3 * rank], torch.device("cpu"), world)
        bench.barrier(world)
        val = bench.whole_job_tokens_per_s(world, tokens_per_step=8192, ms_per_step=red[0])
        q.put((rank, red, val))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_value_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, red, val in res:
        assert red == [11.0, 5.0]                        # max over ranks, element-wise
        assert val == pytest.approx(2 * 8192 / 0.011)   # all ranks' tokens / max time


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert rc == 0 and buf.getvalue() == ""


def test_reference_arm_line_on_rank_zero(monkeypatch):
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                         "--warmup", "1", "--ref-tokens", "8"])
    line = json.loads(buf.getvalue())
    assert rc == 0 and line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_roofline_bound_choice():
    """The bench compares a grouped GEMM with the tensor peak when each weight is used by
    more rows than the flop/byte ridge, else with HBM (weight streaming): the DeepSeek-V3
    and Qwen3 shapes (256 rows per expert) are tensor-bound, the decode micro-batches (about
    6 rows per live expert) stream weights."""
    import bench
    peaks = {"hbm_gbs": 6508.8, "bf16_tflops": 1624.0, "bf16_tflops_sustained": 1372.3}
    assert not bench.streams_weights(65536, 256, peaks)       # DeepSeek-V3-shaped layer
    assert not bench.streams_weights(32768, 128, peaks)       # Qwen3-shaped layer
    assert bench.streams_weights(1024, 170, peaks)            # a decode micro-batch
    assert bench.streams_weights(0, 0, peaks)                 # nothing routed


def test_tensor_peak_follows_the_clock_record():
    import bench
    peaks = {"hbm_gbs": 6508.8, "bf16_tflops": 1624.0, "bf16_tflops_sustained": 1372.3}
    # a short region at the maximum clock: the burst rate
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(full, 0.12, peaks, "measured")[0] == 1624.0
    # the power cap seen briefly, clock still near its maximum: burst
    brief = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(brief, 5.0, peaks, "measured")[0] == 1624.0
    # seconds under the cap with the clock held well down: sustained
    capped = {"sm_mhz": 1310.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    pk, why = bench.tensor_peak(capped, 4.0, peaks, "measured")
    assert pk == 1372.3 and "sustained" in why
    # held down, but the region is short: burst
    assert bench.tensor_peak(capped, 0.6, peaks, "measured")[0] == 1624.0
    # no clock record at all: burst
    assert bench.tensor_peak({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}, 3.0, peaks,
                             "fallback")[0] == 1624.0


def test_copy_bound_takes_the_slower_of_writes_and_all_bytes():
    import bench
    rates = {"write_v4_gbs": 4000.0, "write_bulk_gbs": 5000.0, "copy_gbs": 6000.0}
    # write-heavy (dispatch-like): the writes at the best write rate bound it
    assert abs(bench.copy_bound_ms(1e9, 9e9, rates) - 1e3 * 9e9 / 5e12) < 1e-9
    # read-heavy (combine-like): all bytes at the copy rate
    assert abs(bench.copy_bound_ms(8e9, 1e9, rates) - 1e3 * 9e9 / 6e12) < 1e-9
