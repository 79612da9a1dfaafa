"""The seeded input generator: determinism, random access, distributions, routing."""
import numpy as np

import synth_inputs as si


def test_bits_are_splitmix64_outputs():
    # SplitMix64 seeded with key: output i = mix(key + (i+1)*golden)
    M = (1 << 64) - 1

    def mix(z):
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9 & M
        z = (z ^ (z >> 27)) * 0x94D049BB133111EB & M
        return z ^ (z >> 31)

    seed, stream = 0x5EED0002, 7
    key = mix(seed ^ (stream * 0xD1B54A32D192ED03 & M))
    want = [mix((key + (i + 1) * 0x9E3779B97F4A7C15) & M) for i in range(5, 12)]
    np.testing.assert_array_equal(si.bits(seed, stream, 5, 7), np.array(want, np.uint64))


def test_random_access_and_determinism():
    a = si.normal_bf16(123, 2, 0, 10001, 0.1)
    b = si.normal_bf16(123, 2, 0, 10001, 0.1)
    np.testing.assert_array_equal(a, b)
    for first in (0, 1, 2, 777, 9998):
        np.testing.assert_array_equal(si.normal_bf16(123, 2, first, 3, 0.1), a[first:first + 3])
    assert not np.array_equal(a, si.normal_bf16(124, 2, 0, 10001, 0.1))
    assert not np.array_equal(a, si.normal_bf16(123, 3, 0, 10001, 0.1))


def test_normal_moments():
    z = si.normal_f64(7, 1, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    w = si.bf16_to_f64(si.normal_bf16(7, 1, 0, 200000, 0.25))
    assert abs(w.std() - 0.25) < 0.003


def test_bf16_rounding_matches_torch():
    import torch
    v = si.normal_f32(3, 1, 0, 5000) * 3.7
    mine = si.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)


def test_softmax_router():
    cfg = si.CONFIGS["deepseek_v3"]
    small = si.custom("s", T=64, H=8, I=8, E=cfg.E, k=8, tile=128, seed=cfg.seed,
                      routing="softmax_bias")
    idx, w = si.make_routing(small)
    assert idx.shape == (64, 8) and w.dtype == np.float32
    np.testing.assert_allclose(w.sum(1), 1, rtol=1e-6)
    assert all(len(set(r)) == 8 for r in idx)
    assert np.all(np.diff(w, axis=1) <= 0)          # largest probability first
    # the choice is the top-k of the biased softmax
    logits = si.normal_f32(cfg.seed, si.STREAM_LOGITS, 0, 64 * cfg.E).reshape(64, cfg.E)
    bias = si.normal_f32(cfg.seed, si.STREAM_BIAS, 0, cfg.E, 0.5)
    l = logits.astype(np.float32) + bias
    top = np.argsort(-l.astype(np.float64), axis=1, kind="stable")[:, :8]
    np.testing.assert_array_equal(idx, top)


def test_zipf_router_is_skewed_and_distinct():
    cfg = si.CONFIGS["decode_microbatch"]
    idx, w = si.make_routing(cfg, 0)
    assert idx.shape == (128, 8)
    assert all(len(set(r)) == 8 for r in idx)
    np.testing.assert_allclose(w.sum(1), 1, rtol=1e-6)
    counts = np.bincount(idx.reshape(-1), minlength=cfg.E)
    assert (counts == 0).sum() > 50                 # many experts stay empty
    assert counts.max() >= 64                       # a few are hot
    # micro-batches continue one long draw
    idx1, _ = si.make_routing(cfg, 1)
    big = si.router_zipf(256, 0, cfg.E, cfg.k, cfg.alpha, cfg.seed)[0]
    np.testing.assert_array_equal(big[128:], idx1)


def test_config_shapes():
    c = si.CONFIGS["deepseek_v3"]
    assert (c.T, c.H, c.I, c.E, c.k, c.tile) == (8192, 7168, 2048, 256, 8, 128)
    assert c.pool_rows_max() == 65536 + 256 * 127
    x = si.make_x(si.CONFIGS["tiny"])
    assert x.shape == (256, 256) and x.dtype == np.uint16
    rows = si.make_x_rows(si.CONFIGS["tiny"], np.array([3, 200]))
    np.testing.assert_array_equal(rows, x[[3, 200]])


def test_dy_stream_is_seeded_normal_and_independent_of_x():
    """The backward's upstream gradient: its own seeded stream, N(0, 1) in bf16, the same
    bits on every call, different from x of the same workload, one slice per micro-batch."""
    import numpy as np
    import synth_inputs as si
    cfg = si.custom("dy", T=256, H=256, I=128, E=4, k=2, tile=64, seed=77, micro_batches=2)
    a, b = si.make_dy(cfg), si.make_dy(cfg)
    assert a.dtype == np.uint16 and a.shape == (256, 256) and np.array_equal(a, b)
    assert not np.array_equal(a, si.make_x(cfg))
    assert not np.array_equal(a, si.make_dy(cfg, 1))
    v = si.bf16_to_f64(a)
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.02
