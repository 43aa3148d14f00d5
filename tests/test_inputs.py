"""The seeded input recipe: determinism, row-wise regeneration, layouts."""
import numpy as np

import inputs


def test_counter_based_rows_match_full_tensor():
    cfg = inputs.ROUTING_ONLY
    small = inputs.custom(3, cfg.d, cfg.segments, cfg.seed, cluster_norm=2.0)
    full = inputs.tensor(small, inputs.TENSOR_K, h0=0, nh=3, row0=600, nrows=300)
    again = inputs.tensor(small, inputs.TENSOR_K, h0=0, nh=3, row0=600, nrows=300)
    assert np.array_equal(full, again)
    rows = inputs.rows(small, inputs.TENSOR_K, 2, [600, 777, 899])
    assert np.array_equal(rows, full[2, [0, 177, 299]])


def test_tensors_differ_by_id_and_seed():
    cfg = inputs.custom(1, 64, [inputs.Segment(inputs.SEG_TEXT, 128)], seed=5)
    q = inputs.tensor(cfg, 0)
    k = inputs.tensor(cfg, 1)
    q2 = inputs.tensor(cfg, 0, seed=6)
    assert not np.array_equal(q, k) and not np.array_equal(q, q2)


def test_normal_statistics():
    cfg = inputs.custom(2, 128, [inputs.Segment(inputs.SEG_TEXT, 4096)], seed=3)
    x = inputs.bf16_bits_to_f64(inputs.tensor(cfg, 2))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_cluster_mean_shared_by_frame_and_norm():
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_OUTPUT, 4 * 2000, 4)]
    cfg = inputs.custom(1, 128, segs, seed=9, cluster_norm=2.0)
    q = inputs.bf16_bits_to_f64(inputs.tensor(cfg, 0))[0]
    k = inputs.bf16_bits_to_f64(inputs.tensor(cfg, 1))[0]
    v = inputs.bf16_bits_to_f64(inputs.tensor(cfg, 2))[0]
    for f in range(4):
        rows = slice(64 + f * 2000, 64 + (f + 1) * 2000)
        cq, ck = q[rows].mean(0), k[rows].mean(0)
        assert abs(np.linalg.norm(cq) - 2.0) < 0.4      # noise norm ~ sqrt(128/2000)
        assert np.linalg.norm(cq - ck) < 0.7            # same mean added to Q and K
        assert np.linalg.norm(v[rows].mean(0)) < 0.5    # V has no cluster mean
    assert np.linalg.norm(q[:64].mean(0)) < 2.0         # prefix rows: no mean (noise ~1.41)


def test_workload_layouts():
    for cfg, S in zip(inputs.WORKLOADS, (2048, 16384, 49152, 116883, 116883)):
        seg, times, frame = cfg.layout()
        assert cfg.S == S and len(seg) == S
        video = np.where((seg == 3) | (seg == 4))[0]
        assert video[0] == S - len(video)            # video rows are a contiguous suffix
        assert np.all(times[seg < 3] == 0.0)
    seg, times, frame = inputs.FULL_COMBINED.layout()
    assert list(np.bincount(seg, minlength=5)) == [256, 1013, 810, 57402, 57402]
    g = np.where(seg == 3)[0]
    o = np.where(seg == 4)[0]
    assert times[g[0]] == 0.0 and abs(times[g[-1]] - 26 * 4 / 24) < 1e-6
    assert np.array_equal(times[g], times[o])     # matching temporal grids
    seg1, t1, _ = inputs.TINY_DENSE.layout()
    assert list(np.bincount(seg1, minlength=5)) == [64, 0, 160, 896, 928]


def test_bf16_round_trip():
    x = np.array([1.0, -2.5, 3.14159, 1e-3, 65504.0], np.float32)
    b = inputs.f32_to_bf16_bits(x)
    y = inputs.bf16_bits_to_f64(b)
    assert np.all(np.abs(y - x) <= np.abs(x) * 2 ** -8)
