"""bench.py's host-side legs on CPU: the bounded oracle sample behind `cpu_baseline` and the
reference arm's JSON line (the fp64 oracle timed on the host cores)."""
import argparse
import contextlib
import io
import json

import numpy as np
import pytest

import bench
import inputs


def _small(prefix=True):
    segs = [inputs.Segment(inputs.SEG_TEXT, 70), inputs.Segment(inputs.SEG_AUDIO, 50)] if prefix else []
    segs += [inputs.Segment(inputs.SEG_GUIDE, 4 * 40, 4), inputs.Segment(inputs.SEG_OUTPUT, 4 * 44, 4)]
    cfg = inputs.custom(2, 64, segs, seed=21, cluster_norm=2.0, penalty=inputs.DEFAULT_PENALTY, sparsities=(0.5,))
    seg, times, _ = cfg.layout()
    q, k, v = (inputs.tensor(cfg, t) for t in range(3))
    return cfg, seg, times, q, k, v


@pytest.mark.parametrize("prefix", [True, False])
def test_oracle_sample_covers_every_block_once_when_the_budget_allows(prefix):
    """Every block's eight rows exactly once, also when the edge blocks coincide (no prefix)."""
    cfg, seg, times, q, k, v = _small(prefix)
    flops, secs, desc, rows = bench.oracle_sample(cfg, q, k, v, seg, times, cfg.penalty, 0.5, budget_s=60.0)
    n_blocks = (cfg.S + 63) // 64
    # eight rows of every block (fewer in a ragged last block)
    last_rows = sum(1 for r in (0, 9, 18, 27, 36, 45, 54, 63) if (n_blocks - 1) * 64 + r < cfg.S)
    assert rows == 8 * (n_blocks - 1) + last_rows
    assert flops > 0 and secs > 0
    assert f"{rows} sampled query rows" in desc


def test_oracle_sample_stops_at_its_budget():
    cfg, seg, times, q, k, v = _small()
    _, _, _, rows = bench.oracle_sample(cfg, q, k, v, seg, times, cfg.penalty, 0.5, budget_s=0.0)
    assert rows == 0


def test_reference_arm_prints_one_line_with_the_contract_keys():
    args = argparse.Namespace(gpus=1, steps=1, warmup=3)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(args, 0, 1)
    lines = [ln for ln in out.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and np.isfinite(d["value"])
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # other ranks print nothing
    out2 = io.StringIO()
    with contextlib.redirect_stdout(out2):
        bench.run_reference(args, 1, 2)
    assert out2.getvalue() == ""


class _Plan:
    """The three plan fields the executed-work count reads."""

    def __init__(self, H, n_blocks, first_video_block):
        self.H, self.n_blocks, self.first_video_block = H, n_blocks, first_video_block


def test_executed_work_of_a_dense_plan():
    """Every 128-row tile walks every 64-key block."""
    p = _Plan(3, 37, 0)
    assert bench.executed_mma_pairs(p, None) == 3 * 19 * 37 * 128 * 64


@pytest.mark.parametrize("fvb", [0, 3, 4])
def test_executed_work_when_every_list_is_the_same(fvb):
    """Identical routed lists: every pair's union is the list itself, so a paired tile walks the k routed blocks
    plus the forced ones; the dense prefix tiles (adjacent pairs up to an even block) walk every block."""
    H, nb, k = 2, 90, 7
    nv = nb - fvb
    rng = np.random.default_rng(5)
    lst = np.sort(rng.choice(nv, k, replace=False)) + fvb
    sel = np.broadcast_to(lst, (H, nv, k)).astype(np.int32)
    n_dense = (fvb + 1) // 2
    first = 2 * n_dense
    n_paired_rows = nb - first
    tiles = n_paired_rows // 2 + n_paired_rows % 2
    expect = H * (n_dense * nb + tiles * (k + fvb)) * 128 * 64
    assert bench.executed_mma_pairs(_Plan(H, nb, fvb), sel) == expect


def test_executed_work_of_disjoint_pairs():
    """Two video query blocks with disjoint lists: their tile walks both lists (2k blocks)."""
    H, nb, k = 1, 2, 1
    sel = np.array([[[0], [1]]], np.int32)
    assert bench.executed_mma_pairs(_Plan(H, nb, 0), sel) == 2 * k * 128 * 64
