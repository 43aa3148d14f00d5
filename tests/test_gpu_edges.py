"""GPU parity at the method's edges, through the C ABI (libh3attn), every row against the fp64 oracle.

- The temporal-penalty controls ("Flash Partitions for H3 native temporal alignment", section 1): the
  five (strength, window, falloff, cap) settings the oracle's own pins use, and the reductions of
  section 4 (strength 0 or cap 0 removes the penalty) plus a zero window.
- Times off the latent-frame grid: a gap exactly at the window (no penalty), gaps at the saturation
  point window + falloff sqrt(cap / strength), and many distinct guide times inside one key block (the
  kernel's per-key path).
- The attention kernel's own give-up path: with every wait bounded to one poll the call must report
  H3ATTN_ETIMEOUT, and the next call on the same workspace must be correct again.
"""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import LSE_ABS, compare_outputs, compare_routing, host_bits, make

pytestmark = pytest.mark.gpu

PINNED = [(2.0, 0.20, 0.25, 6.0), (0.5, 0.1, 0.3, 3.0), (8.0, 0.2, 0.25, 12.0), (2.0, 0.0, 0.25, 1.0),
          (2.0, 0.2, 0.05, 6.0)]
REDUCTIONS = [(0.0, 0.2, 0.25, 6.0), (2.0, 0.2, 0.25, 0.0), (2.0, 0.0, 0.25, 6.0)]


def _segs(text, audio, gframes, gtok, oframes, otok):
    segs = [inputs.Segment(inputs.SEG_TEXT, text)] if text else []
    if audio:
        segs.append(inputs.Segment(inputs.SEG_AUDIO, audio))
    segs.append(inputs.Segment(inputs.SEG_GUIDE, gframes * gtok, gframes))
    segs.append(inputs.Segment(inputs.SEG_OUTPUT, oframes * otok, oframes))
    return segs


LAYOUTS = [(128, _segs(20, 30, 3, 37, 3, 41)),      # S = 284: frames straddle blocks, ragged last block
           (64, _segs(64, 160, 5, 100, 5, 110))]    # S = 1274


def _check(cfg, x, times, pen, sparsity):
    """Route (sparsity > 0) and attend on the GPU with the given times; compare every row."""
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel_d, sel = None, None
    if sparsity > 0 and p.n_video_blocks > 0:
        sel_d = h3.route(p, x["q_d"], x["k_d"], ws)
        sel = sel_d.cpu().numpy()
        ref_sel, scores, kth = oracle.route(x["q"], x["k"], x["seg"], sparsity, want_scores=True)
        compare_routing(sel, ref_sel, scores, kth, p.first_video_block, cfg.name)
    times_d = torch.from_numpy(np.ascontiguousarray(times, np.float32)).cuda()
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], times_d, pen=pen, kv_sel=sel_d, ws=ws, lse=True)
    assert h3.check(ws) == h3.OK
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], times, pen=pen, sel=sel)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, f"{cfg.name} pen={pen}")
    assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS


@pytest.mark.parametrize("pen", PINNED + REDUCTIONS)
@pytest.mark.parametrize("d,segs", LAYOUTS)
@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_penalty_controls_every_row(pen, d, segs, sparsity):
    cfg = inputs.custom(2, d, segs, seed=61, cluster_norm=2.0)
    x = make(cfg)
    _check(cfg, x, x["times"], pen, sparsity)


@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_gap_exactly_at_the_window(sparsity):
    """Window 0.25 s; guide frames at 0, 0.5, 1.0 s and output frames at 0.25, 0.75, 1.25 s: every
    gap is an exact binary fraction, among them exactly the window (penalty 0 on both sides of it)."""
    cfg = inputs.custom(2, 128, _segs(40, 0, 3, 40, 3, 44), seed=62, cluster_norm=2.0)
    x = make(cfg)
    seg, _, frame = cfg.layout()
    times = np.zeros(cfg.S, np.float32)
    times[seg == inputs.SEG_GUIDE] = 0.5 * frame[seg == inputs.SEG_GUIDE]
    times[seg == inputs.SEG_OUTPUT] = 0.25 + 0.5 * frame[seg == inputs.SEG_OUTPUT]
    pen = (2.0, 0.25, 0.25, 6.0)
    dts = np.abs(times[seg == inputs.SEG_OUTPUT][:, None] - times[seg == inputs.SEG_GUIDE][None, :])
    assert np.any(dts == np.float32(0.25))
    _check(cfg, x, times, pen, sparsity)


@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_gap_at_the_saturation_point(sparsity):
    """Default controls: dt* = 0.20 + 0.25 sqrt(3) = 0.6330127 s, where the penalty reaches its cap;
    output frames at dt* and dt* -/+ 1 ms from a guide frame at 0."""
    cfg = inputs.custom(2, 128, _segs(40, 0, 2, 60, 3, 44), seed=63, cluster_norm=2.0)
    x = make(cfg)
    seg, _, frame = cfg.layout()
    dstar = 0.20 + 0.25 * np.sqrt(3.0)
    times = np.zeros(cfg.S, np.float32)
    times[seg == inputs.SEG_GUIDE] = 2.0 * frame[seg == inputs.SEG_GUIDE]   # frames at 0 s and 2 s
    times[seg == inputs.SEG_OUTPUT] = (dstar + np.array([-1e-3, 0.0, 1e-3]))[frame[seg == inputs.SEG_OUTPUT]]
    _check(cfg, x, times, inputs.DEFAULT_PENALTY, sparsity)


@pytest.mark.parametrize("pen", [inputs.DEFAULT_PENALTY, (8.0, 0.2, 0.25, 12.0)])
@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_many_guide_times_in_one_block(pen, sparsity):
    """Every guide row at its own time (seeded, 0..1.5 s): each guide key block holds many times, so the
    kernel takes its per-key penalty path on every such block."""
    cfg = inputs.custom(2, 128, _segs(64, 0, 4, 96, 4, 100), seed=64, cluster_norm=2.0)
    x = make(cfg)
    seg = x["seg"]
    times = x["times"].copy()
    g = seg == inputs.SEG_GUIDE
    times[g] = np.random.default_rng(65).uniform(0.0, 1.5, int(g.sum())).astype(np.float32)
    _check(cfg, x, times, pen, sparsity)


def test_attention_gives_up_and_recovers():
    """Every wait of the attention kernel bounded to one poll: the waits run out, the kernel drains its
    own loads and MMAs, releases TMEM and records H3ATTN_ETIMEOUT; with the default bound restored, the
    next call on the same workspace matches the oracle."""
    cfg = inputs.TINY_DENSE
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"])
    ws = h3.workspace(p)
    try:
        h3.set_wait_polls(1)
        h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=inputs.DEFAULT_PENALTY, ws=ws)
        assert h3.check(ws) == h3.ETIMEOUT
    finally:
        h3.set_wait_polls(0)
    assert h3.check(ws) == h3.OK
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=inputs.DEFAULT_PENALTY,
                      ws=ws, lse=True)
    assert h3.check(ws) == h3.OK
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=inputs.DEFAULT_PENALTY)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, "after give-up")
    assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
