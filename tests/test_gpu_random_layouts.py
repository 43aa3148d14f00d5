"""Randomised packings: seeded random mixes of text, image-ref, audio, guide and output segments (frame counts and
sizes, d, sparsity, penalty on or off), routed and attended on the GPU and compared on every row with the oracle;
the int8-QK path too where d = 128."""
import numpy as np
import pytest

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import LSE_ABS, compare_outputs, compare_routing, host_bits, make

pytestmark = pytest.mark.gpu


def _random_config(seed):
    rng = np.random.default_rng(1000 + seed)
    segs = []
    for kind, hi in ((inputs.SEG_TEXT, 200), (inputs.SEG_IMAGE_REF, 120), (inputs.SEG_AUDIO, 150)):
        n = int(rng.integers(0, hi))
        if n and rng.random() < 0.7:
            segs.append(inputs.Segment(kind, n))
    gf = int(rng.integers(0, 7))
    if gf:
        segs.append(inputs.Segment(inputs.SEG_GUIDE, gf * int(rng.integers(10, 220)), gf))
    of = int(rng.integers(1, 9))
    segs.append(inputs.Segment(inputs.SEG_OUTPUT, of * int(rng.integers(10, 260)), of))
    d = int(rng.choice([64, 128]))
    sparsity = float(rng.choice([0.0, 0.5, 0.8, 0.9]))
    pen = inputs.DEFAULT_PENALTY if rng.random() < 0.75 else None
    cfg = inputs.custom(2, d, segs, seed=2000 + seed, cluster_norm=float(rng.choice([0.0, 2.0])))
    return cfg, sparsity, pen


@pytest.mark.parametrize("seed", range(12))
def test_random_packing(seed):
    cfg, sparsity, pen = _random_config(seed)
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel_d = sel = None
    if p.n_video_blocks > 0:
        sel_d = h3.route(p, x["q_d"], x["k_d"], ws)
        sel = sel_d.cpu().numpy()
        ref_sel, scores, kth = oracle.route(x["q"], x["k"], x["seg"], sparsity, want_scores=True)
        compare_routing(sel, ref_sel, scores, kth, p.first_video_block, f"random {seed}")
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel_d, ws=ws,
                      lse=True)
    assert h3.check(ws) == h3.OK
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=pen, sel=sel)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, f"random {seed} (S={S}, d={d}, s={sparsity})")
    assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
    if d == 128:
        o8, l8 = h3.forward_qk8(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel_d,
                                ws=ws, lse=True)
        assert h3.check(ws) == h3.OK
        ref_o8, ref_l8 = oracle.attend_qk8(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=pen, sel=sel)
        compare_outputs(host_bits(o8).reshape(H * S, d), ref_o8, f"random {seed} int8 QK")
        assert np.abs(l8.cpu().numpy().reshape(-1) - ref_l8).max() <= LSE_ABS
