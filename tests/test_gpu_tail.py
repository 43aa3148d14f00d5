"""h3attn_tail_correct (the pooled tail term, "H3 SLA Attention", inputs table, tail_correction) against the
fp64 oracle, and its exactness on blockwise-constant inputs (there the pooled term reproduces the dropped
blocks, so routed attention plus the tail is dense attention)."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import LSE_ABS, compare_outputs, dev_bf16, host_bits, make, sample_rows

pytestmark = pytest.mark.gpu


def _run(cfg, x, sparsity, pen):
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel = h3.route(p, x["q_d"], x["k_d"], ws)
    o, lse = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel, ws=ws,
                        lse=True)
    o_routed = o.clone()
    h3.tail_correct(p, x["v_d"], sel, o, lse, ws)
    torch.cuda.synchronize()
    assert h3.check(ws) == h3.OK
    return p, sel.cpu().numpy(), o, lse, o_routed


def _compare(cfg, x, p, sel, o, lse, pen, heads, rows):
    hh, rr = np.repeat(np.arange(len(heads)), len(rows)), np.tile(rows, len(heads))
    ref_o, ref_l = oracle.attend_tail(x["q"][heads], x["k"][heads], x["v"][heads], x["seg"], x["times"], pen,
                                      sel[heads], hh, rr)
    compare_outputs(host_bits(o)[heads][:, rows].reshape(-1, cfg.d), ref_o, cfg.name + " tail")
    assert np.abs(lse.cpu().numpy()[heads][:, rows].reshape(-1) - ref_l).max() <= LSE_ABS


def test_tail_routing_only():
    cfg = inputs.ROUTING_ONLY
    x = make(cfg)
    p, sel, o, lse, o_routed = _run(cfg, x, 0.85, None)
    rows = sample_rows(cfg.S, [0, 9, 10, 11, 100, 200, 255])
    _compare(cfg, x, p, sel, o, lse, None, [0, 3, 7], rows)
    # the prefix (dense) rows are untouched, the video rows changed
    assert torch.equal(o[:, :640], o_routed[:, :640]) and not torch.equal(o[:, 640:], o_routed[:, 640:])


def test_tail_with_penalty_and_ragged_tail_block():
    segs = [inputs.Segment(inputs.SEG_TEXT, 70), inputs.Segment(inputs.SEG_AUDIO, 90),
            inputs.Segment(inputs.SEG_GUIDE, 6 * 150, 6), inputs.Segment(inputs.SEG_OUTPUT, 6 * 151, 6)]
    cfg = inputs.custom(3, 128, segs, seed=41, cluster_norm=2.0, penalty=inputs.DEFAULT_PENALTY)
    x = make(cfg)
    p, sel, o, lse, _ = _run(cfg, x, 0.7, inputs.DEFAULT_PENALTY)
    assert cfg.S % 64 != 0
    rows = np.unique(np.concatenate([sample_rows(cfg.S, [0, 2, 3, 15, 16, p.n_blocks - 1]), [cfg.S - 1]]))
    _compare(cfg, x, p, sel, o, lse, inputs.DEFAULT_PENALTY, [0, 2], rows)


def test_tail_is_exact_for_blockwise_constant_inputs():
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_AUDIO, 64),
            inputs.Segment(inputs.SEG_OUTPUT, 32 * 64, 32)]
    cfg = inputs.custom(2, 128, segs, seed=5, cluster_norm=2.0)
    x = make(cfg)
    for t, key in enumerate(("q", "k", "v")):
        a = x[key].copy()
        for b in range(0, cfg.S, 64):
            a[:, b:b + 64] = a[:, b:b + 1]
        x[key] = a
        x[key + "_d"] = dev_bf16(a)
    p, sel, o, lse, o_routed = _run(cfg, x, 0.75, None)
    ws = h3.workspace(p)
    o_dense, l_dense = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=None, kv_sel=None,
                                  ws=ws, lse=True)
    diff_tail = (o.float() - o_dense.float()).abs().max().item()
    diff_routed = (o_routed.float() - o_dense.float()).abs().max().item()
    assert diff_routed > 5 * diff_tail and diff_tail < 2e-2, (diff_routed, diff_tail)
    assert (lse - l_dense).abs().max().item() < 2e-2
