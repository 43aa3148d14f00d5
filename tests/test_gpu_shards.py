"""Head-sharded call (the multi-GPU split of "H3 SLA Attention", "How it works": the quoted speed-up is an
eight-GPU figure): every step of the path is independent per head, so N ranks each route and attend a
contiguous range of heads with no collective.  On one GPU the shards run in sequence through the C ABI,
each with a plan of its own head count and Q/K/V/O/kv_sel pointers offset by its first head; the
assembled result must match the oracle (routing and outputs) exactly as an unsharded call does."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from bench import head_range
from parity import LSE_ABS, compare_outputs, compare_routing, host_bits, make, sample_rows

pytestmark = pytest.mark.gpu


def _segs(text, audio, gframes, gtok, oframes, otok):
    segs = [inputs.Segment(inputs.SEG_TEXT, text)] if text else []
    if audio:
        segs.append(inputs.Segment(inputs.SEG_AUDIO, audio))
    if gframes:
        segs.append(inputs.Segment(inputs.SEG_GUIDE, gframes * gtok, gframes))
    segs.append(inputs.Segment(inputs.SEG_OUTPUT, oframes * otok, oframes))
    return segs


def _sharded_call(cfg, x, sparsity, pen, n):
    H, S, d = cfg.H, cfg.S, cfg.d
    p_full = h3.plan(H, S, d, x["seg"], sparsity=sparsity)
    sel_all = torch.empty((H, p_full.n_video_blocks, p_full.k), dtype=torch.int32, device="cuda")
    o_all = torch.empty((H, S, d), dtype=torch.bfloat16, device="cuda")
    lse_all = torch.empty((H, S), dtype=torch.float32, device="cuda")
    covered = np.zeros(H, int)
    for rank in range(n):
        h0, nh = head_range(H, n, rank)
        covered[h0:h0 + nh] += 1
        p = h3.plan(nh, S, d, x["seg"], sparsity=sparsity)
        ws = h3.workspace(p)
        # contiguous views at head h0: the pointers a rank holding only these heads would pass
        q, k, v = x["q_d"][h0:h0 + nh], x["k_d"][h0:h0 + nh], x["v_d"][h0:h0 + nh]
        sel = h3.route(p, q, k, ws, kv_sel=sel_all[h0:h0 + nh])
        h3.forward(p, q, k, v, x["seg_d"], x["times_d"], pen=pen, kv_sel=sel, ws=ws, out=o_all[h0:h0 + nh],
                   lse=lse_all[h0:h0 + nh])
        assert h3.check(ws) == h3.OK
    assert np.all(covered == 1)
    return p_full, sel_all.cpu().numpy(), o_all, lse_all


@pytest.mark.parametrize("n", [2, 3])
def test_head_shards_routing_only_workload(n):
    """Workload 2's shape (S = 16,384, H = 8, d = 128, sparsity 0.85): routing of every head and sampled
    rows of every head against the oracle."""
    cfg = inputs.ROUTING_ONLY
    x = make(cfg)
    p, sel, o, lse = _sharded_call(cfg, x, 0.85, None, n)
    ref, scores, kth = oracle.route(x["q"], x["k"], x["seg"], 0.85, want_scores=True)
    compare_routing(sel, ref, scores, kth, p.first_video_block, f"{n} shards")
    rows = sample_rows(cfg.S, [0, 9, 10, 11, 100, 200, 255])
    hh = np.repeat(np.arange(cfg.H), len(rows))
    rr = np.tile(rows, cfg.H)
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=None, sel=sel, heads=hh, rows=rr)
    compare_outputs(host_bits(o)[:, rows].reshape(-1, cfg.d), ref_o, f"{n} shards")
    assert np.abs(lse.cpu().numpy()[:, rows].reshape(-1) - ref_l).max() <= LSE_ABS


@pytest.mark.parametrize("n", [2, 3])
@pytest.mark.parametrize("seed", [71, 72])
def test_head_shards_random_packing(n, seed):
    """A seeded random packing with guide and output video and the default penalty, 5 heads: every row."""
    rng = np.random.default_rng(seed)
    segs = _segs(int(rng.integers(1, 200)), int(rng.integers(0, 150)), int(rng.integers(2, 5)),
                 int(rng.integers(20, 90)), int(rng.integers(2, 5)), int(rng.integers(20, 90)))
    cfg = inputs.custom(5, 128, segs, seed=seed, cluster_norm=2.0, penalty=inputs.DEFAULT_PENALTY)
    x = make(cfg)
    sparsity = 0.6
    p, sel, o, lse = _sharded_call(cfg, x, sparsity, inputs.DEFAULT_PENALTY, n)
    if p.n_video_blocks > 0:
        ref, scores, kth = oracle.route(x["q"], x["k"], x["seg"], sparsity, want_scores=True)
        compare_routing(sel, ref, scores, kth, p.first_video_block, f"{n} shards")
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=inputs.DEFAULT_PENALTY,
                                 sel=sel if p.n_video_blocks > 0 else None)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, f"{n} shards")
    assert np.abs(lse.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
