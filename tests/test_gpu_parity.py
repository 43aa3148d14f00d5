"""GPU parity against the fp64 oracle, through the C ABI (libh3attn)."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import (LSE_ABS, compare_outputs, compare_routing, dev_bf16, host_bits, make, sample_rows)

pytestmark = pytest.mark.gpu

PEN = inputs.DEFAULT_PENALTY


def _layout(text, audio, gframes, gtok, oframes, otok):
    segs = [inputs.Segment(inputs.SEG_TEXT, text)] if text else []
    if audio:
        segs.append(inputs.Segment(inputs.SEG_AUDIO, audio))
    if gframes:
        segs.append(inputs.Segment(inputs.SEG_GUIDE, gframes * gtok, gframes))
    if oframes:
        segs.append(inputs.Segment(inputs.SEG_OUTPUT, oframes * otok, oframes))
    return segs


# ------------------------------------------------------------------ pooling

@pytest.mark.parametrize("d,segs", [
    (128, _layout(256, 384, 0, 0, 41, 384)),           # config-2 packing
    (64, _layout(20, 30, 3, 37, 3, 41)),               # ragged tail (S = 284)
    (128, _layout(1, 0, 0, 0, 0, 0)),                  # S = 1
])
def test_pool_matches_oracle(d, segs):
    cfg = inputs.custom(3, d, segs, seed=21, cluster_norm=2.0)
    x = make(cfg)
    seg = x["seg"]
    p = h3.plan(cfg.H, cfg.S, d, seg)
    got = h3.pool(p, x["k_d"]).cpu().numpy()
    ref = oracle.pool(x["k"])
    assert got.shape == ref.shape
    assert np.abs(got - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())
    if p.n_blocks > 2:
        part = h3.pool(p, x["q_d"], first_block=1, n_out=p.n_blocks - 2).cpu().numpy()
        assert np.abs(part - oracle.pool(x["q"])[:, 1:-1]).max() <= 1e-6 * max(1.0, np.abs(ref).max())


# ------------------------------------------------------------------ routing

def _route_and_compare(cfg, sparsity, heads=None):
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel = h3.route(p, x["q_d"], x["k_d"], ws).cpu().numpy()
    assert h3.check(ws) == h3.OK
    heads = list(range(cfg.H)) if heads is None else heads
    ref, scores, kth = oracle.route(x["q"][heads], x["k"][heads], x["seg"], sparsity, want_scores=True)
    compare_routing(sel[heads], ref, scores, kth, p.first_video_block, cfg.name)
    return p, x, sel, ws


def test_route_routing_only():
    _route_and_compare(inputs.ROUTING_ONLY, 0.85)


@pytest.mark.parametrize("sparsity", [0.0, 0.60, 0.85, 0.90])
def test_route_mid_clip_all_heads(sparsity):
    _route_and_compare(inputs.MID_CLIP, sparsity)


def test_route_more_than_2048_video_blocks():
    """2,100 video blocks: past the register-resident top-k (2,048), so the
    shared-memory one selects; one head, d = 64."""
    segs = _layout(64, 0, 0, 0, 30, 70 * 64)
    cfg = inputs.custom(1, 64, segs, seed=17, cluster_norm=2.0)
    p, _, _, _ = _route_and_compare(cfg, 0.9)
    assert p.n_video_blocks == 2100


def test_route_many_equal_scores():
    """Repeated key blocks make whole groups of equal pooled scores: the
    selection must still take the lowest blocks of a tied group."""
    segs = _layout(64, 0, 0, 0, 12, 64 * 20)
    cfg = inputs.custom(2, 128, segs, seed=23, cluster_norm=2.0)
    x = make(cfg, device=None)
    k = x["k"].copy()
    for b in range(1, cfg.S // 64):
        k[:, b * 64:(b + 1) * 64] = k[:, (1 + b % 7) * 64:(2 + b % 7) * 64]   # 7 distinct video key blocks
    p = h3.plan(2, cfg.S, 128, x["seg"], sparsity=0.7)
    ws = h3.workspace(p)
    sel = h3.route(p, dev_bf16(x["q"]), dev_bf16(k), ws).cpu().numpy()
    ref, _, _ = oracle.route(x["q"], k, x["seg"], 0.7)
    assert np.array_equal(sel, ref)


def test_route_tie_goes_to_lower_block():
    segs = _layout(64, 0, 0, 0, 8, 64)
    cfg = inputs.custom(2, 128, segs, seed=5, cluster_norm=2.0)
    x = make(cfg, device=None)
    k = x["k"].copy()
    k[:, 4 * 64:5 * 64] = k[:, 7 * 64:8 * 64]      # blocks 4 and 7 score identically
    p = h3.plan(2, cfg.S, 128, x["seg"], sparsity=0.5)
    ws = h3.workspace(p)
    sel = h3.route(p, dev_bf16(x["q"]), dev_bf16(k), ws).cpu().numpy()
    ref, _, _ = oracle.route(x["q"], k, x["seg"], 0.5)
    assert np.array_equal(sel, ref)


# ---------------------------------------------------------------- attention

def _forward_all_rows(cfg, sparsity, pen, routed=True, lse=True):
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel_d = None
    sel = None
    if routed and p.n_video_blocks > 0:
        sel_d = h3.route(p, x["q_d"], x["k_d"], ws)
        sel = sel_d.cpu().numpy()
        ref_sel, scores, kth = oracle.route(x["q"], x["k"], x["seg"], sparsity, want_scores=True)
        compare_routing(sel, ref_sel, scores, kth, p.first_video_block, cfg.name)
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel_d, ws=ws,
                      lse=lse)
    assert h3.check(ws) == h3.OK
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=pen, sel=sel)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, cfg.name)
    if lse:
        assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
    return x, p


RAGGED = [
    (128, _layout(0, 0, 0, 0, 1, 1)),            # S = 1
    (128, _layout(10, 0, 1, 20, 1, 33)),         # S = 63
    (64, _layout(10, 5, 1, 25, 1, 25)),          # S = 65
    (128, _layout(0, 7, 2, 30, 2, 30)),          # S = 127
    (64, _layout(9, 0, 2, 30, 2, 30)),           # S = 129
    (128, _layout(20, 30, 3, 37, 3, 41)),        # S = 284
    (128, _layout(64, 160, 5, 100, 5, 110)),     # S = 1274
]


@pytest.mark.parametrize("d,segs", RAGGED)
@pytest.mark.parametrize("pen", [None, PEN])
def test_forward_dense_ragged(d, segs, pen):
    cfg = inputs.custom(2, d, segs, seed=33, cluster_norm=0.0)
    _forward_all_rows(cfg, 0.0, pen, routed=False)


@pytest.mark.parametrize("d,segs", RAGGED[4:])
@pytest.mark.parametrize("sparsity", [0.5, 0.8])
def test_forward_routed_ragged(d, segs, sparsity):
    cfg = inputs.custom(2, d, segs, seed=44, cluster_norm=2.0)
    _forward_all_rows(cfg, sparsity, PEN, routed=True)


@pytest.mark.parametrize("sparsity", [0.5, 0.9])
def test_forward_routed_paired_groups(sparsity):
    """Odd first video block (3): the dense prefix ends on a mixed tile (2, 3)
    and the overlap pairing covers blocks 4..100, three full groups of 32 and
    one lone block; every row of both heads checked."""
    segs = _layout(100, 30, 3, 300, 9, 600)
    cfg = inputs.custom(2, 128, segs, seed=55, cluster_norm=2.0)
    _, p = _forward_all_rows(cfg, sparsity, PEN, routed=True)
    assert p.first_video_block == 3 and p.n_blocks == 101


@pytest.mark.parametrize("segs,fvb,nb", [
    (_layout(0, 0, 4, 200, 5, 230), 0, 31),        # all video: every tile is a paired one
    (_layout(100, 30, 0, 0, 1, 150), 3, 5),        # video block 3 in the mixed dense tile, block 4 alone
    (_layout(128, 0, 0, 0, 1, 40), 2, 3),          # one video block after an even prefix: a lone tile
    (_layout(64, 0, 0, 0, 1, 40), 1, 2),           # one video block inside the dense tile (0, 1)
    (_layout(70, 0, 1, 60, 1, 100), 2, 4),         # 70 prefix rows: video blocks 2 and 3 paired
])
def test_forward_routed_pairing_edges(segs, fvb, nb):
    cfg = inputs.custom(2, 64, segs, seed=57, cluster_norm=2.0)
    _, p = _forward_all_rows(cfg, 0.5, PEN, routed=True)
    assert p.first_video_block == fvb and p.n_blocks == nb


@pytest.mark.parametrize("segs,sparsity,fvb,nb,k", [
    (_layout(0, 0, 0, 0, 1, 192), 0.7, 0, 3, 1),       # all video, three blocks: a pair and a lone one-step tile
    (_layout(0, 0, 2, 300, 2, 340), 0.999, 0, 20, 1),  # all video, k = 1: tiles of one or two steps
    (_layout(100, 0, 0, 0, 1, 576), 0.95, 2, 11, 1),   # two forced blocks, k = 1
])
def test_forward_routed_single_block_lists(segs, sparsity, fvb, nb, k):
    """Routed lists of one key block: the shortest tiles (a lone query block with one step, or a pair whose
    union is one or two blocks), every row against the oracle."""
    cfg = inputs.custom(2, 128, segs, seed=58, cluster_norm=2.0)
    _, p = _forward_all_rows(cfg, sparsity, PEN, routed=True)
    assert (p.first_video_block, p.n_blocks, p.k) == (fvb, nb, k)


def test_tiny_dense_biased():
    cfg = inputs.TINY_DENSE
    x = make(cfg)
    o, l = h3.dense_biased(x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=PEN, lse=True)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=PEN)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, cfg.name)
    assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
    # same numbers through the planned entry point at sparsity 0
    _forward_all_rows(cfg, 0.0, PEN, routed=True)


def test_peaked_scores_tiny_dense():
    """Q x 4 makes the softmax peaked (max-abs binding), still within tolerance."""
    cfg = inputs.TINY_DENSE
    x = make(cfg, device=None)
    qf = inputs.bf16_bits_to_f64(x["q"]) * 4.0
    q4 = inputs.f32_to_bf16_bits(qf.astype(np.float32)).reshape(x["q"].shape)
    o, _ = h3.dense_biased(dev_bf16(q4), dev_bf16(x["k"]), dev_bf16(x["v"]), torch.from_numpy(x["seg"]).cuda(),
                           torch.from_numpy(x["times"]).cuda(), pen=PEN)
    ref_o, _ = oracle.attend(q4, x["k"], x["v"], x["seg"], x["times"], pen=PEN)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, "tiny dense peaked")


def _sampled_forward(cfg, sparsity, pen, heads, blocks, x=None):
    x = make(cfg) if x is None else x
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel_d = h3.route(p, x["q_d"], x["k_d"], ws) if sparsity > 0 else None
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel_d, ws=ws,
                      lse=True)
    assert h3.check(ws) == h3.OK
    sel = None
    if sel_d is not None:
        sel = sel_d.cpu().numpy()[heads]
        ref_sel, scores, kth = oracle.route(x["q"][heads], x["k"][heads], x["seg"], sparsity, want_scores=True)
        compare_routing(sel, ref_sel, scores, kth, p.first_video_block, cfg.name)
    rows = sample_rows(cfg.S, blocks)
    hh = np.repeat(np.arange(len(heads)), len(rows))
    rr = np.tile(rows, len(heads))
    ref_o, ref_l = oracle.attend(x["q"][heads], x["k"][heads], x["v"][heads], x["seg"], x["times"], pen=pen,
                                 sel=sel, heads=hh, rows=rr)
    og = host_bits(o)[heads][:, rows].reshape(-1, cfg.d)
    compare_outputs(og, ref_o, cfg.name)
    lg = l.cpu().numpy()[heads][:, rows].reshape(-1)
    assert np.abs(lg - ref_l).max() <= LSE_ABS
    return x, p


def test_routing_only_routed():
    cfg = inputs.ROUTING_ONLY
    _sampled_forward(cfg, 0.85, None, heads=list(range(8)), blocks=[0, 5, 9, 10, 11, 100, 200, 255])


@pytest.mark.parametrize("sparsity", [0.0, 0.60, 0.85, 0.90])
def test_mid_clip_sampled(sparsity):
    cfg = inputs.MID_CLIP
    _sampled_forward(cfg, sparsity, None, heads=[0, 31, 55], blocks=[0, 25, 26, 27, 28, 300, 600, 767])


@pytest.mark.parametrize("cfg", [inputs.FULL_DENSE, inputs.FULL_COMBINED], ids=lambda c: c.name)
def test_full_size_sampled(cfg):
    """S = 116,883, H = 56, d = 128: forced/mixed block 32, first video block 33,
    the guide/output boundary block 929, frame-straddling blocks and the 19-row tail."""
    _sampled_forward(cfg, cfg.sparsities[0], PEN, heads=[0, 55],
                     blocks=[0, 31, 32, 33, 34, 100, 500, 928, 929, 930, 1500, 1825, 1826])


def test_maximum_sequence_length():
    """The largest supported sequence, S = 524,288 (8,192 blocks; 8,182 video blocks routed to k = 819 at
    sparsity 0.9 by the shared-memory top-k), one head, d = 128, guide and output video with the penalty: routing
    of every video query block, then sampled rows of the prefix, the first video blocks, the guide/output boundary
    and the last block against the oracle."""
    segs = _layout(256, 384, 32, 8182, 32, 8182)
    cfg = inputs.custom(1, 128, segs, seed=81, cluster_norm=2.0)
    assert cfg.S == 524288
    p, x, sel, ws = _route_and_compare(cfg, 0.9)
    assert (p.n_blocks, p.n_video_blocks, p.k) == (8192, 8182, 819)
    o, l = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=PEN,
                      kv_sel=torch.from_numpy(sel).cuda(), ws=ws, lse=True)
    assert h3.check(ws) == h3.OK
    boundary = (256 + 384 + 32 * 8182) // 64
    rows = sample_rows(cfg.S, [0, 9, 10, 11, 4000, boundary, boundary + 1, 8190, 8191], rows_per_block=(0, 31, 63))
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=PEN, sel=sel,
                                 heads=np.zeros(len(rows), np.int32), rows=rows)
    compare_outputs(host_bits(o)[0, rows], ref_o, "S = 524,288")
    assert np.abs(l.cpu().numpy()[0, rows] - ref_l).max() <= LSE_ABS


def test_full_combined_routing_all_heads():
    """Workload 5 routing (S = 116,883, 1,794 video blocks, k = 180) for all 56 heads against the oracle."""
    _route_and_compare(inputs.FULL_COMBINED, inputs.FULL_COMBINED.sparsities[0])


# ---------------------------------------------------------- failure paths

def test_bounded_wait_reports_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    h3.selftest_timeout(ws, 1000)
    assert h3.check(ws) == h3.ETIMEOUT
    assert h3.check(ws) == h3.OK          # the status word was cleared


def test_corrupt_routed_list_is_flagged_not_used():
    cfg = inputs.custom(1, 128, _layout(64, 0, 0, 0, 8, 64), seed=3, cluster_norm=2.0)
    x = make(cfg)
    p = h3.plan(1, cfg.S, 128, x["seg"], sparsity=0.5)
    ws = h3.workspace(p)
    sel = h3.route(p, x["q_d"], x["k_d"], ws)
    bad = sel.clone()
    bad[0, 0, 0] = 100000                 # far outside the key blocks
    bad[0, 1, 1] = 0                      # a forced block is not a video block
    h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=None, kv_sel=bad, ws=ws)
    assert h3.check(ws) == h3.EDATA
