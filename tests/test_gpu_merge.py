"""h3attn_merge (the Flash-Partitions merge, "Flash Partitions for H3 native temporal alignment", section 4)
against the fp64 oracle merge, and composed with the routed forward: attention over two disjoint key-block
sets merged equals attention over their union."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import LSE_ABS, compare_outputs, dev_bf16, host_bits, make

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,n,log_w", [(128, 1, None), (128, 3, [0.0, -1.5, 0.7]), (64, 2, [0.0, -np.inf]),
                                       (128, 8, None)])
def test_merge_matches_oracle(d, n, log_w):
    rng = np.random.default_rng(11 + n)
    H, S = 3, 777
    o_bits = [inputs.f32_to_bf16_bits(rng.normal(size=(H, S, d)).astype(np.float32)) for _ in range(n)]
    lse = [rng.normal(0, 4, size=(H, S)).astype(np.float32) for _ in range(n)]
    lse[0][1, 5] = -np.inf                       # one partition attended nothing for this row
    o_d = [dev_bf16(b) for b in o_bits]
    l_d = [torch.from_numpy(x).cuda() for x in lse]
    o, l = h3.merge(o_d, l_d, log_w=log_w, lse=True)
    ref_o, ref_l = oracle.merge(np.stack([inputs.bf16_bits_to_f64(b).reshape(H * S, d) for b in o_bits]),
                                np.stack([x.astype(np.float64).reshape(-1) for x in lse]),
                                None if log_w is None else np.array(log_w, np.float64).astype(np.float32))
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, "merge")
    lg = l.cpu().numpy().reshape(-1).astype(np.float64)
    assert np.array_equal(np.isneginf(lg), np.isneginf(ref_l))   # rows that attended nothing
    fin = np.isfinite(ref_l)
    assert np.abs(lg[fin] - ref_l[fin]).max() <= 1e-4


def test_merge_in_place_and_nothing_attended():
    H, S, d = 1, 64, 128
    o0 = torch.randn(H, S, d, device="cuda").to(torch.bfloat16)
    keep = o0.clone()
    l0 = torch.full((H, S), -float("inf"), device="cuda")
    o, l = h3.merge([o0], [l0], out=o0, lse=True)
    assert o.data_ptr() == o0.data_ptr()
    assert torch.all(o.float() == 0) and torch.all(torch.isinf(l)) and not torch.equal(keep, o0)


def _all_video_case(H=2, n_frames=8, d=128):
    segs = [inputs.Segment(inputs.SEG_OUTPUT, n_frames * 512, n_frames)]
    return inputs.custom(H, d, segs, seed=31, cluster_norm=2.0)


def test_forward_over_disjoint_halves_merges_to_dense():
    """No prefix rows, so every query block attends exactly its routed list: two lists splitting the key
    blocks in halves give two disjoint partitions whose merge is the dense attention."""
    cfg = _all_video_case()
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=0.5)
    nv = p.n_video_blocks
    assert p.first_video_block == 0 and p.k == nv // 2
    ws = h3.workspace(p)
    halves = []
    for lo in (0, nv // 2):
        sel = torch.arange(lo, lo + p.k, dtype=torch.int32, device="cuda").expand(cfg.H, nv, p.k).contiguous()
        halves.append(h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=None, kv_sel=sel,
                                 ws=ws, lse=True))
    o_m, l_m = h3.merge([h[0] for h in halves], [h[1] for h in halves], lse=True)
    o_dense, l_dense = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=None, kv_sel=None,
                                  ws=ws, lse=True)
    assert h3.check(ws) == h3.OK
    # both against the oracle's dense attention on sampled rows
    rows = np.array([0, 1, 63, 64, 1000, 2047, 2048, 4095])
    hh, rr = np.repeat(np.arange(cfg.H), len(rows)), np.tile(rows, cfg.H)
    ref_o, ref_l = oracle.attend(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=None, sel=None, heads=hh, rows=rr)
    for o, l, what in ((o_m, l_m, "merged halves"), (o_dense, l_dense, "dense")):
        compare_outputs(host_bits(o)[:, rows].reshape(-1, cfg.d), ref_o, what)
        assert np.abs(l.cpu().numpy()[:, rows].reshape(-1) - ref_l).max() <= LSE_ABS
    # and the merged normaliser is the dense one up to fp32 rounding
    assert torch.allclose(l_m, l_dense, atol=1e-4, rtol=0)
