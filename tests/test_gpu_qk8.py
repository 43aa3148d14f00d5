"""Int8 QK path ("H3 SLA Attention", inputs table, use_int8_qk) through the C ABI: the quantiser's codes and
scales bit for bit against the oracle's, and the attention against the oracle's int8-QK definition."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import LSE_ABS, compare_outputs, host_bits, make, sample_rows
from test_gpu_parity import _layout

pytestmark = pytest.mark.gpu

PEN = inputs.DEFAULT_PENALTY


def _check_quant(cfg, x, heads=None, rows=None):
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"])
    q8, k8, sq, sk = h3.quantize_qk(p, x["q_d"], x["k_d"])
    torch.cuda.synchronize()
    heads = list(range(cfg.H)) if heads is None else heads
    rows = np.arange(cfg.S) if rows is None else rows
    for src, codes, scales in ((x["q"], q8, sq), (x["k"], k8, sk)):
        sub = src[heads][:, rows]
        rc, rs = oracle.quantize_rows(sub)
        gc = codes.cpu().numpy()[heads][:, rows]
        gs = scales.cpu().numpy()[heads][:, rows]
        assert np.array_equal(gc, rc)
        assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))
    stride = p.n_blocks * 64
    if stride > cfg.S:
        assert not sq.cpu().numpy()[:, cfg.S:].any() and not sk.cpu().numpy()[:, cfg.S:].any()


@pytest.mark.parametrize("d,segs", [(128, _layout(20, 30, 3, 37, 3, 41)), (64, _layout(9, 0, 2, 30, 2, 30)),
                                    (128, _layout(64, 160, 5, 100, 5, 110))])
def test_quantize_bit_exact(d, segs):
    cfg = inputs.custom(2, d, segs, seed=61, cluster_norm=2.0)
    _check_quant(cfg, make(cfg))


def test_quantize_zero_and_scaled_rows():
    """A zero row (scale 0, codes 0) and rows with a single large entry."""
    cfg = inputs.custom(1, 128, _layout(10, 0, 1, 40, 1, 40), seed=62)
    x = make(cfg, device=None)
    q = x["q"].copy()
    q[0, 3] = 0
    q[0, 5, 7] = inputs.f32_to_bf16_bits(np.float32([300.0]))[0]
    x["q"] = q
    x["q_d"] = torch.from_numpy(q.view(np.int16)).cuda().view(torch.bfloat16)
    x["k_d"] = torch.from_numpy(x["k"].view(np.int16)).cuda().view(torch.bfloat16)
    _check_quant(cfg, x)


def test_quantize_rows_with_tiny_maximum():
    """Rows whose max |x| is 2^-120 (finite 127 / max) and 2^-130 (a bf16 subnormal: 127 / max overflows in
    fp32, so nonzero elements saturate to +-127 and zeros stay 0): the kernel takes the same fp32 decisions
    as the oracle's quantiser (pinned by hand in the oracle pins)."""
    cfg = inputs.custom(1, 128, _layout(10, 0, 1, 40, 1, 40), seed=63)
    x = make(cfg, device=None)
    q = x["q"].copy()
    q[0, 2] = 0
    q[0, 2, :4] = [0x0380, 0x0300, 0x8380, 0x0000]
    q[0, 6] = 0
    q[0, 6, :4] = [0x0008, 0x8004, 0x0000, 0x0001]
    x["q"] = q
    x["q_d"] = torch.from_numpy(q.view(np.int16)).cuda().view(torch.bfloat16)
    x["k_d"] = torch.from_numpy(x["k"].view(np.int16)).cuda().view(torch.bfloat16)
    _check_quant(cfg, x)


def _qk8_all_rows(cfg, sparsity, pen, routed=True):
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    sel_d = h3.route(p, x["q_d"], x["k_d"], ws) if routed and p.n_video_blocks > 0 else None
    o, l = h3.forward_qk8(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen, kv_sel=sel_d, ws=ws,
                          lse=True)
    assert h3.check(ws) == h3.OK
    sel = None if sel_d is None else sel_d.cpu().numpy()
    ref_o, ref_l = oracle.attend_qk8(x["q"], x["k"], x["v"], x["seg"], x["times"], pen=pen, sel=sel)
    H, S, d = x["q"].shape
    compare_outputs(host_bits(o).reshape(H * S, d), ref_o, cfg.name + " int8 QK")
    assert np.abs(l.cpu().numpy().reshape(-1) - ref_l).max() <= LSE_ABS
    return x, p, sel_d, ws, o


@pytest.mark.parametrize("segs", [_layout(9, 0, 2, 30, 2, 30), _layout(20, 30, 3, 37, 3, 41),
                                  _layout(64, 160, 5, 100, 5, 110), _layout(100, 30, 3, 300, 9, 600)])
@pytest.mark.parametrize("routed", [True, False])
def test_forward_qk8_matches_int8_oracle(segs, routed):
    cfg = inputs.custom(2, 128, segs, seed=63, cluster_norm=2.0)
    _qk8_all_rows(cfg, 0.8, PEN, routed=routed)


def test_forward_qk8_no_penalty_and_close_to_bf16():
    """Without the penalty too; and the int8 output stays within a few percent of the bf16 path's."""
    cfg = inputs.custom(2, 128, _layout(64, 160, 5, 100, 5, 110), seed=64, cluster_norm=2.0)
    x, p, sel_d, ws, o8 = _qk8_all_rows(cfg, 0.8, None)
    o, _ = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=None, kv_sel=sel_d, ws=ws)
    a = inputs.bf16_bits_to_f64(host_bits(o8))
    b = inputs.bf16_bits_to_f64(host_bits(o))
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0.0 < rel <= 0.03, rel


def test_forward_qk8_full_size_sampled():
    """S = 116,883, H = 56, d = 128 at sparsity 0.90 with the penalty: sampled rows of two heads."""
    cfg = inputs.FULL_COMBINED
    x = make(cfg)
    p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=cfg.sparsities[0])
    ws = h3.workspace(p)
    sel_d = h3.route(p, x["q_d"], x["k_d"], ws)
    o, l = h3.forward_qk8(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=PEN, kv_sel=sel_d, ws=ws,
                          lse=True)
    assert h3.check(ws) == h3.OK
    heads = [0, 55]
    rows = sample_rows(cfg.S, [0, 32, 33, 500, 929, 1500, 1826])
    sel = sel_d.cpu().numpy()[heads]
    hh = np.repeat(np.arange(len(heads)), len(rows))
    rr = np.tile(rows, len(heads))
    ref_o, ref_l = oracle.attend_qk8(x["q"][heads], x["k"][heads], x["v"][heads], x["seg"], x["times"], pen=PEN,
                                     sel=sel, heads=hh, rows=rr)
    compare_outputs(host_bits(o)[heads][:, rows].reshape(-1, cfg.d), ref_o, "full size int8 QK")
    assert np.abs(l.cpu().numpy()[heads][:, rows].reshape(-1) - ref_l).max() <= LSE_ABS
