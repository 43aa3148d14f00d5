"""h3attn_attend_host: the whole call from page-locked host memory, head chunks
pipelined over three streams.  Every step is independent per head, so the
result must equal the device-resident route + forward bit for bit."""
import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
import oracle
from parity import compare_outputs, make

pytestmark = pytest.mark.gpu


def _pinned(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


def _case(cfg, sparsity, pen, chunk_heads, same_stream=False):
    x = make(cfg)
    H, S, d = cfg.H, cfg.S, cfg.d
    p = h3.plan(H, S, d, x["seg"], sparsity=sparsity)
    ws = h3.workspace(p)
    routed = p.n_video_blocks > 0 and p.k < p.n_video_blocks
    # reference: device-resident call
    sel_ref = h3.route(p, x["q_d"], x["k_d"], ws) if routed else None
    o_ref, lse_ref = h3.forward(p, x["q_d"], x["k_d"], x["v_d"], x["seg_d"], x["times_d"], pen=pen,
                                kv_sel=sel_ref, ws=ws, lse=True)
    torch.cuda.synchronize()
    assert h3.check(ws) == h3.OK
    # host pipeline
    host = {t: _pinned(x[t].view(np.int16)) for t in ("q", "k", "v")}  # bf16 bits [H][S][d]
    seg_h, times_h = _pinned(x["seg"]), _pinned(x["times"])
    o_h = torch.empty((H, S, d), dtype=torch.int16).pin_memory()
    lse_h = torch.empty((H, S), dtype=torch.float32).pin_memory()
    dev = {t: torch.empty((H, S, d), dtype=torch.bfloat16, device="cuda") for t in ("q", "k", "v", "o")}
    seg_d = torch.empty(S, dtype=torch.uint8, device="cuda")
    times_d = torch.empty(S, dtype=torch.float32, device="cuda")
    lse_d = torch.empty((H, S), dtype=torch.float32, device="cuda")
    sel_d = torch.empty((H, p.n_video_blocks, p.k), dtype=torch.int32, device="cuda") if routed else None
    ws2 = h3.workspace(p)
    main = torch.cuda.Stream()
    cin = main if same_stream else torch.cuda.Stream()
    cout = main if same_stream else torch.cuda.Stream()
    h3.attend_host(p, host["q"], host["k"], host["v"], seg_h, times_h, o_h, q=dev["q"], k=dev["k"], v=dev["v"],
                   seg=seg_d, times=times_d, o=dev["o"], ws=ws2, kv_sel=sel_d, pen=pen, lse_host=lse_h, lse=lse_d,
                   chunk_heads=chunk_heads, stream=main, copy_in_stream=cin, copy_out_stream=cout)
    main.synchronize()
    assert h3.check(ws2, stream=main) == h3.OK
    got = o_h.numpy().view(np.uint16)
    ref = o_ref.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref), "host pipeline differs from the device-resident call"
    assert np.array_equal(lse_h.numpy(), lse_ref.cpu().numpy())
    if routed:
        assert np.array_equal(sel_d.cpu().numpy(), sel_ref.cpu().numpy())
    return x, p, got, sel_d


@pytest.mark.parametrize("chunk_heads", [1, 3, 8])
def test_host_pipeline_routing_only(chunk_heads):
    cfg = inputs.ROUTING_ONLY
    x, p, got, sel = _case(cfg, 0.85, None, chunk_heads)
    # and a few rows against the oracle
    heads, rows = [0, cfg.H - 1], np.array([0, 700, 5000, 16383])
    hh, rr = np.repeat(np.arange(len(heads)), len(rows)), np.tile(rows, len(heads))
    ref_o, _ = oracle.attend(x["q"][heads], x["k"][heads], x["v"][heads], x["seg"], x["times"], pen=None,
                             sel=sel.cpu().numpy()[heads], heads=hh, rows=rr)
    compare_outputs(got[heads][:, rows].reshape(-1, cfg.d), ref_o, "host pipeline")


def test_host_pipeline_dense_with_penalty_one_stream():
    segs = [inputs.Segment(inputs.SEG_TEXT, 64), inputs.Segment(inputs.SEG_AUDIO, 160),
            inputs.Segment(inputs.SEG_GUIDE, 8 * 112, 8), inputs.Segment(inputs.SEG_OUTPUT, 8 * 116, 8)]
    cfg = inputs.custom(5, 64, segs, seed=77, cluster_norm=2.0, penalty=inputs.DEFAULT_PENALTY)
    _case(cfg, 0.0, inputs.DEFAULT_PENALTY, 2, same_stream=True)
