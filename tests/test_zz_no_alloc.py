"""h3attn_route_static: routing for callers that cannot allocate device memory.

Such a caller (a framework that owns all device memory through its own pool, a
loop that must not pay cudaMalloc's implicit synchronisation, a host with a
fixed memory budget) cannot hand over a workspace, so this entry point keeps
its pooled-centroid scratch in a fixed array inside the library.  These tests
call it through the C ABI and check it returns exactly what h3attn_route
returns, on consecutive calls: the larger problem first, then a smaller one
(which must not pick up what the larger one left in the shared array), then the
smaller one again (same result).  The status word of the static calls must read
OK afterwards."""
import ctypes

import numpy as np
import pytest
import torch

import biased_attention_video_b200 as h3
import inputs
from parity import make


def _route_static_abi(p, q, k):
    sel = torch.full((p.H, p.n_video_blocks, p.k), -1, dtype=torch.int32, device=q.device)
    rc = h3.lib().h3attn_route_static(ctypes.byref(p), q.data_ptr(), k.data_ptr(), sel.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == h3.OK, h3.lib().h3attn_strerror(rc)
    return sel


@pytest.mark.gpu
def test_route_static_matches_route_on_consecutive_calls():
    mid = inputs.MID_CLIP
    mid8 = inputs.custom(8, mid.d, mid.segments, mid.seed, cluster_norm=mid.cluster_norm)
    cases = [(mid8, 0.60), (inputs.ROUTING_ONLY, 0.85), (inputs.ROUTING_ONLY, 0.85)]
    made = {}
    results = []
    for cfg, s in cases:
        x = made.setdefault(cfg.name, make(cfg))
        p = h3.plan(cfg.H, cfg.S, cfg.d, x["seg"], sparsity=s)
        static_sel = _route_static_abi(p, x["q_d"], x["k_d"])
        assert h3.lib().h3attn_route_static_check(torch.cuda.current_stream().cuda_stream) == h3.OK
        ws = h3.workspace(p)
        ref = h3.route(p, x["q_d"], x["k_d"], ws)
        torch.cuda.synchronize()
        assert h3.check(ws) == h3.OK
        assert torch.equal(static_sel, ref), cfg.name
        results.append(static_sel.cpu().numpy())
    assert np.array_equal(results[1], results[2])


def test_route_static_rejects_problems_beyond_its_scratch():
    """Checked on the host before any device work: 56 heads x 1794 video blocks x d=128 is too large."""
    seg, _, _ = inputs.FULL_COMBINED.layout()
    p = h3.plan(56, 116883, 128, seg, sparsity=0.9)
    fake = 1 << 40
    assert h3.lib().h3attn_route_static(ctypes.byref(p), fake, fake, fake, None) == h3.EWORKSPACE
