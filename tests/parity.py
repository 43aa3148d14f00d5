"""Helpers shared by the GPU parity tests: device upload of generated inputs,
tolerances and comparisons against the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import inputs
import oracle

# Output tolerances for bf16 I/O with fp32 accumulation (maximum absolute and
# relative Frobenius error against the fp64 oracle).
MAX_ABS = 2e-2
REL_FRO = 1e-2
LSE_ABS = 2e-2
# Routing: a block whose oracle pooled score lies within NEAR_TIE of the k-th
# score may differ; at most NEAR_TIE_FRACTION of the query blocks may differ.
NEAR_TIE = 1e-4
NEAR_TIE_FRACTION = 1e-3


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def make(cfg: inputs.Config, device="cuda"):
    seg, times, _ = cfg.layout()
    q = inputs.tensor(cfg, inputs.TENSOR_Q)
    k = inputs.tensor(cfg, inputs.TENSOR_K)
    v = inputs.tensor(cfg, inputs.TENSOR_V)
    d = dict(seg=seg, times=times, q=q, k=k, v=v)
    if device is not None:
        d.update(q_d=dev_bf16(q, device), k_d=dev_bf16(k, device), v_d=dev_bf16(v, device),
                 seg_d=torch.from_numpy(seg).to(device), times_d=torch.from_numpy(times).to(device))
    return d


def compare_outputs(o_gpu_bits: np.ndarray, o_ref: np.ndarray, what: str = ""):
    """o_gpu_bits: bf16 bits [n][d]; o_ref: fp64 [n][d]."""
    o = inputs.bf16_bits_to_f64(o_gpu_bits)
    err = np.abs(o - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-300))
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {REL_FRO}"
    return max_abs, rel


def compare_routing(sel_gpu: np.ndarray, sel_ref: np.ndarray, scores: np.ndarray, kth: np.ndarray,
                    first_video_block: int, what: str = ""):
    """Sets must agree exactly except near-ties (oracle score within NEAR_TIE of the k-th)."""
    H, nv, kk = sel_ref.shape
    assert sel_gpu.shape == sel_ref.shape
    differing = 0
    for h in range(H):
        for i in range(nv):
            g = sel_gpu[h, i]
            assert np.all(np.diff(g) > 0), f"{what}: list not strictly ascending"
            assert g.min() >= first_video_block and g.max() < first_video_block + nv
            if np.array_equal(g, sel_ref[h, i]):
                continue
            differing += 1
            sym = set(g.tolist()) ^ set(sel_ref[h, i].tolist())
            for b in sym:
                s = scores[h, i, b - first_video_block]
                assert abs(s - kth[h, i]) <= NEAR_TIE, f"{what}: h{h} qb{i} block {b} score {s} kth {kth[h, i]}"
    assert differing <= NEAR_TIE_FRACTION * H * nv + 1e-9, f"{what}: {differing} of {H * nv} query blocks differ"
    return differing


def sample_rows(S: int, block_ids, rows_per_block=(0, 1, 31, 32, 62, 63)):
    rows = []
    for b in block_ids:
        for r in rows_per_block:
            x = b * 64 + r
            if x < S:
                rows.append(x)
    return np.array(sorted(set(rows)), np.int32)
