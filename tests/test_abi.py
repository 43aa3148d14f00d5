"""C-ABI library: loads without a GPU, exports every declared symbol, host-side
plan logic and argument validation (no device work)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import biased_attention_video_b200 as h3
import inputs
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "h3attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h3attn_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    path = h3.lib_path()
    h3.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (h3attn_\w+)", out))
    decl = declared_functions()
    assert decl, "no declarations parsed"
    assert set(decl) <= exported, set(decl) - exported
    assert set(decl) == set(h3.EXPORTS)
    for name in decl:
        getattr(h3.lib(), name)


def test_library_targets_sm100a():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", h3.lib_path()], capture_output=True,
                         text=True).stdout
    assert "sm_100a" in out


@pytest.mark.parametrize("cfg", inputs.WORKLOADS, ids=lambda c: c.name)
def test_plan_matches_oracle_block_classes(cfg):
    seg, _, _ = cfg.layout()
    for s in cfg.sparsities:
        p = h3.plan(cfg.H, cfg.S, cfg.d, seg, sparsity=s)
        cls = oracle.block_classes(seg)
        assert p.n_blocks == len(cls)
        assert p.first_video_block == p.n_forced == int(cls.sum())
        assert np.all(cls[:p.first_video_block] == 1) and np.all(cls[p.first_video_block:] == 0)
        assert p.n_video_blocks == len(cls) - int(cls.sum())
        if p.n_video_blocks:
            assert p.k == oracle.k_for(p.n_video_blocks, s)


def test_plan_known_values():
    seg_full, _, _ = inputs.FULL_COMBINED.layout()
    p = h3.plan(56, 116883, 128, seg_full, sparsity=0.90)
    assert (p.n_blocks, p.first_video_block, p.n_video_blocks, p.k, p.prefix_rows) == (1827, 33, 1794, 180, 2079)
    seg_r, _, _ = inputs.ROUTING_ONLY.layout()
    p2 = h3.plan(8, 16384, 128, seg_r, sparsity=0.85)
    assert (p2.n_blocks, p2.first_video_block, p2.n_video_blocks, p2.k) == (256, 10, 246, 37)


def test_plan_rejects_bad_arguments():
    seg = np.array([0] * 10 + [4] * 100, np.uint8)
    with pytest.raises(h3.H3Error) as e:
        h3.plan(2, 110, 96, seg)
    assert e.value.code == h3.EUNSUPPORTED
    with pytest.raises(h3.H3Error) as e:
        h3.plan(2, 110, 128, seg, sparsity=1.0)
    assert e.value.code == h3.EINVAL
    with pytest.raises(h3.H3Error) as e:
        h3.plan(2, 110, 128, seg, block=128)
    assert e.value.code == h3.EUNSUPPORTED
    bad = seg.copy()
    bad[50] = 2  # audio row inside the video suffix
    with pytest.raises(h3.H3Error) as e:
        h3.plan(2, 110, 128, bad)
    assert e.value.code == h3.EUNSUPPORTED
    bad = seg.copy()
    bad[3] = 9
    with pytest.raises(h3.H3Error) as e:
        h3.plan(2, 110, 128, bad)
    assert e.value.code == h3.EINVAL


def test_plan_size_limits():
    """The largest sequence is 8,192 blocks (S = 524,288: block ids fit the kernels' 14-bit list entries and the
    lists fit shared memory); one row more, S = 0 or H = 0 is rejected before any device work."""
    S = 8192 * 64
    seg = np.concatenate([np.zeros(640, np.uint8), np.full(S - 640, 4, np.uint8)])
    p = h3.plan(1, S, 128, seg, sparsity=0.9)
    assert (p.n_blocks, p.first_video_block, p.n_video_blocks, p.k) == (8192, 10, 8182, 819)
    seg1 = np.concatenate([seg, np.full(1, 4, np.uint8)])
    with pytest.raises(h3.H3Error) as e:
        h3.plan(1, S + 1, 128, seg1)
    assert e.value.code == h3.EUNSUPPORTED
    seg0 = np.zeros(128, np.uint8)
    for H, SS in ((0, 128), (1, 0), (1, -5)):
        out = h3.Plan()
        assert h3.lib().h3attn_plan_init(ctypes.byref(out), H, SS, 128, 64, 0.0, seg0.ctypes.data) == h3.EINVAL


def test_plan_without_video_is_dense():
    seg = np.zeros(300, np.uint8)
    p = h3.plan(1, 300, 64, seg)
    assert p.n_video_blocks == 0 and p.first_video_block == p.n_blocks == 5 and p.k == 0


def test_host_validation_before_any_device_work():
    L = h3.lib()
    seg = np.array([0] * 64 + [4] * 192, np.uint8)
    p = h3.plan(1, 256, 128, seg, sparsity=0.5)
    # null tensors
    assert L.h3attn_forward(ctypes.byref(p), None, None, None, None, None, None, None, None, None, None, 0,
                            None) == h3.EINVAL
    fake = 1 << 40  # never dereferenced: validation fails first
    ws_need = L.h3attn_workspace_bytes(ctypes.byref(p))
    assert ws_need > 0
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake, None, None, fake, None, fake, 16,
                            None) == h3.EWORKSPACE
    assert L.h3attn_forward(ctypes.byref(p), fake + 2, fake, fake, fake, fake, None, None, fake, None, fake,
                            ws_need, None) == h3.EALIGN
    pen = h3.Penalty(*h3.DEFAULT_PENALTY)
    # times is read as float32 when the penalty is on; kv_sel as int32
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake + 2, ctypes.byref(pen), None, fake, None,
                            fake, ws_need, None) == h3.EALIGN
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake, ctypes.byref(pen), fake + 2, fake, None,
                            fake, ws_need, None) == h3.EALIGN
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake, None, None, fake, fake + 1, fake,
                            ws_need, None) == h3.EALIGN
    bad_pen = h3.Penalty(2.0, 0.2, 0.0, 6.0)  # falloff 0 with the penalty on
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake, ctypes.byref(bad_pen), None, fake, None,
                            fake, ws_need, None) == h3.EINVAL
    nan_pen = h3.Penalty(float("nan"), 0.2, 0.25, 6.0)
    assert L.h3attn_forward(ctypes.byref(p), fake, fake, fake, fake, fake, ctypes.byref(nan_pen), None, fake, None,
                            fake, ws_need, None) == h3.EINVAL
    assert L.h3attn_route(ctypes.byref(p), fake, fake, fake, fake, 8, None) == h3.EWORKSPACE
    assert L.h3attn_pool(ctypes.byref(p), fake, 2, 9, fake, None) == h3.EINVAL
    assert L.h3attn_dense_biased(1, 256, 80, fake, fake, fake, fake, fake, None, fake, None, fake, 1 << 20,
                                 None) == h3.EUNSUPPORTED
    # host-buffer pipeline: argument checks come before any copy or launch
    args = [fake] * 17
    assert L.h3attn_attend_host(ctypes.byref(p), *args[:5], None, *args[5:16], ws_need, 0, None, None,
                                None) == h3.EINVAL  # chunk_heads 0
    assert L.h3attn_attend_host(ctypes.byref(p), *args[:5], None, *args[5:16], ws_need, 2, None, None,
                                None) == h3.EINVAL  # chunk_heads > H
    assert L.h3attn_attend_host(ctypes.byref(p), *args[:5], None, *args[5:16], 16, 1, None, None,
                                None) == h3.EWORKSPACE
    # partition merge: counts, pointers, d
    ptrs = (ctypes.c_void_p * 9)(*([fake] * 9))
    assert L.h3attn_merge(0, ptrs, ptrs, None, 1, 64, 128, fake, None, None) == h3.EINVAL
    assert L.h3attn_merge(9, ptrs, ptrs, None, 1, 64, 128, fake, None, None) == h3.EINVAL
    assert L.h3attn_merge(2, ptrs, ptrs, None, 1, 64, 96, fake, None, None) == h3.EUNSUPPORTED
    bad_w = (ctypes.c_float * 2)(0.0, float("nan"))
    assert L.h3attn_merge(2, ptrs, ptrs, bad_w, 1, 64, 128, fake, None, None) == h3.EINVAL
    p.k = 0  # corrupt plan
    assert L.h3attn_workspace_bytes(ctypes.byref(p)) == 0
    for code in [0, -1, -2, -3, -4, -5, -6, -7, -99]:
        assert isinstance(L.h3attn_strerror(code), bytes)


def test_plan_k_matches_oracle_for_decimal_sparsities():
    """k = ceil((1 - sparsity) nV) read in double precision: 0.9 of 2,100 video
    blocks keeps 210 (a float 0.9 would give 211)."""
    import oracle
    for nv, sp in [(2100, 0.9), (1794, 0.9), (100, 0.85), (7, 0.5), (8000, 0.95), (3, 0.0)]:
        S = 64 + nv * 64
        seg = np.array([0] * 64 + [4] * (nv * 64), np.uint8)
        p = h3.plan(1, S, 64, seg, sparsity=sp)
        assert p.n_video_blocks == nv
        assert p.k == oracle.k_for(nv, sp), (nv, sp, p.k)
    assert h3.plan(1, 64 + 2100 * 64, 64, np.array([0] * 64 + [4] * 2100 * 64, np.uint8), sparsity=0.9).k == 210


def test_qk8_validation_before_any_device_work():
    L = h3.lib()
    fake = 1 << 40  # never dereferenced: validation fails first
    seg = np.array([0] * 64 + [4] * 192, np.uint8)
    p64 = h3.plan(1, 256, 64, seg, sparsity=0.5)
    need = L.h3attn_qk8_workspace_bytes(ctypes.byref(p64))
    assert need >= 2 * 256 * 64 + 2 * 256 * 4
    assert L.h3attn_forward_qk8(ctypes.byref(p64), fake, fake, fake, fake, None, None, None, fake, None, fake,
                                1 << 30, fake, need, None) == h3.EUNSUPPORTED
    p = h3.plan(1, 256, 128, seg, sparsity=0.5)
    need = L.h3attn_qk8_workspace_bytes(ctypes.byref(p))
    assert L.h3attn_quantize_qk(ctypes.byref(p), None, fake, fake, need, None) == h3.EINVAL
    assert L.h3attn_quantize_qk(ctypes.byref(p), fake, fake, fake, need - 1, None) == h3.EWORKSPACE
    assert L.h3attn_quantize_qk(ctypes.byref(p), fake + 2, fake, fake, need, None) == h3.EALIGN
    assert L.h3attn_forward_qk8(ctypes.byref(p), fake, fake, fake, fake, None, None, None, fake, None, fake,
                                1 << 30, fake, 16, None) == h3.EWORKSPACE
