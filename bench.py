"""Benchmark of one call of the hot path: block routing (pool + pooled score +
top-k) followed by the fused biased attention over the routed tiles, at the
full H3 packing S = 116,883, H = 56, d = 128, sparsity 0.90, default temporal
penalty (workload "full combined").

Prints one JSON line.  value = effective attention TFLOP/s over all ranks
(4*d FLOPs per attended (query, key, head) triple, valid pairs only) with the
inputs resident in HBM; e2e = the same metric through the C ABI with host
buffers (h3attn_attend_host: host->device copy of Q, K, V, seg, times and
device->host copy of O inside the timed region, pipelined per chunk of heads).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: torchrun, one process per GPU; every rank runs its own independent
call (its own seeded input), no collective on the data path (weak scaling).
The reference arm times the fp64 CPU oracle on a bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import inputs  # noqa: E402

WORKLOAD = "full combined: S=116883 (text 256|image-ref 1013|audio 810|guide 27x2126|output 27x2126), " \
           "H=56, d=128, bf16, block 64, sparsity 0.90 (k=180 of 1794 video KV blocks), default penalty"
WORKLOAD_DENSE = "full dense biased: S=116883 (text 256|image-ref 1013|audio 810|guide 27x2126|output 27x2126), " \
                 "H=56, d=128, bf16, sparsity 0 (every key), default penalty"
METRIC = "effective attention TFLOP/s (S=116883, H=56, d=128, sparsity 0.90, penalty on)"
METRIC_DENSE = "effective attention TFLOP/s (S=116883, H=56, d=128, dense, penalty on)"


# DRAM bytes of one attn_kernel launch as ncu counted them (dram__bytes_read.sum + dram__bytes_write.sum of one
# 8-head launch of the routed packing, captured with --clock-control none), scaled by heads: a stored figure, not a
# per-run measurement.  Valid only for the kernel sources it was taken from (attn.cu and softmax.cuh, hashed
# together); reported as null once either changes.
ATTN_TRAFFIC = {"source_sha256_prefix": "c5dfca8afeb2c7de", "bytes_per_head": (1.843117568e9 + 0.230613760e9) / 8}
ATTN_SOURCES = ("attn.cu", "softmax.cuh")


def attn_source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "biased_attention_video_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic_bytes(H: int):
    if not attn_source_digest().startswith(ATTN_TRAFFIC["source_sha256_prefix"]):
        return None
    return ATTN_TRAFFIC["bytes_per_head"] * H


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def effective_pairs(p, sel: np.ndarray | None) -> int:
    """Sum over heads and query rows of the attended (valid) keys."""
    S, B = p.S, 64
    nkb = p.n_blocks
    rows = np.minimum(B, S - np.arange(nkb) * B).astype(np.int64)
    if sel is None:
        return int(p.H) * S * S
    forced_keys = int(rows[:p.first_video_block].sum())
    dense_pairs = int(rows[:p.first_video_block].sum()) * S
    routed_keys = rows[sel].sum(axis=-1) + forced_keys      # [H][nV]
    vrows = rows[p.first_video_block:]
    return int(p.H) * dense_pairs + int((routed_keys * vrows[None, :]).sum())


def executed_mma_pairs(p, sel: np.ndarray | None) -> int:
    """(query, key) pairs the tensor cores actually process: per 128-row tile, the union
    of its two query blocks' key lists, one 64-key block per step.  The tiles are the
    kernel's: adjacent blocks over the dense prefix (rounded up to an even block), then
    the video blocks paired within groups of 32 by greedy largest list overlap (ties to
    the lowest pair), an odd block out alone."""
    nkb = p.n_blocks
    if sel is None:
        return int(p.H) * ((nkb + 1) // 2) * nkb * 128 * 64
    fvb, H, kk = p.first_video_block, int(p.H), sel.shape[2]
    n_dense = (fvb + 1) // 2
    total = H * n_dense * nkb                 # a dense block makes its tile dense: every key block
    first = 2 * n_dense
    nv = nkb - fvb
    G = 32
    iu = np.triu_indices(G, 1)
    tie = ((31 - iu[0]) * 32 + (31 - iu[1])).astype(np.int64)
    for g0 in range(first, nkb, G):
        gs = min(G, nkb - g0)
        bits = np.zeros((H, G, nv), np.float32)
        hh, ii = np.meshgrid(np.arange(H), np.arange(gs), indexing="ij")
        lst = sel[:, g0 - fvb:g0 - fvb + gs] - fvb                  # [H][gs][k]
        bits[hh[..., None], ii[..., None], lst] = 1.0
        ov = np.einsum("hav,hbv->hab", bits, bits).astype(np.int64)[:, iu[0], iu[1]]
        alive = np.zeros((H, G), bool)
        alive[:, :gs] = True
        for _ in range(gs // 2):
            ok = alive[:, iu[0]] & alive[:, iu[1]]
            key = np.where(ok, ov * 1024 + tie[None, :], -1)
            c = key.argmax(axis=1)
            u = 2 * kk - ov[np.arange(H), c]
            total += int((u + fvb).sum())
            alive[np.arange(H), iu[0][c]] = False
            alive[np.arange(H), iu[1][c]] = False
        if gs % 2:
            total += H * (kk + fvb)
    return int(total) * 128 * 64


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank runs its own independent call: the workload's seed shifted by the rank."""
    return base_seed + rank


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise maximum of per-rank timings (all ranks take part; no-op for one rank)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def head_range(H: int, world: int, rank: int):
    """Heads [h0, h0 + nh) of rank `rank` when one call's H heads are split over `world` ranks: contiguous,
    sizes differing by at most one, together covering every head once.  Every step of the path is
    independent per head, so the shards need no collective."""
    base, extra = divmod(H, world)
    nh = base + (1 if rank < extra else 0)
    h0 = rank * base + min(rank, extra)
    return h0, nh


def sum_over_ranks(values, world: int, device="cpu"):
    """Element-wise sum over ranks (no-op for one rank)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()]


def whole_job_tflops(flops_per_call: float, calls_per_rank: int, world: int, ms: float) -> float:
    """Aggregate throughput of all ranks: every rank did calls_per_rank calls in at most ms."""
    return world * flops_per_call * calls_per_rank / (ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            lines = [ln.strip() for ln in f if ln.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(cfg, q, k, v, seg, times, pen, sparsity, budget_s: float, head: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload: full routing of one
    head plus attention for sampled query rows of that head (dense and routed rows).
    Returns (effective FLOPs done, seconds, description)."""
    import oracle

    t0 = time.perf_counter()
    qh, kh, vh = q[head:head + 1], k[head:head + 1], v[head:head + 1]
    sel, _, _ = oracle.route(qh, kh, seg, sparsity)
    t_route = time.perf_counter() - t0
    nkb = (cfg.S + 63) // 64
    cls = oracle.block_classes(seg)
    fvb = int(cls.sum())
    # the edge blocks first (first and last prefix block, first video block, the
    # ragged last block), then every other block in a seeded random order; eight
    # rows of each; the time budget decides how far down the list it gets
    rng = np.random.default_rng(1234)
    edge = list(dict.fromkeys(b for b in (0, fvb - 1, fvb, nkb - 1) if 0 <= b < nkb))
    blocks = edge + [int(b) for b in rng.permutation(nkb) if int(b) not in edge]
    rows_done, flops = 0, 0
    rows_all = [b * 64 + r for b in blocks for r in (0, 9, 18, 27, 36, 45, 54, 63) if b * 64 + r < cfg.S]
    rows_per_key = np.minimum(64, cfg.S - np.arange(nkb) * 64)
    forced_keys = int(rows_per_key[:fvb].sum())
    i = 0
    while i < len(rows_all) and time.perf_counter() - t0 < budget_s:
        chunk = np.array(rows_all[i:i + 8], np.int32)
        oracle.attend(qh, kh, vh, seg, times, pen=pen, sel=sel, heads=np.zeros(len(chunk), np.int32), rows=chunk)
        for x in chunk:
            qb = x // 64
            keys = cfg.S if qb < fvb else forced_keys + int(rows_per_key[sel[0, qb - fvb]].sum())
            flops += 4 * cfg.d * keys
        rows_done += len(chunk)
        i += 8
    secs = time.perf_counter() - t0
    desc = (f"oracle fp64 on {oracle.threads()} threads: routing of head {head} "
            f"({t_route:.2f} s, {int(cls.size - fvb)}^2 pooled scores) + attention of {rows_done} sampled "
            f"query rows of that head (dense prefix rows and routed video rows)")
    return flops, secs, desc, rows_done


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, rank 0 only."""
    if rank != 0:
        return
    cfg = inputs.FULL_COMBINED
    seg, times, _ = cfg.layout()
    small = inputs.custom(1, cfg.d, cfg.segments, cfg.seed, cluster_norm=cfg.cluster_norm)
    q, k, v = (inputs.tensor(small, t) for t in range(3))
    import oracle

    total_flops, total_s, desc = 0, 0.0, ""
    for i in range(args.warmup + args.steps):
        f, s, desc, _ = oracle_sample(cfg, q, k, v, seg, times, cfg.penalty, cfg.sparsities[0], budget_s=4.0)
        if i >= args.warmup:
            total_flops += f
            total_s += s
    value = total_flops / total_s / 1e12
    line = {"metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "per step: bounded oracle sample of the workload"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _time_calls(torch, fn, steps: int, warmup: int, stream) -> float:
    """Mean CUDA-event time (ms) of `steps` back-to-back calls after `warmup` untimed ones."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def extra_configs(args, h3, dev, stream, host, qd, kd, vd, o):
    """Configuration 4 (dense biased attention at the full packing, default penalty) and configuration 3 (the
    mid clip at sparsity 0, 0.60, 0.85, 0.90, no penalty, routing included in the call).  Inputs resident in
    HBM; each call far above L2 (Q+K+V = 5.0 GB and 2.1 GB)."""
    import torch
    peaks, _ = measured_peaks()
    peak = peaks["bf16_tflops_sustained"]
    steps, warmup = max(1, min(args.steps, 5)), 3
    out = {}

    # configuration 4: the full packing, dense; inputs of its own seed into the same buffers
    cfg = inputs.FULL_DENSE
    seg, times, _ = cfg.layout()
    for i, t in enumerate(("q", "k", "v")):
        inputs.tensor(cfg, i, out=host[t].numpy().view(np.uint16))
    for src, dst in ((host["q"], qd), (host["k"], kd), (host["v"], vd)):
        dst.view(torch.int16).view(-1).copy_(src)
    seg_d = torch.from_numpy(seg).to(dev)
    times_d = torch.from_numpy(times).to(dev)
    p = h3.plan(cfg.H, cfg.S, cfg.d, seg)
    ws = h3.workspace(p, dev)
    ms = _time_calls(torch, lambda: h3.forward(p, qd, kd, vd, seg_d, times_d, pen=cfg.penalty, ws=ws, out=o),
                     steps, warmup, stream)
    if h3.check(ws) != h3.OK:
        raise RuntimeError("device status after the dense call")
    flops = 4.0 * cfg.d * cfg.H * cfg.S * cfg.S
    out["full_dense"] = {
        "workload": "full dense biased: S=116883 (same packing as the headline), H=56, d=128, bf16, sparsity 0, "
                    "default penalty on output->guide pairs, seed 1004",
        "ms_per_call": ms, "effective_tflop_per_call": flops / 1e12, "effective_tflops": flops / (ms * 1e-3) / 1e12,
        "frac_of_sustained_peak": flops / (ms * 1e-3) / 1e12 / peak, "steps": steps, "warmup": warmup}
    del ws

    # configuration 3: the mid clip, sparsity sweep (routing + attention per call)
    cfg = inputs.MID_CLIP
    seg, times, _ = cfg.layout()
    q3, k3, v3 = (torch.from_numpy(inputs.tensor(cfg, i).view(np.int16)).to(dev).view(torch.bfloat16)
                  for i in range(3))
    seg_d = torch.from_numpy(seg).to(dev)
    times_d = torch.from_numpy(times).to(dev)
    o3 = torch.empty_like(q3)
    sweep = []
    for s in cfg.sparsities:
        p = h3.plan(cfg.H, cfg.S, cfg.d, seg, sparsity=s)
        ws = h3.workspace(p, dev)
        routed = p.n_video_blocks > 0 and p.k < p.n_video_blocks
        sel = torch.empty((cfg.H, p.n_video_blocks, p.k), dtype=torch.int32, device=dev) if routed else None

        def call():
            if routed:
                h3.route(p, q3, k3, ws, kv_sel=sel)
            h3.forward(p, q3, k3, v3, seg_d, times_d, pen=None, kv_sel=sel, ws=ws, out=o3)

        ms_call = _time_calls(torch, call, steps, warmup, stream)
        ms_fwd = _time_calls(torch, lambda: h3.forward(p, q3, k3, v3, seg_d, times_d, pen=None, kv_sel=sel, ws=ws,
                                                       out=o3), steps, 1, stream)
        ms_route = _time_calls(torch, lambda: h3.route(p, q3, k3, ws, kv_sel=sel), steps, 1, stream) if routed else 0.0
        if h3.check(ws) != h3.OK:
            raise RuntimeError(f"device status after the mid-clip call at sparsity {s}")
        flops = 4.0 * cfg.d * effective_pairs(p, sel.cpu().numpy() if routed else None)
        sweep.append({"sparsity": s, "k": int(p.k), "ms_per_call": ms_call, "attention_ms": ms_fwd,
                      "route_ms": ms_route,
                      "effective_tflop_per_call": flops / 1e12, "effective_tflops": flops / (ms_call * 1e-3) / 1e12,
                      "attention_tflops": flops / (ms_fwd * 1e-3) / 1e12,
                      "attention_frac_of_sustained_peak": flops / (ms_fwd * 1e-3) / 1e12 / peak})
        del ws, sel
    out["mid_clip_sweep"] = {"workload": "mid clip: S=49152 (text 256|image-ref 1024|audio 400|video 24x1978), "
                                         "H=56, d=128, bf16, block 64, no penalty, seed 1003",
                             "steps": steps, "warmup": warmup, "points": sweep}
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import biased_attention_video_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = inputs.FULL_DENSE if args.workload == "full_dense" else inputs.FULL_COMBINED
    if args.heads is not None:
        cfg = inputs.custom(args.heads, cfg.d, cfg.segments, cfg.seed, cluster_norm=cfg.cluster_norm,
                            penalty=cfg.penalty, sparsities=cfg.sparsities, name=f"{cfg.name} ({args.heads} heads)")
    sharded = args.shard == "heads"
    # weak scaling: every rank its own independent call (seed shifted by the rank); head sharding: one call
    # (one seed), each rank its contiguous range of heads
    seed = cfg.seed if sharded else rank_seed(cfg.seed, rank)
    seg, times, _ = cfg.layout()
    if sharded and world > cfg.H:
        raise SystemExit(f"--shard heads needs at most {cfg.H} ranks")
    h0, H = head_range(cfg.H, world, rank) if sharded else (0, cfg.H)
    S, d = cfg.S, cfg.d
    sparsity = cfg.sparsities[0]
    pen = cfg.penalty

    # inputs generated straight into pinned host memory (also the e2e sources)
    n = H * S * d
    host = {t: torch.empty(n, dtype=torch.int16, pin_memory=True) for t in ("q", "k", "v")}
    for i, t in enumerate(("q", "k", "v")):
        inputs.tensor(cfg, i, h0=h0, nh=H, out=host[t].numpy().view(np.uint16), seed=seed)
    seg_h = torch.from_numpy(seg).pin_memory()
    times_h = torch.from_numpy(times).pin_memory()
    o_h = torch.empty(n, dtype=torch.int16, pin_memory=True)
    qd, kd, vd = (host[t].to(dev).view(torch.bfloat16).view(H, S, d) for t in ("q", "k", "v"))
    seg_d, times_d = seg_h.to(dev), times_h.to(dev)
    p = h3.plan(H, S, d, seg, sparsity=sparsity)
    ws = h3.workspace(p, dev)
    routed = p.n_video_blocks > 0 and p.k < p.n_video_blocks
    sel = torch.empty((H, p.n_video_blocks, p.k), dtype=torch.int32, device=dev) if routed else None
    o = torch.empty_like(qd)
    stream = torch.cuda.current_stream(dev)

    ev = {"r0": [], "r1": [], "f0": [], "f1": []}

    def step(record=False):
        if record:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
        if routed:
            h3.route(p, qd, kd, ws, kv_sel=sel)
        if record:
            e[1].record(stream)
            e[2].record(stream)
        h3.forward(p, qd, kd, vd, seg_d, times_d, pen=pen, kv_sel=sel, ws=ws, out=o)
        if record:
            e[3].record(stream)
            for key, x in zip(("r0", "r1", "f0", "f1"), e):
                ev[key].append(x)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = h3.check(ws)
    if status != h3.OK:
        raise RuntimeError(f"device status {status} after warm-up")
    sel_h = sel.cpu().numpy() if routed else None
    pairs = effective_pairs(p, sel_h)
    eff_flops = 4 * d * pairs
    mma_pairs = executed_mma_pairs(p, sel_h)

    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    status = h3.check(ws)
    if status != h3.OK:
        raise RuntimeError(f"device status {status} in timed region")
    ms = t_start.elapsed_time(t_end)
    route_ms = sum(a.elapsed_time(b) for a, b in zip(ev["r0"], ev["r1"])) / args.steps
    fwd_ms = sum(a.elapsed_time(b) for a, b in zip(ev["f0"], ev["f1"])) / args.steps

    # end to end through the C ABI from pinned host buffers
    h2d = 3 * n * 2 + S + 4 * S
    d2h = n * 2
    qh_v, kh_v, vh_v = host["q"], host["k"], host["v"]

    # the public host-buffer call: head chunks pipelined over three streams
    copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_step():
        h3.attend_host(p, qh_v, kh_v, vh_v, seg_h, times_h, o_h, q=qd, k=kd, v=vd, seg=seg_d, times=times_d, o=o,
                       ws=ws, kv_sel=sel, pen=pen, chunk_heads=min(args.chunk_heads, H), stream=stream,
                       copy_in_stream=copy_in, copy_out_stream=copy_out)

    e2e_ms = float("nan")
    if not args.no_e2e:
        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1)
        if h3.check(ws) != h3.OK:
            raise RuntimeError("device status after e2e")

    # partition merge (h3attn_merge) at full size: two partitions of this call's O/LSE shape, HBM-bound
    merge_ms = float("nan")
    if not args.no_merge:
        lse_a = torch.zeros((H, S), dtype=torch.float32, device=dev)
        lse_b = torch.full((H, S), -0.5, dtype=torch.float32, device=dev)
        o2 = torch.empty_like(o)
        l2 = torch.empty_like(lse_a)
        for _ in range(3):
            h3.merge([o, qd], [lse_a, lse_b], out=o2, lse=l2)
        m0 = torch.cuda.Event(enable_timing=True)
        m1 = torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(args.steps):
            h3.merge([o, qd], [lse_a, lse_b], out=o2, lse=l2)
        m1.record(stream)
        torch.cuda.synchronize(dev)
        merge_ms = m0.elapsed_time(m1) / args.steps
        del lse_a, lse_b, o2, l2

    # pooled tail term (h3attn_tail_correct) at full size: after route + forward with LSE on this call's
    # inputs; its kernels read V's video rows, the pooled scores, the weights and the O/LSE of video rows
    tail_ms = float("nan")
    if not args.no_tail and routed:
        lse_t = torch.empty((H, S), dtype=torch.float32, device=dev)
        tail_ws = h3.tail_workspace(p, dev)
        h3.route(p, qd, kd, ws, kv_sel=sel)
        h3.forward(p, qd, kd, vd, seg_d, times_d, pen=pen, kv_sel=sel, ws=ws, out=o, lse=lse_t)
        h3.tail_correct(p, vd, sel, o, lse_t, ws, tail_ws=tail_ws)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            h3.tail_correct(p, vd, sel, o, lse_t, ws, tail_ws=tail_ws)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        tail_ms = t0.elapsed_time(t1) / args.steps
        if h3.check(ws) != h3.OK:
            raise RuntimeError("device status after the tail correction")
        del lse_t, tail_ws

    # int8 QK (h3attn_forward_qk8: per-token quantisation of Q and K, then the attention with int8 QK
    # products) at full size on this call's routed lists, and its deviation from the bf16 path's O
    qk8_ms = quant_ms = float("nan")
    qk8_rel = None
    if not args.no_qk8 and d == 128:
        qws = h3.qk8_workspace(p, dev)
        o8 = torch.empty_like(o)
        if routed:
            h3.route(p, qd, kd, ws, kv_sel=sel)
        for _ in range(2):
            h3.forward_qk8(p, qd, kd, vd, seg_d, times_d, pen=pen, kv_sel=sel, ws=ws, qk8_ws=qws, out=o8)
        q0 = torch.cuda.Event(enable_timing=True)
        q1 = torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for _ in range(args.steps):
            h3.forward_qk8(p, qd, kd, vd, seg_d, times_d, pen=pen, kv_sel=sel, ws=ws, qk8_ws=qws, out=o8)
        q1.record(stream)
        q0b = torch.cuda.Event(enable_timing=True)
        q1b = torch.cuda.Event(enable_timing=True)
        q0b.record(stream)
        for _ in range(args.steps):
            h3.quantize_qk(p, qd, kd, qws)
        q1b.record(stream)
        torch.cuda.synchronize(dev)
        qk8_ms = q0.elapsed_time(q1) / args.steps
        quant_ms = q0b.elapsed_time(q1b) / args.steps
        if h3.check(ws) != h3.OK:
            raise RuntimeError("device status after the int8 QK call")
        h3.forward(p, qd, kd, vd, seg_d, times_d, pen=pen, kv_sel=sel, ws=ws, out=o)
        num = den = 0.0
        for hh in range(H):
            a = o8[hh].float()
            b = o[hh].float()
            num += float(torch.sum((a - b) ** 2))
            den += float(torch.sum(b * b))
        qk8_rel = (num / den) ** 0.5
        del qws, o8

    # the other measured configurations of the call, on this GPU (one process): the dense biased call at the
    # full packing (the 60 % target's S, 391.7 TFLOP) and the mid clip's sparsity sweep
    extra = None
    if not args.no_extra and world == 1 and args.heads is None and args.workload == "full_combined":
        extra = extra_configs(args, h3, dev, stream, host, qd, kd, vd, o)

    # max over ranks; with head sharding the job's work is the sum of the ranks' shares
    ms, e2e_ms, fwd_ms, route_ms, merge_ms, tail_ms, qk8_ms, quant_ms = max_over_ranks(
        [ms, e2e_ms, fwd_ms, route_ms, merge_ms, tail_ms, qk8_ms, quant_ms], world, dev)
    local_flops, local_mma = eff_flops, mma_pairs
    if sharded:
        eff_flops, mma_pairs = sum_over_ranks([eff_flops, mma_pairs], world, dev)

    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    ms_step = ms / args.steps
    # whole job: weak scaling = world independent calls; sharded = one call split over the ranks
    job_world = 1 if sharded else world
    value = whole_job_tflops(eff_flops, args.steps, job_world, ms)
    e2e_value = whole_job_tflops(eff_flops, args.steps, job_world, e2e_ms)
    attn_tflops = (local_flops if sharded else eff_flops) / (fwd_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    route_bytes = 2 * H * p.n_video_blocks * 64 * d * 2  # Q and K video rows, read once by the pool
    dense_run = args.workload == "full_dense"
    line = {
        "metric": METRIC_DENSE if dense_run else METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded counter-based generator, cluster-mean Q/K)",
        "config": {"workload": WORKLOAD_DENSE if dense_run else WORKLOAD, "H": cfg.H, "S": S, "d": d, "block": 64,
                   "sparsity": sparsity,
                   "parallelism": (f"head-sharded over {world} GPUs (rank 0: heads {h0}..{h0 + H - 1})" if sharded
                                   else f"{world} independent calls, one per GPU"),
                   "k": int(p.k), "seed": seed, "l2": "no flush: Q+K+V = 5.0 GB per step, far above the 126 MB L2",
                   "effective_tflop_per_call": eff_flops / 1e12,
                   "executed_mma_tflop_per_call": 4 * d * mma_pairs / 1e12,
                   "route_ms": route_ms, "attention_ms": fwd_ms},
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak,
                     # the stored capture is of the routed workload; the dense one has none
                     "traffic": None if dense_run else attn_traffic_bytes(H),
                     "kernel": "attn_kernel (fused routed attention); achieved = effective FLOPs per launch / "
                               "CUDA-event time of the forward call (kv_desc prep + attention)",
                     "peak_source": f"{peak_kind} bf16_tflops_sustained"},
        "routing": None if not routed else {
            "ms": route_ms, "bytes_read": route_bytes, "gbs": route_bytes / (route_ms * 1e-3) / 1e9,
            "hbm_peak_gbs": peaks["hbm_gbs"]},
        "merge": None if args.no_merge else {
            "kernel": "merge_kernel (h3attn_merge: two partitions, O bf16 [H][S][d] + LSE f32, out O + LSE)",
            "ms": merge_ms, "bytes": 3 * H * S * (d * 2 + 4),
            "gbs": 3 * H * S * (d * 2 + 4) / (merge_ms * 1e-3) / 1e9, "hbm_peak_gbs": peaks["hbm_gbs"]},
        "tail": None if args.no_tail else {
            "kernels": "pool_vt, tail_weights, tail_gemm (tcgen05), tail_merge (h3attn_tail_correct)",
            "ms": tail_ms, "share_of_call": tail_ms / ms_step},
        "qk8": None if (args.no_qk8 or d != 128) else {
            "what": "h3attn_forward_qk8 on the same routed call: per-token int8 quantisation of Q and K "
                    "(quant_rows_kernel) + attn_kernel with int8 QK MMAs; not the headline (reduced precision)",
            "ms": qk8_ms, "quantize_ms": quant_ms,
            "effective_tflops": (local_flops if sharded else eff_flops) / (qk8_ms * 1e-3) / 1e12,
            "vs_bf16_forward": fwd_ms / qk8_ms,
            "quantize_gbs": (2 * H * S * d * 3 + 2 * H * p.n_blocks * 64 * 4) / (quant_ms * 1e-3) / 1e9,
            "rel_fro_vs_bf16": qk8_rel},
        "full_dense": None if extra is None else extra["full_dense"],
        "mid_clip_sweep": None if extra is None else extra["mid_clip_sweep"],
        "gpu_launches": (6 if routed else 2) * args.steps,  # pool_split, score_gemm, topk, kv_desc, pair, attn
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
    }
    if args.no_e2e:
        line["e2e"] = None
    if args.heads is not None:
        line["config"]["workload"] = line["config"]["workload"].replace("H=56", f"H={args.heads}") + \
            " (profiling variant)"
    if not args.no_cpu_baseline and world == 1:
        small = inputs.custom(1, d, cfg.segments, seed, cluster_norm=cfg.cluster_norm)
        qs, ks, vs = (inputs.tensor(small, i) for i in range(3))
        f, s, desc, _ = oracle_sample(cfg, qs, ks, vs, seg, times, pen, sparsity, budget_s=args.cpu_budget)
        import oracle
        line["cpu_baseline"] = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--heads", type=int, default=None,
                    help="run the same packing with fewer heads (profiling captures only; the default is 56)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-merge", action="store_true", help="skip the partition-merge measurement")
    ap.add_argument("--no-tail", action="store_true", help="skip the pooled-tail-term measurement")
    ap.add_argument("--no-qk8", action="store_true", help="skip the int8-QK measurement")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the dense full-size call and the mid-clip sparsity sweep (extra JSON keys)")
    ap.add_argument("--workload", choices=["full_combined", "full_dense"], default="full_combined",
                    help="the timed call: the routed headline workload (default) or the dense biased call at the "
                         "same packing (profiling)")
    ap.add_argument("--shard", choices=["none", "heads"], default="none",
                    help="N>1: 'none' = one independent call per GPU (weak scaling); 'heads' = one call, its heads "
                         "split over the GPUs (strong scaling)")
    ap.add_argument("--chunk-heads", type=int, default=2, help="heads per pipelined chunk of the host-buffer call")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
